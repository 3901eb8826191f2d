// Mask-aware attention backward, query side (dQ), for sm_100a.
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: forward+backward of mask-aware attention.  For the loss sum(O*dO):
//   dQ_i = scale * sum_j dS_ij k_j,  dS_ij = P_ij (dP_ij - D_i),
//   P_ij = exp(scale q_i.k_j - LSE_i) on visible pairs, dP_ij = dO_i.v_j.
//
// Query-stationary persistent CTAs (one per SM): a work item is (batch,
// q-head, 128-row q-tile); it walks the q-tile's non-skipped k-tiles, recomputes
// S and dP on the tensor core, forms dS in registers and accumulates
// dQ += dS K in TMEM, with dS taken from TMEM as the A operand.  Every dQ row
// is produced by exactly one CTA and written once in bf16: no cross-CTA
// reduction, deterministic results.  (The key side, dK/dV, is a separate
// key-stationary kernel.)
//
// TMEM (512 columns): S[0] [0,128), S[1] [128,256) (dS bf16 written over the
// S buffer of its tile: key columns 0-63 as pairs at [0,32), 64-127 at
// [64,96), so each warpgroup overwrites only columns it has read), dP
// [256,384), dQ [384, 384+d).
// MMA issue order: S(0) dP(0) | S(t+1) , dP(t+1) , dQ += dS(t) K(t) | ...
// where dP(t+1) waits only until the compute warps have loaded dP(t) into
// registers (dS(t) is written over S(t), not over dP), so the next tile's dP
// is computed while the compute warps evaluate the current tile.  The compute
// warps can then complete tile t+1 before the MMA warp has seen "dS(t)
// written", so that signal alternates between two barriers by tile parity: a
// parity wait never sees its barrier two phases ahead (tile t+2 needs S(t+2),
// issued only after dQ(t)).
// K tiles (3-deep ring, freed after dQ) and V tiles (2-deep, freed after dP)
// stream through separate rings; the element mask of a partial tile is built
// from the boundary records read straight from global memory (L2-resident),
// turned into per-row bit words by a warp bit-transpose.
// While the tensor core runs S(t+1), dP(t+1) and dQ(t) the compute warps turn
// S(t)/dP(t) into dS(t).
//
// Roles (352 threads): warps 0-7 compute (thread = query row; warpgroup 0
// takes key columns 0-63 of a tile, warpgroup 1 columns 64-127), warp 8 TMA
// producer of Q/dO and the K ring, warp 10 TMA producer of the V ring, warp 9
// MMA issuer; work items reach every role through a ring of mbarriers.  Q and
// dO are released after the item's last S and dP (one tile before its end), so
// the next item's Q/dO load overlaps the current item's last dQ step.
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

namespace qb {
constexpr int kThreads = 352;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kProducer2Warp = 10;
constexpr int kRing = 4;
constexpr int kKStages = 3;  // K tiles: last read by dQ(t)
constexpr int kVStages = 2;  // V tiles: last read by dP(t), freed earlier
constexpr uint32_t kColS = 0, kColDP = 256, kColDQ = 384;
}  // namespace qb

// A decoded work item (batch, q-head, q-tile).  The producer decodes each item
// once and publishes it in the shared-memory ring; the other roles read it
// there.  item >= n_items2 ends the work.
struct __align__(16) QItem {
  int item, b, h, hm, qt, g;
  int cnt;  // entries of the q-tile's block list (for both q-tiles of the block)
  int n;    // entries not skipped for this q-tile
  // forward work list of the q-tile's block
  __device__ __forceinline__ const int* list(const BwdParams& p) const {
    const Shape& sh = p.s;
    return p.flist + (((size_t)b * sh.Hm + hm) * sh.nQB + (qt >> 1)) * sh.nKt;
  }
};

__device__ __forceinline__ QItem decode_q_item(const BwdParams& p, int item) {
  const Shape& sh = p.s;
  QItem it{};
  it.item = item;
  if (item >= p.n_items2) return it;
  const int unit = p.forder[item];
  if (kChecks && (unit < 0 || unit >= p.n_items2)) {
    atomicCAS(p.status, 0, kDevErrBounds);
    it.item = INT_MAX;  // ends the CTA's work
    return it;
  }
  const ItemCoord c = decode_q_item_coord(sh, unit);
  it.b = c.b;
  it.h = c.hkv * sh.G + c.hg;
  it.hm = (sh.Hm == 1) ? 0 : it.h;
  it.qt = c.t;
  it.g = c.t & 1;
  const size_t lrow = ((size_t)it.b * sh.Hm + it.hm) * sh.nQB + (c.t >> 1);
  it.cnt = (it.qt < sh.nQt) ? p.fcount[lrow] : 0;
  it.n = (it.qt < sh.nQt) ? p.qcount[lrow * 2 + it.g] : 0;  // per-q-tile count of the lists
  if (kChecks) {  // the block's k-tile list and this q-tile's share of it
    bool bad = it.cnt < 0 || it.cnt > sh.nKt || it.n < 0 || it.n > it.cnt;
    for (int t = 0; !bad && t < it.cnt; ++t) {
      const int e = it.list(p)[t];
      bad = (e >> 8) < 0 || (e >> 8) >= sh.nKt;
    }
    if (bad) {
      atomicCAS(p.status, 0, kDevErrBounds);
      it.item = INT_MAX;
      return it;
    }
  }
  return it;
}

// Calls f(kt, cls) for the q-tile's non-skipped k-tiles in increasing order.
template <typename F>
__device__ __forceinline__ bool for_each_ktile(const BwdParams& p, const QItem& it, F&& f) {
  const int* list = it.list(p);
  for (int t = 0; t < it.cnt; ++t) {
    const int e = list[t];
    const int cls = (e >> (2 * it.g)) & 3;
    if (cls == kClsSkip) continue;
    if (!f(e >> 8, cls)) return false;
  }
  return true;
}

template <int D>
struct __align__(1024) DqSmem {
  uint8_t q[kTile * D * 2];
  uint8_t dout[kTile * D * 2];
  uint8_t k[qb::kKStages][kTile * D * 2];
  uint8_t v[qb::kVStages][kTile * D * 2];
  QItem ring[qb::kRing];
  uint64_t ring_full[qb::kRing], ring_empty[qb::kRing];
  uint64_t q_full, q_empty;
  uint64_t k_full[qb::kKStages], k_empty[qb::kKStages];
  uint64_t v_full[qb::kVStages], v_empty[qb::kVStages];
  uint64_t s_full[2], dp_full, dp_read, ds_full[2];
  uint64_t dq_full, dq_free;
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
  int no_abort;
};

static_assert(sizeof(DqSmem<128>) <= 232448, "query-side shared memory exceeds the per-CTA limit");
static_assert(sizeof(DqSmem<64>) <= 232448, "query-side shared memory exceeds the per-CTA limit");

// S (or dP) = A B^T over the head dimension, both K-major SW128 (128 x 128).
template <int D>
__device__ __forceinline__ void q_issue_ss(uint32_t d_tmem, const uint8_t* as, const uint8_t* bs) {
  constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
  const uint32_t aa = smem_addr(as), ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, sdesc_sw128(aa + off, 16, 1024), sdesc_sw128(ba + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// dQ (+)= dS[tmem] K: M = 128 rows, N = D, K = 128 keys; K tile read MN-major.
template <int D>
__device__ __forceinline__ void q_issue_dq(uint32_t d_tmem, uint32_t a_tmem, const uint8_t* ks, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
  const uint32_t ka = smem_addr(ks);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)  // dS pairs: keys 0-63 at [0,32), 64-127 at [64,96)
    mma_ts(d_tmem, a_tmem + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), sdesc_sw128(ka + kk * 2048, 16384, 1024),
           idesc, (accumulate || kk > 0) ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(qb::kThreads, 1)
    fm_bwd_dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                     const BwdParams p) {
  using namespace qb;
  constexpr int kTileBytes = kTile * D * 2;
  constexpr int kBoxes = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DqSmem<D>& s = *reinterpret_cast<DqSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Shape& sh = p.s;

  if (smem_addr(smem_raw) & 1023u) {
    if (tid == 0) atomicCAS(p.status, 0, -5);
    return;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&s.ring_full[i], 1);
      mbar_init(&s.ring_empty[i], 10);  // MMA + second producer + lane 0 of the 8 compute warps
    }
    mbar_init(&s.q_full, 1);
    mbar_init(&s.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
    }
    mbar_init(&s.s_full[0], 1);
    mbar_init(&s.s_full[1], 1);
    mbar_init(&s.dp_full, 1);
    mbar_init(&s.dp_read, 256);
    mbar_init(&s.ds_full[0], 256);
    mbar_init(&s.ds_full[1], 256);
    mbar_init(&s.dq_full, 1);
    mbar_init(&s.dq_free, 256);
    mbar_init(&s.teardown, 1);
    s.abort_flag = 0;
    s.no_abort = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_map(&tq);
    tma_prefetch_map(&tk);
    tma_prefetch_map(&tv);
    tma_prefetch_map(&tdo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();
  const uint32_t tmem = s.tmem_base;
  const WaitCtx w{&s.abort_flag, p.status, p.wait_limit_ns, smem_addr(smem_raw), 2};
  uint32_t q_par = 0, q_armed = 0, k_par[kKStages] = {}, v_par[kVStages] = {}, k_armed = 0, v_armed = 0;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      uint32_t kv_iter = 0, act = 0, k = 0;
      bool ok = true;
      // Items are taken one ahead: while one item's tiles stream, the next
      // item's Q and dO are prefetched into L2, so their load (which may only
      // start once the current item's last S and dP have been issued) hits L2.
      auto take = [&](QItem& out) -> bool {
        const int slot = k % kRing;
        if (!mbar_wait(&s.ring_empty[slot], ((k / kRing) & 1) ^ 1, w)) return false;
        const int item = s.abort_flag ? INT_MAX : atomicAdd(p.counter2, 1);
        out = decode_q_item(p, item);
        s.ring[slot] = out;
        mbar_arrive(&s.ring_full[slot]);
        ++k;
        if (out.item < p.n_items2 && out.n > 0) {
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx) {
            tma_prefetch_l2_4d(&tq, bx * 64, out.h, out.qt * kTile, out.b);
            tma_prefetch_l2_4d(&tdo, bx * 64, out.h, out.qt * kTile, out.b);
          }
        }
        return true;
      };
      QItem nxt{};
      ok = take(nxt);
      while (ok && nxt.item < p.n_items2) {
        const QItem it = nxt;
        if (!(ok = take(nxt))) break;
        if (it.n == 0) continue;
        if (!(ok = mbar_wait(&s.q_empty, (act & 1) ^ 1, w))) break;
        mbar_arrive_expect_tx(&s.q_full, 2 * kTileBytes);
        q_par = act & 1;
        q_armed = 1;
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) {
          tma_load_4d(s.q + bx * 16384, &tq, &s.q_full, bx * 64, it.h, it.qt * kTile, it.b);
          tma_load_4d(s.dout + bx * 16384, &tdo, &s.q_full, bx * 64, it.h, it.qt * kTile, it.b);
        }
        ++act;
        ok = for_each_ktile(p, it, [&](int kt, int) {
          const int sk = kv_iter % kKStages;
          const uint32_t pk = (kv_iter / kKStages) & 1;
          const int hkv = it.h / sh.G;
          if (!mbar_wait(&s.k_empty[sk], pk ^ 1, w)) return false;
          mbar_arrive_expect_tx(&s.k_full[sk], kTileBytes);
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_4d(s.k[sk] + bx * 16384, &tk, &s.k_full[sk], bx * 64, hkv, kt * kTile, it.b);
          k_par[sk] = pk;
          k_armed |= 1u << sk;
          ++kv_iter;
          return true;
        });
      }
    }
  } else if (warp == kProducer2Warp) {
    // second producer: the V ring
    if (lane == 0) {
      uint32_t kv_iter = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int slot = k % kRing;
        if (!(ok = mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w))) break;
        const QItem it = s.ring[slot];
        mbar_arrive(&s.ring_empty[slot]);
        if (it.item >= p.n_items2) break;
        if (it.n == 0) continue;
        ok = for_each_ktile(p, it, [&](int kt, int) {
          const int sv = kv_iter % kVStages;
          const uint32_t pv = (kv_iter / kVStages) & 1;
          if (!mbar_wait(&s.v_empty[sv], pv ^ 1, w)) return false;
          mbar_arrive_expect_tx(&s.v_full[sv], kTileBytes);
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_4d(s.v[sv] + bx * 16384, &tv, &s.v_full[sv], bx * 64, it.h / sh.G, kt * kTile, it.b);
          v_par[sv] = pv;
          v_armed |= 1u << sv;
          ++kv_iter;
          return true;
        });
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      uint32_t kv_iter = 0, tc = 0, act = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int slot = k % kRing;
        if (!(ok = mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w))) break;
        const QItem it = s.ring[slot];
        mbar_arrive(&s.ring_empty[slot]);
        if (it.item >= p.n_items2) break;
        const int n = it.n;
        if (n == 0) continue;
        if (!(ok = mbar_wait(&s.q_full, act & 1, w))) break;
        // tile j uses K stage (kv_iter + j) % kKStages, V stage (kv_iter + j) % kVStages
        // and S buffer (tc + j) & 1
        {
          const int sk = kv_iter % kKStages, sv = kv_iter % kVStages;
          if (!(ok = mbar_wait(&s.k_full[sk], (kv_iter / kKStages) & 1, w))) break;
          tc_fence_after();
          q_issue_ss<D>(tmem + kColS + (tc & 1) * 128, s.q, s.k[sk]);
          mma_commit(&s.s_full[tc & 1]);
          if (!(ok = mbar_wait(&s.v_full[sv], (kv_iter / kVStages) & 1, w))) break;
          tc_fence_after();
          q_issue_ss<D>(tmem + kColDP, s.dout, s.v[sv]);
          mma_commit(&s.dp_full);
          mma_commit(&s.v_empty[sv]);
          if (n == 1) mma_commit(&s.q_empty);  // Q and dO read for the last time
        }
        for (int j = 0; j < n; ++j) {
          const uint32_t kj = kv_iter + j, tj = tc + j;
          const int sk = kj % kKStages, sk2 = (kj + 1) % kKStages, sv2 = (kj + 1) % kVStages;
          const int bf = tj & 1;
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&s.k_full[sk2], ((kj + 1) / kKStages) & 1, w))) break;
            tc_fence_after();
            q_issue_ss<D>(tmem + kColS + (bf ^ 1) * 128, s.q, s.k[sk2]);  // S(j+1): its buffer held dS(j-1)
            mma_commit(&s.s_full[bf ^ 1]);
          }
          if (j + 1 < n) {
            // dP(j+1) as soon as the compute warps hold dP(j) in registers
            if (!(ok = mbar_wait(&s.dp_read, tj & 1, w) && mbar_wait(&s.v_full[sv2], ((kj + 1) / kVStages) & 1, w)))
              break;
            tc_fence_after();
            q_issue_ss<D>(tmem + kColDP, s.dout, s.v[sv2]);
            mma_commit(&s.dp_full);
            mma_commit(&s.v_empty[sv2]);
            if (j + 2 == n) mma_commit(&s.q_empty);  // last S and dP of the item issued
          }
          if (j == 0 && !(ok = mbar_wait(&s.dq_free, (act & 1) ^ 1, w))) break;  // previous dQ read out
          if (!(ok = mbar_wait(&s.ds_full[tj & 1], (tj >> 1) & 1, w))) break;
          tc_fence_after();
          q_issue_dq<D>(tmem + kColDQ, tmem + kColS + bf * 128, s.k[sk], j > 0);  // dQ += dS K
          mma_commit(&s.k_empty[sk]);
        }
        if (!ok) break;
        kv_iter += n;
        tc += n;
        ++act;
        mma_commit(&s.dq_full);
      }
    }
  } else {
    // ---------------- compute warpgroups: thread = query row, 64 key columns each ----------------
    const int wg = warp >> 2, wq = warp & 3;
    const int rl = wq * 32 + lane;  // row within the q-tile
    const uint32_t tb = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t c0 = wg * 64;
    uint32_t tc = 0, act = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int slot = k % kRing;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w)))) break;
      const QItem it = s.ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.ring_empty[slot]);
      if (it.item >= p.n_items2) break;
      if (it.qt >= sh.nQt) continue;
      const int row = it.qt * kTile + rl;
      const bool valid = row < sh.Nq;
      __nv_bfloat16* dqrow = p.dq + (((size_t)it.b * sh.Nq + (valid ? row : 0)) * sh.Hq + it.h) * D + wg * (D / 2);
      if (it.n == 0) {  // every k-tile skipped: dQ = 0
        if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dqrow);
#pragma unroll
          for (int i = 0; i < D / 16; ++i) d4[i] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const size_t roff = ((size_t)it.b * sh.Hq + it.h) * sh.nQt * kTile + (size_t)it.qt * kTile + rl;
      const float lse2 = p.lse2[roff];
      const float drow = p.dsum[roff];
      const int4* recs = p.rec + ((size_t)it.b * sh.Hm + it.hm) * sh.nKt * kTile;
      const int rbase = it.qt * kTile + wq * 32;  // first row of this warp
      ok = for_each_ktile(p, it, [&](int kt, int cls) {
        const int bf = tc & 1;
        const bool need = cls == kClsPartial;
        // this lane's two key columns of the warpgroup's half (read early; L2-resident)
        int4 ra = make_int4(0, 0, 0, 0), rb = ra;
        if (need) {
          ra = recs[(size_t)kt * kTile + c0 + lane];
          rb = recs[(size_t)kt * kTile + c0 + 32 + lane];
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full[bf], (tc >> 1) & 1, w))) return false;
        if (!__all_sync(0xffffffffu, mbar_wait(&s.dp_full, tc & 1, w))) return false;
        tc_fence_after();
        uint32_t sv[64], dv[64];
        tmem_ld32x(tb + kColS + bf * 128 + c0, sv);
        tmem_ld32x(tb + kColS + bf * 128 + c0 + 32, sv + 32);
        tmem_ld32x(tb + kColDP + c0, dv);
        tmem_ld32x(tb + kColDP + c0 + 32, dv + 32);
        uint32_t mbits0 = 0, mbits1 = 0;
        if (need) {  // per-column row words, transposed to per-row column words
          mbits0 = warp_transpose32(column_row_bits(ra, rbase), lane);
          mbits1 = warp_transpose32(column_row_bits(rb, rbase), lane);
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s.dp_read);  // dP(j) is in registers: the tensor core may overwrite it
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float pv = fast_exp2(fmaf(__uint_as_float(sv[i]), p.scale_log2, -lse2));
          const uint32_t bits = (i < 32) ? mbits0 : mbits1;
          pv = ((bits >> (i & 31)) & 1u) ? 0.f : pv;
          sv[i] = __float_as_uint(pv * (__uint_as_float(dv[i]) - drow));
        }
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
        tmem_st32x(tb + kColS + bf * 128 + c0, pk);  // bf16 pairs over this warpgroup's own S columns
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.ds_full[tc & 1]);
        ++tc;
        return true;
      });
      if (!ok) break;
      // epilogue: warpgroup wg writes head-dim columns [wg*D/2, (wg+1)*D/2) of its rows
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.dq_full, act & 1, w)))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t rr[32];
        tmem_ld32x(tb + kColDQ + wg * (D / 2) + c * 32, rr);
        tmem_ld_wait();
        uint32_t pk2[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk2[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * p.scale, __uint_as_float(rr[2 * i + 1]) * p.scale);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 4; ++i) st_global_v4_na(dqrow + c * 32 + i * 8, pk2[4 * i], pk2[4 * i + 1], pk2[4 * i + 2], pk2[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s.dq_free);
      ++act;
    }
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (s.abort_flag) {
    const WaitCtx w2{&s.no_abort, p.status, p.wait_limit_ns, smem_addr(smem_raw), 2};
    if (warp == kMmaWarp && lane == 0) {
      mma_commit(&s.teardown);
      (void)mbar_wait(&s.teardown, 0, w2);
    }
    if (warp == kProducerWarp && lane == 0) {
      if (q_armed) (void)mbar_wait(&s.q_full, q_par, w2);
      for (int st = 0; st < kKStages; ++st)
        if (k_armed & (1u << st)) (void)mbar_wait(&s.k_full[st], k_par[st], w2);
    }
    if (warp == kProducer2Warp && lane == 0) {
      for (int st = 0; st < kVStages; ++st)
        if (v_armed & (1u << st)) (void)mbar_wait(&s.v_full[st], v_par[st], w2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_dq_d(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& tdo, int grid, cudaStream_t st) {
  const int smem = (int)sizeof(DqSmem<D>);
  cudaError_t e = ensure_smem_limit((const void*)fm_bwd_dq_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int prof = profile_begin(2, st);
  note_launch();
  fm_bwd_dq_kernel<D><<<grid, qb::kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  profile_end(prof, st);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, int grid, cudaStream_t st) {
  if (p.s.d == 128) return launch_dq_d<128>(p, tq, tk, tv, tdo, grid, st);
  return launch_dq_d<64>(p, tq, tk, tv, tdo, grid, st);
}

}  // namespace fm
