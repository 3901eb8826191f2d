// Mask-aware attention backward, key side (dK, dV), for sm_100a.
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: forward+backward of mask-aware attention.  For the loss sum(O*dO):
//   dV_j = sum_i P_ij dO_i,   dK_j = scale * sum_i dS_ij q_i,
//   dS = P o (dP - D),  dP = dO V^T,  D_i = rowsum(dO_i o O_i).
// dQ is produced by a separate query-stationary kernel (bwd_dq_sm100.cu), so
// this kernel does no cross-CTA reduction at all.
//
// KV-stationary persistent CTAs, one per SM.  A work item is (batch, KV head,
// 128-key tile): K and V stay in shared memory, dV and dK accumulate in TMEM
// over every q-head of the GQA group and every non-skipped 128-row q-tile.
// TMEM (512 columns at d = 128):
//   S^T [0,128) (P^T bf16 written over it)   dP^T [128,256) (dS^T bf16 over it)
// (bf16 pairs of query columns 0-63 at the region's [0,32), of 64-127 at
// [64,96): each compute warpgroup overwrites only TMEM columns it has read)
//   dV [256, 256+d)                          dK [256+d, 256+2d)
// The MMA warp issues, per q-tile t:
//   ... dV(t) = P^T(t) dO(t) ; S^T(t+1) = K Q(t+1)^T ; dK(t) = dS^T(t) Q(t) ;
//   dP^T(t+1) = V dO(t+1)^T ...
// Q tiles (3-deep ring, freed after dK), dO tiles (2-deep, freed after dV)
// and the rows' LSE2 / D (2-deep, freed by the compute warps) stream through
// separate rings, so each is refilled as soon as its last reader is done.
// Tensor-core instructions of one thread execute in issue order, so S^T(t+1)
// may overwrite the S^T region right after dV(t) (which reads P^T(t) from it)
// and dP^T(t+1) right after dK(t).  While the tensor core runs dV(t)+S^T(t+1)
// the compute warps turn dP^T(t) into dS^T(t); while it runs dK(t)+dP^T(t+1)
// they turn S^T(t+1) into P^T(t+1).
//
// Roles (352 threads): warps 0-7 compute (two warpgroups; thread = key lane,
// warpgroup 0 takes query columns 0-63 of the tile, warpgroup 1 columns
// 64-127), warp 8 TMA producer of K and Q, warp 10 TMA producer of V, dO and
// the LSE2 / D rows, warp 9 MMA issuer.  K is released after the item's last
// S^T and V after its last dP^T, so the next item's K/V load overlaps the
// current item's last q-tile.  Work items reach every
// role through a ring of mbarriers (no CTA-wide barrier between items).
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>

#include "bwd_items.cuh"
#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

namespace kvb {
constexpr int kThreads = 352;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kProducer2Warp = 10;
constexpr int kRing = 4;
constexpr int kQStages = 3;   // Q tiles: last read by dK(t)
constexpr int kDoStages = 2;  // dO tiles: last read by dV(t), freed earlier
constexpr int kLStages = 2;   // LSE2 / D rows: last read by the compute warps
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256;
}  // namespace kvb

template <int D>
struct __align__(1024) DkdvSmem {
  uint8_t k[kTile * D * 2];
  uint8_t v[kTile * D * 2];
  uint8_t q[kvb::kQStages][kTile * D * 2];
  uint8_t dout[kvb::kDoStages][kTile * D * 2];
  float lse2[kvb::kLStages][kTile];
  float dsum[kvb::kLStages][kTile];
  KvItem ring[kvb::kRing];
  uint64_t ring_full[kvb::kRing], ring_empty[kvb::kRing];
  uint64_t k_full, k_empty, v_full, v_empty;
  uint64_t q_full[kvb::kQStages], q_empty[kvb::kQStages];
  uint64_t do_full[kvb::kDoStages], do_empty[kvb::kDoStages];
  uint64_t l_full[kvb::kLStages], l_empty[kvb::kLStages];
  uint64_t s_full, dp_full, p_full, ds_full;
  uint64_t dkdv_full, dkdv_free;
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
  int no_abort;
};

static_assert(sizeof(DkdvSmem<128>) <= 232448, "key-side shared memory exceeds the per-CTA limit");
static_assert(sizeof(DkdvSmem<64>) <= 232448, "key-side shared memory exceeds the per-CTA limit");

// D[tmem] = A B^T, both K-major SW128 over the head dimension (128 x 128 tile).
template <int D>
__device__ __forceinline__ void kv_issue_ss(uint32_t d_tmem, const uint8_t* as, const uint8_t* bs) {
  constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
  const uint32_t aa = smem_addr(as), ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, sdesc_sw128(aa + off, 16, 1024), sdesc_sw128(ba + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// D[tmem] (+)= A[tmem] B, B = [128 rows (K) x D] tile read MN-major.  A (bf16
// pairs) holds K-columns 0-63 at a_tmem + [0,32) and 64-127 at a_tmem + [64,96):
// each compute warpgroup writes its half inside the TMEM columns it read.
template <int D>
__device__ __forceinline__ void kv_issue_ts(uint32_t d_tmem, uint32_t a_tmem, const uint8_t* bs, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
  const uint32_t ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ts(d_tmem, a_tmem + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), sdesc_sw128(ba + kk * 2048, 16384, 1024),
           idesc, (accumulate || kk > 0) ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(kvb::kThreads, 1)
    fm_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const BwdParams p) {
  using namespace kvb;
  constexpr int kTileBytes = kTile * D * 2;
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kColDK = kColDV + D;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DkdvSmem<D>& s = *reinterpret_cast<DkdvSmem<D>*>(smem_raw);
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
    mbar_init(&s.k_full, 1);
    mbar_init(&s.k_empty, 1);
    mbar_init(&s.v_full, 1);
    mbar_init(&s.v_empty, 1);
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&s.q_full[i], 1);
      mbar_init(&s.q_empty[i], 1);
    }
    for (int i = 0; i < kDoStages; ++i) {
      mbar_init(&s.do_full[i], 1);
      mbar_init(&s.do_empty[i], 1);
    }
    for (int i = 0; i < kLStages; ++i) {
      mbar_init(&s.l_full[i], 1);
      mbar_init(&s.l_empty[i], 256);
    }
    mbar_init(&s.s_full, 1);
    mbar_init(&s.dp_full, 1);
    mbar_init(&s.p_full, 256);
    mbar_init(&s.ds_full, 256);
    mbar_init(&s.dkdv_full, 1);
    mbar_init(&s.dkdv_free, 256);
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
  const WaitCtx w{&s.abort_flag, p.status, p.wait_limit_ns, smem_addr(smem_raw), 1};
  uint32_t kv_par = 0, kv_armed = 0, vv_par = 0, vv_armed = 0;
  uint32_t q_par[kQStages] = {}, do_par[kDoStages] = {}, l_par[kLStages] = {};
  uint32_t q_armed = 0, do_armed = 0, l_armed = 0;

  if (warp == kProducerWarp) {
    // first producer: the item's K tile and every q-tile's Q
    if (lane == 0) {
      uint32_t sq = 0, act = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int slot = k % kRing;
        if (!(ok = mbar_wait(&s.ring_empty[slot], ((k / kRing) & 1) ^ 1, w))) break;
        const int item = s.abort_flag ? INT_MAX : atomicAdd(p.counter, 1);
        const KvItem it = decode_kv_item(p, item);
        s.ring[slot] = it;
        mbar_arrive(&s.ring_full[slot]);
        if (item >= p.n_items) break;
        if (it.total == 0) continue;
        if (!(ok = mbar_wait(&s.k_empty, (act & 1) ^ 1, w))) break;  // last S^T of the previous item done
        mbar_arrive_expect_tx(&s.k_full, kTileBytes);
        kv_par = act & 1;
        kv_armed = 1;
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx)
          tma_load_4d(s.k + bx * 16384, &tk, &s.k_full, bx * 64, it.hkv, it.kt * kTile, it.b);
        ++act;
        ok = for_each_qtile(p, it, [&](int, int h, int, int qt, int) {
          const int sqi = sq % kQStages;
          const uint32_t pq = (sq / kQStages) & 1;
          if (!mbar_wait(&s.q_empty[sqi], pq ^ 1, w)) return false;
          mbar_arrive_expect_tx(&s.q_full[sqi], kTileBytes);
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_4d(s.q[sqi] + bx * 16384, &tq, &s.q_full[sqi], bx * 64, h, qt * kTile, it.b);
          q_par[sqi] = pq;
          q_armed |= 1u << sqi;
          ++sq;
          return true;
        });
      }
    }
  } else if (warp == kProducer2Warp) {
    // second producer: the item's V tile, every q-tile's dO and LSE2 / D rows
    if (lane == 0) {
      uint32_t sq = 0, act = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int slot = k % kRing;
        if (!(ok = mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w))) break;
        const KvItem it = s.ring[slot];
        mbar_arrive(&s.ring_empty[slot]);
        if (it.item >= p.n_items) break;
        if (it.total == 0) continue;
        if (!(ok = mbar_wait(&s.v_empty, (act & 1) ^ 1, w))) break;  // last dP^T of the previous item done
        mbar_arrive_expect_tx(&s.v_full, kTileBytes);
        vv_par = act & 1;
        vv_armed = 1;
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx)
          tma_load_4d(s.v + bx * 16384, &tv, &s.v_full, bx * 64, it.hkv, it.kt * kTile, it.b);
        ++act;
        ok = for_each_qtile(p, it, [&](int, int h, int, int qt, int) {
          const int sdo = sq % kDoStages, sl = sq % kLStages;
          const uint32_t pd = (sq / kDoStages) & 1, pl = (sq / kLStages) & 1;
          if (!mbar_wait(&s.do_empty[sdo], pd ^ 1, w)) return false;
          mbar_arrive_expect_tx(&s.do_full[sdo], kTileBytes);
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_4d(s.dout[sdo] + bx * 16384, &tdo, &s.do_full[sdo], bx * 64, h, qt * kTile, it.b);
          do_par[sdo] = pd;
          do_armed |= 1u << sdo;
          if (!mbar_wait(&s.l_empty[sl], pl ^ 1, w)) return false;
          mbar_arrive_expect_tx(&s.l_full[sl], 2 * kTile * 4);
          const size_t roff = ((size_t)it.b * sh.Hq + h) * sh.nQt * kTile + (size_t)qt * kTile;
          bulk_load(s.lse2[sl], p.lse2 + roff, kTile * 4, &s.l_full[sl]);
          bulk_load(s.dsum[sl], p.dsum + roff, kTile * 4, &s.l_full[sl]);
          l_par[sl] = pl;
          l_armed |= 1u << sl;
          ++sq;
          return true;
        });
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      uint32_t sq = 0, tc = 0, act = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int slot = k % kRing;
        if (!(ok = mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w))) break;
        const KvItem it = s.ring[slot];
        mbar_arrive(&s.ring_empty[slot]);
        if (it.item >= p.n_items) break;
        const int n = it.total;
        if (n == 0) continue;
        // first q-tile: S^T and dP^T
        {
          const int sqi = sq % kQStages, sdo = sq % kDoStages;
          if (!(ok = mbar_wait(&s.k_full, act & 1, w) && mbar_wait(&s.q_full[sqi], (sq / kQStages) & 1, w))) break;
          tc_fence_after();
          kv_issue_ss<D>(tmem + kColS, s.k, s.q[sqi]);
          mma_commit(&s.s_full);
          if (n == 1) mma_commit(&s.k_empty);  // K read for the last time
          if (!(ok = mbar_wait(&s.v_full, act & 1, w) && mbar_wait(&s.do_full[sdo], (sq / kDoStages) & 1, w))) break;
          tc_fence_after();
          kv_issue_ss<D>(tmem + kColDP, s.v, s.dout[sdo]);
          mma_commit(&s.dp_full);
          if (n == 1) mma_commit(&s.v_empty);  // V read for the last time
        }
        for (int j = 0; j < n; ++j) {
          const uint32_t sj = sq + j, tj = tc + j;
          const int sqi = sj % kQStages, sdo = sj % kDoStages;
          const int sqi2 = (sj + 1) % kQStages, sdo2 = (sj + 1) % kDoStages;
          const uint32_t par = tj & 1;
          if (j == 0 && !(ok = mbar_wait(&s.dkdv_free, (act & 1) ^ 1, w))) break;  // previous item read out
          if (!(ok = mbar_wait(&s.p_full, par, w))) break;
          tc_fence_after();
          kv_issue_ts<D>(tmem + kColDV, tmem + kColS, s.dout[sdo], j > 0);  // dV += P^T dO
          mma_commit(&s.do_empty[sdo]);                                     // dO(j) read for the last time
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&s.q_full[sqi2], ((sj + 1) / kQStages) & 1, w))) break;
            tc_fence_after();
            kv_issue_ss<D>(tmem + kColS, s.k, s.q[sqi2]);  // S^T(j+1), after dV(j) read P^T(j)
            mma_commit(&s.s_full);
            if (j + 2 == n) mma_commit(&s.k_empty);  // K read for the last time
          }
          if (!(ok = mbar_wait(&s.ds_full, par, w))) break;
          tc_fence_after();
          kv_issue_ts<D>(tmem + kColDK, tmem + kColDP, s.q[sqi], j > 0);  // dK += dS^T Q
          mma_commit(&s.q_empty[sqi]);                                     // Q(j) read for the last time
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&s.do_full[sdo2], ((sj + 1) / kDoStages) & 1, w))) break;
            tc_fence_after();
            kv_issue_ss<D>(tmem + kColDP, s.v, s.dout[sdo2]);  // dP^T(j+1), after dK(j) read dS^T(j)
            mma_commit(&s.dp_full);
            if (j + 2 == n) mma_commit(&s.v_empty);  // V read for the last time
          }
        }
        if (!ok) break;
        sq += n;
        tc += n;
        ++act;
        mma_commit(&s.dkdv_full);
      }
    }
  } else {
    // ---------------- compute warpgroups: thread = key, 64 query columns each ----------------
    const int wg = warp >> 2, wq = warp & 3;
    const int jl = wq * 32 + lane;  // key lane
    const uint32_t tb = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t c0 = wg * 64;  // first query column of this warpgroup
    uint32_t sq = 0, tc = 0, act = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int slot = k % kRing;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w)))) break;
      const KvItem it = s.ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.ring_empty[slot]);
      if (it.item >= p.n_items) break;
      const int key = it.kt * kTile + jl;
      if (it.total > 0) {
        int cur_hm = -1;
        int4 rec = make_int4(0, 0, 0, 0);
        ok = for_each_qtile(p, it, [&](int, int, int hm, int qt, int cls) {
          if (hm != cur_hm) {
            rec = p.rec[(((size_t)it.b * sh.Hm + hm) * sh.nKt + it.kt) * kTile + jl];
            cur_hm = hm;
          }
          const int sl = sq % kLStages;
          const uint32_t par = tc & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full, par, w))) return false;
          if (!__all_sync(0xffffffffu, mbar_wait(&s.l_full[sl], (sq / kLStages) & 1, w))) return false;
          tc_fence_after();
          const float* l2 = s.lse2[sl] + c0;
          const float* dsm = s.dsum[sl] + c0;
          const bool need = cls == kClsPartial;
          // this key's masked rows among the warpgroup's 64 query rows, as two
          // 32-bit words (interval arithmetic on the column's boundaries)
          uint32_t mw0 = 0u, mw1 = 0u;
          if (need) {
            const int row0 = qt * kTile + c0;
            mw0 = column_row_bits(rec, row0);
            mw1 = column_row_bits(rec, row0 + 32);
          }
          // P^T for 64 query columns, in place over the loaded S^T values
          uint32_t pr[64];
          tmem_ld32x(tb + kColS + c0, pr);
          tmem_ld32x(tb + kColS + c0 + 32, pr + 32);
          tmem_ld_wait();
#pragma unroll
          for (int i4 = 0; i4 < 16; ++i4) {  // 16-byte broadcast reads of the rows' LSE2
            const float4 lv = reinterpret_cast<const float4*>(l2)[i4];
            const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int i = i4 * 4 + u;
              const float pv = fast_exp2(fmaf(__uint_as_float(pr[i]), p.scale_log2, -lq[u]));
              const uint32_t bit = ((i < 32 ? mw0 : mw1) >> (i & 31)) & 1u;
              pr[i] = bit ? 0u : __float_as_uint(pv);
            }
          }
          {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
            tmem_st32x(tb + kColS + c0, pk);  // bf16 pairs over this warpgroup's own S^T columns
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&s.p_full);
          // dS^T = P^T o (dP^T - D)
          if (!__all_sync(0xffffffffu, mbar_wait(&s.dp_full, par, w))) return false;
          tc_fence_after();
          {
            uint32_t r[64];
            tmem_ld32x(tb + kColDP + c0, r);
            tmem_ld32x(tb + kColDP + c0 + 32, r + 32);
            tmem_ld_wait();
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {  // 16-byte broadcast reads of the rows' D
              const float4 dv4 = reinterpret_cast<const float4*>(dsm)[i4];
              const float dq4[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int i = i4 * 4 + u;
                pr[i] = __float_as_uint(__uint_as_float(pr[i]) * (__uint_as_float(r[i]) - dq4[u]));
              }
            }
          }
          {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
            tmem_st32x(tb + kColDP + c0, pk);  // bf16 pairs over this warpgroup's own dP^T columns
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&s.ds_full);
          mbar_arrive(&s.l_empty[sl]);  // LSE2 / D of this q-tile no longer read
          ++sq;
          ++tc;
          return true;
        });
        if (!ok) break;
        // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.dkdv_full, act & 1, w)))) break;
        tc_fence_after();
        const bool valid = key < sh.Nk;
        const size_t off = (((size_t)it.b * sh.Nk + (valid ? key : 0)) * sh.Hkv + it.hkv) * D;
        __nv_bfloat16* dst = (wg == 0 ? p.dv : p.dk) + off;
        const float mul = (wg == 0) ? 1.f : p.scale;
        const uint32_t col = (wg == 0) ? kColDV : kColDK;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32x(tb + col + c * 32, rr);
          tmem_ld_wait();
          uint32_t pk2[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk2[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * mul, __uint_as_float(rr[2 * i + 1]) * mul);
          if (valid) {
#pragma unroll
            for (int i = 0; i < 4; ++i) st_global_v4_na(dst + c * 32 + i * 8, pk2[4 * i], pk2[4 * i + 1], pk2[4 * i + 2], pk2[4 * i + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(&s.dkdv_free);
        ++act;
      } else if (key < sh.Nk) {
        // no q-tile reaches this key tile: dK = dV = 0 (each warpgroup one of them)
        const size_t off = (((size_t)it.b * sh.Nk + key) * sh.Hkv + it.hkv) * D;
        uint4* d4 = reinterpret_cast<uint4*>((wg == 0 ? p.dv : p.dk) + off);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) d4[i] = make_uint4(0, 0, 0, 0);
      }
    }
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (s.abort_flag) {
    const WaitCtx w2{&s.no_abort, p.status, p.wait_limit_ns, smem_addr(smem_raw), 1};
    if (warp == kMmaWarp && lane == 0) {
      mma_commit(&s.teardown);
      (void)mbar_wait(&s.teardown, 0, w2);
    }
    if (warp == kProducerWarp && lane == 0) {
      if (kv_armed) (void)mbar_wait(&s.k_full, kv_par, w2);
      for (int st = 0; st < kQStages; ++st)
        if (q_armed & (1u << st)) (void)mbar_wait(&s.q_full[st], q_par[st], w2);
    }
    if (warp == kProducer2Warp && lane == 0) {
      if (vv_armed) (void)mbar_wait(&s.v_full, vv_par, w2);
      for (int st = 0; st < kDoStages; ++st)
        if (do_armed & (1u << st)) (void)mbar_wait(&s.do_full[st], do_par[st], w2);
      for (int st = 0; st < kLStages; ++st)
        if (l_armed & (1u << st)) (void)mbar_wait(&s.l_full[st], l_par[st], w2);
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
static cudaError_t launch_dkdv_d(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& tdo, int grid, cudaStream_t st) {
  const int smem = (int)sizeof(DkdvSmem<D>);
  cudaError_t e = ensure_smem_limit((const void*)fm_bwd_dkdv_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int prof = profile_begin(1, st);
  note_launch();
  fm_bwd_dkdv_kernel<D><<<grid, kvb::kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  profile_end(prof, st);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, int grid, cudaStream_t st) {
  if (p.s.d == 128) return launch_dkdv_d<128>(p, tq, tk, tv, tdo, grid, st);
  return launch_dkdv_d<64>(p, tq, tk, tv, tdo, grid, st);
}

}  // namespace fm
