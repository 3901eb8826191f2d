// Mask-aware attention backward in one key-stationary pass (dQ, dK, dV), for
// sm_100a.
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: forward+backward of mask-aware attention.  For the loss sum(O*dO):
//   dV_j = sum_i P_ij dO_i,   dK_j = scale * sum_i dS_ij q_i,
//   dQ_i = scale * sum_j dS_ij k_j,
//   dS = P o (dP - D),  dP = dO V^T,  D_i = rowsum(dO_i o O_i).
// Each (query tile, key tile) pair is visited once: S, dP and dS are formed
// once and feed all three gradients (the method's 5 matmuls per pair).  dK and
// dV accumulate in TMEM over the whole GQA group; each pair's dQ contribution
// dS K leaves the SM as fp32 bulk reductions (the TMA unit's
// cp.reduce.async.bulk, two of 32 KiB per pair at d = 128) into a tiled
// accumulator in global memory laid out so that each half of a tile's dQ is
// one contiguous range, which a finalize kernel scales and converts to bf16.  dK and dV are deterministic; dQ's fp32 sums depend on
// the order in which the CTAs' reductions land.
//
// KV-stationary persistent CTAs, one per SM.  A work item is (batch, KV head,
// 128-key tile); K and V stay in shared memory.  TMEM (512 columns at d = 128):
//   S^T [0,128) (P^T bf16 written over it)
//   dP^T [128,256) (dS^T bf16 written over it; then dQ(t) [128, 128+d))
//   dV [256, 256+d)   dK [256+d, 256+2d)
// (bf16 pairs of query columns 0-63 at the region's [0,32), of 64-127 at
// [64,96): each compute warpgroup overwrites only TMEM columns it has read.)
// The compute warps also write dS^T(t) as bf16 into shared memory (rows = keys,
// 128-byte swizzle): as the A operand of dQ(t) = dS(t) K it is read MN-major.
// MMA issue order per q-tile t:
//   dV(t) = P^T(t) dO(t) ; S^T(t+1) = K Q(t+1)^T ;
//   dK(t) += dS^T(t) Q(t) ; dQ(t) = dS(t) K  (into the dP^T region) ;
//   dP^T(t+1) = V dO(t+1)^T  (once dQ(t) has been read out of TMEM)
// Tensor-core instructions of one thread execute in issue order, so S^T(t+1)
// may overwrite the S^T region right after dV(t), and dQ(t) the dP^T region
// right after dK(t) has read dS^T(t) from it.
// A fourth warpgroup reads dQ(t) out of TMEM (freeing the region for
// dP^T(t+1) as soon as the loads complete) and sends it as fp32 reductions:
// only it waits on the L2's reduction rate (about 20 bytes per clock per SM
// when every SM reduces), never the compute warps' chain.
//
// Roles (512 threads, registers split per warpgroup with setmaxnreg): warps
// 0-7 compute (two warpgroups; thread = key lane; warpgroup 0 takes query
// columns 0-63, warpgroup 1 64-127), warps 8-11 the dQ read-out (thread =
// query row), warp 12 TMA producer of K and Q, warp 14 TMA producer of V, dO
// and the LSE2 / D rows, warp 13 MMA issuer, warp 15 idle.
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>

#include "bwd_items.cuh"
#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

namespace fb {
constexpr int kThreads = 512;
constexpr int kDrainWarp0 = 8;  // warps 8-11: the dQ read-out warpgroup
constexpr int kProducerWarp = 12, kMmaWarp = 13, kProducer2Warp = 14;  // warp 15 idles
constexpr int kRing = 4;
constexpr int kQStages = 2;   // Q tiles: last read by dK(t)
constexpr int kDoStages = 1;  // dO tiles: last read by dV(t); dO(t+1) is needed only after dQ(t) is read out
// Registers per thread after the per-warpgroup split (setmaxnreg): compute,
// dQ read-out, and the producer/MMA warpgroup.  The block is launched with
// 128 per thread; the shares must not add up to more than that total.
constexpr int kRegCompute = 160, kRegDrain = 72, kRegControl = 120;
static_assert(2 * 128 * kRegCompute + 128 * kRegDrain + 128 * kRegControl <= kThreads * 128,
              "the register split must fit the launch's registers");
constexpr int kLStages = 2;   // LSE2 / D rows: last read by the compute warps
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256;
constexpr uint32_t kColDQ = kColDP;  // dQ(t) reuses the dP^T region
}  // namespace fb

template <int D>
struct __align__(1024) FusedSmem {
  uint8_t k[kTile * D * 2];
  uint8_t v[kTile * D * 2];
  uint8_t q[fb::kQStages][kTile * D * 2];
  uint8_t dout[fb::kDoStages][kTile * D * 2];
  // dS^T bf16 (rows = keys, box g = query columns [64g, 64g+64), SW128); once
  // dQ(t) has read it, the fp32 dQ(t) columns 0-63 staged for reduction
  uint8_t ds[2][kTile * 64 * 2];
  float4 stage[16 * kTile];  // fp32 dQ(t) columns 64-127 staged for reduction
  float lse2[fb::kLStages][kTile];
  float dsum[fb::kLStages][kTile];
  KvItem ring[fb::kRing];
  uint64_t ring_full[fb::kRing], ring_empty[fb::kRing];
  uint64_t k_full, k_empty, v_full, v_empty;
  uint64_t q_full[fb::kQStages], q_empty[fb::kQStages];
  uint64_t do_full[fb::kDoStages], do_empty[fb::kDoStages];
  uint64_t l_full[fb::kLStages], l_empty[fb::kLStages];
  uint64_t s_full, dp_full, p_full, ds_full, dq_full, dq_free;
  uint64_t staged;      // the read-out warpgroup wrote dQ(t) into the two buffers
  uint64_t dsbuf_free;  // the reduction has read the dS buffer: dS(t+1) may be written
  uint64_t buf_free;    // the reductions have read both buffers: dQ(t+1) may be staged
  uint64_t dkdv_full, dkdv_free;
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
  int no_abort;
};

static_assert(sizeof(FusedSmem<128>) <= 232448, "fused backward shared memory exceeds the per-CTA limit");
static_assert(sizeof(FusedSmem<64>) <= 232448, "fused backward shared memory exceeds the per-CTA limit");

// D[tmem] = A B^T, both K-major SW128 over the head dimension (128 x 128 tile).
template <int D>
__device__ __forceinline__ void fb_issue_ss(uint32_t d_tmem, const uint8_t* as, const uint8_t* bs) {
  constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
  const uint32_t aa = smem_addr(as), ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, sdesc_sw128(aa + off, 16, 1024), sdesc_sw128(ba + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// D[tmem] (+)= A[tmem] B, B = [128 rows (K) x D] tile read MN-major; A (bf16
// pairs) holds K-columns 0-63 at a_tmem + [0,32) and 64-127 at a_tmem + [64,96).
template <int D>
__device__ __forceinline__ void fb_issue_ts(uint32_t d_tmem, uint32_t a_tmem, const uint8_t* bs, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
  const uint32_t ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ts(d_tmem, a_tmem + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), sdesc_sw128(ba + kk * 2048, 16384, 1024),
           idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// dQ(t) = dS(t) K: M = 128 query rows, N = D, K = 128 keys.  A = dS from the
// shared dS^T buffer (rows = keys, queries contiguous in two 64-column SW128
// boxes) read MN-major; B = the K tile (rows = keys, d contiguous) read
// MN-major.  One K-step covers 16 key rows (2048 bytes of each box).
template <int D>
__device__ __forceinline__ void fb_issue_dq(uint32_t d_tmem, const uint8_t* ds, const uint8_t* ks) {
  constexpr uint32_t idesc = idesc_bf16(128, D, true, true);
  const uint32_t da = smem_addr(ds), ka = smem_addr(ks);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ss(d_tmem, sdesc_sw128(da + kk * 2048, 16384, 1024), sdesc_sw128(ka + kk * 2048, 16384, 1024), idesc,
           kk > 0 ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(fb::kThreads, 1)
    fm_bwd_fused_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                        const BwdParams p) {
  using namespace fb;
  constexpr int kTileBytes = kTile * D * 2;
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kColDK = kColDV + D;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  FusedSmem<D>& s = *reinterpret_cast<FusedSmem<D>*>(smem_raw);
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
      mbar_init(&s.ring_empty[i], 14);  // MMA + second producer + lane 0 of the 8 compute and 4 read-out warps
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
    mbar_init(&s.dq_full, 1);
    mbar_init(&s.dq_free, 128);  // the read-out warpgroup
    mbar_init(&s.staged, 128);
    mbar_init(&s.dsbuf_free, 1);
    mbar_init(&s.buf_free, 1);
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
  const WaitCtx w{&s.abort_flag, p.status, p.wait_limit_ns, smem_addr(smem_raw), 4};
  uint32_t kv_par = 0, kv_armed = 0, vv_par = 0, vv_armed = 0;
  uint32_t q_par[kQStages] = {}, do_par[kDoStages] = {}, l_par[kLStages] = {};
  uint32_t q_armed = 0, do_armed = 0, l_armed = 0;

  // Every role starts with its warpgroup's register share (setmaxnreg; all
  // warps of a warpgroup execute the same one).
  if (warp == kProducerWarp) {
    setmaxnreg_dec<kRegControl>();
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
        if (!(ok = mbar_wait(&s.k_empty, (act & 1) ^ 1, w))) break;  // last dQ of the previous item done
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
    setmaxnreg_dec<kRegControl>();
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
    setmaxnreg_dec<kRegControl>();
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
        // first q-tile: S^T and dP^T (the latter once the previous item's last
        // dQ has been read out of the dP^T region)
        {
          const int sqi = sq % kQStages, sdo = sq % kDoStages;
          if (!(ok = mbar_wait(&s.k_full, act & 1, w) && mbar_wait(&s.q_full[sqi], (sq / kQStages) & 1, w))) break;
          tc_fence_after();
          fb_issue_ss<D>(tmem + kColS, s.k, s.q[sqi]);
          mma_commit(&s.s_full);
          if (!(ok = mbar_wait(&s.v_full, act & 1, w) && mbar_wait(&s.do_full[sdo], (sq / kDoStages) & 1, w))) break;
          if (tc > 0 && !(ok = mbar_wait(&s.dq_free, (tc - 1) & 1, w))) break;
          tc_fence_after();
          fb_issue_ss<D>(tmem + kColDP, s.v, s.dout[sdo]);
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
          fb_issue_ts<D>(tmem + kColDV, tmem + kColS, s.dout[sdo], j > 0);  // dV += P^T dO
          mma_commit(&s.do_empty[sdo]);                                     // dO(j) read for the last time
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&s.q_full[sqi2], ((sj + 1) / kQStages) & 1, w))) break;
            tc_fence_after();
            fb_issue_ss<D>(tmem + kColS, s.k, s.q[sqi2]);  // S^T(j+1), after dV(j) read P^T(j)
            mma_commit(&s.s_full);
          }
          if (!(ok = mbar_wait(&s.ds_full, par, w))) break;
          tc_fence_after();
          fb_issue_ts<D>(tmem + kColDK, tmem + kColDP, s.q[sqi], j > 0);  // dK += dS^T Q
          mma_commit(&s.q_empty[sqi]);                                     // Q(j) read for the last time
          fb_issue_dq<D>(tmem + kColDQ, s.ds[0], s.k);                     // dQ(j) = dS K, after dK(j) read dS^T
          mma_commit(&s.dq_full);
          if (j + 1 == n) mma_commit(&s.k_empty);  // K read for the last time
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&s.dq_free, par, w) &&  // dQ(j) read out of the dP^T region
                       mbar_wait(&s.do_full[sdo2], ((sj + 1) / kDoStages) & 1, w)))
              break;
            tc_fence_after();
            fb_issue_ss<D>(tmem + kColDP, s.v, s.dout[sdo2]);  // dP^T(j+1)
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
  } else if (warp >= kDrainWarp0 && warp < kDrainWarp0 + 4) {
    // ---------------- dQ read-out warpgroup: thread = query row (TMEM lane) ----------------
    // Copies dQ(t) from TMEM into shared memory in the accumulator tile's
    // layout (columns 0-63 into the dS buffer, which dQ(t) has finished
    // reading, 64-127 into the staging buffer), 64 columns (two loads) at a
    // time, frees the TMEM region once the last load has completed
    // (dP^T(t+1) may then be issued), and has one thread
    // hand both halves to the TMA unit as asynchronous bulk fp32 reductions
    // into [B, Hq, nQt, D/4, 128, 4].  Only that thread waits on the L2's
    // reduction rate (about 20 bytes per clock per SM when every SM reduces):
    // it releases the dS buffer, then the staging buffer, as the reductions
    // read them.
    setmaxnreg_dec<kRegDrain>();
    const int wq = warp & 3;
    const int jl = wq * 32 + lane;
    const uint32_t tb = tmem + ((uint32_t)(wq * 32) << 16);
    const bool elected = (wq == 0 && lane == 0);
    float4* lo = reinterpret_cast<float4*>(s.ds[0]);  // 32 KiB: chunks 0 .. D/8 - 1
    float4* hi = s.stage;                              // chunks D/8 .. D/4 - 1
    uint32_t tc = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int slot = k % kRing;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w)))) break;
      const KvItem it = s.ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.ring_empty[slot]);
      if (it.item >= p.n_items) break;
      if (it.total == 0) continue;
      ok = for_each_qtile(p, it, [&](int, int h, int, int qt, int) {
        // the previous reductions have read both buffers; dQ(t) has completed
        if (tc > 0 && !__all_sync(0xffffffffu, mbar_wait(&s.buf_free, (tc - 1) & 1, w))) return false;
        if (!__all_sync(0xffffffffu, mbar_wait(&s.dq_full, tc & 1, w))) return false;
        tc_fence_after();
#pragma unroll
        for (int cp = 0; cp < D / 64; ++cp) {  // 64 columns (two loads in flight) at a time
          uint32_t r[64];
          tmem_ld32x(tb + kColDQ + cp * 64, r);
          tmem_ld32x(tb + kColDQ + cp * 64 + 32, r + 32);
          tmem_ld_wait();
          if (cp == D / 64 - 1) {  // every column read: the region may take dP^T(t+1)
            tc_fence_before();
            mbar_arrive(&s.dq_free);
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int c = 2 * cp + h2;
            float4* dst = (c < D / 64) ? lo + c * 8 * kTile : hi + (c - D / 64) * 8 * kTile;
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4)
              dst[c4 * kTile + jl] =
                  make_float4(__uint_as_float(r[32 * h2 + 4 * c4]), __uint_as_float(r[32 * h2 + 4 * c4 + 1]),
                              __uint_as_float(r[32 * h2 + 4 * c4 + 2]), __uint_as_float(r[32 * h2 + 4 * c4 + 3]));
          }
        }
        fence_async_smem();
        mbar_arrive(&s.staged);
        bool issued = true;
        if (elected) {
          issued = mbar_wait(&s.staged, tc & 1, w);
          if (issued) {
            float* acc = p.dqacc + (((size_t)it.b * sh.Hq + h) * sh.nQt + qt) * ((size_t)kTile * D);
            constexpr uint32_t kHalfBytes = (D / 8) * kTile * 16;
            bulk_reduce_add_f32(acc, lo, kHalfBytes);
            bulk_commit_group();
            bulk_reduce_add_f32(acc + (D / 8) * kTile * 4, hi, kHalfBytes);
            bulk_commit_group();
            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");  // the dS buffer has been read
            mbar_arrive(&s.dsbuf_free);
            bulk_wait_read_all();
            mbar_arrive(&s.buf_free);
          }
        }
        if (!__all_sync(0xffffffffu, issued)) return false;
        ++tc;
        return true;
      });
    }
    if (elected) bulk_wait_all();  // every reduction has landed before the CTA ends
  } else if (warp < 8) {
    setmaxnreg_inc<kRegCompute>();
    // ---------------- compute warpgroups ----------------
    // S^T / dP^T: thread = key lane, warpgroup wg takes query columns
    // [64 wg, 64 wg + 64).  dQ: thread = query row (the same TMEM lane),
    // warpgroup wg takes dQ columns [wg D/2, wg D/2 + D/2).
    const int wg = warp >> 2, wq = warp & 3;
    const int jl = wq * 32 + lane;  // TMEM lane: key for S^T/dP^T, query row for dQ
    const uint32_t tb = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t c0 = wg * 64;  // first query column of this warpgroup
    uint8_t* ds_row = s.ds[wg] + jl * 128;  // this key's row of the warpgroup's dS^T box
    const int sw = jl & 7;                  // 128-byte swizzle of the row's 16-byte chunks
    uint32_t sq = 0, tc = 0, act = 0;
    bool ok = true;
    // Reads dQ(t) (parity par) out of TMEM into fp32 reductions of its tile in
    // the accumulator ([B, Hq, nQt, D/4, 128, 4]); frees the TMEM region once
    // the loads have completed, then issues the reductions.
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
        ok = for_each_qtile(p, it, [&](int j, int h, int hm, int qt, int cls) {
          if (hm != cur_hm) {
            rec = p.rec[(((size_t)it.b * sh.Hm + hm) * sh.nKt + it.kt) * kTile + jl];
            cur_hm = hm;
          }
          const int sl = sq % kLStages;
          const uint32_t par = tc & 1;
          // this key's masked rows among the warpgroup's 64 query rows, as two
          // 32-bit words (interval arithmetic on the column's boundaries)
          uint32_t mw0 = 0u, mw1 = 0u;
          if (cls == kClsPartial) {
            const int row0 = qt * kTile + c0;
            mw0 = column_row_bits(rec, row0);
            mw1 = column_row_bits(rec, row0 + 32);
          }
          if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full, par, w))) return false;
          if (!__all_sync(0xffffffffu, mbar_wait(&s.l_full[sl], (sq / kLStages) & 1, w))) return false;
          tc_fence_after();
          const float* l2 = s.lse2[sl] + c0;
          const float* dsm = s.dsum[sl] + c0;
          // P^T for 64 query columns in two halves of 32, each written back as
          // 16 bf16 pairs over S^T columns this warpgroup has read
          uint32_t pr[64];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32x(tb + kColS + c0 + half * 32, pr + half * 32);
            tmem_ld_wait();
            const uint32_t mw = half ? mw1 : mw0;
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {  // 16-byte broadcast reads of the rows' LSE2
              const float4 lv = reinterpret_cast<const float4*>(l2 + half * 32)[i4];
              const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int i = half * 32 + i4 * 4 + u;
                const float pv = fast_exp2(fmaf(__uint_as_float(pr[i]), p.scale_log2, -lq[u]));
                pr[i] = ((mw >> (i & 31)) & 1u) ? 0u : __float_as_uint(pv);
              }
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(pr[half * 32 + 2 * i]), __uint_as_float(pr[half * 32 + 2 * i + 1]));
            tmem_st16(tb + kColS + c0 + half * 16, pk);
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
            // and the same 64 values into this key's row of the shared dS^T box,
            // once the previous q-tile's dQ staged there has been read by its reduction
            if (tc > 0 && !__all_sync(0xffffffffu, mbar_wait(&s.dsbuf_free, (tc - 1) & 1, w))) return false;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(ds_row + ((c ^ sw) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
          fence_async_smem();
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
  } else {
    setmaxnreg_dec<kRegControl>();  // warp 15: idle, in the producer/MMA warpgroup
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (s.abort_flag) {
    const WaitCtx w2{&s.no_abort, p.status, p.wait_limit_ns, smem_addr(smem_raw), 4};
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

// ----------------------------------------------------------------------------
// dQ finalize: dQ = bf16(scale * acc), from the tiled fp32 accumulator to the
// [B, Nq, Hq, D] layout.  One CTA per (batch, q-head, q-tile), 64 columns at a
// time through shared memory: the accumulator is read in its own order (each
// warp 512 contiguous bytes), rows are written as whole 128-byte segments.
// HBM-bound: 4 bytes read and 2 written per element.
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fm_dq_finalize_kernel(BwdParams p) {
  const Shape& sh = p.s;
  constexpr int kPad = 68;  // row stride in floats (64 + 4): 16-byte aligned, spreads banks
  __shared__ __align__(16) float tile[kTile * kPad];
  const int64_t n_tiles = (int64_t)sh.B * sh.Hq * sh.nQt;
  const int t = threadIdx.x;
  const float sc = p.scale;
  for (int64_t tix = blockIdx.x; tix < n_tiles; tix += gridDim.x) {
    const int qt = (int)(tix % sh.nQt);
    const int64_t bh = tix / sh.nQt;
    const int h = (int)(bh % sh.Hq), b = (int)(bh / sh.Hq);
    const float4* acc = reinterpret_cast<const float4*>(p.dqacc + tix * ((int64_t)kTile * D));
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
      // 16 four-column chunks x 128 rows of this half: 2048 float4, 8 per thread
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int f = t + 256 * i;
        const int c = f >> 7, r = f & 127;
        const float4 x = acc[(half * 16 + c) * kTile + r];
        *reinterpret_cast<float4*>(&tile[r * kPad + 4 * c]) = x;
      }
      __syncthreads();
      // 128 rows x 64 columns as bf16: 8 threads per row, 16 bytes each
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int r = pass * 32 + (t >> 3), seg = t & 7;
        const int i = qt * kTile + r;
        if (i < sh.Nq) {
          const float* src = &tile[r * kPad + seg * 8];
          const float4 a = *reinterpret_cast<const float4*>(src);
          const float4 c = *reinterpret_cast<const float4*>(src + 4);
          uint4 o;
          o.x = pack_bf16x2(a.x * sc, a.y * sc);
          o.y = pack_bf16x2(a.z * sc, a.w * sc);
          o.z = pack_bf16x2(c.x * sc, c.y * sc);
          o.w = pack_bf16x2(c.z * sc, c.w * sc);
          *reinterpret_cast<uint4*>(p.dq + (((size_t)b * sh.Nq + i) * sh.Hq + h) * D + half * 64 + seg * 8) = o;
        }
      }
      __syncthreads();
    }
  }
}

template <int D>
static cudaError_t launch_fused_d(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const CUtensorMap& tdo, int grid, cudaStream_t st) {
  const int smem = (int)sizeof(FusedSmem<D>);
  cudaError_t e = ensure_smem_limit((const void*)fm_bwd_fused_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int prof = profile_begin(4, st);
  note_launch();
  fm_bwd_fused_kernel<D><<<grid, fb::kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  profile_end(prof, st);
  return cudaGetLastError();
}

cudaError_t launch_bwd_fused(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, int grid, cudaStream_t st) {
  if (p.s.d == 128) return launch_fused_d<128>(p, tq, tk, tv, tdo, grid, st);
  return launch_fused_d<64>(p, tq, tk, tv, tdo, grid, st);
}

cudaError_t launch_dq_finalize(const BwdParams& p, int max_blocks, cudaStream_t st) {
  const int64_t n_tiles = (int64_t)p.s.B * p.s.Hq * p.s.nQt;
  if (n_tiles == 0) return cudaSuccess;
  int64_t blocks = n_tiles;
  if (blocks > max_blocks) blocks = max_blocks;  // grid-stride loop over the tiles
  const int prof = profile_begin(5, st);
  note_launch();
  if (p.s.d == 128)
    fm_dq_finalize_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(p);
  else
    fm_dq_finalize_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(p);
  profile_end(prof, st);
  return cudaGetLastError();
}

}  // namespace fm
