// Mask-aware attention forward for sm_100a.
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: attention forward driven by the column-wise mask, skipping tiles
// that the boundary vectors prove fully masked and applying the element mask
// only on partially masked tiles.  The page's kernel is a Hopper design
// (TMA/WGMMA with three warp roles); this one is written for Blackwell:
//
//   * persistent CTAs (one per SM) take work items -- (batch, q-head, block of
//     two 128-row q-tiles) -- from a longest-first list through an atomic
//     counter;
//   * warp 8 issues TMA loads (Q once per item; K, V and, for tiles that need
//     it, the 2 KiB boundary records through a multi-stage ring);
//   * warp 9 issues tcgen05 MMAs: S_g = Q_g K^T into TMEM, O_g += P_g V with
//     P_g read from TMEM (bf16, written over S_g);
//   * warps 0-3 and 4-7 are the softmax groups of q-tiles 0 and 1: one thread
//     per query row, S read with tcgen05.ld, online softmax in the exp2
//     domain, O rescaled in TMEM only when a row maximum grows by more than
//     2^8 (otherwise the stale maximum is kept, exact after the final 1/l).
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 after O0.
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

template <int D>
struct FwdCfg {
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kTileBytes = kTile * D * 2;  // one 128-row bf16 tile
  static constexpr int kBoxes = D / 64;             // 64-column (128-byte) TMA boxes per tile
  static constexpr int kThreads = 320;
  static constexpr int kProducerWarp = 8;
  static constexpr int kMmaWarp = 9;
};

template <int D>
struct __align__(1024) FwdSmem {
  uint8_t q[2][FwdCfg<D>::kTileBytes];
  uint8_t k[FwdCfg<D>::kStages][FwdCfg<D>::kTileBytes];
  uint8_t v[FwdCfg<D>::kStages][FwdCfg<D>::kTileBytes];
  int4 mask[FwdCfg<D>::kStages][kTile];
  uint64_t q_full;
  uint64_t k_full[FwdCfg<D>::kStages];
  uint64_t v_full[FwdCfg<D>::kStages];
  uint64_t kv_empty[FwdCfg<D>::kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
  int no_abort;
  int item;
};

// S = Q K^T: M = 128 rows, N = 128 keys, K = D; both operands K-major SW128.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, const uint8_t* qs, const uint8_t* ks) {
  constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
  const uint32_t qa = smem_addr(qs), ka = smem_addr(ks);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V: M = 128 rows, N = D, K = 128 keys.  P from TMEM (bf16 pairs,
// 8 columns per 16 keys); V is MN-major (d contiguous) SW128.
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, const uint8_t* vs, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
  const uint32_t va = smem_addr(vs);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(va + kk * 2048, 16384, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ void tmem_ld32p(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32p(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::kThreads, 1)
    fm_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int kStages = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  FwdSmem<D>& s = *reinterpret_cast<FwdSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Shape& sh = p.s;

  if (smem_addr(smem_raw) & 1023u) {  // SW128 operands need 1024-byte alignment
    if (tid == 0) atomicCAS(p.status, 0, -5);
    return;
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.kv_empty[i], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s.s_full[g], 1);
      mbar_init(&s.p_full[g], 128);
      mbar_init(&s.o_full[g], 1);
    }
    mbar_init(&s.teardown, 1);
    s.abort_flag = 0;
    s.no_abort = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::kProducerWarp && lane == 0) {
    tma_prefetch_map(&tq);
    tma_prefetch_map(&tk);
    tma_prefetch_map(&tv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const WaitCtx w{&s.abort_flag, p.status, p.wait_limit_ns};

  // Per-role counters; every role walks the same tiles in the same order.
  uint32_t kv_iter = 0;    // position in the K/V ring
  uint32_t tile_cnt = 0;   // tiles processed (parity of s_full / p_full)
  uint32_t act_cnt = 0;    // items with at least one tile (parity of q_full / o_full)
  uint32_t q_par = 0, k_par[kStages] = {}, v_par[kStages] = {};  // producer: last armed phases
  uint32_t k_armed = 0, q_armed = 0;

  for (;;) {
    if (tid == 0) s.item = s.abort_flag ? INT_MAX : atomicAdd(p.counter, 1);
    __syncthreads();
    const int item = s.item;
    if (item >= p.n_items) break;
    const ItemCoord c = decode_fwd_item(sh, p.order[item]);
    const int b = c.b, qb = c.t, hkv = c.hkv;
    const int h = hkv * sh.G + c.hg;
    const int hm = (sh.Hm == 1) ? 0 : h;
    const size_t lrow = ((size_t)b * sh.Hm + hm) * sh.nQB + qb;
    const int* list = p.flist + lrow * sh.nKt;
    const int n = p.fcount[lrow];

    if (warp == Cfg::kProducerWarp) {
      if (lane == 0 && n > 0) {
        mbar_arrive_expect_tx(&s.q_full, 2 * Cfg::kTileBytes);
        q_par = act_cnt & 1;
        q_armed = 1;
#pragma unroll
        for (int g = 0; g < 2; ++g)
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_4d(s.q[g] + bx * 16384, &tq, &s.q_full, bx * 64, h, qb * 256 + g * kTile, b);
        for (int t = 0; t < n; ++t, ++kv_iter) {
          const int e = list[t];
          const int kt = e >> 8;
          const bool need = ((e & 3) != kClsFull) || (((e >> 2) & 3) != kClsFull) || ((e >> 4) & 1);
          const int st = kv_iter % kStages;
          const uint32_t ph = (kv_iter / kStages) & 1;
          if (!mbar_wait(&s.kv_empty[st], ph ^ 1, w)) break;
          mbar_arrive_expect_tx(&s.k_full[st], Cfg::kTileBytes + (need ? kTile * 16 : 0));
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_4d(s.k[st] + bx * 16384, &tk, &s.k_full[st], bx * 64, hkv, kt * kTile, b);
          if (need)
            bulk_load(s.mask[st], p.rec + (((size_t)b * sh.Hm + hm) * sh.nKt + kt) * kTile, kTile * 16,
                      &s.k_full[st]);
          mbar_arrive_expect_tx(&s.v_full[st], Cfg::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_4d(s.v[st] + bx * 16384, &tv, &s.v_full[st], bx * 64, hkv, kt * kTile, b);
          k_par[st] = ph;
          v_par[st] = ph;
          k_armed |= 1u << st;
        }
      }
    } else if (warp == Cfg::kMmaWarp) {
      if (lane == 0 && n > 0) {
        bool ok = mbar_wait(&s.q_full, act_cnt & 1, w);
        tc_fence_after();
        for (int t = 0; ok && t < n; ++t) {
          const int st = kv_iter % kStages;
          const uint32_t ph = (kv_iter / kStages) & 1;
          const int st2 = (kv_iter + 1) % kStages;
          const uint32_t ph2 = ((kv_iter + 1) / kStages) & 1;
          if (t == 0) {
            if (!(ok = mbar_wait(&s.k_full[st], ph, w))) break;
            tc_fence_after();
            issue_qk<D>(tmem + 0, s.q[0], s.k[st]);
            mma_commit(&s.s_full[0]);
            issue_qk<D>(tmem + 128, s.q[1], s.k[st]);
            mma_commit(&s.s_full[1]);
          }
          if (!(ok = mbar_wait(&s.v_full[st], ph, w) && mbar_wait(&s.p_full[0], tile_cnt & 1, w))) break;
          tc_fence_after();
          issue_pv<D>(tmem + 256, tmem + 0, s.v[st], t > 0);
          if (t == n - 1) mma_commit(&s.o_full[0]);
          if (t + 1 < n) {
            if (!(ok = mbar_wait(&s.k_full[st2], ph2, w))) break;
            tc_fence_after();
            issue_qk<D>(tmem + 0, s.q[0], s.k[st2]);
            mma_commit(&s.s_full[0]);
          }
          if (!(ok = mbar_wait(&s.p_full[1], tile_cnt & 1, w))) break;
          tc_fence_after();
          issue_pv<D>(tmem + 256 + D, tmem + 128, s.v[st], t > 0);
          if (t == n - 1) mma_commit(&s.o_full[1]);
          mma_commit(&s.kv_empty[st]);
          if (t + 1 < n) {
            issue_qk<D>(tmem + 128, s.q[1], s.k[st2]);
            mma_commit(&s.s_full[1]);
          }
          ++kv_iter;
          ++tile_cnt;
        }
      }
    } else {
      // ---------------- softmax groups ----------------
      const int g = warp >> 2, wq = warp & 3;
      const int row = qb * 256 + g * kTile + wq * 32 + lane;
      const uint32_t tb = tmem + ((uint32_t)(wq * 32) << 16);
      const uint32_t s_col = g * 128, o_col = 256 + g * D;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int t = 0; t < n; ++t) {
        const int e = list[t];
        const int cls = (e >> (2 * g)) & 3;
        const bool need = (cls != kClsFull) || ((e >> 4) & 1);
        const int st = kv_iter % kStages;
        const uint32_t ph = (kv_iter / kStages) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[g], tile_cnt & 1, w));
        if (need && ok) ok = __all_sync(0xffffffffu, mbar_wait(&s.k_full[st], ph, w));
        if (!ok) break;
        tc_fence_after();
        uint32_t raw[128];
        tmem_ld32p(tb + s_col + 0, raw + 0);
        tmem_ld32p(tb + s_col + 32, raw + 32);
        tmem_ld32p(tb + s_col + 64, raw + 64);
        tmem_ld32p(tb + s_col + 96, raw + 96);
        tmem_ld_wait();
        float x[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] = __uint_as_float(raw[i]) * p.scale_log2;
        if (need) {
          // Bit j of word c: column 32c + j is masked for this row.  Built with
          // a rolled loop (the boundary records are smem broadcasts), then
          // applied with bit tests on the unrolled register array.
          const int4* mrec = s.mask[st];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t bits = 0;
#pragma unroll 4
            for (int j = 0; j < 32; ++j) {
              const int4 r = mrec[c * 32 + j];
              const bool masked = (r.x <= row && row < r.y) || (r.z <= row && row < r.w);
              bits |= (masked ? 1u : 0u) << j;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) x[c * 32 + j] = ((bits >> j) & 1u) ? -INFINITY : x[c * 32 + j];
          }
        }
        float mx8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) mx8[j] = x[j];
#pragma unroll
        for (int i = 8; i < 128; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], x[i]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        // Lazy rescale: only when the maximum grows by more than 8 (log2 units).
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m_run + 8.f) {
          alpha = fast_exp2(m_run - mx);  // 0 when m_run = -inf
          rescale = (m_run != -INFINITY);
          m_run = mx;
          l_run *= alpha;
        }
        const float mref = (m_run == -INFINITY) ? 0.f : m_run;
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 32 columns -> 16 packed bf16 pairs per store
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = fast_exp2(x[c * 32 + 2 * i] - mref);
            const float a1 = fast_exp2(x[c * 32 + 2 * i + 1] - mref);
            sum4[i & 3] += a0 + a1;
            pk[i] = pack_bf16x2(a0, a1);
          }
          tmem_st16(tb + s_col + c * 16, pk);
        }
        l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        // O correction (the previous P V of this q-tile has completed: the
        // commit that signalled this S was issued after it).
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32p(tb + o_col + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32p(tb + o_col + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.p_full[g]);
        ++kv_iter;
        ++tile_cnt;
      }
      // ---------------- epilogue ----------------
      if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.o_full[g], act_cnt & 1, w));
      if (ok) {
        tc_fence_after();
        const bool valid = row < sh.Nq;
        const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
        __nv_bfloat16* orow = p.o + (((size_t)b * sh.Nq + (valid ? row : 0)) * sh.Hq + h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (n > 0) {
            tmem_ld32p(tb + o_col + c * 32, o);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          uint32_t pkd[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pkd[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2], pkd[4 * i + 3]);
          }
        }
        if (valid)
          p.lse[((size_t)b * sh.Hq + h) * sh.Nq + row] =
              (l_run > 0.f) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      }
    }
    if (n > 0) ++act_cnt;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // ---------------- teardown ----------------
  if (s.abort_flag) {
    // Let copies and MMAs that are still in flight land before the CTA's
    // shared memory and tensor memory are released.
    const WaitCtx w2{&s.no_abort, p.status, p.wait_limit_ns};
    if (warp == Cfg::kMmaWarp && lane == 0) {
      mma_commit(&s.teardown);
      (void)mbar_wait(&s.teardown, 0, w2);
    }
    if (warp == Cfg::kProducerWarp && lane == 0) {
      if (q_armed) (void)mbar_wait(&s.q_full, q_par, w2);
      for (int st = 0; st < kStages; ++st)
        if (k_armed & (1u << st)) {
          (void)mbar_wait(&s.k_full[st], k_par[st], w2);
          (void)mbar_wait(&s.v_full[st], v_par[st], w2);
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_fwd_d(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, int grid, cudaStream_t st) {
  const int smem = (int)sizeof(FwdSmem<D>);
  cudaError_t e = ensure_smem_limit((const void*)fm_fwd_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  profile_begin(0, st);
  note_launch();
  fm_fwd_kernel<D><<<grid, FwdCfg<D>::kThreads, smem, st>>>(tq, tk, tv, p);
  profile_end(0, st);
  return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       int grid, cudaStream_t st) {
  if (p.s.d == 128) return launch_fwd_d<128>(p, tq, tk, tv, grid, st);
  return launch_fwd_d<64>(p, tq, tk, tv, grid, st);
}

}  // namespace fm
