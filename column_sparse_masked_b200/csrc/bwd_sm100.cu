// Mask-aware attention backward for sm_100a.
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: the mask-aware kernel covers forward and backward.  For the loss
// sum(O * dO) with P = softmax(scale * Q K^T + mask):
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),  D_i = rowsum(dO_i o O_i),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Blackwell design, KV-stationary: a persistent CTA takes a work item
// (batch, KV head, 128-key tile), keeps K and V in shared memory and dK, dV in
// tensor memory, and walks the non-skipped q-tiles of every q-head that shares
// the KV head (so dK/dV of a GQA group accumulate on chip).  Per q-tile:
//   S^T  = K Q^T    -> TMEM [0,128)      (tcgen05, both operands K-major)
//   dP^T = V dO^T   -> TMEM [128,256)
//   P^T  = exp2(S^T * scale*log2e - LSE2)  written back as bf16 over S^T
//   dV  += P^T dO   (A = P^T from TMEM, B = dO MN-major)
//   dS^T = P^T o (dP^T - D)  written as bf16 over dP^T and into shared memory
//   dK  += dS^T Q   (A = dS^T from TMEM, B = Q MN-major)
//   dQ   = dS K     -> TMEM [0, d)  (A = dS MN-major from smem, B = K MN-major)
//   dQ is added into an fp32 accumulator in global memory (vector reductions).
// Thread t of the compute warpgroup owns key (lane) t for S^T/dP^T, and query
// row t when it reads the dQ tile.  The element mask is evaluated only on
// partial tiles; each thread holds its key's four boundaries in registers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kStages = 2;
  static constexpr int kThreads = 192;
  static constexpr int kProducerWarp = 4;
  static constexpr int kMmaWarp = 5;
};

template <int D>
struct __align__(1024) BwdSmem {
  uint8_t k[BwdCfg<D>::kTileBytes];
  uint8_t v[BwdCfg<D>::kTileBytes];
  uint8_t q[2][BwdCfg<D>::kTileBytes];
  uint8_t dout[2][BwdCfg<D>::kTileBytes];
  uint8_t ds[kTile * kTile * 2];  // dS, MN-major over q: [key][q] in two 64-wide SW128 atoms
  float lse2[2][kTile];
  float dsum[2][kTile];
  uint64_t kv_full, qd_full[2], qd_empty[2], sp_full, p_full, ds_full, dq_full, s_free, dkdv_full, dv_done,
      teardown;
  uint32_t tmem_base;
  int abort_flag;
  int no_abort;
  int item;
};

// D[tmem] = A B^T with both operands K-major SW128 over the head dimension.
template <int D>
__device__ __forceinline__ void issue_ss_kmajor(uint32_t d_tmem, const uint8_t* as, const uint8_t* bs) {
  constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
  const uint32_t aa = smem_addr(as), ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, sdesc_sw128(aa + off, 16, 1024), sdesc_sw128(ba + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// D[tmem] (+)= A[tmem] B where B is a [128 rows (K) x D (N)] MN-major tile.
template <int D>
__device__ __forceinline__ void issue_ts_mn(uint32_t d_tmem, uint32_t a_tmem, const uint8_t* bs, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
  const uint32_t ba = smem_addr(bs);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(ba + kk * 2048, 16384, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// dQ[tmem] = dS K: A = dS (M = 128 q, K = 128 keys, MN-major), B = K tile (MN-major).
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, const uint8_t* ds, const uint8_t* ks) {
  constexpr uint32_t idesc = idesc_bf16(128, D, true, true);
  const uint32_t da = smem_addr(ds), ka = smem_addr(ks);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ss(d_tmem, sdesc_sw128(da + kk * 2048, 16384, 1024), sdesc_sw128(ka + kk * 2048, 16384, 1024), idesc,
           kk > 0 ? 1u : 0u);
}

__device__ __forceinline__ void tmem_ld32q(uint32_t taddr, uint32_t* r) {
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

__device__ __forceinline__ void tmem_st16q(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    fm_bwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                  const BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  BwdSmem<D>& s = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Shape& sh = p.s;

  if (smem_addr(smem_raw) & 1023u) {
    if (tid == 0) atomicCAS(p.status, 0, -5);
    return;
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.qd_full[i], 1);
      mbar_init(&s.qd_empty[i], 1);
    }
    mbar_init(&s.sp_full, 1);
    mbar_init(&s.p_full, 128);
    mbar_init(&s.ds_full, 128);
    mbar_init(&s.dq_full, 1);
    mbar_init(&s.s_free, 128);
    mbar_init(&s.dkdv_full, 1);
    mbar_init(&s.dv_done, 1);
    mbar_init(&s.teardown, 1);
    s.abort_flag = 0;
    s.no_abort = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::kProducerWarp && lane == 0) {
    tma_prefetch_map(&tq);
    tma_prefetch_map(&tk);
    tma_prefetch_map(&tv);
    tma_prefetch_map(&tdo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const WaitCtx w{&s.abort_flag, p.status, p.wait_limit_ns};

  uint32_t qd_iter = 0, tile_cnt = 0, act_cnt = 0;
  uint32_t kv_par = 0, kv_armed = 0, qd_par[2] = {0, 0}, qd_armed = 0;

  for (;;) {
    if (tid == 0) s.item = s.abort_flag ? INT_MAX : atomicAdd(p.counter, 1);
    __syncthreads();
    const int item = s.item;
    if (item >= p.n_items) break;
    const int unit = p.order[item / sh.Eb];
    const int esub = item % sh.Eb;
    const int kt = unit % sh.nKt;
    const int mu = (unit / sh.nKt) % sh.Mu;
    const int b = unit / (sh.nKt * sh.Mu);
    const int hkv = mu * sh.Eb + esub;
    int total = 0;
    for (int gi = 0; gi < sh.G; ++gi) {
      const int h = hkv * sh.G + gi;
      const int hm = (sh.Hm == 1) ? 0 : h;
      total += p.bcount[((size_t)b * sh.Hm + hm) * sh.nKt + kt];
    }

    if (warp == Cfg::kProducerWarp) {
      if (lane == 0 && total > 0) {
        mbar_arrive_expect_tx(&s.kv_full, 2 * Cfg::kTileBytes);
        kv_par = act_cnt & 1;
        kv_armed = 1;
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_4d(s.k + bx * 16384, &tk, &s.kv_full, bx * 64, hkv, kt * kTile, b);
          tma_load_4d(s.v + bx * 16384, &tv, &s.kv_full, bx * 64, hkv, kt * kTile, b);
        }
        bool ok = true;
        for (int gi = 0; ok && gi < sh.G; ++gi) {
          const int h = hkv * sh.G + gi;
          const int hm = (sh.Hm == 1) ? 0 : h;
          const size_t lrow = ((size_t)b * sh.Hm + hm) * sh.nKt + kt;
          const int* list = p.blist + lrow * sh.nQt;
          const int cnt = p.bcount[lrow];
          for (int t = 0; t < cnt; ++t, ++qd_iter) {
            const int qt = list[t] >> 2;
            const int st = qd_iter & 1;
            const uint32_t ph = (qd_iter >> 1) & 1;
            if (!(ok = mbar_wait(&s.qd_empty[st], ph ^ 1, w))) break;
            mbar_arrive_expect_tx(&s.qd_full[st], 2 * Cfg::kTileBytes + 2 * kTile * 4);
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
              tma_load_4d(s.q[st] + bx * 16384, &tq, &s.qd_full[st], bx * 64, h, qt * kTile, b);
              tma_load_4d(s.dout[st] + bx * 16384, &tdo, &s.qd_full[st], bx * 64, h, qt * kTile, b);
            }
            const size_t roff = ((size_t)b * sh.Hq + h) * sh.nQt * kTile + (size_t)qt * kTile;
            bulk_load(s.lse2[st], p.lse2 + roff, kTile * 4, &s.qd_full[st]);
            bulk_load(s.dsum[st], p.dsum + roff, kTile * 4, &s.qd_full[st]);
            qd_par[st] = ph;
            qd_armed |= 1u << st;
          }
        }
      }
    } else if (warp == Cfg::kMmaWarp) {
      if (lane == 0 && total > 0) {
        bool ok = mbar_wait(&s.kv_full, act_cnt & 1, w);
        tc_fence_after();
        bool first = true;
        for (int gi = 0; ok && gi < sh.G; ++gi) {
          const int h = hkv * sh.G + gi;
          const int hm = (sh.Hm == 1) ? 0 : h;
          const int cnt = p.bcount[((size_t)b * sh.Hm + hm) * sh.nKt + kt];
          for (int t = 0; t < cnt; ++t) {
            const int st = qd_iter & 1;
            const uint32_t ph = (qd_iter >> 1) & 1;
            if (!(ok = mbar_wait(&s.qd_full[st], ph, w) && mbar_wait(&s.s_free, (tile_cnt & 1) ^ 1, w))) break;
            tc_fence_after();
            issue_ss_kmajor<D>(tmem + 0, s.k, s.q[st]);        // S^T
            issue_ss_kmajor<D>(tmem + 128, s.v, s.dout[st]);   // dP^T
            mma_commit(&s.sp_full);
            if (!(ok = mbar_wait(&s.p_full, tile_cnt & 1, w))) break;
            tc_fence_after();
            issue_ts_mn<D>(tmem + 256, tmem + 0, s.dout[st], !first);  // dV += P^T dO
            mma_commit(&s.dv_done);
            if (!(ok = mbar_wait(&s.ds_full, tile_cnt & 1, w))) break;
            tc_fence_after();
            issue_ts_mn<D>(tmem + 256 + D, tmem + 128, s.q[st], !first);  // dK += dS^T Q
            if (!(ok = mbar_wait(&s.dv_done, tile_cnt & 1, w))) break;  // P^T no longer read
            issue_dq<D>(tmem + 0, s.ds, s.k);                            // dQ = dS K
            mma_commit(&s.dq_full);
            mma_commit(&s.qd_empty[st]);
            first = false;
            ++tile_cnt;
            ++qd_iter;
          }
        }
        if (ok) mma_commit(&s.dkdv_full);
      }
    } else {
      // ---------------- compute warpgroup ----------------
      const int jl = warp * 32 + lane;  // key lane; also the q row when reading dQ
      const int key = kt * kTile + jl;
      const uint32_t tb = tmem + ((uint32_t)(warp * 32) << 16);
      bool ok = true;
      for (int gi = 0; ok && gi < sh.G; ++gi) {
        const int h = hkv * sh.G + gi;
        const int hm = (sh.Hm == 1) ? 0 : h;
        const size_t lrow = ((size_t)b * sh.Hm + hm) * sh.nKt + kt;
        const int* list = p.blist + lrow * sh.nQt;
        const int cnt = p.bcount[lrow];
        const int4 rec = p.rec[lrow * kTile + jl];
        for (int t = 0; t < cnt; ++t) {
          const int e = list[t];
          const int qt = e >> 2;
          const bool need = (e & 3) == kClsPartial;
          const int st = qd_iter & 1;
          const uint32_t ph = (qd_iter >> 1) & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&s.sp_full, tile_cnt & 1, w));
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s.qd_full[st], ph, w));
          if (!ok) break;
          tc_fence_after();
          const float* l2 = s.lse2[st];
          const float* dsm = s.dsum[st];
          const int row0 = qt * kTile;
          float pr[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32q(tb + c * 32, r);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int qi = c * 32 + i;
              float pv = fast_exp2(__uint_as_float(r[i]) * p.scale_log2 - l2[qi]);
              if (need) {
                const int row = row0 + qi;
                const bool masked = (rec.x <= row && row < rec.y) || (rec.z <= row && row < rec.w);
                pv = masked ? 0.f : pv;
              }
              pr[qi] = pv;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pr[c * 32 + 2 * i], pr[c * 32 + 2 * i + 1]);
            tmem_st16q(tb + c * 16, pk);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&s.p_full);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32q(tb + 128 + c * 32, r);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int q0 = c * 32 + 2 * i;
              const float d0 = pr[q0] * (__uint_as_float(r[2 * i]) - dsm[q0]);
              const float d1 = pr[q0 + 1] * (__uint_as_float(r[2 * i + 1]) - dsm[q0 + 1]);
              pk[i] = pack_bf16x2(d0, d1);
            }
            tmem_st16q(tb + 128 + c * 16, pk);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const int col8 = c * 4 + ch;  // group of 8 q values
              const uint32_t off = (col8 >> 3) * 16384 + jl * 128 + (((col8 & 7) ^ (jl & 7)) << 4);
              *reinterpret_cast<uint4*>(s.ds + off) =
                  make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
          }
          tmem_st_wait();
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(&s.ds_full);
          ok = __all_sync(0xffffffffu, mbar_wait(&s.dq_full, tile_cnt & 1, w));
          if (!ok) break;
          tc_fence_after();
          const int qrow = row0 + jl;
          const bool qvalid = qrow < sh.Nq;
          float* dst = p.dqacc + (((size_t)b * sh.Nq + (qvalid ? qrow : 0)) * sh.Hq + h) * D;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32q(tb + c * 32, r);
            tmem_ld_wait();
            if (qvalid) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                red_add_v4(dst + c * 32 + 4 * i, __uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                           __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
            }
          }
          tc_fence_before();
          mbar_arrive(&s.s_free);
          ++tile_cnt;
          ++qd_iter;
        }
      }
      // ---------------- epilogue: dK, dV of this key tile ----------------
      if (ok && total > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.dkdv_full, act_cnt & 1, w));
      if (ok) {
        tc_fence_after();
        const bool valid = key < sh.Nk;
        const size_t off = (((size_t)b * sh.Nk + (valid ? key : 0)) * sh.Hkv + hkv) * D;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + off;
          const float mul = (which == 0) ? 1.f : p.scale;
          const uint32_t col = 256 + which * D;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            if (total > 0) {
              tmem_ld32q(tb + col + c * 32, r);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = 0u;
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
            if (valid) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      }
    }
    if (total > 0) ++act_cnt;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // ---------------- teardown ----------------
  if (s.abort_flag) {
    const WaitCtx w2{&s.no_abort, p.status, p.wait_limit_ns};
    if (warp == Cfg::kMmaWarp && lane == 0) {
      mma_commit(&s.teardown);
      (void)mbar_wait(&s.teardown, 0, w2);
    }
    if (warp == Cfg::kProducerWarp && lane == 0) {
      if (kv_armed) (void)mbar_wait(&s.kv_full, kv_par, w2);
      for (int st = 0; st < 2; ++st)
        if (qd_armed & (1u << st)) (void)mbar_wait(&s.qd_full[st], qd_par[st], w2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------------
// preprocess: D = rowsum(dO * O), LSE in log2 units, zeroed dQ accumulator.
// One warp per (b, row, h) of the padded row range; h fastest (coalesced).
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fm_bwd_pre_kernel(BwdPreParams p) {
  const Shape& s = p.s;
  const int npad = s.nQt * kTile;
  const int64_t rows = (int64_t)s.B * npad * s.Hq;
  const int lane = threadIdx.x & 31;
  for (int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; r < rows;
       r += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int h = (int)(r % s.Hq);
    const int i = (int)((r / s.Hq) % npad);
    const int b = (int)(r / ((int64_t)s.Hq * npad));
    const size_t ridx = ((size_t)b * s.Hq + h) * npad + i;
    if (i >= s.Nq) {
      if (lane == 0) {
        p.dsum[ridx] = 0.f;
        p.lse2[ridx] = INFINITY;
      }
      continue;
    }
    const size_t base = (((size_t)b * s.Nq + i) * s.Hq + h) * D;
    constexpr int kPer = D / 32;  // elements per lane (2 or 4)
    float acc = 0.f;
    if (kPer == 4) {
      const uint2 ov = *reinterpret_cast<const uint2*>(p.o + base + lane * 4);
      const uint2 gv = *reinterpret_cast<const uint2*>(p.dout + base + lane * 4);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 a = __bfloat1622float2(o2[j]), c = __bfloat1622float2(g2[j]);
        acc += a.x * c.x + a.y * c.y;
      }
      *reinterpret_cast<float4*>(p.dqacc + base + lane * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const uint32_t ov = *reinterpret_cast<const uint32_t*>(p.o + base + lane * 2);
      const uint32_t gv = *reinterpret_cast<const uint32_t*>(p.dout + base + lane * 2);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv));
      acc = a.x * c.x + a.y * c.y;
      *reinterpret_cast<float2*>(p.dqacc + base + lane * 2) = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const float l = p.lse[((size_t)b * s.Hq + h) * s.Nq + i];
      p.dsum[ridx] = acc;
      p.lse2[ridx] = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
    }
  }
}

__global__ void fm_dq_finalize_kernel(DqFinParams p) {
  const int64_t n4 = p.n / 4;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n4; t += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(p.dqacc)[t];
    uint2 o;
    o.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    o.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    reinterpret_cast<uint2*>(p.dq)[t] = o;
  }
}

// ----------------------------------------------------------------------------
template <int D>
static cudaError_t launch_bwd_d(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const CUtensorMap& tdo, int grid, cudaStream_t st) {
  const int smem = (int)sizeof(BwdSmem<D>);
  cudaError_t e = ensure_smem_limit((const void*)fm_bwd_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  profile_begin(1, st);
  note_launch();
  fm_bwd_kernel<D><<<grid, BwdCfg<D>::kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  profile_end(1, st);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, int grid, cudaStream_t st) {
  if (p.s.d == 128) return launch_bwd_d<128>(p, tq, tk, tv, tdo, grid, st);
  return launch_bwd_d<64>(p, tq, tk, tv, tdo, grid, st);
}

cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t st) {
  const int64_t rows = (int64_t)p.s.B * p.s.nQt * kTile * p.s.Hq;
  if (rows == 0) return cudaSuccess;
  int64_t blocks = (rows * 32 + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (p.s.d == 128)
    { note_launch(); fm_bwd_pre_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(p);
    }
  else
    { note_launch(); fm_bwd_pre_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(p);
    }
  return cudaGetLastError();
}

cudaError_t launch_dq_finalize(const DqFinParams& p, cudaStream_t st) {
  if (p.n == 0) return cudaSuccess;
  int64_t blocks = (p.n / 4 + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  { note_launch(); fm_dq_finalize_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fm
