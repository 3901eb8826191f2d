// Backward preprocess for sm_100a: per query row, D = rowsum(dO o O) (the
// shortcut for sum_j P_ij dP_ij of the softmax backward) and LSE converted to
// log2 units, written over a row range padded to whole 128-row tiles (padded
// rows: D = 0, LSE2 = +inf so that every P of such a row is 0).  A row with no
// visible key (LSE = -inf) also gets LSE2 = +inf.
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: the mask-aware kernels cover forward and backward.
#include <cuda_runtime.h>
#include <cmath>

#include "common.cuh"
#include "launchers.h"

namespace fm {

// ----------------------------------------------------------------------------
// preprocess: D = rowsum(dO * O) and LSE in log2 units, per padded row.
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
    } else {
      const uint32_t ov = *reinterpret_cast<const uint32_t*>(p.o + base + lane * 2);
      const uint32_t gv = *reinterpret_cast<const uint32_t*>(p.dout + base + lane * 2);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv));
      acc = a.x * c.x + a.y * c.y;
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

}  // namespace fm
