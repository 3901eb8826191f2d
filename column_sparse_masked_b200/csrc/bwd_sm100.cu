// Backward preprocess for sm_100a: per query row, D = rowsum(dO o O) (the
// shortcut for sum_j P_ij dP_ij of the softmax backward) and LSE converted to
// log2 units, written over a row range padded to whole 128-row tiles (padded
// rows: D = 0, LSE2 = +inf so that every P of such a row is 0).  A row with no
// visible key (LSE = -inf) also gets LSE2 = +inf.
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: the mask-aware kernels cover forward and backward.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>

#include "common.cuh"
#include "launchers.h"

namespace fm {

// ----------------------------------------------------------------------------
// preprocess: D = rowsum(dO * O) and LSE in log2 units, per padded row (and,
// for the fused backward, zeroing of its fp32 dQ accumulator).
// Half a warp per (b, row, h) of the padded row range, h fastest (coalesced):
// each lane loads 16 bytes of O and of dO, a warp covers two rows per step.
// The kernel is bound by reading O and dO once from HBM.
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fm_bwd_pre_kernel(BwdPreParams p) {
  const Shape& s = p.s;
  const int npad = s.nQt * kTile;
  const int64_t rows = (int64_t)s.B * npad * s.Hq;
  constexpr int kLanes = D / 8;  // lanes per row (16 bytes = 8 elements each): 16 or 8
  constexpr int kRowsPerWarp = 32 / kLanes;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanes, sl = lane % kLanes;
  const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  if (p.dqacc) {  // fused backward: zero the fp32 dQ accumulator (16-byte stores, grid-stride)
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < p.dqacc_vec4;
         t += (int64_t)gridDim.x * blockDim.x)
      p.dqacc[t] = z;
  }
  for (int64_t r0 = warp0 * kRowsPerWarp; r0 < rows; r0 += nwarps * kRowsPerWarp) {
    const int64_t r = r0 + sub;
    const bool in = r < rows;
    const int h = (int)(r % s.Hq);
    const int i = (int)((r / s.Hq) % npad);
    const int b = (int)(r / ((int64_t)s.Hq * npad));
    const bool real = in && i < s.Nq;
    float acc = 0.f;
    if (real) {
      const size_t base = (((size_t)b * s.Nq + i) * s.Hq + h) * D + sl * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(p.o + base);
      const uint4 gv = *reinterpret_cast<const uint4*>(p.dout + base);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 a = __bfloat1622float2(o2[j]), c = __bfloat1622float2(g2[j]);
        acc = fmaf(a.x, c.x, fmaf(a.y, c.y, acc));
      }
    }
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in && sl == 0) {
      const size_t ridx = ((size_t)b * s.Hq + h) * npad + i;
      if (real) {
        const float l = p.lse[((size_t)b * s.Hq + h) * s.Nq + i];
        p.dsum[ridx] = acc;
        p.lse2[ridx] = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
      } else {
        p.dsum[ridx] = 0.f;
        p.lse2[ridx] = INFINITY;
      }
    }
  }
}

cudaError_t launch_bwd_pre(const BwdPreParams& p, int max_blocks, cudaStream_t st) {
  const int64_t rows = (int64_t)p.s.B * p.s.nQt * kTile * p.s.Hq;
  if (rows == 0) return cudaSuccess;
  const int rows_per_block = (p.s.d == 128 ? 2 : 4) * 8;
  int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (blocks > max_blocks) blocks = max_blocks;  // grid-stride loop over the rows
  note_launch();
  if (p.s.d == 128)
    fm_bwd_pre_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(p);
  else
    fm_bwd_pre_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace fm
