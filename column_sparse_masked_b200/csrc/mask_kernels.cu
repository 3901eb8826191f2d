// Mask-side kernels: boundary-record preparation and the per-k-tile block
// summary, tile classification into per-block work lists, the longest-first
// order of scheduling units, clip-shift-max localisation and the closed-form
// count of unmasked pairs.
//
// Method: "FlashMask-3 targets masked distributed attention on Hopper GPUs",
// In-depth insight -- the column-wise mask (four query-axis boundary vectors
// per key column), tiles decided from O(n) data, and the exchange-free
// clip-shift-max localisation of a query chunk.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <climits>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

// ----------------------------------------------------------------------------
// 1. padded boundary records + block summary, one CTA per (k-tile, hm, b)
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(128) mask_prep_kernel(MaskPrepParams p) {
  griddep_wait();
  griddep_launch_dependents();
  const int kt = blockIdx.x, hm = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;
  const int j = kt * kTile + t;
  const size_t row = (size_t)b * p.Hm + hm;
  const bool real = j < p.Nk;
  int4 r = make_int4(0, INT_MAX, 0, 0);  // padded column: hidden from every row
  if (real) {
    const size_t idx = row * p.Nk + j;
    r.x = p.lts ? p.lts[idx] : 0;
    r.y = p.lte ? p.lte[idx] : 0;
    r.z = p.uts ? p.uts[idx] : 0;
    r.w = p.ute ? p.ute[idx] : 0;
  }
  p.rec[(row * p.nKt + kt) * kTile + t] = r;
  if (kChecks && real && p.status) {
    const bool bad = (p.lts && (r.x < 0 || r.x > p.Nq)) || (p.lte && (r.y < 0 || r.y > p.Nq)) ||
                     (p.uts && (r.z < 0 || r.z > p.Nq)) || (p.ute && (r.w < 0 || r.w > p.Nq));
    if (bad) atomicCAS(p.status, 0, kDevErrBounds);
  }
  // min/max over the real columns of the tile
  int v[8];
  v[kMnLts] = real ? r.x : INT_MAX; v[kMxLts] = real ? r.x : INT_MIN;
  v[kMnLte] = real ? r.y : INT_MAX; v[kMxLte] = real ? r.y : INT_MIN;
  v[kMnUts] = real ? r.z : INT_MAX; v[kMxUts] = real ? r.z : INT_MIN;
  v[kMnUte] = real ? r.w : INT_MAX; v[kMxUte] = real ? r.w : INT_MIN;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      v[e] = min(v[e], __shfl_xor_sync(0xffffffffu, v[e], off));
      v[e + 1] = max(v[e + 1], __shfl_xor_sync(0xffffffffu, v[e + 1], off));
    }
  }
  __shared__ int part[4][8];
  if ((t & 31) == 0)
#pragma unroll
    for (int e = 0; e < 8; ++e) part[t >> 5][e] = v[e];
  __syncthreads();
  if (t < 8) {
    int a = part[0][t];
    for (int w = 1; w < 4; ++w) a = (t & 1) ? max(a, part[w][t]) : min(a, part[w][t]);
    p.ksum[(row * p.nKt + kt) * 8 + t] = a;
  }
}

// Block-wide exclusive prefix of a 0/1 flag over 128 threads; returns the
// position of this thread among the set flags and writes the total.
__device__ __forceinline__ int block_compact128(bool flag, int* warp_tot, int* total) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int pos = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[w] = __popc(bal);
  __syncthreads();
  int base = 0;
  for (int i = 0; i < w; ++i) base += warp_tot[i];
  if (t == 0) *total = warp_tot[0] + warp_tot[1] + warp_tot[2] + warp_tot[3];
  __syncthreads();
  return base + pos;
}

// ----------------------------------------------------------------------------
// 2a. forward work lists: per (b, hm, block of two q-tiles) the k-tiles that
//     are not skipped for at least one of the two q-tiles, in increasing order;
//     with paired q-heads a block is one q-tile, whose class both halves share
// ----------------------------------------------------------------------------
__device__ void plan_fwd_body(const PlanParams& p, int qb) {
  const Shape& s = p.s;
  const int hm = blockIdx.y, b = blockIdx.z;
  const size_t row = (size_t)b * s.Hm + hm;
  const int qt0 = s.fpair ? qb : 2 * qb, qt1 = s.fpair ? qb : 2 * qb + 1;
  const int r00 = qt0 * kTile, r01 = min(r00 + kTile, s.Nq);
  const int r10 = qt1 * kTile, r11 = min(r10 + kTile, s.Nq);
  const bool ragged_k = (s.Nk % kTile) != 0;
  int* list = p.flist + (row * s.nFB + qb) * s.nKt;
  __shared__ int warp_tot[4];
  __shared__ int total;
  __shared__ int qc[2];
  if (threadIdx.x < 2) qc[threadIdx.x] = 0;
  __syncthreads();  // the per-q-tile counts are zeroed before any warp adds to them
  int count = 0;
  for (int base = 0; base < s.nKt; base += kTile) {
    const int kt = base + threadIdx.x;
    int c0 = kClsSkip, c1 = kClsSkip;
    if (kt < s.nKt) {
      int sm[8];
      const int* src = p.ksum + (row * s.nKt + kt) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) sm[e] = src[e];
      c0 = classify_tile(sm, r00, r01);
      if (s.fpair) c1 = c0;
      else if (qt1 < s.nQt) c1 = classify_tile(sm, r10, r11);
    }
    const bool keep = (c0 != kClsSkip) || (c1 != kClsSkip);
    const unsigned b0 = __ballot_sync(0xffffffffu, c0 != kClsSkip);
    const unsigned b1 = __ballot_sync(0xffffffffu, c1 != kClsSkip);
    if ((threadIdx.x & 31) == 0) {
      atomicAdd(&qc[0], __popc(b0));
      atomicAdd(&qc[1], __popc(b1));
    }
    const int pos = block_compact128(keep, warp_tot, &total);
    if (keep) list[count + pos] = fwd_entry(kt, c0, c1, (ragged_k && kt == s.nKt - 1) ? 1 : 0);
    count += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.fcount[row * s.nFB + qb] = count;
  if (threadIdx.x < 2) p.qcount[(row * s.nFB + qb) * 2 + threadIdx.x] = qc[threadIdx.x];
}

// ----------------------------------------------------------------------------
// 2b. backward work lists: per (b, hm, k-tile) the q-tiles that are not skipped
// ----------------------------------------------------------------------------
__device__ void plan_bwd_body(const PlanParams& p, int kt) {
  const Shape& s = p.s;
  const int hm = blockIdx.y, b = blockIdx.z;
  const size_t row = (size_t)b * s.Hm + hm;
  int sm[8];
  const int* src = p.ksum + (row * s.nKt + kt) * 8;
#pragma unroll
  for (int e = 0; e < 8; ++e) sm[e] = src[e];
  int* list = p.blist + (row * s.nKt + kt) * s.nQt;
  __shared__ int warp_tot[4];
  __shared__ int total;
  int count = 0;
  for (int base = 0; base < s.nQt; base += kTile) {
    const int qt = base + threadIdx.x;
    int c = kClsSkip;
    if (qt < s.nQt) c = classify_tile(sm, qt * kTile, min(qt * kTile + kTile, s.Nq));
    const bool keep = c != kClsSkip;
    const int pos = block_compact128(keep, warp_tot, &total);
    if (keep) list[count + pos] = bwd_entry(qt, c);
    count += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.bcount[row * s.nKt + kt] = count;
}

__global__ void __launch_bounds__(128) plan_fwd_kernel(PlanParams p) {
  griddep_wait();
  griddep_launch_dependents();
  plan_fwd_body(p, blockIdx.x);
}

__global__ void __launch_bounds__(128) plan_bwd_kernel(PlanParams p) {
  griddep_wait();
  griddep_launch_dependents();
  plan_bwd_body(p, blockIdx.x);
}

// Both list sets of the backward in one launch: blocks [0, nKt) build the
// key-side lists, blocks [nKt, nKt + nQB) the query-side (forward) lists.
__global__ void __launch_bounds__(128) plan_both_kernel(PlanParams p) {
  griddep_wait();
  griddep_launch_dependents();
  const int x = blockIdx.x;
  if (x < p.s.nKt)
    plan_bwd_body(p, x);
  else
    plan_fwd_body(p, x - p.s.nKt);
}

// ----------------------------------------------------------------------------
// 2c. class export [B, Hm, nQt, nKt]
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(128) classify_export_kernel(PlanParams p) {
  const Shape& s = p.s;
  const int qt = blockIdx.x, hm = blockIdx.y, b = blockIdx.z;
  const size_t row = (size_t)b * s.Hm + hm;
  const int r0 = qt * kTile, r1 = min(r0 + kTile, s.Nq);
  for (int kt = threadIdx.x; kt < s.nKt; kt += blockDim.x) {
    int sm[8];
    const int* src = p.ksum + (row * s.nKt + kt) * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) sm[e] = src[e];
    p.cls[(row * s.nQt + qt) * s.nKt + kt] = (uint8_t)classify_tile(sm, r0, r1);
  }
}

// ----------------------------------------------------------------------------
// 3. work order of the persistent kernels (one CTA per order, in smem).
//    Items are indexed group-major ((batch, KV head) groups), so the natural
//    order keeps one group's data together in L2.  With wave > 0 the items of
//    `wave` consecutive groups are taken longest-first: ascending wave index,
//    descending cost.  With a single wave the order is a counting sort over
//    cost buckets (histogram, scan, scatter); the order of equal-cost items is
//    left to the atomics, which changes which CTA takes an item, never what
//    any output element is computed from.  With several waves a bitonic sort
//    of  key = wave index << 48 | (cost_cap - cost) << 32 | item  keeps the
//    index order of equal-cost items.  Also zeroes the work counter of the
//    kernel that follows.
// ----------------------------------------------------------------------------
constexpr int kSortMax = 16384;

__device__ __forceinline__ unsigned item_cost(const SortParams& p, int i) {
  const Shape& s = p.s;
  if (p.mode == 0) {
    const ItemCoord c = decode_fwd_item(s, i);
    const int h = c.hkv * s.G + (s.fpair ? 2 * c.hg : c.hg), hm = (s.Hm == 1) ? 0 : h;
    return (unsigned)p.count[((size_t)c.b * s.Hm + hm) * s.nFB + c.t];
  }
  if (p.mode == 1) {
    const ItemCoord c = decode_kv_item_coord(s, i);
    unsigned cost = 0;
    for (int g = 0; g < s.G; ++g) {
      const int h = c.hkv * s.G + g, hm = (s.Hm == 1) ? 0 : h;
      cost += (unsigned)p.count[((size_t)c.b * s.Hm + hm) * s.nKt + c.t];
    }
    return cost;
  }
  const ItemCoord c = decode_q_item_coord(s, i);
  const int h = c.hkv * s.G + c.hg, hm = (s.Hm == 1) ? 0 : h;
  return (unsigned)p.count[((size_t)c.b * s.Hm + hm) * (s.nQB * 2) + c.t];
}

// Exclusive scan of one int per thread over the block (blockDim.x <= 1024).
__device__ int block_exclusive_scan(int v, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) wsum[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? wsum[warp - 1] : 0);
  __syncthreads();
  return excl;
}

__device__ void counting_sort_body(const SortParams& p, int* sm) {
  const int n = p.n_items, nb = p.n_buckets, C = p.cost_cap;
  const int t = threadIdx.x, nt = blockDim.x;
  int* bkt = sm;          // [n] bucket of each item
  int* pos = sm + n;      // [n] rank within its bucket
  int* hist = sm + 2 * n; // [nb] counts, then start offsets
  __shared__ int wsum[32];
  for (int b = t; b < nb; b += nt) hist[b] = 0;
  __syncthreads();
  for (int u = t; u < n; u += nt) {
    const int cost = min((int)item_cost(p, u), C);
    const int wv = (u / p.items_per_group) / p.wave;
    const int b = wv * (C + 1) + (C - cost);  // ascending wave, descending cost
    bkt[u] = b;
    pos[u] = atomicAdd(&hist[b], 1);
  }
  __syncthreads();
  const int chunk = (nb + nt - 1) / nt, b0 = t * chunk, b1 = min(b0 + chunk, nb);
  int sum = 0;
  for (int b = b0; b < b1; ++b) sum += hist[b];
  int run = block_exclusive_scan(sum, wsum);
  for (int b = b0; b < b1; ++b) {
    const int c = hist[b];
    hist[b] = run;
    run += c;
  }
  __syncthreads();
  for (int u = t; u < n; u += nt) p.order[hist[bkt[u]] + pos[u]] = u;
}

__device__ void sort_units_body(const SortParams& p, unsigned long long* keys) {
  const int n = p.n_items;
  const int t = threadIdx.x;
  if (t == 0) p.counter[0] = 0;
  if (p.wave <= 0 || n > kSortMax) {  // natural group-major order
    for (int u = t; u < n; u += blockDim.x) p.order[u] = u;
    return;
  }
  if (p.n_buckets > 0) {
    counting_sort_body(p, reinterpret_cast<int*>(keys));
    return;
  }
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  for (int u = t; u < np2; u += blockDim.x) {
    unsigned long long key = ~0ull;
    if (u < n) {
      const unsigned cost = min(item_cost(p, u), (unsigned)p.cost_cap);
      const unsigned long long wv = (unsigned long long)((u / p.items_per_group) / p.wave);
      key = (wv << 48) | ((unsigned long long)((unsigned)p.cost_cap - cost) << 32) | (unsigned)u;
    }
    keys[u] = key;
  }
  __syncthreads();
  for (int k = 2; k <= np2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = t; i < np2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & k) == 0;
          const unsigned long long a = keys[i], c = keys[ixj];
          if ((a > c) == up) {
            keys[i] = c;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int u = t; u < n; u += blockDim.x) p.order[u] = (int)(keys[u] & 0xffffffffu);
}

// One block per order: block b sorts the units of p[b] (two independent sorts
// share a launch).
struct SortPair {
  SortParams p[2];
};
__global__ void __launch_bounds__(1024) sort_units_kernel(SortPair sp) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ unsigned long long keys[];
  sort_units_body(sp.p[blockIdx.x], keys);
}

// ----------------------------------------------------------------------------
// 4. clip-shift-max localisation
// ----------------------------------------------------------------------------
__global__ void localize_kernel(const int32_t* in, int32_t* out, int64_t n, int32_t a, int32_t b) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    const int32_t x = min(in[t], b) - a;  // clip to the chunk end, shift to local rows
    out[t] = max(x, 0);                   // max with zero
  }
}

struct Chunks {
  int32_t a[64], b[64];
  int n;
};

__global__ void localize_multi_kernel(const int32_t* in, int32_t* out, int64_t n, Chunks c) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t x = in[t];
    int64_t acc = 0;
    for (int k = 0; k < c.n; ++k) acc += min(max(x, (int64_t)c.a[k]), (int64_t)c.b[k]) - c.a[k];
    out[t] = (int32_t)acc;
  }
}

// ----------------------------------------------------------------------------
// 5. unmasked pairs, closed form per key column (one CTA, deterministic)
//    masked_j = |L n [0,Nq)| + |U n [0,Nq)| - |L n U n [0,Nq)|
// ----------------------------------------------------------------------------
__device__ __forceinline__ int64_t overlap_len(int64_t a, int64_t b, int64_t lo, int64_t hi) {
  const int64_t x = max(a, lo), y = min(b, hi);
  return y > x ? y - x : 0;
}

__global__ void __launch_bounds__(1024) count_unmasked_kernel(MaskPrepParams p, int Hq, int Nq, int64_t* out) {
  const int64_t total = (int64_t)p.B * p.Hm * p.Nk;
  const int64_t weight = (p.Hm == 1) ? Hq : 1;
  unsigned long long acc = 0;
  for (int64_t t = threadIdx.x; t < total; t += blockDim.x) {
    const int64_t lts = p.lts ? p.lts[t] : 0, lte = p.lte ? p.lte[t] : 0;
    const int64_t uts = p.uts ? p.uts[t] : 0, ute = p.ute ? p.ute[t] : 0;
    const int64_t mL = overlap_len(lts, lte, 0, Nq);
    const int64_t mU = overlap_len(uts, ute, 0, Nq);
    const int64_t mLU = overlap_len(max(lts, uts), min(lte, ute), 0, Nq);
    acc += (unsigned long long)((Nq - (mL + mU - mLU)) * weight);
  }
  __shared__ unsigned long long red[32];
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    *out = (int64_t)s;
  }
}

// ----------------------------------------------------------------------------
// 5b. unmasked pairs of each 128-row q-tile (the work a sparsity-aware chunk
//     split evens out), one CTA per q-tile, same closed form restricted to the
//     tile's rows [r0, r1):  unmasked_j = (r1 - r0) - |L n R| - |U n R| + |L n U n R|
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) tile_costs_kernel(MaskPrepParams p, int Hq, int Nq, int64_t* out) {
  const int qt = blockIdx.x;
  const int64_t r0 = (int64_t)qt * kTile, r1 = min(r0 + kTile, (int64_t)Nq);
  const int64_t total = (int64_t)p.B * p.Hm * p.Nk;
  const int64_t weight = (p.Hm == 1) ? Hq : 1;
  unsigned long long acc = 0;
  for (int64_t t = threadIdx.x; t < total; t += blockDim.x) {
    const int64_t lts = p.lts ? p.lts[t] : 0, lte = p.lte ? p.lte[t] : 0;
    const int64_t uts = p.uts ? p.uts[t] : 0, ute = p.ute ? p.ute[t] : 0;
    const int64_t mL = overlap_len(lts, lte, r0, r1);
    const int64_t mU = overlap_len(uts, ute, r0, r1);
    const int64_t mLU = overlap_len(max(lts, uts), min(lte, ute), r0, r1);
    acc += (unsigned long long)((r1 - r0 - (mL + mU - mLU)) * weight);
  }
  __shared__ unsigned long long red[8];
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    out[qt] = (int64_t)s;
  }
}

// ----------------------------------------------------------------------------
// 6. bounded-wait self test: waits on a barrier that nothing arrives on
// ----------------------------------------------------------------------------
__global__ void wait_timeout_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx w{&abort_flag, status, limit_ns, smem_addr(&bar), 3};
    (void)mbar_wait(&bar, 0, w);  // gives up after limit_ns, records the timeout
  }
  __syncthreads();
}

// ----------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------
cudaError_t launch_mask_prep(const MaskPrepParams& p, cudaStream_t st) {
  if (p.B == 0 || p.Hm == 0 || p.nKt == 0) return cudaSuccess;
  { note_launch(); mask_prep_kernel<<<dim3(p.nKt, p.Hm, p.B), 128, 0, st>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_plan_fwd(const PlanParams& p, cudaStream_t st) {
  if (p.s.B == 0 || p.s.nFB == 0) return cudaSuccess;
  return launch_after(plan_fwd_kernel, dim3(p.s.nFB, p.s.Hm, p.s.B), dim3(128), 0, st, p);
}

cudaError_t launch_plan_both(const PlanParams& p, cudaStream_t st) {
  if (p.s.B == 0 || p.s.nKt + p.s.nQB == 0) return cudaSuccess;
  return launch_after(plan_both_kernel, dim3(p.s.nKt + p.s.nQB, p.s.Hm, p.s.B), dim3(128), 0, st, p);
}

cudaError_t launch_plan_bwd(const PlanParams& p, cudaStream_t st) {
  if (p.s.B == 0 || p.s.nKt == 0) return cudaSuccess;
  return launch_after(plan_bwd_kernel, dim3(p.s.nKt, p.s.Hm, p.s.B), dim3(128), 0, st, p);
}

cudaError_t launch_classify_export(const PlanParams& p, cudaStream_t st) {
  if (p.s.B == 0 || p.s.nQt == 0 || p.s.nKt == 0) return cudaSuccess;
  { note_launch(); classify_export_kernel<<<dim3(p.s.nQt, p.s.Hm, p.s.B), 128, 0, st>>>(p);
  }
  return cudaGetLastError();
}

static size_t sort_smem(const SortParams& p) {
  if (p.wave <= 0 || p.n_items > kSortMax) return 0;
  if (p.n_buckets > 0) return (size_t)(2 * p.n_items + p.n_buckets) * sizeof(int);
  int np2 = 1;
  while (np2 < p.n_items) np2 <<= 1;
  return (size_t)np2 * sizeof(unsigned long long);
}

void finish_sort_params(SortParams& p) {
  // cost bound per mode: k-tiles of a q-block (forward), q-tiles of the group
  // (key side), k-tiles of a q-tile (query side)
  const Shape& s = p.s;
  const int64_t bound = (p.mode == 1) ? (int64_t)s.G * s.nQt : (int64_t)s.nKt;
  p.cost_cap = (int)(bound < 0xFFFF ? bound : 0xFFFF);
  p.n_buckets = 0;
  if (p.wave <= 0 || p.n_items <= 0 || p.n_items > kSortMax || p.items_per_group <= 0) return;
  const int64_t groups = (p.n_items + p.items_per_group - 1) / p.items_per_group;
  const int64_t waves = (groups + p.wave - 1) / p.wave;
  // With several L2 waves the index order of equal-cost items (neighbouring
  // tiles of one group, which share K/V or Q/dO) is worth keeping: the
  // bitonic sort keeps it, the counting sort does not.  With one wave (few
  // items, global longest-first) the counting sort is used.
  if (waves != 1) return;
  const int64_t nb = waves * (p.cost_cap + 1);
  if ((2 * (int64_t)p.n_items + nb) * (int64_t)sizeof(int) <= (int64_t)kSortMax * 8) p.n_buckets = (int)nb;
}

cudaError_t launch_sort_units(const SortParams* ps, int count, cudaStream_t st) {
  if (count < 1 || count > 2) return cudaErrorInvalidValue;
  SortPair sp{};
  size_t smem = 0;
  for (int i = 0; i < count; ++i) {
    sp.p[i] = ps[i];
    smem = sort_smem(ps[i]) > smem ? sort_smem(ps[i]) : smem;
  }
  cudaError_t e = ensure_smem_limit((const void*)sort_units_kernel, (int)(kSortMax * sizeof(unsigned long long)));
  if (e != cudaSuccess) return e;
  return launch_after(sort_units_kernel, dim3(count), dim3(1024), smem, st, sp);
}

cudaError_t launch_localize(const int32_t* in, int32_t* out, int64_t n, int32_t a, int32_t b, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  { note_launch(); localize_kernel<<<(unsigned)(blocks < 65535 ? blocks : 65535), 256, 0, st>>>(in, out, n, a, b);
  }
  return cudaGetLastError();
}

cudaError_t launch_localize_multi(const int32_t* in, int32_t* out, int64_t n, const int32_t* starts,
                                  const int32_t* ends, int nchunks, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  Chunks c{};
  c.n = nchunks;
  for (int k = 0; k < nchunks; ++k) {
    c.a[k] = starts[k];
    c.b[k] = ends[k];
  }
  const int64_t blocks = (n + 255) / 256;
  { note_launch(); localize_multi_kernel<<<(unsigned)(blocks < 65535 ? blocks : 65535), 256, 0, st>>>(in, out, n, c);
  }
  return cudaGetLastError();
}

cudaError_t launch_count_unmasked(const MaskPrepParams& p, int Hq, int Nq, int64_t* out, cudaStream_t st) {
  { note_launch(); count_unmasked_kernel<<<1, 1024, 0, st>>>(p, Hq, Nq, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_tile_costs(const MaskPrepParams& p, int Hq, int Nq, int64_t* out, cudaStream_t st) {
  const int nqt = (Nq + kTile - 1) / kTile;
  if (nqt == 0) return cudaSuccess;
  { note_launch(); tile_costs_kernel<<<nqt, 256, 0, st>>>(p, Hq, Nq, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t st) {
  { note_launch(); wait_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  }
  return cudaGetLastError();
}

}  // namespace fm

namespace fm {

// ----------------------------------------------------------------------------
// 7. merge of partial attention results over disjoint key sets (context
//    parallelism with overlap: each received key chunk is attended as soon as
//    it lands).  Per row: lse = log(sum_c exp(lse_c)), o = sum_c exp(lse_c - lse) o_c.
//    16 threads per (batch, row, head), each 8 columns (16-byte loads/stores).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) merge_partials_kernel(MergeParams p) {
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.69314718055994531f;
  const int lanes = p.d / 8;  // threads per row
  const int64_t rows = (int64_t)p.B * p.Nq * p.Hq;
  const int64_t t0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  for (int64_t t = t0; t < rows * lanes; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t / lanes;  // row index in [B, Nq, Hq] order
    const int sl = (int)(t % lanes);
    const int h = (int)(r % p.Hq);
    const int64_t bi = r / p.Hq;
    const int i = (int)(bi % p.Nq), b = (int)(bi / p.Nq);
    const size_t lidx = ((size_t)b * p.Hq + h) * p.Nq + i;
    float m = -INFINITY;
    for (int c = 0; c < p.n; ++c) m = fmaxf(m, p.lse[c][lidx]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float lse_out = -INFINITY;
    if (m != -INFINITY) {
      float wsum = 0.f;
      for (int c = 0; c < p.n; ++c) wsum += exp2f((p.lse[c][lidx] - m) * kLog2e);
      const float inv = 1.f / wsum;
      for (int c = 0; c < p.n; ++c) {
        const float wgt = exp2f((p.lse[c][lidx] - m) * kLog2e) * inv;
        if (wgt == 0.f) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(p.o[c] + r * p.d + sl * 8);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(v2[u]);
          acc[2 * u] = fmaf(wgt, f.x, acc[2 * u]);
          acc[2 * u + 1] = fmaf(wgt, f.y, acc[2 * u + 1]);
        }
      }
      lse_out = m + log2f(wsum) * kLn2;
    }
    uint4 out;
    out.x = pack_bf16x2(acc[0], acc[1]);
    out.y = pack_bf16x2(acc[2], acc[3]);
    out.z = pack_bf16x2(acc[4], acc[5]);
    out.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(p.out_o + r * p.d + sl * 8) = out;
    if (sl == 0) p.out_lse[lidx] = lse_out;
  }
}

cudaError_t launch_merge_partials(const MergeParams& p, int max_blocks, cudaStream_t st) {
  const int64_t threads = (int64_t)p.B * p.Nq * p.Hq * (p.d / 8);
  if (threads == 0) return cudaSuccess;
  int64_t blocks = (threads + 255) / 256;
  if (blocks > max_blocks) blocks = max_blocks;
  note_launch();
  merge_partials_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace fm
