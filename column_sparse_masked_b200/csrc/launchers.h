// Host-side launchers of the kernels; each returns the launch status.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace fm {

cudaError_t launch_mask_prep(const MaskPrepParams& p, cudaStream_t st);
cudaError_t launch_plan_fwd(const PlanParams& p, cudaStream_t st);
cudaError_t launch_plan_bwd(const PlanParams& p, cudaStream_t st);
// Key-side and query-side lists of the backward in one launch.
cudaError_t launch_plan_both(const PlanParams& p, cudaStream_t st);
cudaError_t launch_classify_export(const PlanParams& p, cudaStream_t st);
// Sorts the work items of count (1 or 2) independent orders, one block each.
cudaError_t launch_sort_units(const SortParams* ps, int count, cudaStream_t st);
// Fills cost_cap and n_buckets (chooses the counting sort when it fits).
void finish_sort_params(SortParams& p);
cudaError_t launch_localize(const int32_t* in, int32_t* out, int64_t n, int32_t a, int32_t b, cudaStream_t st);
cudaError_t launch_localize_multi(const int32_t* in, int32_t* out, int64_t n, const int32_t* starts,
                                  const int32_t* ends, int nchunks, cudaStream_t st);
cudaError_t launch_count_unmasked(const MaskPrepParams& p, int Hq, int Nq, int64_t* out, cudaStream_t st);
// Unmasked pairs of each 128-row q-tile over batches and Hq q-heads: out[ceil(Nq/128)].
cudaError_t launch_tile_costs(const MaskPrepParams& p, int Hq, int Nq, int64_t* out, cudaStream_t st);
cudaError_t launch_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t st);
cudaError_t launch_merge_partials(const MergeParams& p, int max_blocks, cudaStream_t st);

// Forward / backward attention kernels.  `grid` is the persistent CTA count.
cudaError_t launch_fwd(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       int grid, cudaStream_t st);
cudaError_t launch_bwd_pre(const BwdPreParams& p, int max_blocks, cudaStream_t st);
// Backward, key side (dK, dV) and query side (dQ); both persistent, grid CTAs.
cudaError_t launch_bwd_dkdv(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, int grid, cudaStream_t st);
cudaError_t launch_bwd_dq(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, int grid, cudaStream_t st);
// Fused backward (dQ, dK, dV in one key-stationary pass; dQ into p.dqacc) and
// the conversion of the fp32 dQ accumulator into bf16 dQ.
cudaError_t launch_bwd_fused(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, int grid, cudaStream_t st);
cudaError_t launch_dq_finalize(const BwdParams& p, int max_blocks, cudaStream_t st);

// Launch bookkeeping: counts every launch.
void note_launch();

// Launches `kernel` after the previous kernel of the stream with programmatic
// stream serialisation: the kernel may be scheduled while its predecessor
// finishes and must call griddep_wait() before reading that kernel's outputs.
// Used only where the predecessor in the stream is a kernel of this library
// (not an event wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}
// Kernel timing (while profiling is on): begin records a start event on st and
// returns a handle (-1 when nothing was recorded); end records the matching
// stop event.  Kinds: 0 forward, 1 backward key side, 2 backward query side
// (split backward), 3 the backward's attention unit (split: the two kernels,
// fork to join; fused: the fused kernel and the dQ finalize), 4 the fused
// backward kernel, 5 the dQ finalize.
int profile_begin(int kind, cudaStream_t st);
void profile_end(int handle, cudaStream_t st);

// Raises a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_smem_limit(const void* func, int bytes);

}  // namespace fm
