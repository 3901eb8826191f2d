/*
 * flashmask.h -- C ABI of the B200 (sm_100a) column-sparse masked attention
 * library.
 *
 * The method: "FlashMask-3 targets masked distributed attention on Hopper
 * GPUs", section "In-depth insight".  A structured attention mask is stored
 * column-wise: for every key column j four int32 query-axis boundaries
 * LTS[j], LTE[j], UTS[j], UTE[j] (O(n) storage instead of O(n^2)).  Query row
 * i is masked for key j iff
 *
 *     LTS[j] <= i < LTE[j]   or   UTS[j] <= i < UTE[j]      (half-open)
 *
 * An interval with start >= end is empty.  That encoding covers causal,
 * document, prefix-LM, share-question, sliding-window and block-sparse masks.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library never allocates or frees device memory; scratch space is passed
 *    in as `workspace` (size from the *_workspace_size queries).
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream) and returns 0 or a negative FLASHMASK_ERR_*
 *    code.  Argument errors are detected on the host before any launch.
 *  - Layouts (contiguous, row-major, bf16 = IEEE bfloat16 bit patterns):
 *      q, o, dout, dq      [B, Nq, Hq, d]
 *      k, v, dk, dv        [B, Nk, Hkv, d]
 *      lse                 [B, Hq, Nq]   float32, natural log of the
 *                                        row's softmax normaliser
 *      lts, lte, uts, ute  [B, Hm, Nk]   int32
 *    q-head h reads KV head h / (Hq / Hkv) and mask head (Hm == 1 ? 0 : h).
 *  - A NULL (lts, lte) pair or a NULL (uts, ute) pair means that interval is
 *    empty for every column.
 *  - scale <= 0 selects 1/sqrt(d).
 *  - Supported: d in {64, 128}; Hq % Hkv == 0; Hm in {1, Hq}; any
 *    Nq, Nk >= 0 (ragged tails are handled); all pointers 16-byte aligned.
 *  - Tiles are 128 query rows x 128 key columns.
 *  - Device-side failures (a bounded wait that timed out) are recorded in a
 *    per-device status word that flashmask_get_status() reads and clears.
 *  - Work items of the persistent kernels are taken longest-first in waves of
 *    (batch, KV head) groups whose shared data fit an L2 budget (64 MiB by
 *    default; the environment variable FLASHMASK_WAVE_BUDGET_MB overrides it,
 *    read at each call: a tuning knob that changes the order of the work,
 *    never its results beyond fp32 summation order in the fused backward's dQ).
 *  - Mask values are applied literally, in or out of [0, Nq].  The checks
 *    build of the library (libflashmask_checks.so, the same entry points
 *    compiled with FLASHMASK_CHECKS) also records FLASHMASK_ERR_BOUNDS in the
 *    status word for a mask value outside [0, Nq] and for any work-order or
 *    work-list index out of range; a work item that fails a check is skipped,
 *    so no access is made with a bad index.
 */
#ifndef FLASHMASK_H_
#define FLASHMASK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLASHMASK_OK 0
#define FLASHMASK_ERR_INVALID_ARG (-1) /* null pointer, negative size, bad head counts   */
#define FLASHMASK_ERR_UNSUPPORTED (-2) /* d not in {64,128}, sizes above int32 ranges     */
#define FLASHMASK_ERR_ALIGN (-3)       /* a pointer is not 16-byte aligned                */
#define FLASHMASK_ERR_WORKSPACE (-4)   /* workspace missing or smaller than required      */
#define FLASHMASK_ERR_CUDA (-5)        /* a CUDA runtime call or launch failed            */
#define FLASHMASK_ERR_TIMEOUT (-6)     /* a kernel's bounded wait expired (status word)   */
#define FLASHMASK_ERR_NO_DEVICE (-7)   /* no sm_100 device current                        */
#define FLASHMASK_ERR_TOO_LARGE (-8)   /* problem needs more than the static no-alloc scratch */
#define FLASHMASK_ERR_BOUNDS (-9)      /* checks build: mask value outside [0, Nq], or an internal
                                          index out of range (status word)                   */

/* Problem shape.  B batch, Hq query heads, Hkv key/value heads, Hm mask heads
 * (1 or Hq), Nq query rows, Nk key columns, d head dimension. */
typedef struct flashmask_dims {
  int32_t B, Hq, Hkv, Hm, Nq, Nk, d;
} flashmask_dims;

/* Bytes of workspace flashmask_fwd needs for `dims` (mask summary, padded
 * boundary records, per-tile work lists, scheduler order), whichever forward
 * item kind (flashmask_set_fwd_pairing) the call uses. */
size_t flashmask_fwd_workspace_size(const flashmask_dims* dims);

/*
 * Forward: O = softmax(scale * Q K^T + mask) V per (batch, q-head) and
 * LSE = m + ln(sum exp(s - m)) per row ("FlashMask-3 targets masked
 * distributed attention on Hopper GPUs", In-depth insight: mask-aware
 * attention forward).  Tiles that the per-tile min/max summary proves fully
 * masked are skipped; the element mask is applied only on partially masked
 * tiles.  Rows with no visible key produce O = 0 and LSE = -inf.
 * Outputs: o (bf16, written in full), lse (fp32, written in full).
 */
int flashmask_fwd(const void* q, const void* k, const void* v, const int32_t* lts, const int32_t* lte,
                  const int32_t* uts, const int32_t* ute, float scale, const flashmask_dims* dims, void* o,
                  float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the library's static device scratch used by flashmask_fwd_noalloc. */
#define FLASHMASK_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * Forward that allocates nothing: the same computation and outputs as
 * flashmask_fwd, but its scratch (mask records, block summary, work lists,
 * scheduler order) lives in one file-scope device array of
 * FLASHMASK_NOALLOC_SCRATCH_BYTES inside the library instead of a
 * caller-provided workspace.  (No counterpart in the paper: this is an
 * interface convenience, not part of the method.)
 *
 * For callers that cannot allocate device memory while they run: a serving
 * process that reserves its whole memory budget at start-up and treats any
 * later allocation as a fault, or a plugin whose host framework owns the
 * device allocator and offers its plugins no way to request workspace.
 * The caller still owns and passes q, k, v, the mask vectors, o and lse.
 *
 *  - Every GPU that loads the library holds the 16 MiB array until the
 *    process exits, whether or not this entry point is used.
 *  - The first call on a device looks up the array's device address with
 *    that device current (once per device); make that first call before
 *    any stream capture.
 *  - Problems whose forward workspace (flashmask_fwd_workspace_size) exceeds
 *    the array are rejected with FLASHMASK_ERR_TOO_LARGE before any launch;
 *    the 16 MiB covers, e.g., one 131072-token sequence with one mask head.
 *  - All calls share the one array and it keeps the previous call's
 *    contents; each call writes everything it later reads (and resets its
 *    work counter) itself.  Calls whose kernels overlap on the GPU -- on
 *    different streams, or from different host threads -- race on the
 *    array: serialise them.
 * No cudaMalloc, cudaFree or other allocating routine is called.
 */
int flashmask_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* lts, const int32_t* lte,
                          const int32_t* uts, const int32_t* ute, float scale, const flashmask_dims* dims,
                          void* o, float* lse, void* stream);

/* Bytes of workspace flashmask_bwd needs (forward's plus the backward lists,
 * per-row D = rowsum(dO*O) and LSE in log2 units over whole 128-row tiles, and
 * the fused backward's fp32 dQ accumulator, 4 * B * Hq * ceil(Nq/128) * 128 * d
 * bytes).  The same size serves both backward modes. */
size_t flashmask_bwd_workspace_size(const flashmask_dims* dims);

/* Backward modes (process-wide, flashmask_set_bwd_mode). */
#define FLASHMASK_BWD_FUSED 0 /* default: one key-stationary pass, dQ by fp32 reductions   */
#define FLASHMASK_BWD_SPLIT 1 /* key-side dK/dV kernel + query-side dQ kernel, deterministic */

/*
 * Backward of the forward above for the loss sum(O * dO) (same page and
 * section: the mask-aware kernels cover both passes): dQ, dK, dV.  dK and dV
 * sum the contributions of the Hq/Hkv q-heads that share a KV head.  `o` and
 * `lse` must be the forward's outputs for the same inputs.  Key columns that
 * no row sees get dK = dV = 0; fully masked rows get dQ = 0.  Outputs are
 * written in full.
 *
 * FLASHMASK_BWD_FUSED (default): each non-skipped (q-tile, k-tile) pair is
 * visited once by a key-stationary kernel that forms S, dP and dS once and
 * computes all five matmuls of the pair; dK and dV are accumulated on chip
 * and written once (deterministic); each pair's dQ contribution is added into
 * an fp32 accumulator in the workspace with fp32 reductions, and a finalize
 * kernel writes dQ = bf16(scale * acc).  dQ is therefore exact up to the
 * order of fp32 additions, which varies from run to run.
 * FLASHMASK_BWD_SPLIT: a key-stationary dK/dV kernel and a query-stationary
 * dQ kernel that recomputes S and dP (1.4x the matmul work); every output
 * element is written by exactly one CTA, no atomics: bit-reproducible.
 *
 * Streams: the preprocess (each row's D = rowsum(dO*O) and LSE in log2 units;
 * in fused mode also zeroing the dQ accumulator) runs on a stream the library
 * owns (one per device, created on first use), ordered after the call's
 * earlier work on `stream` by an event; the mask summary, lists and orders run
 * on `stream` meanwhile.  In split mode the dQ kernel also runs on the
 * library's stream, joined back to `stream` by another event.  Either way
 * everything the call writes is complete in `stream` order when the call's
 * last operation there completes.  Concurrent calls from several host threads
 * share the library's stream and are serialised on it.
 */
int flashmask_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                  const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute, float scale,
                  const flashmask_dims* dims, void* dq, void* dk, void* dv, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * Tile classification (the block summary of the method: per key tile the
 * min/max of each boundary vector).  cls is uint8 [B, Hm, ceil(Nq/128),
 * ceil(Nk/128)].  With mn_X/mx_X the min/max of X over the tile's columns
 * and the q-tile's rows [r0, r1), r1 = min(r0 + 128, Nq):
 *   0 skip     (mx_LTS <= r0 && mn_LTE >= r1) || (mx_UTS <= r0 && mn_UTE >= r1)
 *   2 full     (mn_LTS >= r1 || mx_LTE <= r0 || mn_LTS >= mx_LTE) &&
 *              (mn_UTS >= r1 || mx_UTE <= r0 || mn_UTS >= mx_UTE)
 *   1 partial  otherwise.
 * Uses the forward workspace.
 */
int flashmask_classify(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                       const flashmask_dims* dims, uint8_t* cls, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * Clip-shift-max localisation (same page and section: each query chunk's
 * mask is derived locally from the global vectors, with no data exchanged
 * between chunks): for the contiguous query chunk [a, b),
 * out[t] = max(min(in[t], b) - a, 0) for t < n.  Applied to each of the four
 * vectors, the result encodes exactly rows [a, b) of the full mask.  in and
 * out are device int32 arrays of n elements (may alias).  0 <= a <= b.
 */
int flashmask_localize(const int32_t* in, int32_t* out, int64_t n, int32_t a, int32_t b, void* stream);

/*
 * Localisation onto several increasing, disjoint chunks [starts[c], ends[c])
 * concatenated in order into one local query sequence (a rank that holds
 * several chunks of the sequence): out[t] = sum_c (clamp(in[t], starts[c],
 * ends[c]) - starts[c]).  starts/ends are HOST arrays of nchunks (<= 64)
 * values.
 */
int flashmask_localize_multi(const int32_t* in, int32_t* out, int64_t n, const int32_t* starts,
                             const int32_t* ends, int32_t nchunks, void* stream);

/*
 * Number of unmasked (i, j) pairs over all batches and all Hq query heads,
 * written as one int64 to the device pointer `pairs` (closed form per key
 * column; used for the effective-FLOP count 4*d*pairs forward, 10*d*pairs
 * backward).
 */
int flashmask_count_unmasked(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                             const flashmask_dims* dims, int64_t* pairs, void* stream);

/*
 * Merge of partial attention results over DISJOINT key sets (the same rows
 * attended to n separate key chunks, e.g. by a context-parallel rank as each
 * chunk arrives; same page and section: compute/communication overlap).  Per
 * row of every (batch, q-head): lse = ln(sum_c exp(lse_c)) and
 * o = sum_c exp(lse_c - lse) * o_c -- exactly the attention over the union of
 * the key sets, up to the rounding of the bf16 partials.  Rows with
 * lse_c = -inf for every c get o = 0, lse = -inf.  o_parts / lse_parts: HOST
 * arrays of n (1..16) device pointers to bf16 [B, Nq, Hq, d] and fp32
 * [B, Hq, Nq]; o, lse: outputs of the same shapes (not aliasing any part).  Uses
 * dims->B, Hq, Nq, d.
 */
int flashmask_merge_partials(const void* const* o_parts, const float* const* lse_parts, int32_t n,
                             const flashmask_dims* dims, void* o, float* lse, void* stream);

/*
 * Work of each 128-row query tile: costs[t] (device int64, ceil(Nq/128)
 * entries, 16-byte aligned) receives the number of unmasked (i, j) pairs with
 * row i in [128 t, min(128 t + 128, Nq)), over all batches, all Hq query heads
 * and all Nk key columns (closed form per key column restricted to the tile's
 * rows, one CTA per q-tile).  These are the per-tile loads that
 * flashmask_balance_chunks evens out across context-parallel ranks (same page
 * and section: the sparsity-aware load balancer).  Uses dims->B, Hq, Hm, Nq,
 * Nk (Hkv and d are only checked).  Errors as flashmask_count_unmasked.
 */
int flashmask_tile_costs(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                         const flashmask_dims* dims, int64_t* costs, void* stream);

/*
 * Sparsity-aware split of a query sequence into `parts` contiguous chunks of
 * whole q-tiles, one per context-parallel rank.  The same page and section
 * name a sparsity-aware load balancer (HCC-IPO) without its rule; read here as
 * making the ranks' unmasked-pair counts as even as possible.  A rank's mask
 * then follows from the global vectors by flashmask_localize on its chunk.
 * costs: HOST array of n >= 0 int64 values >= 0, the work of each q-tile (its
 * unmasked (row, key) pairs over heads and batches).  bounds: HOST array of
 * parts + 1 int32, filled with 0 = bounds[0] <= ... <= bounds[parts] = n;
 * chunk p is q-tiles [bounds[p], bounds[p+1]).  The largest chunk cost is the
 * smallest possible; every chunk is non-empty when n >= parts (otherwise the
 * first n chunks hold one tile each).  *max_cost (may be NULL) receives that
 * largest cost.  Pure host computation: no device, no stream.  Returns
 * FLASHMASK_ERR_INVALID_ARG for parts <= 0, n < 0, NULL arrays, a negative
 * cost or a total above INT64_MAX / 4.
 */
int flashmask_balance_chunks(const int64_t* costs, int32_t n, int32_t parts, int32_t* bounds, int64_t* max_cost);

/* Selects the backward mode (FLASHMASK_BWD_FUSED or FLASHMASK_BWD_SPLIT) for
 * every later flashmask_bwd call of the process; FLASHMASK_ERR_INVALID_ARG
 * for any other value.  flashmask_get_bwd_mode returns the current one. */
int flashmask_set_bwd_mode(int32_t mode);
int flashmask_get_bwd_mode(void);

/* Forward work items (process-wide, for every later forward call).  With
 * on = 1 (the default) and a shape with one mask head and an even number of
 * q-heads per KV head, an item is one 128-row q-tile of two q-heads that share
 * a KV head: both halves see the same key tiles, so no tile is computed for a
 * half that skips it.  Otherwise (on = 0, or any other shape) an item is two
 * consecutive q-tiles of one q-head, which compute the union of their key
 * tiles (the tiles one of them skips contribute exact zeros).  Outputs are
 * bit-identical either way.  FLASHMASK_ERR_INVALID_ARG for values other than
 * 0 and 1.  flashmask_get_fwd_pairing returns the current setting. */
int flashmask_set_fwd_pairing(int32_t on);
int flashmask_get_fwd_pairing(void);

/* Synchronises the current device, returns its status word (0 or a negative
 * FLASHMASK_ERR_* code written by a kernel) and resets it to 0. */
int flashmask_get_status(void);

/* Synchronises the current device and copies into info[5] the description of
 * the bounded wait that caused the first FLASHMASK_ERR_TIMEOUT since the
 * status word was last cleared (left unchanged when none occurred since):
 * info[0] kernel (0 forward, 1 backward key side, 2 backward query side,
 * 3 the flashmask_test_wait_timeout self-test, 4 fused backward), info[1] byte offset of the
 * mbarrier in that kernel's shared-memory block, info[2] the phase parity
 * waited for, info[3] block index, info[4] thread index.  Returns
 * FLASHMASK_ERR_INVALID_ARG for a NULL info. */
int flashmask_get_timeout_info(int32_t* info);

/* Sets the limit of every bounded device-side wait, in nanoseconds (default
 * 2e9).  Values <= 0 restore the default.  Host-side setting, process-wide. */
void flashmask_set_wait_limit_ns(int64_t ns);

/* Caps the persistent grid of the attention kernels at n CTAs (0, the
 * default, restores one CTA per SM).  With a small cap one CTA walks many
 * work items in a row, so tests can drive every item-to-item hand-over of the
 * persistent kernels (ring wrap-round, buffer hand-over, phase flips) on
 * problems small enough to check element by element.  Results do not depend
 * on the cap.  Host-side setting, process-wide; FLASHMASK_ERR_INVALID_ARG
 * for n < 0. */
int flashmask_set_max_ctas(int32_t n);

/* Launches one CTA whose only job is a bounded wait on a barrier that nothing
 * arrives on; the wait gives up after `limit_ns` and records
 * FLASHMASK_ERR_TIMEOUT in the status word.  Used to test the failure path
 * without hanging or faulting the GPU. */
int flashmask_test_wait_timeout(int64_t limit_ns, void* stream);

/*
 * Kernel timing for benchmarks.  While enabled (on != 0), every launch of an
 * attention kernel is bracketed by a CUDA event pair recorded on the stream it
 * runs on, and so is the backward's attention unit as a whole (on the call's
 * stream).  flashmask_profiler_read() waits for the recorded events and fills
 * ms[6] / launches[6] (either may be NULL) with the summed milliseconds and
 * counts of kind 0 = forward, 1 = split backward key side (dK, dV), 2 = split
 * backward query side (dQ), 3 = the backward's attention unit (split: kinds 1
 * and 2, which run concurrently, from before the first launch to after both
 * completed; fused: the fused kernel and the dQ finalize), 4 = fused backward
 * kernel, 5 = dQ finalize, then clears them.  Event pairs are pooled (at most
 * 4096 outstanding).  Host-side, process-wide.
 */
int flashmask_profiler_enable(int on);
int flashmask_profiler_read(double* ms, int64_t* launches);

/* Number of kernels this library has launched since the process started
 * (every kind: summary, lists, ordering, preprocess, attention, helpers). */
int64_t flashmask_launch_count(void);

/* Human-readable text of an error code (static storage). */
const char* flashmask_strerror(int code);

/* Library version, 10000 * major + 100 * minor + patch. */
int flashmask_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLASHMASK_H_ */
