// Host side of the C ABI declared in include/flashmask.h: argument checks,
// workspace carving, TMA descriptor encoding and the launch sequence of each
// entry point.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/flashmask.h"
#include "common.cuh"
#include "launchers.h"

namespace fm {

// Per-device status word written by kernels (bounded-wait timeouts).
// [0] status word; [1..5] the wait behind the first timeout since the status
// was last cleared: kernel, barrier offset in the kernel's shared-memory
// struct, parity, block, thread.
__device__ int g_status_word[8];

namespace {

std::atomic<int64_t> g_wait_limit_ns{2000000000LL};
std::atomic<int> g_max_ctas{0};  // 0: one persistent CTA per SM
std::atomic<int> g_bwd_mode{FLASHMASK_BWD_FUSED};
std::atomic<int> g_fwd_pairing{1};

// Persistent grid of an attention kernel: one CTA per SM, at most one per
// work item, at most the process-wide cap when one is set.
int persistent_grid(int64_t n_items, int sm_count) {
  int64_t g = n_items < sm_count ? n_items : sm_count;
  const int cap = g_max_ctas.load(std::memory_order_relaxed);
  if (cap > 0 && g > cap) g = cap;
  return (int)g;
}

// NVTX range around an entry point (visible in a profiler's timeline; a no-op
// when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
thread_local char g_last_cuda_error[256] = "";
std::mutex g_mu;

struct DeviceInfo {
  int sm_count = 0;
  int cc = 0;
  int* status = nullptr;
};

int current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLASHMASK_ERR_NO_DEVICE;
  // Binds the device's primary context to the calling thread: a thread that
  // has made no CUDA call yet (an autograd worker, a user thread) has none,
  // and tensor-map encoding needs one.
  if (cudaSetDevice(dev) != cudaSuccess) return FLASHMASK_ERR_NO_DEVICE;
  static std::unordered_map<int, DeviceInfo> cache;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    DeviceInfo di;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FLASHMASK_ERR_NO_DEVICE;
    di.cc = major * 10 + minor;
    if (di.cc != 100) return FLASHMASK_ERR_NO_DEVICE;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&di.status), g_status_word) != cudaSuccess)
      return FLASHMASK_ERR_CUDA;
    it = cache.emplace(dev, di).first;
  }
  *out = it->second;
  return FLASHMASK_OK;
}

// The library's second stream of the current device, with the fork/join
// events of one backward call (the mutex serialises their use between host
// threads).  Null if it could not be created: the caller's stream alone is used.
struct AuxStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, pre = nullptr, plan = nullptr, join = nullptr;
  std::mutex mu;
};
// Joins the second stream back to the caller's stream if a call returns early
// (an error after the fork), so that none of the call's work stays unordered
// with respect to the caller's later work on its stream.
struct JoinOnExit {
  AuxStream* ax = nullptr;
  cudaStream_t st = nullptr;
  bool armed = false;
  ~JoinOnExit() {
    if (armed) {
      cudaEventRecord(ax->join, ax->stream);
      cudaStreamWaitEvent(st, ax->join, 0);
    }
  }
};

AuxStream* aux_stream() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  static std::unordered_map<int, AuxStream*> cache;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  AuxStream* a = new AuxStream();
  if (cudaStreamCreateWithFlags(&a->stream, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&a->fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&a->pre, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&a->plan, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&a->join, cudaEventDisableTiming) != cudaSuccess) {
    delete a;  // handles of a failed set-up are left to the context (none is used)
    a = nullptr;
  }
  cache.emplace(dev, a);
  return a;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D map over a [B, N, H, d] bf16 tensor: box = 64 columns x 1 head x box_rows rows.
int make_map(CUtensorMap* m, const void* ptr, int B, int N, int H, int d, int box_rows = kTile) {
  auto enc = encode_fn();
  if (!enc) return FLASHMASK_ERR_CUDA;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r == CUDA_SUCCESS) return FLASHMASK_OK;
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return FLASHMASK_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const flashmask_dims* dm) {
  if (!dm) return FLASHMASK_ERR_INVALID_ARG;
  const flashmask_dims& d = *dm;
  if (d.B < 0 || d.Hq <= 0 || d.Hkv <= 0 || d.Hm <= 0 || d.Nq < 0 || d.Nk < 0) return FLASHMASK_ERR_INVALID_ARG;
  if (d.Hq % d.Hkv != 0) return FLASHMASK_ERR_INVALID_ARG;
  if (d.Hm != 1 && d.Hm != d.Hq) return FLASHMASK_ERR_INVALID_ARG;
  if (d.d != 64 && d.d != 128) return FLASHMASK_ERR_UNSUPPORTED;
  if (d.Nq > (1 << 30) || d.Nk > (1 << 30)) return FLASHMASK_ERR_UNSUPPORTED;
  const Shape s = make_shape(d.B, d.Hq, d.Hkv, d.Hm, d.Nq, d.Nk, d.d);
  if (s.n_q_items >= INT_MAX || s.n_kv_items >= INT_MAX)
    return FLASHMASK_ERR_UNSUPPORTED;
  return FLASHMASK_OK;
}

int check_masks(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute) {
  if ((lts == nullptr) != (lte == nullptr)) return FLASHMASK_ERR_INVALID_ARG;
  if ((uts == nullptr) != (ute == nullptr)) return FLASHMASK_ERR_INVALID_ARG;
  for (const int32_t* p : {lts, lte, uts, ute})
    if (p && !aligned16(p)) return FLASHMASK_ERR_ALIGN;
  return FLASHMASK_OK;
}

int check_ws(const void* ws, size_t have, size_t need) {
  if (need == 0) return FLASHMASK_OK;
  if (!ws || have < need) return FLASHMASK_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return FLASHMASK_ERR_ALIGN;
  return FLASHMASK_OK;
}

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return FLASHMASK_OK;
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "CUDA runtime or launch failure in %s: %s", what,
           cudaGetErrorString(e));
  return FLASHMASK_ERR_CUDA;
}

#define FM_TRY(x)                       \
  do {                                  \
    int _rc = (x);                      \
    if (_rc != FLASHMASK_OK) return _rc; \
  } while (0)
#define FM_CUDA(x) FM_TRY(cuda_status((x), #x))

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / std::sqrt((float)d); }

// Steps shared by forward, backward and classify: padded boundary records
// and the per-k-tile block summary.
MaskPrepParams prep_params(const Shape& s, const WsLayout& L, uint8_t* ws, const int32_t* lts, const int32_t* lte,
                           const int32_t* uts, const int32_t* ute, int* status) {
  MaskPrepParams mp{};
  mp.lts = lts; mp.lte = lte; mp.uts = uts; mp.ute = ute;
  mp.B = s.B; mp.Hm = s.Hm; mp.Nk = s.Nk; mp.nKt = s.nKt;
  mp.Nq = s.Nq;
  mp.status = status;
  mp.rec = reinterpret_cast<int4*>(ws + L.rec);
  mp.ksum = reinterpret_cast<int*>(ws + L.ksum);
  return mp;
}

// ---- launch counter and kernel profiler ----
std::atomic<int64_t> g_launches{0};
std::atomic<int> g_profiling{0};
struct ProfRec {
  cudaEvent_t start = nullptr, stop = nullptr;
  int kind = 0;
  bool closed = false;
};
std::vector<ProfRec> g_prof_pool;  // guarded by g_mu
size_t g_prof_used = 0;
constexpr size_t kProfMax = 4096;

// Groups per longest-first wave: as many (batch, KV head) groups as keep the
// data a group's items share (Q/dO -- and, in the fused backward, the fp32 dQ
// accumulator -- for the key side, K/V otherwise) within an L2 budget (half of
// the 126 MB L2 by default; FLASHMASK_WAVE_BUDGET_MB overrides it, a tuning
// knob read at each call); 0 (natural, position order) when a single group is
// larger than that.  Small problems (fewer than 16 items per SM) order all
// groups together for load balance unless the budget is set explicitly.
size_t wave_budget_bytes(bool* explicit_budget) {
  const char* e = getenv("FLASHMASK_WAVE_BUDGET_MB");
  if (e && *e) {
    const long mb = strtol(e, nullptr, 10);
    if (mb > 0) {
      *explicit_budget = true;
      return (size_t)mb << 20;
    }
  }
  *explicit_budget = false;
  return (size_t)64 << 20;
}

int wave_groups(size_t group_bytes, int n_groups, int64_t n_items, int sm_count) {
  bool explicit_budget = false;
  const size_t budget = wave_budget_bytes(&explicit_budget);
  // With few items per CTA the tail of the longest-first order decides the
  // makespan: order all groups together.
  if (group_bytes == 0 || (!explicit_budget && n_items < (int64_t)16 * sm_count)) return n_groups;
  const size_t w = budget / group_bytes;
  if (w == 0) return 0;
  return (int)(w < (size_t)n_groups ? w : (size_t)n_groups);
}

}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// A begin/end pair is recorded only while profiling is on.
constexpr int kProfKinds = 6;

int profile_begin(int kind, cudaStream_t st) {
  if (!g_profiling.load(std::memory_order_relaxed)) return -1;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_prof_used >= kProfMax) return -1;
  if (g_prof_used == g_prof_pool.size()) {
    ProfRec r;
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return -1;
    g_prof_pool.push_back(r);
  }
  const size_t h = g_prof_used;
  ProfRec* r = &g_prof_pool[h];
  r->kind = kind;
  r->closed = false;
  if (cudaEventRecord(r->start, st) != cudaSuccess) return -1;
  ++g_prof_used;
  return (int)h;
}

void profile_end(int handle, cudaStream_t st) {
  if (handle < 0) return;
  std::lock_guard<std::mutex> lock(g_mu);
  if ((size_t)handle >= g_prof_used) return;
  ProfRec& r = g_prof_pool[handle];
  if (cudaEventRecord(r.stop, st) == cudaSuccess) r.closed = true;
}

cudaError_t ensure_smem_limit(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::unordered_map<const void*, uint64_t> done;  // bit per device
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = done.find(func);
    if (it != done.end() && dev < 64 && (it->second >> dev) & 1u) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  if (dev < 64) done[func] |= (uint64_t)1 << dev;
  return cudaSuccess;
}

}  // namespace fm

using namespace fm;

extern "C" {

size_t flashmask_fwd_workspace_size(const flashmask_dims* d) {
  if (check_dims(d) != FLASHMASK_OK) return 0;
  // sized for paired q-heads whenever the shape allows them (the larger
  // layout), so the size holds whichever item kind a call uses
  return make_layout(make_shape(d->B, d->Hq, d->Hkv, d->Hm, d->Nq, d->Nk, d->d, true)).fwd_bytes;
}

size_t flashmask_bwd_workspace_size(const flashmask_dims* d) {
  if (check_dims(d) != FLASHMASK_OK) return 0;
  return make_layout(make_shape(d->B, d->Hq, d->Hkv, d->Hm, d->Nq, d->Nk, d->d)).bwd_bytes;
}

int flashmask_fwd(const void* q, const void* k, const void* v, const int32_t* lts, const int32_t* lte,
                  const int32_t* uts, const int32_t* ute, float scale, const flashmask_dims* dims, void* o,
                  float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx("flashmask_fwd");
  FM_TRY(check_dims(dims));
  FM_TRY(check_masks(lts, lte, uts, ute));
  const flashmask_dims& d = *dims;
  const Shape s = make_shape(d.B, d.Hq, d.Hkv, d.Hm, d.Nq, d.Nk, d.d, g_fwd_pairing.load() != 0);
  if ((int64_t)s.B * s.Nq == 0) return FLASHMASK_OK;
  if (!q || !o || !lse || (s.Nk > 0 && (!k || !v))) return FLASHMASK_ERR_INVALID_ARG;
  for (const void* p : {q, k, v, (const void*)o, (const void*)lse})
    if (p && !aligned16(p)) return FLASHMASK_ERR_ALIGN;
  const WsLayout L = make_layout(s);
  FM_TRY(check_ws(workspace, workspace_bytes, L.fwd_bytes));
  DeviceInfo di;
  FM_TRY(current_device(&di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  CUtensorMap tq, tk, tv;
  FM_TRY(make_map(&tq, q, s.B, s.Nq, s.Hq, s.d));
  if (s.Nk > 0) {
    FM_TRY(make_map(&tk, k, s.B, s.Nk, s.Hkv, s.d));
    FM_TRY(make_map(&tv, v, s.B, s.Nk, s.Hkv, s.d));
  } else {  // never read: every work list is empty
    FM_TRY(make_map(&tk, workspace, 1, 1, 1, s.d));
    tv = tk;
  }
  const MaskPrepParams mp = prep_params(s, L, ws, lts, lte, uts, ute, di.status);
  FM_CUDA(launch_mask_prep(mp, st));

  PlanParams pp{};
  pp.s = s;
  pp.ksum = mp.ksum;
  pp.fcount = reinterpret_cast<int*>(ws + L.fcount);
  pp.flist = reinterpret_cast<int*>(ws + L.flist);
  pp.qcount = reinterpret_cast<int*>(ws + L.qcount);
  FM_CUDA(launch_plan_fwd(pp, st));

  SortParams sp{};
  sp.s = s;
  sp.mode = 0;
  sp.count = pp.fcount;
  sp.order = reinterpret_cast<int*>(ws + L.forder);
  sp.counter = reinterpret_cast<int*>(ws + L.counters);
  sp.n_items = (int)s.n_fwd_items;
  sp.items_per_group = s.nFB * s.fG;
  sp.wave = wave_groups((size_t)s.Nk * s.d * 2 * 2, s.B * s.Hkv, s.n_fwd_items, di.sm_count);
  finish_sort_params(sp);
  FM_CUDA(launch_sort_units(&sp, 1, st));

  FwdParams fp{};
  fp.s = s;
  fp.scale_log2 = resolve_scale(scale, s.d) * 1.4426950408889634f;
  fp.rec = mp.rec;
  fp.flist = pp.flist;
  fp.fcount = pp.fcount;
  fp.order = sp.order;
  fp.counter = sp.counter;
  fp.n_items = (int)s.n_fwd_items;
  fp.o = static_cast<__nv_bfloat16*>(o);
  fp.lse = lse;
  fp.status = di.status;
  fp.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
  const int grid = persistent_grid(fp.n_items, di.sm_count);
  if (grid > 0) FM_CUDA(launch_fwd(fp, tq, tk, tv, grid, st));
  return FLASHMASK_OK;
}

int flashmask_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                  const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute, float scale,
                  const flashmask_dims* dims, void* dq, void* dk, void* dv, void* workspace,
                  size_t workspace_bytes, void* stream) {
  NvtxRange nvtx("flashmask_bwd");
  FM_TRY(check_dims(dims));
  FM_TRY(check_masks(lts, lte, uts, ute));
  const flashmask_dims& d = *dims;
  const Shape s = make_shape(d.B, d.Hq, d.Hkv, d.Hm, d.Nq, d.Nk, d.d);
  if (s.B == 0) return FLASHMASK_OK;
  const bool has_q = s.Nq > 0, has_k = s.Nk > 0;
  if (has_q && (!q || !o || !lse || !dout || !dq)) return FLASHMASK_ERR_INVALID_ARG;
  if (has_k && (!k || !v || !dk || !dv)) return FLASHMASK_ERR_INVALID_ARG;
  for (const void* p : {q, k, v, o, (const void*)lse, dout, (const void*)dq, (const void*)dk, (const void*)dv})
    if (p && !aligned16(p)) return FLASHMASK_ERR_ALIGN;
  const WsLayout L = make_layout(s);
  FM_TRY(check_ws(workspace, workspace_bytes, L.bwd_bytes));
  DeviceInfo di;
  FM_TRY(current_device(&di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float sc = resolve_scale(scale, s.d);

  CUtensorMap tq, tk, tv, tdo;
  if (has_q) {
    FM_TRY(make_map(&tq, q, s.B, s.Nq, s.Hq, s.d));
    FM_TRY(make_map(&tdo, dout, s.B, s.Nq, s.Hq, s.d));
  } else {  // never read: every work list is empty
    FM_TRY(make_map(&tq, workspace, 1, 1, 1, s.d));
    tdo = tq;
  }
  if (has_k) {
    FM_TRY(make_map(&tk, k, s.B, s.Nk, s.Hkv, s.d));
    FM_TRY(make_map(&tv, v, s.B, s.Nk, s.Hkv, s.d));
  } else {
    FM_TRY(make_map(&tk, workspace, 1, 1, 1, s.d));
    tv = tk;
  }
  // The preprocess (D, LSE2; HBM-bound) does not depend on the mask: it runs
  // on the library's second stream while the caller's stream builds the lists
  // and orders.  The query-side kernel follows it there.
  AuxStream* ax = aux_stream();
  std::unique_lock<std::mutex> ax_lock;
  if (ax) ax_lock = std::unique_lock<std::mutex>(ax->mu);
  JoinOnExit join_guard;  // destroyed before the lock is released
  join_guard.ax = ax;
  join_guard.st = st;
  const bool fused = g_bwd_mode.load(std::memory_order_relaxed) == FLASHMASK_BWD_FUSED;
  BwdPreParams bp{};
  bp.s = s;
  bp.o = static_cast<const __nv_bfloat16*>(o);
  bp.dout = static_cast<const __nv_bfloat16*>(dout);
  bp.lse = lse;
  bp.lse2 = reinterpret_cast<float*>(ws + L.lse2);
  bp.dsum = reinterpret_cast<float*>(ws + L.dsum);
  if (fused) {  // the preprocess also zeroes the fp32 dQ accumulator
    bp.dqacc = reinterpret_cast<float4*>(ws + L.dqacc);
    bp.dqacc_vec4 = (int64_t)(dqacc_bytes(s) / 16);
  }
  const int pre_blocks = 64 * di.sm_count;
  if (ax) {
    FM_CUDA(cudaEventRecord(ax->fork, st));
    FM_CUDA(cudaStreamWaitEvent(ax->stream, ax->fork, 0));
    join_guard.armed = true;
    if (has_q) FM_CUDA(launch_bwd_pre(bp, pre_blocks, ax->stream));
    FM_CUDA(cudaEventRecord(ax->pre, ax->stream));
  } else if (has_q) {
    FM_CUDA(launch_bwd_pre(bp, pre_blocks, st));
  }

  const MaskPrepParams mp = prep_params(s, L, ws, lts, lte, uts, ute, di.status);
  FM_CUDA(launch_mask_prep(mp, st));

  if (fused) {
    // one key-stationary pass: key-side lists and order only
    PlanParams pp{};
    pp.s = s;
    pp.ksum = mp.ksum;
    pp.bcount = reinterpret_cast<int*>(ws + L.bcount);
    pp.blist = reinterpret_cast<int*>(ws + L.blist);
    FM_CUDA(launch_plan_bwd(pp, st));
    SortParams sb{};
    sb.s = s;
    sb.mode = 1;
    sb.count = pp.bcount;
    sb.order = reinterpret_cast<int*>(ws + L.border);
    sb.counter = reinterpret_cast<int*>(ws + L.counters) + 1;
    sb.n_items = (int)s.n_kv_items;
    sb.items_per_group = s.nKt;
    // a group's items share its q-heads' Q and dO (bf16) and dQ accumulator rows (fp32)
    sb.wave = wave_groups((size_t)s.G * s.Nq * s.d * (2 + 2 + 4), s.B * s.Hkv, s.n_kv_items, di.sm_count);
    finish_sort_params(sb);
    if (sb.n_items > 0) FM_CUDA(launch_sort_units(&sb, 1, st));
    BwdParams kp{};
    kp.s = s;
    kp.scale = sc;
    kp.scale_log2 = sc * 1.4426950408889634f;
    kp.rec = mp.rec;
    kp.blist = pp.blist;
    kp.bcount = pp.bcount;
    kp.order = sb.order;
    kp.counter = sb.counter;
    kp.n_items = (int)s.n_kv_items;
    kp.lse2 = bp.lse2;
    kp.dsum = bp.dsum;
    kp.dq = static_cast<__nv_bfloat16*>(dq);
    kp.dk = static_cast<__nv_bfloat16*>(dk);
    kp.dv = static_cast<__nv_bfloat16*>(dv);
    kp.dqacc = reinterpret_cast<float*>(ws + L.dqacc);
    kp.status = di.status;
    kp.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
    const int grid = persistent_grid(kp.n_items, di.sm_count);
    if (ax) {
      FM_CUDA(cudaStreamWaitEvent(st, ax->pre, 0));  // D, LSE2 and the zeroed accumulator
      join_guard.armed = false;                      // nothing of this call is left on the second stream
    }
    const int prof = profile_begin(3, st);
    if (grid > 0) FM_CUDA(launch_bwd_fused(kp, tq, tk, tv, tdo, grid, st));
    if (has_q) FM_CUDA(launch_dq_finalize(kp, 64 * di.sm_count, st));
    profile_end(prof, st);
    return FLASHMASK_OK;
  }

  // split backward -- key side: per k-tile q-tile lists, longest-first units
  PlanParams pp{};
  pp.s = s;
  pp.ksum = mp.ksum;
  pp.bcount = reinterpret_cast<int*>(ws + L.bcount);
  pp.blist = reinterpret_cast<int*>(ws + L.blist);
  pp.fcount = reinterpret_cast<int*>(ws + L.fcount);
  pp.flist = reinterpret_cast<int*>(ws + L.flist);
  pp.qcount = reinterpret_cast<int*>(ws + L.qcount);
  // key-side lists (per k-tile q-tile lists) and query-side lists (the
  // forward's per q-block k-tile lists, per q-tile counts) in one launch
  FM_CUDA(launch_plan_both(pp, st));
  int* counters = reinterpret_cast<int*>(ws + L.counters);
  SortParams sb{};
  sb.s = s;
  sb.mode = 1;
  sb.count = pp.bcount;
  sb.order = reinterpret_cast<int*>(ws + L.border);
  sb.counter = counters + 1;
  sb.n_items = (int)s.n_kv_items;
  sb.items_per_group = s.nKt;
  sb.wave = wave_groups((size_t)s.G * s.Nq * s.d * 2 * 2, s.B * s.Hkv, s.n_kv_items, di.sm_count);
  finish_sort_params(sb);
  SortParams sf{};
  sf.s = s;
  sf.mode = 2;
  sf.count = pp.qcount;
  sf.order = reinterpret_cast<int*>(ws + L.qorder);
  sf.counter = counters + 2;
  sf.n_items = (int)s.n_q_items;
  sf.items_per_group = s.nQt * s.G;
  sf.wave = wave_groups((size_t)s.Nk * s.d * 2 * 2, s.B * s.Hkv, s.n_q_items, di.sm_count);
  finish_sort_params(sf);
  {
    SortParams both[2];
    int nsort = 0;
    if (sb.n_items > 0) both[nsort++] = sb;
    if (sf.n_items > 0) both[nsort++] = sf;
    if (nsort > 0) FM_CUDA(launch_sort_units(both, nsort, st));
  }

  BwdParams kp{};
  kp.s = s;
  kp.scale = sc;
  kp.scale_log2 = sc * 1.4426950408889634f;
  kp.rec = mp.rec;
  kp.blist = pp.blist;
  kp.bcount = pp.bcount;
  kp.order = sb.order;
  kp.counter = sb.counter;
  kp.n_items = (int)s.n_kv_items;
  kp.flist = pp.flist;
  kp.fcount = pp.fcount;
  kp.qcount = pp.qcount;
  kp.forder = sf.order;
  kp.counter2 = sf.counter;
  kp.n_items2 = (int)s.n_q_items;
  kp.lse2 = bp.lse2;
  kp.dsum = bp.dsum;
  kp.dq = static_cast<__nv_bfloat16*>(dq);
  kp.dk = static_cast<__nv_bfloat16*>(dk);
  kp.dv = static_cast<__nv_bfloat16*>(dv);
  kp.status = di.status;
  kp.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
  const int grid_kv = persistent_grid(kp.n_items, di.sm_count);
  const int grid_q = (has_q && kp.n_items2 > 0) ? persistent_grid(kp.n_items2, di.sm_count) : 0;
  // The key-side and query-side kernels are independent (same inputs,
  // disjoint outputs).  The query side runs on the library's second stream
  // and is joined back to the caller's stream, so its CTAs take the SMs that
  // the key side's CTAs free as they run out of work.
  if (ax) {
    const int prof = profile_begin(3, st);
    FM_CUDA(cudaStreamWaitEvent(st, ax->pre, 0));           // key side reads D and LSE2
    FM_CUDA(cudaEventRecord(ax->plan, st));
    FM_CUDA(cudaStreamWaitEvent(ax->stream, ax->plan, 0));  // query side reads the lists and orders
    if (grid_kv > 0) FM_CUDA(launch_bwd_dkdv(kp, tq, tk, tv, tdo, grid_kv, st));
    if (grid_q > 0) FM_CUDA(launch_bwd_dq(kp, tq, tk, tv, tdo, grid_q, ax->stream));
    FM_CUDA(cudaEventRecord(ax->join, ax->stream));
    FM_CUDA(cudaStreamWaitEvent(st, ax->join, 0));
    join_guard.armed = false;
    profile_end(prof, st);
  } else {
    const int prof = profile_begin(3, st);
    if (grid_kv > 0) FM_CUDA(launch_bwd_dkdv(kp, tq, tk, tv, tdo, grid_kv, st));
    if (grid_q > 0) FM_CUDA(launch_bwd_dq(kp, tq, tk, tv, tdo, grid_q, st));
    profile_end(prof, st);
  }
  return FLASHMASK_OK;
}

int flashmask_classify(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                       const flashmask_dims* dims, uint8_t* cls, void* workspace, size_t workspace_bytes,
                       void* stream) {
  NvtxRange nvtx("flashmask_classify");
  FM_TRY(check_dims(dims));
  FM_TRY(check_masks(lts, lte, uts, ute));
  const flashmask_dims& d = *dims;
  const Shape s = make_shape(d.B, d.Hq, d.Hkv, d.Hm, d.Nq, d.Nk, d.d);
  if ((int64_t)s.B * s.nQt * s.nKt == 0) return FLASHMASK_OK;
  if (!cls) return FLASHMASK_ERR_INVALID_ARG;
  const WsLayout L = make_layout(s);
  FM_TRY(check_ws(workspace, workspace_bytes, L.fwd_bytes));
  DeviceInfo di;
  FM_TRY(current_device(&di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const MaskPrepParams mp = prep_params(s, L, ws, lts, lte, uts, ute, di.status);
  FM_CUDA(launch_mask_prep(mp, st));
  PlanParams pp{};
  pp.s = s;
  pp.ksum = mp.ksum;
  pp.cls = cls;
  FM_CUDA(launch_classify_export(pp, st));
  return FLASHMASK_OK;
}

int flashmask_localize(const int32_t* in, int32_t* out, int64_t n, int32_t a, int32_t b, void* stream) {
  NvtxRange nvtx("flashmask_localize");
  if (n < 0 || a < 0 || b < a) return FLASHMASK_ERR_INVALID_ARG;
  if (n == 0) return FLASHMASK_OK;
  if (!in || !out) return FLASHMASK_ERR_INVALID_ARG;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  FM_CUDA(launch_localize(in, out, n, a, b, static_cast<cudaStream_t>(stream)));
  return FLASHMASK_OK;
}

int flashmask_localize_multi(const int32_t* in, int32_t* out, int64_t n, const int32_t* starts,
                             const int32_t* ends, int32_t nchunks, void* stream) {
  NvtxRange nvtx("flashmask_localize_multi");
  if (n < 0 || nchunks < 0 || nchunks > 64) return FLASHMASK_ERR_INVALID_ARG;
  if (nchunks > 0 && (!starts || !ends)) return FLASHMASK_ERR_INVALID_ARG;
  for (int c = 0; c < nchunks; ++c) {
    if (starts[c] < 0 || ends[c] < starts[c]) return FLASHMASK_ERR_INVALID_ARG;
    if (c > 0 && starts[c] < ends[c - 1]) return FLASHMASK_ERR_INVALID_ARG;
  }
  if (n == 0) return FLASHMASK_OK;
  if (!in || !out) return FLASHMASK_ERR_INVALID_ARG;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  FM_CUDA(launch_localize_multi(in, out, n, starts, ends, nchunks, static_cast<cudaStream_t>(stream)));
  return FLASHMASK_OK;
}

int flashmask_count_unmasked(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                             const flashmask_dims* dims, int64_t* pairs, void* stream) {
  NvtxRange nvtx("flashmask_count_unmasked");
  FM_TRY(check_dims(dims));
  FM_TRY(check_masks(lts, lte, uts, ute));
  if (!pairs) return FLASHMASK_ERR_INVALID_ARG;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  const flashmask_dims& d = *dims;
  MaskPrepParams mp{};
  mp.lts = lts; mp.lte = lte; mp.uts = uts; mp.ute = ute;
  mp.B = d.B; mp.Hm = d.Hm; mp.Nk = d.Nk;
  FM_CUDA(launch_count_unmasked(mp, d.Hq, d.Nq, pairs, static_cast<cudaStream_t>(stream)));
  return FLASHMASK_OK;
}

int flashmask_tile_costs(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                         const flashmask_dims* dims, int64_t* costs, void* stream) {
  NvtxRange nvtx("flashmask_tile_costs");
  FM_TRY(check_dims(dims));
  FM_TRY(check_masks(lts, lte, uts, ute));
  const flashmask_dims& d = *dims;
  if (d.Nq == 0) return FLASHMASK_OK;
  if (!costs) return FLASHMASK_ERR_INVALID_ARG;
  if (!aligned16(costs)) return FLASHMASK_ERR_ALIGN;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  MaskPrepParams mp{};
  mp.lts = lts; mp.lte = lte; mp.uts = uts; mp.ute = ute;
  mp.B = d.B; mp.Hm = d.Hm; mp.Nk = d.Nk;
  FM_CUDA(launch_tile_costs(mp, d.Hq, d.Nq, costs, static_cast<cudaStream_t>(stream)));
  return FLASHMASK_OK;
}

int flashmask_merge_partials(const void* const* o_parts, const float* const* lse_parts, int32_t n,
                             const flashmask_dims* dims, void* o, float* lse, void* stream) {
  NvtxRange nvtx("flashmask_merge_partials");
  FM_TRY(check_dims(dims));
  if (n < 1 || n > kMaxMergeParts || !o_parts || !lse_parts) return FLASHMASK_ERR_INVALID_ARG;
  const flashmask_dims& d = *dims;
  if ((int64_t)d.B * d.Nq == 0) return FLASHMASK_OK;
  if (!o || !lse) return FLASHMASK_ERR_INVALID_ARG;
  MergeParams mp{};
  for (int c = 0; c < n; ++c) {
    if (!o_parts[c] || !lse_parts[c]) return FLASHMASK_ERR_INVALID_ARG;
    if (!aligned16(o_parts[c]) || !aligned16(lse_parts[c])) return FLASHMASK_ERR_ALIGN;
    mp.o[c] = static_cast<const __nv_bfloat16*>(o_parts[c]);
    mp.lse[c] = lse_parts[c];
  }
  if (!aligned16(o) || !aligned16(lse)) return FLASHMASK_ERR_ALIGN;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  mp.n = n;
  mp.B = d.B; mp.Nq = d.Nq; mp.Hq = d.Hq; mp.d = d.d;
  mp.out_o = static_cast<__nv_bfloat16*>(o);
  mp.out_lse = lse;
  FM_CUDA(launch_merge_partials(mp, 64 * di.sm_count, static_cast<cudaStream_t>(stream)));
  return FLASHMASK_OK;
}

int flashmask_set_bwd_mode(int32_t mode) {
  if (mode != FLASHMASK_BWD_FUSED && mode != FLASHMASK_BWD_SPLIT) return FLASHMASK_ERR_INVALID_ARG;
  g_bwd_mode.store(mode);
  return FLASHMASK_OK;
}

int flashmask_get_bwd_mode(void) { return g_bwd_mode.load(); }

int flashmask_set_fwd_pairing(int32_t on) {
  if (on != 0 && on != 1) return FLASHMASK_ERR_INVALID_ARG;
  g_fwd_pairing.store(on);
  return FLASHMASK_OK;
}

int flashmask_get_fwd_pairing(void) { return g_fwd_pairing.load(); }

int flashmask_set_max_ctas(int32_t n) {
  if (n < 0) return FLASHMASK_ERR_INVALID_ARG;
  g_max_ctas.store(n);
  return FLASHMASK_OK;
}

int flashmask_get_status(void) {
  DeviceInfo di;
  FM_TRY(current_device(&di));
  if (cudaDeviceSynchronize() != cudaSuccess) return FLASHMASK_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, di.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FLASHMASK_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(di.status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FLASHMASK_ERR_CUDA;
  return v;
}

int flashmask_get_timeout_info(int32_t* info) {
  if (!info) return FLASHMASK_ERR_INVALID_ARG;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  if (cudaDeviceSynchronize() != cudaSuccess) return FLASHMASK_ERR_CUDA;
  int v[8] = {};
  if (cudaMemcpy(v, di.status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return FLASHMASK_ERR_CUDA;
  for (int i = 0; i < 5; ++i) info[i] = v[1 + i];
  return FLASHMASK_OK;
}

void flashmask_set_wait_limit_ns(int64_t ns) { g_wait_limit_ns.store(ns > 0 ? ns : 2000000000LL); }

int flashmask_test_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0) return FLASHMASK_ERR_INVALID_ARG;
  DeviceInfo di;
  FM_TRY(current_device(&di));
  FM_CUDA(launch_wait_timeout(di.status, (uint64_t)limit_ns, static_cast<cudaStream_t>(stream)));
  return FLASHMASK_OK;
}

int flashmask_profiler_enable(int on) {
  g_profiling.store(on ? 1 : 0);
  return FLASHMASK_OK;
}

int flashmask_profiler_read(double* ms_out, int64_t* launches_out) {
  std::lock_guard<std::mutex> lock(g_mu);
  double ms[kProfKinds] = {};
  int64_t cnt[kProfKinds] = {};
  int rc = FLASHMASK_OK;
  for (size_t i = 0; i < g_prof_used; ++i) {
    ProfRec& r = g_prof_pool[i];
    if (!r.closed) continue;
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
      rc = FLASHMASK_ERR_CUDA;
      continue;
    }
    const int kd = (r.kind >= 0 && r.kind < kProfKinds) ? r.kind : 0;
    ms[kd] += t;
    cnt[kd] += 1;
  }
  g_prof_used = 0;
  for (int kd = 0; kd < kProfKinds; ++kd) {
    if (ms_out) ms_out[kd] = ms[kd];
    if (launches_out) launches_out[kd] = cnt[kd];
  }
  return rc;
}

int64_t flashmask_launch_count(void) { return g_launches.load(); }

const char* flashmask_strerror(int code) {
  switch (code) {
    case FLASHMASK_OK: return "ok";
    case FLASHMASK_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or head counts)";
    case FLASHMASK_ERR_UNSUPPORTED: return "unsupported configuration (head_dim must be 64 or 128; sizes too large)";
    case FLASHMASK_ERR_ALIGN: return "pointer not 16-byte aligned (workspace: 256-byte)";
    case FLASHMASK_ERR_WORKSPACE: return "workspace missing or too small";
    case FLASHMASK_ERR_CUDA:
      return g_last_cuda_error[0] ? g_last_cuda_error : "CUDA runtime or launch failure";
    case FLASHMASK_ERR_TIMEOUT: return "a device-side bounded wait timed out";
    case FLASHMASK_ERR_NO_DEVICE: return "no sm_100 (B200-class) device is current";
    case FLASHMASK_ERR_BOUNDS:
      return "a mask value outside [0, Nq] or an internal index out of range (checks build)";
    case FLASHMASK_ERR_TOO_LARGE:
      return "problem too large for flashmask_fwd_noalloc: its forward workspace exceeds "
             "FLASHMASK_NOALLOC_SCRATCH_BYTES (16 MiB); use flashmask_fwd with a workspace";
    default: return "unknown error code";
  }
}

int flashmask_version(void) { return 100; }

}  // extern "C"

// ----------------------------------------------------------------------------
// Forward without a caller-provided workspace (see flashmask_fwd_noalloc in
// include/flashmask.h).  For callers that may not allocate device memory once
// running; the forward's scratch lives in this file-scope device array.
// ----------------------------------------------------------------------------
namespace fm {
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[FLASHMASK_NOALLOC_SCRATCH_BYTES];

// Device address of the array, looked up once per device with that device
// current.  In host code the array's name is only a host-side stand-in, so
// the address must come from cudaGetSymbolAddress.
int noalloc_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLASHMASK_ERR_NO_DEVICE;
  static std::unordered_map<int, void*> addr;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = addr.find(dev);
  if (it == addr.end()) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return cuda_status(e == cudaSuccess ? cudaErrorInvalidSymbol : e,
                                                             "cudaGetSymbolAddress(g_noalloc_scratch)");
    it = addr.emplace(dev, p).first;
  }
  *out = it->second;
  return FLASHMASK_OK;
}

}  // namespace
}  // namespace fm

extern "C" int flashmask_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* lts,
                                     const int32_t* lte, const int32_t* uts, const int32_t* ute, float scale,
                                     const flashmask_dims* dims, void* o, float* lse, void* stream) {
  FM_TRY(check_dims(dims));
  const size_t need = flashmask_fwd_workspace_size(dims);
  if (need > (size_t)FLASHMASK_NOALLOC_SCRATCH_BYTES) return FLASHMASK_ERR_TOO_LARGE;
  DeviceInfo di;
  FM_TRY(current_device(&di));  // binds the device's context to this thread first
  void* scratch = nullptr;
  FM_TRY(noalloc_scratch_address(&scratch));
  return flashmask_fwd(q, k, v, lts, lte, uts, ute, scale, dims, o, lse, scratch,
                       (size_t)FLASHMASK_NOALLOC_SCRATCH_BYTES, stream);
}
