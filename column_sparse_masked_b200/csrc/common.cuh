// Definitions shared by the host API and the kernels: tile constants, the
// per-tile class rule, kernel parameter blocks and the workspace layout.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>

namespace fm {

constexpr int kTile = 128;  // rows of a q-tile and columns of a k-tile
constexpr int kClsSkip = 0, kClsPartial = 1, kClsFull = 2;

// Index of the 8 entries of a per-(batch, mask head, k-tile) summary.
enum SummaryIdx { kMnLts = 0, kMxLts, kMnLte, kMxLte, kMnUts, kMxUts, kMnUte, kMxUte };

// Class of the tile (rows [r0, r1)) x (k-tile with summary s).  The summary
// holds min/max of each boundary vector over the k-tile's real columns.
//   skip: one interval covers all rows of the tile in every column;
//   full: no interval reaches any row of the tile in any column.
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: tiles are decided from the O(n) boundary vectors alone.
__host__ __device__ __forceinline__ int classify_tile(const int* s, int r0, int r1) {
  if ((s[kMxLts] <= r0 && s[kMnLte] >= r1) || (s[kMxUts] <= r0 && s[kMnUte] >= r1)) return kClsSkip;
  const bool lt_clear = s[kMnLts] >= r1 || s[kMxLte] <= r0 || s[kMnLts] >= s[kMxLte];
  const bool ut_clear = s[kMnUts] >= r1 || s[kMxUte] <= r0 || s[kMnUts] >= s[kMxUte];
  return (lt_clear && ut_clear) ? kClsFull : kClsPartial;
}

// Forward work-list entry: k-tile index in bits 8.., class of the block's
// first q-tile in bits 0..1, of the second in bits 2..3, bit 4 set on the
// ragged last k-tile (its padded columns must be masked).
__host__ __device__ __forceinline__ int fwd_entry(int kt, int c0, int c1, int ragged) {
  return (kt << 8) | c0 | (c1 << 2) | (ragged << 4);
}
// Backward work-list entry: q-tile index in bits 2.., class in bits 0..1.
__host__ __device__ __forceinline__ int bwd_entry(int qt, int c) { return (qt << 2) | c; }

struct Shape {
  int B, Hq, Hkv, Hm, Nq, Nk, d;
  int G;      // q-heads per KV head
  int nQt;    // q-tiles
  int nKt;    // k-tiles
  int nQB;    // forward blocks of two q-tiles
  int Ef;     // forward: q-heads per scheduling unit (Hq / Hm)
  int Mu;     // backward: scheduling units per (batch, k-tile): 1 if Hm == 1 else Hkv
  int Eb;     // backward: KV heads per unit (Hkv / Mu)
  int64_t n_units_fwd, n_units_bwd;
};

inline Shape make_shape(int B, int Hq, int Hkv, int Hm, int Nq, int Nk, int d) {
  Shape s{};
  s.B = B; s.Hq = Hq; s.Hkv = Hkv; s.Hm = Hm; s.Nq = Nq; s.Nk = Nk; s.d = d;
  s.G = Hq / Hkv;
  s.nQt = (Nq + kTile - 1) / kTile;
  s.nKt = (Nk + kTile - 1) / kTile;
  s.nQB = (s.nQt + 1) / 2;
  s.Ef = Hq / Hm;
  s.Mu = (Hm == 1) ? 1 : Hkv;
  s.Eb = Hkv / s.Mu;
  s.n_units_fwd = (int64_t)B * Hm * s.nQB;
  s.n_units_bwd = (int64_t)B * s.Mu * s.nKt;
  return s;
}

// Workspace layout (byte offsets, each region 256-byte aligned).
struct WsLayout {
  size_t rec, ksum, fcount, flist, forder, counters;       // forward part
  size_t bcount, blist, border, lse2, dsum, dqacc;         // backward part
  size_t fwd_bytes, bwd_bytes;
};

inline size_t ws_align(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout make_layout(const Shape& s) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = ws_align(off + bytes); return o; };
  const size_t bhm = (size_t)s.B * s.Hm;
  L.rec = take(bhm * s.nKt * kTile * 16);
  L.ksum = take(bhm * s.nKt * 8 * 4);
  L.fcount = take(bhm * s.nQB * 4);
  L.flist = take(bhm * s.nQB * s.nKt * 4);
  L.forder = take((size_t)s.n_units_fwd * 4);
  L.counters = take(64);
  L.fwd_bytes = off;
  L.bcount = take(bhm * s.nKt * 4);
  L.blist = take(bhm * s.nKt * s.nQt * 4);
  L.border = take((size_t)s.n_units_bwd * 4);
  L.lse2 = take((size_t)s.B * s.Hq * s.nQt * kTile * 4);
  L.dsum = take((size_t)s.B * s.Hq * s.nQt * kTile * 4);
  L.dqacc = take((size_t)s.B * s.Nq * s.Hq * s.d * 4);
  L.bwd_bytes = off;
  return L;
}

// ----------------------------------------------------------------------------
// kernel parameter blocks
// ----------------------------------------------------------------------------
struct MaskPrepParams {
  const int32_t *lts, *lte, *uts, *ute;  // [B, Hm, Nk]; a null pair = empty intervals
  int B, Hm, Nk, nKt;
  int4* rec;    // [B, Hm, nKt*128] {LTS, LTE, UTS, UTE}; padded columns hide every row
  int* ksum;    // [B, Hm, nKt, 8]
};

struct PlanParams {
  Shape s;
  const int* ksum;
  int* fcount; int* flist;   // forward lists  [B, Hm, nQB] / [B, Hm, nQB, nKt]
  int* bcount; int* blist;   // backward lists [B, Hm, nKt] / [B, Hm, nKt, nQt]
  uint8_t* cls;              // optional export [B, Hm, nQt, nKt]
};

struct SortParams {
  Shape s;
  int mode;               // 0: forward units, 1: backward units
  const int* count;       // fcount or bcount
  int* order;             // out: unit order, descending cost
  int* counter;           // zeroed for the persistent kernel that follows
  int n_units;
};

struct FwdParams {
  Shape s;
  float scale_log2;          // scale * log2(e)
  const int4* rec;
  const int* flist;
  const int* fcount;
  const int* order;
  int* counter;
  int n_items;
  __nv_bfloat16* o;
  float* lse;
  int* status;
  uint64_t wait_limit_ns;
};

struct BwdPreParams {
  Shape s;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  float* lse2;     // [B, Hq, nQt*128]: LSE * log2(e); +inf for empty and padded rows
  float* dsum;     // [B, Hq, nQt*128]: rowsum(dO * O); 0 for padded rows
  float* dqacc;    // [B, Nq, Hq, d] zeroed
};

struct BwdParams {
  Shape s;
  float scale;
  float scale_log2;
  const int4* rec;
  const int* blist;
  const int* bcount;
  const int* order;
  int* counter;
  int n_items;
  const float* lse2;
  const float* dsum;
  float* dqacc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int* status;
  uint64_t wait_limit_ns;
};

struct DqFinParams {
  const float* dqacc;
  __nv_bfloat16* dq;
  float scale;
  int64_t n;  // elements
};

}  // namespace fm
