// Definitions shared by the host API and the kernels: tile constants, the
// per-tile class rule, kernel parameter blocks and the workspace layout.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>

namespace fm {

constexpr int kTile = 128;  // rows of a q-tile and columns of a k-tile

// Checks build (compiled with -DFLASHMASK_CHECKS=1 into a library of its own):
// mask values outside [0, Nq] and out-of-range scheduler indices (work orders,
// list counts and entries) are recorded as FLASHMASK_ERR_BOUNDS in the status
// word; a work item that fails a check is not processed (it ends the CTA's
// work), so no access is made with a bad index.
#ifdef FLASHMASK_CHECKS
constexpr bool kChecks = true;
#else
constexpr bool kChecks = false;
#endif
constexpr int kDevErrBounds = -9;
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
  int nQB;    // blocks of two q-tiles (the query-side lists of the backward)
  // Forward items take two 128-row q-tiles of one q-head (a block of two
  // q-tiles) or, with `fpair`, one q-tile of two q-heads that share a KV head
  // and a mask (GQA with one mask head): both halves then see exactly the
  // same key tiles, so no tile is computed for a q-tile that skips it.
  int fpair;  // forward items pair two q-heads
  int nFB;    // forward blocks: nQB, or nQt with fpair
  int fG;     // forward items per (b, KV head, block): G, or G/2 with fpair
  // Work items of the three attention kernels, indexed group-major: a group
  // is one (batch, KV head), i.e. the data one L2-resident working set shares.
  //   forward   (b, hkv, block, q-head (pair) in group): B*Hkv*fG*nFB items
  //   key side  (b, hkv, k-tile):                         B*Hkv*nKt items
  //   query side(b, hkv, q-tile, q-head in group):        B*Hq*nQt items
  int64_t n_fwd_items, n_kv_items, n_q_items;
};

// Forward items pair q-heads when the shape allows it: one mask head and an
// even number of q-heads per KV head.
inline bool fwd_pairing_possible(int Hq, int Hkv, int Hm) { return Hm == 1 && (Hq / Hkv) % 2 == 0; }

inline Shape make_shape(int B, int Hq, int Hkv, int Hm, int Nq, int Nk, int d, bool fpair = false) {
  Shape s{};
  s.B = B; s.Hq = Hq; s.Hkv = Hkv; s.Hm = Hm; s.Nq = Nq; s.Nk = Nk; s.d = d;
  s.G = Hq / Hkv;
  s.nQt = (Nq + kTile - 1) / kTile;
  s.nKt = (Nk + kTile - 1) / kTile;
  s.nQB = (s.nQt + 1) / 2;
  s.fpair = (fpair && fwd_pairing_possible(Hq, Hkv, Hm)) ? 1 : 0;
  s.nFB = s.fpair ? s.nQt : s.nQB;
  s.fG = s.fpair ? s.G / 2 : s.G;
  s.n_fwd_items = (int64_t)B * Hkv * s.fG * s.nFB;
  s.n_kv_items = (int64_t)B * Hkv * s.nKt;
  s.n_q_items = (int64_t)B * Hq * s.nQt;
  return s;
}

// Workspace layout (byte offsets, each region 256-byte aligned).
struct WsLayout {
  size_t rec, ksum, fcount, flist, qcount, forder, counters;  // forward part
  size_t bcount, blist, border, qorder, lse2, dsum;        // backward part
  size_t dqacc;                                            // fused backward: fp32 dQ accumulator
  size_t fwd_bytes, bwd_bytes;
};

inline size_t ws_align(size_t x) { return (x + 255) & ~size_t(255); }

// fp32 dQ accumulator of the fused backward, one 128-row tile per
// (batch, q-head, q-tile), laid out [B, Hq, nQt, d/4, 128, 4]: four
// consecutive columns of one row are 16 contiguous bytes, and the 128 rows of
// one 4-column chunk are contiguous, so one warp-wide 16-byte reduction of 32
// consecutive rows covers 512 contiguous bytes.
inline size_t dqacc_bytes(const Shape& s) { return (size_t)s.B * s.Hq * s.nQt * kTile * s.d * 4; }

inline WsLayout make_layout(const Shape& s) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = ws_align(off + bytes); return o; };
  const size_t bhm = (size_t)s.B * s.Hm;
  L.rec = take(bhm * s.nKt * kTile * 16);
  L.ksum = take(bhm * s.nKt * 8 * 4);
  L.fcount = take(bhm * s.nFB * 4);
  L.flist = take(bhm * s.nFB * s.nKt * 4);
  L.qcount = take(bhm * s.nFB * 2 * 4);
  L.forder = take((size_t)s.n_fwd_items * 4);
  L.counters = take(64);
  L.fwd_bytes = off;
  L.bcount = take(bhm * s.nKt * 4);
  L.blist = take(bhm * s.nKt * s.nQt * 4);
  L.border = take((size_t)s.n_kv_items * 4);
  L.qorder = take((size_t)s.n_q_items * 4);
  L.lse2 = take((size_t)s.B * s.Hq * s.nQt * kTile * 4);
  L.dsum = take((size_t)s.B * s.Hq * s.nQt * kTile * 4);
  L.dqacc = take(dqacc_bytes(s));
  L.bwd_bytes = off;
  return L;
}

struct ItemCoord {
  int b, hkv, t, hg;  // t = forward block, k-tile or q-tile; hg = q-head (pair) within the GQA group
};
__host__ __device__ __forceinline__ ItemCoord decode_fwd_item(const Shape& s, int i) {
  ItemCoord c;
  c.hg = i % s.fG; i /= s.fG;
  c.t = i % s.nFB; i /= s.nFB;
  c.hkv = i % s.Hkv; c.b = i / s.Hkv;
  return c;
}
__host__ __device__ __forceinline__ ItemCoord decode_kv_item_coord(const Shape& s, int i) {
  ItemCoord c;
  c.hg = 0;
  c.t = i % s.nKt; i /= s.nKt;
  c.hkv = i % s.Hkv; c.b = i / s.Hkv;
  return c;
}
__host__ __device__ __forceinline__ ItemCoord decode_q_item_coord(const Shape& s, int i) {
  ItemCoord c;
  c.hg = i % s.G; i /= s.G;
  c.t = i % s.nQt; i /= s.nQt;
  c.hkv = i % s.Hkv; c.b = i / s.Hkv;
  return c;
}

// ----------------------------------------------------------------------------
// kernel parameter blocks
// ----------------------------------------------------------------------------
struct MaskPrepParams {
  const int32_t *lts, *lte, *uts, *ute;  // [B, Hm, Nk]; a null pair = empty intervals
  int B, Hm, Nk, nKt;
  int Nq;        // checks build: mask values must lie in [0, Nq]
  int* status;   // checks build: where a bad value is recorded
  int4* rec;    // [B, Hm, nKt*128] {LTS, LTE, UTS, UTE}; padded columns hide every row
  int* ksum;    // [B, Hm, nKt, 8]
};

struct PlanParams {
  Shape s;
  const int* ksum;
  int* fcount; int* flist;   // forward lists  [B, Hm, nFB] / [B, Hm, nFB, nKt]
  int* qcount;               // per block slot non-skipped k-tiles [B, Hm, nFB*2]
  int* bcount; int* blist;   // backward lists [B, Hm, nKt] / [B, Hm, nKt, nQt]
  uint8_t* cls;              // optional export [B, Hm, nQt, nKt]
};

// Longest-first order of the work items, in waves of `wave` consecutive
// (batch, KV head) groups (0 = natural group-major order, no sorting).
struct SortParams {
  Shape s;
  int mode;               // 0: forward items, 1: key-side items, 2: query-side items
  const int* count;       // fcount, bcount or qcount
  int* order;             // out: item order
  int* counter;           // zeroed for the persistent kernel that follows
  int n_items;
  int items_per_group;
  int wave;
  int cost_cap;   // costs are clamped to [0, cost_cap]
  int n_buckets;  // > 0: counting sort over (wave, cost) buckets; 0: bitonic sort
};

// Partial attention results over disjoint key sets, merged per row.
constexpr int kMaxMergeParts = 16;
struct MergeParams {
  const __nv_bfloat16* o[kMaxMergeParts];  // [B, Nq, Hq, d]
  const float* lse[kMaxMergeParts];        // [B, Hq, Nq]
  int n, B, Nq, Hq, d;
  __nv_bfloat16* out_o;
  float* out_lse;
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
  float4* dqacc;   // fused backward: accumulator zeroed here (null: none)
  int64_t dqacc_vec4;
};

struct BwdParams {
  Shape s;
  float scale;
  float scale_log2;
  const int4* rec;
  // key side (dK, dV): per (b, hm, k-tile) q-tile lists, units (b, mu, k-tile)
  const int* blist;
  const int* bcount;
  const int* order;
  int* counter;
  int n_items;
  // query side (dQ): per (b, hm, q-block) k-tile lists, units (b, hm, q-block)
  const int* flist;
  const int* fcount;
  const int* qcount;    // [B, Hm, nQB*2]: non-skipped k-tiles per q-tile
  const int* forder;
  int* counter2;
  int n_items2;
  const float* lse2;
  const float* dsum;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dqacc;         // fused backward: [B, Hq, nQt, d/4, 128, 4] fp32, zeroed before the kernel
  int* status;
  uint64_t wait_limit_ns;
};

}  // namespace fm
