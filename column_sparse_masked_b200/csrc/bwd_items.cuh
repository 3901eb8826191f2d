// Work items of the key-stationary backward kernels (batch, KV head, 128-key
// tile) and the walk over their non-skipped q-tiles, shared by the split
// key-side kernel and the fused backward kernel.
#pragma once
#include <climits>

#include "common.cuh"

namespace fm {

// A decoded work item (batch, KV head, k-tile).  The first producer decodes
// each item once and publishes it in the shared-memory ring; the other roles
// read it there.  item >= n_items ends the work.
struct __align__(16) KvItem {
  int item, b, hkv, kt, total;  // total = q-tiles over all q-heads of the group
};

__device__ __forceinline__ KvItem decode_kv_item(const BwdParams& p, int item) {
  const Shape& sh = p.s;
  KvItem it{};
  it.item = item;
  if (item >= p.n_items) return it;
  const int unit = p.order[item];
  if (kChecks && (unit < 0 || unit >= p.n_items)) {
    atomicCAS(p.status, 0, kDevErrBounds);
    it.item = INT_MAX;  // ends the CTA's work
    return it;
  }
  const ItemCoord c = decode_kv_item_coord(sh, unit);
  it.b = c.b;
  it.hkv = c.hkv;
  it.kt = c.t;
  it.total = 0;
  for (int gi = 0; gi < sh.G; ++gi) {
    const int h = it.hkv * sh.G + gi;
    const int hm = (sh.Hm == 1) ? 0 : h;
    const size_t lrow = ((size_t)it.b * sh.Hm + hm) * sh.nKt + it.kt;
    const int cnt = p.bcount[lrow];
    if (kChecks) {  // the q-tile list: a count within [0, nQt], entries in range and not skipped
      bool bad = cnt < 0 || cnt > sh.nQt;
      for (int t = 0; !bad && t < cnt; ++t) {
        const int e = p.blist[lrow * sh.nQt + t];
        bad = (e >> 2) < 0 || (e >> 2) >= sh.nQt || (e & 3) == kClsSkip || (e & 3) > kClsFull;
      }
      if (bad) {
        atomicCAS(p.status, 0, kDevErrBounds);
        it.item = INT_MAX;
        return it;
      }
    }
    it.total += cnt;
  }
  return it;
}

// Calls f(j, h, hm, qt, cls) for the item's q-tiles in the order every role walks them.
template <typename F>
__device__ __forceinline__ bool for_each_qtile(const BwdParams& p, const KvItem& it, F&& f) {
  const Shape& sh = p.s;
  int j = 0;
  for (int gi = 0; gi < sh.G; ++gi) {
    const int h = it.hkv * sh.G + gi;
    const int hm = (sh.Hm == 1) ? 0 : h;
    const size_t lrow = ((size_t)it.b * sh.Hm + hm) * sh.nKt + it.kt;
    const int* list = p.blist + lrow * sh.nQt;
    const int cnt = p.bcount[lrow];
    for (int t = 0; t < cnt; ++t, ++j) {
      const int e = list[t];
      if (!f(j, h, hm, e >> 2, e & 3)) return false;
    }
  }
  return true;
}

}  // namespace fm
