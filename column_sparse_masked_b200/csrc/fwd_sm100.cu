// Mask-aware attention forward for sm_100a.
//
// "FlashMask-3 targets masked distributed attention on Hopper GPUs", In-depth
// insight: attention forward driven by the column-wise mask, skipping tiles
// that the boundary vectors prove fully masked and applying the element mask
// only on partially masked tiles.  The page's kernel is a Hopper design
// (TMA/WGMMA with three warp roles); this one is written for Blackwell:
//
//   * persistent CTAs (one per SM) take work items -- (batch, q-head, block of
//     two 128-row q-tiles), or, when two q-heads share a KV head and the mask,
//     (batch, pair of q-heads, one q-tile), so that both halves see exactly
//     the same key tiles -- from a locality-aware longest-first order through
//     an atomic counter; the producer warp hands each item to the other roles
//     through a ring of mbarriers, so consecutive items overlap (the next
//     item's Q load and first QK^T run while the softmax warps write O);
//   * warp 8 issues TMA loads: Q once per item, and K(0), V(0), K(1), V(1), ...
//     through one ring of tile-sized slots; a K slot is released after the
//     second q-tile's QK^T, a V slot after its P V, so V tiles are requested
//     about two key steps before they are used;
//   * warp 9 issues tcgen05 MMAs: S_g = Q_g K^T into TMEM, O_g += P_g V with
//     P_g read from TMEM (bf16, written over S_g), ping-pong between the two
//     q-tiles: S0 S1 | PV0 S0' PV1 S1' | ...;
//   * warps 0-3 and 4-7 are the softmax groups of q-tiles 0 and 1: one thread
//     per query row; online softmax in the exp2 domain with the scale folded
//     into one FMA per element, O rescaled in TMEM
//     only when a row maximum grows by more than 2^8.
//
// The element mask of a partial tile is built per key column: each lane reads
// the boundary records of 4 columns (L2-resident), turns them into 32-bit words
// over its warp's 32 rows (interval arithmetic), and a 5-step shuffle transpose
// of each 32x32 bit block hands every row its mask bits.  This runs before the
// wait for S, off the softmax critical path.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 after O0.
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "launchers.h"
#include "sm100_primitives.cuh"

namespace fm {

template <int D>
struct FwdCfg {
  static constexpr int kSlots = (D == 128) ? 5 : 10;  // K/V ring slots of one tile each
  static constexpr int kTileBytes = kTile * D * 2;  // one 128-row bf16 tile
  static constexpr int kBoxes = D / 64;             // 64-column (128-byte) TMA boxes per tile
  static constexpr int kThreads = 320;
  static constexpr int kProducerWarp = 8;
  static constexpr int kMmaWarp = 9;
  static constexpr int kRing = 4;
};

// A decoded work item.  The producer decodes each item once (three dependent
// global reads) and publishes it in the shared-memory ring; the other roles
// read it from there.  item = INT_MAX ends the work.
struct __align__(16) FwdItem {
  int item, b, h, hm, hkv, qb, n, e0;  // e0: first entry of the item's tile list
  __device__ __forceinline__ const int* list(const FwdParams& p) const {
    const Shape& sh = p.s;
    return p.flist + (((size_t)b * sh.Hm + hm) * sh.nFB + qb) * sh.nKt;
  }
  // first query row and q-head of half g: two q-tiles of head h, or (paired
  // q-heads) one q-tile of heads h and h + 1
  __device__ __forceinline__ int row0(const Shape& sh, int g) const {
    return sh.fpair ? qb * kTile : qb * 2 * kTile + g * kTile;
  }
  __device__ __forceinline__ int head(const Shape& sh, int g) const { return sh.fpair ? h + g : h; }
};

__device__ __forceinline__ FwdItem decode_fwd(const FwdParams& p, int item) {
  const Shape& sh = p.s;
  FwdItem it{};
  it.item = item;
  if (item >= p.n_items) return it;
  const int unit = p.order[item];
  if (kChecks && (unit < 0 || unit >= p.n_items)) {
    atomicCAS(p.status, 0, kDevErrBounds);
    it.item = INT_MAX;  // ends the CTA's work
    return it;
  }
  const ItemCoord c = decode_fwd_item(sh, unit);
  it.b = c.b;
  it.qb = c.t;
  it.hkv = c.hkv;
  it.h = c.hkv * sh.G + (sh.fpair ? 2 * c.hg : c.hg);
  it.hm = (sh.Hm == 1) ? 0 : it.h;  // paired q-heads share mask head 0
  const size_t lrow = ((size_t)it.b * sh.Hm + it.hm) * sh.nFB + it.qb;
  it.n = p.fcount[lrow];
  if (kChecks) {  // the k-tile list: a count within [0, nKt], entries in range
    bool bad = it.n < 0 || it.n > sh.nKt;
    for (int t = 0; !bad && t < it.n; ++t) {
      const int e = p.flist[lrow * sh.nKt + t];
      bad = (e >> 8) < 0 || (e >> 8) >= sh.nKt || (e & 3) > kClsFull || ((e >> 2) & 3) > kClsFull;
    }
    if (bad) {
      atomicCAS(p.status, 0, kDevErrBounds);
      it.item = INT_MAX;
      return it;
    }
  }
  it.e0 = it.n > 0 ? p.flist[lrow * sh.nKt] : 0;
  return it;
}

template <int D>
struct __align__(1024) FwdSmem {
  uint8_t q[2][FwdCfg<D>::kTileBytes];
  uint8_t slot[FwdCfg<D>::kSlots][FwdCfg<D>::kTileBytes];  // K(t) in ring position 2t, V(t) in 2t+1
  FwdItem ring[FwdCfg<D>::kRing];
  uint64_t ring_full[FwdCfg<D>::kRing], ring_empty[FwdCfg<D>::kRing];
  uint64_t q_full, q_empty;
  uint64_t slot_full[FwdCfg<D>::kSlots];
  uint64_t slot_empty[FwdCfg<D>::kSlots];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_free[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
  int no_abort;
};

static_assert(sizeof(FwdSmem<128>) <= 232448, "forward shared memory exceeds the per-CTA limit");
static_assert(sizeof(FwdSmem<64>) <= 232448, "forward shared memory exceeds the per-CTA limit");

// S = Q K^T: M = 128 rows, N = 128 keys, K = D; both operands K-major SW128.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, const uint8_t* qs, const uint8_t* ks) {
  constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
  const uint32_t qa = smem_addr(qs), ka = smem_addr(ks);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_ss(d_tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V: M = 128 rows, N = D, K = 128 keys.  P from TMEM (bf16 pairs,
// 8 columns per 16 keys); V is MN-major (d contiguous) SW128.
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, const uint8_t* vs, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
  const uint32_t va = smem_addr(vs);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(va + kk * 2048, 16384, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::kThreads, 1)
    fm_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int kSlots = Cfg::kSlots;
  constexpr int kRing = Cfg::kRing;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  FwdSmem<D>& s = *reinterpret_cast<FwdSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Shape& sh = p.s;

  if (smem_addr(smem_raw) & 1023u) {  // SW128 operands need 1024-byte alignment
    if (tid == 0) atomicCAS(p.status, 0, -5);
    return;
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&s.ring_full[i], 1);
      mbar_init(&s.ring_empty[i], 9);  // MMA lane 0 + lane 0 of the 8 softmax warps
    }
    mbar_init(&s.q_full, 1);
    mbar_init(&s.q_empty, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&s.slot_full[i], 1);
      mbar_init(&s.slot_empty[i], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s.s_full[g], 1);
      mbar_init(&s.p_full[g], 128);
      mbar_init(&s.o_full[g], 1);
      mbar_init(&s.o_free[g], 128);
    }
    mbar_init(&s.teardown, 1);
    s.abort_flag = 0;
    s.no_abort = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::kProducerWarp && lane == 0) {
    tma_prefetch_map(&tq);
    tma_prefetch_map(&tk);
    tma_prefetch_map(&tv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the lists, orders and records of the planning kernels
  const uint32_t tmem = s.tmem_base;
  const WaitCtx w{&s.abort_flag, p.status, p.wait_limit_ns, smem_addr(smem_raw), 0};
  uint32_t q_par = 0, q_armed = 0, slot_par = 0, slot_armed = 0;  // producer: copies that may be in flight

  if (warp == Cfg::kProducerWarp) {
    if (lane == 0) {
      uint32_t pos = 0, act = 0, k = 0;  // pos: ring position of the next K/V tile
      bool ok = true;
      // Items are taken one ahead: while one item's tiles stream, the next
      // item's Q is prefetched into L2, so its load (which may only start
      // once the current item's last QK^T has been issued) hits L2.
      auto take = [&](FwdItem& out) -> bool {
        const int slot = k % kRing;
        if (!mbar_wait(&s.ring_empty[slot], ((k / kRing) & 1) ^ 1, w)) return false;
        const int item = s.abort_flag ? INT_MAX : atomicAdd(p.counter, 1);
        out = decode_fwd(p, item);
        s.ring[slot] = out;
        mbar_arrive(&s.ring_full[slot]);
        ++k;
        if (out.item < p.n_items && out.n > 0) {
#pragma unroll
          for (int g = 0; g < 2; ++g)
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx)
              tma_prefetch_l2_4d(&tq, bx * 64, out.head(sh, g), out.row0(sh, g), out.b);
        }
        return true;
      };
      FwdItem nxt{};
      ok = take(nxt);
      while (ok && nxt.item < p.n_items) {
        const FwdItem it = nxt;
        if (!(ok = take(nxt))) break;
        if (it.n == 0) continue;
        const int* list = it.list(p);
        if (!(ok = mbar_wait(&s.q_empty, (act & 1) ^ 1, w))) break;
        mbar_arrive_expect_tx(&s.q_full, 2 * Cfg::kTileBytes);
        q_par = act & 1;
        q_armed = 1;
#pragma unroll
        for (int g = 0; g < 2; ++g)
#pragma unroll
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_4d(s.q[g] + bx * 16384, &tq, &s.q_full, bx * 64, it.head(sh, g), it.row0(sh, g), it.b);
        ++act;
        for (int t = 0; t < it.n && ok; ++t) {
          const int kt = (t == 0 ? it.e0 : list[t]) >> 8;
#pragma unroll
          for (int kv = 0; kv < 2; ++kv, ++pos) {  // K(t), then V(t)
            const int sl = pos % kSlots;
            const uint32_t ph = (pos / kSlots) & 1;
            if (!(ok = mbar_wait(&s.slot_empty[sl], ph ^ 1, w))) break;
            mbar_arrive_expect_tx(&s.slot_full[sl], Cfg::kTileBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx)
              tma_load_4d(s.slot[sl] + bx * 16384, kv ? &tv : &tk, &s.slot_full[sl], bx * 64, it.hkv, kt * kTile, it.b);
            slot_par = (slot_par & ~(1u << sl)) | (ph << sl);
            slot_armed |= 1u << sl;
          }
        }
      }
    }
  } else if (warp == Cfg::kMmaWarp) {
    if (lane == 0) {
      uint32_t pos = 0, tile_cnt = 0, act = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int slot = k % kRing;
        if (!(ok = mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w))) break;
        const FwdItem it = s.ring[slot];
        mbar_arrive(&s.ring_empty[slot]);
        if (it.item >= p.n_items) break;
        const int n = it.n;
        if (n == 0) continue;
        if (!(ok = mbar_wait(&s.q_full, act & 1, w))) break;
        tc_fence_after();
        for (int t = 0; t < n; ++t, pos += 2) {
          // ring slots of K(t+1) and V(t)
          const int sv = (pos + 1) % kSlots;
          const uint32_t pv_ph = ((pos + 1) / kSlots) & 1;
          const int sk2 = (pos + 2) % kSlots;
          const uint32_t k2_ph = ((pos + 2) / kSlots) & 1;
          if (t == 0) {
            const int sk = pos % kSlots;
            if (!(ok = mbar_wait(&s.slot_full[sk], (pos / kSlots) & 1, w))) break;
            tc_fence_after();
            issue_qk<D>(tmem + 0, s.q[0], s.slot[sk]);
            mma_commit(&s.s_full[0]);
            issue_qk<D>(tmem + 128, s.q[1], s.slot[sk]);
            mma_commit(&s.s_full[1]);
            mma_commit(&s.slot_empty[sk]);
            if (n == 1) mma_commit(&s.q_empty);
          }
          if (!(ok = mbar_wait(&s.slot_full[sv], pv_ph, w) && mbar_wait(&s.p_full[0], tile_cnt & 1, w))) break;
          if (t == 0 && !(ok = mbar_wait(&s.o_free[0], (act & 1) ^ 1, w))) break;  // previous O0 read out
          tc_fence_after();
          issue_pv<D>(tmem + 256, tmem + 0, s.slot[sv], t > 0);
          if (t == n - 1) mma_commit(&s.o_full[0]);
          if (t + 1 < n) {
            if (!(ok = mbar_wait(&s.slot_full[sk2], k2_ph, w))) break;
            tc_fence_after();
            issue_qk<D>(tmem + 0, s.q[0], s.slot[sk2]);
            mma_commit(&s.s_full[0]);
          }
          if (!(ok = mbar_wait(&s.p_full[1], tile_cnt & 1, w))) break;
          if (t == 0 && !(ok = mbar_wait(&s.o_free[1], (act & 1) ^ 1, w))) break;
          tc_fence_after();
          issue_pv<D>(tmem + 256 + D, tmem + 128, s.slot[sv], t > 0);
          if (t == n - 1) mma_commit(&s.o_full[1]);
          mma_commit(&s.slot_empty[sv]);
          if (t + 1 < n) {
            issue_qk<D>(tmem + 128, s.q[1], s.slot[sk2]);
            mma_commit(&s.s_full[1]);
            mma_commit(&s.slot_empty[sk2]);
            if (t + 2 == n) mma_commit(&s.q_empty);  // last QK^T of the item issued
          }
          ++tile_cnt;
        }
        if (!ok) break;
        ++act;
      }
    }
  } else {
    // ---------------- softmax groups: thread = query row ----------------
    const int g = warp >> 2, wq = warp & 3;
    const uint32_t tb = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_col = g * 128, o_col = 256 + g * D;
    const float sl2 = p.scale_log2;
    // O rows go out as 32-byte stores when the output allows it (rows are
    // Hq * D * 2 bytes apart, a multiple of 32).
    const bool o_v8 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
    uint32_t tile_cnt = 0, act = 0, k = 0;
    bool ok = true;
    // The item loop is software-pipelined: the next item is taken from the
    // ring and decoded (dependent global reads) before this item's epilogue.
    FwdItem it{};
    it.item = INT_MAX;
    if ((ok = __all_sync(0xffffffffu, mbar_wait(&s.ring_full[0], 0, w)))) it = s.ring[0];
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&s.ring_empty[0]);
    k = 1;
    int e = it.e0;
    while (ok && it.item < p.n_items) {
      const int n = it.n;
      const int* list = it.list(p);
      const int rbase = it.row0(sh, g) + wq * 32;  // first row of this warp
      const int row = rbase + lane;
      const int4* recs = p.rec + ((size_t)it.b * sh.Hm + it.hm) * sh.nKt * kTile;
      float m_run = -INFINITY, l_run = 0.f;  // m_run in scaled log2 units
      for (int t = 0; t < n; ++t) {
        const int e_next = (t + 1 < n) ? list[t + 1] : 0;  // in flight during this tile
        const int cls = (e >> (2 * g)) & 3;
        const bool need = (cls != kClsFull) || ((e >> 4) & 1);
        uint32_t mw[4] = {0u, 0u, 0u, 0u};
        if (need) {
          // column words (this lane's 4 columns) -> row words by transposition
          const int4* mrec = recs + (size_t)(e >> 8) * kTile;
          int4 r4[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) r4[c] = __ldg(mrec + c * 32 + lane);
#pragma unroll
          for (int c = 0; c < 4; ++c) mw[c] = warp_transpose32(column_row_bits(r4[c], rbase), lane);
        }
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[g], tile_cnt & 1, w)))) break;
        tc_fence_after();
        float x[128];
        uint32_t* raw = reinterpret_cast<uint32_t*>(x);
        tmem_ld32x(tb + s_col + 0, raw + 0);
        tmem_ld32x(tb + s_col + 32, raw + 32);
        tmem_ld32x(tb + s_col + 64, raw + 64);
        tmem_ld32x(tb + s_col + 96, raw + 96);
        tmem_ld_wait();
        if (need) {
#pragma unroll
          for (int i = 0; i < 128; ++i) x[i] = ((mw[i >> 5] >> (i & 31)) & 1u) ? -INFINITY : x[i];
        }
        // row maximum of the raw logits (the scale is positive)
        float m4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) m4[j] = max3f(x[j], x[4 + j], x[8 + j]);
#pragma unroll
        for (int i = 12; i + 7 < 128; i += 8)
#pragma unroll
          for (int j = 0; j < 4; ++j) m4[j] = max3f(m4[j], x[i + j], x[i + 4 + j]);
        m4[0] = max3f(m4[0], x[124], x[125]);
        m4[1] = max3f(m4[1], x[126], x[127]);
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
        // Lazy rescale: only when the maximum grows by more than 8 (log2 units).
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m_run + 8.f) {
          alpha = fast_exp2(m_run - mx);  // 0 when m_run = -inf
          rescale = (m_run != -INFINITY);
          m_run = mx;
          l_run *= alpha;
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 32 columns -> 16 packed bf16 pairs per store
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = fast_exp2(fmaf(x[c * 32 + 2 * i], sl2, neg_m));
            const float a1 = fast_exp2(fmaf(x[c * 32 + 2 * i + 1], sl2, neg_m));
            sa += a0;
            sb += a1;
            pk[i] = pack_bf16x2(a0, a1);
          }
          tmem_st16(tb + s_col + c * 16, pk);
        }
        l_run += sa + sb;
        // O correction (the previous P V of this q-tile has completed: the
        // commit that signalled this S was issued after it).
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32x(tb + o_col + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32x(tb + o_col + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.p_full[g]);
        ++tile_cnt;
        e = e_next;
      }
      if (!ok) break;
      // next item: take it from the ring and decode it now
      const FwdItem cur = it;
      {
        const int slot = k % kRing;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.ring_full[slot], (k / kRing) & 1, w)))) break;
        it = s.ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.ring_empty[slot]);
        ++k;
        e = it.e0;
      }
      // ---------------- epilogue of the current item ----------------
      if (n > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&s.o_full[g], act & 1, w)))) break;
      tc_fence_after();
      const bool valid = row < sh.Nq;
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const int hg_out = cur.head(sh, g);
      __nv_bfloat16* orow = p.o + (((size_t)cur.b * sh.Nq + (valid ? row : 0)) * sh.Hq + hg_out) * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o[64];
        if (n > 0) {
          tmem_ld32x(tb + o_col + c * 64, o);
          tmem_ld32x(tb + o_col + c * 64 + 32, o + 32);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] = 0u;
        }
        uint32_t pkd[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          pkd[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (valid) {
          if (o_v8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) st_global_v8_na(orow + c * 64 + i * 16, pkd + 8 * i);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) st_global_v4_na(orow + c * 64 + i * 8, pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2], pkd[4 * i + 3]);
          }
        }
      }
      if (n > 0) {
        tc_fence_before();
        mbar_arrive(&s.o_free[g]);
        ++act;
      }
      if (valid)
        p.lse[((size_t)cur.b * sh.Hq + hg_out) * sh.Nq + row] =
            (l_run > 0.f) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (s.abort_flag) {
    // Let copies and MMAs that are still in flight land before the CTA's
    // shared memory and tensor memory are released.
    const WaitCtx w2{&s.no_abort, p.status, p.wait_limit_ns, smem_addr(smem_raw), 0};
    if (warp == Cfg::kMmaWarp && lane == 0) {
      mma_commit(&s.teardown);
      (void)mbar_wait(&s.teardown, 0, w2);
    }
    if (warp == Cfg::kProducerWarp && lane == 0) {
      if (q_armed) (void)mbar_wait(&s.q_full, q_par, w2);
      for (int sl = 0; sl < kSlots; ++sl)
        if (slot_armed & (1u << sl)) (void)mbar_wait(&s.slot_full[sl], (slot_par >> sl) & 1, w2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_fwd_d(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, int grid, cudaStream_t st) {
  const int smem = (int)sizeof(FwdSmem<D>);
  cudaError_t e = ensure_smem_limit((const void*)fm_fwd_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int prof = profile_begin(0, st);
  const cudaError_t le = launch_after(fm_fwd_kernel<D>, dim3(grid), dim3(FwdCfg<D>::kThreads), smem, st, tq, tk, tv, p);
  profile_end(prof, st);
  return le;
}

cudaError_t launch_fwd(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       int grid, cudaStream_t st) {
  if (p.s.d == 128) return launch_fwd_d<128>(p, tq, tk, tv, grid, st);
  return launch_fwd_d<64>(p, tq, tk, tv, grid, st);
}

}  // namespace fm
