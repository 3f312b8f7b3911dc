// Key sequence ("slots") of one (sequence, KV head) for the attention kernels.
//
// Dense: slot s is key s, s < L.
// Sparse (Focus-dLLM method steps (5): I_p = sinks U kept prompt blocks U current
// block, each key once): slots are laid out as
//   [ current block [g0, g1) ]             padded to gen_pad slots (a multiple of box_rows >= G)
//   [ kept block 0 | kept block 1 | ... ]  each padded to pad_bs = round_up(bs, 8)
//   [ sinks ]                              one slot per listed sink; sinks inside a kept
//                                          block or the current block, out-of-range and
//                                          repeated entries are dropped (invalid slots);
//                                          padded to a multiple of box_rows
// Padding slots are invalid (masked out of the softmax). Every box_rows-aligned group of
// slots inside the current block or a kept block is one contiguous run of keys and can be
// fetched by one TMA box; sink slots are fetched row by row. The sinks come last: with
// tiles claimed a ring's depth ahead of their use, the slow row-by-row gather is issued
// while earlier tiles are still being consumed, instead of holding up the first tile.
#pragma once

#include "focus_common.cuh"

namespace focus {

struct SlotLayout {
  int n_slots;      // total slots (keys + padding)
  int n_sinks;      // sink slots [sink_start, sink_start + n_sinks), one per listed sink
  int blk_start;    // first slot of the kept blocks (the current block starts at slot 0)
  int sink_start;   // first slot of the sinks
  int pad_bs;       // slots per kept block
  int nvb;          // kept blocks (valid entries of the block list)
  int last_size;    // valid keys of the last kept block (short when it ends at P)
  FastDiv pad_div;  // division by pad_bs for any slot offset below n_slots + 128
};

// One warp builds the layout of (b, h) from `pf` (layout_prefetch of the same lists): copies the kept-block list to s_blk (up to
// max_blocks entries) and the de-duplicated sinks to s_sinks (up to max_sinks). The block
// list has its valid entries first, ascending, then -1; sinks are ascending among valid
// entries. gen_pad = slots given to the current block, box_rows = rows per TMA box (a
// power of two dividing gen_pad and round_up(bs, 8)); pad_div divides by round_up(bs, 8)
// (exact below n_slots + 128), bs_div by bs (exact below L). Lane 0 writes *out; the
// layout is also returned to every lane of the warp.
// The first 64 block entries and 32 sinks, fetched together (one memory round trip) and
// early, before the caller's other set-up work.
struct LayoutPrefetch {
  int b0, b1, s0;
};
__device__ __forceinline__ LayoutPrefetch layout_prefetch(const int32_t* blk_g, int C, const int32_t* snk_g, int S) {
  const int lane = threadIdx.x & 31;
  LayoutPrefetch pf;
  pf.b0 = (lane < C) ? blk_g[lane] : -1;
  pf.b1 = (32 + lane < C) ? blk_g[32 + lane] : -1;
  pf.s0 = (lane < S) ? snk_g[lane] : -1;
  return pf;
}

// The block part of the layout of (b, h), built by one warp from `pf` (layout_prefetch of
// the same lists): copies the kept-block list to s_blk (up to max_blocks entries; valid
// entries first, ascending, then -1) and places the segments. The sink segment has a
// fixed size, n_sinks = min(S, max_sinks) slots rounded up to box_rows, so no slot
// position depends on which sinks survive de-duplication (dedupe_sinks). gen_pad = slots
// given to the current block, box_rows = rows per TMA box (a power of two dividing gen_pad
// and round_up(bs, 8)); pad_div divides by round_up(bs, 8) (exact below n_slots + 128).
// Lane 0 writes *out; the layout is also returned to every lane of the warp.
__device__ __forceinline__ SlotLayout build_block_layout(const LayoutPrefetch& pf, const int32_t* blk_g, int C, int S,
                                                         int P, int bs, int gen_pad, int box_rows,
                                                         const FastDiv& pad_div, int* s_blk, int max_blocks,
                                                         int max_sinks, SlotLayout* out) {
  const int lane = threadIdx.x & 31;
  int nvb = 0;
  for (int i0 = 0; i0 < C; i0 += 32) {
    const int i = i0 + lane;
    const int v = i0 == 0 ? pf.b0 : i0 == 32 ? pf.b1 : ((i < C) ? blk_g[i] : -1);
    const unsigned m = __ballot_sync(0xffffffffu, v >= 0);
    if (v >= 0 && i < max_blocks) s_blk[i] = v;
    nvb += __popc(m);
    if (m != 0xffffffffu) break;   // valid entries come first
  }
  nvb = min(nvb, max_blocks);
  __syncwarp();
  SlotLayout sl;
  sl.pad_bs = (bs + 7) & ~7;
  sl.nvb = nvb;
  sl.last_size = nvb > 0 ? min(bs, P - s_blk[nvb - 1] * bs) : bs;
  sl.n_sinks = min(S, max_sinks);
  sl.blk_start = gen_pad;
  sl.sink_start = sl.blk_start + nvb * sl.pad_bs;
  sl.n_slots = sl.sink_start + ((sl.n_sinks + box_rows - 1) & ~(box_rows - 1));
  sl.pad_div = pad_div;
  if (lane == 0) *out = sl;
  return sl;
}

// The same layout when the kept-block list is already in s_blk, complete and ascending
// with nvb valid entries first (the fused kernel's own top-C): no list walk, one load.
__device__ __forceinline__ SlotLayout fused_block_layout(const int* s_blk, int nvb, int S, int P, int bs,
                                                         int gen_pad, int box_rows, const FastDiv& pad_div,
                                                         int max_blocks, int max_sinks, SlotLayout* out) {
  const int lane = threadIdx.x & 31;
  nvb = min(max(nvb, 0), max_blocks);
  SlotLayout sl;
  sl.pad_bs = (bs + 7) & ~7;
  sl.nvb = nvb;
  sl.last_size = nvb > 0 ? min(bs, P - s_blk[nvb - 1] * bs) : bs;
  sl.n_sinks = min(S, max_sinks);
  sl.blk_start = gen_pad;
  sl.sink_start = sl.blk_start + nvb * sl.pad_bs;
  sl.n_slots = sl.sink_start + ((sl.n_sinks + box_rows - 1) & ~(box_rows - 1));
  sl.pad_div = pad_div;
  if (lane == 0) *out = sl;
  return sl;
}

// Sink slots of (b, h), by one warp after build_block_layout: s_sinks[i], i < sl.n_sinks
// (slot sink_start + i), is sink i, or -1 when it is dropped -- out of range, inside the
// current block [g0, g1), a repeat of the previous entry (the list is ascending among its
// valid entries) or inside a kept block. bs_div divides by bs (exact below L).
__device__ __forceinline__ void dedupe_sinks(const LayoutPrefetch& pf, const int32_t* snk_g, const SlotLayout& sl,
                                             int L, int P, int g0, int g1, const FastDiv& bs_div, const int* s_blk,
                                             int* s_sinks) {
  const int lane = threadIdx.x & 31;
  int prev_last = -1;
  for (int i0 = 0; i0 < sl.n_sinks; i0 += 32) {
    const int i = i0 + lane;
    const int j = i0 == 0 ? pf.s0 : ((i < sl.n_sinks) ? snk_g[i] : -1);
    const int jprev = __shfl_up_sync(0xffffffffu, j, 1);
    const int before = (lane == 0) ? prev_last : jprev;
    bool keep = (j >= 0) && (j < L) && !(j >= g0 && j < g1) && (j != before);
    if (keep && j < P) {
      const int jb = static_cast<int>(bs_div.div(static_cast<uint32_t>(j)));
      int lo = 0, hi = sl.nvb - 1;
      while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int v = s_blk[mid];
        if (v == jb) {
          keep = false;
          break;
        }
        if (v < jb) lo = mid + 1;
        else hi = mid - 1;
      }
    }
    if (i < sl.n_sinks) s_sinks[i] = keep ? j : -1;
    prev_last = __shfl_sync(0xffffffffu, j, 31);
  }
  __syncwarp();
}

// First key of the contiguous run starting at group slot gs (box-aligned), or -1 when the
// group lies in the sink segment or past the end (fetched row by row / zero-filled).
template <bool SPARSE>
__device__ __forceinline__ int group_key0(const SlotLayout& sl, const int* s_blk, int bs, int g0, int gs) {
  if (!SPARSE) return gs;
  if (gs >= sl.sink_start) return -1;
  if (gs < sl.blk_start) return g0 + gs;
  const int rel = gs - sl.blk_start;
  const int i = static_cast<int>(sl.pad_div.div(static_cast<uint32_t>(rel)));
  return s_blk[i] * bs + (rel - i * sl.pad_bs);
}

// Key of a sink-segment slot, or -1 for padding and dropped sinks.
__device__ __forceinline__ int sink_slot_key(const SlotLayout& sl, const int* s_sinks, int slot) {
  const int i = slot - sl.sink_start;
  return (i >= 0 && i < sl.n_sinks) ? s_sinks[i] : -1;
}

// Whether a slot holds a key of the set (not padding, not a dropped sink, not past the end).
template <bool SPARSE>
__device__ __forceinline__ bool slot_valid(const SlotLayout& sl, const int* s_sinks, int L, int bs, int G, int slot) {
  if (!SPARSE) return slot < L;
  if (slot < sl.blk_start) return slot < G;
  if (slot >= sl.sink_start) {
    const int i = slot - sl.sink_start;
    return i < sl.n_sinks && s_sinks[i] >= 0;
  }
  const int rel = slot - sl.blk_start;
  const int i = static_cast<int>(sl.pad_div.div(static_cast<uint32_t>(rel)));
  const int r = rel - i * sl.pad_bs;
  return r < ((i == sl.nvb - 1) ? sl.last_size : bs);
}

}  // namespace focus
