// Key sequence ("slots") of one (sequence, KV head) for the attention kernels.
//
// Dense: slot s is key s, s < L.
// Sparse (Focus-dLLM method steps (5): I_p = sinks U kept prompt blocks U current
// block, each key once): slots are laid out as
//   [ kept block 0 | kept block 1 | ... ]  each padded to pad_bs = round_up(bs, 8)
//   [ current block [g0, g1) ]             padded to gen_pad slots (a multiple of 8 >= G)
//   [ de-duplicated sinks ]                sinks inside a kept block or the current
//                                          block, out-of-range and repeated entries dropped
// Padding slots are invalid (masked out of the softmax). Every box_rows-aligned group of
// slots inside a block or the current block is one contiguous run of keys and can be
// fetched by one TMA box; sink slots are fetched row by row.
#pragma once

#include "focus_common.cuh"

namespace focus {

struct SlotLayout {
  int n_slots;      // total slots (keys + padding)
  int gen_start;    // first slot of the current block
  int sink_start;   // first slot of the sink segment
  int pad_bs;       // slots per kept block
  int nvb;          // kept blocks (valid entries of the block list)
  int last_size;    // valid keys of the last kept block (short when it ends at P)
  int n_fsinks;     // sinks that remain after de-duplication
  FastDiv pad_div;  // division by pad_bs for any slot below n_slots + 128
};

// One warp builds the layout of (b, h): copies the kept-block list to s_blk (up to
// max_blocks entries) and the de-duplicated sinks to s_sinks (up to max_sinks). The block
// list has its valid entries first, ascending, then -1; sinks are ascending among valid
// entries. gen_pad = slots given to the current block. Lane 0 writes *out; the layout is
// also returned to every lane of the warp.
__device__ __forceinline__ SlotLayout build_sparse_layout(const int32_t* blk_g, int C, const int32_t* snk_g, int S,
                                                          int L, int P, int bs, int g0, int g1, int gen_pad, int* s_blk,
                                                          int max_blocks, int* s_sinks, int max_sinks,
                                                          SlotLayout* out) {
  const int lane = threadIdx.x & 31;
  // the first 64 block entries and 32 sinks are fetched together (one memory round trip)
  const int pre_b0 = (lane < C) ? blk_g[lane] : -1;
  const int pre_b1 = (32 + lane < C) ? blk_g[32 + lane] : -1;
  const int pre_s0 = (lane < S) ? snk_g[lane] : -1;
  int nvb = 0;
  for (int i0 = 0; i0 < C; i0 += 32) {
    const int i = i0 + lane;
    const int v = i0 == 0 ? pre_b0 : i0 == 32 ? pre_b1 : ((i < C) ? blk_g[i] : -1);
    const unsigned m = __ballot_sync(0xffffffffu, v >= 0);
    if (v >= 0 && i < max_blocks) s_blk[i] = v;
    nvb += __popc(m);
    if (m != 0xffffffffu) break;   // valid entries come first
  }
  nvb = min(nvb, max_blocks);
  __syncwarp();
  int last_size = bs;
  if (nvb > 0) last_size = min(bs, P - s_blk[nvb - 1] * bs);
  int nf = 0, prev_last = -1;
  for (int i0 = 0; i0 < S; i0 += 32) {
    const int i = i0 + lane;
    const int j = i0 == 0 ? pre_s0 : ((i < S) ? snk_g[i] : -1);
    const int jprev = __shfl_up_sync(0xffffffffu, j, 1);
    const int before = (lane == 0) ? prev_last : jprev;
    bool keep = (j >= 0) && (j < L) && !(j >= g0 && j < g1) && (j != before);
    if (keep && j < P) {
      const int jb = j / bs;
      int lo = 0, hi = nvb - 1;
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
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    const int pos = nf + __popc(m & ((1u << lane) - 1u));
    if (keep && pos < max_sinks) s_sinks[pos] = j;
    nf += __popc(m);
    prev_last = __shfl_sync(0xffffffffu, j, 31);
  }
  SlotLayout sl;
  sl.pad_bs = (bs + 7) & ~7;
  sl.nvb = nvb;
  sl.last_size = last_size;
  sl.gen_start = nvb * sl.pad_bs;
  sl.sink_start = sl.gen_start + gen_pad;
  sl.n_fsinks = min(nf, max_sinks);
  sl.n_slots = sl.sink_start + sl.n_fsinks;
  sl.pad_div.init(static_cast<uint32_t>(sl.pad_bs), static_cast<uint32_t>(sl.n_slots + 128));
  if (lane == 0) *out = sl;
  return sl;
}

// First key of the contiguous run starting at group slot gs (box-aligned), or -1 when the
// group lies in the sink segment / past the end (fetched row by row).
template <bool SPARSE>
__device__ __forceinline__ int group_key0(const SlotLayout& sl, const int* s_blk, int bs, int g0, int gs) {
  if (!SPARSE) return gs;
  if (gs < sl.gen_start) {
    const int i = static_cast<int>(sl.pad_div.div(static_cast<uint32_t>(gs)));
    return s_blk[i] * bs + (gs - i * sl.pad_bs);
  }
  if (gs < sl.sink_start) return g0 + (gs - sl.gen_start);
  return -1;
}

// Key of a sink-segment slot, or -1 past the end.
__device__ __forceinline__ int sink_slot_key(const SlotLayout& sl, const int* s_sinks, int slot) {
  return (slot >= sl.sink_start && slot < sl.n_slots) ? s_sinks[slot - sl.sink_start] : -1;
}

// Whether a slot holds a key of the set (not padding, not past the end).
template <bool SPARSE>
__device__ __forceinline__ bool slot_valid(const SlotLayout& sl, int L, int bs, int G, int slot) {
  if (!SPARSE) return slot < L;
  if (slot < sl.gen_start) {
    const int i = static_cast<int>(sl.pad_div.div(static_cast<uint32_t>(slot)));
    const int r = slot - i * sl.pad_bs;
    return r < ((i == sl.nvb - 1) ? sl.last_size : bs);
  }
  if (slot < sl.sink_start) return (slot - sl.gen_start) < G;
  return slot < sl.n_slots;
}

}  // namespace focus
