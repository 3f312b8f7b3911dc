// Block-wide top-k selection shared by the block (top-C) and sink (top-S) kernels.
//
// Order: larger key first, ties to the lower index. Keys are order-preserving 32-bit
// images of the scores (float_order_key), so -0.0 and +0.0 tie.
//   1. Radix select, 8 bits per pass (at most 4 passes), finds T = the k-th largest key
//      and how many keys equal to T are taken. A pass whose boundary digit is taken
//      whole ends the search early: T is then a prefix, compared under its mask. Histograms use warp-aggregated shared atomics
//      (lanes with the same digit add once), so a digit shared by every key does not
//      serialise the CTA; one warp locates the digit with a lane-parallel suffix scan.
//   2. Ordered selection: each warp owns a contiguous segment of indices; a first walk
//      counts keys > T and == T per warp, one block barrier turns the counts into
//      offsets, and a second walk writes the selected indices in ascending order.
#pragma once

#include "focus_common.cuh"

namespace focus {

// Exclusive prefix sum of a 0/1 flag over the CTA in thread order; also returns the total.
// Every thread of the CTA must call it (it synchronises the CTA).
__device__ __forceinline__ int block_excl_scan(bool flag, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) s_warp[warp] = __popc(m);
  __syncthreads();
  int before = 0;
  total = 0;
  for (int w = 0; w < nwarps; ++w) {
    const int c = s_warp[w];
    if (w < warp) before += c;
    total += c;
  }
  __syncthreads();
  return before + in_warp;
}

struct TopkShared {
  int hist[256];
  int s_warp[32];
  int w_gt[32];
  int w_eq[32];
  uint32_t prefix;
  uint32_t mask;           // bits of prefix that are fixed
  int remaining;
};

// key_of(i) -> uint32 key for i in [0, n). Writes out[0 .. min(k, n)) ascending and -1 into
// out[min(k, n) .. cap). Every thread of the CTA (a multiple of 32 threads) must call it.
template <typename KeyFn>
__device__ void block_topk_ascending(KeyFn key_of, int n, int k, int32_t* out, int cap, TopkShared& sm) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
  k = min(k, n);
  if (k <= 0) {
    for (int i = tid; i < cap; i += nt) out[i] = -1;
    return;
  }
  if (k >= n) {
    for (int i = tid; i < cap; i += nt) out[i] = (i < n) ? i : -1;
    return;
  }
  if (tid == 0) {
    sm.prefix = 0u;
    sm.mask = 0u;
    sm.remaining = k;
  }
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = tid; i < 256; i += nt) sm.hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for (int base = 0; base < n; base += nt) {
      const int i = base + tid;
      uint32_t bin = 256u;                       // no digit: outside the candidate set
      if (i < n) {
        const uint32_t key = key_of(i);
        if ((key & hi_mask) == prefix) bin = (key >> shift) & 255u;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending); find the digit holding the
      // remaining-th largest candidate
      int c[8], own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sm.hist[255 - 8 * lane - j];
        own += c[j];
      }
      int incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int rem = sm.remaining;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= rem);
      const int L = __ffs(hit) - 1;              // always found: the counts add up to >= rem
      if (lane == L) {
        int cum = incl - own;
        int digit = 0;
        int whole = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + c[j] >= rem) {
            digit = 255 - 8 * lane - j;
            whole = c[j];
            break;
          }
          cum += c[j];
        }
        sm.remaining = rem - cum;
        sm.prefix = prefix | (static_cast<uint32_t>(digit) << shift);
        // the digit's keys are all taken: no lower bit can change the selection
        sm.mask = (whole == rem - cum) ? (0xFFFFFFFFu << shift) : 0u;
      }
    }
    __syncthreads();
    if (sm.mask != 0u) break;
  }
  const uint32_t T = sm.prefix;
  const uint32_t M = sm.mask != 0u ? sm.mask : 0xFFFFFFFFu;   // a full search fixes every bit
  const int take_eq = sm.remaining;              // keys equal to T (under M) to keep, lowest indices first
  // ordered selection over warp-owned contiguous segments
  const int seg = ((n + nwarps - 1) / nwarps + 31) & ~31;
  const int w_begin = min(n, warp * seg), w_end = min(n, w_begin + seg);
  int gt = 0, eq = 0;
  for (int base = w_begin; base < w_end; base += 32) {
    const int i = base + lane;
    uint32_t key = 0u;
    if (i < w_end) key = key_of(i) & M;
    gt += __popc(__ballot_sync(0xffffffffu, i < w_end && key > T));
    eq += __popc(__ballot_sync(0xffffffffu, i < w_end && key == T));
  }
  if (lane == 0) {
    sm.w_gt[warp] = gt;
    sm.w_eq[warp] = eq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += sm.w_gt[w];
    eq_before += sm.w_eq[w];
  }
  int run_eq = eq_before;
  int run_sel = gt_before + min(eq_before, take_eq);
  const unsigned lt = (1u << lane) - 1u;
  for (int base = w_begin; base < w_end; base += 32) {
    const int i = base + lane;
    uint32_t key = 0u;
    if (i < w_end) key = key_of(i) & M;
    const bool is_gt = i < w_end && key > T;
    const bool is_eq = i < w_end && key == T;
    const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = is_gt || (is_eq && run_eq + __popc(meq & lt) < take_eq);
    const unsigned msel = __ballot_sync(0xffffffffu, sel);
    const int pos = run_sel + __popc(msel & lt);
    if (sel && pos < cap) out[pos] = i;
    run_eq += __popc(meq);
    run_sel += __popc(msel);
  }
  for (int i = k + tid; i < cap; i += nt) out[i] = -1;
}

}  // namespace focus
