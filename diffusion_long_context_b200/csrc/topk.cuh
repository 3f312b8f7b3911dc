// Block-wide top-k selection shared by the block (top-C) and sink (top-S) kernels.
//
// Order: larger key first, ties to the lower index. Keys are order-preserving 32-bit
// images of the scores (float_order_key), so -0.0 and +0.0 tie. An 8-bit radix select
// (four histogram passes) finds the k-th largest key T; one ordered pass then keeps
// every key > T and the lowest-index keys == T, writing the indices in ascending order.
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
  uint32_t prefix;
  int remaining;
};

// key_of(i) -> uint32 key for i in [0, n). Writes out[0 .. min(k, n)) ascending and -1 into
// out[min(k, n) .. cap). Every thread of the CTA must call it.
template <typename KeyFn>
__device__ void block_topk_ascending(KeyFn key_of, int n, int k, int32_t* out, int cap, TopkShared& sm) {
  const int tid = threadIdx.x, nt = blockDim.x;
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
    sm.remaining = k;
  }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = tid; i < 256; i += nt) sm.hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for (int i = tid; i < n; i += nt) {
      const uint32_t key = key_of(i);
      if ((key & hi_mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid == 0) {
      int cum = 0, rem = sm.remaining, sel = 0;
      for (int bin = 255; bin >= 0; --bin) {
        const int h = sm.hist[bin];
        if (cum + h >= rem) {
          sel = bin;
          break;
        }
        cum += h;
      }
      sm.remaining = rem - cum;
      sm.prefix = prefix | (static_cast<uint32_t>(sel) << shift);
    }
    __syncthreads();
  }
  const uint32_t T = sm.prefix;
  const int take_eq = sm.remaining;   // keys equal to T to keep (lowest indices first)
  int run_eq = 0, run_sel = 0;
  for (int base = 0; base < n; base += nt) {
    const int i = base + tid;
    const uint32_t key = (i < n) ? key_of(i) : 0u;
    const bool gt = (i < n) && key > T;
    const bool eq = (i < n) && key == T;
    int eq_total = 0, sel_total = 0;
    const int eq_pos = run_eq + block_excl_scan(eq, sm.s_warp, eq_total);
    const bool sel = gt || (eq && eq_pos < take_eq);
    const int pos = run_sel + block_excl_scan(sel, sm.s_warp, sel_total);
    if (sel && pos < cap) out[pos] = i;
    run_eq += eq_total;
    run_sel += sel_total;
  }
  for (int i = k + tid; i < cap; i += nt) out[i] = -1;
}

}  // namespace focus
