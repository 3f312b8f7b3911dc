// Block-wide top-k selection shared by the block (top-C) and sink (top-S) kernels.
//
// Order: larger key first, ties to the lower index. Keys are order-preserving 32-bit
// images of the scores (float_order_key), so -0.0 and +0.0 tie. Two forms:
//   block_topk_small (n <= KPT * blockDim.x): keys in registers, offset by the block
//     minimum; the first 8-bit radix digit is the top of the spanned range, so smooth
//     scores spread over the 256 bins and one or two passes usually fix the k-th key.
//     One packed (greater, equal) block scan then places the selection in index order.
//   block_topk_ascending (any n): keys read through key_of each pass.
//     1. Radix select, 8 bits per pass (at most 4 passes), finds T = the k-th largest key
//        and how many keys equal to T are taken. Histograms use warp-aggregated shared
//        atomics; one warp locates the digit with a lane-parallel suffix scan. A pass
//        whose boundary digit is taken whole ends the search early.
//     2. Ordered selection: each warp owns a contiguous segment of indices; a first walk
//        counts keys > T and == T per warp, one block barrier turns the counts into
//        offsets, and a second walk writes the selected indices in ascending order.
#pragma once

#include "focus_common.cuh"

namespace focus {

// Per-warp values in shared memory (one int per warp, at most 32 warps), combined by one
// warp in parallel: lane w reads entry w and a warp reduction finishes. A serial loop over
// the entries costs one shared-memory round trip per entry.
__device__ __forceinline__ int warp_sum_first(const int* arr, int upto) {
  const int lane = threadIdx.x & 31;
  return __reduce_add_sync(0xffffffffu, lane < upto ? arr[lane] : 0);
}
__device__ __forceinline__ uint32_t warp_min_of(const int* arr, int n) {
  const int lane = threadIdx.x & 31;
  return __reduce_min_sync(0xffffffffu, lane < n ? static_cast<uint32_t>(arr[lane]) : 0xFFFFFFFFu);
}
__device__ __forceinline__ uint32_t warp_max_of(const int* arr, int n) {
  const int lane = threadIdx.x & 31;
  return __reduce_max_sync(0xffffffffu, lane < n ? static_cast<uint32_t>(arr[lane]) : 0u);
}

// Exclusive prefix sum of a 0/1 flag over the CTA in thread order; also returns the total.
// Every thread of the CTA must call it (it synchronises the CTA).
__device__ __forceinline__ int block_excl_scan(bool flag, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) s_warp[warp] = __popc(m);
  __syncthreads();
  const int before = warp_sum_first(s_warp, warp);
  total = warp_sum_first(s_warp, nwarps);
  __syncthreads();
  return before + in_warp;
}

struct TopkShared {
  int hist[256];
  int hist2[256];          // second histogram (block_topk_small alternates the two)
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
  const int gt_before = warp_sum_first(sm.w_gt, warp), eq_before = warp_sum_first(sm.w_eq, warp);
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

// Top-k for small n (n <= KPT * blockDim.x): same contract and order as
// block_topk_ascending. Thread t holds the keys of indices [KPT*t, KPT*t + KPT) in
// registers. The keys are first offset by the block minimum, and the first radix digit is
// the top 8 bits of the range actually spanned (max - min), so a smooth score
// distribution spreads over all 256 bins and one or two passes usually find the k-th key.
// The two histograms alternate, so each pass needs two block barriers. The ordered
// output comes from one block scan of per-thread (greater, equal) counts packed in one
// word (n < 65536).
// key[j] holds the key of index KPT * threadIdx.x + j (any value when that index >= n).
// key[j] holds the key of index KPT * threadIdx.x + j (any value when that index >= n);
// the array is overwritten.
// priv (optional): 2 * (blockDim.x / 32) * 257 ints of shared memory for per-warp
// histograms (padded so that the warps' copies of a bin sit in different banks); with it
// a bin holding most of the keys costs no cross-warp atomic serialisation.
// wide (optional): 2048 + 64 ints of shared memory. With it the first pass takes 11 bits
// (a 2048-bin histogram and its 64-bin coarse sums, searched coarse then fine), which for
// a few hundred smooth keys almost always isolates the k-th key in one pass.
template <int KPT>
__device__ void block_topk_small_regs(uint32_t (&key)[KPT], int n, int k, int32_t* out, int cap,
                                      TopkShared& sm, int* priv = nullptr, int* wide = nullptr) {
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
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (tid * KPT + j < n) {
      kmin = min(kmin, key[j]);
      kmax = max(kmax, key[j]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    sm.w_gt[warp] = static_cast<int>(kmin);
    sm.w_eq[warp] = static_cast<int>(kmax);
  }
  for (int i = tid; i < 256; i += nt) sm.hist[i] = 0;
  if (priv)
    for (int i = tid; i < nwarps * 257; i += nt) priv[i] = 0;
  if (wide)
    for (int i = tid; i < 2048 + 64; i += nt) wide[i] = 0;
  __syncthreads();
  kmin = warp_min_of(sm.w_gt, nwarps);
  kmax = warp_max_of(sm.w_eq, nwarps);
  // relative keys rk = key - kmin in [0, range] (in place); fixed part: rk >> hi == P
  const uint32_t range = kmax - kmin;
#pragma unroll
  for (int j = 0; j < KPT; ++j) key[j] -= kmin;
  int hi = 32 - __clz(range);          // bits spanned (0 when every key is equal)
  uint32_t P = 0u;
  int remaining = k;
  int buf = 0;
  bool whole = (range == 0u);          // all keys equal: take the lowest indices
  auto warp_incl_scan = [&](int v) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    return v;
  };
  if (wide && hi >= 11 && !whole) {
    int* fine = wide;
    int* coarse = wide + 2048;
    const int lo = hi - 11;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      if (tid * KPT + j < n) {
        const uint32_t f = (key[j] >> lo) & 2047u;
        atomicAdd(&fine[f], 1);
        atomicAdd(&coarse[f >> 5], 1);
      }
    }
    __syncthreads();
    // coarse digit: lane l owns coarse bins 63-2l, 62-2l (descending)
    const int ca = coarse[63 - 2 * lane], cb = coarse[62 - 2 * lane];
    const int incl = warp_incl_scan(ca + cb);
    const int excl = incl - (ca + cb);
    const int L = __ffs(__ballot_sync(0xffffffffu, incl >= remaining)) - 1;
    const bool first = excl + ca >= remaining;
    const int cd = __shfl_sync(0xffffffffu, first ? 63 - 2 * lane : 62 - 2 * lane, L);
    remaining -= __shfl_sync(0xffffffffu, first ? excl : excl + ca, L);
    // fine digit inside coarse bin cd: lane l owns fine bin cd*32 + 31 - l
    const int cf = fine[cd * 32 + 31 - lane];
    const int incl2 = warp_incl_scan(cf);
    const int L2 = __ffs(__ballot_sync(0xffffffffu, incl2 >= remaining)) - 1;
    const int cnt = __shfl_sync(0xffffffffu, cf, L2);
    remaining -= __shfl_sync(0xffffffffu, incl2 - cf, L2);
    whole = (cnt == remaining);
    P = static_cast<uint32_t>(cd * 32 + 31 - L2);
    hi = lo;
  }
  while (hi > 0 && !whole) {
    const int lo = max(0, hi - 8);
    int* hist = buf ? sm.hist2 : sm.hist;
    int* other = buf ? sm.hist : sm.hist2;
    int* whist = hist;                   // where this warp counts
    if (priv) {
      int* pcur = priv + buf * nwarps * 257;
      int* poth = priv + (buf ^ 1) * nwarps * 257;
      for (int i = tid; i < nwarps * 257; i += nt) poth[i] = 0;   // cleared for the next pass
      whist = pcur + warp * 257;
    } else {
      for (int i = tid; i < 256; i += nt) other[i] = 0;           // cleared for the next pass
    }
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const int i = tid * KPT + j;
      const uint32_t rk = key[j];
      if (i < n && (hi >= 32 || (rk >> hi) == P)) atomicAdd(&whist[(rk >> lo) & ((1u << (hi - lo)) - 1u)], 1);
    }
    __syncthreads();
    if (priv) {
      const int* pcur = priv + buf * nwarps * 257;
      for (int b = tid; b < 256; b += nt) {
        int tot = 0;
        for (int w = 0; w < nwarps; ++w) tot += pcur[w * 257 + b];
        hist[b] = tot;
      }
      __syncthreads();
    }
    // every warp locates the digit holding the remaining-th largest candidate (no extra
    // barrier: each warp reaches the same answer from the same counts). Lane l owns
    // digits 255-8l .. 248-8l in descending order.
    {
      int c[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) c[jj] = hist[255 - 8 * lane - jj];
      int pre[8];
      pre[0] = c[0];
#pragma unroll
      for (int jj = 1; jj < 8; ++jj) pre[jj] = pre[jj - 1] + c[jj];
      const int own = pre[7];
      int incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - own;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= remaining);
      const int L = __ffs(hit) - 1;
      // in lane L: the first jj with excl + pre[jj] >= remaining (branch-free)
      int jsel = 0;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) jsel += (excl + pre[jj] < remaining) ? 1 : 0;
      int before = excl, cnt = 0;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        before += (jj < jsel) ? c[jj] : 0;
        cnt = (jj == jsel) ? c[jj] : cnt;
      }
      const int digit = __shfl_sync(0xffffffffu, 255 - 8 * lane - jsel, L);
      cnt = __shfl_sync(0xffffffffu, cnt, L);
      remaining -= __shfl_sync(0xffffffffu, before, L);
      whole = (cnt == remaining);
      P = (P << (hi - lo)) | static_cast<uint32_t>(digit);
      hi = lo;
    }
    buf ^= 1;
    __syncthreads();                   // this pass's histogram is read before it is cleared again
  }
  // keys above the threshold: (rk >> hi) > P; at the threshold: == P (hi = 0 after a
  // full search; every key when all are equal, P = 0)
  const int take_eq = remaining;
  int gt = 0, eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int i = tid * KPT + j;
    const uint32_t v = (hi >= 32) ? 0u : (key[j] >> hi);
    gt += (i < n && v > P) ? 1 : 0;
    eq += (i < n && v == P) ? 1 : 0;
  }
  // exclusive block scan of (gt | eq << 16) in thread order == index order
  const int packed = gt | (eq << 16);
  int incl = packed;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) sm.s_warp[warp] = incl;
  __syncthreads();
  const int before = incl - packed + warp_sum_first(sm.s_warp, warp);
  int gtb = before & 0xFFFF, eqb = before >> 16;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int i = tid * KPT + j;
    const uint32_t v = (hi >= 32) ? 0u : (key[j] >> hi);
    const bool is_gt = i < n && v > P;
    const bool is_eq = i < n && v == P;
    const bool sel = is_gt || (is_eq && eqb < take_eq);
    const int pos = gtb + min(eqb, take_eq);
    if (sel && pos < cap) out[pos] = i;
    gtb += is_gt ? 1 : 0;
    eqb += is_eq ? 1 : 0;
  }
  for (int i = k + tid; i < cap; i += nt) out[i] = -1;
}

template <int KPT, typename KeyFn>
__device__ void block_topk_small(KeyFn key_of, int n, int k, int32_t* out, int cap, TopkShared& sm,
                                 int* wide = nullptr) {
  uint32_t key[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int i = threadIdx.x * KPT + j;
    key[j] = i < n ? key_of(i) : 0u;
  }
  block_topk_small_regs<KPT>(key, n, k, out, cap, sm, nullptr, wide);
}

// Top-k of float order keys (float_order_key) over the whole CTA, two keys per thread:
// the k largest of s_keys[0 .. n), n <= 2 * blockDim.x, with the same result as
// block_topk_small_regs (ties at the threshold go to the lowest indices; out[0 .. k)
// ascending, -1 in out[k .. cap)). blockDim.x must be a multiple of 32 and at least 256;
// s_keys must be readable (8-byte aligned) up to 2 * blockDim.x entries. Every thread of
// the CTA calls it; out is complete after the caller's next CTA barrier.
// The first pass counts the keys in 2048 bins LINEAR in the scores' value between their
// minimum and maximum. The bin is a monotone function of the value, so every key of a
// higher bin is strictly larger; where the bin that holds the threshold holds exactly
// the keys still wanted (the common case: evenly spread scores leave one or two keys in
// that bin), the selection is settled by this one pass. Otherwise the keys of that bin
// are ranked exactly by 8-bit radix passes over their order keys relative to the bin's
// smallest key. Prefix counts use ballots and per-warp totals, so the whole selection
// costs five CTA barriers when the first pass settles it.
// fine: 2048 ints of shared memory (16-byte aligned).
template <bool FLOAT_IN = false>
__device__ void cta_topk_linear(const uint32_t* s_keys, int n, int k, int32_t* out, int cap, int* fine,
                                TopkShared& sm) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  k = min(k, n);
  if (k <= 0 || k >= n) {
    for (int i = tid; i < cap; i += nt) out[i] = (i < k) ? i : -1;
    return;
  }
  // ---- keys, minimum and maximum; the histogram is cleared meanwhile
  const int i0 = 2 * tid;
  const uint2 kv = reinterpret_cast<const uint2*>(s_keys)[tid];
  uint32_t key0 = kv.x, key1 = kv.y;
  if (FLOAT_IN) {
    key0 = float_order_key(__uint_as_float(key0));
    key1 = float_order_key(__uint_as_float(key1));
  }
  const bool p0 = i0 < n, p1 = i0 + 1 < n;
  uint32_t kmin = min(p0 ? key0 : 0xFFFFFFFFu, p1 ? key1 : 0xFFFFFFFFu);
  uint32_t kmax = max(p0 ? key0 : 0u, p1 ? key1 : 0u);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    sm.w_gt[warp] = static_cast<int>(kmin);
    sm.w_eq[warp] = static_cast<int>(kmax);
  }
  for (int i = tid; i < 2048 / 4; i += nt) reinterpret_cast<int4*>(fine)[i] = make_int4(0, 0, 0, 0);
  __syncthreads();
  kmin = warp_min_of(sm.w_gt, nw);
  kmax = warp_max_of(sm.w_eq, nw);
  // ---- linear value bins (bin 0 for every key when the span is zero or not finite)
  const float vmin = order_key_to_float(kmin);
  const float vspan = order_key_to_float(kmax) - vmin;
  const float scale = (vspan > 0.f && vspan <= 3.0e38f) ? 2048.f / vspan : 0.f;
  auto bin_of = [&](uint32_t key) {
    return static_cast<int>(fminf((order_key_to_float(key) - vmin) * scale, 2047.f));
  };
  const int b0 = p0 ? bin_of(key0) : -1, b1 = p1 ? bin_of(key1) : -1;
  if (p0) atomicAdd(&fine[b0], 1);
  if (p1) atomicAdd(&fine[b1], 1);
  __syncthreads();
  // ---- the bin holding the k-th largest: thread u < 256 owns bins 2047 - 8u .. 2040 - 8u
  {
    int c[8];
    if (tid < 256) {
      const int4 hq = reinterpret_cast<const int4*>(fine)[511 - 2 * tid];
      const int4 lq = reinterpret_cast<const int4*>(fine)[510 - 2 * tid];
      c[0] = hq.w; c[1] = hq.z; c[2] = hq.y; c[3] = hq.x;
      c[4] = lq.w; c[5] = lq.z; c[6] = lq.y; c[7] = lq.x;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) c[j] = 0;
    }
    const int own = ((c[0] + c[1]) + (c[2] + c[3])) + ((c[4] + c[5]) + (c[6] + c[7]));
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) sm.s_warp[warp] = incl;
    __syncthreads();
    incl += warp_sum_first(sm.s_warp, warp);
    const int excl = incl - own;
    if (excl < k && incl >= k) {       // exactly one thread
      int rem = k - excl, pb = 2047 - 8 * tid, cnt = c[0];
#pragma unroll
      for (int j = 0; j < 7; ++j) {
        if (rem <= cnt) break;
        rem -= cnt;
        --pb;
        cnt = c[j + 1];
      }
      sm.prefix = static_cast<uint32_t>(pb);
      sm.remaining = rem;
      sm.mask = static_cast<uint32_t>(cnt);
    }
    __syncthreads();
  }
  const int pb = static_cast<int>(sm.prefix);
  int remaining = sm.remaining;
  bool whole = static_cast<int>(sm.mask) == remaining;
  // ---- exact ranking inside bin pb (hi = 32: no prefix; there the keys of bin pb all tie)
  int hi = 32;
  uint32_t P = 0u, cmin = 0u;
  const bool refine = !whole;
  if (refine) {
    const bool c0 = b0 == pb, c1 = b1 == pb;
    uint32_t lmin = min(c0 ? key0 : 0xFFFFFFFFu, c1 ? key1 : 0xFFFFFFFFu);
    uint32_t lmax = max(c0 ? key0 : 0u, c1 ? key1 : 0u);
    lmin = __reduce_min_sync(0xffffffffu, lmin);
    lmax = __reduce_max_sync(0xffffffffu, lmax);
    if (lane == 0) {
      sm.w_gt[warp] = static_cast<int>(lmin);
      sm.w_eq[warp] = static_cast<int>(lmax);
    }
    __syncthreads();
    cmin = warp_min_of(sm.w_gt, nw);
    const uint32_t cmax = warp_max_of(sm.w_eq, nw);
    hi = 32 - __clz(cmax - cmin);      // 0: the candidates are equal, lowest indices win
    while (hi > 0 && !whole) {
      const int lo = max(0, hi - 8);
      __syncthreads();                 // the previous pass's histogram has been read
      for (int i = tid; i < 256; i += nt) sm.hist[i] = 0;
      __syncthreads();
      const uint32_t r0 = key0 - cmin, r1 = key1 - cmin;
      const uint32_t dmask = (1u << (hi - lo)) - 1u;
      if (c0 && (hi >= 32 || (r0 >> hi) == P)) atomicAdd(&sm.hist[(r0 >> lo) & dmask], 1);
      if (c1 && (hi >= 32 || (r1 >> hi) == P)) atomicAdd(&sm.hist[(r1 >> lo) & dmask], 1);
      __syncthreads();
      // every warp finds the same digit; lane l owns digits 255 - 8l .. 248 - 8l
      int c[8], pre[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) c[jj] = sm.hist[255 - 8 * lane - jj];
      pre[0] = c[0];
#pragma unroll
      for (int jj = 1; jj < 8; ++jj) pre[jj] = pre[jj - 1] + c[jj];
      int incl = pre[7];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      const int excl = incl - pre[7];
      const int L = __ffs(__ballot_sync(0xffffffffu, incl >= remaining)) - 1;
      int jsel = 0;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) jsel += (excl + pre[jj] < remaining) ? 1 : 0;
      int before = excl, cnt = 0;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        before += (jj < jsel) ? c[jj] : 0;
        cnt = (jj == jsel) ? c[jj] : cnt;
      }
      const int digit = __shfl_sync(0xffffffffu, 255 - 8 * lane - jsel, L);
      cnt = __shfl_sync(0xffffffffu, cnt, L);
      remaining -= __shfl_sync(0xffffffffu, before, L);
      whole = (cnt == remaining);
      P = (P << (hi - lo)) | static_cast<uint32_t>(digit);
      hi = lo;
    }
  }
  // ---- output: selected = bin > pb, or bin == pb with prefix > P, or the first `remaining`
  // keys (in index order) of bin pb with prefix == P; positions from ballots
  const int take_eq = remaining;
  auto classify = [&](uint32_t key, int b, bool& g, bool& e) {
    const uint32_t v = (hi >= 32) ? 0u : ((key - cmin) >> hi);
    g = b > pb || (b == pb && v > P);
    e = b == pb && v == P;
  };
  bool g0, e0, g1, e1;
  classify(key0, b0, g0, e0);
  classify(key1, b1, g1, e1);
  const unsigned G0 = __ballot_sync(0xffffffffu, g0), G1 = __ballot_sync(0xffffffffu, g1);
  const unsigned E0 = __ballot_sync(0xffffffffu, e0), E1 = __ballot_sync(0xffffffffu, e1);
  if (refine) __syncthreads();         // every thread has read the refinement's per-warp values
  if (lane == 0) {
    sm.w_gt[warp] = __popc(G0) + __popc(G1);
    sm.w_eq[warp] = __popc(E0) + __popc(E1);
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  int gtb = __popc(G0 & lt) + __popc(G1 & lt) + warp_sum_first(sm.w_gt, warp);
  int eqb = __popc(E0 & lt) + __popc(E1 & lt) + warp_sum_first(sm.w_eq, warp);
  if (g0 || (e0 && eqb < take_eq)) {
    const int pos = gtb + min(eqb, take_eq);
    if (pos < cap) out[pos] = i0;
  }
  gtb += g0 ? 1 : 0;
  eqb += e0 ? 1 : 0;
  if (g1 || (e1 && eqb < take_eq)) {
    const int pos = gtb + min(eqb, take_eq);
    if (pos < cap) out[pos] = i0 + 1;
  }
  for (int i = k + tid; i < cap; i += nt) out[i] = -1;
}

}  // namespace focus
