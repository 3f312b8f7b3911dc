// Attention-sink identification.
//
// Focus-dLLM summary page, "核心方法" (core method) and "方法步骤详情" (method steps)
// step (3): the attention distribution of the dense sink layer, aggregated over the
// active queries (column sums produced by the dense attention call), picks the sinks;
// deeper sparse layers reuse them unchanged (cross-layer consistency, abstract).
// Long rows: a cluster of CTAs per (sequence, KV head), each selecting the top-S of its
// share, then CTA 0 selecting among the candidates. Otherwise one CTA per (sequence, KV
// head): block-wide radix top-S over the L column sums (held in registers up to L = 32768,
// else staged in or read from memory).
#include "focus_common.cuh"
#include "topk.cuh"

namespace focus {

// The L column sums of (b, h) are staged in shared memory, as order keys, when they fit
// (STAGE = true); the block-wide radix selection then reads shared memory only.
template <bool STAGE>
__global__ void __launch_bounds__(1024) sink_topk_kernel(const float* __restrict__ colsum, int L, int S,
                                                         int32_t* __restrict__ sinks) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  extern __shared__ float s_row[];
  __shared__ TopkShared tk;
  const int bh = blockIdx.x;
  const float* row = colsum + static_cast<size_t>(bh) * L;
  int32_t* out = sinks + static_cast<size_t>(bh) * S;
  if (STAGE) {
    uint32_t* s_key = reinterpret_cast<uint32_t*>(s_row);
    if ((L & 3) == 0) {
      for (int i = threadIdx.x; i < L / 4; i += blockDim.x) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(row) + i);
        reinterpret_cast<uint4*>(s_key)[i] =
            make_uint4(float_order_key(v.x), float_order_key(v.y), float_order_key(v.z), float_order_key(v.w));
      }
    } else {
      for (int i = threadIdx.x; i < L; i += blockDim.x) s_key[i] = float_order_key(__ldg(row + i));
    }
    __syncthreads();
    block_topk_ascending([&](int i) { return s_key[i]; }, L, S, out, S, tk);
  } else {
    block_topk_ascending([&](int i) { return float_order_key(__ldg(row + i)); }, L, S, out, S, tk);
  }
}

constexpr int kSinkStageMaxBytes = 160 * 1024;
constexpr int kSinkThreads = 512;

// L <= KPT * 512: thread t holds the column sums of [KPT*t, KPT*t + KPT) in registers
// (16-byte loads when the row is 16-byte aligned) and the register top-k selects.
template <int KPT>
__global__ void __launch_bounds__(kSinkThreads) sink_topk_regs_kernel(const float* __restrict__ colsum, int L, int S,
                                                                      int32_t* __restrict__ sinks, int vec) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  __shared__ TopkShared tk;
  const int bh = blockIdx.x;
  const float* row = colsum + static_cast<size_t>(bh) * L;
  const int i0 = threadIdx.x * KPT;
  uint32_t key[KPT];
  if (vec && i0 + KPT <= L) {
#pragma unroll
    for (int j = 0; j < KPT / 4; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + i0) + j);
      key[4 * j] = float_order_key(v.x);
      key[4 * j + 1] = float_order_key(v.y);
      key[4 * j + 2] = float_order_key(v.z);
      key[4 * j + 3] = float_order_key(v.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) key[j] = (i0 + j < L) ? float_order_key(__ldg(row + i0 + j)) : 0u;
  }
  block_topk_small_regs<KPT>(key, L, S, sinks + static_cast<size_t>(bh) * S, S, tk);
}

// Cluster form for long rows: the cs CTAs of (b, h) each take a contiguous share of the L
// columns (chunk, a multiple of 4) and select its local top-S. The global top-S lies in
// the union of the local ones. Every CTA pushes its S candidates (order key, column) into
// CTA 0's shared memory over DSMEM, in rank order, so the candidate list is in ascending
// column order and a tie between candidates resolves to the lower column, as in one
// selection over the whole row. After a cluster barrier CTA 0 selects the top-S of the
// cs * S candidates.
template <int KPT>
__global__ void __launch_bounds__(kSinkThreads, 2) sink_topk_cluster_kernel(const float* __restrict__ colsum, int L,
                                                                         int S, int chunk,
                                                                         int32_t* __restrict__ sinks, int vec) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  extern __shared__ uint32_t s_dyn[];
  uint32_t* s_key = s_dyn;                                   // [chunk] order keys of this share
  int32_t* s_loc = reinterpret_cast<int32_t*>(s_dyn + chunk);    // [S] local selection
  uint32_t* s_ckey = s_dyn + chunk + S;                       // [cs * S] candidates (CTA 0)
  int32_t* s_cidx = reinterpret_cast<int32_t*>(s_ckey + static_cast<size_t>(gridDim.x) * S);
  int32_t* s_pos = s_cidx + static_cast<size_t>(gridDim.x) * S;  // [S] positions chosen by CTA 0
  int* s_priv = reinterpret_cast<int*>(s_pos + S);           // per-warp histograms
  int* s_wide = s_priv + 2 * (kSinkThreads / 32) * 257;      // [2048 + 64] 11-bit first-pass histogram
  __shared__ TopkShared tk;
  const int cs = gridDim.x, rank = blockIdx.x;
  const int bh = blockIdx.y;
  const int c0 = rank * chunk;
  const int n = min(chunk, L - c0);                          // >= S (host-checked)
  const float* row = colsum + static_cast<size_t>(bh) * L + c0;
  const int i0 = threadIdx.x * KPT;
  uint32_t key[KPT];
  if (vec && i0 + KPT <= n) {
#pragma unroll
    for (int j = 0; j < KPT / 4; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + i0) + j);
      key[4 * j] = float_order_key(v.x);
      key[4 * j + 1] = float_order_key(v.y);
      key[4 * j + 2] = float_order_key(v.z);
      key[4 * j + 3] = float_order_key(v.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) key[j] = (i0 + j < n) ? float_order_key(__ldg(row + i0 + j)) : 0u;
  }
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    if (i0 + j < n) s_key[i0 + j] = key[j];
  block_topk_small_regs<KPT>(key, n, S, s_loc, S, tk, s_priv, s_wide);
  __syncthreads();
  const uint32_t ck0 = smem_u32(s_ckey), ci0 = smem_u32(s_cidx);
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const int c = s_loc[i];
    const uint32_t slot = static_cast<uint32_t>(rank * S + i) * 4u;
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(dsmem_addr(ck0 + slot, 0)), "r"(s_key[c]) : "memory");
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(dsmem_addr(ci0 + slot, 0)), "r"(c0 + c) : "memory");
  }
  cluster_sync();                // every candidate is in CTA 0
  if (rank != 0) return;
  const int nc = cs * S;
  auto ckey = [&](int i) { return s_ckey[i]; };
  if (nc <= kSinkThreads) block_topk_small<1>(ckey, nc, S, s_pos, S, tk, s_wide);
  else if (nc <= 2 * kSinkThreads) block_topk_small<2>(ckey, nc, S, s_pos, S, tk, s_wide);
  else block_topk_small<4>(ckey, nc, S, s_pos, S, tk, s_wide);
  __syncthreads();
  int32_t* out = sinks + static_cast<size_t>(bh) * S;
  for (int i = threadIdx.x; i < S; i += blockDim.x) out[i] = s_cidx[s_pos[i]];
}

}  // namespace focus

using namespace focus;

extern "C" int focus_sink_identify(const float* colsum, int B, int Hkv, int L, int S, int32_t* sinks, void* stream) {
  FOCUS_CHECK_ARG(colsum && sinks, "null pointer argument");
  FOCUS_CHECK_ARG(B >= 0 && Hkv >= 1 && L >= 1 && S >= 1 && S <= 4096, "bad sizes (L=%d S=%d)", L, S);
  if (B == 0) return FOCUS_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // cluster form: cs CTAs per (b, h) while two CTAs per SM cover the grid and every share
  // holds at least S columns and at most 16 per thread
  int cs = 1;
  while (cs < 8 && B * Hkv * cs * 2 <= 2 * device_sm_count() && L >= cs * 2 * S && cs * 2 * S <= 4 * kSinkThreads)
    cs *= 2;
  if (cs > 1 && (L + cs - 1) / cs <= 16 * kSinkThreads) {
    const int chunk = ((L + cs - 1) / cs + 3) & ~3;
    if (L - (cs - 1) * chunk >= S) {
      const int vec = ((reinterpret_cast<uintptr_t>(colsum) & 15u) == 0 && (L & 3) == 0) ? 1 : 0;
      const size_t smem =
          (static_cast<size_t>(chunk) + S + 2 * static_cast<size_t>(cs) * S + S + 2 * (kSinkThreads / 32) * 257 +
           2048 + 64) * 4;
      cudaError_t e;
      if (chunk <= 8 * kSinkThreads) {
        auto kern = sink_topk_cluster_kernel<8>;
        if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(kern), 200 * 1024, "sink top-S"))
          return st_attr;
        e = launch_k_cluster(kern, dim3(cs, B * Hkv), dim3(kSinkThreads), smem, st, cs, colsum, L, S, chunk, sinks,
                             vec);
      } else {
        auto kern = sink_topk_cluster_kernel<16>;
        if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(kern), 200 * 1024, "sink top-S"))
          return st_attr;
        e = launch_k_cluster(kern, dim3(cs, B * Hkv), dim3(kSinkThreads), smem, st, cs, colsum, L, S, chunk, sinks,
                             vec);
      }
      note_launch();
      if (e != cudaSuccess) {
        set_error("sink top-S launch: %s", cudaGetErrorString(e));
        return FOCUS_ERR_CUDA;
      }
      return FOCUS_OK;
    }
  }
  if (L <= 64 * kSinkThreads) {
    // 16-byte loads need every row 16-byte aligned: the base and L * 4 bytes
    const int vec = ((reinterpret_cast<uintptr_t>(colsum) & 15u) == 0 && (L & 3) == 0) ? 1 : 0;
    cudaError_t e;
    if (L <= 8 * kSinkThreads)
      e = launch_k(sink_topk_regs_kernel<8>, dim3(B * Hkv), dim3(kSinkThreads), 0, st, colsum, L, S, sinks, vec);
    else if (L <= 16 * kSinkThreads)
      e = launch_k(sink_topk_regs_kernel<16>, dim3(B * Hkv), dim3(kSinkThreads), 0, st, colsum, L, S, sinks, vec);
    else if (L <= 32 * kSinkThreads)
      e = launch_k(sink_topk_regs_kernel<32>, dim3(B * Hkv), dim3(kSinkThreads), 0, st, colsum, L, S, sinks, vec);
    else
      e = launch_k(sink_topk_regs_kernel<64>, dim3(B * Hkv), dim3(kSinkThreads), 0, st, colsum, L, S, sinks, vec);
    note_launch();
    if (e != cudaSuccess) {
      set_error("sink top-S launch: %s", cudaGetErrorString(e));
      return FOCUS_ERR_CUDA;
    }
    return FOCUS_OK;
  }
  const size_t stage_bytes = static_cast<size_t>(L) * sizeof(float);
  const bool stage = stage_bytes <= kSinkStageMaxBytes && (reinterpret_cast<uintptr_t>(colsum) & 15u) == 0;
  cudaError_t e;
  if (stage) {
    if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(sink_topk_kernel<true>),
                                                   kSinkStageMaxBytes, "sink top-S"))
      return st_attr;
    e = launch_k(sink_topk_kernel<true>, dim3(B * Hkv), dim3(1024), stage_bytes, static_cast<cudaStream_t>(stream),
                 colsum, L, S, sinks);
  } else {
    e = launch_k(sink_topk_kernel<false>, dim3(B * Hkv), dim3(1024), 0, static_cast<cudaStream_t>(stream), colsum, L,
                 S, sinks);
  }
  note_launch();
  if (e != cudaSuccess) {
    set_error("sink top-S launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}
