// Attention-sink identification.
//
// Focus-dLLM summary page, "核心方法" (core method) and "方法步骤详情" (method steps)
// step (3): the attention distribution of the dense sink layer, aggregated over the
// active queries (column sums produced by the dense attention call), picks the sinks;
// deeper sparse layers reuse them unchanged (cross-layer consistency, abstract).
// One CTA per (sequence, KV head): block-wide radix top-S over the L column sums.
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

}  // namespace focus

using namespace focus;

extern "C" int focus_sink_identify(const float* colsum, int B, int Hkv, int L, int S, int32_t* sinks, void* stream) {
  FOCUS_CHECK_ARG(colsum && sinks, "null pointer argument");
  FOCUS_CHECK_ARG(B >= 0 && Hkv >= 1 && L >= 1 && S >= 1 && S <= 4096, "bad sizes (L=%d S=%d)", L, S);
  if (B == 0) return FOCUS_OK;
  const size_t stage_bytes = static_cast<size_t>(L) * sizeof(float);
  const bool stage = stage_bytes <= kSinkStageMaxBytes && (reinterpret_cast<uintptr_t>(colsum) & 15u) == 0;
  cudaError_t e;
  if (stage) {
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(sink_topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSinkStageMaxBytes);
      cfg = true;
    }
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
