// Allocation-free entry point: focus_sparse_attention with its split-KV scratch in a
// library-owned static device array instead of a caller-provided workspace.
//
// For callers that cannot call cudaMalloc (allocation forbidden while a stream is being
// captured, plugin enqueue paths, fixed up-front memory reservations). The kernels and
// the result are those of focus_sparse_attention.
#include <mutex>

#include "focus_common.cuh"

namespace focus {
namespace {

// The scratch itself. In host code `g_sparse_scratch` is only a host-side stand-in for the
// symbol; its device address comes from cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_sparse_scratch[FOCUS_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
void* g_scratch_dev_ptr[kMaxDev] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error("cudaGetDevice failed: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDev) {
    set_error("device ordinal %d out of range", dev);
    return FOCUS_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_dev_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sparse_scratch);
    if (e != cudaSuccess || !p) {
      set_error("cudaGetSymbolAddress of the scratch array failed: %s", cudaGetErrorString(e));
      return FOCUS_ERR_CUDA;
    }
    g_scratch_dev_ptr[dev] = p;
  }
  *out = g_scratch_dev_ptr[dev];
  return FOCUS_OK;
}

}  // namespace
}  // namespace focus

extern "C" int focus_sparse_attention_noalloc(const focus_bf16* Q_active, const int32_t* n_active,
                                              const focus_bf16* K, const focus_bf16* V, const int32_t* sinks, int S,
                                              const int32_t* blocks, int C, int bs, int P, int g0, int g1, int B,
                                              int Hq, int Hkv, int L, int d, int acap, float scale,
                                              focus_bf16* O_active, void* stream) {
  const size_t need = focus_sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1);
  if (need > FOCUS_NOALLOC_SCRATCH_BYTES) {
    focus::set_error("split-KV scratch of %zu bytes exceeds the %zu-byte static array", need,
                     static_cast<size_t>(FOCUS_NOALLOC_SCRATCH_BYTES));
    return FOCUS_ERR_CAPACITY;
  }
  void* ws = nullptr;
  const int st = focus::scratch_address(&ws);
  if (st != FOCUS_OK) return st;
  return focus_sparse_attention(Q_active, n_active, K, V, sinks, S, blocks, C, bs, P, g0, g1, B, Hq, Hkv, L, d, acap,
                                scale, O_active, ws, FOCUS_NOALLOC_SCRATCH_BYTES, stream);
}
