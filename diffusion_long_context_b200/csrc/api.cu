// Host-side plumbing shared by every entry point of libfocus.so: status strings, the
// per-thread last-error message, the launch counter and the device error word.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "focus_common.cuh"

namespace focus {

namespace {
thread_local char t_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};
__device__ int g_device_error_word = 0;
constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};
int g_sm_count[kMaxDevices] = {0};
std::mutex g_mutex;
// dynamic shared memory each kernel is configured for, per device ordinal
std::mutex g_attr_mutex;
std::map<std::pair<int, const void*>, int> g_smem_attr;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return (dev >= 0 && dev < kMaxDevices) ? dev : 0;
}
}  // namespace

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("FOCUS_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

void note_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

int device_sm_count() {
  const int dev = current_device();
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

cudaError_t ensure_dynamic_smem(const void* kernel, int bytes) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  const auto key = std::make_pair(dev, kernel);
  const auto it = g_smem_attr.find(key);
  if (it != g_smem_attr.end() && it->second >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_smem_attr[key] = bytes;
  return e;
}

int configure_dynamic_smem(const void* kernel, int bytes, const char* what) {
  const cudaError_t e = ensure_dynamic_smem(kernel, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    set_error("%s: setting %d bytes of dynamic shared memory: %s", what, bytes, cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

int* device_error_word() {
  const int dev = current_device();
  if (!g_err_ptr[dev]) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_err_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_error_word) == cudaSuccess) g_err_ptr[dev] = static_cast<int*>(p);
    }
  }
  return g_err_ptr[dev];
}

}  // namespace focus

extern "C" const char* focus_status_string(int status) {
  switch (status) {
    case FOCUS_OK: return "FOCUS_OK";
    case FOCUS_ERR_INVALID_ARG: return "FOCUS_ERR_INVALID_ARG";
    case FOCUS_ERR_UNSUPPORTED: return "FOCUS_ERR_UNSUPPORTED";
    case FOCUS_ERR_CUDA: return "FOCUS_ERR_CUDA";
    case FOCUS_ERR_CAPACITY: return "FOCUS_ERR_CAPACITY";
    case FOCUS_ERR_DEVICE_CHECK: return "FOCUS_ERR_DEVICE_CHECK";
    default: return "FOCUS_ERR_UNKNOWN";
  }
}

extern "C" const char* focus_last_error(void) { return focus::t_last_error; }

extern "C" uint64_t focus_launch_count(void) { return focus::g_launches.load(std::memory_order_relaxed); }

extern "C" int focus_device_error(int* code_out) {
  int* p = focus::device_error_word();
  if (!p) {
    focus::set_error("device error word unavailable");
    return FOCUS_ERR_CUDA;
  }
  int code = 0;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpy(&code, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    focus::set_error("reading the device error word failed: %s", cudaGetErrorString(cudaGetLastError()));
    return FOCUS_ERR_CUDA;
  }
  if (code_out) *code_out = code;
  if (code != 0) {
    const int zero = 0;
    cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    focus::set_error("device check failed with code %d", code);
    return FOCUS_ERR_DEVICE_CHECK;
  }
  return FOCUS_OK;
}
