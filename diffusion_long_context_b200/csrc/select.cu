// Past Confidence-Guided Indicator (PCGI) + window expansion, and the active-row gather.
//
// Focus-dLLM summary page, "方法步骤详情" (method steps), steps (1) and (2): the top-k
// still-[MASK] positions of the current block by the previous step's confidence,
// k = floor(rho * n(t)), each widened to a window of size w; the union is I_active.
//
// One CTA per sequence, one thread per position of the current block (G <= 1024).
// Rank of a candidate = number of candidates ahead of it in (conf desc, index asc)
// order, so the top-k set needs no sort; both lists are compacted in position order
// with warp ballots and a block-level prefix sum.
#include "focus_common.cuh"
#include "topk.cuh"

namespace focus {

__global__ void select_queries_kernel(const float* __restrict__ conf, const uint8_t* __restrict__ mask, int L,
                                      int g0, int G, int k_req, int w, int32_t* __restrict__ i_focus,
                                      int32_t* __restrict__ n_focus, int kcap, int32_t* __restrict__ i_active,
                                      int32_t* __restrict__ n_active, int acap) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  __shared__ float s_conf[1024];
  __shared__ uint8_t s_cand[1024];
  __shared__ uint8_t s_sel[1024];
  __shared__ int s_warp[32];
  const int b = blockIdx.x, t = threadIdx.x;
  bool cand = false;
  float c = 0.f;
  if (t < G) {
    cand = mask[static_cast<size_t>(b) * L + g0 + t] != 0;
    c = conf[static_cast<size_t>(b) * G + t];
  }
  s_conf[t] = c;
  s_cand[t] = cand ? 1 : 0;
  const int n_cand = __syncthreads_count(cand);
  const int k = min(k_req, n_cand);
  int rank = 0;
  if (cand) {
    for (int j = 0; j < G; ++j) {
      if (!s_cand[j]) continue;
      const float cj = s_conf[j];
      rank += (cj > c) || (cj == c && j < t);   // -0.0 == +0.0 under IEEE comparison
    }
  }
  const bool sel = cand && rank < k;
  s_sel[t] = sel ? 1 : 0;
  int n_sel = 0;
  const int pos_f = block_excl_scan(sel, s_warp, n_sel);   // contains __syncthreads
  if (sel && pos_f < kcap) i_focus[static_cast<size_t>(b) * kcap + pos_f] = g0 + t;
  // q is active iff some selected p has q in [p - w/2, p - w/2 + w - 1]
  bool act = false;
  if (t < G) {
    const int lo = max(0, t - (w - 1) + w / 2), hi = min(G - 1, t + w / 2);
    for (int p = lo; p <= hi; ++p) act |= (s_sel[p] != 0);
  }
  int n_act = 0;
  const int pos_a = block_excl_scan(act, s_warp, n_act);
  if (act && pos_a < acap) i_active[static_cast<size_t>(b) * acap + pos_a] = g0 + t;
  for (int j = n_sel + t; j < kcap; j += blockDim.x) i_focus[static_cast<size_t>(b) * kcap + j] = -1;
  for (int j = n_act + t; j < acap; j += blockDim.x) i_active[static_cast<size_t>(b) * acap + j] = -1;
  if (t == 0) {
    n_focus[b] = min(n_sel, kcap);
    n_active[b] = min(n_act, acap);
  }
}

// X [n_mat, B, H, L, d] -> X_rows [n_mat, B, H, cap, d], one thread per 16-byte chunk.
__global__ void gather_rows_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ rows,
                                   const int32_t* __restrict__ n_rows, int B, int H, int L, int chunks, int cap,
                                   long long total, uint4* __restrict__ out, int* dev_err) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % chunks);
  long long r = idx / chunks;
  const int i = static_cast<int>(r % cap);
  r /= cap;
  const long long mbh = r;                 // (m * B + b) * H + h
  const int b = static_cast<int>((mbh / H) % B);
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (i < n_rows[b]) {
    const int src = rows[static_cast<size_t>(b) * cap + i];
    if (src >= 0 && src < L) {
      v = __ldg(X + (mbh * L + src) * chunks + c);
    } else {
      record_dev_error(dev_err, DEV_ERR_BAD_INDEX);
    }
  }
  out[idx] = v;
}

// Inverse of gather_rows: one thread per 16-byte chunk of a (matrix, b, h, listed row).
__global__ void scatter_rows_kernel(uint4* __restrict__ X, const int32_t* __restrict__ rows,
                                    const int32_t* __restrict__ n_rows, int B, int H, int L, int chunks, int cap,
                                    long long total, const uint4* __restrict__ src_rows, int* dev_err) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % chunks);
  long long r = idx / chunks;
  const int i = static_cast<int>(r % cap);
  r /= cap;
  const long long mbh = r;                 // (m * B + b) * H + h
  const int b = static_cast<int>((mbh / H) % B);
  if (i >= n_rows[b]) return;
  const int dst = rows[static_cast<size_t>(b) * cap + i];
  if (dst < 0 || dst >= L) {
    record_dev_error(dev_err, DEV_ERR_BAD_INDEX);
    return;
  }
  X[(mbh * L + dst) * chunks + c] = __ldg(src_rows + idx);
}

}  // namespace focus

using namespace focus;

extern "C" int focus_select_queries(const float* conf_prev, const uint8_t* mask, int B, int L, int g0, int g1,
                                    int n_t, float rho, int w, int32_t* i_focus, int32_t* n_focus, int kcap,
                                    int32_t* i_active, int32_t* n_active, int acap, void* stream) {
  FOCUS_CHECK_ARG(conf_prev && mask && i_focus && n_focus && i_active && n_active, "null pointer argument");
  FOCUS_CHECK_ARG(B >= 0 && L >= 1 && 0 <= g0 && g0 < g1 && g1 <= L, "need 0 <= g0 < g1 <= L (g0=%d g1=%d L=%d)",
                  g0, g1, L);
  const int G = g1 - g0;
  if (G > 1024) {
    set_error("current block of %d positions exceeds 1024", G);
    return FOCUS_ERR_UNSUPPORTED;
  }
  FOCUS_CHECK_ARG(n_t >= 0 && rho >= 0.f && w >= 1 && kcap >= 1 && acap >= 1, "bad n_t/rho/w/kcap/acap");
  const double kd = static_cast<double>(rho) * static_cast<double>(n_t);
  const long long k_req = static_cast<long long>(kd);   // floor for kd >= 0
  const int k_cap_needed = static_cast<int>(k_req < G ? k_req : G);
  if (kcap < k_cap_needed) {
    set_error("kcap %d < min(floor(rho*n_t), G) = %d", kcap, k_cap_needed);
    return FOCUS_ERR_CAPACITY;
  }
  const long long a_need = static_cast<long long>(k_cap_needed) * w;
  if (acap < (a_need < G ? a_need : G)) {
    set_error("acap %d < min(G, k*w) = %lld", acap, a_need < G ? a_need : static_cast<long long>(G));
    return FOCUS_ERR_CAPACITY;
  }
  if (B == 0) return FOCUS_OK;
  const int threads = ((G + 31) / 32) * 32;
  const cudaError_t e = launch_k(select_queries_kernel, dim3(B), dim3(threads), 0, static_cast<cudaStream_t>(stream),
                                 conf_prev, mask, L, g0, G, k_cap_needed, w, i_focus, n_focus, kcap, i_active,
                                 n_active, acap);
  note_launch();
  if (e != cudaSuccess) {
    set_error("select_queries launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

extern "C" int focus_gather_rows(const focus_bf16* X, const int32_t* rows, const int32_t* n_rows, int n_mat, int B,
                                 int H, int L, int d, int cap, focus_bf16* X_rows, void* stream) {
  FOCUS_CHECK_ARG(X && rows && n_rows && X_rows, "null pointer argument");
  FOCUS_CHECK_ARG(n_mat >= 0 && B >= 0 && H >= 1 && L >= 1 && cap >= 1, "bad sizes");
  FOCUS_CHECK_ARG(d % 8 == 0 && d > 0, "d must be a positive multiple of 8");
  FOCUS_CHECK_ARG(aligned16(X) && aligned16(X_rows), "tensors must be 16-byte aligned");
  const int chunks = d / 8;
  const long long total = static_cast<long long>(n_mat) * B * H * cap * chunks;
  if (total == 0) return FOCUS_OK;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  FOCUS_CHECK_ARG(blocks < (1LL << 31), "too large");
  const cudaError_t e =
      launch_k(gather_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
               static_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(X), rows, n_rows, B, H, L, chunks,
               cap, total, reinterpret_cast<uint4*>(X_rows), device_error_word());
  note_launch();
  if (e != cudaSuccess) {
    set_error("gather_rows launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

extern "C" int focus_scatter_rows(focus_bf16* X, const int32_t* rows, const int32_t* n_rows, int n_mat, int B, int H,
                                  int L, int d, int cap, const focus_bf16* X_rows, void* stream) {
  FOCUS_CHECK_ARG(X && rows && n_rows && X_rows, "null pointer argument");
  FOCUS_CHECK_ARG(n_mat >= 0 && B >= 0 && H >= 1 && L >= 1 && cap >= 1, "bad sizes");
  FOCUS_CHECK_ARG(d % 8 == 0 && d > 0, "d must be a positive multiple of 8");
  FOCUS_CHECK_ARG(aligned16(X) && aligned16(X_rows), "tensors must be 16-byte aligned");
  const int chunks = d / 8;
  const long long total = static_cast<long long>(n_mat) * B * H * cap * chunks;
  if (total == 0) return FOCUS_OK;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  FOCUS_CHECK_ARG(blocks < (1LL << 31), "too large");
  const cudaError_t e =
      launch_k(scatter_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
               static_cast<cudaStream_t>(stream), reinterpret_cast<uint4*>(X), rows, n_rows, B, H, L, chunks, cap,
               total, reinterpret_cast<const uint4*>(X_rows), device_error_word());
  note_launch();
  if (e != cudaSuccess) {
    set_error("scatter_rows launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}
