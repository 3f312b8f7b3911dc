// Prompt-block pruning: representative keys and relevance top-C.
//
// Focus-dLLM summary page, "方法步骤详情" (method steps), step (4): the prompt is cut
// into contiguous blocks, each represented by the mean of its keys; a relevance score
// R_b of the active queries to each block keeps the top-C blocks. The page leaves the
// aggregation open; the reading taken: R_b^h = mean over the active queries and the query
// heads of KV group h of q . kbar_b / sqrt(d), which equals qbar_h . kbar_b / sqrt(d).
#include <algorithm>

#include "focus_common.cuh"
#include "topk.cuh"

namespace focus {

// kbar[bh, j, :] = mean of K[bh, j*bs : min(P, (j+1)*bs), :]. One CTA per (block, head);
// 16-byte coalesced loads (one row = CH threads), fp32 accumulation, shared-memory reduction.
template <int D>
__global__ void __launch_bounds__(256) block_means_kernel(const __nv_bfloat16* __restrict__ K, int L, int P, int bs,
                                                          int nb, float* __restrict__ kbar) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  constexpr int CH = D / 8;
  constexpr int RL = 256 / CH;            // rows in flight per pass
  __shared__ float red[RL][D + 4];
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int c = threadIdx.x % CH, rl = threadIdx.x / CH;
  const int r0 = blk * bs;
  const int size = min(bs, P - r0);
  const uint4* src = reinterpret_cast<const uint4*>(K + (static_cast<size_t>(bh) * L + r0) * D) + c;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int r = rl; r < size; r += RL) {
    const uint4 v = __ldg(src + static_cast<size_t>(r) * CH);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rl][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int q = 0; q < RL; ++q) s += red[q][threadIdx.x];
    kbar[(static_cast<size_t>(bh) * nb + blk) * D + threadIdx.x] = s / static_cast<float>(size);
  }
}

constexpr int kSelectThreads = 512;

// One cluster of `gridDim.x` CTAs per (sequence, KV head). Every CTA forms qbar and scores
// its share of the blocks (8 kbar rows in flight per warp), pushing R into CTA 0's shared
// memory through DSMEM; after a cluster barrier CTA 0 selects the top-C.
template <int D>
__global__ void __launch_bounds__(kSelectThreads) block_select_kernel(
    const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ n_active, const float* __restrict__ kbar, int Hq,
    int Hkv, int acap, FastDiv acap_div, int nb, int C, int32_t* __restrict__ blocks, float* __restrict__ scores) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  constexpr int PARTS = kSelectThreads / D;
  extern __shared__ float s_R[];           // [nb] gathered in CTA 0, then [2048 + 64] top-C histogram
  __shared__ float s_part[PARTS][D];
  __shared__ float s_qbar[D];
  __shared__ TopkShared tk;
  const int cs = gridDim.x, rank = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / Hkv, h = bh % Hkv;
  const int g = Hq / Hkv;
  const int A = min(n_active[b], acap);
  const int dim = threadIdx.x % D, part = threadIdx.x / D;
  float acc = 0.f;
  const int rows = g * A;
  // Row slot r = (head r / acap, position r % acap). Every slot is loaded and positions
  // >= A are masked afterwards, so the loads do not wait for n_active.
  const int nr = g * acap;
  for (int r0 = part; r0 < nr; r0 += PARTS * 8) {         // 8 rows in flight per thread
    __nv_bfloat16 v[8];
    int pos[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = r0 + PARTS * u;
      v[u] = __float2bfloat16_rn(0.f);
      pos[u] = acap;
      if (r < nr) {
        const int rh = static_cast<int>(acap_div.div(static_cast<uint32_t>(r)));
        pos[u] = r - rh * acap;
        v[u] = Q[((static_cast<size_t>(b) * Hq + h * g + rh) * acap + pos[u]) * D + dim];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += pos[u] < A ? __bfloat162float(v[u]) : 0.f;
  }
  s_part[part][dim] = acc;
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll
    for (int p = 0; p < PARTS; ++p) sum += s_part[p][threadIdx.x];
    s_qbar[threadIdx.x] = rows > 0 ? sum / static_cast<float>(rows) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int LANES = D / 4;             // float4 per lane
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane < LANES) qv = reinterpret_cast<const float4*>(s_qbar)[lane];
  const float* kb = kbar + static_cast<size_t>(bh) * nb * D;
  const int chunk = (nb + cs - 1) / cs;
  const int j_begin = rank * chunk, j_end = min(nb, j_begin + chunk);
  const uint32_t sR0 = smem_u32(s_R);
  constexpr int UNR = 8;
  constexpr int NW = kSelectThreads / 32;
  for (int j0 = j_begin + warp * UNR; j0 < j_end; j0 += NW * UNR) {
    float4 kv[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int j = j0 + u;
      kv[u] = (j < j_end && lane < LANES)
                  ? __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D) + lane)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      float p = qv.x * kv[u].x + qv.y * kv[u].y + qv.z * kv[u].z + qv.w * kv[u].w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      const int j = j0 + u;
      if (lane == 0 && j < j_end) {
        const float R = p * inv_sqrt_d;
        if (cs > 1) {
          asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dsmem_addr(sR0 + 4u * j, 0)), "f"(R) : "memory");
        } else {
          s_R[j] = R;
        }
        if (scores) scores[static_cast<size_t>(bh) * nb + j] = R;
      }
    }
  }
  if (cs > 1) cluster_sync();   // every share of R is in CTA 0
  else __syncthreads();
  if (rank != 0) return;
  int32_t* out = blocks + static_cast<size_t>(bh) * C;
  auto key_of = [&](int i) { return float_order_key(s_R[i]); };
  int* wide = reinterpret_cast<int*>(s_R + ((nb + 3) & ~3));
  if (nb <= 2 * kSelectThreads) cta_topk_linear<true>(reinterpret_cast<const uint32_t*>(s_R), nb, C, out, C, wide, tk);
  else if (nb <= 4 * kSelectThreads) block_topk_small<4>(key_of, nb, C, out, C, tk, wide);
  else block_topk_ascending(key_of, nb, C, out, C, tk);
}

}  // namespace focus

using namespace focus;

extern "C" int focus_block_means(const focus_bf16* K, int B, int Hkv, int L, int d, int P, int bs, float* kbar,
                                 void* stream) {
  FOCUS_CHECK_ARG(K && kbar, "null pointer argument");
  FOCUS_CHECK_ARG(B >= 0 && Hkv >= 1 && L >= 1 && 1 <= P && P <= L && bs >= 1, "bad sizes (P=%d L=%d bs=%d)", P, L, bs);
  FOCUS_CHECK_ARG(aligned16(K) && aligned16(kbar), "tensors must be 16-byte aligned");
  if (d != 64 && d != 128) {
    set_error("head dim %d unsupported (64 or 128)", d);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (B == 0) return FOCUS_OK;
  const int nb = (P + bs - 1) / bs;
  FOCUS_CHECK_ARG(static_cast<long long>(B) * Hkv < 65536, "B*Hkv must be < 65536");
  dim3 grid(nb, B * Hkv);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* k = reinterpret_cast<const __nv_bfloat16*>(K);
  const cudaError_t e = d == 128 ? launch_k(block_means_kernel<128>, grid, dim3(256), 0, s, k, L, P, bs, nb, kbar)
                                 : launch_k(block_means_kernel<64>, grid, dim3(256), 0, s, k, L, P, bs, nb, kbar);
  note_launch();
  if (e != cudaSuccess) {
    set_error("block_means launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

extern "C" int focus_block_select(const focus_bf16* Q_active, const int32_t* n_active, const float* kbar, int B,
                                  int Hq, int Hkv, int d, int acap, int nb, int C, int32_t* blocks, float* scores_opt,
                                  void* stream) {
  FOCUS_CHECK_ARG(Q_active && n_active && kbar && blocks, "null pointer argument");
  FOCUS_CHECK_ARG(B >= 0 && Hq >= 1 && Hkv >= 1 && Hq % Hkv == 0 && acap >= 1 && nb >= 1 && C >= 1,
                  "bad sizes (Hq=%d Hkv=%d acap=%d nb=%d C=%d)", Hq, Hkv, acap, nb, C);
  FOCUS_CHECK_ARG(aligned16(kbar), "kbar must be 16-byte aligned");
  FOCUS_CHECK_ARG(static_cast<long long>(B) * Hkv < 65536, "B*Hkv must be < 65536");
  if (d != 64 && d != 128) {
    set_error("head dim %d unsupported (64 or 128)", d);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (nb > 49152) {
    set_error("nb=%d exceeds 49152 blocks", nb);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (B == 0) return FOCUS_OK;
  const size_t smem = (static_cast<size_t>((nb + 3) & ~3) + 2048 + 64) * sizeof(float);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(Q_active);
  // cluster of cs CTAs per (sequence, KV head), cs a power of two with B*Hkv*cs <= SMs
  FastDiv acap_div;
  acap_div.init(static_cast<uint32_t>(acap), static_cast<uint32_t>(Hq / Hkv) * static_cast<uint32_t>(acap) + 4096u);
  const int units = B * Hkv;
  int cs = 1;
  while (cs < 8 && units * cs * 2 <= device_sm_count() && (nb + cs * 2 - 1) / (cs * 2) >= 16) cs *= 2;
  cudaError_t err;
  if (d == 128) {
    if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(block_select_kernel<128>),
                            static_cast<int>(std::max<size_t>(smem, 80 * 1024)), "block_select"))
      return st_attr;
    err = launch_k_cluster(block_select_kernel<128>, dim3(cs, units), dim3(kSelectThreads), smem, s, cs, q,
                           n_active, kbar, Hq, Hkv, acap, acap_div, nb, C, blocks, scores_opt);
  } else {
    if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(block_select_kernel<64>),
                            static_cast<int>(std::max<size_t>(smem, 80 * 1024)), "block_select"))
      return st_attr;
    err = launch_k_cluster(block_select_kernel<64>, dim3(cs, units), dim3(kSelectThreads), smem, s, cs, q,
                           n_active, kbar, Hq, Hkv, acap, acap_div, nb, C, blocks, scores_opt);
  }
  note_launch();
  if (err != cudaSuccess) {
    set_error("block_select launch: %s", cudaGetErrorString(err));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}
