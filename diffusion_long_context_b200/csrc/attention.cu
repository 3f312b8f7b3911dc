// Bidirectional flash attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One kernel serves both attentions of the Focus-dLLM step:
//   * dense  (method steps (3) and the block-entry full refresh): every query row of a
//     KV-head group attends over all L keys;
//   * sparse (method steps (5)): the active queries attend over the key set
//     I_p = sinks U selected prompt blocks U current block, gathered tile by tile.
//
// CTA = 128 packed query rows of one KV-head group (row r <-> query head r / qcap,
// query r % qcap), one split of that group's key sequence. Six warps:
//   warps 0-3 : softmax (one query row per thread, reading S from TMEM), O rescale,
//               epilogue;
//   warp 4    : producer -- TMA (3-D tiled, SWIZZLE_128B, 8-row boxes) for contiguous
//               key runs, plain 16-byte loads for scattered sink rows;
//   warp 5    : tcgen05.mma issuer (one thread) and TMEM owner.
// Per 128-key tile: S = Q K^T (M=128, N=128, K=d) into TMEM, softmax in registers,
// P (bf16) to shared memory, O += P V (M=128, N=d, K=128) into TMEM.
//
// The sparse key sequence is laid out as slots (slots.cuh): the current block, then each
// kept block padded to a multiple of 8 slots, then the de-duplicated sinks. Every
// box-aligned group of slots of a block or of the current block is a contiguous key run
// and is fetched by one TMA box per 64-column atom; sink slots are fetched row by row.
// Padding slots are masked out of the softmax.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "focus_common.cuh"
#include "slots.cuh"

namespace focus {

// decode_attention.cu
bool decode_supported(int d, int Hq, int Hkv, int qcap, int L, int S, int C, bool sparse);
int decode_attention(const __nv_bfloat16* Q, const int32_t* n_q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                     __nv_bfloat16* O, float* lse_out, const int32_t* sinks, const int32_t* blocks, int S, int C, int bs,
                     int P, int g0, int g1, bool sparse, int B, int Hq, int Hkv, int L, int qcap, float scale_log2,
                     cudaStream_t stream, const float* kbar = nullptr, int nb = 0, int32_t* blocks_out = nullptr,
                     float* colsum = nullptr, int32_t* sinks_out = nullptr, int S_out = 0,
                     bool* sinks_done = nullptr);
bool decode_fused_supported(int d, int Hq, int Hkv, int qcap, int L, int S, int C, int nb);
// refresh.cu
bool refresh_supported(int d, int B, int Hq, int Hkv, int qcap, int sms);
int refresh_attention(const __nv_bfloat16* Q, const int32_t* n_q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                      __nv_bfloat16* O, int B, int Hq, int Hkv, int L, int qcap, float scale_log2,
                      cudaStream_t stream, float* kbar = nullptr, int P = 0, int bs = 1);

constexpr int kBM = 128;            // query rows per CTA (tcgen05 M)
constexpr int kBN = 128;            // keys per tile
constexpr int kStages = 2;          // K/V pipeline depth
constexpr int kThreads = 192;       // 6 warps
constexpr int kMaxSinks = 1024;     // sinks per KV head handled by the sparse kernel
constexpr int kMaxBlocks = 1024;    // kept blocks per KV head handled by the sparse kernel
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

struct AttnArgs {
  const __nv_bfloat16* Q;
  const int32_t* n_q;     // [B] or null (all qcap rows valid)
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  __nv_bfloat16* O;
  float* part_o;          // [splits, B, Hq, qcap, D] when n_splits > 1
  float* part_lse;        // [splits, B, Hq, qcap]
  float* lse_out;         // [B, Hq, qcap] (log2 domain) or null; written when n_splits == 1
  const int32_t* sinks;   // [B, Hkv, S]
  const int32_t* blocks;  // [B, Hkv, C]
  int B, Hq, Hkv, L, qcap, g;
  int n_splits, tiles_per_split;
  int box_rows;           // rows per TMA box (divides 128)
  int gen_pad;            // slots of the current block in the sparse layout (multiple of box_rows)
  FastDiv pad_div, bs_div;  // by round_up(bs, 8) and bs (host-computed)
  int S, C, bs, P, g0, g1;
  float scale_log2;
  int* dev_err;
};

struct __align__(8) AttnBook {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full, s_free, p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort_flag;
  SlotLayout sl;
  int blk[kMaxBlocks];
  int fsinks[kMaxSinks];
};

template <int D>
struct AttnSmem {
  static constexpr uint32_t kTile = kBN * D * 2;        // one 128-row bf16 tile
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;
  static constexpr uint32_t kV = kK + kStages * kTile;
  static constexpr uint32_t kP = kV + kStages * kTile;  // 128 x 128 bf16
  static constexpr uint32_t kBook = kP + kBM * kBN * 2;
  static constexpr uint32_t kBytes = kBook + sizeof(AttnBook) + 1024;  // + alignment slack
};

// Packed query row held by TMEM lane / A-operand row `lane`. Rows are spread across the
// four 32-lane quadrants (row j -> lane (j % 4) * 32 + j / 4) so that a partly filled tile
// (32 active queries of an MHA head) keeps all four softmax warps busy.
__device__ __forceinline__ int lane_to_row(int lane) { return (lane & 31) * 4 + (lane >> 5); }

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 500000000ull) return false;
  }
  return true;
}

template <int D, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const AttnArgs a) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  using SM = AttnSmem<D>;
  constexpr int CH = D / 8;                // 16-byte chunks per row
  constexpr int ATOMS = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  uint8_t* sP = smem + SM::kP;
  AttnBook* bk = reinterpret_cast<AttnBook*>(smem + SM::kBook);

  const int warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x, mtile = blockIdx.y;
  const int bh = blockIdx.z;               // b * Hkv + kvh
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int nq_b = a.n_q ? a.n_q[b] : a.qcap;
  const int rows_total = a.g * a.qcap;

  // ---------------------------------------------------------------- prologue
  if (warp == kMmaWarp) {
    tmem_alloc(&bk->tmem_base, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bk->full[s], 1);
      mbar_init(&bk->empty[s], 1);
    }
    mbar_init(&bk->s_full, 1);
    mbar_init(&bk->s_free, 4);
    mbar_init(&bk->p_full, 4);
    mbar_init(&bk->pv_done, 1);
    mbar_init(&bk->drain, 1);
    bk->abort_flag = 0;
    fence_mbar_init();
  }
  if (SPARSE) {
    if (warp == 0) {
      const int32_t* blk_g = a.blocks + static_cast<size_t>(bh) * a.C;
      const int32_t* snk_g = a.sinks ? a.sinks + static_cast<size_t>(bh) * a.S : nullptr;
      const LayoutPrefetch pf = layout_prefetch(blk_g, a.C, snk_g, a.S);
      const SlotLayout sl0 = build_block_layout(pf, blk_g, a.C, a.S, a.P, a.bs, a.gen_pad, a.box_rows, a.pad_div,
                                                bk->blk, kMaxBlocks, kMaxSinks, &bk->sl);
      dedupe_sinks(pf, snk_g, sl0, a.L, a.P, a.g0, a.g1, a.bs_div, bk->blk, bk->fsinks);
    }
  } else if (threadIdx.x == 0) {
    bk->sl.n_slots = a.L;
  }
  // Q rows -> SWIZZLE_128B K-major tile; P tile cleared once.
  for (int idx = threadIdx.x; idx < kBM * CH; idx += kThreads) {
    const int r = idx / CH, c = idx % CH;
    const int R = mtile * kBM + lane_to_row(r);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (R < rows_total) {
      const int hq = kvh * a.g + R / a.qcap, i = R % a.qcap;
      if (i < nq_b)
        v = __ldg(reinterpret_cast<const uint4*>(a.Q + ((static_cast<size_t>(b) * a.Hq + hq) * a.qcap + i) * D) + c);
    }
    *reinterpret_cast<uint4*>(sQ + sw128_offset(r, c, kBM)) = v;
  }
  for (int idx = threadIdx.x; idx < kBM * kBN * 2 / 16; idx += kThreads)
    reinterpret_cast<uint4*>(sP)[idx] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = bk->tmem_base;
  const uint32_t tS = tmem;          // columns [0, 128): S, fp32
  const uint32_t tO = tmem + 128;    // columns [128, 128 + D): O, fp32
  const SlotLayout sl = bk->sl;
  const int n_slots = sl.n_slots;
  const int total_tiles = (n_slots + kBN - 1) / kBN;
  const int t_begin = split * a.tiles_per_split;
  const int t_end = min(total_tiles, t_begin + a.tiles_per_split);
  const int n_it = max(0, t_end - t_begin);
  volatile int* abort_flag = &bk->abort_flag;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    const int BR = a.box_rows;
    const int ngroups = kBN / BR;
    const __nv_bfloat16* Kbh = a.K + static_cast<size_t>(bh) * a.L * D;
    const __nv_bfloat16* Vbh = a.V + static_cast<size_t>(bh) * a.L * D;
    int issued = 0;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % kStages;
      if (it >= kStages) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bk->empty[s], ((it / kStages) - 1) & 1, abort_flag, a.dev_err,
                                               DEV_ERR_TIMEOUT_PRODUCER)))
          break;
      }
      const int slot0 = (t_begin + it) * kBN;
      uint8_t* dK = sK + s * SM::kTile;
      uint8_t* dV = sV + s * SM::kTile;
      if (lane == 0) {
        uint32_t tma_groups = 0;
        for (int grp = 0; grp < ngroups; ++grp)
          if (group_key0<SPARSE>(sl, bk->blk, a.bs, a.g0, slot0 + grp * BR) >= 0) ++tma_groups;
        mbar_expect_tx(&bk->full[s], tma_groups * ATOMS * 2u * static_cast<uint32_t>(BR) * 128u);
        for (int grp = 0; grp < ngroups; ++grp) {
          const int key0 = group_key0<SPARSE>(sl, bk->blk, a.bs, a.g0, slot0 + grp * BR);
          if (key0 < 0) continue;
#pragma unroll
          for (int at = 0; at < ATOMS; ++at) {
            const uint32_t off = at * (kBN * 128) + grp * BR * 128;
            tma_load_3d(smem_u32(dK + off), &tmK, &bk->full[s], at * 64, key0, bh);
            tma_load_3d(smem_u32(dV + off), &tmV, &bk->full[s], at * 64, key0, bh);
          }
        }
      }
      if (SPARSE) {
        // sink rows (and slots past the end, zero-filled) by cp.async, 16 bytes per lane
        bool any_rows = false;
        for (int grp = 0; grp < ngroups; ++grp) {
          if (group_key0<SPARSE>(sl, bk->blk, a.bs, a.g0, slot0 + grp * BR) >= 0) continue;
          any_rows = true;
          for (int idx = lane; idx < BR * CH; idx += 32) {
            const int rr = idx / CH, c = idx % CH;
            const int row = grp * BR + rr;
            const int key = sink_slot_key(sl, bk->fsinks, slot0 + row);
            const uint32_t src_bytes = key >= 0 ? 16u : 0u;
            const size_t koff = static_cast<size_t>(key >= 0 ? key : 0) * D + c * 8;
            cp_async16(smem_u32(dK + sw128_offset(row, c, kBN)), Kbh + koff, src_bytes);
            cp_async16(smem_u32(dV + sw128_offset(row, c, kBN)), Vbh + koff, src_bytes);
          }
        }
        if (any_rows) {
          cp_async_wait_all();
          fence_proxy_async_smem();
        }
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(&bk->full[s]);
      __syncwarp();
      ++issued;
    }
    // never leave with copies in flight
    if (lane == 0) {
      for (int j = max(0, issued - kStages); j < issued; ++j) wait_drain(&bk->full[j % kStages], (j / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      // Descriptors are formed once; a K step or a stage adds a constant to the 14-bit
      // start-address field (address >> 4), which cannot carry: shared memory < 256 KB.
      const uint64_t q_desc = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t p_desc = sw128_desc(smem_u32(sP), 16, 1024);
      const uint64_t k_desc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t v_desc0 = sw128_desc(smem_u32(sV), kBN * 128, 1024);
      constexpr uint32_t kTileDesc = SM::kTile >> 4;
      bool ok = true;
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(&bk->p_full, j & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint64_t vd = v_desc0 + static_cast<uint64_t>((j % kStages) * kTileDesc);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_bf16(tO, p_desc + (ks >> 2) * (kBM * 128 / 16) + (ks & 3) * 2, vd + ks * (2048 / 16), idesc_pv,
                   (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bk->pv_done);
        mma_commit(&bk->empty[j % kStages]);
        return true;
      };
      for (int it = 0; it < n_it && ok; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&bk->full[s], (it / kStages) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) break;
        if (it > 0 && !mbar_wait(&bk->s_free, (it - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint64_t kd = k_desc0 + static_cast<uint64_t>(s * kTileDesc);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * (kBN * 128 / 16) + (ks & 3) * 2;
          mma_bf16(tS, q_desc + koff, kd + koff, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bk->s_full);
        if (it > 0) ok = issue_pv(it - 1);
      }
      if (ok && n_it > 0 && !*abort_flag) issue_pv(n_it - 1);
      // all MMAs done before TMEM is released
      mma_commit(&bk->drain);
      wait_drain(&bk->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0..3
    const int r = threadIdx.x;                      // TMEM lane == row of the A operand
    const int R = mtile * kBM + lane_to_row(r);
    const int hq = kvh * a.g + (R < rows_total ? R / a.qcap : 0);
    const int qi = R % a.qcap;
    const bool row_exists = R < rows_total;
    const bool row_valid = row_exists && qi < nq_b;
    const bool warp_active = __any_sync(0xffffffffu, row_valid);
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bk->s_full, it & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_SOFTMAX))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kBN];
      if (warp_active) {
        // validity of the 128 slots of this tile: 4 ballots, lane evaluates slot lane + 32 q
        unsigned vm[4];
        const int slot0 = (t_begin + it) * kBN;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          vm[q] = __ballot_sync(0xffffffffu,
                                slot_valid<SPARSE>(sl, bk->fsinks, a.L, a.bs, a.g1 - a.g0, slot0 + q * 32 + lane));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t rg[32];
          tmem_ld32(tS + lane_addr + c * 32, rg);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            sv[c * 32 + j] = ((vm[c] >> j) & 1u) ? __uint_as_float(rg[j]) * a.scale_log2 : -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->s_free);

      float alpha = 1.f;
      bool need_rescale = false;
      if (warp_active) {
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < kBN; ++j) mt = fmaxf(mt, sv[j]);
        const float m_new = fmaxf(m_ref, mt);
        // keep the reference maximum unless it grows by more than 2^8 (p stays <= 256)
        if (m_new > m_ref + 8.f || (m_ref == -INFINITY && m_new > -INFINITY)) {
          alpha = (m_ref == -INFINITY) ? 0.f : exp2_approx(m_ref - m_new);
          m_ref = m_new;
          need_rescale = true;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          sv[j] = exp2_approx(sv[j] - m_use);
          ls += sv[j];
        }
        l_sum = l_sum * alpha + ls;
      }
      if (it > 0) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bk->pv_done, (it - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_SOFTMAX))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (warp_active && __any_sync(0xffffffffu, need_rescale && alpha != 1.f)) {
          const float al = need_rescale ? alpha : 1.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t rg[32];
            tmem_ld32(tO + lane_addr + c * 32, rg);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) rg[j] = __float_as_uint(__uint_as_float(rg[j]) * al);
            tmem_st32(tO + lane_addr + c * 32, rg);
          }
          tmem_st_wait();
        }
      }
      if (warp_active) {
#pragma unroll
        for (int c = 0; c < kBN / 8; ++c) {
          uint4 v;
          v.x = pack_bf16x2(sv[c * 8 + 0], sv[c * 8 + 1]);
          v.y = pack_bf16x2(sv[c * 8 + 2], sv[c * 8 + 3]);
          v.z = pack_bf16x2(sv[c * 8 + 4], sv[c * 8 + 5]);
          v.w = pack_bf16x2(sv[c * 8 + 6], sv[c * 8 + 7]);
          *reinterpret_cast<uint4*>(sP + sw128_offset(r, c, kBM)) = v;
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->p_full);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n_it > 0) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bk->pv_done, (n_it - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_EPILOGUE));
      tc_fence_after();
    }
    if (ok) {
      const size_t row_off = (static_cast<size_t>(b) * a.Hq + hq) * a.qcap + qi;
      const bool have_o = n_it > 0 && l_sum > 0.f;
      const float lse2 = have_o ? ((m_ref == -INFINITY ? 0.f : m_ref) + __log2f(l_sum)) : -INFINITY;
      const float inv_l = (row_valid && have_o) ? 1.f / l_sum : 0.f;
      const bool do_ld = warp_active && n_it > 0;      // warp-uniform: tcgen05.ld is collective
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rg[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) rg[j] = 0u;
        if (do_ld) {
          tmem_ld32(tO + lane_addr + c * 32, rg);
          tmem_ld_wait();
        }
        if (a.n_splits == 1) {
          if (row_exists) {
            __nv_bfloat16* orow = a.O + row_off * D + c * 32;
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(rg[j4 * 8 + 0]) * inv_l, __uint_as_float(rg[j4 * 8 + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(rg[j4 * 8 + 2]) * inv_l, __uint_as_float(rg[j4 * 8 + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(rg[j4 * 8 + 4]) * inv_l, __uint_as_float(rg[j4 * 8 + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(rg[j4 * 8 + 6]) * inv_l, __uint_as_float(rg[j4 * 8 + 7]) * inv_l);
              reinterpret_cast<uint4*>(orow)[j4] = v;
            }
          }
        } else if (row_valid) {
          float* po = a.part_o + (static_cast<size_t>(split) * a.B * a.Hq * a.qcap + row_off) * D + c * 32;
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4)
            reinterpret_cast<float4*>(po)[j4] =
                make_float4(__uint_as_float(rg[j4 * 4 + 0]) * inv_l, __uint_as_float(rg[j4 * 4 + 1]) * inv_l,
                            __uint_as_float(rg[j4 * 4 + 2]) * inv_l, __uint_as_float(rg[j4 * 4 + 3]) * inv_l);
        }
      }
      if (row_valid) {
        if (a.n_splits == 1) {
          if (a.lse_out) a.lse_out[row_off] = lse2;
        } else {
          a.part_lse[static_cast<size_t>(split) * a.B * a.Hq * a.qcap + row_off] = lse2;
        }
      }
    } else if (row_valid && a.n_splits > 1) {
      // a wait ran out: this split contributes nothing, so the combine never merges a
      // partial left in the workspace by an earlier call
      const size_t row_off = (static_cast<size_t>(b) * a.Hq + hq) * a.qcap + qi;
      a.part_lse[static_cast<size_t>(split) * a.B * a.Hq * a.qcap + row_off] = -INFINITY;
    }
    if (warp_active) tmem_ld_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Merge split partials: O = sum_s 2^(lse_s - lse) O_s, lse = log2 sum_s 2^lse_s. One warp per row.
template <int D>
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                    const int32_t* __restrict__ n_q, int B, int Hq, int qcap, int n_splits,
                                    __nv_bfloat16* __restrict__ O, float* __restrict__ lse_out) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int total = B * Hq * qcap;
  if (row >= total) return;
  const int qi = row % qcap;
  const int b = row / (Hq * qcap);
  const int nq = n_q ? n_q[b] : qcap;
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float lse = -INFINITY;
  if (qi < nq) {
    float mx = -INFINITY;
    for (int s = 0; s < n_splits; ++s) mx = fmaxf(mx, part_lse[static_cast<size_t>(s) * total + row]);
    float wsum = 0.f;
    if (mx > -INFINITY) {
      for (int s = 0; s < n_splits; ++s) {
        const float ls = part_lse[static_cast<size_t>(s) * total + row];
        if (ls == -INFINITY) continue;
        const float wgt = exp2_approx(ls - mx);
        wsum += wgt;
        const float* po = part_o + (static_cast<size_t>(s) * total + row) * D + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += wgt * po[e];
      }
      const float inv = 1.f / wsum;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] *= inv;
      lse = mx + __log2f(wsum);
    }
  }
  __nv_bfloat16* orow = O + static_cast<size_t>(row) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2) reinterpret_cast<uint32_t*>(orow)[e / 2] = pack_bf16x2(acc[e], acc[e + 1]);
  if (lse_out && qi < nq) lse_out[row] = lse;
}

// ------------------------------------------------------------------------- sink column sums
// colsum[b, h, j] = sum over valid query rows r of the group of 2^(scale_log2 * q_r . k_j - lse2_r).
// Swap-AB: S^T = K Q^T (M = 128 keys, N = padded group rows) so that each thread owns one
// key and the sum over queries is thread-local. The S^T accumulator is double-buffered in
// TMEM, so the MMA of tile i+1 overlaps the exp-sum of tile i. The K ring is as deep as
// shared memory allows (6 stages for up to 64 group rows, else 3), because K is the only
// stream and its bytes in flight bound the bandwidth.
constexpr int kColMaxStages = 6;

struct ColsumArgs {
  const __nv_bfloat16* Q;
  const int32_t* n_q;
  const float* lse2;      // [B, Hq, qcap], log2 domain
  float* colsum;          // [B, Hkv, L]
  int B, Hq, Hkv, L, qcap, g, n_pad, tmem_cols;
  int tiles_per_cta;
  int box_rows;           // rows per TMA box (divides 128)
  float scale_log2;
  int* dev_err;
};

struct __align__(8) ColBook {
  uint64_t full[kColMaxStages];
  uint64_t empty[kColMaxStages];
  uint64_t acc_full[2], acc_free[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  float lse2[256];
};

template <int D, int STAGES>
struct ColSmem {
  static constexpr int kQRows = STAGES > 3 ? 64 : 256;     // group rows the Q area holds
  static constexpr uint32_t kTile = kBN * D * 2;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQRows * D * 2;
  static constexpr uint32_t kBook = kK + STAGES * kTile;
  static constexpr uint32_t kBytes = kBook + sizeof(ColBook) + 1024;
  static_assert(STAGES <= kColMaxStages, "too many stages");
  static_assert(kBytes <= 232448, "colsum kernel exceeds the 227 KB of shared memory per CTA");
};

template <int D, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    colsum_kernel(const __grid_constant__ CUtensorMap tmK128, const ColsumArgs a) {
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  using SM = ColSmem<D, STAGES>;
  constexpr int kColStages = STAGES;
  constexpr int CH = D / 8;
  constexpr int ATOMS = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  ColBook* bk = reinterpret_cast<ColBook*>(smem + SM::kBook);
  const int warp = warp_id(), lane = lane_id();
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int nq_b = a.n_q ? a.n_q[b] : a.qcap;
  const int rows_total = a.g * a.qcap;
  const int n_pad = a.n_pad;

  if (warp == kMmaWarp) {
    tmem_alloc(&bk->tmem_base, a.tmem_cols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kColStages; ++s) {
      mbar_init(&bk->full[s], 1);
      mbar_init(&bk->empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bk->acc_full[i], 1);
      mbar_init(&bk->acc_free[i], 4);
    }
    mbar_init(&bk->drain, 1);
    bk->abort_flag = 0;
    fence_mbar_init();
  }
  for (int idx = threadIdx.x; idx < n_pad * CH; idx += kThreads) {
    const int r = idx / CH, c = idx % CH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows_total) {
      const int hq = kvh * a.g + r / a.qcap, i = r % a.qcap;
      if (i < nq_b)
        v = __ldg(reinterpret_cast<const uint4*>(a.Q + ((static_cast<size_t>(b) * a.Hq + hq) * a.qcap + i) * D) + c);
    }
    *reinterpret_cast<uint4*>(sQ + sw128_offset(r, c, n_pad)) = v;
  }
  for (int r = threadIdx.x; r < 256; r += kThreads) {
    float v = INFINITY;   // padded / invalid rows contribute 2^(-inf) = 0
    if (r < rows_total) {
      const int hq = kvh * a.g + r / a.qcap, i = r % a.qcap;
      if (i < nq_b) v = a.lse2[(static_cast<size_t>(b) * a.Hq + hq) * a.qcap + i];
    }
    bk->lse2[r] = v;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = bk->tmem_base;
  const int total_tiles = (a.L + kBN - 1) / kBN;
  const int t_begin = blockIdx.x * a.tiles_per_cta;
  const int t_end = min(total_tiles, t_begin + a.tiles_per_cta);
  const int n_it = max(0, t_end - t_begin);
  volatile int* abort_flag = &bk->abort_flag;

  if (warp == kProducerWarp) {
    int issued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tmK128);
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kColStages;
        if (it >= kColStages &&
            !mbar_wait(&bk->empty[s], ((it / kColStages) - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_PRODUCER))
          break;
        mbar_arrive_expect_tx(&bk->full[s], ATOMS * kBN * 128);
        for (int r0 = 0; r0 < kBN; r0 += a.box_rows)
          for (int at = 0; at < ATOMS; ++at)
            tma_load_3d(smem_u32(sK + s * SM::kTile + at * (kBN * 128) + r0 * 128), &tmK128, &bk->full[s], at * 64,
                        (t_begin + it) * kBN + r0, bh);
        ++issued;
      }
      for (int j = max(0, issued - kColStages); j < issued; ++j)
        wait_drain(&bk->full[j % kColStages], (j / kColStages) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, n_pad, false, false);
      // descriptors formed once; K steps and stages add constants to the start-address field
      const uint64_t q_desc = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc0 = sw128_desc(smem_u32(sK), 16, 1024);
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kColStages;
        const int ab = it & 1;
        if (!mbar_wait(&bk->full[s], (it / kColStages) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) break;
        if (it >= 2 && !mbar_wait(&bk->acc_free[ab], ((it - 2) >> 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA))
          break;
        tc_fence_after();
        const uint64_t kd = k_desc0 + static_cast<uint64_t>(s * (SM::kTile >> 4));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16(tmem + ab * n_pad, kd + (ks >> 2) * (kBN * 128 / 16) + (ks & 3) * 2,
                   q_desc + (ks >> 2) * (n_pad * 128 / 16) + (ks & 3) * 2, idesc, ks > 0 ? 1u : 0u);
        mma_commit(&bk->acc_full[ab]);
        mma_commit(&bk->empty[s]);
      }
      mma_commit(&bk->drain);
      wait_drain(&bk->drain, 0);
    }
    __syncwarp();
  } else {
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    float* out = a.colsum + static_cast<size_t>(bh) * a.L;
    for (int it = 0; it < n_it; ++it) {
      const int ab = it & 1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&bk->acc_full[ab], (it >> 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_EPILOGUE)))
        break;
      tc_fence_after();
      float sum = 0.f;
      for (int c0 = 0; c0 < n_pad; c0 += 32) {
        uint32_t rg[32];
        tmem_ld32(tmem + lane_addr + ab * n_pad + c0, rg);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = c0 + j;
          if (col < n_pad) sum += exp2_approx(__uint_as_float(rg[j]) * a.scale_log2 - bk->lse2[col]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->acc_free[ab]);
      const int key = (t_begin + it) * kBN + threadIdx.x;
      if (key < a.L) out[key] = sum;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ------------------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over [B*H, L, D] bf16 (x = D innermost), box {64, box_rows, 1}, SWIZZLE_128B,
// out-of-range rows read as zero.
int make_kv_map(CUtensorMap* map, const void* base, int BH, int L, int D, int box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled is unavailable (driver entry point lookup failed)");
    return FOCUS_ERR_CUDA;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (CUresult %d) for [%d, %d, %d]", static_cast<int>(r), BH, L, D);
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int pow2_rows(int x, int cap) {
  int r = 8;
  while (r * 2 <= cap && x % (r * 2) == 0) r *= 2;
  return r;
}

// Rows per TMA box: whole tiles for contiguous keys; for the sparse slot layout the
// largest power of two that keeps every box inside one kept block or the current block.
int box_rows_for(bool sparse, int L, int bs, int G) {
  (void)G;
  int cap = kBN;
  while (cap > L && cap > 8) cap >>= 1;
  if (!sparse) return cap;
  return pow2_rows((bs + 7) & ~7, cap);
}

// The sink segment and the current block are padded to whole boxes so that every box
// stays in one segment.
int gen_pad_for(int box_rows, int G) { return (G + box_rows - 1) / box_rows * box_rows; }


struct AttnPlan {
  bool decode;            // few-query swap-AB kernel (decode_attention.cu) serves this call
  bool refresh;           // many-row kernel (refresh.cu) serves this dense call
  int n_mtiles, n_splits, tiles_per_split;
  size_t lse_bytes, part_lse_bytes, part_o_bytes, total;
};

// Split plan of a call. The decode kernel merges its splits inside a cluster and needs
// workspace only for the log-sum-exp consumed by the column-sum pass.
AttnPlan plan_attention(int B, int Hq, int Hkv, int d, int qcap, int kv_cap, bool want_lse, int L, int S, int C,
                        bool sparse) {
  AttnPlan p{};
  const int g = Hq / Hkv;
  if (decode_supported(d, Hq, Hkv, qcap, L, S, C, sparse)) {
    p.decode = true;                   // merges its splits in the cluster; column sums in-kernel
    p.n_splits = 1;
    return p;
  }
  if (!sparse && !want_lse && refresh_supported(d, B, Hq, Hkv, qcap, device_sm_count())) {
    p.refresh = true;                  // every row block streams all keys: no splits, no workspace
    p.n_splits = 1;
    return p;
  }
  p.n_mtiles = (g * qcap + kBM - 1) / kBM;
  const int max_tiles = std::max(1, (kv_cap + kBN - 1) / kBN);
  const long units = static_cast<long>(B) * Hkv * p.n_mtiles;
  const int sms = device_sm_count();
  int splits = 1;
  if (units < sms) splits = static_cast<int>(std::max(1L, sms / std::max(1L, units)));
  splits = std::min(splits, max_tiles);
  p.tiles_per_split = (max_tiles + splits - 1) / splits;
  p.n_splits = (max_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  const size_t rows = static_cast<size_t>(B) * Hq * qcap;
  p.lse_bytes = want_lse ? align256(rows * 4) : 0;
  p.part_lse_bytes = p.n_splits > 1 ? align256(rows * p.n_splits * 4) : 0;
  p.part_o_bytes = p.n_splits > 1 ? align256(rows * p.n_splits * d * 4) : 0;
  p.total = p.lse_bytes + p.part_lse_bytes + p.part_o_bytes;
  return p;
}

template <int D, bool SPARSE>
int launch_attention(const AttnArgs& args, const CUtensorMap& mk, const CUtensorMap& mv, int n_mtiles,
                     cudaStream_t stream) {
  using SM = AttnSmem<D>;
  auto kern = attn_fwd_kernel<D, SPARSE>;
  if (const int st = configure_dynamic_smem(reinterpret_cast<const void*>(kern), static_cast<int>(SM::kBytes),
                                            "attention kernel"))
    return st;
  dim3 grid(args.n_splits, n_mtiles, args.B * args.Hkv);
  const cudaError_t e = launch_k(kern, grid, dim3(kThreads), SM::kBytes, stream, mk, mv, args);
  note_launch();
  if (e != cudaSuccess) {
    set_error("attention launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return launch_status(SPARSE ? "sparse attention kernel" : "dense attention kernel");
}

template <int D>
int launch_combine(const AttnArgs& a, cudaStream_t stream) {
  const int rows = a.B * a.Hq * a.qcap;
  const int warps = 8;
  const cudaError_t e = launch_k(attn_combine_kernel<D>, dim3((rows + warps - 1) / warps), dim3(warps * 32), 0,
                                 stream, a.part_o, a.part_lse, a.n_q, a.B, a.Hq, a.qcap, a.n_splits, a.O,
                                 a.lse_out);
  note_launch();
  if (e != cudaSuccess) {
    set_error("combine launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

template <int D, int STAGES>
int launch_colsum(const __nv_bfloat16* Q, const int32_t* n_q, const __nv_bfloat16* K, const float* lse2, float* colsum,
                  int B, int Hq, int Hkv, int L, int qcap, float scale_log2, cudaStream_t stream) {
  using SM = ColSmem<D, STAGES>;
  CUtensorMap mk;
  const int box_rows = box_rows_for(false, L, 0, 0);
  int st = make_kv_map(&mk, K, B * Hkv, L, D, box_rows);
  if (st != FOCUS_OK) return st;
  ColsumArgs c{};
  c.box_rows = box_rows;
  c.Q = Q;
  c.n_q = n_q;
  c.lse2 = lse2;
  c.colsum = colsum;
  c.B = B;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.L = L;
  c.qcap = qcap;
  c.g = Hq / Hkv;
  c.n_pad = ((c.g * qcap + 15) / 16) * 16;
  c.tmem_cols = 2 * c.n_pad <= 32 ? 32 : 2 * c.n_pad <= 64 ? 64 : 2 * c.n_pad <= 128 ? 128 : 2 * c.n_pad <= 256 ? 256 : 512;
  c.scale_log2 = scale_log2;
  c.dev_err = device_error_word();
  const int total_tiles = (L + kBN - 1) / kBN;
  const int units = B * Hkv;
  const int sms = device_sm_count();
  int chunks = std::max(1, sms / std::max(1, units));
  chunks = std::min(chunks, total_tiles);
  c.tiles_per_cta = (total_tiles + chunks - 1) / chunks;
  chunks = (total_tiles + c.tiles_per_cta - 1) / c.tiles_per_cta;
  auto kern = colsum_kernel<D, STAGES>;
  if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(kern), static_cast<int>(SM::kBytes),
                                                 "colsum kernel"))
    return st_attr;
  dim3 grid(chunks, units);
  const cudaError_t e = launch_k(kern, grid, dim3(kThreads), SM::kBytes, stream, mk, c);
  note_launch();
  if (e != cudaSuccess) {
    set_error("colsum launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

// The deep ring needs the group rows to fit the 64-row Q area.
template <int D>
int run_colsum(const __nv_bfloat16* Q, const int32_t* n_q, const __nv_bfloat16* K, const float* lse2, float* colsum,
               int B, int Hq, int Hkv, int L, int qcap, float scale_log2, cudaStream_t stream) {
  const int n_pad = ((Hq / Hkv * qcap + 15) / 16) * 16;
  if (n_pad <= ColSmem<D, 6>::kQRows)
    return launch_colsum<D, 6>(Q, n_q, K, lse2, colsum, B, Hq, Hkv, L, qcap, scale_log2, stream);
  return launch_colsum<D, 3>(Q, n_q, K, lse2, colsum, B, Hq, Hkv, L, qcap, scale_log2, stream);
}

template <int D, bool SPARSE>
int run_attention(AttnArgs args, const AttnPlan& plan, void* ws, float* colsum, cudaStream_t stream,
                  int32_t* sinks_out = nullptr, int S_out = 0, bool* sinks_done = nullptr) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (sinks_done) *sinks_done = false;
  if (plan.refresh)
    return refresh_attention(args.Q, args.n_q, args.K, args.V, args.O, args.B, args.Hq, args.Hkv, args.L, args.qcap,
                             args.scale_log2, stream);
  if (plan.decode) {
    // the decode kernel forms the column sums (and, where it can, the sinks) itself
    return decode_attention(args.Q, args.n_q, args.K, args.V, args.O, nullptr, args.sinks, args.blocks, args.S,
                            args.C, args.bs, args.P, args.g0, args.g1, SPARSE, args.B, args.Hq, args.Hkv, args.L,
                            args.qcap, args.scale_log2, stream, nullptr, 0, nullptr, SPARSE ? nullptr : colsum,
                            sinks_out, S_out, sinks_done);
  }
  args.box_rows = box_rows_for(SPARSE, args.L, args.bs, args.g1 - args.g0);
  args.gen_pad = gen_pad_for(args.box_rows, args.g1 - args.g0);
  if (SPARSE) {
    const int pad_bs = (args.bs + 7) & ~7;
    const long long n_max = static_cast<long long>(args.C) * pad_bs + args.gen_pad +
                            gen_pad_for(args.box_rows, std::min(args.S, kMaxSinks)) + 2 * kBN;
    args.pad_div.init(static_cast<uint32_t>(pad_bs), static_cast<uint32_t>(std::min<long long>(n_max, 0xFFFFFFFFll)));
    args.bs_div.init(static_cast<uint32_t>(std::max(args.bs, 1)), static_cast<uint32_t>(args.L));
  }
  CUtensorMap mk, mv;
  int st = make_kv_map(&mk, args.K, args.B * args.Hkv, args.L, D, args.box_rows);
  if (st != FOCUS_OK) return st;
  st = make_kv_map(&mv, args.V, args.B * args.Hkv, args.L, D, args.box_rows);
  if (st != FOCUS_OK) return st;
  args.lse_out = plan.lse_bytes ? reinterpret_cast<float*>(w) : nullptr;
  args.part_lse = plan.part_lse_bytes ? reinterpret_cast<float*>(w + plan.lse_bytes) : nullptr;
  args.part_o = plan.part_o_bytes ? reinterpret_cast<float*>(w + plan.lse_bytes + plan.part_lse_bytes) : nullptr;
  args.n_splits = plan.n_splits;
  args.tiles_per_split = plan.tiles_per_split;
  args.dev_err = device_error_word();
  st = launch_attention<D, SPARSE>(args, mk, mv, plan.n_mtiles, stream);
  if (st != FOCUS_OK) return st;
  if (plan.n_splits > 1) {
    st = launch_combine<D>(args, stream);
    if (st != FOCUS_OK) return st;
  }
  if (colsum) {
    st = run_colsum<D>(args.Q, args.n_q, args.K, args.lse_out, colsum, args.B, args.Hq, args.Hkv, args.L,
                          args.qcap, args.scale_log2, stream);
  }
  return st;
}

constexpr float kLog2e = 1.4426950408889634f;

int check_common(const void* Q, const void* K, const void* V, const void* O, int B, int Hq, int Hkv, int L, int d,
                 int qcap) {
  FOCUS_CHECK_ARG(Q && K && V && O, "null tensor pointer");
  FOCUS_CHECK_ARG(B >= 0 && Hq >= 1 && Hkv >= 1 && L >= 8 && qcap >= 1,
                  "bad sizes B=%d Hq=%d Hkv=%d L=%d (>= 8) qcap=%d", B, Hq, Hkv, L, qcap);
  FOCUS_CHECK_ARG(Hq % Hkv == 0, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  FOCUS_CHECK_ARG(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O), "tensors must be 16-byte aligned");
  FOCUS_CHECK_ARG(static_cast<long long>(B) * Hkv <= 2147483647LL && static_cast<long long>(L) * d < (1LL << 31),
                  "tensor too large");
  return FOCUS_OK;
}

}  // namespace
}  // namespace focus

using namespace focus;

extern "C" size_t focus_dense_workspace_bytes(int B, int Hq, int Hkv, int L, int d, int qcap, int want_colsum) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || qcap <= 0 || Hq % Hkv) return 0;
  return plan_attention(B, Hq, Hkv, d, qcap, L, want_colsum != 0, L, 0, 0, false).total;
}

extern "C" int focus_dense_attention(const focus_bf16* Q, const int32_t* n_q, const focus_bf16* K,
                                     const focus_bf16* V, int B, int Hq, int Hkv, int L, int d, int qcap, float scale,
                                     focus_bf16* O, float* colsum_opt, void* ws, size_t ws_bytes, void* stream) {
  int st = check_common(Q, K, V, O, B, Hq, Hkv, L, d, qcap);
  if (st != FOCUS_OK) return st;
  if (d != 64 && d != 128) {
    set_error("head dim %d unsupported (64 or 128)", d);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (colsum_opt && (Hq / Hkv) * qcap > 256) {
    set_error("column sums need (Hq/Hkv)*qcap <= 256, got %d", (Hq / Hkv) * qcap);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (B == 0) return FOCUS_OK;
  const AttnPlan plan = plan_attention(B, Hq, Hkv, d, qcap, L, colsum_opt != nullptr, L, 0, 0, false);
  FOCUS_CHECK_ARG(ws_bytes >= plan.total && (plan.total == 0 || ws), "workspace too small: need %zu bytes, got %zu",
                  plan.total, ws_bytes);
  FOCUS_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "workspace must be 256-byte aligned");
  AttnArgs a{};
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  a.n_q = n_q;
  a.K = reinterpret_cast<const __nv_bfloat16*>(K);
  a.V = reinterpret_cast<const __nv_bfloat16*>(V);
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.qcap = qcap;
  a.g = Hq / Hkv;
  a.scale_log2 = scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? run_attention<128, false>(a, plan, ws, colsum_opt, s)
                  : run_attention<64, false>(a, plan, ws, colsum_opt, s);
}

extern "C" int focus_dense_attention_sinks(const focus_bf16* Q, const int32_t* n_q, const focus_bf16* K,
                                           const focus_bf16* V, int B, int Hq, int Hkv, int L, int d, int qcap,
                                           float scale, focus_bf16* O, float* colsum, int S, int32_t* sinks, void* ws,
                                           size_t ws_bytes, void* stream) {
  int st = check_common(Q, K, V, O, B, Hq, Hkv, L, d, qcap);
  if (st != FOCUS_OK) return st;
  FOCUS_CHECK_ARG(colsum && sinks, "null pointer argument");
  FOCUS_CHECK_ARG(S >= 1 && S <= 4096, "bad S=%d", S);
  if (d != 64 && d != 128) {
    set_error("head dim %d unsupported (64 or 128)", d);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if ((Hq / Hkv) * qcap > 256) {
    set_error("column sums need (Hq/Hkv)*qcap <= 256, got %d", (Hq / Hkv) * qcap);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (B == 0) return FOCUS_OK;
  const AttnPlan plan = plan_attention(B, Hq, Hkv, d, qcap, L, true, L, 0, 0, false);
  FOCUS_CHECK_ARG(ws_bytes >= plan.total && (plan.total == 0 || ws), "workspace too small: need %zu bytes, got %zu",
                  plan.total, ws_bytes);
  FOCUS_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "workspace must be 256-byte aligned");
  AttnArgs a{};
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  a.n_q = n_q;
  a.K = reinterpret_cast<const __nv_bfloat16*>(K);
  a.V = reinterpret_cast<const __nv_bfloat16*>(V);
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.qcap = qcap;
  a.g = Hq / Hkv;
  a.scale_log2 = scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool done = false;
  st = d == 128 ? run_attention<128, false>(a, plan, ws, colsum, s, sinks, S, &done)
                : run_attention<64, false>(a, plan, ws, colsum, s, sinks, S, &done);
  if (st != FOCUS_OK || done) return st;
  return focus_sink_identify(colsum, B, Hkv, L, S, sinks, stream);   // the top-S as its own launch
}

extern "C" int focus_full_refresh(const focus_bf16* Q, const focus_bf16* K, const focus_bf16* V, int B, int Hq,
                                  int Hkv, int L, int d, float scale, focus_bf16* O, int P, int bs, float* kbar,
                                  void* ws, size_t ws_bytes, void* stream) {
  int st = check_common(Q, K, V, O, B, Hq, Hkv, L, d, L);
  if (st != FOCUS_OK) return st;
  FOCUS_CHECK_ARG(kbar, "null pointer argument");
  FOCUS_CHECK_ARG(1 <= P && P <= L && bs >= 1, "need 1 <= P <= L and bs >= 1 (P=%d bs=%d L=%d)", P, bs, L);
  FOCUS_CHECK_ARG(aligned16(kbar), "kbar must be 16-byte aligned");
  if (d != 64 && d != 128) {
    set_error("head dim %d unsupported (64 or 128)", d);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (B == 0) return FOCUS_OK;
  if (refresh_supported(d, B, Hq, Hkv, L, device_sm_count()) && 128 % bs == 0)
    return refresh_attention(reinterpret_cast<const __nv_bfloat16*>(Q), nullptr,
                             reinterpret_cast<const __nv_bfloat16*>(K), reinterpret_cast<const __nv_bfloat16*>(V),
                             reinterpret_cast<__nv_bfloat16*>(O), B, Hq, Hkv, L, L, scale * kLog2e,
                             static_cast<cudaStream_t>(stream), kbar, P, bs);
  // other shapes: the dense attention and the block means as two launches
  st = focus_dense_attention(Q, nullptr, K, V, B, Hq, Hkv, L, d, L, scale, O, nullptr, ws, ws_bytes, stream);
  if (st != FOCUS_OK) return st;
  return focus_block_means(K, B, Hkv, L, d, P, bs, kbar, stream);
}

extern "C" size_t focus_sparse_workspace_bytes(int B, int Hq, int Hkv, int L, int d, int acap, int S, int C, int bs,
                                               int P, int g0, int g1) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || acap <= 0 || Hq % Hkv || bs <= 0 || C <= 0 || S < 0) return 0;
  const int nb = (P + bs - 1) / bs;
  const int br = box_rows_for(true, L, bs, g1 - g0);
  const long kv_cap = static_cast<long>(std::min(C, std::max(nb, 0))) * ((bs + 7) & ~7) + gen_pad_for(br, g1 - g0) +
                      gen_pad_for(br, std::min(S, kMaxSinks));
  return plan_attention(B, Hq, Hkv, d, acap, static_cast<int>(std::min<long>(kv_cap, 1 << 30)), false, L, S, C, true)
      .total;
}

extern "C" int focus_sparse_attention(const focus_bf16* Q_active, const int32_t* n_active, const focus_bf16* K,
                                      const focus_bf16* V, const int32_t* sinks, int S, const int32_t* blocks, int C,
                                      int bs, int P, int g0, int g1, int B, int Hq, int Hkv, int L, int d, int acap,
                                      float scale, focus_bf16* O_active, void* ws, size_t ws_bytes, void* stream) {
  int st = check_common(Q_active, K, V, O_active, B, Hq, Hkv, L, d, acap);
  if (st != FOCUS_OK) return st;
  if (d != 64 && d != 128) {
    set_error("head dim %d unsupported (64 or 128)", d);
    return FOCUS_ERR_UNSUPPORTED;
  }
  FOCUS_CHECK_ARG(n_active && blocks && (S == 0 || sinks), "null index pointer");
  FOCUS_CHECK_ARG(bs >= 1 && C >= 1 && S >= 0, "bad bs=%d C=%d S=%d", bs, C, S);
  if (C > kMaxBlocks) {
    set_error("C=%d exceeds the %d kept blocks per KV head supported", C, kMaxBlocks);
    return FOCUS_ERR_UNSUPPORTED;
  }
  FOCUS_CHECK_ARG(0 <= P && P <= g0 && g0 < g1 && g1 <= L, "need 0 <= P <= g0 < g1 <= L (P=%d g0=%d g1=%d L=%d)", P,
                  g0, g1, L);
  if (S > kMaxSinks) {
    set_error("S=%d exceeds the %d sinks per KV head supported", S, kMaxSinks);
    return FOCUS_ERR_UNSUPPORTED;
  }
  if (B == 0) return FOCUS_OK;
  const int nb = (P + bs - 1) / bs;
  const int br = box_rows_for(true, L, bs, g1 - g0);
  const long kv_cap = static_cast<long>(std::min(C, nb)) * ((bs + 7) & ~7) + gen_pad_for(br, g1 - g0) +
                      gen_pad_for(br, S);
  FOCUS_CHECK_ARG(kv_cap < (1L << 30), "key set too large");
  const AttnPlan plan = plan_attention(B, Hq, Hkv, d, acap, static_cast<int>(kv_cap), false, L, S, C, true);
  FOCUS_CHECK_ARG(ws_bytes >= plan.total && (plan.total == 0 || ws), "workspace too small: need %zu bytes, got %zu",
                  plan.total, ws_bytes);
  FOCUS_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "workspace must be 256-byte aligned");
  AttnArgs a{};
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q_active);
  a.n_q = n_active;
  a.K = reinterpret_cast<const __nv_bfloat16*>(K);
  a.V = reinterpret_cast<const __nv_bfloat16*>(V);
  a.O = reinterpret_cast<__nv_bfloat16*>(O_active);
  a.sinks = sinks;
  a.blocks = blocks;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.qcap = acap;
  a.g = Hq / Hkv;
  a.S = S;
  a.C = C;
  a.bs = bs;
  a.P = P;
  a.g0 = g0;
  a.g1 = g1;
  a.scale_log2 = scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? run_attention<128, true>(a, plan, ws, nullptr, s)
                  : run_attention<64, true>(a, plan, ws, nullptr, s);
}

extern "C" int focus_sparse_attention_fused(const focus_bf16* Q_active, const int32_t* n_active, const focus_bf16* K,
                                            const focus_bf16* V, const float* kbar, int nb, int C,
                                            const int32_t* sinks, int S, int bs, int P, int g0, int g1, int B, int Hq,
                                            int Hkv, int L, int d, int acap, float scale, int32_t* blocks,
                                            focus_bf16* O_active, void* ws, size_t ws_bytes, void* stream) {
  int st = check_common(Q_active, K, V, O_active, B, Hq, Hkv, L, d, acap);
  if (st != FOCUS_OK) return st;
  FOCUS_CHECK_ARG(n_active && kbar && blocks && (S == 0 || sinks), "null pointer argument");
  FOCUS_CHECK_ARG(aligned16(kbar), "kbar must be 16-byte aligned");
  FOCUS_CHECK_ARG(nb == (P + bs - 1) / bs && nb >= 1, "nb (%d) must equal ceil(P / bs)", nb);
  if (!decode_fused_supported(d, Hq, Hkv, acap, L, S, C, nb)) {
    // shapes the fused kernel does not take: the two calls in sequence
    st = focus_block_select(Q_active, n_active, kbar, B, Hq, Hkv, d, acap, nb, C, blocks, nullptr, stream);
    if (st != FOCUS_OK) return st;
    return focus_sparse_attention(Q_active, n_active, K, V, sinks, S, blocks, C, bs, P, g0, g1, B, Hq, Hkv, L, d,
                                  acap, scale, O_active, ws, ws_bytes, stream);
  }
  FOCUS_CHECK_ARG(bs >= 1 && C >= 1 && S >= 0, "bad bs=%d C=%d S=%d", bs, C, S);
  FOCUS_CHECK_ARG(0 <= P && P <= g0 && g0 < g1 && g1 <= L, "need 0 <= P <= g0 < g1 <= L (P=%d g0=%d g1=%d L=%d)", P,
                  g0, g1, L);
  if (B == 0) return FOCUS_OK;
  return decode_attention(reinterpret_cast<const __nv_bfloat16*>(Q_active), n_active,
                          reinterpret_cast<const __nv_bfloat16*>(K), reinterpret_cast<const __nv_bfloat16*>(V),
                          reinterpret_cast<__nv_bfloat16*>(O_active), nullptr, sinks, nullptr, S, C, bs, P, g0, g1, true,
                          B, Hq, Hkv, L, acap, scale * kLog2e, static_cast<cudaStream_t>(stream), kbar, nb, blocks);
}
