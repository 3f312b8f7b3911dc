// Dense bidirectional attention for many query rows on the sm_100a tensor cores: the
// block-entry full refresh of Focus-dLLM (summary page, "半自回归重遮蔽策略" / semi-AR
// remasking: at block entry the whole sequence runs dense attention and the caches are
// refreshed) and any dense call with enough rows to fill the GPU.
//
// CTA = 256 rows of one KV-head group (two 128-row query tiles Q0, Q1; row r of the group
// is query head r / qcap, position r % qcap, and the group's rows are contiguous in Q), all
// L keys in 128-key tiles. Ten warps:
//   warps 0-3  softmax of Q0 (one row per thread), warps 4-7 softmax of Q1;
//   warp 8     producer: TMA for Q once, then K and V tiles through separate rings;
//   warp 9     tcgen05.mma issuer and owner of all 512 tensor-memory columns.
// Tensor memory: S0 | S1 | O0 | O1, 128 fp32 columns each. A softmax thread reads its row
// of S_i, turns it into P = 2^(s*scale*log2e - m) and writes P back as bf16 pairs over the
// first 64 columns of S_i; O_i += P_i V is then issued with P_i as the tensor-memory A
// operand, so P never goes through shared memory. The issue order
//   QK0(0) QK1(0) | PV0(j) QK0(j+1) PV1(j) QK1(j+1) | ...
// lets the tensor cores work on one tile's products while the other warpgroup turns its
// scores into probabilities (MMAs from one thread run in issue order, so QK_i(j+1) writes
// S_i only after PV_i(j) has read P_i). Each row keeps a reference maximum m: p = 2^(s - m)
// while every s stays below m + 8; a tile that would exceed it moves m up and rescales the
// row of O_i in tensor memory (after PV_i(j-1) has landed). Row sums are per-thread.
//
// Block entry (method steps (4): a prompt block is represented by the mean of its keys,
// computed once per generation block): with kbar requested, the K tiles that stream through
// the CTAs anyway also give the block means. K tile t of the prompt is summed by row block
// t mod (row blocks of the head) -- every row block of a head streams every tile, so each
// tile is summed exactly once -- by the producer warp, between issuing tile t + 1 and
// refilling t's ring stage.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "focus_common.cuh"

namespace focus {

constexpr int kRfThreads = 320;
constexpr int kRfProducerWarp = 8;
constexpr int kRfMmaWarp = 9;
constexpr int kRfKStages = 3;
constexpr int kRfVStages = 2;
constexpr int kRfD = 128;

struct RfArgs {
  const int32_t* n_q;      // [B] valid positions per sequence, or null (all qcap)
  __nv_bfloat16* O;        // [B, Hq, qcap, 128]
  int B, Hq, Hkv, L, qcap, g;
  int rows;                // g * qcap rows per KV group
  float scale_log2;
  int* dev_err;
  // block means of the prompt (block entry): kbar [B, Hkv, nb, 128] fp32 of the blocks
  // [j*bs, min(P, (j+1)*bs)), bs dividing 128; null when not wanted
  float* kbar;
  int P, bs, nb;
};

struct __align__(8) RfBook {
  uint64_t q_full;
  uint64_t k_full[kRfKStages], k_empty[kRfKStages];
  uint64_t v_full[kRfVStages], v_empty[kRfVStages];
  uint64_t s_full[2], p_full[2], o_done[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct RfSmem {
  static constexpr uint32_t kTile = 128 * kRfD * 2;                 // 32 KB
  static constexpr uint32_t kQ = 0;                                 // Q0, Q1
  static constexpr uint32_t kK = 2 * kTile;
  static constexpr uint32_t kV = kK + kRfKStages * kTile;
  static constexpr uint32_t kBook = kV + kRfVStages * kTile;
  static constexpr uint32_t kBytes = kBook + sizeof(RfBook) + 1024;
  static_assert(kBytes <= 232448, "refresh kernel exceeds the 227 KB of shared memory per CTA");
};

// D(tmem) (+)= A(tmem) x B(smem desc), kind::f16 (bf16 inputs, fp32 accumulate); A is M x K
// in tensor memory, row m in lane m, K elements packed two to a 32-bit column.
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ bool rf_wait_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 500000000ull) return false;
  }
  return true;
}

// fp32 pairs (f32x2): one instruction forms the exponent arguments of two keys, and one
// adds two probabilities to two of the row-sum chains
__device__ __forceinline__ unsigned long long f2_pack(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__global__ void __launch_bounds__(kRfThreads, 1)
    refresh_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ RfArgs a) {
  using SM = RfSmem;
  constexpr int D = kRfD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  RfBook* bk = reinterpret_cast<RfBook*>(smem + SM::kBook);
  const int warp = warp_id(), lane = lane_id();
  const int m0 = static_cast<int>(blockIdx.x) * 256;
  const int bh = blockIdx.y;                   // b * Hkv + kvh
  const int b = bh / a.Hkv;
  const int n_kt = (a.L + 127) / 128;
  volatile int* abort_flag = &bk->abort_flag;

  // ---- set-up that reads no input (before the wait for the previous kernel)
  if (warp == kRfProducerWarp) {
    if (lane == 0) {
      mbar_init(&bk->q_full, 1);
      for (int s = 0; s < kRfKStages; ++s) {
        mbar_init(&bk->k_full[s], 1);
        mbar_init(&bk->k_empty[s], 1);
      }
      for (int s = 0; s < kRfVStages; ++s) {
        mbar_init(&bk->v_full[s], 1);
        mbar_init(&bk->v_empty[s], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bk->s_full[i], 1);
        mbar_init(&bk->p_full[i], 4);
        mbar_init(&bk->o_done[i], 1);
      }
      mbar_init(&bk->drain, 1);
      bk->abort_flag = 0;
      fence_mbar_init();
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
  } else if (warp == kRfMmaWarp) {
    tmem_alloc(&bk->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();
  const uint32_t tmem = bk->tmem_base;

  if (warp == kRfProducerWarp) {
    // ------------------------------------------------------------ producer
    // Lane 0 issues the copies; with kbar requested the whole warp sums this CTA's prompt
    // tiles (lane l: dims 4l .. 4l+3 of every row, read from the SW128 tile).
    const int n_ptiles = a.kbar ? (a.P + 127) / 128 : 0;
    auto block_means_of = [&](int t) {
      if (t >= n_ptiles || t % static_cast<int>(gridDim.x) != static_cast<int>(blockIdx.x)) return true;
      const int ks = t % kRfKStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&bk->k_full[ks], (t / kRfKStages) & 1, abort_flag, a.dev_err,
                                             DEV_ERR_TIMEOUT_PRODUCER)))
        return false;
      const uint8_t* tile = sK + ks * SM::kTile;
      const int c = lane >> 1;                                // 16-byte chunk of the row
      const uint32_t base = static_cast<uint32_t>((c >> 3) * (128 * 128) + (lane & 1) * 8);
      for (int r0 = 0; r0 < 128; r0 += a.bs) {
        const int blk = (t * 128 + r0) / a.bs;
        const int n = min(a.bs, a.P - blk * a.bs);            // valid rows of the block
        if (n <= 0) break;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = r0; r < r0 + n; ++r) {
          const uint2 v = *reinterpret_cast<const uint2*>(tile + base + r * 128 + (((c & 7) ^ (r & 7)) << 4));
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
          acc.x += f0.x;
          acc.y += f0.y;
          acc.z += f1.x;
          acc.w += f1.y;
        }
        const float inv = 1.f / static_cast<float>(n);
        reinterpret_cast<float4*>(a.kbar + (static_cast<size_t>(bh) * a.nb + blk) * D)[lane] =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      }
      return true;
    };
    int k_issued = 0, v_issued = 0;
    if (lane == 0) {
      // no evict-first hint: the other row blocks of the same KV head, resident at the same
      // time, read the same K and V tiles out of L2
      mbar_arrive_expect_tx(&bk->q_full, 2u * SM::kTile);
      for (int t = 0; t < 2; ++t)
        for (int at = 0; at < 2; ++at)
          tma_load_3d(smem_u32(sQ + t * SM::kTile + at * (128 * 128)), &tmQ, &bk->q_full, at * 64, m0 + t * 128, bh);
    }
    bool ok = true;
    for (int j = 0; j < n_kt && ok; ++j) {
      const int ks = j % kRfKStages, vs = j % kRfVStages;
      if (lane == 0) {
        if (j >= kRfKStages &&
            !mbar_wait(&bk->k_empty[ks], ((j / kRfKStages) - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_PRODUCER))
          ok = false;
        if (ok) {
          mbar_arrive_expect_tx(&bk->k_full[ks], SM::kTile);
          for (int at = 0; at < 2; ++at)
            tma_load_3d(smem_u32(sK + ks * SM::kTile + at * (128 * 128)), &tmK, &bk->k_full[ks], at * 64, j * 128,
                        bh);
          ++k_issued;
        }
        if (ok && j >= kRfVStages &&
            !mbar_wait(&bk->v_empty[vs], ((j / kRfVStages) - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_PRODUCER))
          ok = false;
        if (ok) {
          mbar_arrive_expect_tx(&bk->v_full[vs], SM::kTile);
          for (int at = 0; at < 2; ++at)
            tma_load_3d(smem_u32(sV + vs * SM::kTile + at * (128 * 128)), &tmV, &bk->v_full[vs], at * 64, j * 128,
                        bh);
          ++v_issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // tile j - 1 has been issued a ring's depth before its stage is refilled (by this warp)
      if (ok && j >= 1) ok = block_means_of(j - 1);
    }
    if (ok && n_kt >= 1) block_means_of(n_kt - 1);
    if (lane == 0) {
      // never leave with copies in flight
      rf_wait_drain(&bk->q_full, 0);
      for (int j = max(0, k_issued - kRfKStages); j < k_issued; ++j)
        rf_wait_drain(&bk->k_full[j % kRfKStages], (j / kRfKStages) & 1);
      for (int j = max(0, v_issued - kRfVStages); j < v_issued; ++j)
        rf_wait_drain(&bk->v_full[j % kRfVStages], (j / kRfVStages) & 1);
    }
    __syncwarp();
  } else if (warp == kRfMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t kTileDesc = SM::kTile >> 4;
      // descriptors formed once; a K step or a stage adds a constant to the 14-bit
      // start-address field (address >> 4), which cannot carry: shared memory < 256 KB
      const uint64_t q_desc0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t v_desc0 = sw128_desc(smem_u32(sV), 128 * 128, 1024);
      auto qk = [&](int i, int j) {
        const uint64_t qd = q_desc0 + static_cast<uint64_t>(i * kTileDesc);
        const uint64_t kd = k_desc0 + static_cast<uint64_t>((j % kRfKStages) * kTileDesc);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128 / 16) + (kk & 3) * 2;
          mma_bf16(tmem + i * 128, qd + koff, kd + koff, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bk->s_full[i]);
      };
      auto pv = [&](int i, int j) {
        const uint64_t vd = v_desc0 + static_cast<uint64_t>((j % kRfVStages) * kTileDesc);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_bf16_tmem_a(tmem + 256 + i * 128, tmem + i * 128 + kk * 8, vd + kk * (2048 / 16), idesc_pv,
                          (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bk->o_done[i]);
      };
      bool ok = mbar_wait(&bk->q_full, 0, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA) &&
                mbar_wait(&bk->k_full[0], 0, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA);
      if (ok) {
        tc_fence_after();
        qk(0, 0);
        qk(1, 0);
        mma_commit(&bk->k_empty[0]);
      }
      for (int j = 0; ok && j < n_kt; ++j) {
        const bool more = j + 1 < n_kt;
        const int kn = (j + 1) % kRfKStages;
        ok = mbar_wait(&bk->v_full[j % kRfVStages], (j / kRfVStages) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA) &&
             mbar_wait(&bk->p_full[0], j & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA);
        if (!ok) break;
        tc_fence_after();
        pv(0, j);
        if (more) {
          if (!mbar_wait(&bk->k_full[kn], ((j + 1) / kRfKStages) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA))
            break;
          tc_fence_after();
          qk(0, j + 1);
        }
        if (!mbar_wait(&bk->p_full[1], j & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        pv(1, j);
        mma_commit(&bk->v_empty[j % kRfVStages]);
        if (more) {
          qk(1, j + 1);
          mma_commit(&bk->k_empty[kn]);
        }
      }
      // every MMA has completed before tensor memory is released
      mma_commit(&bk->drain);
      rf_wait_drain(&bk->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0..7
    const int wg = warp >> 2, qd = warp & 3;
    const int rr = wg * 128 + qd * 32 + lane;    // row within this CTA's 256
    const int r = m0 + rr;                       // row of the group
    const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t tS = tmem + wg * 128 + lane_addr;
    const uint32_t tO = tmem + 256 + wg * 128 + lane_addr;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bk->s_full[wg], j & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_SOFTMAX))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the raw scores of this row (the four loads in flight together); the scale is applied
      // inside the exponent's FFMA, and the maximum is taken on raw scores (scale > 0)
      uint32_t sr[128];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sr + 64));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(sr + 96));
      tmem_ld_wait();
      float* sv = reinterpret_cast<float*>(sr);
      const int nvalid = a.L - j * 128;             // keys of this tile inside [0, L)
      if (nvalid < 128) {                           // only the last tile can be partial
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k >= nvalid) sv[k] = -INFINITY;
      }
      // the row maximum over eight independent chains (max is exact in any order)
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = sv[u];
#pragma unroll
      for (int k = 8; k < 128; ++k) mx[k & 7] = fmaxf(mx[k & 7], sv[k]);
      const float mr =
          fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float mt = mr * a.scale_log2;
      // keep the reference maximum unless it grows by more than 2^8 (p stays <= 256)
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + 8.f || (m_ref == -INFINITY && mt > -INFINITY)) {
        alpha = (m_ref == -INFINITY) ? 0.f : exp2_approx(m_ref - mt);
        m_ref = mt;
        rescale = true;
      }
      const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
      const float c2 = a.scale_log2;
      // P over the first 64 columns of S_i, 32 keys at a time. This thread has read its whole
      // row of S, and PV_i(j - 1), which read the previous P, completed before QK_i(j)
      // signalled s_full.
      const unsigned long long c2x2 = f2_pack(c2, c2), nm2 = f2_pack(neg_m, neg_m);
      unsigned long long lsc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};   // four row-sum chains
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(sv[32 * c + 2 * k], sv[32 * c + 2 * k + 1]), c2x2, nm2), x0, x1);
          const float p0 = exp2_approx(x0);
          const float p1 = exp2_approx(x1);
          lsc2[k & 1] = f2_add(lsc2[k & 1], f2_pack(p0, p1));
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);
      }
      float l0, l1, l2, l3;
      f2_unpack(lsc2[0], l0, l1);
      f2_unpack(lsc2[1], l2, l3);
      const float ls = (l0 + l2) + (l1 + l3);
      l_sum = l_sum * alpha + ls;
      if (j > 0 && __any_sync(0xffffffffu, rescale && alpha != 1.f)) {
        // O_i must hold PV_i(j - 1) before its rows are rescaled
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bk->o_done[wg], (j - 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_SOFTMAX))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float al = rescale ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rg[32];
          tmem_ld32(tO + c * 32, rg);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) rg[k] = __float_as_uint(__uint_as_float(rg[k]) * al);
          tmem_st32(tO + c * 32, rg);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->p_full[wg]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n_kt > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&bk->o_done[wg], (n_kt - 1) & 1, abort_flag, a.dev_err,
                                             DEV_ERR_TIMEOUT_EPILOGUE));
    if (ok) {
      tc_fence_after();
      const bool row_exists = r < a.rows;
      const int qh = row_exists ? r / a.qcap : 0;
      const int i = r - qh * a.qcap;
      const int nq = a.n_q ? min(a.n_q[b], a.qcap) : a.qcap;
      const float inv_l = (row_exists && i < nq && l_sum > 0.f) ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow =
          a.O + ((static_cast<size_t>(b) * a.Hq + static_cast<size_t>(bh % a.Hkv) * a.g + qh) * a.qcap + i) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rg[32];
        tmem_ld32(tO + c * 32, rg);
        tmem_ld_wait();
        if (row_exists) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(rg[k4 * 8 + 0]) * inv_l, __uint_as_float(rg[k4 * 8 + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(rg[k4 * 8 + 2]) * inv_l, __uint_as_float(rg[k4 * 8 + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(rg[k4 * 8 + 4]) * inv_l, __uint_as_float(rg[k4 * 8 + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(rg[k4 * 8 + 6]) * inv_l, __uint_as_float(rg[k4 * 8 + 7]) * inv_l);
            reinterpret_cast<uint4*>(orow + c * 32)[k4] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kRfMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 rf_encode_fn() {
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

// [outer, rows, 128] bf16 with 128-row x 64-column boxes (SWIZZLE_128B); rows past `rows`
// read as zeros.
int rf_make_map(CUtensorMap* map, const void* base, int outer, int rows) {
  auto fn = rf_encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled is unavailable (driver entry point lookup failed)");
    return FOCUS_ERR_CUDA;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kRfD), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kRfD) * 2, static_cast<cuuint64_t>(rows) * kRfD * 2};
  cuuint32_t box[3] = {64u, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (CUresult %d) for [%d, %d, 128]", static_cast<int>(r), outer, rows);
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

}  // namespace

// Whether the many-row kernel serves a dense call: d = 128 and enough 256-row blocks to
// give every SM at least one (with fewer rows the split-KV tile kernel keeps the SMs busy).
bool refresh_supported(int d, int B, int Hq, int Hkv, int qcap, int sms) {
  if (d != kRfD) return false;
  const long rows = static_cast<long>(Hq / Hkv) * qcap;
  const long blocks = static_cast<long>(B) * Hkv * ((rows + 255) / 256);
  return rows >= 256 && blocks >= sms && (rows + 255) / 256 <= 2147483647L && static_cast<long>(B) * Hkv <= 65535;
}

int refresh_attention(const __nv_bfloat16* Q, const int32_t* n_q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                      __nv_bfloat16* O, int B, int Hq, int Hkv, int L, int qcap, float scale_log2,
                      cudaStream_t stream, float* kbar, int P, int bs) {
  RfArgs a{};
  a.n_q = n_q;
  a.O = O;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.qcap = qcap;
  a.g = Hq / Hkv;
  a.rows = a.g * qcap;
  a.scale_log2 = scale_log2;
  a.dev_err = device_error_word();
  a.kbar = kbar;
  a.P = P;
  a.bs = bs;
  a.nb = kbar ? (P + bs - 1) / bs : 0;
  CUtensorMap mq, mk, mv;
  int st = rf_make_map(&mq, Q, B * Hkv, a.rows);
  if (st != FOCUS_OK) return st;
  st = rf_make_map(&mk, K, B * Hkv, L);
  if (st != FOCUS_OK) return st;
  st = rf_make_map(&mv, V, B * Hkv, L);
  if (st != FOCUS_OK) return st;
  if (const int s = configure_dynamic_smem(reinterpret_cast<const void*>(refresh_attn_kernel),
                                           static_cast<int>(RfSmem::kBytes), "refresh attention"))
    return s;
  const dim3 grid((a.rows + 255) / 256, B * Hkv);
  const cudaError_t e = launch_k(refresh_attn_kernel, grid, dim3(kRfThreads), RfSmem::kBytes, stream, mq, mk, mv, a);
  note_launch();
  if (e != cudaSuccess) {
    set_error("refresh attention launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

}  // namespace focus
