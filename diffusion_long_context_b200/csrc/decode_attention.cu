// Few-query ("decode") attention on the sm_100a tensor cores, swap-AB form.
//
// Serves the attentions of a Focus-dLLM sparse step, where only the active queries
// (about 32 per head) attend:
//   * dense  (method steps (3)): the active queries over all L keys;
//   * sparse (method steps (5)): the active queries over I_p = sinks U kept prompt
//     blocks U current block (slot layout in slots.cuh).
// With so few queries the 128 keys of a tile are the MMA's M dimension and the queries
// its N dimension (up to 64 rows of a KV group per CTA; larger groups are cut into row
// slices, one cluster each):
//   S^T[key, q] = K_tile . Q^T        (M = 128 keys, N = NQ queries, K = d)   -> TMEM
//   O^T[dim, q] += V_tile^T . P^T      (M = d = 128, N = NQ, K = 128 keys)    -> TMEM
// V_tile^T is the V tile read as an MN-major A operand; P (bf16) is written to shared
// memory query-major. A softmax thread owns one key of the tile (and one dim of O^T).
// Each query keeps a reference maximum m_q shared by all keys: p = 2^(s - m_q) while every
// s stays below m_q + 8; a tile that would exceed it (and the first tile) takes the slow
// path: the exact per-query tile maximum is reduced across the 128 threads, m_q moves up
// and O^T and the row sums are rescaled. Row sums are per-thread partials reduced once
// at the end.
//
// Split-KV: the CTAs of one (sequence, KV head) form a thread-block cluster. CTA r takes
// the key tiles r, r + cs, ... for its first ring round and then claims further tiles from
// a counter in CTA 0 (one claim in flight, planned while its stage drains); the partial
// results (m, l, O) are merged through distributed shared memory -- no workspace and no
// second launch. The fused form first selects the kept blocks itself (relevance + top-C).
//
// Warps: 0-7 softmax / epilogue (two per TMEM lane quadrant, each taking half of the
// query columns), 8 producer (TMA for key runs, cp.async for sink rows), 9 tcgen05.mma
// issuer and TMEM owner. K/V tiles flow through a STAGES-deep ring.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "focus_common.cuh"
#include "slots.cuh"
#include "topk.cuh"

namespace focus {

constexpr int kDecSoftmaxWarps = 8;   // two per TMEM lane quadrant, each half of the queries
constexpr int kDecSoftmaxThreads = kDecSoftmaxWarps * 32;
constexpr int kDecThreads = kDecSoftmaxThreads + 64;
constexpr int kDecD = 128;
constexpr int kDecMaxBlocks = 512;
constexpr int kDecMaxSinks = 512;
// Query rows per KV group the decode kernel serves: above 64 the group's rows are cut into
// slices of 64, one cluster per slice (GQA 7:1 at 32 active queries = 4 slices). Each slice
// streams the group's keys again (from L2 when the slices run together), so beyond a few
// slices the 128-row tile kernel, which reads the keys once per 128 rows, is the better fit.
constexpr int kDecMaxRows = 256;
constexpr int kDecProducerWarp = kDecSoftmaxWarps;
constexpr int kDecMmaWarp = kDecSoftmaxWarps + 1;

struct DecArgs {
  const __nv_bfloat16* Q;      // [B, Hq, qcap, D]
  const int32_t* n_q;          // [B] or null
  const __nv_bfloat16* K;      // [B, Hkv, L, D]
  const __nv_bfloat16* V;
  __nv_bfloat16* O;            // [B, Hq, qcap, D]
  float* lse_out;              // [B, Hq, qcap] log2 domain, or null
  const int32_t* sinks;        // [B, Hkv, S]
  const int32_t* blocks;       // [B, Hkv, C] (unfused sparse)
  const float* kbar;           // [B, Hkv, nb, D] (fused sparse: relevance + top-C in the prologue)
  int32_t* blocks_out;         // [B, Hkv, C] kept blocks written by the fused kernel, or null
  int nb;
  int B, Hq, Hkv, L, qcap, g;
  int n_slices;                // clusters per (b, kv head): the group's rows in slices of NQ
  int box_rows;                // rows per TMA box (divides 128)
  int gen_pad;                 // slots of the current block (multiple of box_rows)
  int S, C, bs, P, g0, g1;
  float scale_log2;
  FastDiv pad_div, bs_div, qcap_div;   // by round_up(bs, 8), bs and qcap (host-computed)
  int* dev_err;
  // dense sink layer (column-sum form): colsum [B, Hkv, L] of the softmax rows, and
  // optionally the top-S columns sinks_out [B, Hkv, S_out] selected by the cluster
  float* colsum;
  int32_t* sinks_out;
  int S_out;
};

struct __align__(8) DecBook {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  SlotLayout sl;
  float mref[64];
  float alpha[64];
  float lfin[64];
  float red[4][64];
  int blk[kDecMaxBlocks];
  int sinks[kDecMaxSinks];
  TopkShared tk;
  uint64_t kb_bar;         // kbar rows staged by bulk copy (fused relevance prologue)
  uint64_t q_bar;          // the group's query rows staged by bulk copy (fused relevance prologue)
  uint32_t qvalid[2];      // bit q: query column q is a real query
  uint32_t tile_ctr;       // next dynamically claimed tile (CTA 0 of the cluster)
  int stage_tile[4];       // tile held by each ring stage, -1 = no more tiles
  // column-sum pass of the sink layer: a K-only ring over the idle K ring and the part of
  // the V ring the merge does not read
  uint64_t c_full[6], c_empty[6], c_sfull[2], c_sfree[2];
  int c_tile[6];           // tile held by each column-sum slot
  int c_stile[2];          // tile whose scores an S buffer holds, -1 = end
  float lse2[64];          // log2-domain log-sum-exp of every query column (+inf: not a query)
};

template <int NQ, int STAGES>
struct DecSmem {
  static constexpr uint32_t kTile = 128 * kDecD * 2;            // 32 KB
  static constexpr uint32_t kQ = 0;                             // NQ rows x 256 B
  static constexpr uint32_t kK = ((NQ * kDecD * 2) + 1023) / 1024 * 1024;
  static constexpr uint32_t kV = kK + STAGES * kTile;
  static constexpr uint32_t kP = kV + STAGES * kTile;           // 2 x (NQ rows x 128 keys bf16)
  static constexpr uint32_t kBook = kP + 2 * NQ * 256;
  static constexpr uint32_t kBytes = kBook + sizeof(DecBook) + 1024;
  static constexpr uint32_t kTmemCols = (3 * NQ <= 128) ? 128 : 256;
  static_assert(kBytes <= 232448, "decode kernel exceeds the 227 KB of shared memory per CTA");
  static_assert(2 * NQ * 256 >= 4 * 4096, "fused relevance scores must fit in the P buffers");
};

__device__ __forceinline__ bool dec_wait_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 500000000ull) return false;
  }
  return true;
}

constexpr int kDecMaxNb = 4096;   // fused relevance scores held in the P buffers

// Top-C for more than 2 * kDecThreads blocks: out of line, so that the fused kernel's
// straight-line prologue stays short (it runs once per launch from a cold instruction cache).
__device__ __noinline__ void dec_top_c_large(const uint32_t* s_key, int nb, int C, int32_t* blk, TopkShared& tk,
                                             int* s_wide) {
  auto key_of = [&](int i) { return s_key[i]; };
  if (nb <= 4 * kDecThreads) block_topk_small<4>(key_of, nb, C, blk, C, tk, s_wide);
  else if (nb <= 8 * kDecThreads) block_topk_small<8>(key_of, nb, C, blk, C, tk, s_wide);
  else block_topk_ascending(key_of, nb, C, blk, C, tk);
}

// ------------------------------------------------------------------ sink layer
// Column sums of the dense sink layer (method steps (3): the attention distribution of the
// sink layer, aggregated over the active queries, identifies the sinks). They run after
// the cluster merge, once the log-sum-exp of every query is known:
//   colsum[b, h, key] = sum over query columns q of 2^(scale_log2 * s[key, q] - lse2[q]).
// CTA r takes the 128-key tiles p_n - 1 - r, p_n - 1 - r - cs, ...: from the last tile
// down (the tiles the attention pass read last first), with no claim round trip on the
// producer's path. The pass re-reads K from HBM: an evict-last or evict-normal hint on the
// attention pass's K loads (V evict-first) was measured to leave the column-sum pass at the
// same 6.1 TB/s or slower, i.e. no reuse out of L2 at this size (268 MB of K at 32K).
// K tiles flow through a CS-slot ring
// made of the K ring and the V-ring stages the merge does not read; S^T = K_tile . Q^T
// lands in the two S buffers of tensor memory; each softmax thread owns one key, the two
// query halves of a key are added through shared memory, and the key's sum is stored.
// Each key lane also keeps the largest sum it produced (one per tile residue it % m,
// m = ceil(S / 128)) in gmax: the bound decode_sink_topk starts from.
template <int NQ, int STAGES>
__device__ __noinline__ void decode_colsum_phase(const CUtensorMap* tmK, const DecArgs& a, DecBook* bk, uint8_t* sK,
                                                 uint8_t* sV, const uint8_t* sQ, uint32_t tmem, int bh, int rank,
                                                 int cs, uint32_t* gmax) {
  using SM = DecSmem<NQ, STAGES>;
  constexpr int D = kDecD;
  constexpr int QH = NQ / 2;
  constexpr uint32_t kPart = NQ * D * 4 + NQ * 8;              // the merge's partials, V ring start
  constexpr int V0 = static_cast<int>((kPart + SM::kTile - 1) / SM::kTile);
  constexpr int CS = STAGES + (STAGES > V0 ? STAGES - V0 : 0);
  static_assert(CS >= 2 && CS <= 6, "column-sum ring");
  const int warp = warp_id(), lane = lane_id();
  volatile int* abort_flag = &bk->abort_flag;
  __syncthreads();                             // lse2 of every query is in place
  if (*abort_flag) return;                     // uniform: read after a CTA barrier
  const int p_n = (a.L + 127) / 128;
  const int BR = a.box_rows;                   // dense layout: boxes of BR consecutive keys
  const int ngroups = 128 / BR;
  auto slot_addr = [&](int sl) -> uint8_t* {
    return sl < STAGES ? sK + sl * SM::kTile : sV + (V0 + sl - STAGES) * SM::kTile;
  };
  if (warp == kDecProducerWarp) {
    if (lane == 0) {
      const uint64_t l2_once = l2_evict_first_policy();   // the last read of these K rows
      for (int it = 0;; ++it) {
        const int sl = it % CS;
        if (it >= CS && !mbar_wait(&bk->c_empty[sl], ((it / CS) - 1) & 1, abort_flag, a.dev_err,
                                   DEV_ERR_TIMEOUT_PRODUCER))
          break;
        const int tile = p_n - 1 - (rank + it * cs);
        if (tile < 0) {
          bk->c_tile[sl] = -1;
          mbar_arrive(&bk->c_full[sl]);
          break;
        }
        int nbox = 0;
        for (int grp = 0; grp < ngroups; ++grp) nbox += (tile * 128 + grp * BR < a.L) ? 1 : 0;
        bk->c_tile[sl] = tile;
        mbar_arrive_expect_tx(&bk->c_full[sl], static_cast<uint32_t>(nbox * 2 * BR * 128));
        uint8_t* dK = slot_addr(sl);
        for (int grp = 0; grp < nbox; ++grp)
          for (int at = 0; at < 2; ++at)
            tma_load_3d_hint(smem_u32(dK + at * (128 * 128) + grp * BR * 128), tmK, &bk->c_full[sl], at * 64,
                             tile * 128 + grp * BR, bh, l2_once);
      }
    }
    __syncwarp();
  } else if (warp == kDecMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, NQ, false, false);
      const uint64_t q_desc = sw128_desc(smem_u32(sQ), 16, 1024);
      for (int it = 0;; ++it) {
        const int sl = it % CS, sb = it & 1;
        int tile = -1;
        if (mbar_wait(&bk->c_full[sl], (it / CS) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) tile = bk->c_tile[sl];
        // S buffer sb (and its tile id) are free once the softmax warps are done with tile it - 2
        if (it >= 2 && !mbar_wait(&bk->c_sfree[sb], ((it - 2) >> 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA))
          tile = -1;
        bk->c_stile[sb] = tile;
        if (tile >= 0) {
          tc_fence_after();
          const uint64_t kd = sw128_desc(smem_u32(slot_addr(sl)), 16, 1024);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_bf16(tmem + sb * NQ, kd + (ks >> 2) * (128 * 128 / 16) + (ks & 3) * 2,
                     q_desc + (ks >> 2) * (NQ * 128 / 16) + (ks & 3) * 2, idesc_qk, ks > 0 ? 1u : 0u);
          mma_commit(&bk->c_sfull[sb]);
          mma_commit(&bk->c_empty[sl]);
        } else {
          mbar_arrive(&bk->c_sfull[sb]);       // stands in for the commit
        }
        mbar_arrive(&bk->c_sfull[sb]);         // publishes c_stile[sb]
        if (tile < 0) break;
      }
    }
    __syncwarp();
  } else {
    const int t = threadIdx.x & 127, q0 = (warp >> 2) * QH;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* hbuf = &bk->red[0][0];              // [2][128]: the second query half's sums
    // group maxima for the top-S (decode_sink_topk): key lane t, tile residue it % m
    const int m = max(1, min(4, (a.S_out + 127) / 128));
    uint32_t gm[4] = {0u, 0u, 0u, 0u};
    int u = 0;                                 // it % m
    float lse[QH];
#pragma unroll
    for (int q = 0; q < QH; ++q) lse[q] = bk->lse2[q0 + q];
    for (int it = 0;; ++it) {
      const int sb = it & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bk->c_sfull[sb], (it >> 1) & 1, abort_flag, a.dev_err,
                                                        DEV_ERR_TIMEOUT_SOFTMAX));
      const int tile = ok ? bk->c_stile[sb] : -1;
      if (bar_red_or(1, kDecSoftmaxThreads, tile < 0 || *abort_flag != 0)) break;
      tc_fence_after();
      uint32_t rg[QH];
      tmem_ld_cols<QH>(tmem + lane_addr + sb * NQ + q0, rg);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->c_sfree[sb]);
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < QH; ++q) acc += exp2_approx(__uint_as_float(rg[q]) * a.scale_log2 - lse[q]);
      if (warp >= 4) hbuf[sb * 128 + t] = acc;
      named_bar_sync(1, kDecSoftmaxThreads);
      const int key = tile * 128 + t;
      if (warp < 4 && key < a.L) {
        const float v = acc + hbuf[sb * 128 + t];
        a.colsum[static_cast<size_t>(bh) * a.L + key] = v;
        const uint32_t kv = float_order_key(v);
#pragma unroll
        for (int x = 0; x < 4; ++x)
          if (x == u) gm[x] = max(gm[x], kv);
      }
      if (++u == m) u = 0;
    }
    if (warp < 4)
      for (int x = 0; x < m; ++x) gmax[x * 128 + t] = gm[x];
  }
}

// Top-S sinks of the sink layer's column sums, selected inside the cluster (core method:
// the sinks found at the sink layer are reused by every deeper layer). Order: larger
// column sum first, ties to the lower column; the output lists the S columns ascending.
//
// Each CTA selects the top-S of the columns its own column-sum pass produced (its tiles
// t0, t0 + cs, ...), then CTA 0 selects the top-S of the cs * S candidates:
//  1. A lower bound T of this CTA's S-th largest column sum: during the pass every key
//     lane t (and, for S > 128, every tile residue it % m) keeps the maximum of the sums it
//     produced, so there are 128 * m >= S group maxima, each one of the sums; the S-th
//     largest of them is at most the S-th largest sum. Every sum of the top-S is >= T.
//  2. The sums >= T are appended to a candidate list (a shared counter; typically a few
//     dozen of the 8192 columns at 32K). Each is packed as (order key << 32) | ~column, so
//     that one 64-bit comparison orders by sum and then by lower column, and all packed
//     values are distinct.
//  3. The top-S of the candidates by rank counting (rank = number of larger packed values).
//     When more candidates than kSinkCand qualify (many equal sums), the CTA runs the
//     general radix selection over all its columns instead.
//  4. Each CTA writes its S best into CTA 0 (distributed shared memory); after a cluster
//     barrier CTA 0 ranks the cs * S candidates the same way and writes the S columns of
//     the top-S in ascending order.
constexpr int kSinkCand = 1024;              // candidates a CTA ranks directly
constexpr int kSinkCand0 = 2048;             // cs * S candidates of the cluster (CTA 0)

__device__ __forceinline__ uint64_t sink_pack(uint32_t key, int col) {
  return (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(col));
}
__device__ __forceinline__ int sink_col(uint64_t p) { return static_cast<int>(~static_cast<uint32_t>(p)); }

// Rank of every packed value v[i], i < n, among v[0 .. n) (the number of larger values;
// the nonzero values are distinct): v[i] goes to out[rank] when rank < k, so out comes out
// in descending order.
__device__ __forceinline__ void sink_rank_select(const uint64_t* v, int n, int k, uint64_t* out) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint64_t x = v[i];
    int r = 0;
    for (int j = 0; j < n; ++j) r += v[j] > x ? 1 : 0;
    if (r < k) out[r] = x;
  }
}

__device__ __noinline__ void decode_sink_topk(const DecArgs& a, DecBook* bk, uint8_t* ws, const uint32_t* gmax, int bh,
                                              int rank, int cs) {
  const int S = a.S_out;
  const int ng = 128 * max(1, min(4, (S + 127) / 128));   // group maxima (decode_colsum_phase)
  const int p_n = (a.L + 127) / 128;
  const int last = p_n - 1 - rank;                     // this CTA's highest tile
  const int n_own = last >= 0 ? last / cs + 1 : 0;
  const int t0 = last - (n_own - 1) * cs;              // its lowest tile
  const int n_pos = n_own * 128;                       // its positions, in ascending column order
  uint64_t* cand = reinterpret_cast<uint64_t*>(ws);                    // [kSinkCand]
  uint64_t* best = cand + kSinkCand;                                   // [kDecMaxSinks]
  uint64_t* cand0 = best + kDecMaxSinks;                               // [kSinkCand0] (CTA 0)
  int* s_cnt = reinterpret_cast<int*>(cand0 + kSinkCand0);
  uint32_t* s_T = reinterpret_cast<uint32_t*>(s_cnt + 1);
  int32_t* s_pos = reinterpret_cast<int32_t*>(s_T + 1);                // [kDecMaxSinks] (fallback)
  const float* row = a.colsum + static_cast<size_t>(bh) * a.L;
  auto col_of = [&](int pos) { return (t0 + (pos >> 7) * cs) * 128 + (pos & 127); };
  if (threadIdx.x == 0) {
    *s_cnt = 0;
    *s_T = 0u;
  }
  for (int i = threadIdx.x; i < S; i += blockDim.x) best[i] = 0ull;
  __syncthreads();
  // 1. T = the S-th largest group maximum (equal maxima ranked by group index)
  for (int i = threadIdx.x; i < ng; i += blockDim.x) {
    const uint32_t x = gmax[i];
    int r = 0;
    for (int j = 0; j < ng; ++j) {
      const uint32_t y = gmax[j];
      r += (y > x || (y == x && j < i)) ? 1 : 0;
    }
    if (r == S - 1) *s_T = x;
  }
  __syncthreads();
  const uint32_t T = *s_T;
  // 2. the candidates: this CTA's column sums >= T
  for (int pos = threadIdx.x; pos < n_pos; pos += blockDim.x) {
    const int col = col_of(pos);
    if (col >= a.L) continue;
    const uint32_t key = float_order_key(__ldcg(row + col));
    if (key >= T) {
      const int slot = atomicAdd(s_cnt, 1);
      if (slot < kSinkCand) cand[slot] = sink_pack(key, col);
    }
  }
  __syncthreads();
  const int n_cand = *s_cnt;
  // 3. this CTA's top-S, descending
  if (n_cand <= kSinkCand) {
    sink_rank_select(cand, n_cand, S, best);
  } else {
    // many equal sums: the radix selection over all of this CTA's columns (ties to the
    // lower position, i.e. the lower column)
    auto key_of = [&](int pos) {
      const int col = col_of(pos);
      return col < a.L ? float_order_key(__ldcg(row + col)) : 0u;
    };
    block_topk_ascending(key_of, n_pos, S, s_pos, S, bk->tk);
    __syncthreads();
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
      const int pos = s_pos[i];
      const int col = pos >= 0 ? col_of(pos) : a.L;
      cand[i] = col < a.L ? sink_pack(float_order_key(__ldcg(row + col)), col) : 0ull;
    }
    __syncthreads();
    sink_rank_select(cand, S, S, best);
  }
  __syncthreads();
  // 4. the S best of every CTA into CTA 0 (list r at cand0[r * S]), then the cluster's top-S
  const uint32_t c0 = smem_u32(cand0);
  for (int i = threadIdx.x; i < S; i += blockDim.x)
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(dsmem_addr(c0 + static_cast<uint32_t>(rank * S + i) * 8u, 0)),
                 "l"(best[i])
                 : "memory");
  if (cs > 1) cluster_sync();
  else __syncthreads();
  if (rank != 0) return;
  // rank of a candidate = its index in its own (descending) list + the entries larger than
  // it in every other list (binary search); the S of rank < S are the top-S
  for (int i = threadIdx.x; i < S; i += blockDim.x) best[i] = 0ull;
  __syncthreads();
  for (int e = threadIdx.x; e < cs * S; e += blockDim.x) {
    const uint64_t x = cand0[e];
    if (x == 0ull) continue;
    const int r = e / S;
    int rk = e - r * S;
    for (int o = 0; o < cs; ++o) {
      if (o == r) continue;
      const uint64_t* lst = cand0 + o * S;
      int lo = 0, hi = S;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (lst[mid] > x) lo = mid + 1;
        else hi = mid;
      }
      rk += lo;
    }
    if (rk < S) best[rk] = x;
  }
  __syncthreads();
  // the S columns in ascending order (S <= L, so all S are columns)
  int32_t* out = a.sinks_out + static_cast<size_t>(bh) * S;
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const int ci = sink_col(best[i]);
    int r = 0;
    for (int j = 0; j < S; ++j) r += sink_col(best[j]) < ci ? 1 : 0;
    out[r] = ci;
  }
}

template <int NQ, int STAGES, bool SPARSE, bool FUSED, bool COLSUM>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ DecArgs a) {
  using SM = DecSmem<NQ, STAGES>;
  constexpr int D = kDecD;
  constexpr int CH = D / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  uint8_t* sP = smem + SM::kP;
  DecBook* bk = reinterpret_cast<DecBook*>(smem + SM::kBook);

  const int warp = warp_id(), lane = lane_id();
  const int cs = gridDim.x;                    // CTAs per (b, h) == cluster size
  const int rank = blockIdx.x;
  // cluster (blockIdx.y) = (sequence b, KV head kvh, row slice): the slice holds the
  // group rows row0 .. row0 + n_rows - 1 (row r <-> query head kvh*g + r / qcap, position
  // r % qcap); every slice of a group streams the same keys
  const int bh = static_cast<int>(blockIdx.y) / a.n_slices;
  const int row0 = (static_cast<int>(blockIdx.y) - bh * a.n_slices) * NQ;
  const int b = bh / a.Hkv, kvh = bh % a.Hkv;
  const int n_rows = min(NQ, a.g * a.qcap - row0);   // rows of this slice
  const int G = a.g1 - a.g0;
  const FastDiv qdiv = a.qcap_div;             // query column q <-> (head q / qcap, row q % qcap)

  // ---------------------------------------------------------------- setup
  // Work that reads no input of the call runs before the wait for the previous kernel on
  // the stream (with programmatic dependent launch it overlaps that kernel's tail): the
  // pipeline barriers, the tensor-map prefetch, the tile counter, the tensor-memory
  // allocation and, in the fused form, an L2 prefetch of this CTA's share of the block
  // means (a cache hint only: the copy that uses them is issued after the wait).
  volatile int* abort_flag = &bk->abort_flag;
  const int BR = a.box_rows;
  const int ngroups = 128 / BR;
  const __nv_bfloat16* Kbh = a.K + static_cast<size_t>(bh) * a.L * D;
  const __nv_bfloat16* Vbh = a.V + static_cast<size_t>(bh) * a.L * D;
  int issued = 0;
  const uint64_t l2_stream = l2_evict_first_policy();   // K/V rows are read once per call
  // kept-block list and sinks of this (b, h): their first entries are fetched right away
  const int32_t* blk_g = FUSED ? bk->blk : a.blocks + static_cast<size_t>(bh) * a.C;
  const int32_t* snk_g = a.sinks ? a.sinks + static_cast<size_t>(bh) * a.S : nullptr;
  LayoutPrefetch pf{};
  SlotLayout sl_p{};
  int p_n = 0;                 // tiles of this (b, h)
  bool p_more = true;          // the end marker is not issued yet
  // fetch tile `tile` into ring stage `it % STAGES`: TMA boxes from parallel lanes, rows
  // outside key runs by cp.async. With `defer`, a stage that used cp.async is left
  // un-arrived (returns true): the caller completes it with finish_deferred.
  // The stage-independent part of fetching a tile (its group keys and which groups are
  // TMA boxes), so that the producer can work it out while the tile's stage is still busy.
  struct TilePlan {
    unsigned tma_mask;
    int k0a, k0b;            // group key of this lane's op j = lane and j = lane + 32
  };
  const unsigned all_groups = (1u << ngroups) - 1u;     // ngroups <= 16
  auto plan_tile = [&](int tile) -> TilePlan {
    const int slot0 = tile * 128;
    const int key0 = (lane < ngroups) ? group_key0<SPARSE>(sl_p, bk->blk, a.bs, a.g0, slot0 + lane * BR) : -1;
    TilePlan pl;
    pl.tma_mask = __ballot_sync(0xffffffffu, key0 >= 0) & all_groups;
    // op j: group j / 4 (ops j >= 32 exist only when ngroups > 8); the key is looked up once
    pl.k0a = __shfl_sync(0xffffffffu, key0, lane >> 2);
    pl.k0b = __shfl_sync(0xffffffffu, key0, 8 + (lane >> 2));
    return pl;
  };
  auto produce_planned = [&](int it, int tile, const TilePlan& pl, bool defer) -> bool {
    const int s = it % STAGES;
    const int slot0 = tile * 128;
    uint8_t* dK = sK + s * SM::kTile;
    uint8_t* dV = sV + s * SM::kTile;
    const unsigned tma_mask = pl.tma_mask;
    if (lane == 0) mbar_expect_tx(&bk->full[s], __popc(tma_mask) * 2u * 2u * static_cast<uint32_t>(BR) * 128u);
    __syncwarp();
    // op j: group j / 4, atom (j / 2) & 1, K for even j, V for odd j; one op per lane
    const int k0a = pl.k0a, k0b = pl.k0b;
    for (int j = lane; j < ngroups * 4; j += 32) {
      const int grp = j >> 2;
      if (!((tma_mask >> grp) & 1u)) continue;
      const int k0 = j < 32 ? k0a : k0b;
      const int at = (j >> 1) & 1;
      const uint32_t off = at * (128 * 128) + grp * BR * 128;
      if (j & 1) tma_load_3d_hint(smem_u32(dV + off), &tmV, &bk->full[s], at * 64, k0, bh, l2_stream);
      else tma_load_3d_hint(smem_u32(dK + off), &tmK, &bk->full[s], at * 64, k0, bh, l2_stream);
    }
    if (SPARSE && tma_mask != all_groups) {
      // Sink rows (and rows past the end) by cp.async, 16 bytes per lane: lane l moves
      // chunk l % CH of rows l / CH, l / CH + 32 / CH, ... The V rows of slots without a
      // key are zero-filled (their P is 0, and 0 * NaN is not 0); their K rows are not
      // fetched at all (their scores are masked).
      static_assert(32 % CH == 0, "a row's 16-byte chunks must tile a warp");
      const int c = lane % CH;
      for (int grp = 0; grp < ngroups; ++grp) {
        if ((tma_mask >> grp) & 1u) continue;
        for (int row = grp * BR + lane / CH; row < (grp + 1) * BR; row += 32 / CH) {
          const int key = sink_slot_key(sl_p, bk->sinks, slot0 + row);
          const size_t koff = static_cast<size_t>(key >= 0 ? key : 0) * D + c * 8;
          const uint32_t so = sw128_offset(row, c, 128);
          if (key >= 0) cp_async16(smem_u32(dK + so), Kbh + koff, 16u);
          cp_async16(smem_u32(dV + so), Vbh + koff, key >= 0 ? 16u : 0u);
        }
      }
      if (defer) {
        if (lane == 0) bk->stage_tile[s] = tile;
        __syncwarp();
        ++issued;
        return true;
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) {
      bk->stage_tile[s] = tile;
      mbar_arrive(&bk->full[s]);
    }
    __syncwarp();
    ++issued;
    return false;
  };
  auto produce = [&](int it, int tile, bool defer) -> bool { return produce_planned(it, tile, plan_tile(tile), defer); };
  // complete the deferred stages (bit s of `stages`) once their cp.async rows have landed
  auto finish_deferred = [&](unsigned stages) {
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0)
      for (int st = 0; st < STAGES; ++st)
        if ((stages >> st) & 1u) mbar_arrive(&bk->full[st]);
    __syncwarp();
  };
  // no more tiles: stage `it % STAGES` carries the end marker (plain arrive, no bytes)
  auto produce_end = [&](int it) {
    if (lane == 0) {
      bk->stage_tile[it % STAGES] = -1;
      mbar_arrive(&bk->full[it % STAGES]);
    }
    __syncwarp();
  };
  // Tiles of this (b, h): CTA `rank` takes tiles rank, rank + cs, ... for its first STAGES
  // stages; after that every CTA claims the next tile from the counter in CTA 0.
  // The counter's initialisation is ordered before any claim by a cluster barrier: the
  // relevance prologue's own, else a split barrier around the prologue.
  // Pipeline barriers and the tensor-map prefetch (producer warp, lane 0).
  auto init_pipeline = [&]() {
    if (lane == 0) {
      for (int st = 0; st < STAGES; ++st) {
        mbar_init(&bk->full[st], 1);
        mbar_init(&bk->empty[st], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bk->s_full[i], 1);
        mbar_init(&bk->s_free[i], kDecSoftmaxWarps);
        mbar_init(&bk->p_full[i], kDecSoftmaxWarps);
        mbar_init(&bk->pv_done[i], 1);
      }
      mbar_init(&bk->drain, 1);
      if (FUSED) {
        mbar_init(&bk->kb_bar, 1);
        mbar_init(&bk->q_bar, 1);
      }
      if (COLSUM) {
        for (int st = 0; st < 6; ++st) {
          mbar_init(&bk->c_full[st], 1);
          mbar_init(&bk->c_empty[st], 1);
        }
        for (int i = 0; i < 2; ++i) {
          mbar_init(&bk->c_sfull[i], 2);      // the MMAs' commit + the tile id published
          mbar_init(&bk->c_sfree[i], kDecSoftmaxWarps);
        }
      }
      bk->abort_flag = 0;
      if (rank == 0) bk->tile_ctr = static_cast<uint32_t>(cs * STAGES);
      fence_mbar_init();
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
  };
  // fused form: this CTA's contiguous share [j_begin, j_end) of the block means
  const int kb_chunk = FUSED ? (a.nb + cs - 1) / cs : 0;
  const int j_begin = FUSED ? min(a.nb, rank * kb_chunk) : 0;
  const int j_end = FUSED ? min(a.nb, j_begin + kb_chunk) : 0;
  const float* kb = FUSED ? a.kbar + static_cast<size_t>(bh) * a.nb * D : nullptr;
  if (warp == kDecProducerWarp) {
    init_pipeline();
    if (FUSED && lane == 0 && j_begin < j_end)
      bulk_prefetch_l2(kb + static_cast<size_t>(j_begin) * D, static_cast<uint32_t>((j_end - j_begin) * D * 4));
  } else if (warp == kDecMmaWarp) {
    tmem_alloc(&bk->tmem_base, SM::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();              // barriers initialised, tensor memory allocated
  tc_fence_after();

  griddep_wait();               // inputs may come from the previous kernel on the stream
  griddep_launch_dependents();

  // ---------------------------------------------------------------- prologue
  // The producer warp builds the slot layout and issues the first STAGES tiles before the
  // CTA barrier; meanwhile the other warps stage Q. The fused form first stages the group's
  // query rows (into the idle K ring) and its first round of block means (into the idle V
  // ring) by bulk copies, issued before anything else.
  constexpr int kKbRound = STAGES >= 3 ? 128 : 120;            // kbar rows per round
  // (Measured: loading the slice's rows by TMA straight into the SW128 operand and summing
  // qbar from there took 0.2 us longer than the raw copy and the layout pass below.)
  if (FUSED && threadIdx.x == 0) {
    const uint32_t qbytes = static_cast<uint32_t>(a.g * a.qcap * D * 2);
    mbar_arrive_expect_tx(&bk->q_bar, qbytes);
    bulk_load(smem_u32(sK), a.Q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * a.g) * a.qcap * D,
              qbytes, &bk->q_bar);
    if (j_begin < j_end) {
      const int nrow = min(kKbRound, j_end - j_begin);
      mbar_arrive_expect_tx(&bk->kb_bar, static_cast<uint32_t>(nrow * D * 4));
      bulk_load(smem_u32(sV), kb + static_cast<size_t>(j_begin) * D, static_cast<uint32_t>(nrow * D * 4),
                &bk->kb_bar);
    }
  }
  const int nq_b = a.n_q ? min(a.n_q[b], a.qcap) : a.qcap;
  if (SPARSE && warp == kDecProducerWarp) {
    // kept-block list and sinks of this (b, h): their first entries are fetched right away
    if (FUSED) pf.s0 = (snk_g && lane < a.S) ? snk_g[lane] : -1;
    else pf = layout_prefetch(blk_g, a.C, snk_g, a.S);
  }
  if (!FUSED && cs > 1) cluster_arrive();
  if (FUSED) {
    // ---- block relevance R_b = qbar . kbar_b / sqrt(d) and top-C (method steps (4)) ----
    // This CTA scores the contiguous kbar rows [j_begin, j_end). They are staged into the
    // (still idle) V ring by bulk copies of up to kKbRound rows; the group's query rows
    // (contiguous in Q) are staged into the (still idle) K ring by one bulk copy issued
    // with the first round, and qbar is summed from there.
    constexpr int RG = kDecThreads / 64;                       // qbar row groups
    static_assert(kKbRound * D * 4 + (RG + 1) * D * 4 <= STAGES * SM::kTile, "kbar round exceeds the V ring");
    static_assert(kDecMaxRows * D * 2 <= STAGES * SM::kTile, "the group's query rows exceed the K ring");
    uint8_t* const sQraw = sK;                                 // [g * qcap][D] bf16
    const __nv_bfloat162* s_qrows = reinterpret_cast<const __nv_bfloat162*>(sQraw);
    float* s_kb = reinterpret_cast<float*>(sV);                // [kKbRound][D]
    float* s_part = s_kb + kKbRound * D;                       // [RG][D]
    float* s_qbar = s_part + RG * D;                           // [D]
    uint32_t* s_key = reinterpret_cast<uint32_t*>(sP);        // [nb] order keys of R, in every CTA
    const int rows = a.g * nq_b;
    const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
    const int nr = a.g * a.qcap;
    const uint32_t sK0 = smem_u32(s_key);
    auto issue_round = [&](int j0) {
      const int nrow = min(kKbRound, j_end - j0);
      mbar_arrive_expect_tx(&bk->kb_bar, static_cast<uint32_t>(nrow * D * 4));
      bulk_load(smem_u32(s_kb), kb + static_cast<size_t>(j0) * D, static_cast<uint32_t>(nrow * D * 4), &bk->kb_bar);
    };
    // qbar over the group's valid rows: RG row groups x 64 dim pairs. Row r is query head
    // r / qcap at position i = r % qcap, valid when i < nq_b.
    {
      const int t = threadIdx.x, dp = t % 64, rg = t / 64;
      float2 acc = make_float2(0.f, 0.f);
      mbar_wait(&bk->q_bar, 0, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_PRODUCER);
      int i = rg;                                   // rg < RG <= qcap is not assumed
      while (i >= a.qcap) i -= a.qcap;
#pragma unroll 4
      for (int r = rg; r < nr; r += RG) {
        if (i < nq_b) {
          const float2 f = __bfloat1622float2(s_qrows[r * (D / 2) + dp]);
          acc.x += f.x;
          acc.y += f.y;
        }
        i += RG;
        while (i >= a.qcap) i -= a.qcap;
      }
      s_part[rg * D + 2 * dp] = acc.x;
      s_part[rg * D + 2 * dp + 1] = acc.y;
    }
    // this slice's rows as the MMA's K-major SW128 Q operand, from the staged copy (the
    // fence after the top-C orders these writes before the tensor cores read them)
    for (int idx = threadIdx.x; idx < NQ * CH; idx += kDecThreads) {
      const int q = idx / CH, c = idx % CH;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (q < n_rows) {
        const int r = row0 + q;
        const int qh = static_cast<int>(qdiv.div(static_cast<uint32_t>(r)));
        if (r - qh * a.qcap < nq_b) v = *reinterpret_cast<const uint4*>(sQraw + static_cast<size_t>(r) * (D * 2) + c * 16);
      }
      *reinterpret_cast<uint4*>(sQ + sw128_offset(q, c, NQ)) = v;
    }
    __syncthreads();
    if (threadIdx.x < D) {
      float q = 0.f;
#pragma unroll
      for (int g = 0; g < RG; ++g) q += s_part[g * D + threadIdx.x];
      s_qbar[threadIdx.x] = rows > 0 ? q / static_cast<float>(rows) : 0.f;
    }
    __syncthreads();
    // R of the staged rows: warp w scores groups of 16 rows, lane l holding dims
    // 4l .. 4l+3 of every row of the group; a warp reduce-scatter leaves row g*16 + l/2's
    // score in lanes l and l^1. The order key of every score is broadcast to each CTA.
    const float4 qv = reinterpret_cast<const float4*>(s_qbar)[lane];
    for (int j0 = j_begin, round = 0; j0 < j_end; j0 += kKbRound, ++round) {
      const int nrow = min(kKbRound, j_end - j0);
      mbar_wait(&bk->kb_bar, round & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_PRODUCER);
      for (int g0 = warp * 16; g0 < nrow; g0 += kDecThreads / 2) {
        float part[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float4 kv = reinterpret_cast<const float4*>(s_kb + static_cast<size_t>(g0 + r) * D)[lane];
          part[r] = (qv.x * kv.x + qv.y * kv.y) + (qv.z * kv.z + qv.w * kv.w);
        }
        warp_sum_scatter16(part);              // row g0 + lane / 2 in lanes 2i, 2i + 1
        if ((lane & 1) == 0 && g0 + (lane >> 1) < nrow) {
          const int j = j0 + g0 + (lane >> 1);
          const uint32_t key = float_order_key(part[0] * inv_sqrt_d);
          if (cs > 1) {
            for (int r = 0; r < cs; ++r)
              asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(dsmem_addr(sK0 + 4u * j, r)), "r"(key)
                           : "memory");
          } else {
            s_key[j] = key;
          }
        }
      }
      if (j0 + kKbRound < j_end) {
        __syncthreads();               // every warp is done with this round's rows
        if (threadIdx.x == 0) issue_round(j0 + kKbRound);
      }
    }
    if (cs > 1) cluster_sync();   // every CTA holds all nb keys
    else __syncthreads();
    int* s_wide = reinterpret_cast<int*>(sK + 4096);          // 11-bit first pass (over the staged rows)
    if (a.nb <= 2 * kDecThreads) cta_topk_linear(s_key, a.nb, a.C, bk->blk, a.C, s_wide, bk->tk);
    else dec_top_c_large(s_key, a.nb, a.C, bk->blk, bk->tk, s_wide);
    // the K and V rings were written and read through the generic proxy above; the
    // producer's TMA writes them next
    fence_proxy_async_smem();
    __syncthreads();
    if (rank == 0 && row0 == 0 && a.blocks_out)
      for (int i = threadIdx.x; i < a.C; i += kDecThreads) a.blocks_out[static_cast<size_t>(bh) * a.C + i] = bk->blk[i];
  }
  if (warp == kDecProducerWarp) {
    if (SPARSE && FUSED) {
      sl_p = fused_block_layout(bk->blk, min(a.C, a.nb), a.S, a.P, a.bs, a.gen_pad, a.box_rows, a.pad_div,
                                kDecMaxBlocks, kDecMaxSinks, &bk->sl);
    } else if (SPARSE) {
      sl_p = build_block_layout(pf, blk_g, a.C, a.S, a.P, a.bs, a.gen_pad, a.box_rows, a.pad_div, bk->blk,
                                kDecMaxBlocks, kDecMaxSinks, &bk->sl);
    } else {
      sl_p.n_slots = a.L;
      if (lane == 0) bk->sl = sl_p;
    }
    p_n = (sl_p.n_slots + 127) / 128;
    __syncwarp();
    // the layout and the barriers are ready: release the other warps, then fill the ring
    // (a tile gathered row by row completes after the TMA tiles behind it are issued)
    named_bar_arrive(2, kDecThreads);
    // Tiles of kept blocks and of the current block do not need the sinks: the sinks are
    // de-duplicated just before the first tile that holds sink slots (the sink segment ends
    // the layout), at the latest before any tile beyond this first round.
    bool sinks_ready = !SPARSE;
    auto ensure_sinks = [&]() {
      if (SPARSE && !sinks_ready) {
        dedupe_sinks(pf, snk_g, sl_p, a.L, a.P, a.g0, a.g1, a.bs_div, bk->blk, bk->sinks);
        sinks_ready = true;
      }
    };
    unsigned deferred = 0;
    for (int it = 0; it < STAGES; ++it) {
      const int tile = rank + it * cs;
      if (tile >= p_n) {
        produce_end(it);
        p_more = false;
        break;
      }
      if ((tile + 1) * 128 > sl_p.sink_start) ensure_sinks();
      if (produce(it, tile, true)) deferred |= 1u << it;
    }
    ensure_sinks();
    if (deferred) finish_deferred(deferred);
    if (!FUSED && cs > 1) cluster_wait();   // the claim counter is initialised
  }
  if (warp != kDecProducerWarp) {
    // Q rows (query q <-> head kvh*g + q/qcap, position q%qcap) as a K-major SW128 B
    // operand; rows are loaded before the valid count is known and masked afterwards
    const int qt = warp < kDecProducerWarp ? threadIdx.x : threadIdx.x - 32;   // dense index without the producer
    for (int idx = qt; !FUSED && idx < NQ * CH; idx += kDecThreads - 32) {   // (fused: staged in the prologue)
      const int q = idx / CH, c = idx % CH;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (q < n_rows) {
        const int r = row0 + q;
        const int qh = static_cast<int>(qdiv.div(static_cast<uint32_t>(r)));
        const int hq = kvh * a.g + qh, i = r - qh * a.qcap;
        v = __ldg(reinterpret_cast<const uint4*>(a.Q + ((static_cast<size_t>(b) * a.Hq + hq) * a.qcap + i) * D) + c);
        if (i >= nq_b) v = make_uint4(0u, 0u, 0u, 0u);
      }
      *reinterpret_cast<uint4*>(sQ + sw128_offset(q, c, NQ)) = v;
    }
    if (threadIdx.x < NQ) {
      bk->mref[threadIdx.x] = -INFINITY;
      bk->alpha[threadIdx.x] = 1.f;
    }
    if (warp < 2) {
      const int q = threadIdx.x;
      const int qh = static_cast<int>(qdiv.div(static_cast<uint32_t>(row0 + q)));
      const unsigned m = __ballot_sync(0xffffffffu, q < NQ && q < n_rows && (row0 + q - qh * a.qcap) < nq_b);
      if (lane == 0) bk->qvalid[warp] = m;
    }
    fence_proxy_async_smem();
  }
  if (warp != kDecProducerWarp) {
    tc_fence_before();
    named_bar_sync(2, kDecThreads);      // layout, barriers, TMEM and Q are ready
    tc_fence_after();
    if (!FUSED && cs > 1) cluster_wait();
  }

  const uint32_t tmem = bk->tmem_base;
  const SlotLayout sl = bk->sl;
  int n_it = 0;                                  // tiles this CTA processed (set by each role)
  constexpr int QH = NQ / 2;                     // query columns per softmax thread
  float lsum[QH];
#pragma unroll
  for (int q = 0; q < QH; ++q) lsum[q] = 0.f;

  if (warp == kDecProducerWarp) {
    // ------------------------------------------------------------ producer
    // A wait that ran out raises the abort flag, which ends the other roles' loops; the
    // end marker is then not issued.
    bool drained_marker = !p_more;
    if (p_more) {
      const uint32_t ctr = smem_u32(&bk->tile_ctr);
      // Lane 0 claims the next tile right after issuing the current one; the claim (a round
      // trip to CTA 0) is first read after the next stage wait, so it never delays a load.
      // The claimed tile is planned while its stage is still busy (the claim has long
      // returned by then), so a freed stage is refilled at once.
      // The sparse layout ends with the sink segment, whose rows are gathered one by one:
      // its last tile is handed out in the middle of the claims (claim m), so that the
      // gather is issued while the claiming CTA still has other tiles to consume and the
      // claims after it rebalance the cluster, instead of ending some CTA's work late.
      const int m_sink = max(cs * STAGES, p_n / 2);
      auto claim_tile = [&](int c) {
        if (!SPARSE || m_sink >= p_n - 1 || c < m_sink || c >= p_n) return c;
        return c == m_sink ? p_n - 1 : c - 1;
      };
      int claim = 0;
      if (lane == 0) claim = static_cast<int>(dsmem_atomic_add(ctr, 0, 1u));
      for (int it = STAGES;; ++it) {
        const int s = it % STAGES;
        const int tile = claim_tile(__shfl_sync(0xffffffffu, claim, 0));
        TilePlan pl{0u, 0, 0};
        if (tile < p_n) pl = plan_tile(tile);
        if (!__all_sync(0xffffffffu, mbar_wait(&bk->empty[s], ((it / STAGES) - 1) & 1, abort_flag, a.dev_err,
                                               DEV_ERR_TIMEOUT_PRODUCER)))
          break;
        if (tile >= p_n) {
          produce_end(it);
          drained_marker = true;
          break;
        }
        produce_planned(it, tile, pl, false);
        if (lane == 0) claim = static_cast<int>(dsmem_atomic_add(ctr, 0, 1u));
      }
    }
    // wait for the copies still in flight; the end marker (issue index `issued`) shares its
    // stage with tile issued - STAGES, which had completed before the marker was issued
    if (lane == 0)
      for (int j = max(0, issued - STAGES + (drained_marker ? 1 : 0)); j < issued; ++j)
        dec_wait_drain(&bk->full[j % STAGES], (j / STAGES) & 1);
    __syncwarp();
  } else if (warp == kDecMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, NQ, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, NQ, true, false);
      const uint32_t tO = tmem + 2 * NQ;
      // Descriptors are formed once; a K step or a stage adds a constant to the 14-bit
      // start-address field (address >> 4), which cannot carry: shared memory < 256 KB.
      const uint64_t q_desc = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t v_desc0 = sw128_desc(smem_u32(sV), 128 * 128, 1024);
      const uint64_t p_desc0 = sw128_desc(smem_u32(sP), 16, 1024);
      constexpr uint32_t kTileDesc = SM::kTile >> 4;
      bool ok = true;
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1;
        if (!mbar_wait(&bk->p_full[pb], (j >> 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint64_t vd = v_desc0 + static_cast<uint64_t>((j % STAGES) * kTileDesc);
        const uint64_t pd = p_desc0 + static_cast<uint64_t>(pb * (NQ * 256 / 16));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16(tO, vd + ks * (2048 / 16), pd + (ks >> 2) * (NQ * 128 / 16) + (ks & 3) * 2, idesc_pv,
                   (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bk->pv_done[pb]);
        mma_commit(&bk->empty[j % STAGES]);
        return true;
      };
      // QK runs one tile ahead of PV: QK(j + 1) only needs the S buffer that softmax(j - 1)
      // has already read, so it is issued before PV(j), which waits for softmax(j)'s P.
      // (Two tiles ahead would hold PV(j) behind the load of tile j + 2, whose ring stage
      // is only freed by PV(j - 1): the loads in flight would shrink to one tile.)
      constexpr int LA = 1;
      int q_next = 0, n_end = -1;          // next QK tile; tile index of the end marker
      // QK of tile it; at the end marker, releases the softmax warps and returns false
      auto issue_qk = [&](int it) -> bool {
        const int s = it % STAGES, sb = it & 1;
        if (!mbar_wait(&bk->full[s], (it / STAGES) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          return false;
        }
        if (bk->stage_tile[s] < 0) {
          n_end = it;
          mbar_arrive(&bk->s_full[sb]);
          return false;
        }
        if (it >= 2 && !mbar_wait(&bk->s_free[sb], ((it - 2) >> 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          return false;
        }
        tc_fence_after();
        const uint64_t kd = k_desc0 + static_cast<uint64_t>(s * kTileDesc);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16(tmem + sb * NQ, kd + (ks >> 2) * (128 * 128 / 16) + (ks & 3) * 2,
                   q_desc + (ks >> 2) * (NQ * 128 / 16) + (ks & 3) * 2, idesc_qk, ks > 0 ? 1u : 0u);
        mma_commit(&bk->s_full[sb]);
        return true;
      };
      while (q_next < LA && n_end < 0 && ok && issue_qk(q_next)) ++q_next;
      for (int j = 0; ok; ++j) {
        if (n_end >= 0 && j >= n_end) break;
        if (n_end < 0 && issue_qk(q_next)) ++q_next;
        if (!ok) break;
        ok = issue_pv(j);
      }
      n_it = max(n_end, 0);
      mma_commit(&bk->drain);
      dec_wait_drain(&bk->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0..7
    // Warp w reads TMEM lane quadrant w % 4 (keys 32*(w%4) .. +31 of the tile, or dims of
    // O^T) and query half w / 4 (columns q0 .. q0 + QH - 1).
    const int t = threadIdx.x & 127;                   // key of the tile == TMEM lane == dim of O^T
    const int qd = warp & 3;
    const int q0 = (warp >> 2) * QH;
    const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t tO = tmem + 2 * NQ;
    const uint64_t qvalid =
        (bk->qvalid[0] | (static_cast<uint64_t>(bk->qvalid[1]) << 32)) >> q0;   // bit q: column q0 + q is real
    // The loop ends, in all eight warps at once, at the end marker or when a wait ran out.
    // A warp whose wait ran out inside an iteration finishes it without waits or
    // tensor-memory access, so that all eight warps take the same named-barrier steps.
    bool ok = true;
    int it = 0;
    for (;; ++it) {
      const int sb = it & 1;
      if (ok)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bk->s_full[sb], (it >> 1) & 1, abort_flag, a.dev_err, DEV_ERR_TIMEOUT_SOFTMAX));
      int tile = -1;
      if (ok) {
        // the stage's tile id, published by the producer before it completed full[stage]
        ok = __all_sync(0xffffffffu, mbar_wait(&bk->full[it % STAGES], (it / STAGES) & 1, abort_flag, a.dev_err,
                                               DEV_ERR_TIMEOUT_SOFTMAX));
        if (ok) tile = bk->stage_tile[it % STAGES];
      }
      if (bar_red_or(1, kDecSoftmaxThreads, tile < 0 || *abort_flag != 0)) break;
      float sv[QH];
#pragma unroll
      for (int q = 0; q < QH; ++q) sv[q] = 0.f;
      if (ok) {
        tc_fence_after();
        uint32_t rg[QH];
        tmem_ld_cols<QH>(tmem + lane_addr + sb * NQ + q0, rg);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < QH; ++q) sv[q] = __uint_as_float(rg[q]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->s_free[sb]);
      const bool kv = ok && slot_valid<SPARSE>(sl, bk->sinks, a.L, a.bs, G, tile * 128 + t);
      bool over = false;
#pragma unroll
      for (int q = 0; q < QH; ++q) {
        sv[q] = (kv && ((qvalid >> q) & 1ull)) ? sv[q] * a.scale_log2 : -INFINITY;
        over |= sv[q] > bk->mref[q0 + q] + 8.f;
      }
      if (bar_red_or(1, kDecSoftmaxThreads, over)) {
        // exact per-query maximum of this tile, then move the references up
        // (one redux per query on the order-preserving integer image of the score)
#pragma unroll
        for (int q = 0; q < QH; ++q) {
          const uint32_t m = __reduce_max_sync(0xffffffffu, float_order_key(sv[q]));
          if (lane == 0) bk->red[qd][q0 + q] = __uint_as_float(m);
        }
        named_bar_sync(1, kDecSoftmaxThreads);
        if (threadIdx.x < NQ) {
          const int tq = threadIdx.x;
          const uint32_t k01 = max(__float_as_uint(bk->red[0][tq]), __float_as_uint(bk->red[1][tq]));
          const uint32_t k23 = max(__float_as_uint(bk->red[2][tq]), __float_as_uint(bk->red[3][tq]));
          const float mt = order_key_to_float(max(k01, k23));
          const float mo = bk->mref[tq];
          const float mn = fmaxf(mo, mt);
          if (mn > mo + 8.f || (mo == -INFINITY && mn > -INFINITY)) {
            bk->alpha[tq] = (mo == -INFINITY) ? 0.f : exp2_approx(mo - mn);
            bk->mref[tq] = mn;
          } else {
            bk->alpha[tq] = 1.f;
          }
        }
        named_bar_sync(1, kDecSoftmaxThreads);
        bool any_scale = false;
#pragma unroll
        for (int q = 0; q < QH; ++q) {
          const float al = bk->alpha[q0 + q];
          lsum[q] *= al;
          any_scale |= al != 1.f;
        }
        any_scale = __any_sync(0xffffffffu, any_scale);
        if (it > 0 && any_scale && ok) {
          // O^T must hold PV of the previous tile before it is rescaled
          ok = __all_sync(0xffffffffu, mbar_wait(&bk->pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag,
                                                 a.dev_err, DEV_ERR_TIMEOUT_SOFTMAX));
          if (ok) {
            tc_fence_after();
            uint32_t rg[QH];
            tmem_ld_cols<QH>(tO + lane_addr + q0, rg);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < QH; ++q) rg[q] = __float_as_uint(__uint_as_float(rg[q]) * bk->alpha[q0 + q]);
            tmem_st_cols<QH>(tO + lane_addr + q0, rg);
            tmem_st_wait();
          }
        }
      }
      // P^T of this key: p = 2^(s - m_q)
#pragma unroll
      for (int q = 0; q < QH; ++q) {
        const float m = bk->mref[q0 + q];
        sv[q] = exp2_approx(sv[q] - (m == -INFINITY ? 0.f : m));
        lsum[q] += sv[q];
      }
      if (it >= 2 && ok)
        ok = __all_sync(0xffffffffu, mbar_wait(&bk->pv_done[sb], ((it - 2) >> 1) & 1, abort_flag, a.dev_err,
                                               DEV_ERR_TIMEOUT_SOFTMAX));
      if (ok) {
        uint8_t* pbuf = sP + sb * (NQ * 256);
        const uint32_t col = static_cast<uint32_t>((t & 7) * 2);
#pragma unroll
        for (int q = 0; q < QH; ++q) {
          const __nv_bfloat16 hv = __float2bfloat16_rn(sv[q]);
          *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_offset(q0 + q, t >> 3, NQ) + col) = hv;
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bk->p_full[sb]);
    }
    n_it = it;
    // row sums (while the last PV is still running): reduce the per-key partials over the
    // 32 lanes of each warp (reduce-scatter), then over the four lane quadrants; the
    // epilogue's CTA barrier orders lfin
    if constexpr (QH % 32 == 0) {
      warp_sum_scatter<QH>(lsum);
#pragma unroll
      for (int j = 0; j < QH / 32; ++j) bk->red[qd][q0 + lane * (QH / 32) + j] = lsum[j];
    } else {
      warp_sum_scatter16(lsum);
      if ((lane & 1) == 0) bk->red[qd][q0 + (lane >> 1)] = lsum[0];
    }
    named_bar_sync(1, kDecSoftmaxThreads);
    if (threadIdx.x < NQ) {
      const int tq = threadIdx.x;
      bk->lfin[tq] = (bk->red[0][tq] + bk->red[1][tq]) + (bk->red[2][tq] + bk->red[3][tq]);
    }
    if (ok && n_it > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bk->pv_done[(n_it - 1) & 1], ((n_it - 1) >> 1) & 1, abort_flag,
                                             a.dev_err, DEV_ERR_TIMEOUT_EPILOGUE));
      tc_fence_after();
    }
    if (!ok) bk->abort_flag = 1;
  }

  // ---------------------------------------------------------------- epilogue
  // Every CTA leaves its partial result (unnormalised O^T, m and l of every query) in its
  // own V ring, idle once its loop is done. After one cluster barrier, CTA r merges the
  // queries [r * qpc, (r + 1) * qpc) from the partials of all CTAs of the cluster, read over
  // distributed shared memory with 16-byte loads; a split barrier (arrive after the reads,
  // wait before exit) keeps every CTA's partials resident until all readers are done.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool have_o = (n_it > 0) && !bk->abort_flag;
  static_assert(NQ * D * 4 + NQ * 8 <= STAGES * SM::kTile, "partials exceed the V ring");
  float* part_o = reinterpret_cast<float*>(sV);                      // [NQ][D]
  float2* part_ml = reinterpret_cast<float2*>(part_o + NQ * D);      // [NQ] (m, l)
  if (warp < kDecSoftmaxWarps) {
    // warp w: dims of lane quadrant w % 4, query half w / 4
    const int t = threadIdx.x & 127, q0 = (warp >> 2) * QH;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t rg[QH];
#pragma unroll
    for (int j = 0; j < QH; ++j) rg[j] = 0u;
    if (have_o) {
      tmem_ld_cols<QH>(tmem + 2 * NQ + lane_addr + q0, rg);
      tmem_ld_wait();
    }
#pragma unroll
    for (int j = 0; j < QH; ++j) part_o[(q0 + j) * D + t] = __uint_as_float(rg[j]);
    if (threadIdx.x < NQ)
      part_ml[threadIdx.x] = make_float2(bk->mref[threadIdx.x], have_o ? bk->lfin[threadIdx.x] : 0.f);
  }
  tc_fence_before();
  if (cs > 1) cluster_sync();        // every partial of the cluster is in place
  else __syncthreads();
  if (!COLSUM && warp == kDecMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, SM::kTmemCols);
  }
  const int qpc = (n_rows + cs - 1) / cs;
  // lane: dims 4*lane .. 4*lane+3; warp: queries rank*qpc + warp + 8k, two per batch. A
  // batch's partials are all requested before any is used. Every warp arrives on the
  // cluster barrier once the values of all its remote loads have been used (so the loads
  // are complete and nothing needs publishing: a relaxed arrive), and waits on it at the
  // very end.
  const uint32_t po = smem_u32(part_o), pm = smem_u32(part_ml);
  auto load_q = [&](int q, bool v, float4 (&ov)[8], float2 (&ml)[8]) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      ov[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      ml[r] = make_float2(-INFINITY, 0.f);
      if (v && r < cs) {
        ml[r] = dsmem_ld_v2(dsmem_addr(pm + static_cast<uint32_t>(q) * 8u, r));
        ov[r] = dsmem_ld_v4(dsmem_addr(po + static_cast<uint32_t>(q * D + 4 * lane) * 4u, r));
      }
    }
  };
  // merged maximum M and row sum l of a query from the CTAs' (m, l); w[r] = 2^(m_r - M)
  auto merge_ml = [&](const float2 (&ml)[8], float& M, float& l, float (&w)[8]) {
    M = -INFINITY;
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (ml[r].y > 0.f) M = fmaxf(M, ml[r].x);
    l = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      w[r] = ml[r].y > 0.f ? exp2_approx(ml[r].x - M) : 0.f;
      l += w[r] * ml[r].y;
    }
  };
  if constexpr (COLSUM) {
    // every CTA needs the log-sum-exp of every query column for its column sums: the
    // producer warp, idle now, forms it while the softmax warps merge
    for (int q = lane; warp == kDecProducerWarp && q < NQ; q += 32) {
      float v = INFINITY;                     // not a query: 2^(s - inf) = 0
      if (q < n_rows) {
        const int r = row0 + q;
        const int qh = static_cast<int>(qdiv.div(static_cast<uint32_t>(r)));
        if (r - qh * a.qcap < nq_b) {
          float2 ml[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            ml[c] = c < cs ? dsmem_ld_v2(dsmem_addr(smem_u32(part_ml) + static_cast<uint32_t>(q) * 8u, c))
                           : make_float2(-INFINITY, 0.f);
          float M, l, w[8];
          merge_ml(ml, M, l, w);
          if (l > 0.f) v = M + __log2f(l);
        }
      }
      bk->lse2[q] = v;
    }
  }
  auto finish_q = [&](int q, const float4 (&ov)[8], const float2 (&ml)[8]) {
    float M, l, w[8];
    merge_ml(ml, M, l, w);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float wr = w[r] * inv;
      o.x += wr * ov[r].x;
      o.y += wr * ov[r].y;
      o.z += wr * ov[r].z;
      o.w += wr * ov[r].w;
    }
    const int r = row0 + q;
    const int qh = static_cast<int>(qdiv.div(static_cast<uint32_t>(r)));
    const int hq = kvh * a.g + qh, i = r - qh * a.qcap;
    if (i >= nq_b) o = make_float4(0.f, 0.f, 0.f, 0.f);
    uint2 pk;
    pk.x = pack_bf16x2(o.x, o.y);
    pk.y = pack_bf16x2(o.z, o.w);
    const size_t row = (static_cast<size_t>(b) * a.Hq + hq) * a.qcap + i;
    *reinterpret_cast<uint2*>(a.O + row * D + 4 * lane) = pk;
    if (lane == 0 && a.lse_out && i < nq_b) a.lse_out[row] = M + __log2f(l);
  };
  if (warp < kDecSoftmaxWarps) {
    constexpr int W = kDecSoftmaxWarps;
    for (int qi0 = warp; qi0 < qpc; qi0 += 2 * W) {
      const int qa = rank * qpc + qi0, qb = qa + W;
      const bool va = qa < n_rows, vb = (qi0 + W < qpc) && qb < n_rows;
      float4 ova[8], ovb[8];
      float2 mla[8], mlb[8];
      load_q(qa, va, ova, mla);
      load_q(qb, vb, ovb, mlb);
      if (va) finish_q(qa, ova, mla);
      if (vb) finish_q(qb, ovb, mlb);
    }
  }
  if (cs > 1) cluster_arrive_relaxed();   // this warp's reads of the partials are done
  if constexpr (COLSUM)
    decode_colsum_phase<NQ, STAGES>(&tmK, a, bk, sK, sV, sQ, tmem, bh, rank, cs, reinterpret_cast<uint32_t*>(sP));
  if (cs > 1) cluster_wait();             // no CTA leaves while its partials may still be read
  if constexpr (COLSUM) {
    // the column sums are visible to the whole cluster
    __threadfence();
    tc_fence_before();
    if (cs > 1) cluster_sync();
    else __syncthreads();
    if (warp == kDecMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, SM::kTmemCols);
    }
    // every CTA of the cluster takes the same barriers here, also after a wait ran out (the
    // sinks are then undefined, and the device error word says so)
    if (a.sinks_out) decode_sink_topk(a, bk, sK, reinterpret_cast<const uint32_t*>(sP), bh, rank, cs);
  }
}

// ------------------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 dec_encode_fn() {
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

int dec_make_map(CUtensorMap* map, const void* base, int BH, int L, int box_rows) {
  auto fn = dec_encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled is unavailable (driver entry point lookup failed)");
    return FOCUS_ERR_CUDA;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDecD), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDecD) * 2, static_cast<cuuint64_t>(L) * kDecD * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

template <int NQ, int STAGES, bool SPARSE, bool FUSED, bool COLSUM>
int max_active_clusters(int cs) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(dev, cs);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  auto kern = decode_attn_kernel<NQ, STAGES, SPARSE, FUSED, COLSUM>;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), static_cast<int>(DecSmem<NQ, STAGES>::kBytes)) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, 1, 1);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = DecSmem<NQ, STAGES>::kBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cs;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[key] = n;
  return n;
}

template <int NQ, int STAGES, bool SPARSE, bool FUSED, bool COLSUM>
int choose_cluster(int units) {
  const int sms = device_sm_count();
  for (int cs : {8, 4, 2}) {
    if (units * cs > sms) continue;
    if (max_active_clusters<NQ, STAGES, SPARSE, FUSED, COLSUM>(cs) >= units) return cs;
  }
  return 1;
}

// Whether the cluster's fused top-S (decode_sink_topk) serves S sinks over L columns with
// cs CTAs: S group maxima per CTA at most 4 x 128, and the cs * S candidates in CTA 0.
bool plan_sink_topk(int L, int S, int cs) {
  return S >= 1 && S <= kDecMaxSinks && S <= L && cs * S <= kSinkCand0;
}

template <int NQ, int STAGES, bool SPARSE, bool FUSED, bool COLSUM = false>
int run_decode(const DecArgs& a0, cudaStream_t stream, bool* sinks_done = nullptr) {
  DecArgs a = a0;
  CUtensorMap mk, mv;
  int st = dec_make_map(&mk, a.K, a.B * a.Hkv, a.L, a.box_rows);
  if (st != FOCUS_OK) return st;
  st = dec_make_map(&mv, a.V, a.B * a.Hkv, a.L, a.box_rows);
  if (st != FOCUS_OK) return st;
  a.dev_err = device_error_word();
  a.n_slices = (a.g * a.qcap + NQ - 1) / NQ;
  const int units = a.B * a.Hkv * a.n_slices;
  if (units > 65535) {
    set_error("decode attention: %d (sequence, KV head, row slice) units exceed the grid", units);
    return FOCUS_ERR_UNSUPPORTED;
  }
  const int cs = choose_cluster<NQ, STAGES, SPARSE, FUSED, COLSUM>(units);
  if (COLSUM && a.sinks_out) {
    if (!plan_sink_topk(a.L, a.S_out, cs)) a.sinks_out = nullptr;
    if (sinks_done) *sinks_done = a.sinks_out != nullptr;
  }
  auto kern = decode_attn_kernel<NQ, STAGES, SPARSE, FUSED, COLSUM>;
  if (const int st_attr = configure_dynamic_smem(reinterpret_cast<const void*>(kern),
                                                 static_cast<int>(DecSmem<NQ, STAGES>::kBytes),
                                                 "decode attention"))
    return st_attr;
  const cudaError_t e =
      launch_k_cluster(kern, dim3(cs, units), dim3(kDecThreads), DecSmem<NQ, STAGES>::kBytes, stream, cs, mk, mv, a);
  note_launch();
  if (e != cudaSuccess) {
    set_error("decode attention launch: %s", cudaGetErrorString(e));
    return FOCUS_ERR_CUDA;
  }
  return FOCUS_OK;
}

int pow2_divisor(int x, int cap) {
  int r = 8;
  while (r * 2 <= cap && x % (r * 2) == 0) r *= 2;
  return r;
}

}  // namespace

// Whether the decode kernel serves this shape (else the 128-row tile kernel does). A sparse
// call takes up to kDecMaxRows query rows per KV group, in slices of 64 rows that stream
// the same (few) kept keys. A dense call takes at most one slice: every slice would stream
// all L keys through a 2-deep ring, and the tile kernel, which reads the keys once per 128
// rows with every SM busy, does better there.
bool decode_supported(int d, int Hq, int Hkv, int qcap, int L, int S, int C, bool sparse) {
  const int rows = (Hq / Hkv) * qcap;
  return d == kDecD && rows <= (sparse ? kDecMaxRows : 64) && L >= 8 && S <= kDecMaxSinks && C <= kDecMaxBlocks;
}

// Fused relevance + top-C is used when kbar is given (blocks is then ignored).
bool decode_fused_supported(int d, int Hq, int Hkv, int qcap, int L, int S, int C, int nb) {
  return decode_supported(d, Hq, Hkv, qcap, L, S, C, true) && nb >= 1 && nb <= kDecMaxNb;
}

int decode_attention(const __nv_bfloat16* Q, const int32_t* n_q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                     __nv_bfloat16* O, float* lse_out, const int32_t* sinks, const int32_t* blocks, int S, int C, int bs,
                     int P, int g0, int g1, bool sparse, int B, int Hq, int Hkv, int L, int qcap, float scale_log2,
                     cudaStream_t stream, const float* kbar, int nb, int32_t* blocks_out, float* colsum,
                     int32_t* sinks_out, int S_out, bool* sinks_done) {
  DecArgs a{};
  a.Q = Q;
  a.n_q = n_q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.lse_out = lse_out;
  a.sinks = sinks;
  a.blocks = blocks;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.qcap = qcap;
  a.g = Hq / Hkv;
  a.S = S;
  a.C = C;
  a.bs = bs;
  a.P = P;
  a.g0 = g0;
  a.g1 = g1;
  a.scale_log2 = scale_log2;
  int cap = 128;
  while (cap > L) cap >>= 1;
  if (sparse) {
    // boxes stay inside one kept block; the current block is padded to whole boxes
    a.box_rows = pow2_divisor((bs + 7) & ~7, cap);
    a.gen_pad = (g1 - g0 + a.box_rows - 1) / a.box_rows * a.box_rows;
  } else {
    a.box_rows = cap;
    a.gen_pad = 0;
  }
  {
    const int pad_bs = (bs + 7) & ~7;
    const long long n_max = static_cast<long long>(C) * pad_bs + a.gen_pad +
                            (std::min(S, kDecMaxSinks) + a.box_rows - 1) / a.box_rows * a.box_rows + 256;
    a.pad_div.init(static_cast<uint32_t>(pad_bs), static_cast<uint32_t>(std::min<long long>(n_max, 0xFFFFFFFFll)));
    a.bs_div.init(static_cast<uint32_t>(std::max(bs, 1)), static_cast<uint32_t>(L));
    a.qcap_div.init(static_cast<uint32_t>(qcap), static_cast<uint32_t>(a.g * qcap));
  }
  const int nrows = a.g * qcap;
  if (kbar) {
    a.kbar = kbar;
    a.nb = nb;
    a.blocks_out = blocks_out;
    return nrows <= 32 ? run_decode<32, 3, true, true>(a, stream) : run_decode<64, 2, true, true>(a, stream);
  }
  if (sinks_done) *sinks_done = false;
  if (!sparse && colsum) {
    // the sink layer: attention, column sums and (when the cluster can select them) sinks
    a.colsum = colsum;
    a.sinks_out = sinks_out;
    a.S_out = S_out;
    return nrows <= 32 ? run_decode<32, 3, false, false, true>(a, stream, sinks_done)
                       : run_decode<64, 2, false, false, true>(a, stream, sinks_done);
  }
  if (nrows <= 32)
    return sparse ? run_decode<32, 3, true, false>(a, stream) : run_decode<32, 3, false, false>(a, stream);
  return sparse ? run_decode<64, 2, true, false>(a, stream) : run_decode<64, 2, false, false>(a, stream);
}

}  // namespace focus
