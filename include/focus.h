/*
 * focus.h -- C ABI of libfocus.so, the B200 (sm_100a) implementation of the
 * Focus-dLLM sparse denoising-step attention.
 *
 * Source of the operations: "Focus-dLLM: Accelerating Long-Context Diffusion LLM
 * Inference via Confidence-Guided Context Focusing" (summary page of arXiv
 * 2602.02159), section "方法步骤详情" (method steps) steps (1)-(5), and section
 * "核心方法" (core method). At a block-entry step the whole sequence runs dense
 * attention; at every other step:
 *   (1) PCGI picks the top-k still-[MASK] positions by the previous step's
 *       confidence, k = floor(rho * n(t))                     -> focus_select_queries
 *   (2) each is widened to a window of size w -> I_active     -> focus_select_queries
 *   (3) the first layers run full attention; the attention distribution of the
 *       sink layer picks the attention sinks                   -> focus_dense_attention,
 *                                                                focus_sink_identify
 *   (4) prompt blocks are represented by their mean key, scored against the
 *       active queries, and the top-C kept                     -> focus_block_means,
 *                                                                focus_block_select
 *   (5) the active queries attend over I_p = sinks U kept blocks U current block
 *                                                              -> focus_sparse_attention
 *
 * Conventions shared by every call:
 *   - Every pointer is a DEVICE pointer unless stated otherwise. The caller owns all
 *     memory (tensors and workspace); the library allocates nothing.
 *   - bf16 tensors are passed as `focus_bf16` (raw IEEE bfloat16 bits).
 *   - Layouts are dense row-major: K, V [B, Hkv, L, d]; Q [B, Hq, qcap, d];
 *     query head hq uses KV head hq / (Hq / Hkv).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *     enqueues work on it and never synchronises the host; counts (n_focus,
 *     n_active) stay on the device.
 *   - Every call returns a focus_status. Arguments are validated before any launch;
 *     an invalid call launches nothing and returns FOCUS_ERR_INVALID_ARG (or
 *     FOCUS_ERR_UNSUPPORTED / FOCUS_ERR_CAPACITY) with a message in
 *     focus_last_error(). A failed launch returns FOCUS_ERR_CUDA.
 *   - Index outputs are sorted ascending; unused tail slots hold -1.
 *   - Every top-k orders by (score descending, index ascending): ties go to the
 *     lower index and -0.0 equals +0.0. Scores must be finite.
 *   - A kernel wait that runs out (2 s) records a code in the device error word
 *     (read it with focus_device_error) and the kernel returns early; outputs of
 *     that call are then undefined.
 */
#ifndef FOCUS_H_
#define FOCUS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(FOCUS_BUILD) && defined(__GNUC__)
#define FOCUS_API __attribute__((visibility("default")))
#else
#define FOCUS_API
#endif

typedef uint16_t focus_bf16;

typedef enum {
  FOCUS_OK = 0,
  FOCUS_ERR_INVALID_ARG = -1,
  FOCUS_ERR_UNSUPPORTED = -2,
  FOCUS_ERR_CUDA = -3,
  FOCUS_ERR_CAPACITY = -4,
  FOCUS_ERR_DEVICE_CHECK = -5
} focus_status;

/* Human-readable name of a status code. Never NULL. */
FOCUS_API const char* focus_status_string(int status);

/* Message of the last failing call on this host thread ("" if none). Never NULL. */
FOCUS_API const char* focus_last_error(void);

/* Number of kernels this library has launched in this process (all threads). */
FOCUS_API uint64_t focus_launch_count(void);

/* Synchronises the current device, copies the device error word to *code_out (0 = no
 * error) and clears it. Returns FOCUS_ERR_DEVICE_CHECK if the word was set. */
FOCUS_API int focus_device_error(int* code_out);

/*
 * (1)+(2) PCGI and window expansion -- method steps (1) and (2).
 * conf_prev [B, G] fp32, G = g1 - g0: c_{t-1} of position g0 + j at conf_prev[b, j].
 * mask [B, L] uint8, nonzero = still [MASK]. Candidates: masked positions of the current
 * block [g0, g1). k = min(floor(rho * n_t), #candidates); I_focus = the top-k candidates
 * by conf. Each p in I_focus becomes [p - w/2, p - w/2 + w - 1] clipped to [g0, g1);
 * I_active = the sorted union.
 * Outputs: i_focus [B, kcap], n_focus [B], i_active [B, acap], n_active [B] (int32).
 * Requires 0 <= g0 < g1 <= L, G <= 1024, n_t >= 0, rho >= 0, w >= 1,
 * kcap >= min(floor(rho*n_t), G), acap >= min(G, kcap * w) (else FOCUS_ERR_CAPACITY).
 */
FOCUS_API int focus_select_queries(const float* conf_prev, const uint8_t* mask, int B, int L, int g0, int g1, int n_t,
                         float rho, int w, int32_t* i_focus, int32_t* n_focus, int kcap, int32_t* i_active,
                         int32_t* n_active, int acap, void* stream);

/*
 * Gathers rows of a stack of head-major matrices by per-batch row lists (the queries of
 * the active positions). X [n_mat, B, H, L, d] -> X_rows [n_mat, B, H, cap, d] with
 * X_rows[m, b, h, i] = X[m, b, h, rows[b, i]] for i < n_rows[b], zero otherwise.
 * rows [B, cap] and n_rows [B] int32 (device). Row indices outside [0, L) are written
 * as zero rows and flagged in the device error word (code 5).
 */
FOCUS_API int focus_gather_rows(const focus_bf16* X, const int32_t* rows, const int32_t* n_rows, int n_mat, int B, int H,
                      int L, int d, int cap, focus_bf16* X_rows, void* stream);

/*
 * Approximate-KV-cache refresh (Focus-dLLM summary page, "近似KV缓存" / approximate KV
 * cache: a token of the refresh set U(t) takes its recomputed key and value, every other
 * token keeps its cached one). The inverse of focus_gather_rows: for every matrix m,
 * X[m, b, h, rows[b, i]] = X_rows[m, b, h, i] for i < n_rows[b]; all other rows of X are
 * left unchanged. X [n_mat, B, H, L, d] (the K or V cache of n_mat layers, updated in
 * place), X_rows [n_mat, B, H, cap, d], rows [B, cap] and n_rows [B] int32 (device), e.g.
 * I_active (or I_focus) from focus_select_queries. Row lists must not repeat a row (the
 * selection outputs are ascending and unique). Indices outside [0, L) are skipped and
 * flagged in the device error word (code 5). d a multiple of 8; X and X_rows 16-byte
 * aligned. The pages have no fused form of this step; it runs as one scatter launch.
 */
FOCUS_API int focus_scatter_rows(focus_bf16* X, const int32_t* rows, const int32_t* n_rows, int n_mat, int B, int H,
                                 int L, int d, int cap, const focus_bf16* X_rows, void* stream);

/*
 * (4a) Block representative keys -- method steps (4): the prompt [0, P) is cut into
 * nb = ceil(P / bs) contiguous blocks; kbar[b, h, j] = mean of K[b, h, j*bs : min(P,(j+1)*bs)].
 * K [B, Hkv, L, d] bf16 -> kbar [B, Hkv, nb, d] fp32. Requires 1 <= P <= L, bs >= 1,
 * d in {64, 128}, K 16-byte aligned.
 */
FOCUS_API int focus_block_means(const focus_bf16* K, int B, int Hkv, int L, int d, int P, int bs, float* kbar,
                      void* stream);

/*
 * (4b) Block relevance and top-C -- method steps (4).
 * R[b, h, j] = mean over the n_active[b] active queries and the Hq/Hkv query heads of
 * KV group h of q . kbar[b, h, j] / sqrt(d) (0 when n_active[b] == 0).
 * blocks[b, h, :] = the top-min(C, nb) blocks, ascending, -1 tail.
 * Q_active [B, Hq, acap, d] bf16; n_active [B]; kbar [B, Hkv, nb, d] fp32;
 * scores_opt: NULL or [B, Hkv, nb] fp32 receiving R. Requires nb <= 49152, C >= 1,
 * d in {64, 128}.
 */
FOCUS_API int focus_block_select(const focus_bf16* Q_active, const int32_t* n_active, const float* kbar, int B, int Hq,
                       int Hkv, int d, int acap, int nb, int C, int32_t* blocks, float* scores_opt,
                       void* stream);

/*
 * (3) Dense bidirectional attention -- method steps (3) and the block-entry full refresh.
 * For query i < n_q[b] (all qcap rows when n_q == NULL) of head hq:
 *   O[b, hq, i] = softmax_j(scale * q_i . k_j) V over all L keys (fp32 accumulation).
 * Rows i >= n_q[b] of O are written as zero.
 * colsum_opt: NULL, or [B, Hkv, L] fp32 receiving the sink importance
 *   colsum[b, h, j] = sum over the group's query heads and the valid queries of p_ij
 *   (requires (Hq/Hkv) * qcap <= 256).
 * ws/ws_bytes: device workspace of at least focus_dense_workspace_bytes(...) bytes,
 *   256-byte aligned (may be NULL when that size is 0).
 * Requires d in {64, 128}, Hq % Hkv == 0, L >= 8, Q/K/V/O 16-byte aligned.
 */
FOCUS_API int focus_dense_attention(const focus_bf16* Q, const int32_t* n_q, const focus_bf16* K, const focus_bf16* V,
                          int B, int Hq, int Hkv, int L, int d, int qcap, float scale, focus_bf16* O,
                          float* colsum_opt, void* ws, size_t ws_bytes, void* stream);

FOCUS_API size_t focus_dense_workspace_bytes(int B, int Hq, int Hkv, int L, int d, int qcap, int want_colsum);

/*
 * Block entry in one call -- "半自回归重遮蔽策略" (semi-AR remasking: at block entry the whole
 * sequence runs dense attention) and method steps (4) (a prompt block is represented by the
 * mean of its keys, computed once per generation block): O = dense attention of all L
 * queries of Q [B, Hq, L, d] over all L keys (as focus_dense_attention with n_q = NULL,
 * qcap = L) and kbar [B, Hkv, nb, d] fp32 = the block means of the prompt [0, P) in blocks of
 * bs (as focus_block_means). Where the many-row kernel serves the shape (d = 128, enough
 * 256-row blocks to fill the GPU) and bs divides 128, the block means are summed from the K
 * tiles the attention streams anyway: one launch, no second read of K. Otherwise the two
 * calls run in sequence; ws/ws_bytes then serve the dense attention (size them with
 * focus_dense_workspace_bytes(B, Hq, Hkv, L, d, L, 0)). Requires 1 <= P <= L, bs >= 1,
 * kbar 16-byte aligned and the conditions of focus_dense_attention.
 */
FOCUS_API int focus_full_refresh(const focus_bf16* Q, const focus_bf16* K, const focus_bf16* V, int B, int Hq,
                                 int Hkv, int L, int d, float scale, focus_bf16* O, int P, int bs, float* kbar,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * (3) The sink layer in one call -- method steps (3) and core method: dense attention of the
 * active queries (as focus_dense_attention), the sink importance colsum [B, Hkv, L] (as its
 * colsum_opt) and the sinks [B, Hkv, S] = top-min(S, L) columns of colsum per KV head,
 * ascending, -1 tail (as focus_sink_identify). Where the few-query kernel serves the shape
 * (d = 128, (Hq/Hkv) * qcap <= 64) the attention and the column sums run in one launch:
 * after the cluster merge the kernel re-reads the K tiles, most recently read first, for
 * the column sums. The same launch also selects the sinks within the cluster when
 * S <= 512, S <= L and (CTAs per KV head) x S <= 2048; otherwise the top-S runs as a
 * second launch. Other shapes run the calls in sequence. colsum and sinks are both written in every case. Requires 1 <= S <= 4096
 * and the conditions of focus_dense_attention with column sums; ws/ws_bytes as there.
 */
FOCUS_API int focus_dense_attention_sinks(const focus_bf16* Q, const int32_t* n_q, const focus_bf16* K,
                                          const focus_bf16* V, int B, int Hq, int Hkv, int L, int d, int qcap,
                                          float scale, focus_bf16* O, float* colsum, int S, int32_t* sinks, void* ws,
                                          size_t ws_bytes, void* stream);

/*
 * (3) Sink identification -- core method / method steps (3): the attention distribution
 * of the sink layer, aggregated over the active queries, picks the S sinks per KV head,
 * reused by every deeper sparse layer. sinks[b, h, :] = top-min(S, L) of colsum[b, h, :],
 * ascending, -1 tail. colsum [B, Hkv, L] fp32 -> sinks [B, Hkv, S] int32. Requires
 * 1 <= S <= 4096.
 */
FOCUS_API int focus_sink_identify(const float* colsum, int B, int Hkv, int L, int S, int32_t* sinks, void* stream);

/*
 * (5) Sparse attention -- method steps (5): for each active query (i < n_active[b]) of
 * head hq (KV head h): O_active[b, hq, i] = softmax over I_p of scale * q . k, applied to V,
 * with I_p = sinks[b, h, :] U (blocks [j*bs, min(P, (j+1)*bs)) for j in blocks[b, h, :])
 * U [g0, g1) taken as a SET (a key named twice counts once). Negative entries of
 * sinks/blocks are ignored; entries must otherwise lie in [0, L) and [0, nb). Rows
 * i >= n_active[b] of O_active are written as zero.
 * ws/ws_bytes: at least focus_sparse_workspace_bytes(...) bytes, 256-byte aligned.
 * Requires d in {64, 128}, L >= 8, 0 <= P <= g0 < g1 <= L, bs >= 1, 0 <= S <= 1024,
 * 1 <= C <= 1024, blocks sorted ascending among their valid entries.
 */
FOCUS_API int focus_sparse_attention(const focus_bf16* Q_active, const int32_t* n_active, const focus_bf16* K,
                           const focus_bf16* V, const int32_t* sinks, int S, const int32_t* blocks, int C, int bs,
                           int P, int g0, int g1, int B, int Hq, int Hkv, int L, int d, int acap, float scale,
                           focus_bf16* O_active, void* ws, size_t ws_bytes, void* stream);

/*
 * (4b)+(5) Block relevance, top-C and sparse attention of one layer in a single launch --
 * method steps (4) and (5). Same results as focus_block_select (kept blocks written to
 * blocks [B, Hkv, C], -1 tail) followed by focus_sparse_attention on them. kbar
 * [B, Hkv, nb, d] fp32 with nb = ceil(P / bs). Shapes outside the fused kernel's range
 * (d != 128, more than 256 query rows per KV head, nb > 4096, C > 512 or S > 512) run the
 * two calls in sequence; ws/ws_bytes then serve focus_sparse_attention (size them with
 * focus_sparse_workspace_bytes).
 */
FOCUS_API int focus_sparse_attention_fused(const focus_bf16* Q_active, const int32_t* n_active, const focus_bf16* K,
                                           const focus_bf16* V, const float* kbar, int nb, int C,
                                           const int32_t* sinks, int S, int bs, int P, int g0, int g1, int B, int Hq,
                                           int Hkv, int L, int d, int acap, float scale, int32_t* blocks,
                                           focus_bf16* O_active, void* ws, size_t ws_bytes, void* stream);

FOCUS_API size_t focus_sparse_workspace_bytes(int B, int Hq, int Hkv, int L, int d, int acap, int S, int C, int bs, int P,
                                    int g0, int g1);

/*
 * Allocation-free variant of focus_sparse_attention. The paper has no counterpart: this
 * entry point exists for callers that cannot call cudaMalloc, e.g. code that runs while a
 * stream is being captured in a mode that forbids allocation, plugin hosts whose enqueue
 * path must not allocate, or servers that reserve all device memory up front. It takes the
 * same arguments minus the workspace and computes the same result.
 *
 * Scratch: the split-KV partials live in one library-owned device array of
 * FOCUS_NOALLOC_SCRATCH_BYTES bytes (a static __device__ array: every GPU that loads the
 * library holds it until the process exits). A call whose partials would need more
 * (focus_sparse_workspace_bytes(...) > FOCUS_NOALLOC_SCRATCH_BYTES) returns
 * FOCUS_ERR_CAPACITY and launches nothing. The call allocates nothing.
 * The first call on a device looks the array's device address up (cudaGetSymbolAddress,
 * with that device current) and caches it per device ordinal; make that first call before
 * any stream capture. The cached address is only valid for the device context it was
 * taken in: after a cudaDeviceReset (or any other teardown of the primary context) it is
 * stale, and this entry point must not be called again in that process.
 * All calls share the array and it keeps the previous call's contents; every element a
 * call reads is written earlier by the same call, so nothing has to be cleared (a split
 * whose kernel gave up on a timed-out wait marks its partial empty). Calls that overlap
 * on the GPU (e.g. on two streams without ordering) race on the array. After a call that
 * leaves the device error word set (focus_device_error), its output is undefined.
 */
#define FOCUS_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

FOCUS_API int focus_sparse_attention_noalloc(const focus_bf16* Q_active, const int32_t* n_active,
                                             const focus_bf16* K, const focus_bf16* V, const int32_t* sinks, int S,
                                             const int32_t* blocks, int C, int bs, int P, int g0, int g1, int B,
                                             int Hq, int Hkv, int L, int d, int acap, float scale,
                                             focus_bf16* O_active, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FOCUS_H_ */
