"""Oracle for the Focus-dLLM sparse denoising-step attention (plain, slow, fp64, CPU).

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import this module. The product path (the CUDA
library and its Python binding) never imports, links or calls it, and this module
imports nothing from the product package.

Source of every definition: "Focus-dLLM: Accelerating Long-Context Diffusion LLM
Inference via Confidence-Guided Context Focusing" (summary page of arXiv 2602.02159),
section "方法步骤详情" (method steps), steps (1)-(5), and section "核心方法" (core
method) for PCGI and sink-aware pruning; the English abstract on the paperdance.org
card for cross-layer sink reuse. Readings taken where the pages are silent (numbered
o1..o22 with the design notes):
  * PCGI candidates are the still-[MASK] positions of the current block [g0, g1).
  * k = floor(rho * n_t), clamped to the number of candidates.
  * a window of size w around p is [p - w//2, p - w//2 + w - 1], clipped to [g0, g1).
  * block relevance R_b^h = mean over active queries i and the query heads of KV
    group h of q_i . kbar_b / sqrt(d); an empty active set gives R = 0.
  * sink importance = sum over active queries (and the group's query heads) of the
    softmax probability of each key column; every one of the L columns is a candidate.
  * the sparse key set I_p = sinks U selected prompt blocks U [g0, g1), as a set.
  * every top-k orders by (score descending, index ascending), -0.0 == +0.0, and
    returns its indices ascending. Scores must be finite.

Everything is computed in float64 from the exact (widened) bf16 / fp32 inputs.
Parity status: every function here is pinned by tests/test_oracle_pins.py
(brute force, closed forms, library routines, planted structure); the composed
step schedule is pinned only by composition of its parts. The top-k margins of the
fixed seeds (how far each selected set is from a near-tie) are recorded by
tests/golden/make_topk_margins.py.
"""
from __future__ import annotations

import math
from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np


# --------------------------------------------------------------------------- top-k
def top_k_ascending(scores: np.ndarray, k: int) -> np.ndarray:
    """The k best indices under (score desc, index asc), returned in ascending order.

    Every top-k of the method (PCGI "选取top-k个最高的[MASK]位置", block "top-C",
    sinks) uses this order. Ties go to the lower index.
    """
    s = np.asarray(scores, dtype=np.float64).reshape(-1)
    if not np.all(np.isfinite(s)):
        raise ValueError("oracle top-k: scores must be finite")
    s = np.where(s == 0.0, 0.0, s)          # -0.0 and +0.0 are the same key
    k = max(0, min(int(k), s.size))
    idx = np.arange(s.size)
    order = np.lexsort((idx, -s))           # primary: -score ascending; secondary: index
    return np.sort(order[:k]).astype(np.int64)


def top_k_margin(scores: np.ndarray, k: int) -> float:
    """Gap between the k-th and (k+1)-th best score: how far the kept set of a top-k is
    from changing. inf when no score is dropped (k <= 0 or k >= n); 0 on a boundary tie,
    where only the index order decides."""
    s = np.sort(np.asarray(scores, dtype=np.float64).reshape(-1))[::-1]
    if k <= 0 or k >= s.size:
        return math.inf
    return float(s[k - 1] - s[k])


def top_k_relative_margin(scores: np.ndarray, k: int) -> float:
    """top_k_margin relative to the magnitude of the k-th best score (inf as above; the
    gap itself when the k-th score is 0)."""
    gap = top_k_margin(scores, k)
    if not math.isfinite(gap):
        return gap
    s = np.sort(np.asarray(scores, dtype=np.float64).reshape(-1))[::-1]
    ref = abs(float(s[k - 1]))
    return gap / ref if ref > 0.0 else gap


# ------------------------------------------------------- step (1)+(2): PCGI + windows
def select_queries(conf_prev: np.ndarray, mask: np.ndarray, g0: int, g1: int,
                   n_t: int, rho: float, w: int) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Past Confidence-Guided Indicator and window expansion.

    Method steps (1): among positions still [MASK], take the top-k by the previous
    step's confidence c_{t-1}, k = floor(rho * n(t)) -> I_focus. Method steps (2):
    expand each p in I_focus to a local window of size w; the union is I_active.

    conf_prev: [B, G] with conf_prev[b, p - g0] = c_{t-1} at position p.
    mask:      [B, L], nonzero = still [MASK].
    Returns per-batch ascending int64 arrays (I_focus, I_active).
    """
    B = conf_prev.shape[0]
    k_req = int(math.floor(float(rho) * float(n_t)))
    focus_all, active_all = [], []
    for b in range(B):
        cand = [p for p in range(g0, g1) if mask[b, p] != 0]
        k = min(k_req, len(cand))
        cand_scores = np.array([conf_prev[b, p - g0] for p in cand], dtype=np.float64)
        chosen = top_k_ascending(cand_scores, k) if cand else np.zeros(0, np.int64)
        focus = np.array(sorted(cand[i] for i in chosen), dtype=np.int64)
        active = set()
        for p in focus:
            lo = p - w // 2
            for q in range(max(g0, lo), min(g1 - 1, lo + w - 1) + 1):
                active.add(q)
        focus_all.append(focus)
        active_all.append(np.array(sorted(active), dtype=np.int64))
    return focus_all, active_all


def gather_rows(X: np.ndarray, rows: Sequence[np.ndarray], cap: int) -> np.ndarray:
    """X[b, h, rows[b][i]] into [B, H, cap, d]; rows past len(rows[b]) are zero."""
    B, H, _, d = X.shape
    out = np.zeros((B, H, cap, d), dtype=np.float64)
    for b in range(B):
        r = np.asarray(rows[b], dtype=np.int64)
        out[b, :, :r.size] = X[b][:, r]
    return out


# --------------------------------------------------------- step (4): block means
def refresh_rows(X: np.ndarray, rows: Sequence[np.ndarray], X_new: np.ndarray) -> np.ndarray:
    """Approximate KV cache (summary page, "近似KV缓存"): a token i of the refresh set U(t)
    takes its recomputed state, every other token keeps the cached one:
    X'[b, h, i] = X_new[b, h, k] where rows[b][k] == i, else X[b, h, i].
    X [B, H, L, d], X_new [B, H, cap, d] (row k of sequence b for k < len(rows[b]))."""
    out = X.copy()
    for b, r in enumerate(rows):
        for k, i in enumerate(r):
            out[b, :, int(i)] = X_new[b, :, k]
    return out


def block_means(K: np.ndarray, P: int, bs: int) -> np.ndarray:
    """Representative key of each prompt block = mean of the block's keys.

    Method steps (4): prompt tokens [0, P) are cut into contiguous blocks of bs; a
    block's representative key is the mean of its keys. A short last block averages
    only its valid rows. K: [B, Hkv, L, d] -> kbar [B, Hkv, nb, d].
    """
    B, H, _, d = K.shape
    nb = -(-P // bs)
    kbar = np.zeros((B, H, nb, d), dtype=np.float64)
    for blk in range(nb):
        r0, r1 = blk * bs, min(P, (blk + 1) * bs)
        kbar[:, :, blk] = K[:, :, r0:r1].mean(axis=2)
    return kbar


# ---------------------------------------------- step (4): relevance R_b + top-C
def block_relevance(Q_active: np.ndarray, n_active: Sequence[int],
                    kbar: np.ndarray) -> np.ndarray:
    """R_b^h = mean over active queries i and query heads of group h of q_i . kbar_b / sqrt(d).

    Method steps (4) ("计算候选查询与每个块的相关性分数R_b"). Q_active [B, Hq, acap, d],
    kbar [B, Hkv, nb, d] -> R [B, Hkv, nb]. An empty active set gives R = 0.
    """
    B, Hq, _, d = Q_active.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    g = Hq // Hkv
    R = np.zeros((B, Hkv, nb), dtype=np.float64)
    for b in range(B):
        A = int(n_active[b])
        if A == 0:
            continue
        for h in range(Hkv):
            q = Q_active[b, h * g:(h + 1) * g, :A].reshape(g * A, d)   # every (head, query)
            dots = (q @ kbar[b, h].T) / math.sqrt(d)                   # [g*A, nb]
            R[b, h] = dots.mean(axis=0)
    return R


def block_select(Q_active: np.ndarray, n_active: Sequence[int], kbar: np.ndarray,
                 C: int) -> Tuple[np.ndarray, np.ndarray]:
    """Top-C prompt blocks per KV head by R_b. Returns (blocks [B,Hkv,C] with -1 tail, R)."""
    R = block_relevance(Q_active, n_active, kbar)
    B, Hkv, nb = R.shape
    blocks = np.full((B, Hkv, C), -1, dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            sel = top_k_ascending(R[b, h], min(C, nb))
            blocks[b, h, :sel.size] = sel
    return blocks, R


# ----------------------------------------------- step (3) / block entry: dense attention
def dense_attention(Q: np.ndarray, n_q: Optional[Sequence[int]], K: np.ndarray,
                    V: np.ndarray, scale: float, want_colsum: bool = False):
    """Full bidirectional attention over all L keys.

    Method steps (3): the first l_dense layers run full attention; at a block-entry
    step the whole sequence does (use_sparse = False). For query i of head hq (KV head
    h = hq // g): s_ij = scale * q_i . k_j, p_ij = softmax_j(s_ij), o_i = sum_j p_ij v_j.
    With want_colsum, the sink importance of column j for KV head h is
    colsum[b, h, j] = sum over the group's query heads and the valid queries of p_ij
    (core method: sinks are found from the attention distribution of the dense layer).

    Q [B, Hq, nq, d] (rows >= n_q[b] ignored and returned as zero), K/V [B, Hkv, L, d].
    Returns (O [B, Hq, nq, d], colsum [B, Hkv, L] or None, lse [B, Hq, nq] natural log).
    """
    B, Hq, nq, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    g = Hq // Hkv
    O = np.zeros((B, Hq, nq, d), dtype=np.float64)
    lse = np.full((B, Hq, nq), -np.inf, dtype=np.float64)
    colsum = np.zeros((B, Hkv, L), dtype=np.float64) if want_colsum else None
    for b in range(B):
        n = nq if n_q is None else int(n_q[b])
        if n == 0:
            continue
        for hq in range(Hq):
            h = hq // g
            s = (Q[b, hq, :n] @ K[b, h].T) * scale             # [n, L]
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            p = e / l
            O[b, hq, :n] = p @ V[b, h]
            lse[b, hq, :n] = (m + np.log(l))[:, 0]
            if want_colsum:
                colsum[b, h] += p.sum(axis=0)
    return O, colsum, lse


# ------------------------------------------------------ step (3): sink identification
def sink_identify(colsum: np.ndarray, S: int) -> np.ndarray:
    """Top-S columns of the dense layer's aggregated attention, per KV head.

    Core method / method steps (3): the attention distribution of layer l_dense
    identifies the attention sinks, which every deeper sparse layer reuses unchanged
    (cross-layer consistency, abstract). colsum [B, Hkv, L] -> sinks [B, Hkv, S]
    ascending, -1 tail when S > L.
    """
    B, Hkv, L = colsum.shape
    sinks = np.full((B, Hkv, S), -1, dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            sel = top_k_ascending(colsum[b, h], min(S, L))
            sinks[b, h, :sel.size] = sel
    return sinks


# ------------------------------------------------------- step (5): sparse attention
def sparse_key_set(sinks_bh: np.ndarray, blocks_bh: np.ndarray, bs: int, P: int,
                   g0: int, g1: int) -> np.ndarray:
    """I_p = I_sink U (selected prompt blocks) U [g0, g1), as an ascending set."""
    keys = set(int(j) for j in sinks_bh if j >= 0)
    for blk in blocks_bh:
        if blk < 0:
            continue
        keys.update(range(int(blk) * bs, min(P, (int(blk) + 1) * bs)))
    keys.update(range(g0, g1))
    return np.array(sorted(keys), dtype=np.int64)


def sparse_attention(Q_active: np.ndarray, n_active: Sequence[int], K: np.ndarray,
                     V: np.ndarray, sinks: np.ndarray, blocks: np.ndarray, bs: int,
                     P: int, g0: int, g1: int, scale: float) -> np.ndarray:
    """Method steps (5): the active queries attend, bidirectionally, only over I_p.

    Q_active [B, Hq, acap, d]; sinks [B, Hkv, S]; blocks [B, Hkv, C] (-1 = unused).
    Returns O [B, Hq, acap, d] (rows >= n_active[b] zero).
    """
    B, Hq, acap, d = Q_active.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    O = np.zeros((B, Hq, acap, d), dtype=np.float64)
    for b in range(B):
        A = int(n_active[b])
        if A == 0:
            continue
        for h in range(Hkv):
            Ip = sparse_key_set(sinks[b, h], blocks[b, h], bs, P, g0, g1)
            Kp, Vp = K[b, h, Ip], V[b, h, Ip]
            for hq in range(h * g, (h + 1) * g):
                s = (Q_active[b, hq, :A] @ Kp.T) * scale
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                p = e / e.sum(axis=1, keepdims=True)
                O[b, hq, :A] = p @ Vp
    return O


# ------------------------------------------------------------- the step schedule
def sink_identify_mean_query(Q_active: np.ndarray, n_active: Sequence[int], K: np.ndarray,
                             S: int) -> Tuple[np.ndarray, np.ndarray]:
    """Variant sink importance (summary page, "方法步骤详情" (3): token importance from an
    aggregated query representation): the attention of the group's mean active query,
    softmax_j(qbar . k_j / sqrt(d)), over all L columns. The softmax is monotone in the
    score, so the top-S columns are the top-S of R_j = qbar . k_j / sqrt(d): block relevance
    with every key its own block. Returns (sinks [B,Hkv,S], R)."""
    return block_select(Q_active, n_active, K, S)


def sparse_step(layer_fn: Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]],
                n_layers: int, l_dense: int, conf_prev: np.ndarray, mask: np.ndarray,
                g0: int, g1: int, n_t: int, rho: float, w: int, P: int, bs: int,
                C: int, S: int, acap: int, scale: float, layers_out=None, dense_tail: int = 0,
                relevance: str = "active", sink_agg: str = "probs", layers_eval=None):
    """One non-block-entry denoising step (method steps (1)-(5)).

    layer_fn(l) -> (Q_full [B,Hq,L,d], K, V) in float64. Layers 0..l_dense are dense over
    the active queries; layer l_dense also yields the sinks; deeper layers select top-C
    blocks from their own block means and attend over sinks U blocks U the current block.
    Returns a dict with I_focus, I_active, sinks (and the sink layer's colsum), per-layer
    blocks and relevance scores R, and outputs (only for layers in `layers_out`, default all).
    `layers_eval` (default all) limits which layers are computed at all: layer_fn supplies
    every layer's inputs, so a layer's results depend only on its own inputs and on the
    sinks of layer l_dense (always computed); the skipped layers are simply absent.

    Variants the pages describe: the last `dense_tail` layers also run dense (Dream keeps
    its last 4 layers dense); relevance="focus" scores the blocks with the I_focus rows
    instead of I_active (method steps (4) speaks of the candidate queries);
    sink_agg="mean_query" picks the sinks by the mean active query's attention
    (sink_identify_mean_query) instead of the summed softmax rows.
    """
    focus, active = select_queries(conf_prev, mask, g0, g1, n_t, rho, w)
    n_active = [a.size for a in active]
    out = {"I_focus": focus, "I_active": active, "O": {}, "blocks": {}, "R": {}, "sinks": None}
    want = set(range(n_layers)) if layers_out is None else set(layers_out)
    run = set(range(n_layers)) if layers_eval is None else set(layers_eval) | {l_dense}
    tail0 = max(l_dense + 1, n_layers - dense_tail)
    for l in range(n_layers):
        if l not in run:
            continue
        Q, K, V = layer_fn(l)
        Qa = gather_rows(Q, active, acap)
        if l <= l_dense or l >= tail0:
            sink_layer = l == l_dense
            O, colsum, _ = dense_attention(Qa, n_active, K, V, scale, want_colsum=sink_layer and sink_agg == "probs")
            if sink_layer:
                if sink_agg == "probs":
                    out["sinks"] = sink_identify(colsum, S)
                    out["colsum"] = colsum
                else:
                    out["sinks"], out["sink_scores"] = sink_identify_mean_query(Qa, n_active, K, S)
        else:
            kbar = block_means(K, P, bs)
            if relevance == "focus":
                Qr = gather_rows(Q, focus, g1 - g0)
                blocks, R = block_select(Qr, [f.size for f in focus], kbar, C)
            else:
                blocks, R = block_select(Qa, n_active, kbar, C)
            out["blocks"][l] = blocks
            out["R"][l] = R
            O = sparse_attention(Qa, n_active, K, V, out["sinks"], blocks, bs, P, g0, g1, scale)
        if l in want:
            out["O"][l] = O
    return out
