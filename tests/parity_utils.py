"""Helpers for the GPU-vs-oracle parity tests (comparison only; no method arithmetic)."""
import numpy as np
import torch

# Attention outputs: bf16 inputs, fp32 accumulation, bf16 output vs the fp64 oracle.
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
# Block means: fp32 accumulation of bf16 rows vs fp64.
KBAR_REL = 1e-3


def assert_attention_close(got: torch.Tensor, ref: np.ndarray, rows_valid=None, what="attention"):
    g = got.detach().to("cpu").to(torch.float64).numpy()
    if rows_valid is not None:
        # rows_valid: per-batch number of valid rows along axis 2
        parts_g, parts_r = [], []
        for b, n in enumerate(rows_valid):
            parts_g.append(g[b, :, :n].reshape(-1))
            parts_r.append(ref[b, :, :n].reshape(-1))
            assert np.all(g[b, :, n:] == 0.0), f"{what}: rows past the valid count must be zero"
        gv, rv = np.concatenate(parts_g), np.concatenate(parts_r)
    else:
        gv, rv = g.reshape(-1), ref.reshape(-1)
    assert np.all(np.isfinite(gv)), f"{what}: non-finite output"
    err = np.abs(gv - rv)
    max_abs, mean_abs = float(err.max(initial=0.0)), float(err.mean() if err.size else 0.0)
    assert max_abs <= ATTN_MAX_ABS and mean_abs <= ATTN_MEAN_ABS, \
        f"{what}: max-abs {max_abs:.3e} (<= {ATTN_MAX_ABS}), mean-abs {mean_abs:.3e} (<= {ATTN_MEAN_ABS})"
    return max_abs, mean_abs


def idx_rows(t: torch.Tensor):
    """Device index tensor [..., cap] -> nested python lists without the -1 tail."""
    a = t.detach().to("cpu").numpy()
    flat = a.reshape(-1, a.shape[-1])
    out = [[int(x) for x in row if x >= 0] for row in flat]
    return out


def assert_tail_is_minus_one(t: torch.Tensor, counts):
    a = t.detach().to("cpu").numpy().reshape(-1, t.shape[-1])
    for row, n in zip(a, counts):
        assert np.all(row[n:] == -1), "unused index slots must hold -1"
        assert np.all(np.diff(row[:n]) > 0), "indices must be strictly ascending"


def topk_matches(got, scores, k, rel=1e-4):
    """Exact top-k match (returns True), or a mismatch confined to scores tied within `rel`
    of the k-th score (returns False after checking the GPU set is a valid top-k)."""
    from oracle import focus_oracle as orc
    exp = orc.top_k_ascending(scores, k).tolist()
    if list(got) == exp:
        return True
    s = np.asarray(scores, dtype=np.float64)
    kth = np.sort(s)[::-1][min(k, s.size) - 1]
    tol = rel * max(1.0, abs(kth))
    diff = set(got) ^ set(exp)
    assert len(got) == len(exp), f"top-k size {len(got)} != {len(exp)}"
    assert all(abs(s[i] - kth) <= tol for i in diff), f"top-k mismatch beyond a near-tie: {sorted(diff)}"
    return False


def assert_index_sets(got_t, scores, k, what):
    """Per-(b, h) top-k sets of a device tensor [B, H, cap] vs oracle scores [B, H, n]."""
    got = got_t.detach().to("cpu").numpy()
    ties = 0
    for b in range(got.shape[0]):
        for h in range(got.shape[1]):
            row = [int(x) for x in got[b, h] if x >= 0]
            ties += not topk_matches(row, scores[b, h], k)
            assert np.all(got[b, h, min(k, scores.shape[-1]):] == -1), f"{what}: tail must be -1"
    return ties
