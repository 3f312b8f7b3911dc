"""Pins for the oracle against what the pages and the mathematics fix (CPU only).

Each test checks an oracle function against something other than itself: a
hand-worked example derived from the Focus-dLLM method steps (tests/golden/), brute
force on tiny inputs, a library routine (torch scaled_dot_product_attention in
float64, numpy reduceat), a closed form, an invariant, or planted structure.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import focus_oracle as orc


def _ints(v):
    return [int(x) for x in v]


def _floats(v):
    return [float(x) for x in v]


# ----------------------------------------------------------------------------- top-k
def _dominates(si, i, sj, j):
    """(score desc, index asc) order; -0.0 == +0.0 because 0.0 == -0.0 in IEEE."""
    return si > sj or (si == sj and i < j)


def _brute_top_k(scores, k):
    n = len(scores)
    good = []
    for subset in itertools.combinations(range(n), k):
        inside = set(subset)
        if all(_dominates(scores[i], i, scores[j], j)
               for i in inside for j in range(n) if j not in inside):
            good.append(subset)
    assert len(good) == 1, "the order key must single out exactly one k-subset"
    return list(good[0])


def test_top_k_brute_force_with_ties():
    rng = np.random.default_rng(7)
    for _ in range(400):
        n = int(rng.integers(1, 9))
        vals = rng.choice([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 3.0], size=n)
        k = int(rng.integers(0, n + 1))
        got = orc.top_k_ascending(vals, k).tolist()
        assert got == _brute_top_k(list(vals), k)


def test_top_k_margin_brute_force():
    """The margin is the gap between the worst kept and the best dropped score of the
    brute-forced top-k (0 on a boundary tie, inf when nothing is dropped)."""
    rng = np.random.default_rng(8)
    for _ in range(400):
        n = int(rng.integers(1, 9))
        vals = rng.choice([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 3.0, 7.5], size=n)
        k = int(rng.integers(0, n + 1))
        got = orc.top_k_margin(vals, k)
        if k == 0 or k == n:
            assert got == math.inf
            continue
        kept = set(_brute_top_k(list(vals), k))
        want = min(vals[i] for i in kept) - max(vals[j] for j in range(n) if j not in kept)
        assert got == want
    assert orc.top_k_margin([3.0, 1.0, 2.0], 1) == 1.0
    assert orc.top_k_margin([2.0, 2.0, 1.0], 1) == 0.0
    assert orc.top_k_margin([0.5, -0.0, 0.0], 1) == 0.5
    assert orc.top_k_relative_margin([4.0, 3.0, 1.0], 2) == 2.0 / 3.0
    assert orc.top_k_relative_margin([4.0, 0.0, -1.0], 2) == 1.0
    assert orc.top_k_relative_margin([4.0, 3.0], 2) == math.inf


def test_top_k_golden_ties():
    g = read_golden("sink_topk_ties.txt")
    cs = np.array(_floats(g["colsum"]))
    for key, S in (("top3", 3), ("top4", 4), ("top6", 6)):
        assert orc.top_k_ascending(cs, S).tolist() == _ints(g[key])


def test_top_k_rejects_nan():
    with pytest.raises(ValueError):
        orc.top_k_ascending(np.array([1.0, np.nan]), 1)


# ----------------------------------------------------------------- select_queries
def _golden_select(name, w):
    g = read_golden(name)
    g0, g1, L = int(g["g0"][0]), int(g["g1"][0]), int(g["L"][0])
    mask = np.zeros((1, L), np.uint8)
    mask[0, g0:g1] = _ints(g["mask_block"])
    conf = np.array([_floats(g["conf_block"])], dtype=np.float32)
    focus, active = orc.select_queries(conf, mask, g0, g1, int(g["n_t"][0]),
                                       float(g["rho"][0]), w)
    return g, focus[0].tolist(), active[0].tolist()


@pytest.mark.parametrize("w", [3, 4])
def test_select_queries_golden(w):
    g, focus, active = _golden_select("select_queries_example.txt", w)
    assert focus == _ints(g[f"case_w{w}_focus"])
    assert active == _ints(g[f"case_w{w}_active"])


def test_select_queries_golden_edge():
    g, focus, active = _golden_select("select_queries_edge.txt", 4)
    assert focus == _ints(g["case_w4_focus"])
    assert active == _ints(g["case_w4_active"])


def test_select_queries_brute_force_and_invariants():
    rng = np.random.default_rng(11)
    for trial in range(1500):
        G = int(rng.integers(1, 11))
        g0 = int(rng.integers(0, 5))
        g1 = g0 + G
        L = g1 + int(rng.integers(0, 4))
        mask = np.zeros((1, L), np.uint8)
        mask[0, g0:g1] = rng.integers(0, 2, size=G)
        # a coarse value set makes ties common
        conf = rng.choice(np.float32([0.1, 0.5, 0.5, 0.9, 0.0, -0.0]), size=(1, G)).astype(np.float32)
        n_t = int(rng.integers(0, 4))
        rho = float(rng.choice([1.0, 2.0, 2.5, 4.0]))
        w = int(rng.integers(1, 6))
        focus, active = orc.select_queries(conf, mask, g0, g1, n_t, rho, w)
        focus, active = focus[0].tolist(), active[0].tolist()
        cand = [p for p in range(g0, g1) if mask[0, p]]
        k = min(int(math.floor(rho * n_t)), len(cand))
        # brute force over every k-subset of the candidates
        scores = [float(conf[0, p - g0]) for p in cand]
        expect = sorted(cand[i] for i in _brute_top_k(scores, k)) if cand else []
        assert focus == expect
        # invariants
        assert len(focus) == k
        assert set(focus) <= set(cand)
        assert set(focus) <= set(active) <= set(range(g0, g1))
        assert len(active) <= k * w
        assert active == sorted(set(active))
        # each window is contiguous around its centre: p itself and, when w > 1 and
        # the block allows, its left neighbour (floor(w/2) >= 1) are active
        for p in focus:
            if w > 1 and p - 1 >= g0:
                assert p - 1 in active


def test_select_queries_window_size_inside_block():
    """A lone focus position far from the block edges yields exactly w active positions."""
    L, g0, g1 = 64, 0, 64
    for w in range(1, 9):
        mask = np.zeros((1, L), np.uint8)
        mask[0, 30] = 1
        conf = np.zeros((1, 64), np.float32)
        focus, active = orc.select_queries(conf, mask, g0, g1, 1, 1.0, w)
        assert focus[0].tolist() == [30]
        assert len(active[0]) == w and 30 in active[0].tolist()


# -------------------------------------------------------------------- block means
def test_block_means_against_reduceat():
    rng = np.random.default_rng(3)
    for P, bs in ((64, 16), (70, 16), (5, 8), (33, 1)):
        K = rng.standard_normal((2, 3, P + 9, 5))
        kbar = orc.block_means(K, P, bs)
        starts = np.arange(0, P, bs)
        counts = np.diff(np.append(starts, P))
        sums = np.add.reduceat(K[:, :, :P], starts, axis=2)
        np.testing.assert_allclose(kbar, sums / counts[None, None, :, None], rtol=1e-13, atol=1e-13)
        # total mass: sum_b count_b * kbar_b == sum of all prompt rows
        np.testing.assert_allclose((kbar * counts[None, None, :, None]).sum(axis=2),
                                   K[:, :, :P].sum(axis=2), rtol=1e-12, atol=1e-12)


def test_block_means_bs1_is_identity():
    K = np.random.default_rng(4).standard_normal((1, 2, 12, 4))
    np.testing.assert_array_equal(orc.block_means(K, 10, 1), K[:, :, :10])


# ------------------------------------------------------------------ block_select
def test_block_relevance_golden():
    g = read_golden("block_relevance_example.txt")
    d = int(g["d"][0])
    Q = np.zeros((1, 2, 4, d))
    Q[0, 0, :2] = np.array([_floats(r) for r in g["q_head0"]])
    Q[0, 1, :2] = np.array([_floats(r) for r in g["q_head1"]])
    kbar = np.array([[_floats(r) for r in g["kbar"]]])[:, None]     # [1,1,4,d]
    R = orc.block_relevance(Q, [2], kbar)
    np.testing.assert_allclose(R[0, 0], _floats(g["R"]), rtol=0, atol=1e-15)
    assert orc.block_select(Q, [2], kbar, 2)[0][0, 0].tolist() == _ints(g["top2"])
    assert orc.block_select(Q, [2], kbar, 3)[0][0, 0].tolist() == _ints(g["top3"])


def test_block_relevance_equals_mean_query_closed_form():
    """mean_i (q_i . k) = (mean_i q_i) . k: R from the double sum equals qbar . kbar / sqrt(d)."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, acap, d, nb = 2, 6, 2, 9, 16, 13
    Q = rng.standard_normal((B, Hq, acap, d))
    kbar = rng.standard_normal((B, Hkv, nb, d))
    n_active = [7, 3]
    R = orc.block_relevance(Q, n_active, kbar)
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            qbar = Q[b, h * g:(h + 1) * g, :n_active[b]].mean(axis=(0, 1))
            np.testing.assert_allclose(R[b, h], kbar[b, h] @ qbar / math.sqrt(d), rtol=1e-12, atol=1e-13)


def test_block_select_planted_block_and_brute_force():
    rng = np.random.default_rng(6)
    B, Hq, Hkv, acap, d, nb = 1, 2, 2, 8, 8, 7
    Q = rng.standard_normal((B, Hq, acap, d))
    kbar = rng.standard_normal((B, Hkv, nb, d)) * 0.1
    for h in range(Hkv):
        qbar = Q[0, h, :5].mean(axis=0)
        kbar[0, h, 4] = 10.0 * qbar          # planted: aligned with the mean query
    blocks, R = orc.block_select(Q, [5], kbar, 3)
    for h in range(Hkv):
        assert 4 in blocks[0, h].tolist()
        assert blocks[0, h].tolist() == sorted(_brute_top_k(list(R[0, h]), 3))
    # C larger than nb: everything, -1 tail
    blocks, _ = orc.block_select(Q, [5], kbar, nb + 2)
    assert blocks[0, 0].tolist() == list(range(nb)) + [-1, -1]


def test_block_relevance_empty_active_is_zero():
    R = orc.block_relevance(np.ones((1, 1, 4, 4)), [0], np.ones((1, 1, 3, 4)))
    assert np.all(R == 0.0)


# -------------------------------------------------------------- dense attention
def _sdpa_reference(Q, K, V, n_q, scale):
    """torch scaled_dot_product_attention in float64 on the CPU (library routine)."""
    B, Hq, nq, d = Q.shape
    g = Hq // K.shape[1]
    Kx = torch.from_numpy(np.repeat(K, g, axis=1))
    Vx = torch.from_numpy(np.repeat(V, g, axis=1))
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), Kx, Vx, scale=scale).numpy()
    for b in range(B):
        out[b, :, n_q[b]:] = 0.0
    return out


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (6, 2)])
def test_dense_attention_vs_sdpa(Hq, Hkv):
    rng = np.random.default_rng(8)
    B, nq, L, d = 2, 5, 37, 16
    Q = rng.standard_normal((B, Hq, nq, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    n_q = [5, 3]
    scale = 1 / math.sqrt(d)
    O, colsum, lse = orc.dense_attention(Q, n_q, K, V, scale, want_colsum=True)
    np.testing.assert_allclose(O, _sdpa_reference(Q, K, V, n_q, scale), rtol=1e-11, atol=1e-12)
    # every probability row sums to one -> column sums total (group size) x (valid rows)
    g = Hq // Hkv
    for b in range(B):
        np.testing.assert_allclose(colsum[b].sum(axis=1), g * n_q[b], rtol=1e-12)
    # lse against a library logsumexp
    Kx = np.repeat(K, g, axis=1)
    s = np.einsum("bhqd,bhkd->bhqk", Q, Kx) * scale
    ref_lse = torch.logsumexp(torch.from_numpy(s), dim=-1).numpy()
    for b in range(B):
        np.testing.assert_allclose(lse[b, :, :n_q[b]], ref_lse[b, :, :n_q[b]], rtol=1e-12)


def test_dense_attention_golden_two_keys():
    g = read_golden("attention_two_keys.txt")
    Q = np.array(_floats(g["q"]))[None, None, None, :]
    K = np.array([_floats(r) for r in g["k"]])[None, None]
    V = np.array([_floats(r) for r in g["v"]])[None, None]
    O, colsum, lse = orc.dense_attention(Q, None, K, V, 1.0, want_colsum=True)
    np.testing.assert_allclose(O[0, 0, 0], _floats(g["o"]), rtol=1e-14)
    np.testing.assert_allclose(colsum[0, 0], _floats(g["colsum"]), rtol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], float(g["lse"][0]), rtol=1e-14)


def test_dense_attention_uniform_values():
    rng = np.random.default_rng(9)
    Q = rng.standard_normal((1, 2, 3, 8)) * 3
    K = rng.standard_normal((1, 2, 20, 8))
    v = rng.standard_normal(8)
    V = np.broadcast_to(v, (1, 2, 20, 8)).copy()
    O, _, _ = orc.dense_attention(Q, None, K, V, 0.3)
    np.testing.assert_allclose(O, np.broadcast_to(v, O.shape), rtol=1e-12)


# ---------------------------------------------------------------- sink identify
def test_sinks_recover_planted_positions():
    """Keys planted with +3 u (u along the mean query) dominate the aggregated attention."""
    from diffusion_long_context_b200 import configs, inputs
    cfg = configs.TINY
    st = inputs.step_state(cfg)
    Q, K, V = (inputs.to_f64(t) for t in inputs.make_layer(cfg, 0, "cpu", st.sink_pos))
    focus, active = orc.select_queries(st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, cfg.rho, cfg.w)
    Qa = orc.gather_rows(Q, active, cfg.acap)
    _, colsum, _ = orc.dense_attention(Qa, [a.size for a in active], K, V,
                                       1 / math.sqrt(cfg.d), want_colsum=True)
    sinks = orc.sink_identify(colsum, cfg.S)
    for h in range(cfg.Hkv):
        assert set(st.sink_pos.tolist()) <= set(sinks[0, h].tolist())


def test_sink_identify_brute_force():
    rng = np.random.default_rng(10)
    for _ in range(200):
        L = int(rng.integers(1, 9))
        cs = rng.choice([0.0, 0.5, 0.5, 1.0, 2.0], size=(1, 1, L))
        S = int(rng.integers(1, L + 2))
        got = orc.sink_identify(cs, S)[0, 0]
        k = min(S, L)
        assert got[:k].tolist() == sorted(_brute_top_k(list(cs[0, 0]), k))
        assert (got[k:] == -1).all()


# ------------------------------------------------------------- sparse attention
def test_sparse_key_set_golden():
    g = read_golden("sparse_key_set_example.txt")
    Ip = orc.sparse_key_set(np.array(_ints(g["sinks"])), np.array(_ints(g["blocks"])),
                            int(g["bs"][0]), int(g["P"][0]), int(g["g0"][0]), int(g["g1"][0]))
    assert Ip.tolist() == _ints(g["I_p"])


def test_sparse_equals_dense_when_everything_is_kept():
    """All blocks + every non-prompt, non-current-block position as sinks => I_p = [0, L)."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, L, d, bs = 1, 4, 2, 40, 8, 8
    P, g0, g1 = 24, 24, 32
    Q = rng.standard_normal((B, Hq, 6, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    nb = P // bs
    blocks = np.tile(np.arange(nb), (B, Hkv, 1))
    extra = np.arange(g1, L)
    sinks = np.tile(extra, (B, Hkv, 1))
    scale = 1 / math.sqrt(d)
    Os = orc.sparse_attention(Q, [6], K, V, sinks, blocks, bs, P, g0, g1, scale)
    Od, _, _ = orc.dense_attention(Q, [6], K, V, scale)
    np.testing.assert_allclose(Os, Od, rtol=1e-12, atol=1e-13)


def test_sparse_duplicates_count_once_and_match_masked_sdpa():
    rng = np.random.default_rng(13)
    B, Hq, Hkv, L, d, bs = 1, 2, 1, 48, 8, 8
    P, g0, g1 = 32, 32, 40
    Q = rng.standard_normal((B, Hq, 4, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    scale = 0.4
    blocks = np.array([[[1, 3]]])
    sinks_dup = np.array([[[0, 9, 33, 44]]])     # 9 in block 1, 33 in the current block
    sinks_min = np.array([[[0, 44, -1, -1]]])
    O1 = orc.sparse_attention(Q, [3], K, V, sinks_dup, blocks, bs, P, g0, g1, scale)
    O2 = orc.sparse_attention(Q, [3], K, V, sinks_min, blocks, bs, P, g0, g1, scale)
    np.testing.assert_allclose(O1, O2, rtol=1e-13, atol=1e-14)
    # library reference: SDPA with a boolean key mask over I_p
    keep = np.zeros(L, bool)
    keep[[0, 44]] = True
    keep[8:16] = True
    keep[24:32] = True
    keep[32:40] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q[:, :, :3]), torch.from_numpy(np.repeat(K, 2, axis=1)),
        torch.from_numpy(np.repeat(V, 2, axis=1)), attn_mask=torch.from_numpy(np.broadcast_to(keep, (3, L)).copy()), scale=scale).numpy()
    np.testing.assert_allclose(O1[:, :, :3], ref, rtol=1e-11, atol=1e-12)
    assert np.all(O1[:, :, 3:] == 0.0)


def test_sparse_partial_last_block():
    """P % bs != 0: the last block covers only the valid prompt rows [16, 20), not [16, 24)."""
    Ip = orc.sparse_key_set(np.array([-1]), np.array([2]), 8, 20, 28, 32)
    assert Ip.tolist() == [16, 17, 18, 19, 28, 29, 30, 31]


# ------------------------------------------------------------------ approximate KV-cache refresh
def test_refresh_rows_golden_and_invariants():
    """Summary page, "近似KV缓存": tokens of U(t) take the recomputed state, all others keep
    the cache. Hand-worked case, then the gather/refresh round trip on random data."""
    X = np.arange(2 * 1 * 4 * 2, dtype=np.float64).reshape(2, 1, 4, 2)
    Xn = -np.ones((2, 1, 3, 2))
    Xn[0, 0, 1] = [-5.0, -6.0]
    out = orc.refresh_rows(X, [np.array([1, 3]), np.array([], dtype=np.int64)], Xn)
    want = X.copy()
    want[0, 0, 1] = [-1.0, -1.0]
    want[0, 0, 3] = [-5.0, -6.0]
    assert np.array_equal(out, want)
    assert np.array_equal(X, np.arange(16, dtype=np.float64).reshape(2, 1, 4, 2))   # input untouched
    rng = np.random.default_rng(3)
    Xr = rng.standard_normal((3, 2, 50, 8))
    rows = [np.sort(rng.choice(50, size=n, replace=False)) for n in (0, 7, 50)]
    Xnew = rng.standard_normal((3, 2, 50, 8))
    out = orc.refresh_rows(Xr, rows, Xnew)
    back = orc.gather_rows(out, rows, 50)
    for b, r in enumerate(rows):
        assert np.array_equal(back[b, :, :r.size], Xnew[b, :, :r.size])
        keep = np.setdiff1d(np.arange(50), r)
        assert np.array_equal(out[b, :, keep], Xr[b, :, keep])


# ------------------------------------------------------------------ step variants
def test_mean_query_sinks_against_explicit_softmax():
    """Variant sink importance: the top-S columns of the mean active query's attention row,
    computed here by an explicit fp64 softmax and a full sort, with a planted key."""
    rng = np.random.default_rng(21)
    B, Hq, Hkv, A, L, d, S = 2, 4, 2, 5, 200, 16, 6
    Q = rng.standard_normal((B, Hq, 8, d))
    K = rng.standard_normal((B, Hkv, L, d))
    n_active = [5, 3]
    qbar = np.zeros((B, Hkv, d))
    for b in range(B):
        for h in range(Hkv):
            rows = Q[b, h * 2:(h + 1) * 2, :n_active[b]].reshape(-1, d)
            qbar[b, h] = rows.mean(axis=0)
    K[1, 0, 77] = 5.0 * qbar[1, 0] / np.linalg.norm(qbar[1, 0])      # planted: aligned with qbar
    sinks, _ = orc.sink_identify_mean_query(Q, n_active, K, S)
    for b in range(B):
        for h in range(Hkv):
            s = K[b, h] @ qbar[b, h] / np.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            order = sorted(range(L), key=lambda j: (-p[j], j))[:S]
            assert sinks[b, h].tolist() == sorted(order)
    assert 77 in sinks[1, 0].tolist()


def test_variant_schedules_and_ratio_forms():
    from diffusion_long_context_b200 import configs as cf
    dream = cf.DREAM_16K.replace(dense_tail=4)
    assert dream.dense_layers == [0, 1, 2, 24, 25, 26, 27]
    assert dream.sparse_layers == list(range(3, 24))
    assert cf.FULL_32K.dense_layers == [0, 1, 2] and cf.FULL_32K.sparse_layers == list(range(3, 32))
    r = cf.ratio_forms(cf.FULL_32K)               # alpha = 0.5 of 508 blocks, 1% of 32768 tokens
    assert (r.C, r.S) == (254, 328)
    assert cf.ratio_forms(cf.TINY).C == 7 and cf.ratio_forms(cf.TINY).S == 6


def test_step_layer_subset_equals_the_full_step():
    """sparse_step(layers_eval=...) computes the chosen layers exactly as the full step does:
    the layers' inputs come from layer_fn, so only the sinks carry from layer to layer."""
    from diffusion_long_context_b200 import configs as cf
    from diffusion_long_context_b200 import inputs as inp
    cfg = cf.scaled(cf.LLADA_8K, 768, n_layers=5, Hq=4, Hkv=2, l_dense=1, C=3, S=4, bs=32)
    st = inp.step_state(cfg)
    lay = [tuple(inp.to_f64(t) for t in inp.make_layer(cfg, l, "cpu", st.sink_pos)) for l in range(cfg.n_layers)]
    args = (cfg.n_layers, cfg.l_dense, st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, cfg.rho, cfg.w, cfg.P, cfg.bs,
            cfg.C, cfg.S, cfg.acap, 1 / math.sqrt(cfg.d))
    full = orc.sparse_step(lambda l: lay[l], *args)
    part = orc.sparse_step(lambda l: lay[l], *args, layers_eval=[3])
    assert np.array_equal(full["sinks"], part["sinks"])
    assert sorted(part["blocks"]) == [3] and sorted(part["O"]) == [1, 3]
    assert np.array_equal(full["blocks"][3], part["blocks"][3]) and np.array_equal(full["R"][3], part["R"][3])
    assert np.array_equal(full["O"][3], part["O"][3])
