"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded inputs.

Index sets must match exactly; attention outputs within max-abs 2e-2 / mean-abs 2e-3;
block means within 1e-3 relative. Sizes span several 128-key tiles with ragged tails,
both head dims, MHA and GQA, and the degenerate cases of the method.
"""
import math

import numpy as np
import pytest
import torch

from diffusion_long_context_b200 import configs, inputs
from oracle import focus_oracle as orc
from parity_utils import (KBAR_REL, assert_attention_close, assert_index_sets, assert_tail_is_minus_one,
                          idx_rows, topk_matches)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def F():
    from diffusion_long_context_b200 import build
    build.build()
    from diffusion_long_context_b200 import focus
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return focus


def _i32(shape, fill=-7):
    return torch.full(shape, fill, dtype=torch.int32, device=DEV)


# ------------------------------------------------------------------ select_queries
def _run_select(F, conf, mask, g0, g1, n_t, rho, w, kcap, acap):
    B = mask.shape[0]
    conf_d = torch.from_numpy(conf).to(DEV)
    mask_d = torch.from_numpy(mask).to(DEV)
    i_focus, n_focus = _i32((B, kcap)), _i32((B,))
    i_active, n_active = _i32((B, acap)), _i32((B,))
    F.focus_select_queries(conf_d, mask_d, g0, g1, n_t, rho, w, i_focus, n_focus, i_active, n_active)
    torch.cuda.synchronize()
    return i_focus, n_focus, i_active, n_active


def test_select_queries_tiny_config(F):
    cfg = configs.TINY
    st = inputs.step_state(cfg)
    rho = float(np.float32(cfg.rho))
    i_focus, n_focus, i_active, n_active = _run_select(F, st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, rho,
                                                       cfg.w, cfg.G, cfg.G)
    ef, ea = orc.select_queries(st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, rho, cfg.w)
    assert idx_rows(i_focus) == [ef[0].tolist()]
    assert idx_rows(i_active) == [ea[0].tolist()]
    assert n_focus.tolist() == [len(ef[0])] and n_active.tolist() == [len(ea[0])]
    assert len(ef[0]) == min(cfg.k, cfg.n_masked)
    assert_tail_is_minus_one(i_active, n_active.tolist())


@pytest.mark.parametrize("seed", range(6))
def test_select_queries_random_batches(F, seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(6):
        B = int(rng.integers(1, 65))
        G = int(rng.choice([1, 3, 8, 31, 32, 33, 64, 200, 1024]))
        g0 = int(rng.integers(0, 50))
        g1 = g0 + G
        L = g1 + int(rng.integers(0, 40))
        mask = np.zeros((B, L), np.uint8)
        mask[:, g0:g1] = (rng.random((B, G)) < rng.uniform(0.1, 1.0)).astype(np.uint8)
        mask[:, g1:] = 1
        vals = np.float32([0.0, -0.0, 0.125, 0.5, 0.5, 0.75, 1.0])
        conf = np.where(rng.random((B, G)) < 0.5, rng.choice(vals, (B, G)),
                        rng.random((B, G)).astype(np.float32)).astype(np.float32)
        n_t = int(rng.integers(0, 9))
        rho = float(np.float32(rng.choice([1.0, 2.0, 2.5, 4.0, 8.0])))
        w = int(rng.integers(1, 12))
        k = min(int(math.floor(rho * n_t)), G)
        acap = max(1, min(G, k * w))
        i_focus, n_focus, i_active, n_active = _run_select(F, conf, mask, g0, g1, n_t, rho, w, max(1, k), acap)
        ef, ea = orc.select_queries(conf, mask, g0, g1, n_t, rho, w)
        assert idx_rows(i_focus) == [e.tolist() for e in ef]
        assert idx_rows(i_active) == [e.tolist() for e in ea]
        assert n_focus.tolist() == [len(e) for e in ef]
        assert n_active.tolist() == [len(e) for e in ea]


def test_select_queries_no_masked_positions(F):
    mask = np.zeros((2, 64), np.uint8)
    conf = np.ones((2, 16), np.float32)
    i_focus, n_focus, i_active, n_active = _run_select(F, conf, mask, 40, 56, 4, 4.0, 8, 16, 16)
    assert n_focus.tolist() == [0, 0] and n_active.tolist() == [0, 0]
    assert (i_focus == -1).all() and (i_active == -1).all()


# ------------------------------------------------------------------ gather_rows
def test_gather_rows(F):
    X = inputs.random_bf16((3, 2, 5, 300, 128), seed=5, device=DEV)
    rows = torch.tensor([[7, 8, 299, 0, -1, -1], [1, 2, 3, 4, 5, 6]], dtype=torch.int32, device=DEV)
    n = torch.tensor([4, 6], dtype=torch.int32, device=DEV)
    out = torch.full((3, 2, 5, 6, 128), 9.0, dtype=torch.bfloat16, device=DEV)
    F.focus_gather_rows(X, rows, n, out)
    torch.cuda.synchronize()
    for b, cnt in enumerate([4, 6]):
        r = rows[b, :cnt].long()
        assert torch.equal(out[:, b, :, :cnt], X[:, b][:, :, r])
        assert (out[:, b, :, cnt:] == 0).all()
    assert F.device_error() == 0


# ------------------------------------------------------------------ KV-cache refresh
def test_scatter_rows_matches_oracle_refresh(F):
    """Approximate-KV-cache refresh over a stack of layers: bit-exact against the oracle."""
    X = inputs.random_bf16((3, 2, 5, 300, 128), seed=8, device=DEV)
    Xn = inputs.random_bf16((3, 2, 5, 6, 128), seed=9, device=DEV)
    rows = torch.tensor([[0, 7, 8, 299, -1, -1], [1, 2, 3, 4, 5, 6]], dtype=torch.int32, device=DEV)
    n = torch.tensor([4, 6], dtype=torch.int32, device=DEV)
    ref_in = X.cpu()
    F.focus_scatter_rows(X, rows, n, Xn)
    torch.cuda.synchronize()
    rl = [rows[0, :4].cpu().numpy(), rows[1, :6].cpu().numpy()]
    for m in range(3):
        want = orc.refresh_rows(ref_in[m].float().numpy(), rl, Xn[m].cpu().float().numpy())
        assert np.array_equal(X[m].cpu().float().numpy(), want)
    assert F.device_error() == 0


def test_scatter_rows_empty_and_out_of_range(F):
    X = inputs.random_bf16((2, 2, 40, 64), seed=10, device=DEV)
    before = X.clone()
    Xn = inputs.random_bf16((2, 2, 4, 64), seed=11, device=DEV)
    rows = torch.tensor([[3, 5, -1, -1], [40, 1, -1, -1]], dtype=torch.int32, device=DEV)
    F.focus_scatter_rows(X, rows, torch.tensor([0, 0], dtype=torch.int32, device=DEV), Xn)
    torch.cuda.synchronize()
    assert torch.equal(X, before)                                   # empty refresh sets
    F.focus_scatter_rows(X, rows, torch.tensor([2, 2], dtype=torch.int32, device=DEV), Xn)
    torch.cuda.synchronize()
    assert F.device_error() != 0                                    # row 40 is outside [0, 40)
    assert torch.equal(X[1, :, 1], Xn[1, :, 1]) and torch.equal(X[0, :, 3], Xn[0, :, 0])
    assert torch.equal(X[1, :, 2:], before[1, :, 2:]) and torch.equal(X[0, :, :3], before[0, :, :3])


# ------------------------------------------------------------------ block means
@pytest.mark.parametrize("d,P,bs,L", [(64, 448, 32, 512), (128, 1000, 64, 1100), (128, 333, 128, 400),
                                      (128, 64, 1, 64), (64, 250, 24, 260)])
def test_block_means(F, d, P, bs, L):
    K = inputs.random_bf16((2, 3, L, d), seed=P + bs, device=DEV)
    nb = -(-P // bs)
    kbar = torch.empty((2, 3, nb, d), dtype=torch.float32, device=DEV)
    F.focus_block_means(K, P, bs, kbar)
    torch.cuda.synchronize()
    ref = orc.block_means(inputs.to_f64(K), P, bs)
    got = kbar.cpu().double().numpy()
    assert np.all(np.abs(got - ref) <= KBAR_REL * np.abs(ref) + 1e-6)


# ------------------------------------------------------------------ block select
@pytest.mark.parametrize("Hq,Hkv,d,nb,C,acap", [(4, 4, 64, 14, 4, 32), (32, 32, 128, 508, 64, 32),
                                               (28, 4, 128, 252, 32, 32), (8, 2, 128, 1016, 128, 16),
                                               (4, 4, 128, 7, 16, 32), (2, 1, 64, 3000, 257, 8)])
def test_block_select(F, Hq, Hkv, d, nb, C, acap):
    B = 2
    Q = inputs.random_bf16((B, Hq, acap, d), seed=nb, device=DEV)
    kbar = inputs.random_f32((B, Hkv, nb, d), seed=nb + 1, device=DEV, lo=-1.0, hi=1.0)
    n_active = torch.tensor([acap, max(1, acap // 3)], dtype=torch.int32, device=DEV)
    blocks = _i32((B, Hkv, C))
    scores = torch.empty((B, Hkv, nb), dtype=torch.float32, device=DEV)
    F.focus_block_select(Q, n_active, kbar, C, blocks, scores)
    torch.cuda.synchronize()
    ref_blocks, R = orc.block_select(inputs.to_f64(Q), n_active.tolist(), inputs.to_f64(kbar), C)
    np.testing.assert_allclose(scores.cpu().double().numpy(), R, rtol=1e-4, atol=1e-5)
    got = blocks.cpu().numpy()
    exact = 0
    for b in range(B):
        for h in range(Hkv):
            g = [int(x) for x in got[b, h] if x >= 0]
            exact += topk_matches(g, R[b, h], min(C, nb))
            assert np.all(got[b, h, min(C, nb):] == -1)
    assert exact == B * Hkv, f"{B * Hkv - exact} near-tie top-C sets (checked valid)"


def test_block_select_empty_active_set(F):
    Q = inputs.random_bf16((1, 2, 8, 64), seed=1, device=DEV)
    kbar = inputs.random_f32((1, 2, 10, 64), seed=2, device=DEV)
    blocks = _i32((1, 2, 3))
    F.focus_block_select(Q, torch.zeros(1, dtype=torch.int32, device=DEV), kbar, 3, blocks)
    torch.cuda.synchronize()
    assert blocks.tolist() == [[[0, 1, 2], [0, 1, 2]]]      # R = 0 everywhere: lowest indices


# ------------------------------------------------------------------ sink identify
@pytest.mark.parametrize("L,S,coarse", [(512, 4, False), (32768, 32, False), (1000, 16, True), (7, 16, True),
                                        (65536, 300, False)])
def test_sink_identify(F, L, S, coarse):
    B, Hkv = 2, 3
    if coarse:
        vals = torch.tensor([0.0, -0.0, 0.25, 0.5, 1.0], device=DEV)
        gen = torch.Generator(device=DEV)
        gen.manual_seed(L)
        colsum = vals[torch.randint(0, 5, (B, Hkv, L), generator=gen, device=DEV)].contiguous()
    else:
        colsum = inputs.random_f32((B, Hkv, L), seed=L, device=DEV)
    sinks = _i32((B, Hkv, S))
    F.focus_sink_identify(colsum, S, sinks)
    torch.cuda.synchronize()
    ref = orc.sink_identify(inputs.to_f64(colsum), S)
    assert np.array_equal(sinks.cpu().numpy(), ref)


# ------------------------------------------------------------------ dense attention
DENSE_CASES = [
    # B, Hq, Hkv, L, d, qcap, n_q
    (1, 4, 4, 512, 64, 32, [13]),
    (2, 4, 4, 1000, 128, 32, [32, 5]),
    (1, 28, 4, 1500, 128, 32, [29]),
    (2, 8, 2, 777, 64, 24, [24, 1]),
    (1, 2, 1, 129, 128, 16, [16]),
    (1, 8, 4, 700, 128, 32, [27]),          # 2 query heads per KV head x 32: 64 query columns
    (2, 32, 32, 600, 128, 32, [32, 19]),    # 64 heads: clusters of 2
    (1, 6, 2, 900, 128, 32, [30]),          # 96 rows per KV head: row slices of 64 + 32
    (2, 28, 4, 1100, 128, 24, [24, 7]),     # GQA 7:1, 168 rows per KV head: three row slices
    (1, 16, 1, 700, 128, 32, [32]),         # 512 rows per KV head: the 128-row tile kernel
]


@pytest.mark.parametrize("B,Hq,Hkv,L,d,qcap,n_q", DENSE_CASES)
def test_dense_attention_active_with_colsum(F, B, Hq, Hkv, L, d, qcap, n_q):
    Q = inputs.random_bf16((B, Hq, qcap, d), seed=L, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=L + 1, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=L + 2, device=DEV)
    nq = torch.tensor(n_q, dtype=torch.int32, device=DEV)
    O = torch.full((B, Hq, qcap, d), 7.0, dtype=torch.bfloat16, device=DEV)
    # column sums are served for up to 256 query rows per KV group
    want_colsum = (Hq // Hkv) * qcap <= 256
    colsum = torch.empty((B, Hkv, L), dtype=torch.float32, device=DEV) if want_colsum else None
    scale = 1.0 / math.sqrt(d)
    F.focus_dense_attention(Q, nq, K, V, O, scale=scale, colsum=colsum)
    torch.cuda.synchronize()
    refO, refC, _ = orc.dense_attention(inputs.to_f64(Q), n_q, inputs.to_f64(K), inputs.to_f64(V),
                                        float(np.float32(scale)), want_colsum=True)
    assert_attention_close(O, refO, rows_valid=n_q, what="dense attention")
    if want_colsum:
        np.testing.assert_allclose(colsum.cpu().double().numpy(), refC, rtol=2e-3, atol=1e-6)
    assert F.device_error() == 0


@pytest.mark.parametrize("B,Hq,Hkv,L,d", [(1, 4, 4, 640, 128), (1, 4, 2, 300, 64), (2, 2, 2, 257, 128)])
def test_dense_attention_full_refresh(F, B, Hq, Hkv, L, d):
    Q = inputs.random_bf16((B, Hq, L, d), seed=3 * L, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=3 * L + 1, device=DEV, scale=2.0)
    V = inputs.random_bf16((B, Hkv, L, d), seed=3 * L + 2, device=DEV)
    O = torch.empty((B, Hq, L, d), dtype=torch.bfloat16, device=DEV)
    F.focus_dense_attention(Q, None, K, V, O)
    torch.cuda.synchronize()
    refO, _, _ = orc.dense_attention(inputs.to_f64(Q), None, inputs.to_f64(K), inputs.to_f64(V),
                                     float(np.float32(1.0 / math.sqrt(d))))
    assert_attention_close(O, refO, what="full refresh")


SINK_LAYER_CASES = [
    # B, Hq, Hkv, L, d, qcap, n_q, S
    (1, 32, 32, 4000, 128, 32, [30], 32),     # one launch: attention, column sums, cluster top-S
    (2, 4, 4, 2500, 128, 32, [32, 7], 16),    # clusters of 8 CTAs
    (1, 8, 4, 1200, 128, 32, [27], 8),        # 64 rows per KV head: the 64-column kernel
    (1, 2, 1, 129, 128, 16, [16], 4),         # one partial key tile
    (1, 4, 4, 300, 128, 32, [31], 120),       # S close to L: a CTA holds fewer than S columns
    (1, 4, 4, 3000, 128, 32, [30], 300),      # S > 128: three group maxima per key lane
    (1, 2, 2, 5000, 128, 32, [32], 700),      # S beyond the cluster's candidate room: top-S kernel
    (1, 4, 4, 700, 64, 32, [25], 8),          # d = 64: tile kernel, column-sum kernel, top-S kernel
    (1, 28, 4, 900, 128, 32, [29], 16),       # 224 rows per KV head: tile kernel + column-sum kernel
]


@pytest.mark.parametrize("B,Hq,Hkv,L,d,qcap,n_q,S", SINK_LAYER_CASES)
def test_sink_layer_one_call(F, B, Hq, Hkv, L, d, qcap, n_q, S):
    """focus_dense_attention_sinks against the oracle: output rows, column sums, and the
    top-S sets (bit-exact up to near-ties at the boundary)."""
    Q = inputs.random_bf16((B, Hq, qcap, d), seed=5 * L + S, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=5 * L + S + 1, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=5 * L + S + 2, device=DEV)
    nq = torch.tensor(n_q, dtype=torch.int32, device=DEV)
    O = torch.full((B, Hq, qcap, d), 3.0, dtype=torch.bfloat16, device=DEV)
    colsum = torch.full((B, Hkv, L), -1.0, dtype=torch.float32, device=DEV)
    sinks = torch.full((B, Hkv, S), -7, dtype=torch.int32, device=DEV)
    scale = 1.0 / math.sqrt(d)
    F.focus_dense_attention_sinks(Q, nq, K, V, O, colsum, sinks, scale=scale)
    torch.cuda.synchronize()
    assert F.device_error() == 0
    refO, refC, _ = orc.dense_attention(inputs.to_f64(Q), n_q, inputs.to_f64(K), inputs.to_f64(V),
                                        float(np.float32(scale)), want_colsum=True)
    assert_attention_close(O, refO, rows_valid=n_q, what="sink layer attention")
    np.testing.assert_allclose(colsum.cpu().double().numpy(), refC, rtol=2e-3, atol=1e-6)
    ties = assert_index_sets(sinks, refC, min(S, L), "sink layer sinks")
    assert ties == 0, f"{ties} near-tie sink sets"


@pytest.mark.parametrize("L,S", [(12288, 32), (3000, 200)])
def test_sink_layer_equal_column_sums(F, L, S):
    """Degenerate case: K = 0 makes every score 0, so every column sum is n_q / L exactly
    and the top-S is decided by the tie rule alone (the lowest columns). At 12288 columns
    more columns tie than a CTA's candidate list holds, so each CTA takes the general radix
    selection; at 3000 every column of a CTA is a candidate."""
    B, Hq, Hkv, d, qcap = 1, 4, 4, 128, 32
    Q = inputs.random_bf16((B, Hq, qcap, d), seed=77, device=DEV)
    K = torch.zeros((B, Hkv, L, d), dtype=torch.bfloat16, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=78, device=DEV)
    nq = torch.tensor([29], dtype=torch.int32, device=DEV)
    O = torch.empty((B, Hq, qcap, d), dtype=torch.bfloat16, device=DEV)
    colsum = torch.empty((B, Hkv, L), dtype=torch.float32, device=DEV)
    sinks = torch.full((B, Hkv, S), -7, dtype=torch.int32, device=DEV)
    F.focus_dense_attention_sinks(Q, nq, K, V, O, colsum, sinks)
    torch.cuda.synchronize()
    assert F.device_error() == 0
    c = colsum.cpu()
    assert torch.all(c == c[0, 0, 0]), "column sums of equal scores differ"
    np.testing.assert_allclose(float(c[0, 0, 0]) * L, 29.0, rtol=1e-4)
    expect = torch.arange(S, dtype=torch.int32).expand(B, Hkv, S)
    assert torch.equal(sinks.cpu(), expect)


def test_sink_layer_cluster_top_s_matches_the_top_s_kernel(F):
    """On the 32K step's shape (reduced length) the one-call sink layer's in-cluster top-S
    picks the sets focus_sink_identify picks from the column sums of focus_dense_attention
    (the same kernel; its CTAs claim key tiles dynamically, so the order of the fp32 partial
    sums, and with it the last bits of O and of the column sums, varies between launches)."""
    B, Hq, Hkv, L, d, qcap, S = 1, 32, 32, 12288, 128, 32, 32
    Q = inputs.random_bf16((B, Hq, qcap, d), seed=901, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=902, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=903, device=DEV)
    nq = torch.tensor([30], dtype=torch.int32, device=DEV)
    O1, O2 = (torch.empty((B, Hq, qcap, d), dtype=torch.bfloat16, device=DEV) for _ in range(2))
    c1, c2 = (torch.empty((B, Hkv, L), dtype=torch.float32, device=DEV) for _ in range(2))
    s1, s2 = (torch.empty((B, Hkv, S), dtype=torch.int32, device=DEV) for _ in range(2))
    F.focus_dense_attention_sinks(Q, nq, K, V, O1, c1, s1)
    F.focus_dense_attention(Q, nq, K, V, O2, colsum=c2)
    F.focus_sink_identify(c2, S, s2)
    torch.cuda.synchronize()
    assert F.device_error() == 0
    torch.testing.assert_close(O1.float(), O2.float(), rtol=0, atol=2e-3)
    torch.testing.assert_close(c1, c2, rtol=1e-5, atol=0)
    assert assert_index_sets(s1, c2.double().cpu().numpy(), S, "one-call sinks vs the top-S kernel") == 0
    assert assert_index_sets(s2, c1.double().cpu().numpy(), S, "top-S kernel vs one-call column sums") == 0


MANY_ROW_CASES = [
    # B, Hq, Hkv, L, qcap, n_q (None = all rows): enough 256-row blocks for the many-row kernel
    (1, 16, 16, 2400, 2400, None),          # ragged key tile and ragged row block
    (2, 8, 4, 2700, 2700, None),            # GQA 2:1, two sequences
    (2, 16, 16, 3000, 2048, [2048, 1000]),  # valid-row counts: rows past n_q written as zero
]


@pytest.mark.parametrize("B,Hq,Hkv,L,qcap,n_q", MANY_ROW_CASES)
def test_dense_attention_many_rows(F, B, Hq, Hkv, L, qcap, n_q):
    """The many-row dense kernel (P kept in tensor memory, two query tiles per CTA) against
    the oracle on sampled rows of every head."""
    d = 128
    Q = inputs.random_bf16((B, Hq, qcap, d), seed=7 * L + qcap, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=7 * L + 1, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=7 * L + 2, device=DEV)
    O = torch.full((B, Hq, qcap, d), 5.0, dtype=torch.bfloat16, device=DEV)
    nq = None if n_q is None else torch.tensor(n_q, dtype=torch.int32, device=DEV)
    F.focus_dense_attention(Q, nq, K, V, O)
    torch.cuda.synchronize()
    assert F.device_error() == 0
    rng = np.random.default_rng(L)
    rows = np.sort(np.unique(np.concatenate([rng.choice(qcap, 40, replace=False), [0, qcap - 1]])))
    ridx = torch.as_tensor(rows, device=DEV)
    valid = [qcap] * B if n_q is None else n_q
    scale = float(np.float32(1 / math.sqrt(d)))
    g = Hq // Hkv
    for hq in range(Hq):
        h = hq // g
        q = inputs.to_f64(Q[:, hq:hq + 1, ridx])
        ref, _, _ = orc.dense_attention(q, None, inputs.to_f64(K[:, h:h + 1]), inputs.to_f64(V[:, h:h + 1]), scale)
        for b in range(B):
            keep = rows < valid[b]
            ref[b, :, ~keep] = 0.0                 # rows past the valid count are written as zero
        assert_attention_close(O[:, hq:hq + 1, ridx], ref, what=f"many-row dense head {hq}")


FULL_REFRESH_CASES = [
    # B, Hq, Hkv, L, d, P, bs: block entry (attention of every query + block means)
    (1, 16, 16, 2400, 128, 2336, 64),     # one launch: the means summed from the K stream
    (2, 8, 4, 2700, 128, 2605, 32),       # GQA, a short last block (2605 = 81 * 32 + 13)
    (1, 16, 16, 2400, 128, 2300, 128),    # bs = 128: one block per key tile
    (1, 16, 16, 2400, 128, 2304, 96),     # bs not dividing 128: attention and block means as two calls
    (1, 4, 4, 600, 64, 500, 64),          # d = 64: two calls
]


@pytest.mark.parametrize("B,Hq,Hkv,L,d,P,bs", FULL_REFRESH_CASES)
def test_full_refresh_with_block_means(F, B, Hq, Hkv, L, d, P, bs):
    """focus_full_refresh: every query over all keys (sampled rows of every head) and the
    prompt's block means, against the oracle."""
    Q = inputs.random_bf16((B, Hq, L, d), seed=11 * L + bs, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=11 * L + bs + 1, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=11 * L + bs + 2, device=DEV)
    nb = -(-P // bs)
    O = torch.full((B, Hq, L, d), 5.0, dtype=torch.bfloat16, device=DEV)
    kbar = torch.full((B, Hkv, nb, d), -9.0, dtype=torch.float32, device=DEV)
    F.focus_full_refresh(Q, K, V, O, P, bs, kbar)
    torch.cuda.synchronize()
    assert F.device_error() == 0
    K64 = inputs.to_f64(K)
    ref_kbar = orc.block_means(K64, P, bs)
    got = kbar.cpu().double().numpy()
    assert np.all(np.abs(got - ref_kbar) <= KBAR_REL * np.abs(ref_kbar) + 1e-6), "block means off"
    rng = np.random.default_rng(L + bs)
    rows = np.sort(np.unique(np.concatenate([rng.choice(L, 24, replace=False), [0, L - 1]])))
    ridx = torch.as_tensor(rows, device=DEV)
    scale = float(np.float32(1 / math.sqrt(d)))
    g = Hq // Hkv
    for hq in range(Hq):
        h = hq // g
        q = inputs.to_f64(Q[:, hq:hq + 1, ridx])
        ref, _, _ = orc.dense_attention(q, None, K64[:, h:h + 1], inputs.to_f64(V[:, h:h + 1]), scale)
        assert_attention_close(O[:, hq:hq + 1, ridx], ref, what=f"full refresh head {hq}")


def test_dense_attention_planted_sinks_recovered(F):
    cfg = configs.TINY
    st = inputs.step_state(cfg)
    Qf, K, V = inputs.make_layer(cfg, 0, DEV, st.sink_pos)
    ef, ea = orc.select_queries(st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, cfg.rho, cfg.w)
    rows = torch.full((1, cfg.acap), -1, dtype=torch.int32, device=DEV)
    rows[0, :len(ea[0])] = torch.tensor(ea[0], dtype=torch.int32)
    n = torch.tensor([len(ea[0])], dtype=torch.int32, device=DEV)
    Qa = torch.empty((1, cfg.Hq, cfg.acap, cfg.d), dtype=torch.bfloat16, device=DEV)
    F.focus_gather_rows(Qf, rows, n, Qa)
    O = torch.empty_like(Qa)
    colsum = torch.empty((1, cfg.Hkv, cfg.L), dtype=torch.float32, device=DEV)
    F.focus_dense_attention(Qa, n, K, V, O, colsum=colsum)
    sinks = _i32((1, cfg.Hkv, cfg.S))
    F.focus_sink_identify(colsum, cfg.S, sinks)
    torch.cuda.synchronize()
    _, refC, _ = orc.dense_attention(orc.gather_rows(inputs.to_f64(Qf), ea, cfg.acap), [len(ea[0])],
                                     inputs.to_f64(K), inputs.to_f64(V), 1 / math.sqrt(cfg.d), True)
    for h in range(cfg.Hkv):
        got = [int(x) for x in sinks[0, h].tolist() if x >= 0]
        assert set(st.sink_pos.tolist()) <= set(got)
        topk_matches(got, refC[0, h], cfg.S)


# ------------------------------------------------------------------ sparse attention
SPARSE_CASES = [
    # name, B, Hq, Hkv, d, P, G, L, bs, C, S, acap, n_active
    ("tiny", 1, 4, 4, 64, 448, 32, 512, 32, 4, 4, 32, [21]),
    ("mha_bs64", 2, 4, 4, 128, 1984, 32, 2048, 64, 8, 8, 32, [32, 17]),
    ("gqa", 1, 28, 4, 128, 2048, 32, 2112, 64, 6, 16, 32, [30]),
    ("bs128_allblocks", 1, 2, 2, 128, 1024, 32, 1088, 128, 16, 4, 32, [9]),
    ("bs32_many", 1, 2, 1, 128, 4096, 32, 4160, 32, 64, 32, 32, [32]),
    ("ragged_bs24", 1, 4, 2, 64, 250, 20, 300, 24, 5, 7, 20, [20]),
    ("no_sinks", 1, 2, 2, 128, 512, 32, 544, 64, 3, 0, 32, [11]),
    ("gqa2_nq64", 1, 8, 4, 128, 1024, 32, 1100, 64, 5, 9, 32, [32]),
    ("mha64_heads", 2, 32, 32, 128, 640, 32, 700, 32, 4, 6, 32, [25, 32]),
    ("bs16_mha", 1, 4, 4, 128, 512, 32, 560, 16, 12, 5, 32, [30]),
    ("gqa3_96rows", 2, 6, 2, 128, 1024, 32, 1100, 64, 7, 5, 32, [32, 12]),
    ("gqa16_tile", 1, 16, 1, 128, 1024, 32, 1088, 64, 6, 4, 32, [29]),
]


def _sparse_indices(rng, B, Hkv, P, g0, g1, L, bs, C, S, dup=True):
    nb = -(-P // bs)
    blocks = np.full((B, Hkv, C), -1, np.int32)
    sinks = np.full((B, Hkv, max(S, 1)), -1, np.int32)
    for b in range(B):
        for h in range(Hkv):
            kb = np.sort(rng.choice(nb, size=min(C, nb), replace=False))
            blocks[b, h, :kb.size] = kb
            if S:
                pool = list(range(L))
                s = set(rng.choice(pool, size=S, replace=False).tolist())
                if dup and kb.size:
                    s.pop()
                    s.add(int(kb[0]) * bs)        # a sink inside a kept block
                if dup and S > 2:
                    s.pop()
                    s.add(g0 + 1)                 # a sink inside the current block
                sv = np.sort(np.array(sorted(s)))[:S]
                sinks[b, h, :sv.size] = sv
    return blocks, (sinks if S else None)


@pytest.mark.parametrize("case", SPARSE_CASES, ids=[c[0] for c in SPARSE_CASES])
def test_sparse_attention(F, case):
    name, B, Hq, Hkv, d, P, G, L, bs, C, S, acap, n_act = case
    g0, g1 = P, P + G
    rng = np.random.default_rng(len(name) * 1000 + L)
    blocks, sinks = _sparse_indices(rng, B, Hkv, P, g0, g1, L, bs, C, S)
    Q = inputs.random_bf16((B, Hq, acap, d), seed=L + 11, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=L + 12, device=DEV, scale=1.5)
    V = inputs.random_bf16((B, Hkv, L, d), seed=L + 13, device=DEV)
    O = torch.full((B, Hq, acap, d), 3.0, dtype=torch.bfloat16, device=DEV)
    n_active = torch.tensor(n_act, dtype=torch.int32, device=DEV)
    blocks_d = torch.from_numpy(blocks).to(DEV)
    sinks_d = None if sinks is None else torch.from_numpy(sinks).to(DEV)
    scale = 1.0 / math.sqrt(d)
    F.focus_sparse_attention(Q, n_active, K, V, sinks_d, blocks_d, bs, P, g0, g1, O, scale=scale)
    torch.cuda.synchronize()
    sinks_o = np.full((B, Hkv, 1), -1) if sinks is None else sinks
    ref = orc.sparse_attention(inputs.to_f64(Q), n_act, inputs.to_f64(K), inputs.to_f64(V), sinks_o, blocks, bs,
                               P, g0, g1, float(np.float32(scale)))
    assert_attention_close(O, ref, rows_valid=n_act, what=f"sparse attention ({name})")
    assert F.device_error() == 0


def test_sparse_equals_dense_when_everything_is_kept(F):
    B, Hq, Hkv, d, bs, G = 1, 4, 2, 128, 64, 32
    P = 1024
    g0, g1 = P, P + G
    L = g1 + 64
    Q = inputs.random_bf16((B, Hq, 32, d), seed=1, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=2, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=3, device=DEV)
    n = torch.tensor([32], dtype=torch.int32, device=DEV)
    blocks = torch.arange(P // bs, dtype=torch.int32, device=DEV).repeat(B, Hkv, 1).contiguous()
    sinks = torch.arange(g1, L, dtype=torch.int32, device=DEV).repeat(B, Hkv, 1).contiguous()
    Os = torch.empty((B, Hq, 32, d), dtype=torch.bfloat16, device=DEV)
    Od = torch.empty_like(Os)
    F.focus_sparse_attention(Q, n, K, V, sinks, blocks, bs, P, g0, g1, Os)
    F.focus_dense_attention(Q, n, K, V, Od)
    torch.cuda.synchronize()
    assert (Os.float() - Od.float()).abs().max().item() <= 1e-2


# ------------------------------------------------------------------ composed step
def test_composed_step_small(F):
    """Select -> dense layers (+ sinks) -> block means/select -> sparse layers, vs the oracle."""
    cfg = configs.scaled(configs.LLADA_8K, 1024, n_layers=4, Hq=4, Hkv=4, l_dense=1, C=4, S=8)
    st = inputs.step_state(cfg)
    layers = [inputs.make_layer(cfg, l, DEV, st.sink_pos) for l in range(cfg.n_layers)]
    rho = float(np.float32(cfg.rho))
    conf = torch.from_numpy(st.conf_prev).to(DEV)
    mask = torch.from_numpy(st.mask).to(DEV)
    i_focus, n_focus = _i32((cfg.B, cfg.G)), _i32((cfg.B,))
    i_active, n_active = _i32((cfg.B, cfg.acap)), _i32((cfg.B,))
    F.focus_select_queries(conf, mask, cfg.g0, cfg.g1, cfg.n_t, rho, cfg.w, i_focus, n_focus, i_active, n_active)
    colsum = torch.empty((cfg.B, cfg.Hkv, cfg.L), dtype=torch.float32, device=DEV)
    sinks = _i32((cfg.B, cfg.Hkv, cfg.S))
    outs, blocks_all = {}, {}
    for l, (Qf, K, V) in enumerate(layers):
        Qa = torch.empty((cfg.B, cfg.Hq, cfg.acap, cfg.d), dtype=torch.bfloat16, device=DEV)
        F.focus_gather_rows(Qf, i_active, n_active, Qa)
        O = torch.empty_like(Qa)
        if l <= cfg.l_dense:
            F.focus_dense_attention(Qa, n_active, K, V, O, colsum=colsum if l == cfg.l_dense else None)
            if l == cfg.l_dense:
                F.focus_sink_identify(colsum, cfg.S, sinks)
        else:
            kbar = torch.empty((cfg.B, cfg.Hkv, cfg.nb, cfg.d), dtype=torch.float32, device=DEV)
            F.focus_block_means(K, cfg.P, cfg.bs, kbar)
            blocks = _i32((cfg.B, cfg.Hkv, cfg.C))
            F.focus_block_select(Qa, n_active, kbar, cfg.C, blocks)
            F.focus_sparse_attention(Qa, n_active, K, V, sinks, blocks, cfg.bs, cfg.P, cfg.g0, cfg.g1, O)
            blocks_all[l] = blocks
        outs[l] = O
    torch.cuda.synchronize()
    f64 = [tuple(inputs.to_f64(t) for t in lay) for lay in layers]
    ref = orc.sparse_step(lambda l: f64[l], cfg.n_layers, cfg.l_dense, st.conf_prev, st.mask, cfg.g0, cfg.g1,
                          cfg.n_t, rho, cfg.w, cfg.P, cfg.bs, cfg.C, cfg.S, cfg.acap,
                          float(np.float32(1 / math.sqrt(cfg.d))))
    assert idx_rows(i_focus) == [a.tolist() for a in ref["I_focus"]]
    assert idx_rows(i_active) == [a.tolist() for a in ref["I_active"]]
    for h in range(cfg.Hkv):
        topk_matches([int(x) for x in sinks[0, h].tolist() if x >= 0], ref["colsum"][0, h], cfg.S)
    assert np.array_equal(sinks.cpu().numpy(), ref["sinks"]), "sink sets differ"
    nA = [len(a) for a in ref["I_active"]]
    for l in range(cfg.n_layers):
        if l in blocks_all:
            assert np.array_equal(blocks_all[l].cpu().numpy(), ref["blocks"][l]), f"layer {l} blocks differ"
        assert_attention_close(outs[l], ref["O"][l], rows_valid=nA, what=f"layer {l}")
    assert F.device_error() == 0


# ------------------------------------------------------------------ fused relevance + top-C + sparse attention
FUSED_CASES = [
    # name, B, Hq, Hkv, P, G, L, bs, C, S, acap, n_active
    ("mha_bs64", 1, 4, 4, 2048, 32, 2112, 64, 8, 8, 32, [30]),
    ("mha_b2_bs32", 2, 4, 4, 1024, 32, 1088, 32, 12, 16, 32, [32, 9]),
    ("gqa2", 1, 8, 4, 1500, 32, 1600, 64, 5, 6, 32, [27]),
    ("ragged_bs24", 1, 2, 2, 250, 20, 300, 24, 4, 3, 20, [20]),
    ("gqa7_sliced", 1, 28, 4, 1024, 32, 1100, 64, 6, 8, 32, [31]),       # 224 rows: four row slices
    ("gqa3_b2", 2, 6, 2, 1024, 32, 1100, 64, 7, 5, 32, [32, 12]),         # 96 rows: two slices
    ("gqa16_two_calls", 1, 16, 1, 1024, 32, 1100, 64, 6, 8, 32, [31]),   # 512 rows: two-call path
    # the fused kernel's limits: 4096 blocks (nb), C = 512, S = 512, 64 rows (NQ = 64)
    ("max_nb_c_s", 1, 2, 1, 32768, 32, 32800, 8, 512, 512, 32, [32]),
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=[c[0] for c in FUSED_CASES])
def test_sparse_fused_matches_oracle_and_two_calls(F, case):
    name, B, Hq, Hkv, P, G, L, bs, C, S, acap, n_act = case
    g0, g1 = P, P + G
    d = 128
    rng = np.random.default_rng(len(name) + L)
    Q = inputs.random_bf16((B, Hq, acap, d), seed=L + 31, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=L + 32, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=L + 33, device=DEV)
    n_active = torch.tensor(n_act, dtype=torch.int32, device=DEV)
    nb = -(-P // bs)
    kbar = torch.empty((B, Hkv, nb, d), dtype=torch.float32, device=DEV)
    F.focus_block_means(K, P, bs, kbar)
    sinks = torch.from_numpy(np.sort(np.stack([np.stack([rng.choice(L, S, replace=False) for _ in range(Hkv)])
                                                for _ in range(B)]), axis=-1).astype(np.int32)).to(DEV)
    blocks_f = _i32((B, Hkv, C))
    O_f = torch.full((B, Hq, acap, d), 4.0, dtype=torch.bfloat16, device=DEV)
    F.focus_sparse_attention_fused(Q, n_active, K, V, kbar, C, sinks, bs, P, g0, g1, blocks_f, O_f)
    blocks_2 = _i32((B, Hkv, C))
    O_2 = torch.full((B, Hq, acap, d), 4.0, dtype=torch.bfloat16, device=DEV)
    F.focus_block_select(Q, n_active, kbar, C, blocks_2)
    F.focus_sparse_attention(Q, n_active, K, V, sinks, blocks_2, bs, P, g0, g1, O_2)
    torch.cuda.synchronize()
    assert torch.equal(blocks_f, blocks_2), "fused top-C differs from focus_block_select"
    # oracle: its own block means and relevance from the same inputs
    Q64, K64, V64 = inputs.to_f64(Q), inputs.to_f64(K), inputs.to_f64(V)
    ref_blocks, R = orc.block_select(Q64, n_act, orc.block_means(K64, P, bs), C)
    assert np.array_equal(blocks_f.cpu().numpy(), ref_blocks), "kept blocks differ from the oracle"
    ref = orc.sparse_attention(Q64, n_act, K64, V64, sinks.cpu().numpy(), ref_blocks, bs, P, g0, g1,
                               float(np.float32(1 / math.sqrt(d))))
    assert_attention_close(O_f, ref, rows_valid=n_act, what=f"fused sparse ({name})")
    assert (O_f.float() - O_2.float()).abs().max().item() <= 1e-2
    assert F.device_error() == 0


# ------------------------------------------------------------------ fused top-C on chosen relevance values
# Every active query row is e_0, so q_bar = e_0 and R_j = kbar[j, 0] / sqrt(d) exactly up to
# one monotone rounding: the block scores are set directly. The patterns reach the exact
# ranking passes inside one value bin, ties at the threshold (lowest indices win), the
# all-equal case, and scores of both signs; nb = 500 takes the one-warp selection and
# nb = 700 the CTA-wide one.
def _top_c_scores(pattern, nb, C, rng):
    if pattern == "outlier_cluster":          # one far outlier: all other scores share a bin
        v = -0.5 + np.arange(nb) * 2.0 ** -9
        v[nb // 3] = 1.0e6
    elif pattern == "ties_at_boundary":       # groups of seven equal scores, shuffled
        v = np.floor(rng.permutation(nb) / 7.0) - 20.0
    elif pattern == "all_equal":
        v = np.full(nb, 0.5)
    elif pattern == "near_tie_cluster":       # the C-th score inside a tight cluster
        v = rng.uniform(-1.0, 1.0, nb)
        idx = rng.permutation(nb)
        v[idx[:C - 11]] = rng.uniform(50.0, 100.0, C - 11)
        v[idx[C - 11:C + 29]] = 2.0 + np.arange(40) * 2.0 ** -16
    else:
        raise ValueError(pattern)
    return v.astype(np.float32)


@pytest.mark.parametrize("nb", [500, 700])
@pytest.mark.parametrize("pattern", ["outlier_cluster", "ties_at_boundary", "all_equal", "near_tie_cluster"])
def test_fused_top_c_chosen_scores(F, pattern, nb):
    B, Hq, Hkv, G, bs, C, S, acap, d = 1, 2, 2, 32, 64, 64, 8, 32, 128
    P = nb * bs
    L, g0, g1 = P + G, P, P + G
    rng = np.random.default_rng(nb + len(pattern))
    Qh = np.zeros((B, Hq, acap, d), dtype=np.float32)
    Qh[..., 0] = 1.0
    Q = torch.from_numpy(Qh).to(torch.bfloat16).to(DEV)
    n_act = [29]
    n_active = torch.tensor(n_act, dtype=torch.int32, device=DEV)
    K = inputs.random_bf16((B, Hkv, L, d), seed=nb + 7, device=DEV)
    V = inputs.random_bf16((B, Hkv, L, d), seed=nb + 8, device=DEV)
    kb = np.zeros((B, Hkv, nb, d), dtype=np.float32)
    for h in range(Hkv):
        kb[0, h, :, 0] = _top_c_scores(pattern, nb, C, rng)
    kbar = torch.from_numpy(kb).to(DEV)
    sinks = torch.from_numpy(np.sort(np.stack([np.stack([rng.choice(L, S, replace=False) for _ in range(Hkv)])
                                                for _ in range(B)]), axis=-1).astype(np.int32)).to(DEV)
    blocks_f = _i32((B, Hkv, C))
    O_f = torch.full((B, Hq, acap, d), 4.0, dtype=torch.bfloat16, device=DEV)
    F.focus_sparse_attention_fused(Q, n_active, K, V, kbar, C, sinks, bs, P, g0, g1, blocks_f, O_f)
    blocks_2 = _i32((B, Hkv, C))
    F.focus_block_select(Q, n_active, kbar, C, blocks_2)
    torch.cuda.synchronize()
    ref_blocks, _ = orc.block_select(inputs.to_f64(Q), n_act, kb.astype(np.float64), C)
    assert np.array_equal(blocks_f.cpu().numpy(), ref_blocks), "fused top-C differs from the oracle"
    assert np.array_equal(blocks_2.cpu().numpy(), ref_blocks), "focus_block_select differs from the oracle"
    Q64, K64, V64 = inputs.to_f64(Q), inputs.to_f64(K), inputs.to_f64(V)
    ref = orc.sparse_attention(Q64, n_act, K64, V64, sinks.cpu().numpy(), ref_blocks, bs, P, g0, g1,
                               float(np.float32(1 / math.sqrt(d))))
    assert_attention_close(O_f, ref, rows_valid=n_act, what=f"fused sparse ({pattern}, nb={nb})")
    assert F.device_error() == 0


# ------------------------------------------------------------------ the step sequencer, plain and variants
@pytest.mark.parametrize("variant", ["plain_fused", "dream_tail_focus_meanq_ratio"])
def test_sparse_step_sequencer(F, variant):
    """SparseStep (the product's step schedule) against the oracle's composed step."""
    from diffusion_long_context_b200 import configs as cf
    from diffusion_long_context_b200.step import SparseStep
    cfg = cf.scaled(cf.LLADA_8K, 1024, n_layers=6, Hq=4, Hkv=2, l_dense=1, C=4, S=8)
    fused = True
    if variant != "plain_fused":
        cfg = cf.ratio_forms(cfg.replace(dense_tail=2, relevance="focus", sink_agg="mean_query"))
        fused = False
    st = inputs.step_state(cfg)
    layers = [inputs.make_layer(cfg, l, DEV, st.sink_pos) for l in range(cfg.n_layers)]
    Q_full = torch.stack([lay[0] for lay in layers])
    step = SparseStep(cfg, Q_full, [lay[1] for lay in layers], [lay[2] for lay in layers], device=DEV, fused=fused)
    step.set_state(torch.from_numpy(st.conf_prev), torch.from_numpy(st.mask), non_blocking=False)
    step.block_entry()
    step.run()
    torch.cuda.synchronize()
    f64 = [tuple(inputs.to_f64(t) for t in lay) for lay in layers]
    ref = orc.sparse_step(lambda l: f64[l], cfg.n_layers, cfg.l_dense, st.conf_prev, st.mask, cfg.g0, cfg.g1,
                          cfg.n_t, step.rho, cfg.w, cfg.P, cfg.bs, cfg.C, cfg.S, cfg.acap,
                          float(np.float32(1 / math.sqrt(cfg.d))), dense_tail=cfg.dense_tail,
                          relevance=cfg.relevance, sink_agg=cfg.sink_agg)
    assert idx_rows(step.i_active) == [a.tolist() for a in ref["I_active"]]
    assert np.array_equal(step.sinks.cpu().numpy(), ref["sinks"]), "sink sets differ"
    nA = [len(a) for a in ref["I_active"]]
    assert sorted(ref["blocks"]) == step.sparse_layers
    for l in range(cfg.n_layers):
        if l in step.sparse_layers:
            assert np.array_equal(step.blocks[l].cpu().numpy(), ref["blocks"][l]), f"layer {l} blocks differ"
        assert_attention_close(step.O_active[l], ref["O"][l], rows_valid=nA, what=f"{variant} layer {l}")
    assert F.device_error() == 0


def test_step_graph_with_host_io(F):
    """SparseStep.capture_io: one graph holding the host-state copies in, the step and the
    copies out gives the same host results as the step graph plus separate copies."""
    from diffusion_long_context_b200 import configs as cf
    from diffusion_long_context_b200.step import SparseStep
    cfg = cf.scaled(cf.LLADA_8K, 1024, n_layers=4, Hq=4, Hkv=2, l_dense=1, C=4, S=8)
    st = inputs.step_state(cfg)
    layers = [inputs.make_layer(cfg, l, DEV, st.sink_pos) for l in range(cfg.n_layers)]
    Q_full = torch.stack([lay[0] for lay in layers])
    step = SparseStep(cfg, Q_full, [lay[1] for lay in layers], [lay[2] for lay in layers], device=DEV)
    conf_h = torch.from_numpy(st.conf_prev).pin_memory()
    mask_h = torch.from_numpy(st.mask).pin_memory()
    step.set_state(conf_h, mask_h, non_blocking=False)
    step.block_entry()
    step.capture()
    step.replay()
    torch.cuda.synchronize()
    ref_o, ref_a, ref_n = step.O_active[-1].cpu(), step.i_active.cpu(), step.n_active.cpu()
    step.O_active[-1].zero_()
    step.i_active.fill_(-5)
    out_h = torch.full(ref_o.shape, 7.0, dtype=torch.bfloat16).pin_memory()
    act_h = torch.full(ref_a.shape, -9, dtype=torch.int32).pin_memory()
    nact_h = torch.zeros(ref_n.shape, dtype=torch.int32).pin_memory()
    step.capture_io(conf_h, mask_h, [(out_h, step.O_active[-1]), (act_h, step.i_active), (nact_h, step.n_active)])
    for _ in range(2):
        step.replay_io()
        torch.cuda.current_stream().synchronize()
    assert torch.equal(act_h, ref_a) and torch.equal(nact_h, ref_n)
    # the cluster's tiles are claimed dynamically, so the last bits of O may differ
    torch.testing.assert_close(out_h.float(), ref_o.float(), rtol=0, atol=1e-2)
    step.release()
    assert F.device_error() == 0
