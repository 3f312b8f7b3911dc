"""The pins catch plausible oracle mistakes (CPU only).

Each case plants one mistake in a copy of an oracle function (source edit of the
function, executed in the oracle's namespace and monkeypatched in for the test only)
and asserts that at least one of the named pin tests then fails. The oracle itself is
never modified on disk.
"""
import inspect
import textwrap

import pytest

import test_oracle_pins as pins
from oracle import focus_oracle as orc

MUTATIONS = [
    # (id, function, original text, mistaken text, pins expected to catch it)
    ("window_centre_off_by_one", "select_queries", "lo = p - w // 2", "lo = p - (w - 1) // 2",
     [lambda: pins.test_select_queries_golden(4)]),
    ("window_not_clipped_high", "select_queries", "min(g1 - 1, lo + w - 1)", "lo + w - 1",
     [pins.test_select_queries_golden_edge]),
    ("mask_ignored", "select_queries", "if mask[b, p] != 0", "if True",
     [lambda: pins.test_select_queries_golden(3)]),
    ("k_rounded_up", "select_queries", "k_req = int(math.floor(float(rho) * float(n_t)))",
     "k_req = int(math.ceil(float(rho) * float(n_t)))", [lambda: pins.test_select_queries_golden(3)]),
    ("ties_to_higher_index", "top_k_ascending", "order = np.lexsort((idx, -s))", "order = np.lexsort((-idx, -s))",
     [pins.test_top_k_golden_ties, pins.test_top_k_brute_force_with_ties]),
    ("ascending_scores_picked", "top_k_ascending", "order = np.lexsort((idx, -s))", "order = np.lexsort((idx, s))",
     [pins.test_top_k_golden_ties]),
    ("block_mean_divides_by_bs", "block_means", "kbar[:, :, blk] = K[:, :, r0:r1].mean(axis=2)",
     "kbar[:, :, blk] = K[:, :, r0:r1].sum(axis=2) / bs", [pins.test_block_means_against_reduceat]),
    ("relevance_drops_scale", "block_relevance", "dots = (q @ kbar[b, h].T) / math.sqrt(d)",
     "dots = (q @ kbar[b, h].T)", [pins.test_block_relevance_golden]),
    ("relevance_wrong_group", "block_relevance", "q = Q_active[b, h * g:(h + 1) * g, :A]",
     "q = Q_active[b, h:h + g, :A]", [pins.test_block_relevance_equals_mean_query_closed_form]),
    ("softmax_sign_flipped", "dense_attention", "e = np.exp(s - m)", "e = np.exp(m - s)",
     [lambda: pins.test_dense_attention_vs_sdpa(4, 4)]),
    ("values_transposed_with_keys", "dense_attention", "O[b, hq, :n] = p @ V[b, h]",
     "O[b, hq, :n] = p @ K[b, h]", [lambda: pins.test_dense_attention_vs_sdpa(4, 4)]),
    ("gqa_head_index", "dense_attention", "h = hq // g\n            s = ", "h = hq % Hkv\n            s = ",
     [lambda: pins.test_dense_attention_vs_sdpa(6, 2)]),
    ("colsum_unnormalised", "dense_attention", "colsum[b, h] += p.sum(axis=0)", "colsum[b, h] += e.sum(axis=0)",
     [lambda: pins.test_dense_attention_vs_sdpa(4, 4), pins.test_dense_attention_golden_two_keys]),
    ("scale_dropped", "dense_attention", "s = (Q[b, hq, :n] @ K[b, h].T) * scale",
     "s = (Q[b, hq, :n] @ K[b, h].T)", [lambda: pins.test_dense_attention_vs_sdpa(4, 4)]),
    ("current_block_left_out", "sparse_key_set", "keys.update(range(g0, g1))", "pass",
     [pins.test_sparse_key_set_golden]),
    ("last_block_not_clipped", "sparse_key_set", "min(P, (int(blk) + 1) * bs)", "(int(blk) + 1) * bs",
     [pins.test_sparse_partial_last_block]),
    ("sinks_dropped", "sparse_key_set", "keys = set(int(j) for j in sinks_bh if j >= 0)", "keys = set()",
     [pins.test_sparse_key_set_golden]),
]


def _mutated(fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(orc, fn_name)))
    assert old in src, f"mutation anchor not found in {fn_name}: {old!r}"
    ns = dict(vars(orc))
    exec(compile(src.replace(old, new, 1), f"<mutated {fn_name}>", "exec"), ns)
    return ns[fn_name]


@pytest.mark.parametrize("mid,fn,old,new,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(monkeypatch, mid, fn, old, new, checks):
    monkeypatch.setattr(orc, fn, _mutated(fn, old, new))
    caught = 0
    for check in checks:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake {mid}"


def test_unmutated_oracle_passes_the_same_checks():
    for _, _, _, _, checks in MUTATIONS:
        for check in checks:
            check()
