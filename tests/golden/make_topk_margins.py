"""Writes tests/golden/topk_margins.txt: how far every top-k of the fixed seeds is from a tie.

Every index set of a Focus-dLLM step is a top-k (summary page of arXiv 2602.02159, method
steps (1), (3), (4)): I_focus (top-k of c_{t-1} over the masked positions), the sinks
(top-S of the sink layer's column sums) and the kept blocks of every sparse layer (top-C
of R_b per KV head). The GPU path must reproduce them bit for bit; that is only a fair
demand where the k-th and (k+1)-th scores differ by well more than fp32 rounding. This
script computes, with the fp64 oracle only, the smallest relative margin
(k-th - (k+1)-th) / |k-th| of every set family at the seeded workloads, so that a near-tie
is reported as a property of the input.

The inputs come from diffusion_long_context_b200.inputs on the device the GPU tests use
(torch's CUDA generator when a GPU is present: the values differ from a CPU run), so
run it on a GPU machine:

  python tests/golden/make_topk_margins.py [--out tests/golden/topk_margins.txt] [--quick]

--quick covers the tiny and 8K workloads only. Output lines:
  <workload> <set> n=<number of sets> k=<k> min_rel_margin=<x> at=<where>
"""
from __future__ import annotations

import argparse
import math
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from diffusion_long_context_b200 import configs, inputs  # noqa: E402
from oracle import focus_oracle as orc  # noqa: E402


def _active_rows(Qf, active, cap):
    """Active query rows of the generated Q, widened to float64 (indexing only)."""
    B, H, _, d = Qf.shape
    out = np.zeros((B, H, cap, d))
    for b in range(B):
        r = torch.as_tensor(active[b], dtype=torch.long, device=Qf.device)
        out[b, :, :r.numel()] = inputs.to_f64(Qf[b][:, r])
    return out


def _min_rel(score_sets, k):
    """Smallest relative top-k margin over a list of (label, scores)."""
    best, where = math.inf, "-"
    for label, s in score_sets:
        m = orc.top_k_relative_margin(s, k)
        if m < best:
            best, where = m, label
    return best, where


def margins(cfg, dev, layers=None):
    """Rows (set, n, k, min_rel_margin, where) for one workload."""
    st = inputs.step_state(cfg)
    rho = float(np.float32(cfg.rho))
    scale = float(np.float32(1 / math.sqrt(cfg.d)))
    rows = []
    # I_focus: top-k of c_{t-1} over the masked positions of the current block
    focus, active = orc.select_queries(st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, rho, cfg.w)
    sets = []
    for b in range(cfg.B):
        cand = [p for p in range(cfg.g0, cfg.g1) if st.mask[b, p]]
        sets.append((f"b{b}", np.array([st.conf_prev[b, p - cfg.g0] for p in cand], dtype=np.float64)))
    k = min(cfg.k, cfg.n_masked)
    m, w = _min_rel(sets, k)
    rows.append(("I_focus", len(sets), k, m, w))
    nA = [a.size for a in active]
    # sinks: top-S of the sink layer's column sums
    ld = cfg.l_dense
    Qf, K, V = inputs.make_layer(cfg, ld, dev, st.sink_pos)
    Qa = _active_rows(Qf, active, cfg.acap)
    _, colsum, _ = orc.dense_attention(Qa, nA, inputs.to_f64(K), inputs.to_f64(V), scale, want_colsum=True)
    del Qf, K, V
    sets = [(f"b{b}h{h}", colsum[b, h]) for b in range(cfg.B) for h in range(cfg.Hkv)]
    m, w = _min_rel(sets, min(cfg.S, cfg.L))
    rows.append(("sinks", len(sets), min(cfg.S, cfg.L), m, w))
    # kept blocks: top-C of R_b in every sparse layer
    sparse = [l for l in range(cfg.n_layers) if l > ld] if layers is None else layers
    if not sparse:
        sparse = [ld]           # a one-layer workload: its parity tests select blocks on that layer
    sets = []
    for l in sparse:
        Qf, K, _ = inputs.make_layer(cfg, l, dev, st.sink_pos)
        Qa = _active_rows(Qf, active, cfg.acap)
        kbar = orc.block_means(inputs.to_f64(K), cfg.P, cfg.bs)
        del Qf, K
        R = orc.block_relevance(Qa, nA, kbar)
        sets += [(f"l{l}b{b}h{h}", R[b, h]) for b in range(cfg.B) for h in range(cfg.Hkv)]
    if sets:
        k = min(cfg.C, cfg.nb)
        m, w = _min_rel(sets, k)
        rows.append(("blocks", len(sets), k, m, w))
    return rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=os.path.join(ROOT, "tests", "golden", "topk_margins.txt"))
    ap.add_argument("--quick", action="store_true", help="tiny and 8K workloads only")
    a = ap.parse_args()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    work = [(configs.TINY, None), (configs.LLADA_8K, None)]
    if not a.quick:
        work += [(configs.DREAM_16K, None), (configs.FULL_32K, None)]
        for p in configs.sweep_points():
            work.append((p.replace(n_layers=2, l_dense=0), None))
    lines = [
        "# Smallest relative top-k margin (k-th - (k+1)-th) / |k-th| of every index-set family",
        "# of the seeded workloads, from the fp64 oracle (written by make_topk_margins.py;",
        f"# inputs generated on {dev}). Sets: I_focus per sequence, sinks per (sequence, KV",
        "# head) of the sink layer, kept blocks per (sparse layer, sequence, KV head).",
    ]
    for cfg, layers in work:
        t0 = time.time()
        for name, n, k, m, w in margins(cfg, dev, layers):
            lines.append(f"{cfg.name} {name} n={n} k={k} min_rel_margin={m:.6e} at={w}")
        print(f"{cfg.name}: {time.time() - t0:.1f} s", flush=True)
    with open(a.out, "w") as f:
        f.write("\n".join(lines) + "\n")
    print("\n".join(lines))


if __name__ == "__main__":
    main()
