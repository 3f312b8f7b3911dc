"""One-layer workload for kernel profiling (ncu) of a single Focus-dLLM call.

  python -m diffusion_long_context_b200.profile_case --call sparse|fused|dense|colsum|sinks|select|blocks|means|refresh|entry \
      [--L 32768] [--repeat 3]

Builds one layer of the 32K LLaDA-shaped step (synthetic, seeded), runs the whole step
once so every index set is real, then launches the chosen call `--repeat` times. The
K/V of the layer (537 MB at 32K) is larger than L2.
"""
from __future__ import annotations

import argparse
import math

import torch

from . import configs, inputs
from . import focus as F


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--call", default="sparse",
                    choices=["sparse", "fused", "dense", "colsum", "sinks", "select", "blocks", "means", "refresh",
                             "entry"])
    ap.add_argument("--L", type=int, default=32768)
    ap.add_argument("--repeat", type=int, default=3)
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    c = configs.FULL_32K if a.L == 32768 else configs.scaled(configs.FULL_32K, a.L)
    c = c.replace(n_layers=1, l_dense=0)
    st = inputs.step_state(c)
    Qf, K, V = inputs.make_layer(c, 0, dev, st.sink_pos)
    i32 = dict(dtype=torch.int32, device=dev)
    conf = torch.from_numpy(st.conf_prev).to(dev)
    mask = torch.from_numpy(st.mask).to(dev)
    i_focus, n_focus = torch.empty((c.B, c.G), **i32), torch.empty((c.B,), **i32)
    i_active, n_active = torch.empty((c.B, c.acap), **i32), torch.empty((c.B,), **i32)
    rho = float(torch.tensor(c.rho, dtype=torch.float32))
    Qa = torch.empty((c.B, c.Hq, c.acap, c.d), dtype=torch.bfloat16, device=dev)
    O = torch.empty_like(Qa)
    colsum = torch.empty((c.B, c.Hkv, c.L), dtype=torch.float32, device=dev)
    sinks = torch.empty((c.B, c.Hkv, c.S), **i32)
    kbar = torch.empty((c.B, c.Hkv, c.nb, c.d), dtype=torch.float32, device=dev)
    blocks = torch.empty((c.B, c.Hkv, c.C), **i32)
    ws = torch.empty(max(F.dense_workspace_bytes(c.B, c.Hq, c.Hkv, c.L, c.d, c.acap, True),
                         F.sparse_workspace_bytes(c.B, c.Hq, c.Hkv, c.L, c.d, c.acap, c.S, c.C, c.bs, c.P,
                                                  c.g0, c.g1), 256), dtype=torch.uint8, device=dev)

    def select():
        F.focus_select_queries(conf, mask, c.g0, c.g1, c.n_t, rho, c.w, i_focus, n_focus, i_active, n_active)
        F.focus_gather_rows(Qf, i_active, n_active, Qa)

    def dense():
        F.focus_dense_attention(Qa, n_active, K, V, O, ws=ws)

    def dense_colsum():
        F.focus_dense_attention(Qa, n_active, K, V, O, colsum=colsum, ws=ws)
        F.focus_sink_identify(colsum, c.S, sinks)

    def sink_layer():
        F.focus_dense_attention_sinks(Qa, n_active, K, V, O, colsum, sinks, ws=ws)

    def means():
        F.focus_block_means(K, c.P, c.bs, kbar)

    def blocks_sel():
        F.focus_block_select(Qa, n_active, kbar, c.C, blocks)

    def sparse():
        F.focus_sparse_attention(Qa, n_active, K, V, sinks, blocks, c.bs, c.P, c.g0, c.g1, O, ws=ws)

    def fused():
        F.focus_sparse_attention_fused(Qa, n_active, K, V, kbar, c.C, sinks, c.bs, c.P, c.g0, c.g1, blocks, O,
                                       ws=ws)

    O_full = None

    def refresh():
        F.focus_dense_attention(Qf, None, K, V, O_full, scale=1 / math.sqrt(c.d))

    def entry():
        F.focus_full_refresh(Qf, K, V, O_full, c.P, c.bs, kbar, scale=1 / math.sqrt(c.d))

    select()
    dense_colsum()
    means()
    blocks_sel()
    sparse()
    torch.cuda.synchronize()
    if a.call in ("refresh", "entry"):
        O_full = torch.empty((c.B, c.Hq, c.L, c.d), dtype=torch.bfloat16, device=dev)
    fn = {"sparse": sparse, "fused": fused, "dense": dense, "colsum": dense_colsum, "select": select, "blocks": blocks_sel,
          "means": means, "refresh": refresh, "entry": entry, "sinks": sink_layer}[a.call]
    for _ in range(a.repeat):
        fn()
    torch.cuda.synchronize()
    assert F.device_error() == 0
    print(f"profile_case {a.call} L={c.L} repeat={a.repeat} ok")


if __name__ == "__main__":
    main()
