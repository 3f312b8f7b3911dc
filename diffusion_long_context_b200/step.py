"""The Focus-dLLM denoising step, sequenced over the C-ABI calls.

A non-block-entry step (Focus-dLLM summary page, "方法步骤详情" / method steps (1)-(5)):
  select_queries -> gather the active query rows of every layer -> layers 0..l_dense:
  dense attention (layer l_dense also produces the sink column sums) -> sink top-S ->
  layers > l_dense: block relevance + top-C and sparse attention over sinks U blocks U
  current block (one fused launch per layer, or two calls).
A block-entry step refreshes the block means of every sparse layer (and, for the
comparison, runs the dense full refresh).

This module only allocates buffers and orders the calls on one CUDA stream; every
step of the computation runs in libfocus.so kernels. `SparseStep.capture()` records
the whole step into a CUDA graph so that replay costs one launch from the host.
"""
from __future__ import annotations

import math
from typing import List, Optional

import torch

from . import focus as F
from .configs import FocusConfig


class SparseStep:
    def __init__(self, cfg: FocusConfig, Q_full: torch.Tensor, K: List[torch.Tensor], V: List[torch.Tensor],
                 device="cuda", fused: bool = True):
        """Q_full [n_layers, B, Hq, L, d]; K[l], V[l] [B, Hkv, L, d] (bf16, on `device`).

        fused: each sparse layer runs block relevance + top-C and the sparse attention as
        one launch (focus_sparse_attention_fused), else as two calls. The config's variants
        (dense_tail, relevance, sink_agg) change the schedule; relevance="focus" runs the
        two calls."""
        c = cfg
        self.cfg = c
        self.fused = fused
        self.dev = torch.device(device)
        self.Q_full, self.K, self.V = Q_full, K, V
        self.scale = 1.0 / math.sqrt(c.d)
        self.rho = float(torch.tensor(c.rho, dtype=torch.float32))
        i32 = dict(dtype=torch.int32, device=self.dev)
        bf = dict(dtype=torch.bfloat16, device=self.dev)
        self.kcap = max(1, min(c.k, c.G))
        self.conf_prev = torch.zeros((c.B, c.G), dtype=torch.float32, device=self.dev)
        self.mask = torch.zeros((c.B, c.L), dtype=torch.uint8, device=self.dev)
        self.i_focus = torch.full((c.B, self.kcap), -1, **i32)
        self.n_focus = torch.zeros((c.B,), **i32)
        self.i_active = torch.full((c.B, c.acap), -1, **i32)
        self.n_active = torch.zeros((c.B,), **i32)
        self.Q_active = torch.zeros((c.n_layers, c.B, c.Hq, c.acap, c.d), **bf)
        self.O_active = torch.zeros((c.n_layers, c.B, c.Hq, c.acap, c.d), **bf)
        self.colsum = torch.zeros((c.B, c.Hkv, c.L), dtype=torch.float32, device=self.dev)
        self.sinks = torch.full((c.B, c.Hkv, c.S), -1, **i32)
        self.dense_layers = c.dense_layers
        self.sparse_layers = c.sparse_layers
        # variants: relevance from the I_focus rows needs their queries (and the two-call
        # layer, the fused kernel scores with the rows it attends with); mean-query sinks
        # score every key of the sink layer, held as fp32 "blocks" of one key
        self.Q_focus = (torch.zeros((c.n_layers, c.B, c.Hq, self.kcap, c.d), **bf) if c.relevance == "focus"
                        else None)
        if c.relevance == "focus":
            self.fused = False
        self.k_rows = (torch.zeros((c.B, c.Hkv, c.L, c.d), dtype=torch.float32, device=self.dev)
                       if c.sink_agg == "mean_query" else None)
        self.kbar = {l: torch.zeros((c.B, c.Hkv, c.nb, c.d), dtype=torch.float32, device=self.dev)
                     for l in self.sparse_layers}
        self.blocks = {l: torch.full((c.B, c.Hkv, c.C), -1, **i32) for l in self.sparse_layers}
        dws = F.dense_workspace_bytes(c.B, c.Hq, c.Hkv, c.L, c.d, c.acap, True)
        sws = F.sparse_workspace_bytes(c.B, c.Hq, c.Hkv, c.L, c.d, c.acap, c.S, c.C, c.bs, c.P, c.g0, c.g1)
        self.ws = torch.empty(max(dws, sws, 256), dtype=torch.uint8, device=self.dev)
        self.graph: Optional[torch.cuda.CUDAGraph] = None
        self.graph_io: Optional[torch.cuda.CUDAGraph] = None
        self.launches_per_step: Optional[int] = None

    # ------------------------------------------------------------------ inputs
    def set_state(self, conf_prev: torch.Tensor, mask: torch.Tensor, non_blocking=True):
        self.conf_prev.copy_(conf_prev, non_blocking=non_blocking)
        self.mask.copy_(mask, non_blocking=non_blocking)

    # ------------------------------------------------------------------ block entry
    def block_entry(self, O_full: Optional[torch.Tensor] = None):
        """Block entry. Without O_full: the block means of every sparse layer only (cached for
        the later steps of the block). With O_full [B, Hq, L, d]: the block-entry step proper,
        every layer's dense full refresh into O_full (reused per layer), the sparse layers'
        block means computed in the same launch."""
        c = self.cfg
        if O_full is None:
            for l in self.sparse_layers:
                F.focus_block_means(self.K[l], c.P, c.bs, self.kbar[l])
            return
        for l in range(c.n_layers):
            self.full_refresh_layer(l, O_full)

    def full_refresh_layer(self, l: int, O_full: torch.Tensor):
        """Dense full refresh of layer l: every query of the sequence over all L keys (with the
        layer's block means when it is a sparse layer)."""
        c = self.cfg
        if l in self.kbar:
            F.focus_full_refresh(self.Q_full[l], self.K[l], self.V[l], O_full, c.P, c.bs, self.kbar[l],
                                 scale=self.scale)
        else:
            F.focus_dense_attention(self.Q_full[l], None, self.K[l], self.V[l], O_full, scale=self.scale)

    # ------------------------------------------------------------------ sparse step
    def select(self):
        c = self.cfg
        F.focus_select_queries(self.conf_prev, self.mask, c.g0, c.g1, c.n_t, self.rho, c.w, self.i_focus,
                               self.n_focus, self.i_active, self.n_active)
        F.focus_gather_rows(self.Q_full, self.i_active, self.n_active, self.Q_active)
        if self.Q_focus is not None:
            F.focus_gather_rows(self.Q_full, self.i_focus, self.n_focus, self.Q_focus)

    def dense_layer(self, l: int):
        c = self.cfg
        sink_layer = l == c.l_dense
        probs = sink_layer and c.sink_agg == "probs"
        if probs:
            # attention, column sums and the top-S sinks in one call (one launch where served)
            F.focus_dense_attention_sinks(self.Q_active[l], self.n_active, self.K[l], self.V[l], self.O_active[l],
                                          self.colsum, self.sinks, scale=self.scale, ws=self.ws)
            return
        F.focus_dense_attention(self.Q_active[l], self.n_active, self.K[l], self.V[l], self.O_active[l],
                                scale=self.scale, ws=self.ws)
        if sink_layer:
            # mean-query importance: top-S of qbar . k_j over all L keys (each key a block of one)
            F.focus_block_means(self.K[l], c.L, 1, self.k_rows)
            F.focus_block_select(self.Q_active[l], self.n_active, self.k_rows, c.S, self.sinks)

    def block_select_layer(self, l: int):
        if self.Q_focus is not None:
            F.focus_block_select(self.Q_focus[l], self.n_focus, self.kbar[l], self.cfg.C, self.blocks[l])
        else:
            F.focus_block_select(self.Q_active[l], self.n_active, self.kbar[l], self.cfg.C, self.blocks[l])

    def sparse_attention_layer(self, l: int):
        c = self.cfg
        F.focus_sparse_attention(self.Q_active[l], self.n_active, self.K[l], self.V[l], self.sinks,
                                 self.blocks[l], c.bs, c.P, c.g0, c.g1, self.O_active[l], scale=self.scale,
                                 ws=self.ws)

    def sparse_layer_fused(self, l: int):
        """Block relevance + top-C + sparse attention of layer l in one launch."""
        c = self.cfg
        F.focus_sparse_attention_fused(self.Q_active[l], self.n_active, self.K[l], self.V[l], self.kbar[l], c.C,
                                       self.sinks, c.bs, c.P, c.g0, c.g1, self.blocks[l], self.O_active[l],
                                       scale=self.scale, ws=self.ws)

    def run(self, timers=None):
        """Eager step. `timers` (optional) maps a call kind to a list receiving (start, end) events."""
        c = self.cfg

        def timed(kind, fn, *args):
            if timers is None:
                fn(*args)
                return
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn(*args)
            e.record()
            timers.setdefault(kind, []).append((s, e))

        timed("select", self.select)
        dense = set(self.dense_layers)
        for l in range(c.n_layers):
            if l in dense:
                timed("dense_attention" if l != c.l_dense else "dense_attention_colsum", self.dense_layer, l)
            elif self.fused:
                timed("sparse_layer_fused", self.sparse_layer_fused, l)
            else:
                timed("block_select", self.block_select_layer, l)
                timed("sparse_attention", self.sparse_attention_layer, l)

    # ------------------------------------------------------------------ graphs
    def capture(self):
        before = F.launch_count()
        self.run()                      # warm: configures kernels, touches every buffer
        torch.cuda.synchronize()
        self.launches_per_step = F.launch_count() - before
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.run()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = g
        return g

    def capture_io(self, conf_h: torch.Tensor, mask_h: torch.Tensor, outs):
        """The step with its host traffic in one graph: the pinned host state (conf_h, mask_h)
        is copied in, the step runs, and each (pinned host tensor, device tensor) pair of
        `outs` is copied out, so that one replay_io() is one launch from the host."""
        for t in (conf_h, mask_h, *(h for h, _ in outs)):
            if not t.is_pinned():
                raise ValueError("capture_io needs pinned host tensors")
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.conf_prev.copy_(conf_h, non_blocking=True)
                self.mask.copy_(mask_h, non_blocking=True)
                self.run()
                for h, d in outs:
                    h.copy_(d, non_blocking=True)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph_io = g
        return g

    def replay(self):
        self.graph.replay()

    def replay_io(self):
        self.graph_io.replay()

    def release(self):
        self.graph = None
        self.graph_io = None
