"""Synthetic workload configurations for the Focus-dLLM sparse denoising step.

The Focus-dLLM pages (paper.rainbus.top summary of arXiv 2602.02159, section
"方法步骤详情" / method steps; hyper-parameters in "复现评估" / reproducibility)
measure on LongBench with UltraLLaDA / Dream-7B weights. Neither the datasets nor
the weights exist here, so these seeded synthetic shapes stand in for them:
LLaDA-8B-shaped MHA (32 x 128, 32 layers) and Dream-7B-shaped GQA (28 q / 4 kv
heads x 128, 28 layers) at 8K, 16K and 32K context.

Positions: prompt = [0, P), current generation block = [g0, g1) with g0 = P,
later generation positions [g1, L) are still [MASK].
"""
from __future__ import annotations

import dataclasses
from typing import Optional, List


@dataclasses.dataclass(frozen=True)
class FocusConfig:
    name: str
    B: int                 # independent sequences
    L: int                 # context length (prompt + generation canvas)
    P: int                 # prompt length
    G: int                 # current generation block size (g1 - g0)
    Hq: int                # query heads
    Hkv: int               # key/value heads
    d: int                 # head dim
    n_layers: int
    l_dense: int           # layers 0..l_dense are dense; layer l_dense finds the sinks
    n_masked: int          # still-[MASK] positions inside the current block
    conf_dist: str         # "uniform" -> U(0,1), "beta25" -> Beta(2,5)
    n_t: int               # tokens decoded at this step, n(t)
    rho: float             # expansion factor
    w: int                 # window size
    bs: int                # prompt key block size
    C: int                 # kept prompt blocks
    S: int                 # attention sinks per KV head
    n_planted_sinks: int   # sink positions planted in the keys (same in every layer)
    positional: bool       # add the seeded rank-8 smooth positional component to Q and K
    seed: int
    # variants the pages describe (defaults: the configs' plain schedule)
    dense_tail: int = 0            # the last dense_tail layers also run dense (Dream keeps 4)
    relevance: str = "active"      # block relevance from "active" (I_active) or "focus" (I_focus) rows
    sink_agg: str = "probs"        # sink importance: "probs" (sum of softmax rows) or "mean_query"

    @property
    def g0(self) -> int:
        return self.P

    @property
    def g1(self) -> int:
        return self.P + self.G

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nb(self) -> int:
        return -(-self.P // self.bs)

    @property
    def k(self) -> int:
        """k = floor(rho * n(t)) before clamping to the number of masked positions."""
        import math
        return int(math.floor(float(self.rho) * float(self.n_t)))

    @property
    def acap(self) -> int:
        """Capacity of the active-query list: at most G positions of the current block."""
        return self.G

    @property
    def kv_cap(self) -> int:
        """Upper bound on |I_p| = S + C*bs + G keys (before de-duplication)."""
        return self.S + min(self.C, self.nb) * self.bs + self.G

    @property
    def dense_layers(self) -> List[int]:
        """Layers 0..l_dense, then the last dense_tail layers."""
        tail = range(max(self.l_dense + 1, self.n_layers - self.dense_tail), self.n_layers)
        return list(range(min(self.l_dense + 1, self.n_layers))) + list(tail)

    @property
    def sparse_layers(self) -> List[int]:
        dense = set(self.dense_layers)
        return [l for l in range(self.n_layers) if l not in dense]

    def replace(self, **kw) -> "FocusConfig":
        return dataclasses.replace(self, **kw)


def ratio_forms(cfg: FocusConfig, alpha: float = 0.5, sink_frac: float = 0.01) -> FocusConfig:
    """The pages' ratio forms of C and S (reproducibility section: alpha = 0.5,
    N_sinks = 0.01 x M): C = ceil(alpha * nb) kept prompt blocks and S = ceil(sink_frac * L)
    sinks, L (the context length) standing for M."""
    import math
    return cfg.replace(C=max(1, math.ceil(alpha * cfg.nb)), S=max(1, math.ceil(sink_frac * cfg.L)))


TINY = FocusConfig(
    name="tiny_L512_H4_d64", B=1, L=512, P=448, G=32, Hq=4, Hkv=4, d=64, n_layers=1,
    l_dense=0, n_masked=16, conf_dist="uniform", n_t=2, rho=4.0, w=4, bs=32, C=4, S=4,
    n_planted_sinks=2, positional=False, seed=1001)

LLADA_8K = FocusConfig(
    name="llada8b_mha32x128_L8192", B=1, L=8192, P=7936, G=32, Hq=32, Hkv=32, d=128,
    n_layers=32, l_dense=2, n_masked=16, conf_dist="beta25", n_t=4, rho=4.0, w=8, bs=64,
    C=16, S=16, n_planted_sinks=8, positional=True, seed=2002)

DREAM_16K = FocusConfig(
    name="dream7b_gqa28q4kv_L16384", B=1, L=16384, P=16128, G=32, Hq=28, Hkv=4, d=128,
    n_layers=28, l_dense=2, n_masked=16, conf_dist="beta25", n_t=4, rho=4.0, w=8, bs=64,
    C=32, S=16, n_planted_sinks=8, positional=True, seed=3003)

FULL_32K = FocusConfig(
    name="llada8b_mha32x128_L32768_step", B=1, L=32768, P=32512, G=32, Hq=32, Hkv=32,
    d=128, n_layers=32, l_dense=2, n_masked=16, conf_dist="beta25", n_t=4, rho=4.0, w=8,
    bs=64, C=64, S=32, n_planted_sinks=8, positional=True, seed=4004)

SWEEP_BASE = FocusConfig(
    name="sweep_B4_mha32x128_L32768", B=4, L=32768, P=32512, G=32, Hq=32, Hkv=32, d=128,
    n_layers=1, l_dense=0, n_masked=16, conf_dist="beta25", n_t=4, rho=4.0, w=8, bs=64,
    C=32, S=32, n_planted_sinks=8, positional=True, seed=5005)


def sweep_points():
    """Block size x C grid at rho=4, then rho in {2,4,8} at bs=64, C=32 (w=8, S=32)."""
    pts = []
    for bs in (32, 64, 128):
        for C in (8, 32, 128):
            pts.append(SWEEP_BASE.replace(name=f"sweep_bs{bs}_C{C}_rho4", bs=bs, C=C))
    for rho in (2.0, 8.0):
        pts.append(SWEEP_BASE.replace(name=f"sweep_bs64_C32_rho{int(rho)}", rho=rho))
    return pts


ALL = {c.name: c for c in (TINY, LLADA_8K, DREAM_16K, FULL_32K, SWEEP_BASE)}


def scaled(cfg: FocusConfig, L: int, n_layers: Optional[int] = None, **kw) -> FocusConfig:
    """Same generators at a shorter context: P = L - 2*G (one current block, one future block)."""
    P = L - 2 * cfg.G
    return cfg.replace(name=f"{cfg.name}_at{L}", L=L, P=P,
                       n_layers=cfg.n_layers if n_layers is None else n_layers, **kw)
