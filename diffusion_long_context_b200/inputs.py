"""Seeded synthetic inputs for the Focus-dLLM sparse denoising step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic. Both the CUDA path and the oracle consume its output.

Recipe (the shapes follow LLaDA-8B / Dream-7B attention; values are synthetic):
  * Q, K, V ~ N(0, 1), layout [B, H, L, d], rounded to bf16 at the end.
  * Optional rank-8 smooth positional component, shared by Q and K of a KV-head
    group: for r = 0..3, f_r = 2**r cycles over L, phi_{2r}(p) = sin(2 pi f_r p / L),
    phi_{2r+1}(p) = cos(2 pi f_r p / L); X_p += 0.5 * sum_j phi_j(p) a_j with
    a_j ~ N(0, I_d) per (layer, KV head). Block relevance is then non-uniform.
  * Planted attention sinks at the same positions in every layer: position 0 plus
    seeded prompt positions. k_j += 3 u_h where u_h = sqrt(d) * (unit vector of the
    mean query of KV-head group h over all L positions).
  * Mask [B, L] uint8: prompt [0, P) decoded (0); current block [g0, g1) has
    `n_masked` seeded still-[MASK] positions (1); later blocks [g1, L) are [MASK].
  * Previous-step confidence c_{t-1} [B, G] fp32 on the current block: U(0,1) or
    Beta(2,5) at masked positions; 2.0 at decoded positions (so a kernel that ignores
    the mask picks them and fails parity).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from .configs import FocusConfig


@dataclass
class StepState:
    mask: np.ndarray          # uint8 [B, L]
    conf_prev: np.ndarray     # float32 [B, G]
    sink_pos: np.ndarray      # int64 [n_planted]


def step_state(cfg: FocusConfig) -> StepState:
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    B, L, G = cfg.B, cfg.L, cfg.G
    mask = np.zeros((B, L), dtype=np.uint8)
    mask[:, cfg.g1:] = 1
    conf = np.full((B, G), 2.0, dtype=np.float32)
    for b in range(B):
        pos = rng.choice(G, size=min(cfg.n_masked, G), replace=False)
        mask[b, cfg.g0 + pos] = 1
        if cfg.conf_dist == "uniform":
            vals = rng.uniform(0.0, 1.0, size=pos.size)
        elif cfg.conf_dist == "beta25":
            vals = rng.beta(2.0, 5.0, size=pos.size)
        else:
            raise ValueError(cfg.conf_dist)
        conf[b, pos] = vals.astype(np.float32)
    n_pl = cfg.n_planted_sinks
    if n_pl > 0:
        extra = rng.choice(np.arange(1, cfg.P), size=n_pl - 1, replace=False)
        sink_pos = np.sort(np.concatenate([[0], extra])).astype(np.int64)
    else:
        sink_pos = np.zeros(0, dtype=np.int64)
    return StepState(mask=mask, conf_prev=conf, sink_pos=sink_pos)


def _layer_seed(cfg: FocusConfig, layer: int, salt: int) -> int:
    return (cfg.seed * 1_000_003 + layer * 7919 + salt * 104_729) % (2**62)


def positional_basis(L: int, device) -> torch.Tensor:
    p = torch.arange(L, dtype=torch.float64, device=device)
    cols = []
    for r in range(4):
        f = float(2 ** r)
        cols.append(torch.sin(2.0 * math.pi * f * p / L))
        cols.append(torch.cos(2.0 * math.pi * f * p / L))
    return torch.stack(cols, dim=1).to(torch.float32)  # [L, 8]


def make_layer(cfg: FocusConfig, layer: int, device="cpu", sink_pos=None):
    """Q [B,Hq,L,d], K [B,Hkv,L,d], V [B,Hkv,L,d] as bf16 tensors on `device`."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(_layer_seed(cfg, layer, 1))
    B, L, d, Hq, Hkv, g = cfg.B, cfg.L, cfg.d, cfg.Hq, cfg.Hkv, cfg.group
    Q = torch.randn((B, Hq, L, d), generator=gen, device=device, dtype=torch.float32)
    K = torch.randn((B, Hkv, L, d), generator=gen, device=device, dtype=torch.float32)
    V = torch.randn((B, Hkv, L, d), generator=gen, device=device, dtype=torch.float32)
    if cfg.positional:
        a = torch.randn((Hkv, 8, d), generator=gen, device=device, dtype=torch.float32)
        phi = positional_basis(L, device)                       # [L, 8]
        pos = 0.5 * torch.einsum("lj,hjd->hld", phi, a)           # [Hkv, L, d]
        K += pos.unsqueeze(0)
        Q += pos.repeat_interleave(g, dim=0).unsqueeze(0)
    if sink_pos is None:
        sink_pos = step_state(cfg).sink_pos
    if len(sink_pos) > 0:
        sp = torch.as_tensor(np.asarray(sink_pos), device=device, dtype=torch.long)
        for b in range(B):
            for h in range(Hkv):
                mq = Q[b, h * g:(h + 1) * g].mean(dim=(0, 1))
                nrm = torch.linalg.vector_norm(mq)
                if float(nrm) == 0.0:
                    mq = torch.randn((d,), generator=gen, device=device)
                    nrm = torch.linalg.vector_norm(mq)
                u = math.sqrt(d) * mq / nrm
                K[b, h, sp] += 3.0 * u
    return (Q.to(torch.bfloat16).contiguous(), K.to(torch.bfloat16).contiguous(),
            V.to(torch.bfloat16).contiguous())


def random_bf16(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(seed)
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * scale
    return x.to(torch.bfloat16).contiguous()


def random_f32(shape, seed: int, device="cpu", lo=0.0, hi=1.0) -> torch.Tensor:
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(seed)
    x = torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    return (lo + (hi - lo) * x).contiguous()


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32 tensor to a float64 numpy array on the host."""
    return t.detach().to("cpu").to(torch.float64).numpy()
