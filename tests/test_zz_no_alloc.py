"""The allocation-free sparse attention entry point (GPU).

focus_sparse_attention_noalloc serves callers that cannot call cudaMalloc (allocation
forbidden during stream capture, plugin enqueue paths, servers that reserve all device
memory up front): its split-KV scratch is a library-owned static device array instead of
a caller workspace. This test calls it through the C ABI (ctypes, raw device pointers)
twice in a row on different inputs and checks each output against the regular
focus_sparse_attention on the same inputs (bit for bit: the same kernels run, only the
scratch pointer differs) and against the fp64 oracle, then checks the size limit. It lives in its own
file, collected last, and passes both alone in a fresh process and after the other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from diffusion_long_context_b200 import inputs
from oracle import focus_oracle as orc
from parity_utils import assert_attention_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def F():
    from diffusion_long_context_b200 import build
    build.build()
    from diffusion_long_context_b200 import focus
    return focus


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _case(seed, B=1, Hq=16, Hkv=1, d=128, P=4096, G=32, bs=64, C=32, S=16, acap=32):
    g0, g1 = P, P + G
    L = g1 + 64
    rng = np.random.default_rng(seed)
    nb = P // bs
    blocks = np.sort(np.stack([np.stack([rng.choice(nb, C, replace=False) for _ in range(Hkv)])
                               for _ in range(B)]), axis=-1).astype(np.int32)
    sinks = np.sort(np.stack([np.stack([rng.choice(L, S, replace=False) for _ in range(Hkv)])
                              for _ in range(B)]), axis=-1).astype(np.int32)
    return dict(
        Q=inputs.random_bf16((B, Hq, acap, d), seed=seed, device=DEV),
        K=inputs.random_bf16((B, Hkv, L, d), seed=seed + 1, device=DEV),
        V=inputs.random_bf16((B, Hkv, L, d), seed=seed + 2, device=DEV),
        n=torch.tensor([acap - seed % 5] * B, dtype=torch.int32, device=DEV),
        blocks=torch.from_numpy(blocks).to(DEV), sinks=torch.from_numpy(sinks).to(DEV),
        sizes=(S, C, bs, P, g0, g1, B, Hq, Hkv, L, d, acap))


def _noalloc(F, c, O, stream):
    S, C, bs, P, g0, g1, B, Hq, Hkv, L, d, acap = c["sizes"]
    return F.lib.focus_sparse_attention_noalloc(
        _p(c["Q"]), _p(c["n"]), _p(c["K"]), _p(c["V"]), _p(c["sinks"]), S, _p(c["blocks"]), C, bs, P, g0, g1, B,
        Hq, Hkv, L, d, acap, ctypes.c_float(1.0 / math.sqrt(d)), _p(O), ctypes.c_void_p(stream.cuda_stream))


def test_noalloc_matches_the_workspace_entry_point_twice(F):
    stream = torch.cuda.current_stream()
    # 16 query heads x 32 queries on one KV head (512 rows): the 128-row tile kernel with
    # split-KV partials in the scratch array
    for seed in (11, 12):                                  # two calls in a row, different inputs
        c = _case(seed)
        S, C, bs, P, g0, g1, B, Hq, Hkv, L, d, acap = c["sizes"]
        assert F.sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1) > 0, \
            "the case must exercise the split-KV scratch"
        O_ref = torch.zeros((B, Hq, acap, d), dtype=torch.bfloat16, device=DEV)
        F.focus_sparse_attention(c["Q"], c["n"], c["K"], c["V"], c["sinks"], c["blocks"], bs, P, g0, g1, O_ref)
        O = torch.full((B, Hq, acap, d), 5.0, dtype=torch.bfloat16, device=DEV)
        st = _noalloc(F, c, O, stream)
        assert st == 0, F.last_error()
        torch.cuda.synchronize()
        assert torch.isfinite(O.float()).all()
        assert torch.equal(O, O_ref), "same kernels, other scratch: the outputs must be identical"
        nA = c["n"].cpu().tolist()
        O_orc = orc.sparse_attention(inputs.to_f64(c["Q"]), nA, inputs.to_f64(c["K"]), inputs.to_f64(c["V"]),
                                     c["sinks"].cpu().numpy(), c["blocks"].cpu().numpy(), bs, P, g0, g1,
                                     float(np.float32(1.0 / math.sqrt(d))))
        assert_attention_close(O, O_orc, rows_valid=nA, what=f"noalloc call seed {seed}")
    assert F.device_error() == 0


def test_noalloc_rejects_sizes_beyond_the_static_array(F):
    # 1024 query rows of one head: 18 splits x 1024 rows x 128 x 4 B > 8 MiB of partials
    c = _case(3, Hq=1, Hkv=1, acap=1024, C=64, S=8)
    S, C, bs, P, g0, g1, B, Hq, Hkv, L, d, acap = c["sizes"]
    need = F.sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1)
    if need <= (8 << 20):
        pytest.skip(f"this device plans only {need} bytes of partials for the oversized case")
    O = torch.zeros((B, Hq, acap, d), dtype=torch.bfloat16, device=DEV)
    before = F.launch_count()
    assert _noalloc(F, c, O, torch.cuda.current_stream()) == -4          # FOCUS_ERR_CAPACITY
    assert "exceeds" in F.last_error()
    assert F.launch_count() == before
