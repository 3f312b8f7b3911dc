"""Thin ctypes binding of libfocus.so (argument marshalling only).

Every function here has the name of the C entry point it calls and takes torch tensors
that already live on the GPU; it checks dtype / shape / contiguity, passes raw device
pointers and the current (or given) CUDA stream, and raises FocusError on a non-zero
status. All arithmetic happens in the library's kernels. Importing this module loads
the library and raises ImportError when it has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfocus.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "focus.h")


class FocusError(RuntimeError):
    pass


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m diffusion_long_context_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_i, _f, _p, _sz, _u64 = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64
_SIGS = {
    "focus_status_string": (ctypes.c_char_p, [_i]),
    "focus_last_error": (ctypes.c_char_p, []),
    "focus_launch_count": (_u64, []),
    "focus_device_error": (_i, [ctypes.POINTER(ctypes.c_int)]),
    "focus_select_queries": (_i, [_p, _p, _i, _i, _i, _i, _i, _f, _i, _p, _p, _i, _p, _p, _i, _p]),
    "focus_gather_rows": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p]),
    "focus_scatter_rows": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p]),
    "focus_block_means": (_i, [_p, _i, _i, _i, _i, _i, _i, _p, _p]),
    "focus_block_select": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "focus_dense_attention": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _sz, _p]),
    "focus_dense_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "focus_dense_attention_sinks": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _i, _p, _p, _sz, _p]),
    "focus_full_refresh": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _f, _p, _i, _i, _p, _p, _sz, _p]),
    "focus_sink_identify": (_i, [_p, _i, _i, _i, _i, _p, _p]),
    "focus_sparse_attention": (_i, [_p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                    _p, _p, _sz, _p]),
    "focus_sparse_workspace_bytes": (_sz, [_i] * 12),
    "focus_sparse_attention_noalloc": (_i, [_p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                            _i, _f, _p, _p]),
    "focus_sparse_attention_fused": (_i, [_p, _p, _p, _p, _p, _i, _i, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                          _i, _f, _p, _p, _p, _sz, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_symbols():
    """Names of the entry points declared in include/focus.h."""
    with open(HEADER_PATH) as f:
        return re.findall(r"FOCUS_API\s+[\w\s\*]+?\b(focus_\w+)\s*\(", f.read())


def launch_count() -> int:
    return int(lib.focus_launch_count())


def last_error() -> str:
    return lib.focus_last_error().decode()


def device_error() -> int:
    """Synchronises, returns and clears the device error word (0 = none)."""
    code = ctypes.c_int(0)
    st = lib.focus_device_error(ctypes.byref(code))
    if st not in (0, -5):
        raise FocusError(f"focus_device_error: {last_error()}")
    return code.value


def _check(status: int, name: str):
    if status != 0:
        raise FocusError(f"{name}: {lib.focus_status_string(status).decode()}: {last_error()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


# ----------------------------------------------------------------------------- calls
def focus_select_queries(conf_prev, mask, g0, g1, n_t, rho, w, i_focus, n_focus, i_active, n_active, stream=None):
    _need(conf_prev, torch.float32, "conf_prev", 2)
    _need(mask, torch.uint8, "mask", 2)
    for t, n in ((i_focus, "i_focus"), (n_focus, "n_focus"), (i_active, "i_active"), (n_active, "n_active")):
        _need(t, torch.int32, n)
    B, L = mask.shape
    st = lib.focus_select_queries(_ptr(conf_prev), _ptr(mask), B, L, g0, g1, n_t, float(rho), w, _ptr(i_focus),
                                  _ptr(n_focus), i_focus.shape[-1], _ptr(i_active), _ptr(n_active),
                                  i_active.shape[-1], _stream(stream))
    _check(st, "focus_select_queries")


def focus_gather_rows(X, rows, n_rows, X_rows, stream=None):
    """X [n_mat, B, H, L, d] (or [B, H, L, d]) -> X_rows [..., cap, d]."""
    _need(X, torch.bfloat16, "X")
    _need(X_rows, torch.bfloat16, "X_rows")
    _need(rows, torch.int32, "rows", 2)
    _need(n_rows, torch.int32, "n_rows", 1)
    x = X if X.dim() == 5 else X.unsqueeze(0)
    n_mat, B, H, L, d = x.shape
    cap = rows.shape[1]
    st = lib.focus_gather_rows(_ptr(X), _ptr(rows), _ptr(n_rows), n_mat, B, H, L, d, cap, _ptr(X_rows),
                               _stream(stream))
    _check(st, "focus_gather_rows")


def focus_scatter_rows(X, rows, n_rows, X_rows, stream=None):
    """Approximate-KV-cache refresh: X[..., rows[b, i], :] = X_rows[..., i, :] for i < n_rows[b].

    X [n_mat, B, H, L, d] (or [B, H, L, d]) is updated in place from X_rows [..., cap, d]."""
    _need(X, torch.bfloat16, "X")
    _need(X_rows, torch.bfloat16, "X_rows")
    _need(rows, torch.int32, "rows", 2)
    _need(n_rows, torch.int32, "n_rows", 1)
    x = X if X.dim() == 5 else X.unsqueeze(0)
    n_mat, B, H, L, d = x.shape
    cap = rows.shape[1]
    st = lib.focus_scatter_rows(_ptr(X), _ptr(rows), _ptr(n_rows), n_mat, B, H, L, d, cap, _ptr(X_rows),
                                _stream(stream))
    _check(st, "focus_scatter_rows")


def focus_block_means(K, P, bs, kbar, stream=None):
    _need(K, torch.bfloat16, "K", 4)
    _need(kbar, torch.float32, "kbar", 4)
    B, Hkv, L, d = K.shape
    st = lib.focus_block_means(_ptr(K), B, Hkv, L, d, P, bs, _ptr(kbar), _stream(stream))
    _check(st, "focus_block_means")


def focus_block_select(Q_active, n_active, kbar, C, blocks, scores=None, stream=None):
    _need(Q_active, torch.bfloat16, "Q_active", 4)
    _need(n_active, torch.int32, "n_active", 1)
    _need(kbar, torch.float32, "kbar", 4)
    _need(blocks, torch.int32, "blocks", 3)
    if scores is not None:
        _need(scores, torch.float32, "scores", 3)
    B, Hq, acap, d = Q_active.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    st = lib.focus_block_select(_ptr(Q_active), _ptr(n_active), _ptr(kbar), B, Hq, Hkv, d, acap, nb, C,
                                _ptr(blocks), _ptr(scores), _stream(stream))
    _check(st, "focus_block_select")


def dense_workspace_bytes(B, Hq, Hkv, L, d, qcap, want_colsum):
    return int(lib.focus_dense_workspace_bytes(B, Hq, Hkv, L, d, qcap, 1 if want_colsum else 0))


def sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1):
    return int(lib.focus_sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1))


def _workspace(nbytes, device, ws):
    if nbytes == 0:
        return None, 0
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace needs {nbytes} bytes")
        return ws, ws.numel() * ws.element_size()
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def focus_dense_attention(Q, n_q, K, V, O, scale=None, colsum=None, ws=None, stream=None):
    _need(Q, torch.bfloat16, "Q", 4)
    _need(K, torch.bfloat16, "K", 4)
    _need(V, torch.bfloat16, "V", 4)
    _need(O, torch.bfloat16, "O", 4)
    if n_q is not None:
        _need(n_q, torch.int32, "n_q", 1)
    if colsum is not None:
        _need(colsum, torch.float32, "colsum", 3)
    B, Hq, qcap, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = dense_workspace_bytes(B, Hq, Hkv, L, d, qcap, colsum is not None)
    ws, ws_bytes = _workspace(need, Q.device, ws)
    st = lib.focus_dense_attention(_ptr(Q), _ptr(n_q), _ptr(K), _ptr(V), B, Hq, Hkv, L, d, qcap, float(scale),
                                   _ptr(O), _ptr(colsum), _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "focus_dense_attention")


def focus_dense_attention_sinks(Q, n_q, K, V, O, colsum, sinks, scale=None, ws=None, stream=None):
    """The sink layer: dense attention, column sums and the top-S sinks (S = sinks.shape[2])."""
    _need(Q, torch.bfloat16, "Q", 4)
    _need(K, torch.bfloat16, "K", 4)
    _need(V, torch.bfloat16, "V", 4)
    _need(O, torch.bfloat16, "O", 4)
    _need(colsum, torch.float32, "colsum", 3)
    _need(sinks, torch.int32, "sinks", 3)
    if n_q is not None:
        _need(n_q, torch.int32, "n_q", 1)
    B, Hq, qcap, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = dense_workspace_bytes(B, Hq, Hkv, L, d, qcap, True)
    ws, ws_bytes = _workspace(need, Q.device, ws)
    st = lib.focus_dense_attention_sinks(_ptr(Q), _ptr(n_q), _ptr(K), _ptr(V), B, Hq, Hkv, L, d, qcap, float(scale),
                                         _ptr(O), _ptr(colsum), sinks.shape[2], _ptr(sinks), _ptr(ws), ws_bytes,
                                         _stream(stream))
    _check(st, "focus_dense_attention_sinks")


def focus_full_refresh(Q, K, V, O, P, bs, kbar, scale=None, ws=None, stream=None):
    """Block entry: dense attention of every query (O [B, Hq, L, d]) and the prompt's block
    means kbar [B, Hkv, ceil(P / bs), d] fp32, in one launch where the kernel serves it."""
    _need(Q, torch.bfloat16, "Q", 4)
    _need(K, torch.bfloat16, "K", 4)
    _need(V, torch.bfloat16, "V", 4)
    _need(O, torch.bfloat16, "O", 4)
    _need(kbar, torch.float32, "kbar", 4)
    B, Hq, L, d = Q.shape
    Hkv = K.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = dense_workspace_bytes(B, Hq, Hkv, L, d, L, False)
    ws, ws_bytes = _workspace(need, Q.device, ws)
    st = lib.focus_full_refresh(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, L, d, float(scale), _ptr(O), P, bs, _ptr(kbar),
                                _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "focus_full_refresh")


def focus_sink_identify(colsum, S, sinks, stream=None):
    _need(colsum, torch.float32, "colsum", 3)
    _need(sinks, torch.int32, "sinks", 3)
    B, Hkv, L = colsum.shape
    st = lib.focus_sink_identify(_ptr(colsum), B, Hkv, L, S, _ptr(sinks), _stream(stream))
    _check(st, "focus_sink_identify")


def focus_sparse_attention(Q_active, n_active, K, V, sinks, blocks, bs, P, g0, g1, O_active, scale=None, ws=None,
                           stream=None):
    _need(Q_active, torch.bfloat16, "Q_active", 4)
    _need(n_active, torch.int32, "n_active", 1)
    _need(K, torch.bfloat16, "K", 4)
    _need(V, torch.bfloat16, "V", 4)
    _need(O_active, torch.bfloat16, "O_active", 4)
    _need(blocks, torch.int32, "blocks", 3)
    if sinks is not None:
        _need(sinks, torch.int32, "sinks", 3)
    B, Hq, acap, d = Q_active.shape
    Hkv, L = K.shape[1], K.shape[2]
    S = 0 if sinks is None else sinks.shape[2]
    C = blocks.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1)
    ws, ws_bytes = _workspace(need, Q_active.device, ws)
    st = lib.focus_sparse_attention(_ptr(Q_active), _ptr(n_active), _ptr(K), _ptr(V), _ptr(sinks), S,
                                    _ptr(blocks), C, bs, P, g0, g1, B, Hq, Hkv, L, d, acap, float(scale),
                                    _ptr(O_active), _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "focus_sparse_attention")


def focus_sparse_attention_fused(Q_active, n_active, K, V, kbar, C, sinks, bs, P, g0, g1, blocks, O_active, scale=None,
                                 ws=None, stream=None):
    """Block relevance + top-C + sparse attention of one layer (blocks receives the kept blocks)."""
    _need(Q_active, torch.bfloat16, "Q_active", 4)
    _need(n_active, torch.int32, "n_active", 1)
    _need(K, torch.bfloat16, "K", 4)
    _need(V, torch.bfloat16, "V", 4)
    _need(kbar, torch.float32, "kbar", 4)
    _need(blocks, torch.int32, "blocks", 3)
    _need(O_active, torch.bfloat16, "O_active", 4)
    if sinks is not None:
        _need(sinks, torch.int32, "sinks", 3)
    B, Hq, acap, d = Q_active.shape
    Hkv, L = K.shape[1], K.shape[2]
    nb = kbar.shape[2]
    S = 0 if sinks is None else sinks.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = sparse_workspace_bytes(B, Hq, Hkv, L, d, acap, S, C, bs, P, g0, g1)
    ws, ws_bytes = _workspace(need, Q_active.device, ws)
    st = lib.focus_sparse_attention_fused(_ptr(Q_active), _ptr(n_active), _ptr(K), _ptr(V), _ptr(kbar), nb, C,
                                          _ptr(sinks), S, bs, P, g0, g1, B, Hq, Hkv, L, d, acap, float(scale),
                                          _ptr(blocks), _ptr(O_active), _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "focus_sparse_attention_fused")
