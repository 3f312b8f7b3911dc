"""The C-ABI library loads and exports every entry point include/focus.h declares (CPU only).

No compute call is made here: calls that need a GPU are in the gpu-marked tests. The
argument checks that run before any CUDA call are exercised with null pointers.
"""
import ctypes

import pytest

from diffusion_long_context_b200 import build as focus_build


@pytest.fixture(scope="module")
def F():
    focus_build.build()
    from diffusion_long_context_b200 import focus
    return focus


EXPECTED = {
    "focus_status_string", "focus_last_error", "focus_launch_count", "focus_device_error",
    "focus_select_queries", "focus_gather_rows", "focus_block_means", "focus_block_select",
    "focus_dense_attention", "focus_dense_workspace_bytes", "focus_sink_identify",
    "focus_sparse_attention", "focus_sparse_workspace_bytes",
}


def test_header_declares_the_six_calls(F):
    names = set(F.header_symbols())
    assert EXPECTED <= names
    for call in ("focus_select_queries", "focus_block_means", "focus_block_select",
                 "focus_sink_identify", "focus_sparse_attention", "focus_dense_attention"):
        assert call in names


def test_library_exports_every_declared_symbol(F):
    lib = ctypes.CDLL(F.LIB_PATH)
    for name in F.header_symbols():
        assert hasattr(lib, name), f"{name} declared in focus.h but not exported"


def test_status_strings(F):
    assert F.lib.focus_status_string(0) == b"FOCUS_OK"
    assert F.lib.focus_status_string(-1) == b"FOCUS_ERR_INVALID_ARG"
    assert F.lib.focus_status_string(-4) == b"FOCUS_ERR_CAPACITY"
    assert F.lib.focus_status_string(12345) == b"FOCUS_ERR_UNKNOWN"


def test_invalid_arguments_are_rejected_before_any_launch(F):
    lib = F.lib
    before = lib.focus_launch_count()
    # null pointers
    assert lib.focus_select_queries(None, None, 1, 8, 0, 4, 1, 1.0, 1, None, None, 1, None, None, 4, None) == -1
    assert b"null" in lib.focus_last_error()
    fake = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    # g1 > L
    assert lib.focus_select_queries(fake, fake, 1, 8, 0, 9, 1, 1.0, 1, fake, fake, 1, fake, fake, 4, None) == -1
    # capacity: k = floor(4*2) = 8 > kcap = 2
    assert lib.focus_select_queries(fake, fake, 1, 64, 0, 32, 2, 4.0, 1, fake, fake, 2, fake, fake, 32, None) == -4
    # head dim 96 unsupported
    assert lib.focus_block_means(fake, 1, 1, 64, 96, 64, 8, fake, None) == -2
    # Hq not a multiple of Hkv
    assert lib.focus_dense_attention(fake, None, fake, fake, 1, 6, 4, 64, 128, 8, 0.1, fake, None, None, 0,
                                     None) == -1
    # P > g0 in the sparse call
    assert lib.focus_sparse_attention(fake, fake, fake, fake, fake, 4, fake, 4, 64, 200, 100, 132, 1, 4, 4, 256,
                                      128, 32, 0.1, fake, None, 0, None) == -1
    # unaligned tensor
    assert lib.focus_block_means(ctypes.c_void_p(258), 1, 1, 64, 128, 64, 8, fake, None) == -1
    assert lib.focus_launch_count() == before
