"""B200-native (sm_100a) Focus-dLLM sparse denoising-step attention.

The compute path lives in the C-ABI library `libfocus.so` (csrc/); `focus` is its
thin ctypes binding. `configs` and `inputs` describe and draw synthetic workloads.
Importing this package does not load the CUDA library; `focus` does, and fails loudly
when it is missing.
"""
__all__ = ["configs", "inputs"]
