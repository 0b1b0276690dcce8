"""Exact, IO-aware tiled attention (forward and backward) for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libattn.so`` (hand-written CUDA,
declared in ``include/attn.h``); ``exact_io_aware_58_b200.attn`` is a thin
ctypes binding over it.  PyTorch only provides device memory and streams.
"""

__version__ = "0.1.0"
