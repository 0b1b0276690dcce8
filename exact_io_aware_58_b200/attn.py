"""Thin ctypes binding over libattn.so (the C ABI in include/attn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libattn.so.  PyTorch supplies device memory and the stream.  If the
library is missing the import of a compute entry point fails loudly; there is
no fallback path.

Raw entry points keep the C names and argument order (``attn_fwd``,
``attn_bwd``, ``attn_bwd_deterministic``, ``attn_bwd_workspace_bytes``,
``attn_check_status``, ``attn_status_string``); ``forward`` / ``backward``
allocate the outputs with torch and call them.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

from .build import LIB_PATH

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_MISALIGNED = -3
ATTN_ERR_WORKSPACE = -4
ATTN_ERR_LAUNCH = -5
ATTN_ERR_TIMEOUT = -6
ATTN_ERR_DEVICE = -7

EXPORTED = ("attn_fwd", "attn_fwd_f32out", "attn_fwd_gqa", "attn_fwd_blocksparse", "attn_fwd_varlen", "attn_bwd",
            "attn_bwd_gqa",
            "attn_bwd_blocksparse", "attn_bwd_deterministic", "attn_bwd_workspace_bytes",
            "attn_bwd_deterministic_workspace_bytes", "attn_fwd_fp8", "attn_fwd_kvcache", "attn_fwd_kvcache_fp8",
            "attn_fwd_kvcache_splits", "attn_fwd_kvcache_workspace_bytes",
            "attn_bwd_fused_preprocess", "attn_bwd_fused_dkdvdq", "attn_bwd_fused_dq_convert",
            "attn_bwd_preprocess", "attn_bwd_dkdv",
            "attn_bwd_dq", "attn_bwd_static_workspace", "attn_check_status", "attn_last_error",
            "attn_selftest_wait_timeout",
            "attn_status_string")

# Size of the library-owned workspace used by attn_bwd_static_workspace (bytes).
ATTN_STATIC_WORKSPACE_BYTES = 32 * 1024 * 1024


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = attn_last_error()
        super().__init__(f"{where}: {attn_status_string(status)} ({status})" + (f": {detail}" if detail else ""))


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libattn.so and declare the C signatures (once)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m exact_io_aware_58_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(path)
    i64, vp, f32, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_int
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp]
    lib.attn_fwd_f32out.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp]
    lib.attn_fwd_f32out.restype = i32
    lib.attn_fwd.restype = i32
    lib.attn_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, vp]
    lib.attn_fwd_gqa.restype = i32
    lib.attn_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, vp,
                                 ctypes.c_size_t, vp]
    lib.attn_bwd_gqa.restype = i32
    lib.attn_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, vp]
    lib.attn_fwd_blocksparse.restype = i32
    lib.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, vp]
    lib.attn_fwd_varlen.restype = i32
    lib.attn_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32,
                                         vp, ctypes.c_size_t, vp]
    lib.attn_bwd_blocksparse.restype = i32
    lib.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, f32, f32, f32, vp]
    lib.attn_fwd_fp8.restype = i32
    lib.attn_fwd_kvcache.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i32, f32, i64, vp,
                                     ctypes.c_size_t, vp]
    lib.attn_fwd_kvcache.restype = i32
    lib.attn_fwd_kvcache_fp8.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i32, f32, f32, f32,
                                         i64, vp, ctypes.c_size_t, vp]
    lib.attn_fwd_kvcache_fp8.restype = i32
    lib.attn_fwd_kvcache_splits.argtypes = [i64] * 7
    lib.attn_fwd_kvcache_splits.restype = i64
    lib.attn_fwd_kvcache_workspace_bytes.argtypes = [i64] * 7
    lib.attn_fwd_kvcache_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_deterministic_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.attn_bwd_deterministic_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, f32, vp,
                                           ctypes.c_size_t, vp]
    lib.attn_bwd_deterministic.restype = i32
    lib.attn_bwd_fused_preprocess.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, ctypes.c_size_t, vp]
    lib.attn_bwd_fused_preprocess.restype = i32
    lib.attn_bwd_fused_dkdvdq.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp,
                                          ctypes.c_size_t, vp]
    lib.attn_bwd_fused_dkdvdq.restype = i32
    lib.attn_bwd_fused_dq_convert.argtypes = [vp, i64, i64, i64, i64, f32, vp, ctypes.c_size_t, vp]
    lib.attn_bwd_fused_dq_convert.restype = i32
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp,
                             ctypes.c_size_t, vp]
    lib.attn_bwd.restype = i32
    lib.attn_bwd_preprocess.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, ctypes.c_size_t, vp]
    lib.attn_bwd_preprocess.restype = i32
    lib.attn_bwd_dkdv.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp, ctypes.c_size_t, vp]
    lib.attn_bwd_dkdv.restype = i32
    lib.attn_bwd_dq.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp, ctypes.c_size_t, vp]
    lib.attn_bwd_dq.restype = i32
    lib.attn_bwd_static_workspace.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, f32, vp]
    lib.attn_bwd_static_workspace.restype = i32
    lib.attn_selftest_wait_timeout.argtypes = [vp]
    lib.attn_selftest_wait_timeout.restype = i32
    lib.attn_check_status.argtypes = [vp]
    lib.attn_check_status.restype = i32
    lib.attn_last_error.argtypes = []
    lib.attn_last_error.restype = ctypes.c_char_p
    lib.attn_status_string.argtypes = [i32]
    lib.attn_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def attn_status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()


def attn_last_error() -> str:
    return load_library().attn_last_error().decode()


# The current stream's raw handle without building a torch.cuda.Stream object
# (the public call costs a few microseconds per launch); None on builds without it.
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        if _raw_current_stream is not None:
            return ctypes.c_void_p(_raw_current_stream(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _check_device(name: str, t: torch.Tensor):
    # The library launches on the calling thread's current device (and takes
    # its workspace and default stream from there): every tensor must live on it.
    if t.is_cuda and t.get_device() != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}; call under torch.cuda.device({t.device})")


def _check_bhnd(name: str, t: torch.Tensor, shape=None):
    if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape (B, H, N, d)")
    _check_device(name, t)
    if shape is not None and t.shape != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_lse(t: torch.Tensor, shape):
    B, H, N, _ = shape
    if not t.is_cuda or t.dtype != torch.float32 or t.shape != (B, H, N) or not t.is_contiguous():
        raise ValueError("LSE must be a contiguous CUDA float32 tensor of shape (B, H, N)")
    _check_device("LSE", t)


def attn_fwd(Q, K, V, O, LSE, causal: bool, scale: float, stream=None) -> None:
    """O, LSE <- attention(Q, K, V); all tensors preallocated on the device."""
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("O", O)):
        _check_bhnd(n, t, Q.shape)
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    st = load_library().attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, N, d, int(bool(causal)),
                                 float(scale), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd")


def attn_fwd_f32out(Q, K, V, O, O32, LSE, causal: bool, scale: float, stream=None) -> None:
    """attn_fwd that also writes O32 (fp32, same shape as O): the normalised rows before their bf16 rounding."""
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("O", O)):
        _check_bhnd(n, t, Q.shape)
    if not O32.is_cuda or O32.dtype != torch.float32 or tuple(O32.shape) != tuple(Q.shape) or not O32.is_contiguous():
        raise ValueError("O32 must be a contiguous CUDA fp32 tensor shaped like Q")
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    st = load_library().attn_fwd_f32out(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(O32), _ptr(LSE), B, H, N, d,
                                        int(bool(causal)), float(scale), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_f32out")


def _check_kv(name: str, t: torch.Tensor, q_shape):
    B, H, N, d = q_shape
    if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape (B, H_kv, N, d)")
    _check_device(name, t)
    Hk = t.shape[1]
    if t.shape[0] != B or t.shape[2] != N or t.shape[3] != d or Hk < 1 or H % Hk != 0:
        raise ValueError(f"{name} has shape {tuple(t.shape)}; expected (B, H_kv, N, d) with H % H_kv == 0")
    return Hk


def attn_fwd_gqa(Q, K, V, O, LSE, causal: bool, scale: float, stream=None) -> None:
    """attn_fwd with K, V of shape (B, H_kv, N, d) shared by groups of H / H_kv query heads."""
    _check_bhnd("Q", Q)
    _check_bhnd("O", O, Q.shape)
    Hk = _check_kv("K", K, Q.shape)
    if _check_kv("V", V, Q.shape) != Hk:
        raise ValueError("K and V must have the same number of heads")
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    st = load_library().attn_fwd_gqa(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, Hk, N, d,
                                     int(bool(causal)), float(scale), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_gqa")


def attn_bwd_gqa(Q, K, V, O, dO, LSE, dQ, dK, dV, causal: bool, scale: float, workspace, stream=None) -> None:
    """attn_bwd with K, V, dK, dV of shape (B, H_kv, N, d)."""
    _check_bhnd("Q", Q)
    for n, t in (("O", O), ("dO", dO), ("dQ", dQ)):
        _check_bhnd(n, t, Q.shape)
    Hk = _check_kv("K", K, Q.shape)
    for n, t in (("V", V), ("dK", dK), ("dV", dV)):
        if _check_kv(n, t, Q.shape) != Hk:
            raise ValueError(f"{n} must have the same number of heads as K")
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_gqa(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE), _ptr(dQ), _ptr(dK),
                                     _ptr(dV), B, H, Hk, N, d, int(bool(causal)), float(scale), wp, wb,
                                     _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_gqa")


def _check_mask(mask, B, H, N):
    nt = (N + 127) // 128
    if not mask.is_cuda or mask.dtype != torch.uint8 or not mask.is_contiguous() or \
            tuple(mask.shape) != (B, H, nt, nt):
        raise ValueError(f"block_mask must be a contiguous CUDA uint8 tensor of shape {(B, H, nt, nt)}")


def attn_fwd_blocksparse(Q, K, V, O, LSE, block_mask, causal: bool, scale: float, stream=None) -> None:
    """attn_fwd over the 128x128 blocks selected by block_mask (B, H, ceil(N/128), ceil(N/128))."""
    _check_bhnd("Q", Q)
    _check_bhnd("O", O, Q.shape)
    Hk = _check_kv("K", K, Q.shape)
    if _check_kv("V", V, Q.shape) != Hk:
        raise ValueError("K and V must have the same number of heads")
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    _check_mask(block_mask, B, H, N)
    st = load_library().attn_fwd_blocksparse(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(block_mask), B, H,
                                             Hk, N, d, int(bool(causal)), float(scale), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_blocksparse")


def attn_fwd_varlen(Q, K, V, O, LSE, cu_seqlens, causal: bool, scale: float, stream=None) -> None:
    """Packed sequences: Q, O (total, H, d), K, V (total, H_kv, d) bf16, LSE (H, total) fp32,
    cu_seqlens int32 (n_seqs + 1,) token offsets, all on the current CUDA device."""
    for name, t in (("Q", Q), ("K", K), ("V", V), ("O", O)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape (total, heads, d)")
        _check_device(name, t)
    total, H, d = Q.shape
    if tuple(O.shape) != tuple(Q.shape):
        raise ValueError("O must have Q's shape")
    if K.shape != V.shape or K.shape[0] != total or K.shape[2] != d or K.shape[1] < 1 or H % K.shape[1] != 0:
        raise ValueError(f"K, V have shapes {tuple(K.shape)}, {tuple(V.shape)}; expected (total, H_kv, d)")
    if not LSE.is_cuda or LSE.dtype != torch.float32 or tuple(LSE.shape) != (H, total) or not LSE.is_contiguous():
        raise ValueError("LSE must be a contiguous CUDA float32 tensor of shape (H, total)")
    _check_device("LSE", LSE)
    if not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 \
            or cu_seqlens.numel() < 2 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous CUDA int32 tensor of shape (n_seqs + 1,)")
    _check_device("cu_seqlens", cu_seqlens)
    st = load_library().attn_fwd_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(cu_seqlens),
                                        cu_seqlens.numel() - 1, total, H, K.shape[1], d, int(bool(causal)),
                                        float(scale), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_varlen")


def attn_bwd_blocksparse(Q, K, V, O, dO, LSE, block_mask, dQ, dK, dV, causal: bool, scale: float, workspace,
                         stream=None) -> None:
    """Backward of attn_fwd_blocksparse."""
    _check_bhnd("Q", Q)
    for n, t in (("O", O), ("dO", dO), ("dQ", dQ)):
        _check_bhnd(n, t, Q.shape)
    Hk = _check_kv("K", K, Q.shape)
    for n, t in (("V", V), ("dK", dK), ("dV", dV)):
        if _check_kv(n, t, Q.shape) != Hk:
            raise ValueError(f"{n} must have the same number of heads as K")
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    _check_mask(block_mask, B, H, N)
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_blocksparse(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE),
                                             _ptr(block_mask), _ptr(dQ), _ptr(dK), _ptr(dV), B, H, Hk, N, d,
                                             int(bool(causal)), float(scale), wp, wb, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_blocksparse")


def attn_fwd_fp8(Q8, K8, V8, O, LSE, causal: bool, scale: float, q_descale: float, k_descale: float,
                 v_descale: float, stream=None) -> None:
    """O (bf16), LSE <- attention of the dequantised E4M3 tensors descale * X8.

    Q8 (B, H, N, 128) and K8, V8 (B, H_kv, N, 128) are torch.float8_e4m3fn
    (or uint8 holding E4M3 codes) CUDA tensors; O is bf16 (B, H, N, 128).
    """
    for name, t in (("Q8", Q8), ("K8", K8), ("V8", V8)):
        if not t.is_cuda or t.dtype not in (torch.float8_e4m3fn, torch.uint8) or t.dim() != 4 \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA float8_e4m3fn (or uint8) tensor of rank 4")
    _check_bhnd("O", O, Q8.shape)
    _check_lse(LSE, Q8.shape)
    B, H, N, d = Q8.shape
    if K8.shape != V8.shape or K8.shape[0] != B or K8.shape[2] != N or K8.shape[3] != d or K8.shape[1] < 1 \
            or H % K8.shape[1] != 0:
        raise ValueError(f"K8, V8 have shapes {tuple(K8.shape)}, {tuple(V8.shape)}; expected (B, H_kv, N, d)")
    st = load_library().attn_fwd_fp8(_ptr(Q8), _ptr(K8), _ptr(V8), _ptr(O), _ptr(LSE), B, H, K8.shape[1], N, d,
                                     int(bool(causal)), float(scale), float(q_descale), float(k_descale),
                                     float(v_descale), _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")


def attn_fwd_kvcache_splits(B: int, H: int, H_kv: int, Nq: int, Nk: int, d: int, num_splits: int = 0) -> int:
    return int(load_library().attn_fwd_kvcache_splits(B, H, H_kv, Nq, Nk, d, num_splits))


def attn_fwd_kvcache_workspace_bytes(B: int, H: int, H_kv: int, Nq: int, Nk: int, d: int,
                                     num_splits: int = 0) -> int:
    return int(load_library().attn_fwd_kvcache_workspace_bytes(B, H, H_kv, Nq, Nk, d, num_splits))


def attn_fwd_kvcache(Q, K, V, O, LSE, kv_lens, causal: bool, scale: float, num_splits: int = 0, workspace=None,
                     stream=None) -> None:
    """O, LSE <- attention of Q (B, H, Nq, d) against the cache K, V (B, H_kv, Nk, d).

    kv_lens: int32 CUDA tensor (B,) of valid cache lengths, or None (all Nk).
    workspace: CUDA tensor of at least attn_fwd_kvcache_workspace_bytes() bytes
    when more than one split is used (None allowed with one split).
    """
    _check_bhnd("Q", Q)
    _check_bhnd("O", O, Q.shape)
    _check_lse(LSE, Q.shape)
    B, H, Nq, d = Q.shape
    for name, t in (("K", K), ("V", V)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape (B, H_kv, Nk, d)")
    if K.shape != V.shape or K.shape[0] != B or K.shape[3] != d or K.shape[1] < 1 or H % K.shape[1] != 0:
        raise ValueError(f"K, V have shapes {tuple(K.shape)}, {tuple(V.shape)}; expected (B, H_kv, Nk, d)")
    Hk, Nk = K.shape[1], K.shape[2]
    if kv_lens is not None and (not kv_lens.is_cuda or kv_lens.dtype != torch.int32 or tuple(kv_lens.shape) != (B,)
                                or not kv_lens.is_contiguous()):
        raise ValueError("kv_lens must be a contiguous CUDA int32 tensor of shape (B,)")
    wp, wb = (ctypes.c_void_p(None), 0) if workspace is None else _ws(workspace)
    st = load_library().attn_fwd_kvcache(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE),
                                         ctypes.c_void_p(None) if kv_lens is None else _ptr(kv_lens),
                                         B, H, Hk, Nq, Nk, d, int(bool(causal)), float(scale), int(num_splits),
                                         wp, wb, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_kvcache")


def attn_fwd_kvcache_fp8(Q, K8, V8, O, LSE, kv_lens, causal: bool, scale: float, k_descale: float,
                         v_descale: float, num_splits: int = 0, workspace=None, stream=None) -> None:
    """attn_fwd_kvcache with an E4M3 cache: K8, V8 (B, H_kv, Nk, 128) float8_e4m3fn or uint8 CUDA tensors."""
    _check_bhnd("Q", Q)
    _check_bhnd("O", O, Q.shape)
    _check_lse(LSE, Q.shape)
    B, H, Nq, d = Q.shape
    for name, t in (("K8", K8), ("V8", V8)):
        if not t.is_cuda or t.dtype not in (torch.float8_e4m3fn, torch.uint8) or t.dim() != 4 \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA float8_e4m3fn (or uint8) tensor of rank 4")
    if K8.shape != V8.shape or K8.shape[0] != B or K8.shape[3] != d or K8.shape[1] < 1 or H % K8.shape[1] != 0:
        raise ValueError(f"K8, V8 have shapes {tuple(K8.shape)}, {tuple(V8.shape)}; expected (B, H_kv, Nk, d)")
    if kv_lens is not None and (not kv_lens.is_cuda or kv_lens.dtype != torch.int32 or tuple(kv_lens.shape) != (B,)
                                or not kv_lens.is_contiguous()):
        raise ValueError("kv_lens must be a contiguous CUDA int32 tensor of shape (B,)")
    if workspace is None:
        raise ValueError("attn_fwd_kvcache_fp8 needs a workspace (attn_fwd_kvcache_workspace_bytes)")
    wp, wb = _ws(workspace)
    st = load_library().attn_fwd_kvcache_fp8(_ptr(Q), _ptr(K8), _ptr(V8), _ptr(O), _ptr(LSE),
                                             ctypes.c_void_p(None) if kv_lens is None else _ptr(kv_lens),
                                             B, H, K8.shape[1], Nq, K8.shape[2], d, int(bool(causal)), float(scale),
                                             float(k_descale), float(v_descale), int(num_splits), wp, wb,
                                             _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_kvcache_fp8")


def attn_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_bwd_workspace_bytes(B, H, N, d))


def attn_bwd_deterministic_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().attn_bwd_deterministic_workspace_bytes(B, H, N, d))


def attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, causal: bool, scale: float, workspace, stream=None) -> None:
    """dQ, dK, dV <- backward of attention (one pass over the key tiles; dQ
    summed in an fp32 workspace accumulator); all tensors preallocated on the device."""
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("O", O), ("dO", dO), ("dQ", dQ), ("dK", dK), ("dV", dV)):
        _check_bhnd(n, t, Q.shape)
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE), _ptr(dQ), _ptr(dK),
                                 _ptr(dV), B, H, N, d, int(bool(causal)), float(scale), wp, wb,
                                 _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd")


def attn_bwd_deterministic(Q, K, V, O, dO, LSE, dQ, dK, dV, causal: bool, scale: float, workspace,
                           stream=None) -> None:
    """The bitwise-reproducible backward (separate dK/dV and dQ kernels); K, V,
    dK, dV may have H_kv heads (B, H_kv, N, d)."""
    _check_bhnd("Q", Q)
    for n, t in (("O", O), ("dO", dO), ("dQ", dQ)):
        _check_bhnd(n, t, Q.shape)
    Hk = _check_kv("K", K, Q.shape)
    for n, t in (("V", V), ("dK", dK), ("dV", dV)):
        if _check_kv(n, t, Q.shape) != Hk:
            raise ValueError(f"{n} must have the same number of heads as K")
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_deterministic(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE), _ptr(dQ),
                                               _ptr(dK), _ptr(dV), B, H, Hk, N, d, int(bool(causal)), float(scale),
                                               wp, wb, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_deterministic")


def attn_bwd_static_workspace(Q, K, V, O, dO, LSE, dQ, dK, dV, causal: bool, scale: float, stream=None) -> None:
    """attn_bwd without a caller workspace: for callers that cannot allocate
    device memory; the library's fixed device array (ATTN_STATIC_WORKSPACE_BYTES)
    is used instead.  Calls that overlap on the GPU race on that array."""
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("O", O), ("dO", dO), ("dQ", dQ), ("dK", dK), ("dV", dV)):
        _check_bhnd(n, t, Q.shape)
    _check_lse(LSE, Q.shape)
    B, H, N, d = Q.shape
    st = load_library().attn_bwd_static_workspace(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE), _ptr(dQ),
                                                  _ptr(dK), _ptr(dV), B, H, N, d, int(bool(causal)), float(scale),
                                                  _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_static_workspace")


def _ws(workspace):
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check_device("workspace", workspace)
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def attn_bwd_fused_preprocess(O, dO, LSE, workspace, stream=None) -> None:
    _check_bhnd("O", O)
    _check_bhnd("dO", dO, O.shape)
    _check_lse(LSE, O.shape)
    B, H, N, d = O.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_fused_preprocess(_ptr(O), _ptr(dO), _ptr(LSE), B, H, N, d, wp, wb,
                                                  _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_fused_preprocess")


def attn_bwd_fused_dkdvdq(Q, K, V, dO, dK, dV, causal: bool, scale: float, workspace, stream=None) -> None:
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("dO", dO), ("dK", dK), ("dV", dV)):
        _check_bhnd(n, t, Q.shape)
    B, H, N, d = Q.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_fused_dkdvdq(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(dK), _ptr(dV), B, H, N, d,
                                              int(bool(causal)), float(scale), wp, wb, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_fused_dkdvdq")


def attn_bwd_fused_dq_convert(dQ, scale: float, workspace, stream=None) -> None:
    _check_bhnd("dQ", dQ)
    B, H, N, d = dQ.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_fused_dq_convert(_ptr(dQ), B, H, N, d, float(scale), wp, wb,
                                                  _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_fused_dq_convert")


def attn_bwd_preprocess(O, dO, LSE, workspace, stream=None) -> None:
    _check_bhnd("O", O)
    _check_bhnd("dO", dO, O.shape)
    _check_lse(LSE, O.shape)
    B, H, N, d = O.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_preprocess(_ptr(O), _ptr(dO), _ptr(LSE), B, H, N, d, wp, wb,
                                            _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_preprocess")


def attn_bwd_dkdv(Q, K, V, dO, dK, dV, causal: bool, scale: float, workspace, stream=None) -> None:
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("dO", dO), ("dK", dK), ("dV", dV)):
        _check_bhnd(n, t, Q.shape)
    B, H, N, d = Q.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_dkdv(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(dK), _ptr(dV), B, H, N, d,
                                      int(bool(causal)), float(scale), wp, wb, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_dkdv")


def attn_bwd_dq(Q, K, V, dO, dQ, causal: bool, scale: float, workspace, stream=None) -> None:
    _check_bhnd("Q", Q)
    for n, t in (("K", K), ("V", V), ("dO", dO), ("dQ", dQ)):
        _check_bhnd(n, t, Q.shape)
    B, H, N, d = Q.shape
    wp, wb = _ws(workspace)
    st = load_library().attn_bwd_dq(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(dQ), B, H, N, d,
                                    int(bool(causal)), float(scale), wp, wb, _stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_dq")


def attn_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the failure-path self-test (a bounded wait that runs out)."""
    st = load_library().attn_selftest_wait_timeout(_stream_handle(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_wait_timeout")


def attn_check_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status code."""
    return int(load_library().attn_check_status(_stream_handle(stream)))


# ---------------------------------------------------------------------------
# Convenience wrappers: allocate outputs with torch, then call the C ABI.
# ---------------------------------------------------------------------------

def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def forward(Q, K, V, causal: bool, scale: float | None = None, stream=None):
    """O, LSE for Q (B, H, N, d) and K, V (B, H_kv, N, d); H_kv == H is plain multi-head attention."""
    B, H, N, d = Q.shape
    scale = default_scale(d) if scale is None else scale
    O = torch.empty_like(Q)
    LSE = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    if K.shape[1] == H:
        attn_fwd(Q, K, V, O, LSE, causal, scale, stream)
    else:
        attn_fwd_gqa(Q, K, V, O, LSE, causal, scale, stream)
    return O, LSE


def alloc_workspace(B: int, H: int, N: int, d: int, device, deterministic: bool = False) -> torch.Tensor:
    nbytes = (attn_bwd_deterministic_workspace_bytes if deterministic else attn_bwd_workspace_bytes)(B, H, N, d)
    return torch.empty((max(nbytes, 16) + 15) // 16 * 4, dtype=torch.float32, device=device)


def backward(Q, K, V, O, LSE, dO, causal: bool, scale: float | None = None, workspace=None, stream=None,
             deterministic: bool = False):
    """dQ, dK, dV; ``deterministic`` selects the bitwise-reproducible two-kernel path."""
    B, H, N, d = Q.shape
    scale = default_scale(d) if scale is None else scale
    if workspace is None:
        workspace = alloc_workspace(B, H, N, d, Q.device, deterministic)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    if deterministic:
        attn_bwd_deterministic(Q, K, V, O, dO, LSE, dQ, dK, dV, causal, scale, workspace, stream)
    elif K.shape[1] == H:
        attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, causal, scale, workspace, stream)
    else:
        attn_bwd_gqa(Q, K, V, O, dO, LSE, dQ, dK, dV, causal, scale, workspace, stream)
    return dQ, dK, dV
