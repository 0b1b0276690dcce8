"""The C-ABI library builds, loads without a GPU, exports every symbol that
include/attn.h declares, and rejects bad arguments before launching anything."""

import ctypes
import os
import re

import pytest

from exact_io_aware_58_b200 import attn, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return attn.load_library()


def test_header_declares_the_abi():
    assert _declared_functions() == sorted(attn.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    # and nothing internal leaks out under the attn_ prefix
    out = os.popen(f"nm -D --defined-only {build.LIB_PATH}").read()
    exported = sorted(set(re.findall(r"\bT (attn_[a-z_0-9]+)\b", out)))
    assert exported == _declared_functions()


def test_status_strings(lib):
    for code, name in [(0, "ATTN_OK"), (-1, "ATTN_ERR_INVALID_ARG"), (-2, "ATTN_ERR_UNSUPPORTED"),
                       (-3, "ATTN_ERR_MISALIGNED"), (-4, "ATTN_ERR_WORKSPACE"), (-5, "ATTN_ERR_LAUNCH"),
                       (-6, "ATTN_ERR_TIMEOUT"), (-7, "ATTN_ERR_DEVICE")]:
        assert attn.attn_status_string(code) == name
    assert attn.attn_status_string(42) == "ATTN_ERR_UNKNOWN"


def test_workspace_bytes(lib):
    # deterministic path: two fp32 vectors per head, rows padded to a multiple of 128
    det = attn.attn_bwd_deterministic_workspace_bytes
    assert det(1, 2, 256, 64) == 2 * 4 * 2 * 256
    assert det(8, 32, 16384, 128) == 2 * 4 * 256 * 16384
    assert det(1, 8, 100000, 128) == 2 * 4 * 8 * 100096
    assert det(1, 1, 1, 64) == 2 * 4 * 128
    assert det(1, 1, 1, 96) == 0       # unsupported d
    assert det(0, 1, 1, 64) == 0
    # fused path: the same vectors plus a d-wide fp32 dQ accumulator per padded row
    ws = attn.attn_bwd_workspace_bytes
    assert ws(1, 2, 256, 64) == (2 + 64) * 4 * 2 * 256
    assert ws(8, 32, 16384, 128) == (2 + 128) * 4 * 256 * 16384
    assert ws(1, 8, 100000, 128) == (2 + 128) * 4 * 8 * 100096
    assert ws(1, 1, 1, 96) == 0
    assert ws(0, 1, 1, 64) == 0


# Fake, never-dereferenced device addresses: argument checks happen before any
# CUDA call, so these return synchronously without a GPU.
A = ctypes.c_void_p(0x100000)
MIS = ctypes.c_void_p(0x100008)


def _fwd(lib, B=1, H=1, N=128, d=64, scale=0.125, ptrs=None):
    p = ptrs or [A] * 5
    return lib.attn_fwd(*p, B, H, N, d, 0, scale, None)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, N=0) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, B=0) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == attn.ATTN_ERR_UNSUPPORTED
    assert _fwd(lib, d=256) == attn.ATTN_ERR_UNSUPPORTED
    assert _fwd(lib, scale=0.0) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, scale=-1.0) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd(lib, ptrs=[A, A, None, A, A]) == attn.ATTN_ERR_INVALID_ARG
    for k in range(5):
        p = [A] * 5
        p[k] = MIS
        assert _fwd(lib, ptrs=p) == attn.ATTN_ERR_MISALIGNED


def test_f32out_argument_errors(lib):
    # the fp32 output is required; the forward's own checks apply to the rest
    assert lib.attn_fwd_f32out(A, A, A, A, None, A, 1, 2, 128, 64, 0, 0.125, None) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_f32out(A, A, A, A, MIS, A, 1, 2, 128, 64, 0, 0.125, None) == attn.ATTN_ERR_MISALIGNED
    assert lib.attn_fwd_f32out(A, A, A, A, A, A, 1, 2, 128, 96, 0, 0.125, None) == attn.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fwd_f32out(A, A, A, A, A, A, 1, 2, 0, 64, 0, 0.125, None) == attn.ATTN_ERR_INVALID_ARG


def test_gqa_argument_errors(lib):
    p = [A] * 5
    # H must be a multiple of H_kv, and 1 <= H_kv <= H
    assert lib.attn_fwd_gqa(*p, 1, 4, 3, 128, 64, 0, 0.125, None) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_gqa(*p, 1, 4, 0, 128, 64, 0, 0.125, None) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_gqa(*p, 1, 4, 8, 128, 64, 0, 0.125, None) == attn.ATTN_ERR_INVALID_ARG
    ws = attn.attn_bwd_workspace_bytes(1, 4, 128, 64)
    assert lib.attn_bwd_gqa(*([A] * 9), 1, 4, 3, 128, 64, 1, 0.125, A, ws, None) == attn.ATTN_ERR_INVALID_ARG
    p[1] = MIS
    assert lib.attn_fwd_gqa(*p, 1, 4, 2, 128, 64, 0, 0.125, None) == attn.ATTN_ERR_MISALIGNED


def test_bwd_argument_errors(lib):
    ws = attn.attn_bwd_workspace_bytes(1, 1, 128, 64)

    def bwd(ptrs=None, ws_ptr=A, ws_bytes=ws, d=64):
        p = ptrs or [A] * 9
        return lib.attn_bwd(*p, 1, 1, 128, d, 1, 0.125, ws_ptr, ws_bytes, None)

    assert bwd(ws_bytes=ws - 4) == attn.ATTN_ERR_WORKSPACE
    # the deterministic path's smaller workspace is not enough for the fused path
    assert bwd(ws_bytes=attn.attn_bwd_deterministic_workspace_bytes(1, 1, 128, 64)) == attn.ATTN_ERR_WORKSPACE
    assert bwd(ws_ptr=None) == attn.ATTN_ERR_INVALID_ARG
    assert bwd(ws_ptr=MIS) == attn.ATTN_ERR_MISALIGNED
    assert bwd(d=32) == attn.ATTN_ERR_UNSUPPORTED
    for k in range(9):
        p = [A] * 9
        p[k] = MIS
        assert bwd(ptrs=p) == attn.ATTN_ERR_MISALIGNED


def test_bwd_deterministic_argument_errors(lib):
    ws = attn.attn_bwd_deterministic_workspace_bytes(1, 4, 128, 64)

    def bwd(ptrs=None, ws_ptr=A, ws_bytes=ws, d=64, hk=4):
        p = ptrs or [A] * 9
        return lib.attn_bwd_deterministic(*p, 1, 4, hk, 128, d, 1, 0.125, ws_ptr, ws_bytes, None)

    assert bwd(ws_bytes=ws - 4) == attn.ATTN_ERR_WORKSPACE
    assert bwd(ws_ptr=None) == attn.ATTN_ERR_INVALID_ARG
    assert bwd(ws_ptr=MIS) == attn.ATTN_ERR_MISALIGNED
    assert bwd(d=96) == attn.ATTN_ERR_UNSUPPORTED
    assert bwd(hk=3) == attn.ATTN_ERR_INVALID_ARG
    for k in range(9):
        p = [A] * 9
        p[k] = MIS
        assert bwd(ptrs=p) == attn.ATTN_ERR_MISALIGNED


def test_error_detail_has_no_stray_text(lib):
    # a rejected fp8 call records a formatted detail string
    p = [A] * 5
    assert lib.attn_fwd_fp8(*p, 1, 1, 1, 128, 64, 0, 0.125, 1.0, 1.0, 1.0, None) == attn.ATTN_ERR_UNSUPPORTED
    assert attn.attn_last_error() == "attn_fwd_fp8 supports d = 128 only (got 64)"


def test_python_binding_validates_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q, q, torch.zeros(1, 1, 8), False, 0.125)


def test_kvcache_splits_and_workspace(lib):
    # explicit counts are capped by the number of 128-row key tiles
    assert attn.attn_fwd_kvcache_splits(1, 8, 8, 1, 1000, 128, 3) == 3
    assert attn.attn_fwd_kvcache_splits(1, 8, 8, 1, 1000, 128, 50) == 8
    assert attn.attn_fwd_kvcache_splits(1, 8, 8, 1, 100, 128, 0) == 1
    # decode batch with 64 key/value heads over a 16K cache: many splits, all SMs busy
    s = attn.attn_fwd_kvcache_splits(8, 32, 8, 1, 16384, 128, 0)
    assert 2 <= s <= 128
    # 4 packed rows per key/value head: replicated into the four lane quarters, four partials per chunk
    assert attn.attn_fwd_kvcache_workspace_bytes(8, 32, 8, 1, 16384, 128, 0) == 4 * s * 8 * 32 * 1 * 129 * 4
    # 40 packed rows: one partial per chunk; a single chunk needs no workspace
    assert attn.attn_fwd_kvcache_workspace_bytes(1, 8, 2, 10, 1000, 64, 3) == 3 * 8 * 10 * 65 * 4
    assert attn.attn_fwd_kvcache_workspace_bytes(1, 8, 2, 10, 1000, 64, 1) == 0
    assert attn.attn_fwd_kvcache_workspace_bytes(1, 8, 2, 1, 1000, 64, 1) == 4 * 8 * 1 * 65 * 4
    # a large prefill-sized grid needs no split and no workspace
    assert attn.attn_fwd_kvcache_splits(8, 32, 32, 512, 2048, 128, 0) == 1
    assert attn.attn_fwd_kvcache_workspace_bytes(8, 32, 32, 512, 2048, 128, 0) == 0
    # rejected sizes
    assert attn.attn_fwd_kvcache_splits(1, 8, 3, 1, 100, 128, 0) == 0
    assert attn.attn_fwd_kvcache_workspace_bytes(1, 8, 8, 1, 100, 96, 2) == 0
    assert attn.attn_fwd_kvcache_splits(1, 8, 8, 0, 100, 128, 0) == 0


def test_kvcache_argument_errors(lib):
    p = [A] * 5

    def call(B=1, H=4, Hk=2, Nq=1, Nk=256, d=64, scale=0.125, splits=1, ws=None, ws_bytes=0, lens=None, ptrs=None):
        return lib.attn_fwd_kvcache(*(ptrs or p), lens, B, H, Hk, Nq, Nk, d, 1, scale, splits, ws, ws_bytes, None)

    assert call(Nq=0) == attn.ATTN_ERR_INVALID_ARG
    assert call(Nk=0) == attn.ATTN_ERR_INVALID_ARG
    assert call(Hk=3) == attn.ATTN_ERR_INVALID_ARG
    assert call(d=96) == attn.ATTN_ERR_UNSUPPORTED
    assert call(scale=0.0) == attn.ATTN_ERR_INVALID_ARG
    assert call(splits=-1) == attn.ATTN_ERR_INVALID_ARG
    assert call(lens=ctypes.c_void_p(0x100002)) == attn.ATTN_ERR_MISALIGNED
    for k in range(5):
        q = [A] * 5
        q[k] = MIS
        assert call(ptrs=q) == attn.ATTN_ERR_MISALIGNED
    # two splits need a workspace of the advertised size
    need = attn.attn_fwd_kvcache_workspace_bytes(1, 4, 2, 1, 256, 64, 2)
    assert need == 4 * 2 * 4 * 65 * 4          # 2 packed rows: four partials per chunk
    assert call(splits=2) == attn.ATTN_ERR_INVALID_ARG
    assert call(splits=2, ws=MIS, ws_bytes=need) == attn.ATTN_ERR_MISALIGNED
    assert call(splits=2, ws=A, ws_bytes=need - 4) == attn.ATTN_ERR_WORKSPACE


def test_fp8_argument_errors(lib):
    p = [A] * 5

    def call(d=128, dq=1.0, dk=1.0, dv=1.0, ptrs=None, Hk=2):
        return lib.attn_fwd_fp8(*(ptrs or p), 1, 4, Hk, 256, d, 1, 0.125, dq, dk, dv, None)

    assert call(d=64) == attn.ATTN_ERR_UNSUPPORTED
    assert call(Hk=3) == attn.ATTN_ERR_INVALID_ARG
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert call(dq=bad) == attn.ATTN_ERR_INVALID_ARG
        assert call(dk=bad) == attn.ATTN_ERR_INVALID_ARG
        assert call(dv=bad) == attn.ATTN_ERR_INVALID_ARG
    for k in range(5):
        q = [A] * 5
        q[k] = MIS
        assert call(ptrs=q) == attn.ATTN_ERR_MISALIGNED


def test_kvcache_fp8_argument_errors(lib):
    p = [A] * 5
    ws_ok = attn.attn_fwd_kvcache_workspace_bytes(1, 4, 2, 1, 256, 128, 2)

    def call(H=4, Hk=2, Nq=1, d=128, kd=1.0, vd=1.0, ws=A, ws_bytes=None, ptrs=None):
        wb = ws_ok if ws_bytes is None else ws_bytes
        return lib.attn_fwd_kvcache_fp8(*(ptrs or p), None, 1, H, Hk, Nq, 256, d, 1, 0.125, kd, vd, 2, ws, wb,
                                        None)

    assert call(d=64) == attn.ATTN_ERR_UNSUPPORTED
    assert call(H=64, Hk=1) == attn.ATTN_ERR_UNSUPPORTED        # 64 packed rows per key/value head
    assert call(Nq=17) == attn.ATTN_ERR_UNSUPPORTED             # 2 * 17 = 34 > 32
    for bad in (0.0, -2.0, float("nan")):
        assert call(kd=bad) == attn.ATTN_ERR_INVALID_ARG
        assert call(vd=bad) == attn.ATTN_ERR_INVALID_ARG
    assert call(ws=None) == attn.ATTN_ERR_INVALID_ARG
    assert call(ws_bytes=ws_ok - 4) == attn.ATTN_ERR_WORKSPACE
    for k in range(5):
        q = [A] * 5
        q[k] = MIS
        assert call(ptrs=q) == attn.ATTN_ERR_MISALIGNED


def test_varlen_argument_errors(lib):
    p = [A] * 5

    def call(ptrs=None, cu=A, n_seqs=2, total=300, H=4, Hk=2, d=128, scale=0.1):
        return lib.attn_fwd_varlen(*(ptrs or p), cu, n_seqs, total, H, Hk, d, 1, scale, None)

    assert call(n_seqs=0) == attn.ATTN_ERR_INVALID_ARG
    assert call(total=0) == attn.ATTN_ERR_INVALID_ARG
    assert call(d=96) == attn.ATTN_ERR_UNSUPPORTED
    assert call(Hk=3) == attn.ATTN_ERR_INVALID_ARG
    assert call(scale=0.0) == attn.ATTN_ERR_INVALID_ARG
    assert call(cu=None) == attn.ATTN_ERR_INVALID_ARG
    assert call(cu=ctypes.c_void_p(0x100002)) == attn.ATTN_ERR_MISALIGNED
    for k in range(5):
        q = [A] * 5
        q[k] = MIS
        assert call(ptrs=q) == attn.ATTN_ERR_MISALIGNED
