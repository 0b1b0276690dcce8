"""attn_bwd_static_workspace: the backward for callers that cannot allocate
device memory (the workspace is the library's fixed device array instead of a
caller buffer).  Checked through the C ABI against attn_bwd_deterministic with
a caller workspace -- the same kernels, so the results must be bit for bit
equal -- and, independently, against the fp64 oracle, on two calls in a row
with different sizes, so that the second call runs over whatever the first
left in the shared array.

This file is collected last on purpose: it must pass both on its own in a
fresh process and after every other test.
"""

import ctypes
import math

import pytest
import torch

from exact_io_aware_58_b200 import attn
from exact_io_aware_58_b200.inputs import make_inputs
from oracle import attn_oracle as orc

from ._parity import assert_grad, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _case(B, H, N, d, causal, seed):
    lib = attn.load_library()
    inp = make_inputs(B, H, N, d, seed=seed)
    q, k, v, do = (inp[n].to(DEV) for n in ("Q", "K", "V", "dO"))
    scale = 1.0 / math.sqrt(d)
    o, lse = attn.forward(q, k, v, causal, scale)
    # existing deterministic entry point, caller-allocated workspace
    ref = attn.backward(q, k, v, o, lse, do, causal, scale, deterministic=True)
    # the fixed-workspace entry point, called through the C ABI
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.attn_bwd_static_workspace(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
                                       B, H, N, d, int(causal), scale, stream)
    assert st == attn.ATTN_OK, attn.attn_last_error()
    assert attn.attn_check_status() == attn.ATTN_OK
    for name, got, want in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
        assert torch.equal(got, want), name
    Q, K, V, dO = (f64(inp[n]) for n in ("Q", "K", "V", "dO"))
    for name, got, want in zip(("dQ", "dK", "dV"), (dq, dk, dv), orc.attn_bwd(Q, K, V, dO, scale, causal)):
        assert_grad(f64(got), want, name)


def test_static_workspace_matches_caller_workspace_twice():
    _case(2, 4, 1000, 128, True, seed=21)     # first call in this context: address look-up
    _case(1, 3, 300, 64, False, seed=22)      # second call: smaller sizes over the stale array


def test_static_workspace_rejects_sizes_beyond_its_capacity():
    lib = attn.load_library()
    fake = ctypes.c_void_p(0x100000)
    # B*H*Npad = 2^22 + 128 rows -> 8 bytes per row exceeds 32 MiB
    st = lib.attn_bwd_static_workspace(*([fake] * 9), 1, 1, 2**22 + 1, 128, 1, 0.1, None)
    assert st == attn.ATTN_ERR_WORKSPACE
    assert "ATTN_STATIC_WORKSPACE_BYTES" in attn.attn_last_error()
    assert attn.attn_bwd_deterministic_workspace_bytes(8, 32, 16384, 128) <= attn.ATTN_STATIC_WORKSPACE_BYTES
