"""Out-of-bounds write detection without a sanitizer: every output buffer (O,
LSE, the fp32 copy of O, dQ, dK, dV, the backward workspaces, the split-KV
partials) is a view into a larger allocation whose guard regions before and
after it hold a byte pattern; after each call the guards must be unchanged.
The lengths straddle the 128-row tiles (1, 127, 129, 300, 513), where a store
past the last row would land in the guard after the buffer.  Results are not
checked here (the parity tests do that), only that nothing was written
outside the buffers."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn

from ._parity import Guarded

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _check(named):
    torch.cuda.synchronize()
    assert attn.attn_check_status() == attn.ATTN_OK
    bad = [name for name, g in named.items() if not g.intact()]
    assert not bad, f"writes outside the buffer: {bad}"


def _inputs(B, H, Hk, N, d, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    mk = lambda h: torch.randn((B, h, N, d), generator=g).to(torch.bfloat16).to(DEV)
    return mk(H), mk(Hk), mk(Hk), mk(H)


NS = [1, 127, 129, 300, 513]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", NS)
def test_forward_and_both_backward_paths_stay_in_bounds(N, causal, d):
    B, H = 1, 2
    q, k, v, do = _inputs(B, H, H, N, d, seed=N + d)
    scale = 1 / math.sqrt(d)
    O, LSE = Guarded((B, H, N, d), torch.bfloat16), Guarded((B, H, N), torch.float32)
    O32 = Guarded((B, H, N, d), torch.float32)
    attn.attn_fwd_f32out(q, k, v, O.t, O32.t, LSE.t, causal, scale)
    _check({"O": O, "O32": O32, "LSE": LSE})
    attn.attn_fwd(q, k, v, O.t, LSE.t, causal, scale)
    _check({"O": O, "LSE": LSE})
    for det in (False, True):
        dQ, dK, dV = (Guarded((B, H, N, d), torch.bfloat16) for _ in range(3))
        wsb = (attn.attn_bwd_deterministic_workspace_bytes if det else attn.attn_bwd_workspace_bytes)(B, H, N, d)
        ws = Guarded(None, torch.float32, nbytes=wsb)
        fn = attn.attn_bwd_deterministic if det else attn.attn_bwd
        fn(q, k, v, O.t, do, LSE.t, dQ.t, dK.t, dV.t, causal, scale, ws.t)
        _check({"dQ": dQ, "dK": dK, "dV": dV, "workspace": ws})


@pytest.mark.parametrize("N", NS)
def test_gqa_and_blocksparse_stay_in_bounds(N):
    B, H, Hk, d = 1, 4, 2, 128
    q, k, v, do = _inputs(B, H, Hk, N, d, seed=7 + N)
    scale = 1 / math.sqrt(d)
    O, LSE = Guarded((B, H, N, d), torch.bfloat16), Guarded((B, H, N), torch.float32)
    attn.attn_fwd_gqa(q, k, v, O.t, LSE.t, True, scale)
    _check({"O": O, "LSE": LSE})
    dQ = Guarded((B, H, N, d), torch.bfloat16)
    dK, dV = Guarded((B, Hk, N, d), torch.bfloat16), Guarded((B, Hk, N, d), torch.bfloat16)
    ws = Guarded(None, torch.float32, nbytes=attn.attn_bwd_workspace_bytes(B, H, N, d))
    attn.attn_bwd_gqa(q, k, v, O.t, do, LSE.t, dQ.t, dK.t, dV.t, True, scale, ws.t)
    _check({"dQ": dQ, "dK": dK, "dV": dV, "workspace": ws})
    nt = (N + 127) // 128
    rng = np.random.default_rng(N)
    mask = torch.from_numpy((rng.random((B, H, nt, nt)) < 0.6).astype(np.uint8)).to(DEV)
    attn.attn_fwd_blocksparse(q, k, v, O.t, LSE.t, mask, True, scale)
    _check({"O": O, "LSE": LSE})
    attn.attn_bwd_blocksparse(q, k, v, O.t, do, LSE.t, mask, dQ.t, dK.t, dV.t, True, scale, ws.t)
    _check({"dQ": dQ, "dK": dK, "dV": dV, "workspace": ws})


@pytest.mark.parametrize("N", NS)
def test_fp8_forward_stays_in_bounds(N):
    B, H, Hk, d = 1, 2, 2, 128
    g = torch.Generator("cpu").manual_seed(N)
    q8, k8, v8 = (torch.randn((B, h, N, d), generator=g).to(torch.float8_e4m3fn).to(DEV) for h in (H, Hk, Hk))
    O, LSE = Guarded((B, H, N, d), torch.bfloat16), Guarded((B, H, N), torch.float32)
    attn.attn_fwd_fp8(q8, k8, v8, O.t, LSE.t, True, 1 / math.sqrt(d), 1.0, 1.0, 1.0)
    _check({"O": O, "LSE": LSE})


@pytest.mark.parametrize("Nk", NS)
@pytest.mark.parametrize("Nq", [1, 3])
def test_kvcache_paths_stay_in_bounds(Nq, Nk):
    B, H, Hk, d = 2, 8, 2, 128
    g = torch.Generator("cpu").manual_seed(Nk + Nq)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn((B, Hk, Nk, d), generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn((B, Hk, Nk, d), generator=g).to(torch.bfloat16).to(DEV)
    lens = torch.tensor([Nk, max(0, Nk // 2)], dtype=torch.int32, device=DEV)
    scale = 1 / math.sqrt(d)
    for splits in (1, 3, 0):
        O, LSE = Guarded((B, H, Nq, d), torch.bfloat16), Guarded((B, H, Nq), torch.float32)
        nb = attn.attn_fwd_kvcache_workspace_bytes(B, H, Hk, Nq, Nk, d, splits)
        ws = Guarded(None, torch.float32, nbytes=max(nb, 16))
        attn.attn_fwd_kvcache(q, k, v, O.t, LSE.t, lens, True, scale, splits, ws.t if nb else None)
        _check({"O": O, "LSE": LSE, "partials": ws})
    k8, v8 = k.float().to(torch.float8_e4m3fn), v.float().to(torch.float8_e4m3fn)
    O, LSE = Guarded((B, H, Nq, d), torch.bfloat16), Guarded((B, H, Nq), torch.float32)
    nb = attn.attn_fwd_kvcache_workspace_bytes(B, H, Hk, Nq, Nk, d, 0)
    ws = Guarded(None, torch.float32, nbytes=nb)
    attn.attn_fwd_kvcache_fp8(q, k8, v8, O.t, LSE.t, lens, True, scale, 1.0, 1.0, 0, ws.t)
    _check({"O": O, "LSE": LSE, "partials": ws})
