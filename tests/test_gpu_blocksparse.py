"""GPU parity for block-sparse selection (attn_fwd_blocksparse /
attn_bwd_blocksparse) against the oracle's masked definition: random block
masks, query tiles that select nothing (O = 0, LSE = -inf), key tiles nobody
selects (dK = dV = 0), with and without the causal mask and shared K/V heads."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from oracle import attn_oracle as orc

from ._parity import assert_grad, assert_lse, assert_o, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(B, H, Hk, N, d, causal, density, seed, empty_rows=True):
    g = torch.Generator("cpu").manual_seed(seed)
    mk = lambda h: torch.randn((B, h, N, d), generator=g).to(torch.bfloat16)
    q, k, v, do = mk(H), mk(Hk), mk(Hk), mk(H)
    nt = (N + 127) // 128
    rng = np.random.default_rng(seed)
    mask = (rng.random((B, H, nt, nt)) < density).astype(np.uint8)
    if empty_rows and nt > 1:
        mask[0, 0, nt - 1, :] = 0            # a query tile that selects nothing
        mask[:, :, :, 0] = 0                 # key tile 0 selected by nobody
    scale = 1.0 / math.sqrt(d)
    Q, K, V, dO = (t.to(DEV) for t in (q, k, v, do))
    M = torch.from_numpy(mask).to(DEV)
    O = torch.empty_like(Q)
    LSE = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    attn.attn_fwd_blocksparse(Q, K, V, O, LSE, M, causal, scale)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    ws = attn.alloc_workspace(B, H, N, d, DEV)
    attn.attn_bwd_blocksparse(Q, K, V, O, dO, LSE, M, dQ, dK, dV, causal, scale, ws)
    assert attn.attn_check_status() == attn.ATTN_OK
    Qn, Kn, Vn, dOn = (f64(t) for t in (q, k, v, do))
    mflat = mask.reshape(B * H, nt, nt)
    O_ref, L_ref = orc.attn_fwd_blocksparse(Qn, Kn, Vn, scale, causal, mflat, B, H, Hk)
    o, l = f64(O), f64(LSE)
    empty = np.isneginf(L_ref)
    assert (np.isneginf(l) == empty).all(), "rows without visible keys must have LSE = -inf"
    assert (o[empty] == 0).all()
    assert_o(o, O_ref)
    assert_lse(np.where(empty, 0.0, l), np.where(empty, 0.0, L_ref))
    dQ_ref, dK_ref, dV_ref = orc.attn_bwd_blocksparse(Qn, Kn, Vn, dOn, scale, causal, mflat, B, H, Hk)
    assert_grad(f64(dQ), dQ_ref, "dQ")
    assert_grad(f64(dK), dK_ref, "dK")
    assert_grad(f64(dV), dV_ref, "dV")
    return mask


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [129, 300, 640])
def test_blocksparse_mha(N, causal, d):
    _case(1, 2, 2, N, d, causal, 0.5, seed=600 + N + d + causal)


@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_gqa(causal):
    _case(2, 4, 2, 513, 128, causal, 0.4, seed=610 + causal)


def test_blocksparse_all_selected_equals_dense():
    B, H, N, d = 1, 2, 384, 128
    g = torch.Generator("cpu").manual_seed(620)
    q, k, v = (torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).to(DEV) for _ in range(3))
    M = torch.ones((B, H, 3, 3), dtype=torch.uint8, device=DEV)
    o1, l1 = torch.empty_like(q), torch.empty((B, H, N), device=DEV)
    o2, l2 = attn.forward(q, k, v, True, 0.1)
    attn.attn_fwd_blocksparse(q, k, v, o1, l1, M, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_blocksparse_nothing_selected():
    B, H, N, d = 1, 1, 256, 64
    q = torch.randn((B, H, N, d)).to(torch.bfloat16).to(DEV)
    M = torch.zeros((B, H, 2, 2), dtype=torch.uint8, device=DEV)
    o, l = torch.full_like(q, float("nan")), torch.zeros((B, H, N), device=DEV)
    attn.attn_fwd_blocksparse(q, q, q, o, l, M, False, 0.1)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    ws = attn.alloc_workspace(B, H, N, d, DEV)
    attn.attn_bwd_blocksparse(q, q, q, o, q, l, M, dq, dk, dv, False, 0.1, ws)
    assert attn.attn_check_status() == attn.ATTN_OK
    assert (o == 0).all() and torch.isneginf(l).all()
    assert (dq == 0).all() and (dk == 0).all() and (dv == 0).all()
