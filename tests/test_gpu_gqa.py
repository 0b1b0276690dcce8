"""GPU parity for shared key/value heads (grouped-query / multi-query
attention) through attn_fwd_gqa / attn_bwd_gqa, against the oracle's
expand-and-sum definition on the same seeded bf16 inputs."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from oracle import attn_oracle as orc

from ._parity import assert_grad, assert_lse, assert_o, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _inputs(B, H, Hk, N, d, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    mk = lambda h: torch.randn((B, h, N, d), generator=g).to(torch.bfloat16)
    return mk(H), mk(Hk), mk(Hk), mk(H)


def _check(B, H, Hk, N, d, causal, seed, with_bwd=True):
    q, k, v, do = _inputs(B, H, Hk, N, d, seed)
    scale = 1.0 / math.sqrt(d)
    Q, K, V, dO = (t.to(DEV) for t in (q, k, v, do))
    o, lse = attn.forward(Q, K, V, causal, scale)
    if with_bwd:
        dq, dk, dv = attn.backward(Q, K, V, o, lse, dO, causal, scale)
        assert dk.shape == K.shape and dv.shape == V.shape
    assert attn.attn_check_status() == attn.ATTN_OK
    Qn, Kn, Vn, dOn = (f64(t) for t in (q, k, v, do))
    O_ref, L_ref = orc.attn_fwd_gqa(Qn, Kn, Vn, scale, causal, B, H, Hk)
    assert_o(f64(o), O_ref)
    assert_lse(f64(lse), L_ref)
    if with_bwd:
        dQ_ref, dK_ref, dV_ref = orc.attn_bwd_gqa(Qn, Kn, Vn, dOn, scale, causal, B, H, Hk)
        assert_grad(f64(dq), dQ_ref, "dQ")
        assert_grad(f64(dk), dK_ref, "dK")
        assert_grad(f64(dv), dV_ref, "dV")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hk", [1, 2])
@pytest.mark.parametrize("N", [1, 129, 300])
def test_gqa_small(N, Hk, causal, d):
    _check(2, 4, Hk, N, d, causal, seed=500 + N + Hk + d)


def test_gqa_mid_size_causal():
    _check(2, 16, 4, 2048, 128, True, seed=77)


def test_gqa_entry_with_all_heads_equals_mha():
    q, k, v, do = (t.to(DEV) for t in _inputs(1, 4, 4, 300, 128, 9))
    o1, l1 = torch.empty_like(q), torch.empty(1, 4, 300, device=DEV)
    o2, l2 = torch.empty_like(q), torch.empty(1, 4, 300, device=DEV)
    attn.attn_fwd(q, k, v, o1, l1, True, 0.1)
    attn.attn_fwd_gqa(q, k, v, o2, l2, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
