"""GPU parity of the forward's fp32 output copy (attn_fwd_f32out) against the
oracle with the bare O tolerance 1e-2: the normalised rows before their
rounding to bf16.  The bf16 O that the same call writes must be exactly the
round-to-nearest-even bf16 of that fp32 copy, and O and LSE must equal what
attn_fwd writes for the same inputs (one forward, two output formats).
Covers the outlier workload (rows whose softmax is nearly one-hot, |O| up to
8, where bf16 rounding alone exceeds 1e-2), both masks, both head dims and
ragged tails."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from exact_io_aware_58_b200.inputs import WORKLOADS, make_inputs, workload_inputs
from oracle import attn_oracle as orc

from ._parity import LSE_TOL, O_TOL, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _check(inp, causal, scale, heads=None):
    q, k, v = (inp[n].to(DEV) for n in ("Q", "K", "V"))
    O = torch.empty_like(q)
    O32 = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    L = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
    attn.attn_fwd_f32out(q, k, v, O, O32, L, causal, scale)
    O_b = torch.empty_like(q)
    L_b = torch.empty_like(L)
    attn.attn_fwd(q, k, v, O_b, L_b, causal, scale)
    assert attn.attn_check_status() == attn.ATTN_OK
    assert torch.equal(O, O32.to(torch.bfloat16)), "bf16 O is not the rounding of the fp32 O"
    assert torch.equal(O, O_b) and torch.equal(L, L_b), "attn_fwd_f32out differs from attn_fwd"
    sel = slice(None) if heads is None else heads
    Q, K, V = (f64(inp[n].cpu())[sel] for n in ("Q", "K", "V"))
    O_ref, L_ref = orc.attn_fwd(Q, K, V, scale, causal)
    o32 = f64(O32)[sel]
    assert np.isfinite(o32).all()
    err = float(np.abs(o32 - O_ref).max())
    assert err <= O_TOL, f"fp32 O error {err:.3e} > {O_TOL}"
    assert float(np.abs(f64(L)[sel] - L_ref).max()) <= LSE_TOL
    return err


@pytest.mark.parametrize("causal", [False, True])
def test_outliers_fp32_output_bare_tolerance(causal):
    w = WORKLOADS["fwd_outliers"]
    inp = workload_inputs(w)
    # the oracle on every fourth head keeps the test to seconds (1 % of all
    # rows are outliers, about 20 per head, so every head checked holds some)
    heads = list(range(0, w.B * w.H, 4))
    _check(inp, causal, w.scale, heads=heads)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 129, 300, 513])
def test_small_shapes_fp32_output(N, d, causal):
    inp = make_inputs(1, 2, N, d, seed=700 + N + d + causal, with_dO=False)
    _check(inp, causal, 1.0 / math.sqrt(d))


def test_peaked_rows_fp32_output_within_the_p_rounding_bound():
    # Q scaled up so most rows are nearly one-hot.  There the rounding of P to
    # bf16 (the P reading; relative error up to 2^-8, bf16's unit roundoff)
    # does not average out: with the lazily rescaled p of the dominant key
    # anywhere in [1, 2^8], a row's O carries up to 2^-8 sum_j P_ij |V_jk| of
    # it -- for N(0, 1) values up to ~0.018 on a one-hot row, above the bare
    # 1e-2 (measured 0.0102 here).  So this case is held to that derived bound
    # elementwise, plus 1e-3 for the fp32 scores (|S| reaches ~30 after
    # scaling) and exp2.
    g = torch.Generator("cpu").manual_seed(790)
    B, H, N, d = 1, 2, 384, 128
    scale = 1.0 / math.sqrt(d)
    q = (torch.randn((B, H, N, d), generator=g) * 8.0).to(torch.bfloat16)
    k = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    Q, K, V = (t.to(DEV) for t in (q, k, v))
    O = torch.empty_like(Q)
    O32 = torch.empty(Q.shape, dtype=torch.float32, device=DEV)
    L = torch.empty(Q.shape[:3], dtype=torch.float32, device=DEV)
    attn.attn_fwd_f32out(Q, K, V, O, O32, L, True, scale)
    assert attn.attn_check_status() == attn.ATTN_OK
    assert torch.equal(O, O32.to(torch.bfloat16))
    Qh, Kh, Vh = f64(q), f64(k), f64(v)
    O_ref, L_ref = orc.attn_fwd(Qh, Kh, Vh, scale, True)
    o32 = f64(O32)
    for h in range(B * H):
        s_ = orc.head_scores(Qh[h], Kh[h], scale, True)
        P = np.exp(s_ - s_.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        bound = 2.0 ** -8 * (P @ np.abs(Vh[h])) + 1e-3
        err = np.abs(o32[h] - O_ref[h])
        assert (err <= bound).all(), f"head {h}: max excess {float((err - bound).max()):.3e}"
    assert float(np.abs(f64(L) - L_ref).max()) <= LSE_TOL
