"""GPU parity for the FP8 (E4M3) forward (attn_fwd_fp8) against the oracle's
attention on the dequantised inputs.

What is exact and what is not (from the arithmetic, see the header of
attn_fwd_fp8): the products Q8 K8^T are exact in fp32 and the row statistics
are fp32, so LSE is held to the same 1e-3 as the bf16 path.  O carries the
rounding of P to E4M3: per row, |O - O_ref| <= dv * max|V8| * (2^-4 +
n_visible * 2^-10 / l) + half an ulp of the bf16 output, l = sum_j
exp(S_ij - max_j S_ij).  That bound is checked row by row; on top, the errors
of many rows must be unbiased (least-squares gain of O on O_ref within 1 %)
and small on average (relative Frobenius error within 6 %), which a wrong
scale factor or a dropped tile would break."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from oracle import attn_oracle as orc

from ._parity import LSE_TOL, bf16_half_ulp, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
E4M3_MAX = 448.0


def _quantise(x: torch.Tensor):
    """Per-tensor quantisation of an fp32 tensor to E4M3: (codes, descale)."""
    descale = float(x.abs().max()) / E4M3_MAX
    return (x / descale).to(torch.float8_e4m3fn), descale


def _case(B, H, Hk, N, causal, seed, stats=False, q_gain=1.0):
    d = 128
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, N, d), generator=g) * q_gain
    k = torch.randn((B, Hk, N, d), generator=g)
    v = torch.randn((B, Hk, N, d), generator=g)
    (q8, dq), (k8, dk), (v8, dv) = _quantise(q), _quantise(k), _quantise(v)
    scale = 1.0 / math.sqrt(d)
    O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=DEV)
    LSE = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    attn.attn_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), O, LSE, causal, scale, dq, dk, dv)
    assert attn.attn_check_status() == attn.ATTN_OK
    codes = [t.view(torch.uint8).numpy().reshape(-1, N, d) for t in (q8, k8, v8)]
    O_ref, L_ref = orc.attn_fwd_fp8(*codes, dq, dk, dv, scale, causal, B, H, Hk)
    o, l = f64(O), f64(LSE)
    assert np.isfinite(o).all() and np.isfinite(l).all()
    assert float(np.abs(l - L_ref).max()) <= LSE_TOL

    # row-wise bound from the E4M3 rounding of P
    Qd = dq * orc.e4m3_decode(codes[0])
    Kd = orc.expand_kv(dk * orc.e4m3_decode(codes[1]), B, H, Hk)
    Vd = orc.expand_kv(dv * orc.e4m3_decode(codes[2]), B, H, Hk)
    for h in range(B * H):
        s = orc.head_scores(Qd[h], Kd[h], scale, causal)
        m = s.max(axis=1, keepdims=True)
        lsum = np.exp(s - m).sum(axis=1)
        n_vis = np.isfinite(s).sum(axis=1)
        vmax = np.abs(Vd[h]).max()
        bound = vmax * (2.0 ** -4 + n_vis * 2.0 ** -10 / lsum) * 1.001 + 1e-4
        err = np.abs(o[h] - O_ref[h]).max(axis=1)
        ok = err <= bound + bf16_half_ulp(np.abs(O_ref[h])).max(axis=1)
        assert ok.all(), f"head {h}: row {int(np.argmin(ok))} err {err[~ok][0]:.3e} > bound"
    if stats:
        gain = float((o * O_ref).sum() / (O_ref * O_ref).sum())
        rel = float(np.linalg.norm(o - O_ref) / np.linalg.norm(O_ref))
        assert abs(gain - 1.0) <= 0.01, gain
        assert rel <= 0.06, rel


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 300, 513])
def test_fp8_forward_small(N, causal):
    _case(1, 2, 2, N, causal, seed=900 + N + causal)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_shared_heads_statistics(causal):
    _case(2, 4, 2, 1024, causal, seed=950 + causal, stats=True)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_many_items_per_cta(causal):
    # 2 x 40 query heads on 8 key/value heads, 3 row blocks each: 240 CTAs,
    # more than one wave on the SMs, with a ragged last block (513 rows)
    _case(2, 40, 8, 513, causal, seed=960 + causal, stats=True)


def test_fp8_forward_peaked_rows():
    # queries scaled up so rows put most of their weight on a few keys (the
    # lazy rescale fires and P spans the whole E4M3 range)
    _case(1, 2, 1, 640, True, seed=970, q_gain=6.0)


def test_fp8_rejects_other_head_dims():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float8_e4m3fn, device=DEV)
    O = torch.empty((1, 1, 128, 64), dtype=torch.bfloat16, device=DEV)
    LSE = torch.empty((1, 1, 128), dtype=torch.float32, device=DEV)
    with pytest.raises(attn.AttnError) as e:
        attn.attn_fwd_fp8(q, q, q, O, LSE, False, 0.125, 1.0, 1.0, 1.0)
    assert e.value.status == attn.ATTN_ERR_UNSUPPORTED


@pytest.mark.slow
def test_fp8_long_batch_sampled():
    """The benched size: long_batch (B=8, H=32, N=16384, causal) quantised per
    tensor to E4M3 as the benchmark does; two full heads against the oracle
    with the row-wise bound, 512 sampled rows across all heads, and the gain /
    relative-error statistics over everything checked."""
    from exact_io_aware_58_b200.inputs import WORKLOADS, sample_rows, workload_inputs

    w = WORKLOADS["long_batch"]
    inp = workload_inputs(w, seed=0, device=DEV)

    def q8(x):
        ds = float(x.abs().amax()) / E4M3_MAX
        return (x.float() / ds).to(torch.float8_e4m3fn), ds

    (qf, dq), (kf, dk), (vf, dv) = q8(inp["Q"]), q8(inp["K"]), q8(inp["V"])
    del inp
    O = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=DEV)
    LSE = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=DEV)
    attn.attn_fwd_fp8(qf, kf, vf, O, LSE, True, w.scale, dq, dk, dv)
    assert attn.attn_check_status() == attn.ATTN_OK
    codes = lambda t, h: t.view(-1, w.N, w.d)[h].view(torch.uint8).cpu().numpy()
    dec = lambda t, h, ds: ds * orc.e4m3_decode(codes(t, h))
    got, want = [], []
    heads = np.sort(np.random.default_rng(5).choice(w.B * w.H, 2, replace=False))
    for h in heads:
        Qd, Kd, Vd = dec(qf, h, dq), dec(kf, h, dk), dec(vf, h, dv)
        O_ref, L_ref = orc.attn_fwd(Qd[None], Kd[None], Vd[None], w.scale, True)
        o = O[:, :].reshape(-1, w.N, w.d)[h].float().cpu().numpy().astype(np.float64)
        l = LSE.reshape(-1, w.N)[h].cpu().numpy().astype(np.float64)
        assert np.isfinite(o).all() and float(np.abs(l - L_ref[0]).max()) <= LSE_TOL
        s = orc.head_scores(Qd, Kd, w.scale, True)
        m = s.max(axis=1, keepdims=True)
        lsum = np.exp(s - m).sum(axis=1)
        n_vis = np.isfinite(s).sum(axis=1)
        del s
        bound = np.abs(Vd).max() * (2.0 ** -4 + n_vis * 2.0 ** -10 / lsum) * 1.001 + 1e-4
        err = np.abs(o - O_ref[0]).max(axis=1)
        ok = err <= bound + bf16_half_ulp(np.abs(O_ref[0])).max(axis=1)
        assert ok.all(), f"head {h}: {int((~ok).sum())} rows above the bound"
        got.append(o)
        want.append(O_ref[0])
    rows = sample_rows(w.B, w.H, w.N, 512, 0).numpy()
    bh, ii = rows // w.N, rows % w.N
    for h in np.unique(bh):
        sel = ii[bh == h]
        o_ref, l_ref = orc.attn_fwd_rows(dec(qf, h, dq), dec(kf, h, dk), dec(vf, h, dv), w.scale, True, sel)
        o = O.reshape(-1, w.N, w.d)[h, torch.as_tensor(sel)].float().cpu().numpy().astype(np.float64)
        l = LSE.reshape(-1, w.N)[h, torch.as_tensor(sel)].cpu().numpy().astype(np.float64)
        assert float(np.abs(l - l_ref).max()) <= LSE_TOL
        got.append(o)
        want.append(o_ref)
    g, r = np.concatenate(got), np.concatenate(want)
    gain = float((g * r).sum() / (r * r).sum())
    rel = float(np.linalg.norm(g - r) / np.linalg.norm(r))
    assert abs(gain - 1.0) <= 0.01, gain
    assert rel <= 0.06, rel
