"""GPU parity for decode against an FP8 (E4M3) key/value cache
(attn_fwd_kvcache_fp8): the oracle's cache forward on the dequantised cache.
The kernel forms the scores on the E4M3 key codes with each query row split
into two E4M3 terms (exact for elements of at least 2^-10 of the row's
largest magnitude, within 2^-10 of it in the row's scaled units below that),
widens the value codes exactly and rounds P to f16, so the tolerances are
those of the bf16 path (O 1e-2 plus the output's half ulp, LSE 1e-3).
Covers decode and a few query rows per head, shared key/value heads, both
masks, per-batch lengths with non-finite codes past the length, several
split counts, and query rows whose elements span many binades (the split's
inexact range)."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from oracle import attn_oracle as orc

from ._parity import assert_lse, assert_o, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
E4M3_MAX = 448.0


def _run(B, H, Hk, Nq, Nk, causal, seed, lens=None, splits=0, poison=False, q_spread=0):
    d = 128
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g)
    if q_spread:
        # per-element factors 2^-q_spread .. 2^3: most of a row far below its largest element
        q = q * torch.exp2(torch.randint(-q_spread, 4, q.shape, generator=g).float())
    q = q.to(torch.bfloat16)
    k = torch.randn((B, Hk, Nk, d), generator=g)
    v = torch.randn((B, Hk, Nk, d), generator=g)
    kd, vd = float(k.abs().max()) / E4M3_MAX, float(v.abs().max()) / E4M3_MAX
    k8 = (k / kd).to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = (v / vd).to(torch.float8_e4m3fn).view(torch.uint8)
    if poison and lens is not None:
        for b, L in enumerate(lens):
            k8[b, :, L:] = 0x7F                    # E4M3 NaN
            v8[b, :, L:] = 0xFF                    # E4M3 NaN (negative)
    scale = 1.0 / math.sqrt(d)
    Q, K8, V8 = q.to(DEV), k8.to(DEV), v8.to(DEV)
    O = torch.full_like(Q, 7.0)
    LSE = torch.full((B, H, Nq), 7.0, dtype=torch.float32, device=DEV)
    lens_t = None if lens is None else torch.tensor(lens, dtype=torch.int32, device=DEV)
    nbytes = attn.attn_fwd_kvcache_workspace_bytes(B, H, Hk, Nq, Nk, d, splits)
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device=DEV)
    attn.attn_fwd_kvcache_fp8(Q, K8, V8, O, LSE, lens_t, causal, scale, kd, vd, splits, ws)
    assert attn.attn_check_status() == attn.ATTN_OK
    outs = [orc.attn_fwd_kvcache_fp8(f64(q[b:b + 1]), k8[b:b + 1].numpy().reshape(-1, Nk, d),
                                     v8[b:b + 1].numpy().reshape(-1, Nk, d), kd, vd, scale, causal, 1, H, Hk,
                                     kv_lens=None if lens is None else [lens[b]]) for b in range(B)]
    O_ref = np.concatenate([o for o, _ in outs])
    L_ref = np.concatenate([lv for _, lv in outs])
    o, l = f64(O), f64(LSE)
    empty = np.isneginf(L_ref)
    assert (np.isneginf(l) == empty).all()
    assert (o[empty] == 0).all()
    assert_o(o, O_ref)
    assert_lse(np.where(empty, 0.0, l), np.where(empty, 0.0, L_ref))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nk", [1, 100, 129, 1000, 4097])
def test_fp8_cache_decode(Nk, causal):
    _run(2, 8, 2, 1, Nk, causal, seed=1100 + Nk + causal)


@pytest.mark.parametrize("Hk", [1, 8, 32])
@pytest.mark.parametrize("splits", [0, 1, 5])
def test_fp8_cache_head_groups_and_splits(Hk, splits):
    _run(1, 32, Hk, 1, 2000, True, seed=1200 + Hk + splits, splits=splits)


@pytest.mark.parametrize("Nq", [2, 4])
def test_fp8_cache_few_rows(Nq):
    _run(2, 8, 2, Nq, 700, True, seed=1300 + Nq)


def test_fp8_cache_lengths_with_nan_past_the_length():
    _run(5, 4, 2, 3, 1000, True, seed=1400, lens=[1000, 517, 128, 1, 0], poison=True)


@pytest.mark.parametrize("spread", [12, 24])
def test_fp8_cache_query_rows_spanning_many_binades(spread):
    _run(2, 8, 2, 1, 1500, True, seed=1500 + spread, q_spread=spread)
