"""GPU parity for the key/value-cache forward (attn_fwd_kvcache) against the
oracle's definition: decode (Nq = 1) and multi-row shapes, shared key/value
heads packed into one tile, bottom-right causal alignment, per-batch cache
lengths (including 0 and lengths shorter than Nq), non-finite cache contents
past the valid length, and every split count (one CTA per chunk, merged by
LSE) against the same reference."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from oracle import attn_oracle as orc

from ._parity import assert_lse, assert_o, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _oracle(q, k, v, scale, causal, lens):
    # one batch entry at a time keeps the oracle's expanded key/value copy small
    B, H, Hk = q.shape[0], q.shape[1], k.shape[1]
    outs = [orc.attn_fwd_kvcache(f64(q[b:b + 1]), f64(k[b:b + 1]), f64(v[b:b + 1]), scale, causal, 1, H, Hk,
                                 kv_lens=None if lens is None else [lens[b]]) for b in range(B)]
    return np.concatenate([o for o, _ in outs]), np.concatenate([l for _, l in outs])


def _run(B, H, Hk, Nq, Nk, d, causal, seed, lens=None, splits=0, poison=False, scale=None):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hk, Nk, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hk, Nk, d), generator=g).to(torch.bfloat16)
    if poison and lens is not None:
        # cache rows past each valid length hold NaN / Inf: they must never be weighted
        for b, L in enumerate(lens):
            k[b, :, L:] = float("nan")
            v[b, :, L:] = float("inf")
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    Q, K, V = q.to(DEV), k.to(DEV), v.to(DEV)
    O = torch.full_like(Q, 7.0)
    LSE = torch.full((B, H, Nq), 7.0, dtype=torch.float32, device=DEV)
    lens_t = None if lens is None else torch.tensor(lens, dtype=torch.int32, device=DEV)
    nbytes = attn.attn_fwd_kvcache_workspace_bytes(B, H, Hk, Nq, Nk, d, splits)
    ws = torch.full((max(nbytes, 16) // 4,), float("nan"), dtype=torch.float32, device=DEV) if nbytes else None
    attn.attn_fwd_kvcache(Q, K, V, O, LSE, lens_t, causal, scale, splits, ws)
    assert attn.attn_check_status() == attn.ATTN_OK
    O_ref, L_ref = _oracle(q, k, v, scale, causal, lens)
    o, l = f64(O), f64(LSE)
    empty = np.isneginf(L_ref)
    assert (np.isneginf(l) == empty).all(), "rows without visible keys must have LSE = -inf"
    assert (o[empty] == 0).all()
    assert_o(o, O_ref)
    assert_lse(np.where(empty, 0.0, l), np.where(empty, 0.0, L_ref))
    return attn.attn_fwd_kvcache_splits(B, H, Hk, Nq, Nk, d, splits)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nk", [1, 100, 128, 129, 1000, 4097])
def test_decode_single_query(Nk, causal, d):
    _run(2, 8, 2, 1, Nk, d, causal, seed=700 + Nk + d + causal)


@pytest.mark.parametrize("Hk", [1, 4, 16])
@pytest.mark.parametrize("splits", [0, 1, 3, 7])
def test_decode_head_groups_and_splits(Hk, splits):
    s = _run(2, 16, Hk, 1, 2000, 128, True, seed=720 + Hk + splits, splits=splits)
    if splits:
        assert s == splits


@pytest.mark.parametrize("Nq", [2, 7, 37, 130])
@pytest.mark.parametrize("causal", [False, True])
def test_multi_row_queries(Nq, causal):
    # (H / H_kv) * Nq packed rows: 4 * 130 = 520 spans five row tiles with a ragged last one
    _run(2, 8, 2, Nq, 777, 64, causal, seed=740 + Nq + causal, splits=0)
    _run(1, 4, 1, Nq, 777, 128, causal, seed=760 + Nq + causal, splits=2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("splits", [0, 1, 4])
def test_cache_lengths_with_poisoned_tail(causal, splits):
    # lengths: full, ragged, one tile exactly, a single row, empty, shorter than Nq
    lens = [1000, 517, 128, 1, 0, 3]
    _run(6, 4, 2, 5, 1000, 128, causal, seed=780 + causal + splits, lens=lens, splits=splits, poison=True)


def test_square_shape_matches_plain_forward():
    # Nq = Nk: the cache forward is the square forward (top-left = bottom-right)
    B, H, N, d = 1, 4, 300, 64
    _run(B, H, H, N, N, d, True, seed=800)
    g = torch.Generator("cpu").manual_seed(801)
    q, k, v = (torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).to(DEV) for _ in range(3))
    O1, O2 = torch.empty_like(q), torch.empty_like(q)
    L1, L2 = (torch.empty((B, H, N), dtype=torch.float32, device=DEV) for _ in range(2))
    attn.attn_fwd_kvcache(q, k, v, O1, L1, None, True, 0.125, 1, None)
    attn.attn_fwd(q, k, v, O2, L2, True, 0.125)
    assert attn.attn_check_status() == attn.ATTN_OK
    assert np.abs(f64(O1) - f64(O2)).max() <= 2e-2
    assert np.abs(f64(L1) - f64(L2)).max() <= 1e-3


def test_rescale_stress_rows():
    # a few query rows scaled by 8 make tile maxima jump by far more than the
    # lazy-rescale threshold, so the accumulator is rescaled mid-stream
    B, H, Hk, Nq, Nk, d = 1, 8, 2, 3, 3000, 128
    g = torch.Generator("cpu").manual_seed(820)
    q = torch.randn((B, H, Nq, d), generator=g)
    q[0, 1, 2] *= 8.0
    q[0, 5, 0] *= 8.0
    k = torch.randn((B, Hk, Nk, d), generator=g)
    k[0, 0, 2500] *= 6.0                      # one late dominant key
    v = torch.randn((B, Hk, Nk, d), generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    for splits in (1, 5):
        Q, K, V = q.to(DEV), k.to(DEV), v.to(DEV)
        O = torch.empty_like(Q)
        LSE = torch.empty((B, H, Nq), dtype=torch.float32, device=DEV)
        nbytes = attn.attn_fwd_kvcache_workspace_bytes(B, H, Hk, Nq, Nk, d, splits)
        ws = torch.empty((max(nbytes, 16) // 4,), dtype=torch.float32, device=DEV)
        attn.attn_fwd_kvcache(Q, K, V, O, LSE, None, False, scale, splits, ws)
        assert attn.attn_check_status() == attn.ATTN_OK
        O_ref, L_ref = _oracle(q, k, v, scale, False, None)
        assert_o(f64(O), O_ref)
        assert_lse(f64(LSE), L_ref)


def test_decode_long_cache_sampled():
    # decode batch of the long-batch shape: 8 x 32 query heads over 8 shared
    # cache heads of 16384 rows; every row is checked (one query per head)
    B, H, Hk, Nk, d = 8, 32, 8, 16384, 128
    _run(B, H, Hk, 1, Nk, d, True, seed=840)
