"""GPU parity for the packed variable-length forward (attn_fwd_varlen): many
sequences of different lengths in one (total, H, d) buffer, each attending
only to itself.  Checked against the oracle's per-sequence definition, bit
for bit against attn_fwd_gqa run on each sequence alone, and for writes
outside the buffers (guard regions) and outside the sequences."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from oracle import attn_oracle as orc

from ._parity import Guarded, assert_lse, assert_o

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def h64(t):
    """Tensor -> float64 numpy array of the same shape."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def _packed(lens, H, Hk, d, seed, total=None):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1]) if total is None else total
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((total, H, d), generator=g).to(torch.bfloat16)
    k = torch.randn((total, Hk, d), generator=g).to(torch.bfloat16)
    v = torch.randn((total, Hk, d), generator=g).to(torch.bfloat16)
    return cu, q, k, v


def _run(cu, q, k, v, causal, scale, O=None, LSE=None):
    Q, K, V = (t.to(DEV) for t in (q, k, v))
    total, H, d = q.shape
    O = torch.empty_like(Q) if O is None else O
    LSE = torch.empty((H, total), dtype=torch.float32, device=DEV) if LSE is None else LSE
    attn.attn_fwd_varlen(Q, K, V, O, LSE, torch.from_numpy(cu).to(DEV), causal, scale)
    assert attn.attn_check_status() == attn.ATTN_OK
    return O, LSE


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hk", [1, 4])
def test_varlen_against_oracle(Hk, causal, d):
    lens = [1, 127, 0, 128, 129, 300, 64, 513]
    H = 4
    cu, q, k, v = _packed(lens, H, Hk, d, seed=7 + d + Hk)
    scale = 1.0 / math.sqrt(d)
    O, LSE = _run(cu, q, k, v, causal, scale)
    O_ref, L_ref = orc.attn_fwd_varlen(h64(q), h64(k), h64(v), cu, scale, causal, H, Hk)
    assert_o(h64(O), O_ref)
    assert_lse(h64(LSE), L_ref)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_each_sequence_alone_bitwise(causal):
    lens = [300, 5, 0, 1024, 129, 777]
    H, Hk, d = 8, 2, 128
    cu, q, k, v = _packed(lens, H, Hk, d, seed=41)
    scale = 0.09
    O, LSE = _run(cu, q, k, v, causal, scale)
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        seq = lambda t: t[a:b].transpose(0, 1).unsqueeze(0).contiguous().to(DEV)   # (1, heads, len, d)
        qs, ks, vs = seq(q), seq(k), seq(v)
        os_ = torch.empty_like(qs)
        ls = torch.empty((1, H, b - a), dtype=torch.float32, device=DEV)
        attn.attn_fwd_gqa(qs, ks, vs, os_, ls, causal, scale)
        assert torch.equal(O[a:b], os_[0].transpose(0, 1)), (a, b)
        assert torch.equal(LSE[:, a:b], ls[0]), (a, b)


def test_varlen_many_sequences_random_lengths():
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 700, size=37).tolist()
    H, Hk, d = 4, 4, 128
    cu, q, k, v = _packed(lens, H, Hk, d, seed=6)
    O, LSE = _run(cu, q, k, v, True, 0.1)
    O_ref, L_ref = orc.attn_fwd_varlen(h64(q), h64(k), h64(v), cu, 0.1, True, H, Hk)
    assert_o(h64(O), O_ref)
    assert_lse(h64(LSE), L_ref)


def test_varlen_writes_nothing_outside_buffers_or_sequences():
    # tokens past cu_seqlens[-1] belong to no sequence: their rows stay untouched
    lens = [129, 0, 300, 1]
    H, Hk, d = 4, 2, 64
    cu, q, k, v = _packed(lens, H, Hk, d, seed=9, total=int(sum(lens)) + 77)
    total = q.shape[0]
    og, lg = Guarded((total, H, d), torch.bfloat16), Guarded((H, total), torch.float32)
    og.t.fill_(3.0)
    lg.t.fill_(5.0)
    O, LSE = _run(cu, q, k, v, True, 0.125, O=og.t, LSE=lg.t)
    torch.cuda.synchronize()
    assert og.intact() and lg.intact()
    used = int(cu[-1])
    assert bool((O[used:] == 3.0).all()) and bool((LSE[:, used:] == 5.0).all())
    O_ref, L_ref = orc.attn_fwd_varlen(h64(q), h64(k), h64(v), cu, 0.125, True, H, Hk)
    assert_o(h64(O[:used]), O_ref[:used])
    assert_lse(h64(LSE[:, :used]), L_ref[:, :used])
