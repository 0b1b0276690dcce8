"""The persistent forward walks several work items per CTA, carrying its
barrier phases, K/V ring position and tensor memory from one item to the next
(and, under the causal mask, a separate phase count per query tile, since the
first tile skips the key tile that lies wholly above it).  Every item's
arithmetic is the same whichever CTA runs it and whatever ran before, so a
head computed inside a large launch must equal, bit for bit, the same head
computed alone (one item per CTA).  A wrong phase, ring slot or skipped tile
in the item loop shows up here as a difference in some head."""

import math

import pytest
import torch

from exact_io_aware_58_b200 import attn

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).to(DEV)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 1024, 2048, 2500])
def test_heads_in_a_large_launch_equal_heads_alone(N, causal, d):
    B, H = 1, 48       # 48 heads x ceil(N/256) items: more items than SMs from N = 1024 on
    q, k, v = (_rand((B, H, N, d), seed=N + d + i) for i in range(3))
    scale = 1.0 / math.sqrt(d)
    O = torch.empty_like(q)
    LSE = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    attn.attn_fwd(q, k, v, O, LSE, causal, scale)
    assert attn.attn_check_status() == attn.ATTN_OK
    for h in range(H):
        one = lambda t: t[:, h:h + 1].contiguous()
        o1 = torch.empty((B, 1, N, d), dtype=torch.bfloat16, device=DEV)
        l1 = torch.empty((B, 1, N), dtype=torch.float32, device=DEV)
        attn.attn_fwd(one(q), one(k), one(v), o1, l1, causal, scale)
        assert torch.equal(O[:, h:h + 1], o1), f"O of head {h} differs"
        assert torch.equal(LSE[:, h:h + 1], l1), f"LSE of head {h} differs"
    assert attn.attn_check_status() == attn.ATTN_OK


@pytest.mark.parametrize("causal", [False, True])
def test_shared_kv_heads_in_a_large_launch_equal_groups_alone(causal):
    B, H, Hk, N, d = 2, 32, 4, 1536, 128   # 2 x 32 x 6 = 384 items
    q = _rand((B, H, N, d), seed=11)
    k, v = _rand((B, Hk, N, d), seed=12), _rand((B, Hk, N, d), seed=13)
    scale = 0.1
    O = torch.empty_like(q)
    LSE = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    attn.attn_fwd_gqa(q, k, v, O, LSE, causal, scale)
    assert attn.attn_check_status() == attn.ATTN_OK
    g = H // Hk
    for b in range(B):
        for hk in range(Hk):
            qs = q[b:b + 1, hk * g:(hk + 1) * g].contiguous()
            ks, vs = k[b:b + 1, hk:hk + 1].contiguous(), v[b:b + 1, hk:hk + 1].contiguous()
            o1 = torch.empty_like(qs)
            l1 = torch.empty((1, g, N), dtype=torch.float32, device=DEV)
            attn.attn_fwd_gqa(qs, ks, vs, o1, l1, causal, scale)
            assert torch.equal(O[b:b + 1, hk * g:(hk + 1) * g], o1), (b, hk)
            assert torch.equal(LSE[b:b + 1, hk * g:(hk + 1) * g], l1), (b, hk)
