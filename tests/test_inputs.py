import torch

from exact_io_aware_58_b200.inputs import WORKLOADS, make_inputs, outlier_rows, sample_rows


def test_inputs_are_seeded_bf16_and_ordered():
    a = make_inputs(1, 2, 33, 8, seed=3)
    b = make_inputs(1, 2, 33, 8, seed=3)
    assert list(a) == ["Q", "K", "V", "dO"]
    for k in a:
        assert a[k].dtype == torch.bfloat16 and a[k].shape == (1, 2, 33, 8)
        assert a[k].is_contiguous()
        assert torch.equal(a[k], b[k])
    # Q, K, V, dO come from one generator in that order.
    g = torch.Generator("cpu").manual_seed(3)
    q = torch.randn((1, 2, 33, 8), generator=g)
    assert torch.equal(a["Q"], q.to(torch.bfloat16))


def test_outlier_rows_scaled_by_eight():
    base = make_inputs(2, 2, 50, 4, seed=0, with_dO=False)
    out = make_inputs(2, 2, 50, 4, seed=0, with_dO=False, outlier_frac=0.05)
    rows = outlier_rows(2, 2, 50, 0.05, 0)
    assert rows.numel() == 10 and rows.unique().numel() == 10
    qb, qo = base["Q"].view(-1, 4).float(), out["Q"].view(-1, 4).float()
    mask = torch.zeros(200, dtype=torch.bool); mask[rows] = True
    assert torch.equal(qo[~mask], qb[~mask])
    assert not torch.equal(qo[mask], qb[mask])


def test_sample_rows_distinct():
    r = sample_rows(1, 8, 1000, 512, 0)
    assert r.numel() == 512 and r.unique().numel() == 512 and int(r.max()) < 8000


def test_workload_table():
    w = WORKLOADS["long_batch"]
    assert (w.B, w.H, w.N, w.d, w.causal, w.std) == (8, 32, 16384, 128, (True,), 0.5)
    assert w.flops_fwd(True) == 4 * 16384**2 * 128 * 256 / 2
