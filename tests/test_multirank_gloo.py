"""N>1 path on CPU: two gloo ranks.  Heads are sharded across ranks with no
collective on the data path; each rank's share, computed independently,
reassembles into the single-process result; timing is reduced as the max over
ranks; the whole-job value counts every rank's work."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_58_b200.multi import aggregate_tflops, max_over_ranks, rank_seed, shard_range


def test_shard_range_covers_exactly():
    for total in (1, 2, 7, 256, 1000):
        for world in (1, 2, 3, 8):
            spans = [shard_range(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (a, b), (c, _) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_aggregate_value():
    assert aggregate_tflops(1e12, 4, 1000.0) == pytest.approx(4.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_io_aware_58_b200.inputs import make_inputs
        from oracle import attn_oracle as orc

        # one batch, heads split across ranks
        B, H, N, d = 1, 5, 40, 8
        inp = make_inputs(B, H, N, d, seed=3)
        a, b = shard_range(B * H, world, rank)
        Q, K, V, dO = (inp[n].float().numpy().astype(np.float64).reshape(B * H, N, d) for n in ("Q", "K", "V", "dO"))
        O, L = orc.attn_fwd(Q[a:b], K[a:b], V[a:b], 0.35, True)
        dQ, dK, dV = orc.attn_bwd(Q[a:b], K[a:b], V[a:b], dO[a:b], 0.35, True)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), O=O, L=L, dQ=dQ, dK=dK, dV=dV, a=a, b=b)
        # timing reduction: each rank reports a different time; all see the max
        ms = max_over_ranks([10.0 + rank, 5.0 * (world - rank)])
        assert ms == [10.0 + world - 1, 5.0 * world]
        # weak scaling: ranks draw distinct batches
        seeds = [None] * world
        dist.all_gather_object(seeds, rank_seed(1234, rank))
        assert len(set(seeds)) == world
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_full_result(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    from exact_io_aware_58_b200.inputs import make_inputs
    from oracle import attn_oracle as orc

    B, H, N, d = 1, 5, 40, 8
    inp = make_inputs(B, H, N, d, seed=3)
    Q, K, V, dO = (inp[n].float().numpy().astype(np.float64).reshape(B * H, N, d) for n in ("Q", "K", "V", "dO"))
    O, L = orc.attn_fwd(Q, K, V, 0.35, True)
    dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, 0.35, True)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    covered = sorted((int(p["a"]), int(p["b"])) for p in parts)
    assert covered[0][0] == 0 and covered[-1][1] == B * H
    for name, full in (("O", O), ("L", L), ("dQ", dQ), ("dK", dK), ("dV", dV)):
        got = np.concatenate([p[name] for p in sorted(parts, key=lambda p: int(p["a"]))])
        np.testing.assert_array_equal(got, full)


# ---------------------------------------------------------------------------
# The benchmark's per-rank loop (multi.run_timed) with a host clock and a stub
# step in place of the kernels: barrier + sync around the timed steps, the
# per-segment means, the max over ranks and the whole-job value.
# ---------------------------------------------------------------------------

class _HostClock:
    def mark(self):
        import time
        return time.perf_counter()

    @staticmethod
    def elapsed_ms(a, b):
        return (b - a) * 1e3

    @staticmethod
    def sync():
        pass


def _bench_worker(rank, world, port, out_dir):
    import json
    import time

    from exact_io_aware_58_b200.multi import run_timed

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        calls = []
        nap = 0.004 * (1 + rank)          # rank 1 is the slower one

        def step(mark):                   # two "kernels" per step, marked in between
            calls.append(rank)
            time.sleep(nap)
            mark()
            time.sleep(nap / 2)

        total, seg = run_timed(step, steps=5, warmup=3, clock=_HostClock(), barrier=dist.barrier, n_segments=2)
        assert len(calls) == 8
        vals = max_over_ranks([total] + seg)
        value = aggregate_tflops(1e9, world, vals[0] / 5)
        with open(os.path.join(out_dir, f"b{rank}.json"), "w") as f:
            json.dump({"local": [total] + seg, "max": vals, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_bench_rank_loop_two_gloo_ranks(tmp_path):
    import json

    world = 2
    mp.spawn(_bench_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"b{r}.json")) for r in range(world)]
    # every rank reports the same max, and it is the slower rank's time
    assert res[0]["max"] == res[1]["max"]
    for k in range(3):
        assert res[0]["max"][k] == max(r["local"][k] for r in res)
    assert res[1]["local"][0] > res[0]["local"][0]
    # segment means: ~nap and ~nap/2 per step on the slower rank
    assert res[1]["local"][1] >= 8.0 * 0.95 and res[1]["local"][2] >= 4.0 * 0.95
    # whole-job value: both ranks' work over the slowest rank's per-step time
    assert res[0]["value"] == pytest.approx(1e9 * world / (res[0]["max"][0] / 5 * 1e-3) / 1e12)


def test_rank_envs():
    from exact_io_aware_58_b200.multi import rank_envs

    envs = rank_envs(4, 29511, base_env={"PATH": "/bin"})
    assert [e["RANK"] for e in envs] == ["0", "1", "2", "3"]
    assert [e["LOCAL_RANK"] for e in envs] == ["0", "1", "2", "3"]
    assert all(e["WORLD_SIZE"] == "4" and e["MASTER_ADDR"] == "127.0.0.1" and e["MASTER_PORT"] == "29511"
               and e["PATH"] == "/bin" for e in envs)


def test_bench_gpus_flag_fails_loudly_without_enough_devices():
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "--gpus 2 but only 0 CUDA device" in r.stderr
    env["WORLD_SIZE"] = "2"
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "1"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "must agree" in r.stderr
