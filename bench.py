#!/usr/bin/env python
"""Benchmark: exact attention forward + backward on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: attn_fwd, then the
backward as attn_bwd runs it (attn_bwd_fused_preprocess,
attn_bwd_fused_dkdvdq, attn_bwd_fused_dq_convert), on the long-batch workload
B=8, H=32, N=16384, d=128, causal, bf16 (the configuration whose target is
forward >= 60 % and forward+backward >= 45 % of dense BF16 peak).  Inputs are
1 GiB per tensor (larger than the 126 MB L2), so no L2 flush is needed
between steps.

Metric: attention TFLOP/s of forward+backward, counted as 4 N^2 d per head for
the forward (halved under the causal mask) and 2.5x that for the backward.
The other four workloads (tiny fwd+bwd, the outlier-row forward with both
masks, the d = 64 training shape, the 100K-token causal forward) are measured
in the same run under the key ``configs``; the deterministic backward, shared
key/value heads, block-sparse selection, packed variable-length prefill,
decode against a cache and FP8 have keys of their own.

Multi-GPU: ``--gpus N`` starts N rank processes on this node (one GPU each)
unless it is already running under a launcher that set WORLD_SIZE; every rank
runs its own batch of the same workload (weak scaling, no collective on the
data path); ``value`` is the FLOPs of all ranks over the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on a bounded sample (the exact
causal prefix sub-problem of one head: its first rows/keys), on rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "long_batch"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "attention TFLOP/s fwd and fwd+bwd at 1 B200; % of dense BF16 tensor peak"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "attn_fwd": ("attn_fwd.cuh", "sm100.cuh"),
    "bwd_pre": ("attn_bwd.cuh", "sm100.cuh"),
    "bwd_fused": ("attn_bwd_fused.cuh", "attn_bwd.cuh", "sm100.cuh"),
    "bwd_dq_convert": ("attn_bwd_fused.cuh", "attn_bwd.cuh", "sm100.cuh"),
    "bwd_dkdv": ("attn_bwd.cuh", "sm100.cuh"),
    "bwd_dq": ("attn_bwd.cuh", "sm100.cuh"),
    "kvcache": ("attn_kvcache.cuh", "sm100.cuh"),
    "kvcache_fp8": ("attn_kvcache_fp8.cuh", "attn_kvcache.cuh", "attn_fwd_fp8.cuh", "sm100.cuh"),
    "fp8": ("attn_fwd_fp8.cuh", "sm100.cuh"),
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the source files a kernel is compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_58_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch (read + write) from a committed ncu summary, scaled
    to the full workload, if it was taken on the kernel's current sources."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    ent = rec.get(WORKLOAD, {}).get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.out = os.path.join("/tmp", f"bench_clocks_{os.getpid()}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.out, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.out):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx.append(float(parts[1]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[3:7]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
            os.unlink(self.out)
        except Exception:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def flops_fwd_per_rank(w) -> float:
    return w.flops_fwd(True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from exact_io_aware_58_b200 import attn
    from exact_io_aware_58_b200.inputs import WORKLOADS, workload_inputs
    from exact_io_aware_58_b200.multi import CudaClock, aggregate_tflops, max_over_ranks, rank_seed, run_timed

    wname = args.workload
    w = WORKLOADS[wname]
    resized = bool(args.batch or args.heads or args.seq)
    if resized:
        # smaller cases of the same kernels, for profiler captures only
        import dataclasses
        w = dataclasses.replace(w, B=args.batch or w.B, H=args.heads or w.H, N=args.seq or w.N)

    def traffic(kernel):
        # the committed DRAM records are per launch of the full long-batch step
        return recorded_traffic(kernel) if (wname == WORKLOAD and not resized) else None

    tensor_mb = w.B * w.H * w.N * w.d * 2 / 1e6
    l2_note = (f"inputs {tensor_mb:.0f} MB per tensor > 126 MB L2; no flush" if tensor_mb > 126 else
               f"inputs {tensor_mb:.0f} MB per tensor fit the 126 MB L2 (a profiling case, not a bench number)")
    causal = True
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    attn.load_library()
    stream = torch.cuda.current_stream()
    clock = CudaClock(stream)
    barrier = dist.barrier if world > 1 else None

    inp = workload_inputs(w, seed=rank_seed(1234, rank), device=dev)
    q, k, v, do = inp["Q"], inp["K"], inp["V"], inp["dO"]
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = attn.alloc_workspace(w.B, w.H, w.N, w.d, dev)
    scale = w.scale

    # One step = the forward and the three kernels of attn_bwd, each bracketed
    # by CUDA events on the launching stream.
    def step(mark):
        attn.attn_fwd(q, k, v, o, lse, causal, scale, stream)
        mark()
        attn.attn_bwd_fused_preprocess(o, do, lse, ws, stream)
        mark()
        attn.attn_bwd_fused_dkdvdq(q, k, v, do, dk, dv, causal, scale, ws, stream)
        mark()
        attn.attn_bwd_fused_dq_convert(dq, scale, ws, stream)

    sampler = []

    def start_clock_sampler():
        sampler.append(ClockSampler(local_rank))
        time.sleep(0.3)

    total_ms, seg = run_timed(step, args.steps, args.warmup, clock, barrier, n_segments=4,
                              on_timed_start=start_clock_sampler)
    clk = sampler[0].stop()
    st = attn.attn_check_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(f"device status after timed region: {attn.attn_status_string(st)}")

    names = ["attn_fwd", "bwd_pre", "bwd_fused", "bwd_dq_convert"]
    # max over ranks of the timed-region duration and of the per-kernel means
    vals = max_over_ranks([total_ms] + seg, device=dev)
    total_ms = vals[0]
    per_kernel = dict(zip(names, vals[1:]))
    ms_per_step = total_ms / args.steps
    t_fwd = per_kernel["attn_fwd"]
    t_bwd = per_kernel["bwd_pre"] + per_kernel["bwd_fused"] + per_kernel["bwd_dq_convert"]

    f_fwd = flops_fwd_per_rank(w)
    value = aggregate_tflops(3.5 * f_fwd, world, ms_per_step)
    fwd_tflops = aggregate_tflops(f_fwd, world, t_fwd)
    fwdbwd_kernel_tflops = aggregate_tflops(3.5 * f_fwd, world, t_fwd + t_bwd)

    peaks, peaks_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))

    # Roofline of the dominant kernel: algorithmic FLOPs per launch (GEMMs on
    # the causal half of the score matrix: forward 2; fused backward 5 = the
    # 2.5x backward count) over its CUDA-event mean duration, against the
    # measured burst peak (the sustained figure was measured at a lower SM
    # clock than these kernels run at, so it would overstate the fraction; it
    # is reported beside it).
    alg = {"attn_fwd": f_fwd, "bwd_fused": 2.5 * f_fwd}
    dom = max(alg, key=lambda kname: per_kernel[kname])
    achieved = alg[dom] / (per_kernel[dom] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": burst,
                "peak_kind": f"bf16_tflops burst ({peaks_src})", "unit": "TFLOP/s",
                "frac": round(achieved / burst, 4), "frac_of_sustained": round(achieved / sustained, 4),
                "frac_of_datasheet_2250": round(achieved / 2250.0, 4),
                "alg_flops_per_launch": alg[dom], "traffic": traffic(dom)}

    peak_mem = torch.cuda.max_memory_allocated(dev)

    # --------------------------------------- deterministic backward (3 kernels)
    det = None
    if not args.no_det:
        wsd = attn.alloc_workspace(w.B, w.H, w.N, w.d, dev, deterministic=True)

        def det_step(mark):
            attn.attn_bwd_preprocess(o, do, lse, wsd, stream)
            mark()
            attn.attn_bwd_dkdv(q, k, v, do, dk, dv, causal, scale, wsd, stream)
            mark()
            attn.attn_bwd_dq(q, k, v, do, dq, causal, scale, wsd, stream)

        n_d = max(3, min(args.steps, 5))
        _, dseg = run_timed(det_step, n_d, args.warmup, clock, barrier, n_segments=3)
        assert attn.attn_check_status(stream) == attn.ATTN_OK
        dseg = max_over_ranks(dseg, device=dev)
        det = {"kernel_ms": {"bwd_pre": round(dseg[0], 3), "bwd_dkdv": round(dseg[1], 3), "bwd_dq": round(dseg[2], 3)},
               "bwd_tflops": round(aggregate_tflops(2.5 * f_fwd, world, sum(dseg)), 2),
               "fwdbwd_tflops": round(aggregate_tflops(3.5 * f_fwd, world, t_fwd + sum(dseg)), 2),
               "steps": n_d, "note": "bitwise-reproducible path (separate dK/dV and dQ kernels, 7 GEMMs per tile pair)"}
        del wsd

    # ------------------------------------------------- shared key/value heads
    gqa = None
    if not args.no_gqa and w.H % args.gqa_kv_heads == 0:
        hk = args.gqa_kv_heads
        kg, vg = k[:, :hk].contiguous(), v[:, :hk].contiguous()
        dkg, dvg = torch.empty_like(kg), torch.empty_like(vg)

        def gqa_step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            attn.attn_fwd_gqa(q, kg, vg, o, lse, causal, scale, stream)
            if ev is not None:
                ev[1].record(stream)
            attn.attn_bwd_gqa(q, kg, vg, o, do, lse, dq, dkg, dvg, causal, scale, ws, stream)
            if ev is not None:
                ev[2].record(stream)

        for _ in range(args.warmup):
            gqa_step()
        n_g = max(3, min(args.steps, 5))
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_g)]
        torch.cuda.synchronize()
        for e in gev:
            gqa_step(e)
        torch.cuda.synchronize()
        assert attn.attn_check_status(stream) == attn.ATTN_OK
        gf = sum(e[0].elapsed_time(e[1]) for e in gev) / n_g
        gb = sum(e[1].elapsed_time(e[2]) for e in gev) / n_g
        gf, gb = max_over_ranks([gf, gb], device=dev)
        gqa = {"H_kv": hk, "group": w.H // hk, "ms_fwd": round(gf, 3), "ms_bwd": round(gb, 3),
               "fwd_tflops": round(aggregate_tflops(f_fwd, world, gf), 2),
               "fwdbwd_tflops": round(aggregate_tflops(3.5 * f_fwd, world, gf + gb), 2), "steps": n_g}
        del kg, vg, dkg, dvg

    # ------------------------------------------------- block-sparse selection
    sparse = None
    if not args.no_sparse:
        import numpy as np
        nt = (w.N + 127) // 128
        ii, jj = np.meshgrid(np.arange(nt), np.arange(nt), indexing="ij")
        sel = ((ii - jj >= 0) & (ii - jj < args.sparse_window)) | (jj < args.sparse_sink)
        sel &= jj <= ii                                    # causal: tiles above the diagonal are never visible
        # visible score entries: full tiles below the diagonal, 128*129/2 on it
        vis = float(np.sum(np.where(ii == jj, 128 * 129 / 2, 128 * 128) * sel))
        f_sparse = 4.0 * w.d * vis * w.B * w.H
        mask = torch.from_numpy(np.broadcast_to(sel.astype(np.uint8), (w.B, w.H, nt, nt)).copy()).to(dev)

        def sparse_step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            attn.attn_fwd_blocksparse(q, k, v, o, lse, mask, causal, scale, stream)
            if ev is not None:
                ev[1].record(stream)
            attn.attn_bwd_blocksparse(q, k, v, o, do, lse, mask, dq, dk, dv, causal, scale, ws, stream)
            if ev is not None:
                ev[2].record(stream)

        for _ in range(args.warmup):
            sparse_step()
        n_s = max(3, min(args.steps, 5))
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_s)]
        torch.cuda.synchronize()
        for e in sev:
            sparse_step(e)
        torch.cuda.synchronize()
        assert attn.attn_check_status(stream) == attn.ATTN_OK
        sf = sum(e[0].elapsed_time(e[1]) for e in sev) / n_s
        sb = sum(e[1].elapsed_time(e[2]) for e in sev) / n_s
        sf, sb = max_over_ranks([sf, sb], device=dev)
        sparse = {"pattern": f"causal sliding window of {args.sparse_window} key tiles + first {args.sparse_sink} tiles",
                  "tile_density_vs_causal": round(float(sel.sum()) / float((jj <= ii).sum()), 4),
                  "ms_fwd": round(sf, 3), "ms_bwd": round(sb, 3),
                  "fwd_tflops": round(aggregate_tflops(f_sparse, world, sf), 2),
                  "fwdbwd_tflops": round(aggregate_tflops(3.5 * f_sparse, world, sf + sb), 2), "steps": n_s}
        del mask

    # ------------------------------------- packed variable-length prefill
    # 16 sequences of lengths drawn uniformly in [N/16, N] in one packed
    # (total, H, d) buffer (cu_seqlens), causal, the long-batch heads and
    # head dim; FLOPs counted per sequence (4 L^2 d per head, halved causal).
    varlen = None
    if not args.no_varlen:
        gen = torch.Generator("cpu").manual_seed(rank_seed(77, rank))
        lens = torch.randint(w.N // 16, w.N + 1, (16,), generator=gen).tolist()
        cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0).tolist()), dtype=torch.int32)
        total = int(cu[-1])
        gv = torch.Generator(dev).manual_seed(rank_seed(78, rank))
        qv, kv_, vv = (torch.randn((total, w.H, w.d), generator=gv, device=dev).mul_(w.std).to(torch.bfloat16)
                       for _ in range(3))
        ov = torch.empty_like(qv)
        lv = torch.empty((w.H, total), dtype=torch.float32, device=dev)
        cud = cu.to(dev)
        f_var = sum(4.0 * L * L * w.d * w.H / 2 for L in lens)

        def var_step(mark):
            attn.attn_fwd_varlen(qv, kv_, vv, ov, lv, cud, causal, scale, stream)

        n_v = max(3, min(args.steps, 5))
        _, vseg = run_timed(var_step, n_v, args.warmup, clock, barrier, n_segments=1)
        assert attn.attn_check_status(stream) == attn.ATTN_OK
        tv = max_over_ranks(vseg, device=dev)[0]
        varlen = {"workload": f"16 packed sequences, lengths uniform in [N/16, N] (total {total} tokens), "
                              f"H={w.H}, d={w.d}, causal", "ms_fwd": round(tv, 3),
                  "fwd_tflops": round(aggregate_tflops(f_var, world, tv), 2),
                  "fwd_of_burst": round(aggregate_tflops(f_var, world, tv) / world / burst, 4), "steps": n_v}
        del qv, kv_, vv, ov, lv

    # ------------------------------------------- decode against a KV cache
    # One new query row per head of the same batch against a cache of N rows
    # held in H_kv shared key/value heads: HBM-bound (each cache byte is used
    # by H / H_kv query rows), so its roofline is the measured copy bandwidth.
    kvcache = None
    if not args.no_kvcache and w.H % args.gqa_kv_heads == 0:
        hk = args.gqa_kv_heads
        kc, vc = k[:, :hk].contiguous(), v[:, :hk].contiguous()
        qd = q[:, :, -1:].contiguous()
        od = torch.empty_like(qd)
        lsed = torch.empty((w.B, w.H, 1), dtype=torch.float32, device=dev)
        gen = torch.Generator("cpu").manual_seed(rank_seed(99, rank))
        lens_var = torch.randint(w.N // 2, w.N + 1, (w.B,), generator=gen, dtype=torch.int32)
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        kvcache = {"workload": f"decode: B={w.B}, H={w.H}, H_kv={hk}, Nq=1, Nk={w.N}, d={w.d}, causal",
                   "peak_gbs": hbm, "peak_kind": f"hbm_gbs ({peaks_src})"}
        for name, lens in (("full", None), ("varlen", lens_var)):
            lens_dev = None if lens is None else lens.to(dev)
            splits = attn.attn_fwd_kvcache_splits(w.B, w.H, hk, 1, w.N, w.d, 0)
            wsb = attn.attn_fwd_kvcache_workspace_bytes(w.B, w.H, hk, 1, w.N, w.d, 0)
            wsd = torch.empty((max(wsb, 16) // 4,), dtype=torch.float32, device=dev)
            rows_read = w.B * w.N if lens is None else int(lens.sum())
            alg_bytes = rows_read * hk * w.d * 2 * 2 + 2 * qd.numel() * 2 + lsed.numel() * 4

            def dec():
                attn.attn_fwd_kvcache(qd, kc, vc, od, lsed, lens_dev, causal, scale, 0, wsd, stream)

            for _ in range(max(3, args.warmup)):
                dec()
            # One event pair around back-to-back calls: a call is ~0.1 ms of GPU
            # work, so per-call event pairs would also time the host's launch gap.
            n_d = 50
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(n_d):
                dec()
            ev1.record(stream)
            torch.cuda.synchronize()
            assert attn.attn_check_status(stream) == attn.ATTN_OK
            t_us = ev0.elapsed_time(ev1) / n_d * 1e3
            t_us = max_over_ranks([t_us], device=dev)[0]
            gbs = alg_bytes / (t_us * 1e-6) / 1e9
            kvcache[name] = {"splits": splits, "us": round(t_us, 2), "alg_bytes": alg_bytes,
                             "gb_s": round(gbs, 1), "frac": round(gbs / hbm, 4), "calls": n_d,
                             "traffic": traffic("kvcache") if lens is None else None,
                             "kv_lens": None if lens is None else "uniform in [N/2, N] per batch entry"}
            del wsd
        # the same decode with the cache stored in E4M3 (per-tensor scales): half the bytes
        if w.d == 128:
            kd8 = float(kc.abs().amax()) / 448.0
            vd8 = float(vc.abs().amax()) / 448.0
            kc8 = (kc.float() / kd8).to(torch.float8_e4m3fn)
            vc8 = (vc.float() / vd8).to(torch.float8_e4m3fn)
            wsb = attn.attn_fwd_kvcache_workspace_bytes(w.B, w.H, hk, 1, w.N, w.d, 0)
            wsd = torch.empty((max(wsb, 16) // 4,), dtype=torch.float32, device=dev)

            def dec8():
                attn.attn_fwd_kvcache_fp8(qd, kc8, vc8, od, lsed, None, causal, scale, kd8, vd8, 0, wsd, stream)

            for _ in range(max(3, args.warmup)):
                dec8()
            n_d = 50
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(n_d):
                dec8()
            ev1.record(stream)
            torch.cuda.synchronize()
            assert attn.attn_check_status(stream) == attn.ATTN_OK
            t_us = max_over_ranks([ev0.elapsed_time(ev1) / n_d * 1e3], device=dev)[0]
            alg_bytes = w.B * w.N * hk * w.d * 2 + 2 * qd.numel() * 2 + lsed.numel() * 4
            gbs = alg_bytes / (t_us * 1e-6) / 1e9
            kvcache["fp8_cache"] = {"us": round(t_us, 2), "alg_bytes": alg_bytes, "gb_s": round(gbs, 1),
                                    "frac": round(gbs / hbm, 4), "calls": n_d,
                                    "traffic": traffic("kvcache_fp8"),
                                    "cache": "K, V in E4M3 with per-tensor scales (1 byte per element)"}
            if not args.no_cpu_baseline and rank == 0:
                # the oracle (as it stands) on batch entry 0 of the same decode
                import numpy as np
                from oracle import attn_oracle as orc
                codes = lambda t: t[0:1].view(torch.uint8).cpu().numpy().reshape(-1, w.N, w.d)
                Q64 = qd[0:1].float().cpu().numpy().astype(np.float64).reshape(-1, 1, w.d)
                K8h, V8h = codes(kc8), codes(vc8)
                t = time.perf_counter()
                orc.attn_fwd_kvcache_fp8(Q64, K8h, V8h, kd8, vd8, scale, causal, 1, w.H, hk)
                dt = time.perf_counter() - t
                b1 = hk * w.N * w.d * 2
                kvcache["fp8_cache"]["cpu_oracle"] = {
                    "value": round(b1 / dt / 1e9, 3), "unit": "GB/s", "seconds": round(dt, 3), "kind": "oracle",
                    "sample": "batch entry 0 of the E4M3-cache decode, fp64 numpy"}
            del kc8, vc8, wsd
        if not args.no_cpu_baseline and rank == 0:
            # the oracle (as it stands) on batch entry 0 of the full-cache decode
            import numpy as np
            from oracle import attn_oracle as orc
            h64 = lambda t: t.float().cpu().numpy().astype(np.float64).reshape(-1, t.shape[2], t.shape[3])
            Qh, Kh, Vh = h64(qd[0:1]), h64(kc[0:1]), h64(vc[0:1])
            t = time.perf_counter()
            orc.attn_fwd_kvcache(Qh, Kh, Vh, scale, causal, 1, w.H, hk)
            dt = time.perf_counter() - t
            b1 = hk * w.N * w.d * 2 * 2
            kvcache["cpu_oracle"] = {"value": round(b1 / dt / 1e9, 3), "unit": "GB/s", "seconds": round(dt, 3),
                                     "kind": "oracle", "sample": "batch entry 0 of the full-cache decode, fp64 numpy"}
        del kc, vc

    # ---------------------------------------------------- FP8 (E4M3) forward
    # Same workload and FLOP count as the bf16 forward, inputs quantised per
    # tensor to E4M3; its tensor peak is the measured bf16 peak x 2 (the
    # nominal E4M3 : BF16 dense ratio, 4.5 : 2.25 PFLOP/s).
    fp8 = None
    if not args.no_fp8 and w.d == 128:
        def q8(x):
            ds = float(x.abs().amax()) / 448.0
            return (x.float() / ds).to(torch.float8_e4m3fn), ds

        (qf, dq8), (kf, dk8), (vf, dv8) = q8(q), q8(k), q8(v)

        def fp8_fwd():
            attn.attn_fwd_fp8(qf, kf, vf, o, lse, causal, scale, dq8, dk8, dv8, stream)

        for _ in range(args.warmup):
            fp8_fwd()
        n_f = max(3, min(args.steps, 5))
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_f)]
        torch.cuda.synchronize()
        for e in fev:
            e[0].record(stream)
            fp8_fwd()
            e[1].record(stream)
        torch.cuda.synchronize()
        assert attn.attn_check_status(stream) == attn.ATTN_OK
        tf = sum(e[0].elapsed_time(e[1]) for e in fev) / n_f
        tf = max_over_ranks([tf], device=dev)[0]
        fp8_tf = aggregate_tflops(f_fwd, world, tf)
        fp8 = {"workload": "long_batch forward on E4M3 Q, K, V (per-tensor scales)", "ms_fwd": round(tf, 3),
               "fwd_tflops": round(fp8_tf, 2), "peak": round(2 * burst, 1),
               "peak_kind": f"2 x bf16_tflops ({peaks_src}), nominal E4M3:BF16 ratio",
               "frac": round(fp8_tf / (2 * burst), 4),
               # every exponential on MUFU: 2 x 128 x 128 ex2 per 128-key step at 16 per SM
               # cycle (2048 cycles) against 1024 cycles of E4M3 products caps it at half the peak
               "mufu_cap_frac": 0.5, "frac_of_mufu_cap": round(fp8_tf / (2 * burst) / 0.5, 4),
               "steps": n_f, "traffic": traffic("fp8")}
        if not args.no_cpu_baseline and rank == 0:
            # the oracle on the causal prefix of head (0, 0): first 4096 rows and keys
            import numpy as np
            from oracle import attn_oracle as orc
            rows = 4096
            c8 = lambda t: t[0, 0, :rows].view(torch.uint8).cpu().numpy()[None]
            t = time.perf_counter()
            orc.attn_fwd_fp8(c8(qf), c8(kf), c8(vf), dq8, dk8, dv8, scale, causal, 1, 1, 1)
            dt = time.perf_counter() - t
            fp8["cpu_oracle"] = {"value": round(4.0 * rows * rows * w.d / 2 / dt / 1e12, 6), "unit": "TFLOP/s",
                                 "seconds": round(dt, 3), "kind": "oracle",
                                 "sample": f"causal prefix of head (0,0): first {rows} rows, forward, fp64 numpy"}
        del qf, kf, vf

    # ------------------------------------------- the other four workloads
    configs = None
    if not args.no_configs:
        configs = measure_configs(args, rank, world, dev, stream, clock, barrier, burst, peaks_src)

    # ---------------------------------------------------------------- e2e
    # Through host buffers: every step copies its inputs Q, K, V, dO from
    # pinned host memory to the device and its results O, LSE, dQ, dK, dV back.
    # Steps are pipelined over three streams with two device buffer sets, so
    # step i+1's upload and step i-1's download overlap step i's kernels.
    e2e = None
    if not args.no_e2e:
        del inp
        sets = []
        for b in range(2):
            dev_in = [torch.empty_like(q) for _ in range(4)]
            dev_out = [torch.empty_like(q), torch.empty_like(lse), torch.empty_like(q), torch.empty_like(q),
                       torch.empty_like(q)]
            host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out]
            sets.append((dev_in, dev_out, host_out))
        host_in = [t.cpu().pin_memory() for t in (q, k, v, do)]
        s_up, s_run, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_run = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]
        for e in ev_run + ev_down:
            e.record(s_run)

        def e2e_step(i):
            b = i % 2
            dev_in, dev_out, host_out = sets[b]
            with torch.cuda.stream(s_up):
                s_up.wait_event(ev_run[b])          # inputs of step i-2 no longer read
                for dst, src in zip(dev_in, host_in):
                    dst.copy_(src, non_blocking=True)
                ev_up[b].record(s_up)
            s_run.wait_event(ev_up[b])
            s_run.wait_event(ev_down[b])            # outputs of step i-2 already downloaded
            qi, ki, vi, doi = dev_in
            oo, ll, dqo, dko, dvo = dev_out
            attn.attn_fwd(qi, ki, vi, oo, ll, causal, scale, s_run)
            attn.attn_bwd(qi, ki, vi, oo, doi, ll, dqo, dko, dvo, causal, scale, ws, s_run)
            ev_run[b].record(s_run)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_run[b])
                for dst, src in zip(host_out, dev_out):
                    dst.copy_(src, non_blocking=True)
                ev_down[b].record(s_down)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_up)
        for i in range(n_e2e):
            e2e_step(i)
        b_.record(s_down)
        torch.cuda.synchronize()
        e_ms = max_over_ranks([a.elapsed_time(b_) / n_e2e], device=dev)[0]
        elt = q.element_size()
        h2d = 4 * q.numel() * elt
        d2h = 4 * q.numel() * elt + lse.numel() * 4
        e2e = {"value": round(aggregate_tflops(3.5 * f_fwd, world, e_ms), 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 3),
               "steps": n_e2e, "pipelined": "upload / kernels / download on three streams, two buffer sets"}
        assert attn.attn_check_status(stream) == attn.ATTN_OK
        del sets, host_in

    # ------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(q[0, 0], k[0, 0], v[0, 0], do[0, 0], w, rows=args.cpu_rows)

    assert world == args.gpus
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0, 0.5^2) bf16 Q, K, V, dO; generated on the device)",
        "config": {"workload": f"{wname}: B={w.B} H={w.H} N={w.N} d={w.d} causal, fwd+bwd per step",
                   "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": True, "scale": scale,
                   "global_batch": w.B * world, "seq_len": w.N, "parallelism": f"dp{world} (heads/batches per rank)",
                   "l2": l2_note},
        "fwd_tflops": round(fwd_tflops, 2),
        "fwdbwd_kernel_tflops": round(fwdbwd_kernel_tflops, 2),
        "pct_of_peak": {
            "fwd_of_burst": round(fwd_tflops / world / burst, 4),
            "fwdbwd_of_burst": round(value / world / burst, 4),
            "fwd_of_sustained": round(fwd_tflops / world / sustained, 4),
            "fwdbwd_of_sustained": round(value / world / sustained, 4),
            "fwd_of_datasheet_2250": round(fwd_tflops / world / 2250.0, 4),
            "fwdbwd_of_datasheet_2250": round(value / world / 2250.0, 4),
            "peaks": peaks_src,
        },
        "kernel_ms": {kname: round(t, 3) for kname, t in per_kernel.items()},
        "roofline": roofline,
        "bwd_deterministic": det,
        "configs": configs,
        "gqa": gqa,
        "block_sparse": sparse,
        "varlen": varlen,
        "kvcache": kvcache,
        "fp8": fp8,
        "gpu_launches": 4 * args.steps,      # attn_fwd + the three kernels of attn_bwd per timed step
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "peak_mem_gib": round(peak_mem / 2**30, 3),
        "naive_score_bytes_per_layer": 2 * w.N * w.N * w.B * w.H,
    }
    return line


def _oracle_threads():
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        threads = max([int(i.get("num_threads", 1)) for i in threadpool_info()] + [1])
    except Exception:
        pass
    return threads


def measure_configs(args, rank, world, dev, stream, clock, barrier, burst, peaks_src):
    """TFLOP/s, peak device memory and a bounded oracle sample for the tiny,
    outlier-row, d = 64 training and 100K-token workloads (the long-batch one
    is the main step).  Each timed step runs ``reps`` back-to-back calls so
    that the short ones are not timed as host launch gaps."""
    import numpy as np
    import torch

    from exact_io_aware_58_b200 import attn
    from exact_io_aware_58_b200.inputs import WORKLOADS, sample_rows, workload_inputs
    from exact_io_aware_58_b200.multi import aggregate_tflops, max_over_ranks, rank_seed, run_timed

    plan = [("tiny", 100), ("fwd_outliers", 10), ("train_d64", 10), ("long_context", 1)]
    out = {}
    for name, reps in plan:
        w = WORKLOADS[name]
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        inp = workload_inputs(w, seed=rank_seed(0, rank), device=dev)
        q, k, v = inp["Q"], inp["K"], inp["V"]
        do = inp.get("dO")
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        with_bwd = do is not None
        if with_bwd:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            ws = attn.alloc_workspace(w.B, w.H, w.N, w.d, dev)
        ent = {"shape": {"B": w.B, "H": w.H, "N": w.N, "d": w.d}, "note": w.note, "reps_per_step": reps}
        for causal in w.causal:
            key = "causal" if causal else "non_causal"

            def step(mark):
                for _ in range(reps):
                    attn.attn_fwd(q, k, v, o, lse, causal, w.scale, stream)
                if with_bwd:
                    mark()
                    for _ in range(reps):
                        attn.attn_bwd(q, k, v, o, do, lse, dq, dk, dv, causal, w.scale, ws, stream)

            n = max(3, min(args.steps, 10))
            _, seg = run_timed(step, n, args.warmup, clock, barrier, n_segments=2 if with_bwd else 1)
            assert attn.attn_check_status(stream) == attn.ATTN_OK
            seg = [x / reps for x in max_over_ranks(seg, device=dev)]
            f = w.flops_fwd(causal)
            r = {"ms_fwd": round(seg[0], 5), "fwd_tflops": round(aggregate_tflops(f, world, seg[0]), 2),
                 "fwd_of_burst": round(aggregate_tflops(f, world, seg[0]) / world / burst, 4)}
            if with_bwd:
                r.update({"ms_bwd": round(seg[1], 5),
                          "fwdbwd_tflops": round(aggregate_tflops(3.5 * f, world, seg[0] + seg[1]), 2),
                          "fwdbwd_of_burst": round(aggregate_tflops(3.5 * f, world, seg[0] + seg[1]) / world / burst,
                                                   4)})
            ent[key] = r
        torch.cuda.synchronize()
        ent["peak_mem_gib"] = round((torch.cuda.max_memory_allocated(dev) - base) / 2**30, 4)
        ent["naive_score_bytes"] = 2 * w.N * w.N * w.B * w.H
        ent["peaks"] = peaks_src

        if rank == 0 and world >= 1 and not args.no_cpu_baseline:
            # the oracle as it stands, on a bounded sample of the same inputs
            from oracle import attn_oracle as orc
            h64 = lambda t: t.float().cpu().numpy().astype(np.float64)
            causal = w.causal[-1]
            if name == "long_context":
                rows = sample_rows(w.B, w.H, w.N, w.check_rows, 0).numpy()
                bh, ii = rows // w.N, rows % w.N
                secs, fl = 0.0, 0.0
                for h in np.unique(bh):
                    sel = ii[bh == h]
                    qh, kh, vh = (h64(t.view(-1, w.N, w.d)[h]) for t in (q, k, v))
                    t0 = time.perf_counter()
                    orc.attn_fwd_rows(qh, kh, vh, w.scale, True, sel)
                    secs += time.perf_counter() - t0
                    fl += float(np.sum(4.0 * (sel + 1) * w.d))
                sample = f"{len(rows)} sampled query rows (all heads), causal forward; full job x{w.N * w.H / len(rows):.0f}"
                full = secs * w.N * w.H / len(rows)
            else:
                heads = 2 if name == "tiny" else 1
                qh, kh, vh = (h64(t.view(-1, w.N, w.d)[:heads]) for t in (q, k, v))
                t0 = time.perf_counter()
                orc.attn_fwd(qh, kh, vh, w.scale, causal)
                if with_bwd:
                    orc.attn_bwd(qh, kh, vh, h64(do.view(-1, w.N, w.d)[:heads]), w.scale, causal)
                secs = time.perf_counter() - t0
                fl = (3.5 if with_bwd else 1.0) * w.flops_fwd(causal) * heads / (w.B * w.H)
                sample = (f"{heads} of {w.B * w.H} heads, {'fwd+bwd' if with_bwd else 'fwd'}, "
                          f"{'causal' if causal else 'non-causal'}")
                full = secs * (w.B * w.H) / heads
            ent["cpu_oracle"] = {"value": round(fl / secs / 1e12, 6), "unit": "TFLOP/s", "seconds": round(secs, 3),
                                 "full_job_seconds_extrapolated": round(full, 1), "cores": _oracle_threads(),
                                 "kind": "oracle", "sample": sample + ", fp64 numpy"}
        out[name] = ent
        del inp, q, k, v, o, lse, do
        if with_bwd:
            del dq, dk, dv, ws
        torch.cuda.empty_cache()
    return out


def cpu_baseline_sample(q, k, v, do, w, rows):
    """The oracle (as it stands) on the exact causal prefix sub-problem of one
    head: its first ``rows`` queries see only its first ``rows`` keys, so this
    is a self-contained forward+backward of size ``rows``."""
    import numpy as np
    import torch

    from oracle import attn_oracle as orc

    def host(t):
        return t[:rows].float().cpu().numpy().astype(np.float64)[None]

    Q, K, V, dO = host(q), host(k), host(v), host(do)
    threads = _oracle_threads()
    t = time.perf_counter()
    orc.attn_fwd(Q, K, V, w.scale, True)
    orc.attn_bwd(Q, K, V, dO, w.scale, True)
    dt = time.perf_counter() - t
    flops = 3.5 * 4.0 * rows * rows * w.d / 2
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"causal prefix of head (0,0): first {rows} query rows and keys, fwd+bwd, fp64 numpy"}


def run_reference(args):
    """The oracle timed on the host cores: --warmup + --steps samples."""
    import torch

    from exact_io_aware_58_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS[WORKLOAD]
    rows = args.ref_rows
    inp = make_inputs(1, 1, rows, w.d, seed=1234, std=w.std)
    q, k, v, do = (inp[n][0, 0] for n in ("Q", "K", "V", "dO"))
    for _ in range(args.warmup):
        cpu_baseline_sample(q, k, v, do, w, rows)
    times = []
    res = None
    for _ in range(args.steps):
        res = cpu_baseline_sample(q, k, v, do, w, rows)
        times.append(res["seconds"])
    ms = 1000.0 * sum(times) / len(times)
    flops = 3.5 * 4.0 * rows * rows * w.d / 2
    value = flops / (ms * 1e-3) / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": args.gpus,          # the launch it belongs to; the work itself runs on host cores
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0, 0.5^2), bf16-rounded, fp64 arithmetic)",
        "config": {"workload": f"{WORKLOAD}: B={w.B} H={w.H} N={w.N} d={w.d} causal, fwd+bwd per step",
                   "sample": res["sample"] if res else None},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": res["cores"] if res else None,
                         "kind": "oracle", "sample": res["sample"] if res else None},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def spawn_ranks(n: int) -> int:
    """Run this script as ``n`` rank processes on this node, one GPU each, and
    return the first non-zero exit code (0 if all succeed).  Rank 0 prints the
    JSON line."""
    import socket

    import torch

    from exact_io_aware_58_b200.multi import rank_envs

    visible = torch.cuda.device_count()
    if visible < n:
        raise SystemExit(f"bench.py: --gpus {n} but only {visible} CUDA device(s) are visible")
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [subprocess.Popen([sys.executable, os.path.abspath(__file__), *sys.argv[1:]], env=env)
             for env in rank_envs(n, port)]
    rcs = [p.wait() for p in procs]
    return next((rc for rc in rcs if rc != 0), 0)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gqa", action="store_true", help="skip the shared key/value head measurement")
    ap.add_argument("--no-kvcache", action="store_true", help="skip the decode (key/value cache) measurement")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 forward measurement")
    ap.add_argument("--gqa-kv-heads", type=int, default=8)
    ap.add_argument("--no-sparse", action="store_true", help="skip the block-sparse measurement")
    ap.add_argument("--no-det", action="store_true", help="skip the deterministic backward measurement")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed variable-length prefill measurement")
    ap.add_argument("--no-configs", action="store_true", help="skip the other four workloads")
    ap.add_argument("--sparse-window", type=int, default=16)
    ap.add_argument("--sparse-sink", type=int, default=2)
    ap.add_argument("--cpu-rows", type=int, default=16384)
    ap.add_argument("--ref-rows", type=int, default=8192)
    ap.add_argument("--batch", type=int, default=0, help="override B (profiling captures only)")
    ap.add_argument("--heads", type=int, default=0, help="override H (profiling captures only)")
    ap.add_argument("--seq", type=int, default=0, help="override N (profiling captures only)")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=("tiny", "train_d64", "long_batch"),
                    help="the step's workload (fwd+bwd, causal), for profiling captures only: the bench line is long_batch")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    launched = "WORLD_SIZE" in os.environ
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # host cores only: rank 0 prints the line, other ranks exit without work
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if not launched and args.gpus > 1:
        sys.exit(spawn_ranks(args.gpus))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; they must agree")

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
