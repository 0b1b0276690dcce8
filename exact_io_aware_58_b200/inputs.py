"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and describes workload shapes; it holds
none of the attention arithmetic.  Recipe (the same for every workload):

* ``torch.Generator(device).manual_seed(seed)``, then ``torch.randn`` in
  float32 in the order Q, K, V, dO, each of shape (B, H, N, d), each
  multiplied by ``std``.  ``device`` is "cpu" by default; the largest
  workloads draw on the GPU (CPU ``randn`` needs ~30 s per 2^29 values), and
  the oracle is then given a host copy of exactly those bf16 tensors;
* optionally a fraction of query rows is multiplied by ``outlier_mult``
  (rows drawn without replacement by a generator seeded ``seed + 1``), to
  stress the running-max rescaling of online softmax;
* finally everything is rounded to bfloat16 (round to nearest even).

The oracle sees exactly these bf16 values, upcast to float64, so the parity
error measures the kernels and not the input cast.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "outlier_rows", "sample_rows"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: tuple
    std: float = 1.0
    with_dO: bool = True
    outlier_frac: float = 0.0
    outlier_mult: float = 8.0
    check_rows: int = 0
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops_fwd(self, causal: bool) -> float:
        """Counted forward FLOPs: 4 N^2 d per head, halved under the causal mask."""
        f = 4.0 * self.N * self.N * self.d * self.B * self.H
        return f / 2 if causal else f


# The five workloads of the exact-attention study: a tiny fwd+bwd case, a
# forward case with outlier query rows, a d=64 training shape, the long-batch
# case whose naive score buffer is 256 GiB per layer (16K tokens x 32 heads x
# batch 8), and the 100K-token long-context forward (20 GB of scores per head
# if materialised).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, (False,), note="fwd+bwd, non-causal"),
    "fwd_outliers": Workload("fwd_outliers", 8, 16, 2048, 128, (False, True), with_dO=False,
                             outlier_frac=0.01, note="fwd, 1% of query rows x8"),
    "train_d64": Workload("train_d64", 4, 16, 4096, 64, (True,), note="fwd+bwd, causal"),
    "long_batch": Workload("long_batch", 8, 32, 16384, 128, (True,), std=0.5,
                           note="fwd+bwd, causal, N(0, 0.5^2)"),
    "long_context": Workload("long_context", 1, 8, 100000, 128, (True,), with_dO=False,
                             check_rows=512, note="fwd, causal, 512 sampled check rows"),
}


def outlier_rows(B: int, H: int, N: int, frac: float, seed: int) -> torch.Tensor:
    """Flat (b*H + h)*N + i indices of the rows to scale, drawn without replacement."""
    total = B * H * N
    count = int(round(frac * total))
    g = torch.Generator("cpu").manual_seed(seed + 1)
    return torch.randperm(total, generator=g)[:count]


def sample_rows(B: int, H: int, N: int, count: int, seed: int) -> torch.Tensor:
    """``count`` distinct flat (b*H + h)*N + i row indices, uniform, generator ``seed + 2``."""
    total = B * H * N
    g = torch.Generator("cpu").manual_seed(seed + 2)
    return torch.randperm(total, generator=g)[: min(count, total)]


def make_inputs(B: int, H: int, N: int, d: int, seed: int = 0, std: float = 1.0,
                with_dO: bool = True, outlier_frac: float = 0.0,
                outlier_mult: float = 8.0, device="cpu") -> dict:
    """Q, K, V (and dO) as contiguous bf16 tensors of shape (B, H, N, d) on ``device``."""
    g = torch.Generator(device).manual_seed(seed)
    names = ["Q", "K", "V"] + (["dO"] if with_dO else [])
    out = {}
    for name in names:
        x = torch.randn((B, H, N, d), generator=g, dtype=torch.float32, device=device)
        if std != 1.0:
            x.mul_(std)
        if name == "Q" and outlier_frac > 0:
            rows = outlier_rows(B, H, N, outlier_frac, seed).to(x.device)
            x.view(-1, d)[rows] *= outlier_mult
        out[name] = x.to(torch.bfloat16).contiguous()
    return out


def workload_inputs(w: Workload, seed: int = 0, device="cpu") -> dict:
    return make_inputs(w.B, w.H, w.N, w.d, seed=seed, std=w.std, with_dO=w.with_dO,
                       outlier_frac=w.outlier_frac, outlier_mult=w.outlier_mult, device=device)
