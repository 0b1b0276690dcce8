"""Helpers shared by the GPU parity tests: tolerances and comparisons.

Tolerances (bf16 inputs, fp32 accumulation):
  * O:    max |O - O_ref| <= 1e-2 + half an ulp of bf16 at |O_ref|.  The
          kernel's O is bf16; rounding alone costs up to half an ulp, which is
          already 0.0156 for |O| in [4, 8), so a bare 1e-2 bound cannot hold for
          any bf16 output there.  The extra term is exactly that rounding.
  * LSE:  max |LSE - LSE_ref| <= 1e-3 (fp32 output).
  * dQ, dK, dV: max |g - g_ref| <= 2e-2 * max |g_ref| + 1e-5 per tensor.
          The 1e-5 floor only matters where the reference is identically zero:
          with N = 1, dS = P (dP - D) vanishes in exact arithmetic, but the
          kernel's D comes from the bf16 O, so its dS, and dQ, dK, are ~1e-7.
"""

from __future__ import annotations

import numpy as np
import torch

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_REL = 2e-2
GRAD_ABS_FLOOR = 1e-5


def f64(t: torch.Tensor, n: int | None = None, d: int | None = None) -> np.ndarray:
    """bf16/fp32 tensor -> float64 numpy array; 4-D (B,H,N,d) -> (B*H, N, d)."""
    a = t.detach().to("cpu", torch.float32).numpy().astype(np.float64)
    if a.ndim == 4:
        a = a.reshape(-1, a.shape[2], a.shape[3])
    elif a.ndim == 3:
        a = a.reshape(-1, a.shape[2])
    return a


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.exp2(e - 8.0)


def o_error(o: np.ndarray, o_ref: np.ndarray):
    err = np.abs(o - o_ref)
    bound = O_TOL + bf16_half_ulp(o_ref)
    return float(err.max()), bool((err <= bound).all())


def assert_o(o: np.ndarray, o_ref: np.ndarray, what: str = "O"):
    assert np.isfinite(o).all(), f"{what}: non-finite values"
    mx, ok = o_error(o, o_ref)
    assert ok, f"{what}: max |O - O_ref| = {mx:.3e} exceeds 1e-2 + half-ulp(bf16)"


def assert_lse(l: np.ndarray, l_ref: np.ndarray, what: str = "LSE"):
    assert np.isfinite(l).all(), f"{what}: non-finite values"
    mx = float(np.abs(l - l_ref).max())
    assert mx <= LSE_TOL, f"{what}: max |LSE - LSE_ref| = {mx:.3e} > {LSE_TOL}"


def assert_grad(g: np.ndarray, g_ref: np.ndarray, what: str):
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    ref_max = float(np.abs(g_ref).max())
    mx = float(np.abs(g - g_ref).max())
    assert mx <= GRAD_REL * ref_max + GRAD_ABS_FLOOR, \
        f"{what}: max err {mx:.3e} > {GRAD_REL} * {ref_max:.3e} + {GRAD_ABS_FLOOR}"


GUARD = 64 * 1024          # guard bytes on each side (a multiple of 16: views stay 16-byte aligned)
PATTERN = 0xA5


class Guarded:
    """A CUDA tensor of ``shape``/``dtype`` (or of ``nbytes`` bytes, flat) with
    GUARD bytes of PATTERN on both sides, to detect writes outside it."""

    def __init__(self, shape, dtype, nbytes=None, device="cuda:0"):
        elem = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) if nbytes is None else nbytes // elem
        self.g = GUARD // elem
        self.buf = torch.empty(self.g + self.n + self.g, dtype=dtype, device=device)
        self.buf.view(torch.uint8).fill_(PATTERN)
        self.t = self.buf[self.g:self.g + self.n]
        if nbytes is None:
            self.t = self.t.view(shape)

    def intact(self) -> bool:
        raw = self.buf.view(torch.uint8)
        gb = self.g * self.buf.element_size()
        return bool((raw[:gb] == PATTERN).all()) and bool((raw[raw.numel() - gb:] == PATTERN).all())
