"""Failure detection on the GPU without a fault: a kernel's bounded wait runs
out (a barrier that nothing arrives on); the host sees ATTN_ERR_TIMEOUT from
attn_check_status, the status is cleared, and the same context keeps running
attention correctly (the timed-out kernel released its tensor memory, or the
next kernel's allocation could not proceed)."""

import math

import numpy as np
import pytest
import torch

from exact_io_aware_58_b200 import attn
from exact_io_aware_58_b200.inputs import make_inputs
from oracle import attn_oracle as orc

from ._parity import assert_lse, assert_o, f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    assert attn.attn_check_status() == attn.ATTN_OK
    attn.attn_selftest_wait_timeout()
    assert attn.attn_check_status() == attn.ATTN_ERR_TIMEOUT
    assert attn.attn_check_status() == attn.ATTN_OK          # the status word was cleared
    inp = make_inputs(1, 2, 300, 128, seed=5)
    q, k, v = (inp[n].to("cuda:0") for n in ("Q", "K", "V"))
    o, lse = attn.forward(q, k, v, True, 1 / math.sqrt(128))
    assert attn.attn_check_status() == attn.ATTN_OK
    O_ref, L_ref = orc.attn_fwd(f64(inp["Q"]), f64(inp["K"]), f64(inp["V"]), 1 / math.sqrt(128), True)
    assert_o(f64(o), O_ref)
    assert_lse(f64(lse), L_ref)
