"""Failure detection without a GPU fault, and the device exponentials.

* A kernel whose barrier wait runs out (nothing ever arrives) must give up
  after its cycle budget, record FA_ERR_TIMEOUT, return normally and leave
  the context usable.
* The FMA-pipe exp2 polynomial and the MUFU exp2 against fp64 2^x."""

import numpy as np
import pytest
import torch

from exact_attention_104_b200 import attention_forward, binding
from exact_attention_104_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert binding.fa_device_status() == binding.FA_OK
    assert binding.fa_selftest_wait_timeout(1 << 20) == binding.FA_OK
    assert binding.fa_device_status() == binding.FA_ERR_TIMEOUT
    assert binding.fa_device_status() == binding.FA_OK          # cleared after being read
    w = WORKLOADS["tiny_b1_h2_n128_d64"]
    q, k, v, _ = make_inputs(w, "cuda")
    o, lse = attention_forward(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and binding.fa_device_status() == binding.FA_OK
    assert binding.fa_selftest_wait_timeout(0) == binding.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("use_poly", [False, True])
def test_device_exp2_accuracy(use_poly):
    # dense grid over the softmax argument range (stale max allows up to +8)
    x = torch.linspace(-125.0, 8.0, 1 << 22, dtype=torch.float32, device="cuda")
    x = torch.cat([x, torch.arange(-125, 9, dtype=torch.float32, device="cuda")])   # exact integers
    y = torch.empty_like(x)
    assert binding.fa_selftest_exp2(x, y, use_poly) == binding.FA_OK
    torch.cuda.synchronize()
    xs = x.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs)
    rel = np.abs(y.cpu().numpy().astype(np.float64) / ref - 1)
    if use_poly:
        assert rel.max() <= 1.1e-4                  # fitted bound 1.0e-4, far below bf16's 2^-9
        ints = xs == np.round(xs)
        assert np.all(y.cpu().numpy()[ints] == ref[ints].astype(np.float32))
    else:
        assert rel.max() <= 2.0 ** -20


def test_poly_exp2_underflow_is_tiny_and_non_negative():
    x = torch.tensor([-126.0, -200.0, float("-inf"), -125.5], dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    assert binding.fa_selftest_exp2(x, y, True) == binding.FA_OK
    torch.cuda.synchronize()
    yv = y.cpu().numpy()
    assert np.all(yv >= 0) and np.all(yv < 1e-37)
