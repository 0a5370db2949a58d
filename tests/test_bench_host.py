"""Host-side helpers of bench.py (no GPU): the record of logit extremes."""

import importlib.util
import os

import torch

_spec = importlib.util.spec_from_file_location(
    "bench", os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def _brute(q, k, causal):
    qh, kh = q[0, 0].double(), k[0, 0].double()
    best = 0.0
    for i in range(qh.shape[0]):
        for j in range(kh.shape[0]):
            if causal and j > i:
                continue
            best = max(best, abs(float(qh[i] @ kh[j])))
    return best


def test_logit_extremes_match_brute_force_over_chunks():
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 2, 37, 16, generator=g).bfloat16()
    k = torch.randn(1, 2, 37, 16, generator=g).bfloat16()
    for causal in (False, True):
        r = bench.logit_extremes(q, k, 0.25, causal, rows_per_chunk=8)
        assert abs(r["max_abs_raw"] - _brute(q, k, causal)) < 1e-4
        assert abs(r["max_abs_scaled"] - 0.25 * r["max_abs_raw"]) < 1e-6


def test_logit_extremes_ignore_masked_pairs_and_other_heads():
    q = torch.zeros(1, 2, 8, 4)
    k = torch.zeros(1, 2, 8, 4)
    q[0, 0, 0] = 10.0       # row 0 sees only key 0
    k[0, 0, 5] = 1.0        # key 5 is masked for row 0
    k[0, 0, 0, 0] = 0.5
    q[0, 1] = 100.0         # another head: not sampled
    k[0, 1] = 100.0
    q, k = q.bfloat16(), k.bfloat16()
    assert bench.logit_extremes(q, k, 1.0, True)["max_abs_raw"] == 5.0
    assert bench.logit_extremes(q, k, 1.0, False)["max_abs_raw"] == 40.0


def test_single_rank_time_is_its_own_maximum():
    assert bench.reduce_max_over_ranks(2.5, 1, "cpu") == 2.5
