"""Host-side helpers of bench.py (no GPU): the record of logit extremes and the
bounded CPU-oracle sample."""

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


def test_cpu_sample_rows_are_bounded_strided_and_rotate():
    from exact_attention_104_b200.workloads import WORKLOADS
    w = WORKLOADS["long_b1_h16_n16384_d128_causal"]
    seen = set()
    for step in range(3 * w.Hq):
        h, rows = bench.cpu_sample_rows(w, step)
        assert h == step % w.Hq
        assert len(rows) == bench.CPU_BLOCK_ENTRIES // w.N
        assert rows.min() >= 0 and rows.max() < w.N
        assert (rows[1:] - rows[:-1] == w.N // len(rows)).all()
        seen.add(int(rows[0]))
    assert seen == {0, 1, 2}
    # a short sequence is sampled whole
    h, rows = bench.cpu_sample_rows(WORKLOADS["train_b8_h16_n2048_d128"], 5)
    assert h == 5 and list(rows) == list(range(2048))


def test_cpu_sample_flops_count_visible_pairs():
    import numpy as np
    from exact_attention_104_b200.workloads import Workload
    rows = np.array([0, 3, 9])
    causal = Workload("c", 1, 1, 1, 10, 64, True)
    full = Workload("f", 1, 1, 1, 10, 64, False)
    assert bench.cpu_sample_flops(causal, rows) == 3.5 * 4 * 64 * (1 + 4 + 10)
    assert bench.cpu_sample_flops(full, rows) == 3.5 * 4 * 64 * 3 * 10
