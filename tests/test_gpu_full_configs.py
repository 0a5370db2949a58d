"""GPU parity at the full sizes of the five reference workloads (C2 in both
masking modes), plus the d = 64 and ragged-length workloads, in the launch
configuration bench.py times.  The oracle
computes sampled outputs one head at a time: O and LSE for sampled query rows,
dQ for the same rows and dK, dV for sampled key rows (every query row
contributes to those, so the oracle computes the full probability columns)."""

import pytest

from exact_attention_104_b200.workloads import WORKLOADS

from _parity import assert_within_tolerance, compare_sampled, run_gpu

pytestmark = pytest.mark.gpu

UNITS = {
    "tiny_b1_h2_n128_d64": [(0, 0), (0, 1)],
    "train_b8_h16_n2048_d128": [(0, 0), (7, 15)],
    "train_b8_h16_n2048_d128_causal": [(0, 3), (5, 15)],
    "long_b1_h16_n16384_d128_causal": [(0, 9)],
    "gqa_b4_hq32_hkv8_n4096_d128_causal": [(3, 7)],
    "wide_b2_h8_n8192_d256_bigqk": [(1, 5)],
    "train_b8_h16_n2048_d64": [(2, 11)],
    "ragged_b8_h16_n2000_d128_causal": [(0, 0), (7, 15)],
}


@pytest.mark.parametrize("name", list(UNITS), ids=list(UNITS))
def test_full_size_workload_sampled_parity(name):
    w = WORKLOADS[name]
    g = run_gpu(w)
    err = compare_sampled(w, g, UNITS[name], n_rows=40, seed=sum(map(ord, name)) % 1000)
    print(name, err)
    assert_within_tolerance(err)
