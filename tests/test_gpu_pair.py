"""fa_fwd_pair: the d = 128 forward pass on CTA pairs (tcgen05 cta_group::2),
through the C ABI, against the fp64 oracle: whole tensors on small problems
(one cluster; query-tile counts that leave the last cluster's upper tiles
past N; ragged N; GQA; both masks) and sampled rows at the full sizes of the
d = 128 workloads.  Tolerances are the forward's (O max-abs 2e-2, mean-abs
2e-3; LSE 1e-3)."""

import numpy as np
import pytest
import torch

import oracle
from exact_attention_104_b200 import binding
from exact_attention_104_b200.workloads import WORKLOADS, Workload, make_inputs

from _parity import LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, f64

pytestmark = pytest.mark.gpu


def _run_pair(w):
    q, k, v, _ = make_inputs(w, "cuda")
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device="cuda")
    st = binding.fa_fwd_pair(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.causal, w.scale)
    assert st == binding.FA_OK, binding.fa_status_string(st)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    return q, k, v, o, lse


def _assert_close(eo, el, name):
    msg = f"{name}: O max {eo.max():.3e} mean {eo.mean():.3e} LSE max {el.max():.3e}"
    assert eo.max() <= O_MAX_ABS and eo.mean() <= O_MEAN_ABS and el.max() <= LSE_MAX_ABS, msg


SMALL = [
    Workload("pair_one_cluster", 1, 1, 1, 256, 128, False, 1.0, 81),
    Workload("pair_one_cluster_causal", 1, 1, 1, 512, 128, True, 1.0, 82),
    Workload("pair_five_tiles", 1, 2, 2, 640, 128, False, 1.0, 83),
    Workload("pair_gqa_causal", 2, 4, 2, 768, 128, True, 1.0, 84),
    Workload("pair_ragged", 1, 2, 1, 300, 128, False, 1.0, 85),
    Workload("pair_ragged_causal", 2, 2, 2, 1000, 128, True, 1.0, 86),
    Workload("pair_short", 1, 2, 2, 1, 128, True, 1.0, 87),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_pair_forward_matches_oracle(w):
    q, k, v, o, lse = _run_pair(w)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), w.scale, w.causal)
    _assert_close(np.abs(f64(o) - ro), np.abs(f64(lse) - rl), w.name)


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items() if w.d == 128])
def test_pair_forward_full_size_sampled(name):
    w = WORKLOADS[name]
    q, k, v, o, lse = _run_pair(w)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, w.N - 1], rng.choice(w.N, 24, replace=False)]))
    eo, el = [], []
    for (b, h) in ((0, 0), (w.B - 1, w.Hq - 1)):
        g = h // w.G
        o_r, l_r, _ = oracle.head_forward_rows(f64(q[b, h]), f64(k[b, g]), f64(v[b, g]), w.scale, w.causal, rows)
        eo.append(np.abs(f64(o[b, h][rows]) - o_r))
        el.append(np.abs(f64(lse[b, h][rows]) - l_r))
    _assert_close(np.concatenate([x.ravel() for x in eo]), np.concatenate(el), name)


def test_pair_forward_rejects_other_head_dims():
    w = Workload("pair_d64", 1, 1, 1, 256, 64, False, 1.0, 88)
    q, k, v, _ = make_inputs(w, "cuda")
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 256, device="cuda")
    assert binding.fa_fwd_pair(q, k, v, o, lse, 1, 1, 1, 256, 64, False, w.scale) == binding.FA_ERR_UNSUPPORTED
