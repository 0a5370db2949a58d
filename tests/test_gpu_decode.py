"""GPU parity of the decoding forward pass (fa_fwd_decode, through the C ABI)
against the fp64 oracle's suffix attention: Nq queries that are the last Nq
positions of an Nk-long sequence.  Tolerances are the forward's (O max-abs
2e-2, mean-abs 2e-3; LSE 1e-3)."""

import numpy as np
import pytest
import torch

import oracle
from exact_attention_104_b200 import attention_decode, binding, lib
from exact_attention_104_b200.workloads import DECODE_WORKLOADS, DecodeWorkload, make_decode_inputs

from _parity import LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _short_waits():
    lib().fa_set_wait_cap(1 << 28)
    yield
    lib().fa_set_wait_cap(0)


def _check(w):
    q, k, v = make_decode_inputs(w, "cuda")
    o, lse = attention_decode(q, k, v, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    o_ref, lse_ref = oracle.attention_forward_suffix(f64(q), f64(k), f64(v), w.scale, w.causal)
    err_o = np.abs(f64(o) - o_ref)
    err_l = np.abs(f64(lse) - lse_ref)
    msg = f"{w.name}: O max {err_o.max():.3e} mean {err_o.mean():.3e} LSE max {err_l.max():.3e}"
    assert err_o.max() <= O_MAX_ABS and err_o.mean() <= O_MEAN_ABS and err_l.max() <= LSE_MAX_ABS, msg


# (B, Hq, Hkv, Nq, Nk, d, causal): single key; GQA groups of 4 and 8 rows;
# Nk ragged against the 64-key tiles; Nq = Nk (a whole square problem);
# d = 64, 128, 256.  With more than 16 rows per kv head (G·Nq) the
# tensor-core kernel runs: 40, 64, 128 rows (one 128-row tile, partly
# filled), 160 and 512 rows (two and four tiles), Nk ragged against its
# 128-key tiles, shorter than one tile, and square (Nq = Nk, causal)
CASES = [
    (1, 8, 2, 16, 1000, 128, True),
    (2, 16, 2, 5, 777, 64, False),
    (1, 4, 2, 256, 300, 128, True),
    (1, 2, 1, 200, 200, 256, True),
    (1, 32, 8, 32, 4096, 128, True),
    (2, 8, 1, 20, 20000, 128, False),
    (1, 4, 1, 30, 100, 256, False),
    (1, 1, 1, 1, 1, 128, True),
    (1, 4, 1, 1, 100, 128, True),
    (2, 8, 2, 3, 1000, 64, True),
    (1, 8, 1, 16, 4097, 128, False),
    (1, 2, 2, 16, 16, 256, True),
    (2, 32, 8, 1, 5000, 128, True),
    (1, 4, 4, 5, 64, 256, False),
    (1, 16, 2, 2, 3333, 128, True),
    (1, 2, 1, 7, 129, 64, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_hq{}_hkv{}_nq{}_nk{}_d{}_{}".format(*c[:6], "c" if c[6] else "nc"))
def test_decode_matches_oracle(case):
    B, Hq, Hkv, Nq, Nk, d, causal = case
    _check(DecodeWorkload("dec", B, Hq, Hkv, Nq, Nk, d, causal, 300 + Nk + Nq))


def _random_decode_cases(n, seed):
    """Seeded random decode shapes: d in {64, 128, 256}, kv heads 1..3 with GQA
    ratio 1, 2, 4 or 8, B in 1..2, Nk in 1..5999, Nq in 1..min(Nk, 256), either
    mask: both decode kernels and partial, single and multiple row tiles."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([64, 128, 256]))
        hkv = int(rng.integers(1, 4))
        g = int(rng.choice([1, 2, 4, 8]))
        B = int(rng.integers(1, 3))
        Nk = int(rng.integers(1, 6000))
        Nq = int(rng.integers(1, min(Nk, 256) + 1))
        out.append(DecodeWorkload(f"rdec{i}", B, hkv * g, hkv, Nq, Nk, d, bool(rng.integers(0, 2)), 7000 + i))
    return out


def test_decode_random_shapes_match_oracle():
    # 60 seeded random shapes in one test (a few seconds); every failing shape is reported
    failures = []
    for w in _random_decode_cases(60, 2718):
        try:
            _check(w)
        except AssertionError as e:
            failures.append((w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, str(e)))
    assert not failures, failures


@pytest.mark.parametrize("name", list(DECODE_WORKLOADS))
def test_decode_bench_workload_matches_oracle(name):
    _check(DECODE_WORKLOADS[name])


def test_decode_is_deterministic():
    w = DecodeWorkload("det", 2, 8, 2, 2, 2000, 128, True, 91)
    q, k, v = make_decode_inputs(w, "cuda")
    a = attention_decode(q, k, v, causal=True)
    b = attention_decode(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_decode_tensor_core_path_is_deterministic():
    w = DecodeWorkload("det_tc", 2, 8, 2, 32, 3000, 128, True, 92)
    q, k, v = make_decode_inputs(w, "cuda")
    a = attention_decode(q, k, v, causal=True)
    b = attention_decode(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
