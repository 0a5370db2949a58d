"""Packed batches of sequences with different lengths (fa_fwd_varlen,
fa_bwd_varlen) on the GPU, through the C ABI.

* Small mixed batches (lengths 1, 127, 128, 129, 300, an empty sequence, 513,
  64; GQA 2:1) against the fp64 oracle's per-sequence loop, whole tensors, at
  d = 64, 128, 256, with and without the causal mask.
* The same batches against separate fa_fwd / fa_bwd calls on each sequence:
  a varlen unit runs the same per-tile arithmetic in the same order as the
  fixed-length kernels on that sequence, so O, LSE, dK and dV are identical
  bit for bit; dQ differs only in the order of its fp32 reduce-adds.
* Lengths from 1 to 5000 (GQA 4:1, d = 128), and the benchmark's packed
  batch (16 causal sequences of 256 to 4096 tokens, 16 heads), sampled rows
  of every sequence against the oracle.
* cu_seqlens that breaks its rules: the call computes nothing, leaves the
  outputs untouched and fa_device_status reports FA_ERR_INVALID_ARG."""

import numpy as np
import pytest
import torch

import oracle
from exact_attention_104_b200 import (attention_backward, attention_backward_varlen, attention_forward,
                                      attention_forward_varlen, binding)
from exact_attention_104_b200.workloads import VARLEN_WORKLOADS, VarlenWorkload, make_varlen_inputs, varlen_lengths

from _parity import GRAD_REL_FRO, assert_within_tolerance, f64, rel_fro

pytestmark = pytest.mark.gpu

MIXED = (1, 127, 128, 129, 300, 0, 513, 64)


def _small(d, causal):
    return VarlenWorkload(f"mixed_d{d}_{'c' if causal else 'nc'}", MIXED, 4, 2, d, causal, 3000 + d + causal,
                          3.0 if d == 256 else 1.0)


def _run(w, inputs=None):
    q, k, v, do, cu = inputs if inputs is not None else make_varlen_inputs(w, "cuda")
    o, lse = attention_forward_varlen(q, k, v, cu, w.max_seqlen, causal=w.causal, scale=w.scale)
    dq, dk, dv = attention_backward_varlen(q, k, v, o, lse, do, cu, w.max_seqlen, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    return dict(q=q, k=k, v=v, do=do, cu=cu, o=o, lse=lse, dq=dq, dk=dk, dv=dv)


CASES = [(d, c) for d in (64, 128, 256) for c in (False, True)]


@pytest.mark.parametrize("d,causal", CASES, ids=[f"d{d}-{'causal' if c else 'full'}" for d, c in CASES])
def test_varlen_small_batches_match_oracle(d, causal):
    w = _small(d, causal)
    g = _run(w)
    cu = w.cu_seqlens()
    dq, dk, dv, o, lse = oracle.attention_backward_varlen(f64(g["q"]), f64(g["k"]), f64(g["v"]), f64(g["do"]), cu,
                                                          w.scale, w.causal)
    err_o = np.abs(f64(g["o"]) - o)
    err = {"o_max": float(err_o.max()), "o_mean": float(err_o.mean()),
           "lse_max": float(np.abs(f64(g["lse"]) - lse).max()),
           "dq": rel_fro(f64(g["dq"]), dq), "dk": rel_fro(f64(g["dk"]), dk), "dv": rel_fro(f64(g["dv"]), dv)}
    print(w.name, err)
    assert_within_tolerance(err)


@pytest.mark.parametrize("d,causal", CASES, ids=[f"d{d}-{'causal' if c else 'full'}" for d, c in CASES])
def test_varlen_equals_one_call_per_sequence(d, causal):
    w = _small(d, causal)
    g = _run(w)
    cu = w.cu_seqlens()
    for b in range(len(w.lengths)):
        lo, hi = cu[b], cu[b + 1]
        if hi == lo:
            continue
        sl = lambda t: t[:, lo:hi].unsqueeze(0).contiguous()  # noqa: E731
        q, k, v, do = sl(g["q"]), sl(g["k"]), sl(g["v"]), sl(g["do"])
        o, lse = attention_forward(q, k, v, causal=causal, scale=w.scale)
        dq, dk, dv = attention_backward(q, k, v, o, lse, do, causal=causal, scale=w.scale)
        torch.cuda.synchronize()
        assert torch.equal(o[0], g["o"][:, lo:hi]), (b, "o")
        assert torch.equal(lse[0], g["lse"][:, lo:hi]), (b, "lse")
        assert torch.equal(dk[0], g["dk"][:, lo:hi]), (b, "dk")
        assert torch.equal(dv[0], g["dv"][:, lo:hi]), (b, "dv")
        assert rel_fro(f64(dq[0]), f64(g["dq"][:, lo:hi])) <= 1e-3, (b, "dq")


def _random_batches(n, seed):
    """Seeded random packed batches: 1..8 sequences of 0..599 tokens, d in
    {64, 128, 256}, kv heads 1..2 with GQA ratio 1, 2 or 4, either mask."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([64, 128, 256]))
        hkv = int(rng.integers(1, 3))
        g = int(rng.choice([1, 2, 4]))
        lens = tuple(int(x) for x in rng.integers(0, 600, size=int(rng.integers(1, 9))))
        if sum(lens) < 2:
            lens = lens + (5,)
        causal = bool(rng.integers(0, 2))
        out.append(VarlenWorkload(f"rand{i}_d{d}_hq{hkv * g}_hkv{hkv}_{'c' if causal else 'nc'}", lens, hkv * g, hkv,
                                  d, causal, 9000 + i, 3.0 if d == 256 else 1.0))
    return out


def test_varlen_random_batches_match_oracle():
    # 40 seeded random batches in one test (about 12 s); every failing batch is reported
    failures = []
    for w in _random_batches(40, 4242):
        g = _run(w)
        cu = w.cu_seqlens()
        dq, dk, dv, o, lse = oracle.attention_backward_varlen(f64(g["q"]), f64(g["k"]), f64(g["v"]), f64(g["do"]), cu,
                                                              w.scale, w.causal)
        err_o = np.abs(f64(g["o"]) - o)
        err = {"o_max": float(err_o.max()), "o_mean": float(err_o.mean()),
               "lse_max": float(np.abs(f64(g["lse"]) - lse).max()),
               "dq": rel_fro(f64(g["dq"]), dq), "dk": rel_fro(f64(g["dk"]), dk), "dv": rel_fro(f64(g["dv"]), dv)}
        try:
            assert_within_tolerance(err)
        except AssertionError:
            failures.append((w.name, w.lengths, err))
    assert not failures, failures


def _sampled_errors(w, g, seed, rows_per_seq=12):
    """Sampled rows of every sequence (its first and last rows, the rows
    around the first tile edge, the last tile's first row and random ones),
    on the first and last kv head and all their query heads, against the
    oracle's row-wise forward and sampled backward."""
    cu = w.cu_seqlens()
    rng = np.random.default_rng(seed)
    o_abs, lse_abs, dq_p, dk_p, dv_p = [], [], [], [], []
    for b, n in enumerate(w.lengths):
        if n == 0:
            continue
        lo = cu[b]
        fixed = {0, n - 1, 127, 128, (n - 1) // 128 * 128}
        rows = np.array(sorted({r for r in fixed if 0 <= r < n} |
                               set(rng.choice(n, min(n, rows_per_seq), replace=False))))
        for g_kv in sorted({0, w.Hkv - 1}):
            kh, vh = f64(g["k"][g_kv, lo:lo + n]), f64(g["v"][g_kv, lo:lo + n])
            heads = range(g_kv * w.G, (g_kv + 1) * w.G)
            qh = np.stack([f64(g["q"][h, lo:lo + n]) for h in heads])
            doh = np.stack([f64(g["do"][h, lo:lo + n]) for h in heads])
            for i, h in enumerate(heads):
                o_r, lse_r, _ = oracle.head_forward_rows(qh[i], kh, vh, w.scale, w.causal, rows)
                o_abs.append(np.abs(f64(g["o"][h, lo:lo + n][rows]) - o_r))
                lse_abs.append(np.abs(f64(g["lse"][h, lo:lo + n][rows]) - lse_r))
            dq_r, dk_r, dv_r = oracle.head_backward_sampled(qh, kh, vh, doh, w.scale, w.causal, rows, rows)
            for i, h in enumerate(heads):
                dq_p.append((f64(g["dq"][h, lo:lo + n][rows]), dq_r[i]))
            dk_p.append((f64(g["dk"][g_kv, lo:lo + n][rows]), dk_r))
            dv_p.append((f64(g["dv"][g_kv, lo:lo + n][rows]), dv_r))
    o_abs = np.concatenate([x.ravel() for x in o_abs])
    err = {"o_max": float(o_abs.max()), "o_mean": float(o_abs.mean()),
           "lse_max": float(np.concatenate(lse_abs).max())}
    for name, pairs in (("dq", dq_p), ("dk", dk_p), ("dv", dv_p)):
        err[name] = rel_fro(np.concatenate([p[0].ravel() for p in pairs]),
                            np.concatenate([p[1].ravel() for p in pairs]))
    return err


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_lengths_1_to_5000_sampled(causal):
    lengths = varlen_lengths(10, 1, 5000, 77 + causal, include=(1, 5000, 129))
    w = VarlenWorkload("mixed_1_5000", lengths, 8, 2, 128, causal, 3100 + causal)
    err = _sampled_errors(w, _run(w), 5 + causal)
    print(lengths, err)
    assert_within_tolerance(err)


@pytest.mark.parametrize("name", list(VARLEN_WORKLOADS))
def test_varlen_bench_workload_sampled(name):
    """The packed batch the benchmark times, in the same call sequence."""
    w = VARLEN_WORKLOADS[name]
    err = _sampled_errors(w, _run(w), 11, rows_per_seq=6)
    print(w.name, err)
    assert_within_tolerance(err)


@pytest.mark.parametrize("bad", ["last_not_T", "decreasing", "too_long"])
@pytest.mark.parametrize("d", [128, 256])
def test_varlen_invalid_cu_seqlens_reported_on_device(bad, d):
    w = VarlenWorkload("bad", (100, 200, 50), 2, 1, d, True, 3200)
    q, k, v, do, cu = make_varlen_inputs(w, "cuda")
    max_seqlen = w.max_seqlen
    if bad == "last_not_T":
        cu[-1] = w.T - 1
    elif bad == "decreasing":
        cu[1], cu[2] = 250, 200
    else:
        max_seqlen = 150          # sequence 1 is 200 long
    o = torch.full_like(q, 7.0)
    lse = torch.full((w.Hq, w.T), 7.0, device="cuda")
    ws = torch.empty(binding.fa_fwd_varlen_workspace_bytes(3, w.Hq, w.Hkv, w.T, max_seqlen, d), dtype=torch.uint8,
                     device="cuda")
    st = binding.fa_fwd_varlen(q, k, v, o, lse, cu, 3, w.Hq, w.Hkv, w.T, max_seqlen, d, True, w.scale, ws,
                               ws.numel())
    assert st == binding.FA_OK
    assert binding.fa_device_status() == binding.FA_ERR_INVALID_ARG
    assert bool((o == 7.0).all()) and bool((lse == 7.0).all())
    dq, dk, dv = (torch.full_like(t, 7.0) for t in (q, k, v))
    wsb = torch.empty(binding.fa_bwd_varlen_workspace_bytes(3, w.Hq, w.Hkv, w.T, max_seqlen, d), dtype=torch.uint8,
                      device="cuda")
    st = binding.fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu, 3, w.Hq, w.Hkv, w.T, max_seqlen, d, True,
                               w.scale, wsb, wsb.numel())
    assert st == binding.FA_OK
    assert binding.fa_device_status() == binding.FA_ERR_INVALID_ARG
    for t in (dq, dk, dv):
        assert bool((t == 7.0).all())
    assert binding.fa_device_status() == binding.FA_OK  # reported once
