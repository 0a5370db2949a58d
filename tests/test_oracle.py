"""Pins for the fp64 oracle, checked against what the pages and the mathematics
fix rather than against the oracle itself:

* the worked online-softmax example printed in "深度学习进阶（三十一）FlashAttention：
  IO 感知的精确注意力" §2.1 (golden fixture) and its closed forms;
* the page's claim in the same section that the online result equals safe
  softmax exactly, extended to the blockwise attention update of §2.2;
* rows of P sum to one (the softmax row-sum invariant the "Flash-Attention"
  concept page cites as an SDC check, "Key observations");
* closed forms of the definition (Q = 0, V = 1);
* the library special case: torch's fp64 CPU ``scaled_dot_product_attention``
  and its autograd (the handbook page "FlashAttention", "如何使用 FlashAttention",
  names PyTorch SDPA as the standard entry point);
* central finite differences and gradient invariants for the backward pass;
* the conditional-rescale form of the blockwise update (the FA4 technique the
  concept page lists) against the plain definition for several thresholds,
  with both branches exercised and the e^tau bound on its terms;
* planted mistakes in the oracle, which must make at least one pin fail.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "online_softmax_example.txt")


def _read_golden(path):
    out = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split("=", 1)
            out[key.strip()] = [float(t) for t in val.split(",")]
    return out


# ---------------------------------------------------------------------------
# Online softmax worked example
# ---------------------------------------------------------------------------

def test_online_softmax_worked_example_matches_page():
    g = _read_golden(GOLDEN)
    dec = int(g["decimals"][0])
    m_tr, d_tr, y = oracle.online_softmax(g["x"])
    tol = 0.5 * 10 ** (-dec) + 1e-12
    np.testing.assert_allclose(m_tr, g["m_after_each_step"], atol=tol, rtol=0)
    np.testing.assert_allclose(d_tr, g["d_after_each_step"], atol=tol, rtol=0)
    np.testing.assert_allclose(y, g["softmax"], atol=tol, rtol=0)


def test_online_softmax_worked_example_closed_forms():
    # d_2 = 1 + e^{-1};  d_3 = d_2·e^{-1} + 1;  y = e^{x-3} / d_3
    _, d_tr, y = oracle.online_softmax([2.0, 1.0, 3.0])
    e1 = math.exp(-1.0)
    assert d_tr[0] == 1.0
    assert abs(d_tr[1] - (1 + e1)) < 1e-15
    assert abs(d_tr[2] - ((1 + e1) * e1 + 1)) < 1e-15
    d3 = (1 + e1) * e1 + 1
    np.testing.assert_allclose(y, [math.exp(-1) / d3, math.exp(-2) / d3, 1 / d3], rtol=1e-15)


def test_online_softmax_equals_safe_softmax():
    rng = np.random.default_rng(0)
    for n in (1, 2, 7, 64, 300):
        for sd in (1.0, 30.0, 300.0):
            x = rng.normal(0, sd, n)
            _, d_tr, y = oracle.online_softmax(x)
            np.testing.assert_allclose(y, oracle.safe_softmax(x), rtol=1e-12, atol=1e-300)
            assert abs(d_tr[-1] - np.exp(x - x.max()).sum()) <= 1e-12 * d_tr[-1]


def test_safe_softmax_reduces_to_textbook_and_survives_large_inputs():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 3, (5, 40))
    np.testing.assert_allclose(oracle.safe_softmax(x), oracle.naive_softmax(x), rtol=1e-13)
    big = np.array([1000.0, 999.0, 990.0])
    y = oracle.safe_softmax(big)
    assert np.all(np.isfinite(y)) and abs(y.sum() - 1) < 1e-15
    np.testing.assert_allclose(y, oracle.safe_softmax(big - 1000.0), rtol=1e-15)


# ---------------------------------------------------------------------------
# Blockwise online update inside attention (§2.2) == two-pass safe softmax
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sd", [1.0, 3.0])
def test_blockwise_online_attention_equals_two_pass(causal, sd):
    rng = np.random.default_rng(2 + int(causal))
    N, d = 37, 8
    q = rng.normal(0, sd, (N, d))
    k = rng.normal(0, sd, (N, d))
    v = rng.normal(0, 1, (N, d))
    scale = 1 / math.sqrt(d)
    o_ref, lse_ref, p_ref = oracle.head_forward_rows(q, k, v, scale, causal)
    for trial in range(6):
        cuts = np.sort(rng.choice(np.arange(1, N), size=rng.integers(0, 8), replace=False))
        sizes = np.diff(np.concatenate([[0], cuts, [N]])).tolist()
        o, m, dsum = oracle.blockwise_online_attention(q, k, v, scale, sizes, causal)
        np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(m + np.log(dsum), lse_ref, rtol=1e-12, atol=1e-12)
    # fixed block size form, including a ragged last block
    o, _, _ = oracle.blockwise_online_attention(q, k, v, scale, 16, causal)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)


def test_blockwise_update_running_max_and_normaliser():
    # after the last block m is the row max of the scaled scores and d = Σ e^{S - m}
    rng = np.random.default_rng(4)
    q = rng.normal(0, 2, (5, 4))
    k = rng.normal(0, 2, (11, 4))
    v = rng.normal(0, 1, (11, 4))
    _, m, dsum = oracle.blockwise_online_attention(q, k, v, 0.5, [3, 3, 5])
    s = 0.5 * q @ k.T
    np.testing.assert_allclose(m, s.max(axis=1), rtol=1e-15)
    np.testing.assert_allclose(dsum, np.exp(s - s.max(axis=1, keepdims=True)).sum(axis=1), rtol=1e-13)


def _growing_logits(seed, N=48, d=8):
    # keys whose scores against every query grow from block to block, so the
    # row maximum moves up by several units per block (the rescale branch)
    rng = np.random.default_rng(seed)
    q = rng.normal(0, 1, (N, d))
    q[:, 0] = np.abs(q[:, 0]) + 1.0
    k = rng.normal(0, 1, (N, d))
    k[:, 0] = np.linspace(0.0, 40.0, N)
    v = rng.normal(0, 1, (N, d))
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 0.7, 8 * math.log(2), 1e3])
def test_lazy_rescale_equals_two_pass(causal, tau):
    # conditional rescaling keeps O and l on one reference, so the result is
    # the plain definition for any threshold (exactness, P1 "Core idea")
    cases = [_growing_logits(11), (_rand((40, 8), 12, 3.0), _rand((40, 8), 13, 3.0), _rand((40, 8), 14))]
    for q, k, v in cases:
        scale = 1 / math.sqrt(q.shape[1])
        o_ref, lse_ref, _ = oracle.head_forward_rows(q, k, v, scale, causal)
        ragged = [5, 11, 7, 1, q.shape[0] - 24]  # uneven blocks, one of a single key
        for sizes in (16, ragged, 1):
            o, lse, _, _ = oracle.blockwise_attention_lazy_rescale(q, k, v, scale, sizes, tau, causal)
            np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_lazy_rescale_branches_and_term_bound():
    q, k, v = _growing_logits(21)
    scale = 1 / math.sqrt(q.shape[1])
    # tau = 0: a rescale at every block whose row maximum is larger
    _, _, r0, t0 = oracle.blockwise_attention_lazy_rescale(q, k, v, scale, 8, 0.0)
    assert r0.min() >= 1 and t0 <= 1.0 + 1e-12
    # a threshold above the whole score range: the first block's maximum stays
    # the reference, and terms then exceed 1 (up to e^tau)
    _, _, r1, t1 = oracle.blockwise_attention_lazy_rescale(q, k, v, scale, 8, 1e3)
    assert r1.max() == 0 and t1 > 1.0
    # the kernels' threshold: some rows rescale, fewer times than with tau = 0,
    # and no term exceeds e^tau
    tau = 8 * math.log(2)
    _, _, r2, t2 = oracle.blockwise_attention_lazy_rescale(q, k, v, scale, 8, tau)
    assert 0 < r2.sum() < r0.sum() and t2 <= math.exp(tau) * (1 + 1e-12)


def test_planted_lazy_rescale_mistake_is_caught(monkeypatch):
    # rescaling O but not the normaliser l must break exactness
    def only_o(o, l, m_ref, m_new):
        o2, _ = _orig_lazy_rescale(o, l, m_ref, m_new)
        return o2, l
    _orig_lazy_rescale = oa._lazy_rescale
    monkeypatch.setattr(oa, "_lazy_rescale", only_o)
    q, k, v = _growing_logits(31)
    scale = 1 / math.sqrt(q.shape[1])
    o_ref, lse_ref, _ = oracle.head_forward_rows(q, k, v, scale, False)
    o, lse, r, _ = oracle.blockwise_attention_lazy_rescale(q, k, v, scale, 8, 0.0)
    assert r.sum() > 0
    assert np.abs(lse - lse_ref).max() > 1e-3 or np.abs(o - o_ref).max() > 1e-3


# ---------------------------------------------------------------------------
# Forward: invariants, closed forms, library special case
# ---------------------------------------------------------------------------

def _rand(shape, seed, sd=1.0):
    return np.random.default_rng(seed).normal(0, sd, shape)


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k, v = _rand((16, 8), 5), _rand((16, 8), 6), _rand((16, 8), 7)
    _, _, p = oracle.head_forward_rows(q, k, v, 0.3, causal)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    if causal:
        assert np.all(np.triu(p, 1) == 0)


def test_zero_queries_give_mean_of_values_and_log_n():
    B, H, N, d = 1, 2, 12, 4
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), 8), _rand((B, H, N, d), 9)
    o, lse = oracle.attention_forward(q, k, v, 0.7, causal=False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, math.log(N), rtol=1e-14)
    o, lse = oracle.attention_forward(q, k, v, 0.7, causal=True)
    prefix_mean = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(o, prefix_mean, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, N + 1)), lse.shape), rtol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_give_constant_output(causal):
    q, k = _rand((1, 1, 20, 8), 10, 3.0), _rand((1, 1, 20, 8), 11, 3.0)
    v = np.ones((1, 1, 20, 8))
    o, _ = oracle.attention_forward(q, k, v, 1 / math.sqrt(8), causal)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-13)


def _torch_sdpa(q, k, v, scale, causal):
    G = q.shape[1] // k.shape[1]
    tq = torch.tensor(q)
    tk = torch.tensor(k).repeat_interleave(G, dim=1)
    tv = torch.tensor(v).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale).numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1)])
def test_forward_matches_torch_sdpa_fp64(causal, Hq, Hkv):
    B, N, d = 2, 19, 8
    q = _rand((B, Hq, N, d), 12)
    k = _rand((B, Hkv, N, d), 13)
    v = _rand((B, Hkv, N, d), 14)
    o, lse = oracle.attention_forward(q, k, v, 1 / math.sqrt(d), causal)
    np.testing.assert_allclose(o, _torch_sdpa(q, k, v, 1 / math.sqrt(d), causal), rtol=1e-12, atol=1e-13)
    # LSE against torch.logsumexp of the masked scaled scores
    G = Hq // Hkv
    s = torch.einsum("bhid,bhjd->bhij", torch.tensor(q),
                     torch.tensor(k).repeat_interleave(G, dim=1)) / math.sqrt(d)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-13)


def test_gqa_equals_repeated_heads():
    B, Hq, Hkv, N, d = 1, 4, 2, 10, 4
    q = _rand((B, Hq, N, d), 15)
    k, v = _rand((B, Hkv, N, d), 16), _rand((B, Hkv, N, d), 17)
    o, lse = oracle.attention_forward(q, k, v, 0.5, True)
    o2, lse2 = oracle.attention_forward(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1), 0.5, True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_head_forward_rows_subset_equals_full():
    q, k, v = _rand((30, 4), 18), _rand((30, 4), 19), _rand((30, 4), 20)
    rows = np.array([0, 7, 29])
    o, lse, _ = oracle.head_forward_rows(q, k, v, 0.4, True)
    o_r, lse_r, _ = oracle.head_forward_rows(q, k, v, 0.4, True, rows)
    np.testing.assert_array_equal(o_r, o[rows])
    np.testing.assert_array_equal(lse_r, lse[rows])


# ---------------------------------------------------------------------------
# Backward: finite differences, invariants, library autograd
# ---------------------------------------------------------------------------

def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_forward(q, k, v, scale, causal)
    return float(np.sum(o * do))


@pytest.mark.parametrize("N,d,Hq,Hkv,causal", [
    (1, 1, 1, 1, False), (3, 4, 1, 1, True), (8, 4, 2, 1, False), (17, 1, 2, 2, True), (8, 4, 2, 1, True),
])
def test_backward_matches_central_finite_differences(N, d, Hq, Hkv, causal):
    B = 1
    scale = 1 / math.sqrt(d)
    q = _rand((B, Hq, N, d), 21)
    k = _rand((B, Hkv, N, d), 22)
    v = _rand((B, Hkv, N, d), 23)
    do = _rand((B, Hq, N, d), 24)
    dq, dk, dv, _, _ = oracle.attention_backward(q, k, v, do, scale, causal)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            fm = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            num[idx] = (fp - fm) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
        assert err <= 1e-6, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    # rows of P sum to one  =>  Σ_keys dV = Σ_queries dO (per kv head, over its
    # query heads) and Σ_keys dS = 0 per query row  =>  Σ_keys dK = 0.
    B, Hq, Hkv, N, d = 2, 4, 2, 24, 8
    q, k, v = _rand((B, Hq, N, d), 25), _rand((B, Hkv, N, d), 26), _rand((B, Hkv, N, d), 27)
    do = _rand((B, Hq, N, d), 28)
    dq, dk, dv, _, _ = oracle.attention_backward(q, k, v, do, 0.35, causal)
    G = Hq // Hkv
    do_sum = do.reshape(B, Hkv, G, N, d).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), do_sum, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd_fp64(causal):
    B, Hq, Hkv, N, d = 1, 4, 2, 21, 8
    scale = 1 / math.sqrt(d)
    q, k, v = _rand((B, Hq, N, d), 29), _rand((B, Hkv, N, d), 30), _rand((B, Hkv, N, d), 31)
    do = _rand((B, Hq, N, d), 32)
    dq, dk, dv, o, _ = oracle.attention_backward(q, k, v, do, scale, causal)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    G = Hq // Hkv
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1), is_causal=causal, scale=scale)
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=1e-12, atol=1e-13)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_backward_equals_full(causal):
    B, Hq, Hkv, N, d = 1, 2, 1, 40, 4
    q, k, v = _rand((B, Hq, N, d), 33), _rand((B, Hkv, N, d), 34), _rand((B, Hkv, N, d), 35)
    do = _rand((B, Hq, N, d), 36)
    dq, dk, dv, _, _ = oracle.attention_backward(q, k, v, do, 0.5, causal)
    qr, kr = np.array([0, 5, 39]), np.array([1, 20, 39])
    dq_r, dk_r, dv_r = oracle.head_backward_sampled(q[0], k[0, 0], v[0, 0], do[0], 0.5, causal, qr, kr, row_chunk=16)
    np.testing.assert_allclose(dq_r, dq[0][:, qr], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dk_r, dk[0, 0][kr], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv_r, dv[0, 0][kr], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_row_block_backward_partials_sum_to_full(causal):
    # blocks of query rows (ragged sizes, one block strided) that partition all
    # rows: dQ/O/LSE rows are the full ones, and the dK/dV partials add up to
    # the full gradients of the head
    N, d, s = 37, 5, 0.4
    q, k, v, do = (_rand((1, 1, N, d), 40 + i) for i in range(4))
    dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, do, s, causal)
    blocks = [np.arange(0, 37, 3), np.arange(1, 11, 3), np.setdiff1d(np.arange(N), np.concatenate(
        [np.arange(0, 37, 3), np.arange(1, 11, 3)]))]
    dk_sum, dv_sum = np.zeros((N, d)), np.zeros((N, d))
    for rows in blocks:
        dq_r, dk_p, dv_p, o_r, lse_r = oracle.head_backward_rows(q[0, 0], k[0, 0], v[0, 0], do[0, 0], s, causal,
                                                                 rows)
        np.testing.assert_allclose(dq_r, dq[0, 0][rows], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(o_r, o[0, 0][rows], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse_r, lse[0, 0][rows], rtol=1e-12, atol=1e-13)
        dk_sum += dk_p
        dv_sum += dv_p
    np.testing.assert_allclose(dk_sum, dk[0, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv_sum, dv[0, 0], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# Packed variable-length batches
# ---------------------------------------------------------------------------

VARLEN_CASES = [
    # (lengths, Hq, Hkv): ragged lengths, a length-1 sequence, an empty one, GQA
    ([5, 1, 0, 17, 9], 4, 2),
    ([3, 12], 2, 2),
    ([1], 1, 1),
]


def _sdpa_block_diagonal(q, k, v, lengths, scale, causal):
    """torch fp64 SDPA over the whole packed token axis with a boolean mask
    that lets token i see token j only inside its own sequence (and, causal,
    only j <= i) -- an independent route to the same definition."""
    T = q.shape[1]
    seq = np.repeat(np.arange(len(lengths)), lengths)
    pos = np.concatenate([np.arange(n) for n in lengths]) if T else np.zeros(0, int)
    allowed = seq[:, None] == seq[None, :]
    if causal:
        allowed &= pos[None, :] <= pos[:, None]
    G = q.shape[0] // k.shape[0]
    tq = torch.tensor(q[None], requires_grad=True)
    tk = torch.tensor(k[None], requires_grad=True)
    tv = torch.tensor(v[None], requires_grad=True)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1), attn_mask=torch.tensor(allowed), scale=scale)
    return tq, tk, tv, out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lengths,Hq,Hkv", VARLEN_CASES)
def test_varlen_matches_block_diagonal_sdpa(lengths, Hq, Hkv, causal):
    T, d, s = sum(lengths), 6, 0.45
    cu = np.concatenate([[0], np.cumsum(lengths)])
    q, do = _rand((Hq, T, d), 70), _rand((Hq, T, d), 71)
    k, v = _rand((Hkv, T, d), 72), _rand((Hkv, T, d), 73)
    dq, dk, dv, o, lse = oracle.attention_backward_varlen(q, k, v, do, cu, s, causal)
    o_f, lse_f = oracle.attention_forward_varlen(q, k, v, cu, s, causal)
    np.testing.assert_array_equal(o, o_f)
    np.testing.assert_array_equal(lse, lse_f)
    tq, tk, tv, out = _sdpa_block_diagonal(q, k, v, lengths, s, causal)
    out.backward(torch.tensor(do[None]))
    np.testing.assert_allclose(o, out.detach().numpy()[0], rtol=1e-12, atol=1e-13)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy()[0], rtol=1e-10, atol=1e-12)
    # LSE from its definition, row by row
    for b in range(len(lengths)):
        for i in range(lengths[b]):
            t = cu[b] + i
            keys = np.arange(cu[b], cu[b] + (i + 1 if causal else lengths[b]))
            for h in range(Hq):
                sc = s * (k[h // (Hq // Hkv), keys] @ q[h, t])
                assert abs(lse[h, t] - (sc.max() + np.log(np.exp(sc - sc.max()).sum()))) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_zero_queries_give_sequence_means(causal):
    lengths = [4, 1, 7]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T, d = sum(lengths), 3
    v = _rand((1, T, d), 74)
    o, lse = oracle.attention_forward_varlen(np.zeros((2, T, d)), _rand((1, T, d), 75), v, cu, 0.5, causal)
    for b, n in enumerate(lengths):
        for i in range(n):
            t = cu[b] + i
            seen = v[0, cu[b]:cu[b] + (i + 1 if causal else n)]
            np.testing.assert_allclose(o[:, t], np.broadcast_to(seen.mean(axis=0), (2, d)), rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(lse[:, t], math.log(len(seen)), rtol=1e-13)


def test_varlen_boundary_mistake_is_caught(monkeypatch):
    # plant a mistake in the oracle: every sequence boundary moved one token
    # early, so the first token of each sequence joins the previous one
    orig = oa._varlen_bounds

    def shifted(cu_seqlens, T):
        cu = orig(cu_seqlens, T)
        return [0] + [max(0, c - 1) for c in cu[1:-1]] + [cu[-1]]

    monkeypatch.setattr(oa, "_varlen_bounds", shifted)
    for causal in (False, True):
        with pytest.raises(AssertionError):
            test_varlen_matches_block_diagonal_sdpa([5, 1, 0, 17, 9], 4, 2, causal)


def test_flop_count():
    # 4·B·Hq·N²·d, halved when causal
    assert oracle.attention_flops(8, 16, 2048, 128, False) == 274877906944.0
    assert oracle.attention_flops(8, 16, 2048, 128, True) == 137438953472.0
    assert oracle.attention_flops(1, 2, 128, 64, False) == 8388608.0


# ---------------------------------------------------------------------------
# Fewer queries than keys (decoding): attention_forward_suffix
# ---------------------------------------------------------------------------

def _suffix_check(fn, causal, Nq, Hq, Hkv, seed):
    """The last Nq rows of the square computation over the whole sequence."""
    rng = np.random.default_rng(seed)
    B, N, d = 2, 13, 5
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    o_sq, lse_sq = oracle.attention_forward(q, k, v, 0.6, causal)
    o, lse = fn(q[:, :, N - Nq:], k, v, 0.6, causal)
    np.testing.assert_allclose(o, o_sq[:, :, N - Nq:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_sq[:, :, N - Nq:], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq", [1, 4, 13])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1)])
def test_suffix_equals_last_rows_of_square_attention(causal, Nq, Hq, Hkv):
    _suffix_check(oracle.attention_forward_suffix, causal, Nq, Hq, Hkv, 5 + Nq)


def test_suffix_alignment_mistake_is_caught():
    # a top-left aligned mask (query row r sees keys 0..r) must fail the pin
    def top_left(q, k, v, scale, causal=False):
        q = np.asarray(q, np.float64)
        B, Hq, Nq, d = q.shape
        Hkv, Nk = k.shape[1], k.shape[2]
        o = np.zeros_like(q)
        lse = np.zeros((B, Hq, Nq))
        for b in range(B):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                sc = scale * (q[b, h] @ k[b, g].T)
                if causal:
                    sc = np.where(np.arange(Nk)[None, :] > np.arange(Nq)[:, None], -np.inf, sc)
                m = sc.max(axis=1, keepdims=True)
                e = np.exp(sc - m)
                o[b, h] = e / e.sum(axis=1, keepdims=True) @ v[b, g]
                lse[b, h] = (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
        return o, lse

    with pytest.raises(AssertionError):
        _suffix_check(top_left, True, 4, 2, 2, 9)


def test_suffix_matches_brute_force_loops():
    # every visible key enumerated with scalar exp and explicit sums
    rng = np.random.default_rng(17)
    Nq, Nk, d = 3, 7, 4
    q = rng.standard_normal((1, 1, Nq, d))
    k = rng.standard_normal((1, 1, Nk, d))
    v = rng.standard_normal((1, 1, Nk, d))
    for causal in (False, True):
        o, lse = oracle.attention_forward_suffix(q, k, v, 0.5, causal)
        for r in range(Nq):
            last = (Nk - Nq + r) if causal else Nk - 1
            sc = [0.5 * sum(q[0, 0, r, c] * k[0, 0, j, c] for c in range(d)) for j in range(last + 1)]
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            tot = sum(w)
            for c in range(d):
                ref = sum(w[j] * v[0, 0, j, c] for j in range(last + 1)) / tot
                assert abs(o[0, 0, r, c] - ref) < 1e-12
            assert abs(lse[0, 0, r] - (mx + math.log(tot))) < 1e-12


def test_suffix_closed_forms():
    # Q = 0: O is the mean of the visible values, LSE = ln(number visible);
    # V = 1: O = 1 whatever the scores
    rng = np.random.default_rng(3)
    Nq, Nk, d = 4, 10, 3
    v = rng.standard_normal((1, 2, Nk, d))
    k = rng.standard_normal((1, 2, Nk, d))
    o, lse = oracle.attention_forward_suffix(np.zeros((1, 2, Nq, d)), k, v, 1.0, True)
    for r in range(Nq):
        n_vis = Nk - Nq + r + 1
        np.testing.assert_allclose(o[0, :, r], v[0, :, :n_vis].mean(axis=1), atol=1e-12)
        np.testing.assert_allclose(lse[0, :, r], math.log(n_vis), atol=1e-12)
    o1, _ = oracle.attention_forward_suffix(rng.standard_normal((1, 2, Nq, d)), k, np.ones_like(v), 0.7, True)
    np.testing.assert_allclose(o1, 1.0, atol=1e-12)


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above
# ---------------------------------------------------------------------------

def _pins_pass():
    """Run a compact subset of the pins; return False if any fails."""
    checks = [
        lambda: test_forward_matches_torch_sdpa_fp64(True, 4, 2),
        lambda: test_forward_matches_torch_sdpa_fp64(False, 2, 2),
        lambda: test_zero_queries_give_mean_of_values_and_log_n(),
        lambda: test_backward_matches_torch_autograd_fp64(True),
        lambda: test_backward_invariants(True),
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def test_pins_pass_on_unmodified_oracle():
    assert _pins_pass()


def _mut_scores_no_scale(qh, kh, scale, causal, rows=None, _orig=oa._scores):
    return _orig(qh, kh, 1.0, causal, rows)


def _mut_scores_wrong_mask(qh, kh, scale, causal, rows=None, _orig=oa._scores):
    # masks j >= i instead of j > i (drops the diagonal), keeping row 0 alive
    s = _orig(qh, kh, scale, False, rows)
    if causal:
        r = np.arange(qh.shape[0]) if rows is None else rows
        mask = (np.arange(kh.shape[0])[None, :] >= r[:, None]) & (r[:, None] > 0)
        s = np.where(mask, -np.inf, s)
    return s


def _mut_scores_transposed(qh, kh, scale, causal, rows=None, _orig=oa._scores):
    return _orig(kh, qh, scale, causal, rows)


@pytest.mark.parametrize("mutant", [_mut_scores_no_scale, _mut_scores_wrong_mask, _mut_scores_transposed])
def test_planted_score_mistakes_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(oa, "_scores", mutant)
    assert not _pins_pass()


def test_planted_backward_mistake_is_caught(monkeypatch):
    # drop the D term of dS = P ∘ (dP − D) by zeroing dO·O inside the oracle
    orig_sum = np.sum

    def bad_sum(a, *args, **kw):
        out = orig_sum(a, *args, **kw)
        if kw.get("keepdims") and kw.get("axis") == 1:
            return out * 0.0
        return out

    monkeypatch.setattr(oa.np, "sum", bad_sum)
    try:
        assert not _pins_pass()
    finally:
        monkeypatch.setattr(oa.np, "sum", orig_sum)
