"""fp64 CPU oracle for exact scaled-dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library never
calls it, shares no code with it, and fails loudly rather than falling back to it.

What it computes, and where that is defined
-------------------------------------------
Sources are three web pages about FlashAttention:

* [P1] "Flash-Attention" (Awesome System Papers Wiki concept page), sections
  "Core idea" (核心思想) and "Key observations" (关键观察).
* [P2] "深度学习进阶（三十一）FlashAttention：IO 感知的精确注意力" (rkmt.cn blog),
  section 2.1 "Online Softmax" and section 2.2 "把 Online Softmax 嵌入注意力".
* [P3] "FlashAttention" (LLM inference handbook, kernel-optimization chapter),
  section "attention 为什么一开始就很慢" (standard attention and its three steps).

FlashAttention is *exact*: it reaches the same result as standard attention
(P1 "Core idea"; P2 §2.1 closing remark that the online result equals safe
softmax; P3 standard-attention formula).  The oracle is therefore the plain
definition written out in float64, materialising the score matrix S and the
probability matrix P for each (batch, query head), exactly as P3's three steps
describe (S = Q Kᵀ / √d, softmax, then P V).

Readings taken where the pages are silent:

* scale ``s`` is applied to the scores before the mask and the softmax (P3
  formula uses 1/√d_k; callers pass ``scale``);
* causal: key j is masked for query i when j > i (equal query/key lengths);
* LSE is the natural-log log-sum-exp of the scaled, masked scores of a row;
* GQA: query head h uses key/value head ``h // G`` with ``G = Hq // Hkv``;
* the backward pass is the chain rule on the same definition (the pages only
  say that P is recomputed from Q, K, V and a few per-row statistics, P1
  "Core idea"): dV = Pᵀ dO, dP = dO Vᵀ, D_i = Σ_c dO_ic O_ic,
  dS = P ∘ (dP − D), dQ = s dS K, dK = s dSᵀ Q, with dK and dV summed over the
  G query heads that share a key/value head;
* P2 §2.2 step 5 writes the second term of the O update with ``softmax_j(S_j)``;
  it equals the exact result only if that factor is the *un-normalised*
  ``exp(S_j - m_j)`` (consistent with the step-4 normaliser update), so
  :func:`blockwise_online_attention` uses that reading.

All arrays are numpy float64.  Inputs that were bf16 on the device are upcast
exactly before they reach this module.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "naive_softmax",
    "safe_softmax",
    "online_softmax",
    "blockwise_online_attention",
    "blockwise_attention_lazy_rescale",
    "attention_forward",
    "attention_backward",
    "head_forward_rows",
    "head_backward_rows",
    "head_backward_sampled",
    "attention_forward_suffix",
    "attention_forward_varlen",
    "attention_backward_varlen",
    "attention_flops",
]


# ---------------------------------------------------------------------------
# Softmax forms (P2 §2.1)
# ---------------------------------------------------------------------------

def naive_softmax(x):
    """Textbook softmax y_i = e^{x_i} / Σ_j e^{x_j} (P2 §2.1, first formula).

    Overflows for large inputs; kept only as the special case the safe form
    must agree with on moderate inputs."""
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def safe_softmax(x):
    """Safe softmax: subtract the row maximum m before exponentiating
    (P2 §2.1, second formula).  Entries equal to -inf contribute zero."""
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def online_softmax(x):
    """Streaming (online) softmax of a 1-D vector, one element at a time
    (P2 §2.1): m_i = max(m_{i-1}, x_i), d_i = d_{i-1}·e^{m_{i-1}-m_i} + e^{x_i-m_i},
    starting from m_0 = -inf, d_0 = 0; finally y_i = e^{x_i - m_n} / d_n.

    Returns ``(m_trace, d_trace, y)`` where the traces hold (m_i, d_i) after
    each element, so a test can compare every intermediate the page prints."""
    m_prev = -math.inf
    d_prev = 0.0
    m_trace, d_trace = [], []
    for xi in (float(v) for v in x):
        m_i = max(m_prev, xi)
        # e^{m_{i-1} - m_i} with m_0 = -inf is e^{-inf} = 0
        carry = 0.0 if m_prev == -math.inf else math.exp(m_prev - m_i)
        d_i = d_prev * carry + math.exp(xi - m_i)
        m_trace.append(m_i)
        d_trace.append(d_i)
        m_prev, d_prev = m_i, d_i
    y = [math.exp(float(v) - m_prev) / d_prev for v in x]
    return np.array(m_trace), np.array(d_trace), np.array(y)


def blockwise_online_attention(q, k, v, scale, kv_block, causal=False):
    """One query block attending to KV blocks streamed one at a time, with the
    per-row state (m, d, O) updated after every block as in P2 §2.2 steps 1-5:

      1. S_j = s·Q K_jᵀ
      2. m_j = rowmax(S_j)
      3. m_new = max(m_prev, m_j)
      4. d_new = e^{m_prev - m_new}·d_prev + e^{m_j - m_new}·Σ e^{S_j - m_j}
      5. O_new = (d_prev/d_new)·e^{m_prev - m_new}·O_prev
                 + (e^{m_j - m_new}/d_new)·exp(S_j - m_j) V_j

    In step 5 the page's ``softmax_j(S_j)`` is read as the un-normalised
    ``exp(S_j - m_j)``; with that reading O stays normalised after every step.
    ``kv_block`` is an int (fixed block size) or a list of block sizes summing
    to the number of keys.  q: [M, d], k, v: [N, d].  Returns (O, m, d)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n_keys = k.shape[0]
    if isinstance(kv_block, int):
        sizes = [kv_block] * (n_keys // kv_block)
        if n_keys % kv_block:
            sizes.append(n_keys % kv_block)
    else:
        sizes = list(kv_block)
    assert sum(sizes) == n_keys
    rows = q.shape[0]
    m_prev = np.full(rows, -np.inf)
    d_prev = np.zeros(rows)
    o_prev = np.zeros((rows, v.shape[1]))
    start = 0
    for size in sizes:
        kj, vj = k[start:start + size], v[start:start + size]
        s_j = scale * (q @ kj.T)                                   # step 1
        if causal:
            qi = np.arange(rows)[:, None]
            kj_idx = (start + np.arange(size))[None, :]
            s_j = np.where(kj_idx > qi, -np.inf, s_j)
        m_j = s_j.max(axis=1)                                      # step 2
        m_new = np.maximum(m_prev, m_j)                            # step 3
        # rows whose block is fully masked keep their state unchanged
        alive = np.isfinite(m_j)
        m_j_safe = np.where(alive, m_j, 0.0)
        m_new_safe = np.where(np.isfinite(m_new), m_new, 0.0)
        e_blk = np.where(alive[:, None], np.exp(s_j - m_j_safe[:, None]), 0.0)
        carry_prev = np.where(np.isfinite(m_prev), np.exp(m_prev - m_new_safe), 0.0)
        carry_blk = np.where(alive, np.exp(m_j_safe - m_new_safe), 0.0)
        d_new = carry_prev * d_prev + carry_blk * e_blk.sum(axis=1)   # step 4
        with np.errstate(invalid="ignore", divide="ignore"):
            o_new = ((d_prev / d_new * carry_prev)[:, None] * o_prev
                     + (carry_blk / d_new)[:, None] * (e_blk @ vj))     # step 5
        o_new = np.where((d_new > 0)[:, None], o_new, 0.0)
        m_prev, d_prev, o_prev = m_new, d_new, o_new
        start += size
    return o_prev, m_prev, d_prev


def _lazy_rescale(o, l, m_ref, m_new):
    """Move a row's accumulated output and normaliser from reference maximum
    m_ref to m_new (both scaled by e^{m_ref - m_new}); rows without any term
    yet (m_ref = -inf) hold zeros and stay zero."""
    alpha = np.where(np.isfinite(m_ref), np.exp(np.where(np.isfinite(m_ref), m_ref, 0.0) - m_new), 0.0)
    return alpha[:, None] * o, alpha * l


def blockwise_attention_lazy_rescale(q, k, v, scale, kv_block, tau, causal=False):
    """Blockwise attention with conditional rescaling, the FA4 technique that
    P1 "Key observations" names without giving its rule.  The reading taken:
    every row keeps a reference maximum m_ref and un-normalised accumulators
    O and l, all relative to m_ref.  For each KV block j:

      1. S_j = s·Q K_jᵀ (masked entries -inf), m_j = rowmax(S_j)
      2. if m_ref = -inf or m_j > m_ref + tau: rescale O and l by
         e^{m_ref - m_new} and set m_ref = m_new = max(m_ref, m_j)
         (otherwise keep the stale m_ref)
      3. O += exp(S_j - m_ref) V_j ;  l += Σ exp(S_j - m_ref)

    and at the end O/l, LSE = m_ref + ln l.  Because O and l always share one
    reference the result is the exact softmax for any tau >= 0; tau only
    bounds every term exp(S_j - m_ref) by e^tau.  The pages give no threshold:
    the kernels use 8 in base-2 units of the scaled scores, i.e.
    tau = 8·ln 2 here.  ``kv_block`` is an int or a list of block sizes.
    q: [M, d], k, v: [N, d].  Returns (O, LSE, rescales, max_term): the number
    of rescalings of each row after its first term, and the largest term
    exp(S_j - m_ref) met."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n_keys = k.shape[0]
    if isinstance(kv_block, int):
        sizes = [kv_block] * (n_keys // kv_block)
        if n_keys % kv_block:
            sizes.append(n_keys % kv_block)
    else:
        sizes = list(kv_block)
    assert sum(sizes) == n_keys and tau >= 0
    rows = q.shape[0]
    m_ref = np.full(rows, -np.inf)
    l = np.zeros(rows)
    o = np.zeros((rows, v.shape[1]))
    rescales = np.zeros(rows, np.int64)
    max_term = 0.0
    start = 0
    for size in sizes:
        kj, vj = k[start:start + size], v[start:start + size]
        s_j = scale * (q @ kj.T)                                       # step 1
        if causal:
            qi = np.arange(rows)[:, None]
            kj_idx = (start + np.arange(size))[None, :]
            s_j = np.where(kj_idx > qi, -np.inf, s_j)
        m_j = s_j.max(axis=1)
        need = np.isfinite(m_j) & (~np.isfinite(m_ref) | (m_j > m_ref + tau))   # step 2
        if need.any():
            m_new = np.where(need, np.maximum(m_ref, m_j), m_ref)
            o_s, l_s = _lazy_rescale(o, l, m_ref, m_new)
            o = np.where(need[:, None], o_s, o)
            l = np.where(need, l_s, l)
            rescales += (need & np.isfinite(m_ref)).astype(np.int64)
            m_ref = m_new
        live = np.isfinite(m_ref)
        e = np.where(live[:, None], np.exp(s_j - np.where(live, m_ref, 0.0)[:, None]), 0.0)   # step 3
        if e.size:
            max_term = max(max_term, float(e.max()))
        o = o + e @ vj
        l = l + e.sum(axis=1)
        start += size
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where((l > 0)[:, None], o / l[:, None], 0.0)
        lse = np.where(l > 0, m_ref + np.log(l), -np.inf)
    return out, lse, rescales, max_term


# ---------------------------------------------------------------------------
# Standard attention, materialised (P3 "attention 为什么一开始就很慢")
# ---------------------------------------------------------------------------

def _scores(qh, kh, scale, causal, rows=None):
    """s·Q Kᵀ for one head, with causal masking (key j > query i → -inf).
    ``rows`` selects query rows (default: all)."""
    if rows is None:
        rows = np.arange(qh.shape[0])
    s = scale * (qh[rows] @ kh.T)
    if causal:
        s = np.where(np.arange(kh.shape[0])[None, :] > rows[:, None], -np.inf, s)
    return s


def head_forward_rows(qh, kh, vh, scale, causal, rows=None):
    """Forward pass of one (batch, query head) for the selected query rows.

    qh: [N, d] queries of this head; kh, vh: [N, d] keys/values of the head it
    reads.  Returns (O[rows], LSE[rows], P[rows]) where P is the full
    probability row (safe softmax of the scaled, masked scores)."""
    qh = np.asarray(qh, np.float64)
    kh = np.asarray(kh, np.float64)
    vh = np.asarray(vh, np.float64)
    s = _scores(qh, kh, scale, causal, rows)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    o = p @ vh
    lse = (m + np.log(l))[:, 0]
    return o, lse, p


def attention_forward(q, k, v, scale, causal=False):
    """O = softmax(s·Q Kᵀ [+ causal mask]) V and LSE for every (b, h).

    q: [B, Hq, N, d]; k, v: [B, Hkv, N, d]; Hq must be a multiple of Hkv and
    query head h reads key/value head h // (Hq // Hkv).  Returns
    O [B, Hq, N, d] and LSE [B, Hq, N] (natural log), both float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            o[b, h], lse[b, h], _ = head_forward_rows(q[b, h], k[b, g], v[b, g], scale, causal)
    return o, lse


def attention_backward(q, k, v, do, scale, causal=False):
    """Gradients of the forward pass with respect to Q, K, V given dO.

    Chain rule on the definition (P is recomputed here, never supplied):
      dV_g += Pᵀ dO;  dP = dO Vᵀ;  D_i = Σ_c dO_ic O_ic;  dS = P ∘ (dP − D);
      dQ = s·dS K;  dK_g += s·dSᵀ Q.
    Returns (dq, dk, dv, o, lse) in float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            oh, lse[b, h], p = head_forward_rows(q[b, h], k[b, g], v[b, g], scale, causal)
            o[b, h] = oh
            dv[b, g] += p.T @ do[b, h]
            dp = do[b, h] @ v[b, g].T
            D = np.sum(do[b, h] * oh, axis=1, keepdims=True)
            ds = p * (dp - D)
            dq[b, h] = scale * (ds @ k[b, g])
            dk[b, g] += scale * (ds.T @ q[b, h])
    return dq, dk, dv, o, lse


def head_backward_rows(qh, kh, vh, doh, scale, causal, rows):
    """The share of one block of query rows in the backward pass of one
    (batch, query head).

    Same formulas as :func:`attention_backward`, restricted to the query rows
    ``rows`` (an index array): dQ of those rows is complete (it only involves
    their own rows of P), while dK and dV are sums over query rows, so the
    block contributes the partial sums  dV_part = P[rows]ᵀ dO[rows]  and
    dK_part = s·dS[rows]ᵀ Q[rows].  Summing the partials of blocks that
    partition all rows gives the head's dK and dV.

    qh, doh: [N, d]; kh, vh: [N, d].  Returns (dq_rows [R, d], dk_part [N, d],
    dv_part [N, d], o_rows [R, d], lse_rows [R])."""
    qh = np.asarray(qh, np.float64)
    kh = np.asarray(kh, np.float64)
    vh = np.asarray(vh, np.float64)
    doh = np.asarray(doh, np.float64)
    rows = np.asarray(rows)
    o_r, lse_r, p_r = head_forward_rows(qh, kh, vh, scale, causal, rows)
    do_r = doh[rows]
    dp_r = do_r @ vh.T
    D_r = np.sum(do_r * o_r, axis=1, keepdims=True)
    ds_r = p_r * (dp_r - D_r)
    dq_r = scale * (ds_r @ kh)
    dk_part = scale * (ds_r.T @ qh[rows])
    dv_part = p_r.T @ do_r
    return dq_r, dk_part, dv_part, o_r, lse_r


def head_backward_sampled(q_heads, kh, vh, do_heads, scale, causal, q_rows, k_rows,
                          row_chunk=2048):
    """Sampled backward entries for one key/value head and the G query heads
    that share it, for sizes where materialising whole gradients is too slow.

    q_heads, do_heads: [G, N, d]; kh, vh: [N, d].  Returns
      dq_rows [G, len(q_rows), d]  – dQ of the sampled query rows,
      dk_rows [len(k_rows), d], dv_rows [len(k_rows), d] – dK, dV of the
      sampled key rows, summed over the G query heads.
    Same formulas as :func:`attention_backward`.  dK/dV of a key row need the
    probabilities of that key column for every query row, hence LSE and D for
    every row; those are row-local quantities, computed ``row_chunk`` rows at
    a time only to bound memory (each row is still one exact softmax)."""
    q_heads = np.asarray(q_heads, np.float64)
    do_heads = np.asarray(do_heads, np.float64)
    kh = np.asarray(kh, np.float64)
    vh = np.asarray(vh, np.float64)
    G, N, d = q_heads.shape
    q_rows = np.asarray(q_rows)
    k_rows = np.asarray(k_rows)
    dq_rows = np.zeros((G, len(q_rows), d))
    dk_rows = np.zeros((len(k_rows), d))
    dv_rows = np.zeros((len(k_rows), d))
    for g in range(G):
        qh, doh = q_heads[g], do_heads[g]
        # dQ rows: everything they need is in their own rows
        o_r, _, p_r = head_forward_rows(qh, kh, vh, scale, causal, q_rows)
        dp_r = doh[q_rows] @ vh.T
        D_r = np.sum(doh[q_rows] * o_r, axis=1, keepdims=True)
        dq_rows[g] = scale * ((p_r * (dp_r - D_r)) @ kh)
        # dK/dV rows: need P[:, k_rows] for every query row
        for start in range(0, N, row_chunk):
            rows = np.arange(start, min(N, start + row_chunk))
            o_c, _, p_c = head_forward_rows(qh, kh, vh, scale, causal, rows)
            D_c = np.sum(doh[rows] * o_c, axis=1, keepdims=True)
            p_cols = p_c[:, k_rows]                          # [rows, K]
            dp_cols = doh[rows] @ vh[k_rows].T               # [rows, K]
            ds_cols = p_cols * (dp_cols - D_c)
            dv_rows += p_cols.T @ doh[rows]
            dk_rows += scale * (ds_cols.T @ qh[rows])
    return dq_rows, dk_rows, dv_rows


# ---------------------------------------------------------------------------
# Fewer queries than keys: the queries are the last positions of the sequence
# ---------------------------------------------------------------------------

def attention_forward_suffix(q, k, v, scale, causal=False):
    """Attention of Nq queries against Nk keys when the queries are the last Nq
    positions of an Nk-long sequence (decoding against cached keys and values).

    The pages define the causal mask for equal lengths only (key j is visible
    to the query at position i iff j <= i).  Reading used here: query row r
    sits at position Nk - Nq + r, so key j is masked iff j > Nk - Nq + r; then
    these rows are exactly the last Nq rows of the square computation over the
    whole sequence.  Without the mask every query sees all Nk keys.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] (Nq <= Nk when causal).  Returns
    O [B, Hq, Nq, d] and LSE [B, Hq, Nq] (natural log), float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    pos = (Nk - Nq) + np.arange(Nq)  # sequence position of each query row
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = scale * (q[b, h] @ k[b, g].T)
            if causal:
                s = np.where(np.arange(Nk)[None, :] > pos[:, None], -np.inf, s)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, h] = (e / l) @ v[b, g]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


# ---------------------------------------------------------------------------
# Packed batches of sequences with different lengths
# ---------------------------------------------------------------------------

def _varlen_bounds(cu_seqlens, T):
    cu = [int(c) for c in cu_seqlens]
    assert cu[0] == 0 and cu[-1] == T and all(a <= b for a, b in zip(cu, cu[1:])), cu
    return cu


def attention_forward_varlen(q, k, v, cu_seqlens, scale, causal=False):
    """Attention over a packed batch of independent sequences of different
    lengths ("Flash-Attention" concept page, "Design space and trade-offs":
    ragged batches change which tiles are legal and how work balances).

    Sequence b holds tokens cu_seqlens[b] .. cu_seqlens[b+1]-1 of the packed
    token axis; its queries see only its own keys (causal: key j of the
    sequence is masked for query i of the sequence when j > i, positions
    counted from the sequence's first token).  So every sequence is exactly one
    call of :func:`attention_forward` on its own tokens.

    q: [Hq, T, d]; k, v: [Hkv, T, d] (heads first, sequences back to back along
    the token axis); cu_seqlens: nseq + 1 non-decreasing offsets from 0 to T.
    Returns O [Hq, T, d] and LSE [Hq, T] (natural log), float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    Hq, T, d = q.shape
    cu = _varlen_bounds(cu_seqlens, T)
    o = np.zeros_like(q)
    lse = np.zeros((Hq, T))
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        if hi == lo:
            continue
        ob, lb = attention_forward(q[None, :, lo:hi], k[None, :, lo:hi], v[None, :, lo:hi], scale, causal)
        o[:, lo:hi], lse[:, lo:hi] = ob[0], lb[0]
    return o, lse


def attention_backward_varlen(q, k, v, do, cu_seqlens, scale, causal=False):
    """Gradients of :func:`attention_forward_varlen`: each sequence is one
    call of :func:`attention_backward` on its own tokens (the sequences share
    no keys, so nothing couples their gradients).  Layouts as in the forward;
    do: [Hq, T, d].  Returns (dq, dk, dv, o, lse) in float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    Hq, T, d = q.shape
    cu = _varlen_bounds(cu_seqlens, T)
    dq, dk, dv, o = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(q)
    lse = np.zeros((Hq, T))
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        if hi == lo:
            continue
        r = attention_backward(q[None, :, lo:hi], k[None, :, lo:hi], v[None, :, lo:hi], do[None, :, lo:hi],
                               scale, causal)
        dq[:, lo:hi], dk[:, lo:hi], dv[:, lo:hi], o[:, lo:hi], lse[:, lo:hi] = (x[0] for x in r)
    return dq, dk, dv, o, lse


def attention_flops(B, Hq, N, d, causal):
    """Algorithmic FLOPs of one forward pass: 4·B·Hq·N²·d (two N×N×d matrix
    products), halved when causal.  The backward pass counts 2.5× this."""
    f = 4.0 * B * Hq * N * N * d
    return f / 2 if causal else f
