"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the fp64 oracle on the same bf16 inputs, and compare with the tolerances
of the specification (bf16 O: max-abs <= 2e-2, mean-abs <= 2e-3; LSE: max-abs
<= 1e-3; dQ, dK, dV: relative Frobenius error <= 2e-2)."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_attention_104_b200 import attention_backward, attention_forward, fa_device_status, lib
from exact_attention_104_b200.workloads import Workload, make_inputs

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_FRO = 2e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(a, b) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def run_gpu(w: Workload, inputs=None, bwd=True):
    q, k, v, do = inputs if inputs is not None else make_inputs(w, "cuda")
    o, lse = attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    out = {"q": q, "k": k, "v": v, "do": do, "o": o, "lse": lse}
    if bwd:
        dq, dk, dv = attention_backward(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    st = fa_device_status()
    assert st == 0, f"device status {st}"
    return out


def compare_full(w: Workload, g, bwd=True):
    """Whole-tensor comparison against the oracle (small sizes)."""
    q, k, v, do = (f64(g[n]) for n in ("q", "k", "v", "do"))
    if bwd:
        dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, do, w.scale, w.causal)
    else:
        o, lse = oracle.attention_forward(q, k, v, w.scale, w.causal)
    err = {
        "o_max": float(np.max(np.abs(f64(g["o"]) - o))),
        "o_mean": float(np.mean(np.abs(f64(g["o"]) - o))),
        "lse_max": float(np.max(np.abs(f64(g["lse"]) - lse))),
    }
    if bwd:
        err.update(dq=rel_fro(f64(g["dq"]), dq), dk=rel_fro(f64(g["dk"]), dk), dv=rel_fro(f64(g["dv"]), dv))
    return err


def compare_sampled(w: Workload, g, units, n_rows=48, seed=0, bwd=True):
    """Compare sampled rows of the given (b, kv_head) units against the oracle,
    computed one head at a time; returns the worst errors over the sample."""
    rng = np.random.default_rng(seed)
    N = w.N
    o_abs, lse_abs = [], []
    dq_pairs, dk_pairs, dv_pairs = [], [], []
    for (b, g_kv) in units:
        kh, vh = f64(g["k"][b, g_kv]), f64(g["v"][b, g_kv])
        heads = list(range(g_kv * w.G, (g_kv + 1) * w.G))
        # always include the first and last rows of the sequence and of a tile,
        # and the first row of the last (possibly partial) tile
        last_tile = (N - 1) // 128 * 128
        fixed = np.array(sorted({r for r in (0, 127, 128, N - 128, last_tile - 1, last_tile, N - 1) if 0 <= r < N}))
        rows = np.unique(np.concatenate([fixed, rng.choice(N, min(n_rows, N), replace=False)]))
        krows = np.unique(np.concatenate([fixed, rng.choice(N, min(n_rows, N), replace=False)]))
        qh_all = np.stack([f64(g["q"][b, h]) for h in heads])
        doh_all = np.stack([f64(g["do"][b, h]) for h in heads])
        for i, h in enumerate(heads):
            o_ref, lse_ref, _ = oracle.head_forward_rows(qh_all[i], kh, vh, w.scale, w.causal, rows)
            o_abs.append(np.abs(f64(g["o"][b, h][rows]) - o_ref))
            lse_abs.append(np.abs(f64(g["lse"][b, h][rows]) - lse_ref))
        if bwd:
            dq_r, dk_r, dv_r = oracle.head_backward_sampled(qh_all, kh, vh, doh_all, w.scale, w.causal, rows, krows)
            for i, h in enumerate(heads):
                dq_pairs.append((f64(g["dq"][b, h][rows]), dq_r[i]))
            dk_pairs.append((f64(g["dk"][b, g_kv][krows]), dk_r))
            dv_pairs.append((f64(g["dv"][b, g_kv][krows]), dv_r))
    o_abs = np.concatenate([x.ravel() for x in o_abs])
    err = {"o_max": float(o_abs.max()), "o_mean": float(o_abs.mean()),
           "lse_max": float(np.concatenate(lse_abs).max())}
    if bwd:
        for name, pairs in (("dq", dq_pairs), ("dk", dk_pairs), ("dv", dv_pairs)):
            mine = np.concatenate([p[0].ravel() for p in pairs])
            ref = np.concatenate([p[1].ravel() for p in pairs])
            err[name] = rel_fro(mine, ref)
    return err


def assert_within_tolerance(err: dict, bwd=True):
    msg = str(err)
    assert err["o_max"] <= O_MAX_ABS, msg
    assert err["o_mean"] <= O_MEAN_ABS, msg
    assert err["lse_max"] <= LSE_MAX_ABS, msg
    if bwd:
        for n in ("dq", "dk", "dv"):
            assert err[n] <= GRAD_REL_FRO, msg


def ensure_lib():
    lib()
