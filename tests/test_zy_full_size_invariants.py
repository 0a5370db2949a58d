"""Softmax row sums and gradient column sums on the GPU at every workload's
full size, with no oracle.

The rows of P sum to one (the invariant the "Flash-Attention" concept page
names as a check for silent data corruption, "Key observations").  So with
V = 1 every row of O is 1, up to the rounding of P to bf16 before the PV
product (relative error at most 2^-9 per term, so at most 2^-9 for the row)
and the rounding of O to bf16 (which maps anything that close to 1 to 1).
The log-sum-exp does not depend on V at all, so it must be bit-identical to
the LSE of the same call with the workload's own V.  The decoding pass obeys
the same invariant (its P stays in fp32).

The same fact fixes two column sums of the backward pass over every row:
Σ_keys dV = Σ_queries dO (dV = Pᵀ dO and the rows of P sum to one), and
Σ_keys dK = 0 (Σ_j dS_ij = Σ_j P_ij dP_ij − D_i = 0 because D_i = dO_i·O_i
= Σ_j P_ij dP_ij), both per (batch, kv head), summed over the query heads of
its group.  The tolerances come from emulating the kernels' bf16 roundings
(P, dS, O, dK, dV) in fp64 on N = 1024-2000 heads: relative error of the dV
sum at most 1.6e-3 (d = 256, Q, K ~ N(0, 9)) and |Σ dK| at most 5.2e-3 of
the root-sum-square of the dK rows; a D off by 1 % gives 1.2e-2 for dK and
one key column dropped from P gives 1.5e-2 for dV.

This file is named to be collected after the other GPU tests and before the
no-allocation test, which comes last."""

import pytest
import torch

from exact_attention_104_b200 import attention_backward, attention_decode, attention_forward, binding
from exact_attention_104_b200.workloads import DECODE_WORKLOADS, WORKLOADS, make_decode_inputs, make_inputs

pytestmark = pytest.mark.gpu

# 2^-9 from the bf16 P, with room to spare for fp32 accumulation and 1/l
ROW_SUM_TOL = 1e-2
DV_SUM_REL_TOL = 5e-3
DK_SUM_RATIO_TOL = 1e-2


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_rows_of_p_sum_to_one_at_full_size(name):
    w = WORKLOADS[name]
    q, k, v, _ = make_inputs(w, "cuda")
    _, lse = attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    o1, lse1 = attention_forward(q, k, torch.ones_like(v), causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    err = (o1.float() - 1.0).abs().max().item()
    assert err <= ROW_SUM_TOL, f"{name}: max |O - 1| = {err:.3e} with V = 1"
    assert torch.equal(lse, lse1), f"{name}: the LSE changed with V"


@pytest.mark.parametrize("name", list(DECODE_WORKLOADS))
def test_decode_rows_sum_to_one(name):
    w = DECODE_WORKLOADS[name]
    q, k, v = make_decode_inputs(w, "cuda")
    _, lse = attention_decode(q, k, v, causal=w.causal, scale=w.scale)
    o1, lse1 = attention_decode(q, k, torch.ones_like(v), causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    err = (o1.float() - 1.0).abs().max().item()
    assert err <= ROW_SUM_TOL, f"{name}: max |O - 1| = {err:.3e} with V = 1"
    assert torch.equal(lse, lse1), f"{name}: the LSE changed with V"


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_gradient_column_sums_at_full_size(name):
    w = WORKLOADS[name]
    q, k, v, do = make_inputs(w, "cuda")
    o, lse = attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    dq, dk, dv = attention_backward(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    sum_dv = dv.double().sum(dim=2)                                           # [B, Hkv, d]
    sum_do = do.double().view(w.B, w.Hkv, w.G, w.N, w.d).sum(dim=(2, 3))     # [B, Hkv, d]
    rel_dv = ((sum_dv - sum_do).norm(dim=-1) / sum_do.norm(dim=-1)).max().item()
    dk64 = dk.double()
    ratio_dk = (dk64.sum(dim=2).norm(dim=-1) / dk64.pow(2).sum(dim=(2, 3)).sqrt()).max().item()
    assert rel_dv <= DV_SUM_REL_TOL, f"{name}: |sum dV - sum dO| / |sum dO| = {rel_dv:.3e}"
    assert ratio_dk <= DK_SUM_RATIO_TOL, f"{name}: |sum dK| / rss(dK rows) = {ratio_dk:.3e}"
