"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (for example a plugin inside a host framework that owns every byte of
device memory, or a latency-critical loop that must not call cudaMalloc).  It
takes no workspace and uses the library's fixed 64 MiB device scratch array.

Checked through the C ABI against the ordinary workspace entry point, fa_bwd,
on two calls in a row (the array keeps the previous call's contents, so the
second call shows that nothing stale leaks into the result).  This file is
named to be collected after the parity tests."""

import pytest
import torch

from exact_attention_104_b200 import attention_forward, binding
from exact_attention_104_b200.workloads import Workload, make_inputs

from _parity import GRAD_REL_FRO, f64, rel_fro

pytestmark = pytest.mark.gpu


def _workspace_bwd(w, q, k, v, o, lse, do):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    need = binding.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = binding.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, w.B, w.Hq, w.Hkv, w.N, w.d, w.causal, w.scale, ws, need)
    assert st == binding.FA_OK
    return dq, dk, dv


@pytest.mark.parametrize("w", [
    Workload("na_d128_gqa_causal", 2, 4, 2, 512, 128, True, 1.0, 61),
    Workload("na_d64", 1, 2, 2, 384, 64, False, 1.0, 62),
    Workload("na_d256", 1, 2, 1, 256, 256, False, 1.0, 63),
    Workload("na_d128_ragged_causal", 1, 2, 2, 300, 128, True, 1.0, 65),
], ids=lambda w: w.name)
def test_noalloc_backward_matches_workspace_backward_on_two_calls(w):
    assert binding.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d) <= binding.FA_NOALLOC_SCRATCH_BYTES
    q, k, v, do = make_inputs(w, "cuda")
    o, lse = attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    ref = _workspace_bwd(w, q, k, v, o, lse, do)
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st = binding.fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, w.B, w.Hq, w.Hkv, w.N, w.d, w.causal,
                                    w.scale)
        assert st == binding.FA_OK, binding.fa_status_string(st)
        torch.cuda.synchronize()
        assert binding.fa_device_status() == binding.FA_OK
        for name, mine, theirs in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            err = rel_fro(f64(mine), f64(theirs))
            assert err <= GRAD_REL_FRO, (call, name, err)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    w = Workload("na_big", 8, 16, 16, 2048, 128, False, 1.0, 64)  # needs about 130 MiB (136 MB) of scratch
    assert binding.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d) > binding.FA_NOALLOC_SCRATCH_BYTES
    shape_q = (w.B, w.Hq, w.N, w.d)
    t = lambda: torch.zeros(shape_q, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    q, k, v, o, do, dq, dk, dv = (t() for _ in range(8))
    lse = torch.zeros(w.B, w.Hq, w.N, device="cuda")
    st = binding.fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, w.B, w.Hq, w.Hkv, w.N, w.d, False, w.scale)
    assert st == binding.FA_ERR_UNSUPPORTED
