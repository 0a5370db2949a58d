"""Use patterns beyond one call at a time on the default stream.  A CUDA graph
captures the forward and the backward and replays them.  Two different
problems run concurrently on two streams: the persistent forward and the
banded backward keep no state outside their arguments.  Both must give the
results of the ordinary calls: O, LSE, dK and dV bit for bit (their reduction
order is fixed), and dQ up to the order of its fp32 reduce-adds."""

import pytest
import torch

from exact_attention_104_b200 import attention_backward, attention_forward, binding, lib
from exact_attention_104_b200.workloads import Workload, make_inputs

from _parity import f64, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _short_waits():
    lib().fa_set_wait_cap(1 << 28)
    yield
    lib().fa_set_wait_cap(0)


def _buffers(w, q, k):
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(k)
    ws = torch.empty(binding.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8,
                     device=q.device)
    return o, lse, dq, dk, dv, ws


def _step(w, q, k, v, do, bufs, stream):
    o, lse, dq, dk, dv, ws = bufs
    attention_forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
    attention_backward(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                       stream=stream)


def _assert_same(bufs, ref):
    o, lse, dq, dk, dv, _ = bufs
    ro, rlse, rdq, rdk, rdv, _ = ref
    assert torch.equal(o, ro) and torch.equal(lse, rlse)
    assert torch.equal(dk, rdk) and torch.equal(dv, rdv)
    assert rel_fro(f64(dq), f64(rdq)) <= 1e-3


def test_forward_and_backward_replayed_from_a_cuda_graph():
    w = Workload("graph_gqa_causal", 2, 4, 2, 640, 128, True, 1.0, 71)
    q, k, v, do = make_inputs(w, "cuda")
    ref = _buffers(w, q, k)
    _step(w, q, k, v, do, ref, None)
    bufs = _buffers(w, q, k)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    _step(w, q, k, v, do, bufs, s)  # first calls (attribute set-up) outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _step(w, q, k, v, do, bufs, s)
    for _ in range(3):
        for t in bufs[:5]:
            t.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    _assert_same(bufs, ref)


def test_two_problems_on_two_streams_at_once():
    wa = Workload("streams_a", 2, 4, 4, 1024, 128, False, 1.0, 81)
    wb = Workload("streams_b", 1, 4, 1, 777, 64, True, 1.0, 82)
    ins = [make_inputs(w, "cuda") for w in (wa, wb)]
    refs = []
    for w, (q, k, v, do) in zip((wa, wb), ins):
        r = _buffers(w, q, k)
        _step(w, q, k, v, do, r, None)
        refs.append(r)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [_buffers(w, q, k) for w, (q, k, v, do) in zip((wa, wb), ins)]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for _ in range(3):
        for w, (q, k, v, do), bufs, s in zip((wa, wb), ins, outs, streams):
            with torch.cuda.stream(s):
                _step(w, q, k, v, do, bufs, s)
    torch.cuda.synchronize()
    assert binding.fa_device_status() == binding.FA_OK
    for bufs, ref in zip(outs, refs):
        _assert_same(bufs, ref)
