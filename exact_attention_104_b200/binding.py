"""ctypes binding for libfa_b200.so (argument marshalling only).

Every function here forwards to the C ABI declared in ``include/fa.h``; all
arithmetic runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or the device is unsupported, calls raise ``FAError``.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

# FA_B200_DEBUG=1 selects the debug build (device-side checks, -DFA_DEBUG)
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libfa_b200_debug.so" if os.environ.get("FA_B200_DEBUG") == "1" else "libfa_b200.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_DEVICE_CHECK = range(6)

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fa_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FAError(FA_ERR_UNSUPPORTED, f"{LIB_PATH} is missing; build it with "
                      "`python -m exact_attention_104_b200.build`"
                      + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.fa_fwd.restype = i
    L.fa_fwd_pair.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.fa_fwd_pair.restype = i
    L.fa_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
    L.fa_bwd_workspace_bytes.restype = z
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, z, vp]
    L.fa_bwd.restype = i
    L.fa_device_status.argtypes = [vp]
    L.fa_device_status.restype = i
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_set_wait_cap.argtypes = [ctypes.c_longlong]
    L.fa_set_wait_cap.restype = i
    L.fa_profile_next.argtypes = [vp, vp]
    L.fa_profile_next.restype = i
    L.fa_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
    L.fa_selftest_wait_timeout.restype = i
    L.fa_selftest_exp2.argtypes = [vp, vp, ctypes.c_longlong, i, vp]
    L.fa_selftest_exp2.restype = i
    L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.fa_bwd_noalloc.restype = i
    L.fa_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
    L.fa_decode_workspace_bytes.restype = z
    L.fa_fwd_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, z, vp]
    L.fa_fwd_decode.restype = i
    L.fa_fwd_varlen_workspace_bytes.argtypes = [i, i, i, i, i, i]
    L.fa_fwd_varlen_workspace_bytes.restype = z
    L.fa_bwd_varlen_workspace_bytes.argtypes = [i, i, i, i, i, i]
    L.fa_bwd_varlen_workspace_bytes.restype = z
    L.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, z, vp]
    L.fa_fwd_varlen.restype = i
    L.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, z, vp]
    L.fa_bwd_varlen.restype = i
    _lib = L
    return L


def fa_status_string(status: int) -> str:
    try:
        return lib().fa_status_string(int(status)).decode()
    except FAError:
        return {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
                4: "device wait timed out"}.get(int(status), "unknown status")


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _stream_handle(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != FA_OK:
        raise FAError(status, where)


def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream=None) -> int:
    """Raw C-ABI call; tensors or integer device pointers.  Returns the status."""
    return lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                        int(bool(causal)), float(scale), _stream_handle(stream))


def fa_fwd_pair(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream=None) -> int:
    """Raw C-ABI call of the forward pass on CTA pairs (d = 128).  Returns the
    status."""
    return lib().fa_fwd_pair(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                             int(bool(causal)), float(scale), _stream_handle(stream))


def fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, Hq, Hkv, N, d))


def fa_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, workspace, workspace_bytes,
           stream=None) -> int:
    """Raw C-ABI call; tensors or integer device pointers.  Returns the status."""
    return lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                        B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _ptr(workspace),
                        int(workspace_bytes), _stream_handle(stream))


def fa_selftest_wait_timeout(cap_cycles: int, stream=None) -> int:
    return lib().fa_selftest_wait_timeout(int(cap_cycles), _stream_handle(stream))


def fa_selftest_exp2(x, y, use_poly: bool, stream=None) -> int:
    return lib().fa_selftest_exp2(_ptr(x), _ptr(y), int(x.numel()), int(bool(use_poly)), _stream_handle(stream))


FA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, stream=None) -> int:
    """Raw C-ABI call of the backward pass that uses the library's fixed
    device scratch array instead of a caller workspace (for callers that
    cannot allocate device memory).  Returns the status."""
    return lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, Hq, Hkv, N, d, int(bool(causal)), float(scale),
                                _stream_handle(stream))


def fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d) -> int:
    return lib().fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d)


def fa_fwd_decode(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, workspace, workspace_bytes,
                  stream=None) -> int:
    """Raw C-ABI call of the decoding forward pass (Nq queries, the last
    positions of an Nk-long sequence).  Returns the status."""
    return lib().fa_fwd_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d,
                               int(bool(causal)), float(scale), _ptr(workspace), int(workspace_bytes),
                               _stream_handle(stream))


def fa_fwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d) -> int:
    return int(lib().fa_fwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d))


def fa_bwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d) -> int:
    return int(lib().fa_bwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d))


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, nseq, Hq, Hkv, T, max_seqlen, d, causal, scale, workspace,
                  workspace_bytes, stream=None) -> int:
    """Raw C-ABI call of the packed variable-length forward pass (sequences
    back to back along the token axis of [H, T, d] tensors, boundaries in the
    device int32 tensor cu_seqlens).  Returns the status."""
    return lib().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), nseq, Hq, Hkv, T,
                               max_seqlen, d, int(bool(causal)), float(scale), _ptr(workspace),
                               int(workspace_bytes), _stream_handle(stream))


def fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu_seqlens, nseq, Hq, Hkv, T, max_seqlen, d, causal, scale,
                  workspace, workspace_bytes, stream=None) -> int:
    """Raw C-ABI call of the packed variable-length backward pass.  Returns
    the status."""
    return lib().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(cu_seqlens), nseq, Hq, Hkv, T, max_seqlen, d, int(bool(causal)),
                               float(scale), _ptr(workspace), int(workspace_bytes), _stream_handle(stream))


def fa_profile_next(start_event=None, stop_event=None) -> int:
    """Ask the next fa_fwd / fa_bwd call on this thread to record the given
    torch.cuda.Event objects around its attention kernel."""
    for ev in (start_event, stop_event):
        if ev is not None and not ev.cuda_event:
            ev.record()  # torch creates the underlying cudaEvent lazily
    s = start_event.cuda_event if start_event is not None else None
    e = stop_event.cuda_event if stop_event is not None else None
    return lib().fa_profile_next(s, e)


def fa_device_status(stream=None) -> int:
    return lib().fa_device_status(_stream_handle(stream))


def _shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError(f"incompatible shapes q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    return B, Hq, k.shape[1], N, d


def attention_forward(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None):
    """O, LSE = exact attention of bf16 [B,H,N,d] tensors on the current CUDA
    device (no CPU path).  Returns (o bf16 [B,Hq,N,d], lse fp32 [B,Hq,N])."""
    B, Hq, Hkv, N, d = _shapes(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    _check(fa_fwd(q, k, v, out, lse, B, Hq, Hkv, N, d, causal, scale, stream), "fa_fwd")
    return out, lse


def attention_backward(q, k, v, o, lse, do, causal=False, scale=None, dq=None, dk=None, dv=None,
                       workspace=None, stream=None):
    """dQ, dK, dV of exact attention given the forward outputs and dO."""
    B, Hq, Hkv, N, d = _shapes(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_workspace_bytes(B, Hq, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(fa_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, workspace,
                  workspace.numel() * workspace.element_size(), stream), "fa_bwd")
    return dq, dk, dv


def attention_decode(q, k, v, causal=False, scale=None, out=None, lse=None, workspace=None, stream=None):
    """O, LSE of Nq queries q [B,Hq,Nq,d] against cached k, v [B,Hkv,Nk,d]; the
    queries are the last Nq positions of the sequence (see fa_fwd_decode)."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4 or k.shape != v.shape:
        raise FAError(FA_ERR_INVALID_ARG, "attention_decode: q, k, v must be [B,H,N,d] with k.shape == v.shape")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != d:
        raise FAError(FA_ERR_INVALID_ARG, "attention_decode: batch or head dimension mismatch")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise FAError(FA_ERR_INVALID_ARG, "attention_decode: inputs must be contiguous bf16 CUDA tensors")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=q.device)
    need = fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(fa_fwd_decode(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, workspace,
                         workspace.numel() * workspace.element_size(), stream), "fa_fwd_decode")
    return out, lse


def _varlen_shapes(q, k, v, cu_seqlens):
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape:
        raise FAError(FA_ERR_INVALID_ARG, "varlen: q must be [Hq, T, d] and k, v [Hkv, T, d]")
    Hq, T, d = q.shape
    if k.shape[1] != T or k.shape[2] != d:
        raise FAError(FA_ERR_INVALID_ARG, "varlen: token or head dimension mismatch")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise FAError(FA_ERR_INVALID_ARG, "varlen: q, k, v must be contiguous bf16 CUDA tensors")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise FAError(FA_ERR_INVALID_ARG, "varlen: cu_seqlens must be a 1-D int32 CUDA tensor")
    return Hq, k.shape[0], T, d, cu_seqlens.numel() - 1


def attention_forward_varlen(q, k, v, cu_seqlens, max_seqlen, causal=False, scale=None, out=None, lse=None,
                             workspace=None, stream=None):
    """O, LSE of a packed batch: q [Hq, T, d], k, v [Hkv, T, d] bf16 with the
    sequences back to back along T (boundaries in the int32 CUDA tensor
    cu_seqlens); each sequence attends only to itself.  max_seqlen bounds
    every length.  Returns (o bf16 [Hq, T, d], lse fp32 [Hq, T])."""
    Hq, Hkv, T, d, nseq = _varlen_shapes(q, k, v, cu_seqlens)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, T, dtype=torch.float32, device=q.device)
    need = fa_fwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(fa_fwd_varlen(q, k, v, out, lse, cu_seqlens, nseq, Hq, Hkv, T, max_seqlen, d, causal, scale, workspace,
                         workspace.numel() * workspace.element_size(), stream), "fa_fwd_varlen")
    return out, lse


def attention_backward_varlen(q, k, v, o, lse, do, cu_seqlens, max_seqlen, causal=False, scale=None, dq=None,
                              dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of a packed batch given the forward outputs and dO."""
    Hq, Hkv, T, d, nseq = _varlen_shapes(q, k, v, cu_seqlens)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, max_seqlen, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu_seqlens, nseq, Hq, Hkv, T, max_seqlen, d, causal,
                         scale, workspace, workspace.numel() * workspace.element_size(), stream), "fa_bwd_varlen")
    return dq, dk, dv
