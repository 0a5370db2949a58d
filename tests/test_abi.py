"""C-ABI checks that need no GPU: the library loads, exports every function
``include/fa.h`` declares, and rejects invalid arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

from exact_attention_104_b200 import binding
from exact_attention_104_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.lib()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(fa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_device_status", "fa_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code in range(6):
        assert binding.fa_status_string(code) != "unknown status"
    assert binding.fa_status_string(binding.FA_ERR_DEVICE_CHECK) == "device-side check failed (debug build)"
    assert binding.fa_status_string(99) == "unknown status"


def test_debug_build_compiles_and_exports_the_same_symbols(tmp_path):
    # the -DFA_DEBUG variant (device-side checks of bulk-copy coordinates)
    path = build(force=True, debug=True, out=str(tmp_path / "libfa_b200_debug.so"))
    dbg = ctypes.CDLL(path)
    for name in _declared_functions():
        assert hasattr(dbg, name), name
    dbg.fa_status_string.argtypes = [ctypes.c_int]
    dbg.fa_status_string.restype = ctypes.c_char_p
    assert dbg.fa_status_string(binding.FA_ERR_DEVICE_CHECK) == b"device-side check failed (debug build)"


def test_workspace_bytes_formula(lib):
    # two fp32 row vectors and an fp32 [B,Hq,Np,d] accumulator, each 256-rounded,
    # with Np = N rounded up to a multiple of 128 (per-head padding rows), and
    # 256 bytes for the main kernel's unit counter
    B, Hq, Hkv, N, d = 8, 16, 16, 2048, 128
    rows = B * Hq * N
    assert binding.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) == 2 * rows * 4 + rows * d * 4 + 256
    assert binding.fa_bwd_workspace_bytes(1, 1, 1, 128, 64) == 2 * 512 + 128 * 64 * 4 + 256
    assert binding.fa_bwd_workspace_bytes(1, 1, 1, 100, 64) == 2 * 512 + 128 * 64 * 4 + 256
    assert binding.fa_bwd_workspace_bytes(2, 3, 1, 129, 256) == 2 * 1536 * 4 + 1536 * 256 * 4 + 256
    assert binding.fa_bwd_workspace_bytes(1, 1, 1, 1, 128) == 2 * 512 + 128 * 128 * 4 + 256
    assert binding.fa_bwd_workspace_bytes(1, 3, 2, 128, 64) == 0      # Hq % Hkv != 0
    assert binding.fa_bwd_workspace_bytes(1, 2, 2, 128, 96) == 0      # unsupported d


FAKE = 1 << 20  # an aligned, non-null address; validation must reject before any use


def _fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5,
             B=1, Hq=2, Hkv=2, N=128, d=64, causal=0, scale=0.125, stream=0)
    a.update(kw)
    return binding.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                          a["causal"], a["scale"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA_ERR_INVALID_ARG),
    (dict(lse=0), binding.FA_ERR_INVALID_ARG),
    (dict(k=FAKE * 2 + 8), binding.FA_ERR_INVALID_ARG),          # misaligned
    (dict(Hq=3, Hkv=2), binding.FA_ERR_INVALID_ARG),
    (dict(Hq=0), binding.FA_ERR_INVALID_ARG),
    (dict(B=-1), binding.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), binding.FA_ERR_INVALID_ARG),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(d=0), binding.FA_ERR_INVALID_ARG),
    (dict(B=70000), binding.FA_ERR_UNSUPPORTED),
    (dict(B=1024, Hq=1024, Hkv=1024, N=4096), binding.FA_ERR_UNSUPPORTED),
    (dict(B=1024, Hq=1024, Hkv=1024, N=1921), binding.FA_ERR_UNSUPPORTED),  # B·Hq·pad128(N) = 2^31
    (dict(o=FAKE), binding.FA_ERR_INVALID_ARG),                  # output aliases q
    (dict(lse=FAKE * 4 + 64), binding.FA_ERR_INVALID_ARG),       # lse overlaps o
    (dict(B=0, q=0, k=0, v=0, o=0, lse=0), binding.FA_OK),       # empty problem: nothing to do
    (dict(N=0), binding.FA_OK),
])
def test_fwd_argument_validation(lib, kw, expect):
    assert _fwd(lib, **kw) == expect


def _bwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5, do=FAKE * 6, dq=FAKE * 7, dk=FAKE * 8,
             dv=FAKE * 9, B=1, Hq=2, Hkv=2, N=128, d=64, causal=0, scale=0.125, ws=FAKE * 10, wsb=1 << 20)
    a.update(kw)
    return binding.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"], a["dv"],
                          a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["causal"], a["scale"], a["ws"], a["wsb"], 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(do=0), binding.FA_ERR_INVALID_ARG),
    (dict(ws=0), binding.FA_ERR_INVALID_ARG),
    (dict(ws=FAKE * 10 + 16), binding.FA_ERR_INVALID_ARG),       # workspace not 256-aligned
    (dict(wsb=100), binding.FA_ERR_INVALID_ARG),                 # workspace too small
    (dict(dq=FAKE), binding.FA_ERR_INVALID_ARG),                 # dq aliases q
    (dict(dk=FAKE * 7), binding.FA_ERR_INVALID_ARG),             # dk aliases dq
    (dict(ws=FAKE * 9), binding.FA_ERR_INVALID_ARG),             # workspace aliases dv
    (dict(Hq=4, Hkv=3), binding.FA_ERR_INVALID_ARG),
    (dict(d=32), binding.FA_ERR_UNSUPPORTED),
    (dict(B=1024, Hq=1024, Hkv=1024, N=2047), binding.FA_ERR_UNSUPPORTED),  # padded rows reach 2^31
    (dict(B=0), binding.FA_OK),
])
def test_bwd_argument_validation(lib, kw, expect):
    assert _bwd(lib, **kw) == expect


def test_wait_cap_setter(lib):
    assert lib.fa_set_wait_cap(-1) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_set_wait_cap(1 << 28) == binding.FA_OK
    assert lib.fa_set_wait_cap(0) == binding.FA_OK


def test_decode_workspace_bytes(lib):
    # per-split partial O (fp32, d per row) and (m, l) for every row group of
    # 4, 8 or 16 query rows; grows with the key count until the split count caps
    ws = binding.fa_decode_workspace_bytes
    assert ws(8, 32, 8, 1, 32768, 128) > 0
    assert ws(8, 32, 8, 1, 64, 128) <= ws(8, 32, 8, 1, 4096, 128)
    assert ws(1, 4, 1, 1, 100, 64) % 256 == 0
    assert ws(1, 3, 2, 1, 100, 64) == 0       # Hq % Hkv != 0
    assert ws(1, 2, 2, 1, 100, 96) == 0       # unsupported d
    assert ws(1, 2, 2, 1, 0, 64) == 0         # queries with no key
    assert ws(0, 2, 2, 1, 100, 64) == 0       # empty problem needs nothing
    # more than 16 query rows per kv head: 128-row tiles, 128-key tiles, about
    # one CTA per SM in all (64 units of B8 x Hkv8 -> 2 splits of 128 tiles)
    assert ws(8, 32, 8, 32, 32768, 128) == 2 * 64 * 128 * 128 * 4 + 2 * 64 * 128 * 2 * 4
    # 512 rows -> 4 row tiles; Nk = 300 -> 3 key tiles, one split each at most
    assert ws(1, 4, 2, 256, 300, 128) == 3 * 8 * 128 * 128 * 4 + 3 * 8 * 128 * 2 * 4


def _dec(lib, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5, B=1, Hq=4, Hkv=2, Nq=1, Nk=300, d=128,
             causal=1, scale=0.088, ws=FAKE * 6, wsb=1 << 20)
    a.update(kw)
    return binding.fa_fwd_decode(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"],
                                 a["Nk"], a["d"], a["causal"], a["scale"], a["ws"], a["wsb"], 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA_ERR_INVALID_ARG),
    (dict(ws=0), binding.FA_ERR_INVALID_ARG),
    (dict(k=FAKE * 2 + 8), binding.FA_ERR_INVALID_ARG),          # misaligned
    (dict(ws=FAKE * 6 + 16), binding.FA_ERR_INVALID_ARG),        # workspace not 256-aligned
    (dict(wsb=100), binding.FA_ERR_INVALID_ARG),                 # workspace too small
    (dict(o=FAKE), binding.FA_ERR_INVALID_ARG),                  # output aliases q
    (dict(Hq=3), binding.FA_ERR_INVALID_ARG),                    # Hq % Hkv
    (dict(Nk=0), binding.FA_ERR_INVALID_ARG),                    # queries with no key
    (dict(Nq=301), binding.FA_ERR_INVALID_ARG),                  # causal queries before the first key
    (dict(Nq=300, causal=0), binding.FA_ERR_UNSUPPORTED),        # long query blocks belong to fa_fwd
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(scale=-1.0), binding.FA_ERR_INVALID_ARG),
    (dict(B=0), binding.FA_OK),                                  # empty problem: nothing to do
    (dict(Nq=0), binding.FA_OK),
])
def test_decode_argument_validation(lib, kw, expect):
    assert _dec(lib, **kw) == expect


def test_noalloc_scratch_size_matches_header():
    # the binding's copy of FA_NOALLOC_SCRATCH_BYTES must equal the C #define
    src = open(HEADER).read()
    m = re.search(r"#define\s+FA_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", src)
    assert m, "FA_NOALLOC_SCRATCH_BYTES not found in fa.h"
    value = eval(m.group(1).replace("u", ""), {})  # e.g. "64u * 1024u * 1024u"
    assert value == binding.FA_NOALLOC_SCRATCH_BYTES


def _bwd_noalloc(lib, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5, do=FAKE * 6, dq=FAKE * 7, dk=FAKE * 8,
             dv=FAKE * 9, B=1, Hq=2, Hkv=2, N=128, d=64, causal=0, scale=0.125)
    a.update(kw)
    return binding.fa_bwd_noalloc(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"], a["dv"],
                                  a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["causal"], a["scale"], 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA_ERR_INVALID_ARG),                     # checked before the scratch lookup
    (dict(dv=0), binding.FA_ERR_INVALID_ARG),
    (dict(lse=FAKE * 5 + 4), binding.FA_ERR_INVALID_ARG),        # misaligned
    (dict(Hq=3), binding.FA_ERR_INVALID_ARG),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(B=8, Hq=16, Hkv=16, N=2048, d=128), binding.FA_ERR_UNSUPPORTED),  # beyond the 64 MiB scratch
    (dict(B=0), binding.FA_OK),
])
def test_noalloc_argument_validation(lib, kw, expect):
    assert _bwd_noalloc(lib, **kw) == expect


def test_varlen_workspace_bytes(lib):
    # header + work table (one int2 per 128-row tile, T/128 + nseq bound); the
    # backward adds D and lse2 rows, the fp32 dQ accumulator over padded rows
    # Tp = ceil64(T + 256·nseq) per head, and the unit counter
    r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    nseq, Hq, Hkv, T, d = 3, 4, 2, 1000, 128
    table = r256(8 * ((T + 127) // 128 + nseq))
    assert binding.fa_fwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, 600, d) == 256 + table
    Tp = (T + 256 * nseq + 63) // 64 * 64
    rows_p = Hq * Tp
    assert binding.fa_bwd_varlen_workspace_bytes(nseq, Hq, Hkv, T, 600, d) == \
        256 + table + 2 * r256(rows_p * 4) + r256(rows_p * d * 4) + 256
    assert binding.fa_fwd_varlen_workspace_bytes(3, 3, 2, 1000, 600, 128) == 0      # Hq % Hkv
    assert binding.fa_fwd_varlen_workspace_bytes(3, 4, 2, 1000, 600, 96) == 0       # unsupported d
    assert binding.fa_bwd_varlen_workspace_bytes(3, 4, 2, 1000, 0, 128) == 0        # max_seqlen < 1
    assert binding.fa_bwd_varlen_workspace_bytes(3, 4, 2, 1000, (1 << 20) + 1, 128) == 0
    assert binding.fa_fwd_varlen_workspace_bytes(0, 4, 2, 0, 1, 128) == 256         # empty problem


def _fwd_varlen(lib, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5, cu=FAKE * 6, nseq=3, Hq=4, Hkv=2, T=1000,
             max_seqlen=600, d=128, causal=1, scale=0.088, ws=FAKE * 7, wsb=1 << 20)
    a.update(kw)
    return binding.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"], a["nseq"], a["Hq"], a["Hkv"],
                                 a["T"], a["max_seqlen"], a["d"], a["causal"], a["scale"], a["ws"], a["wsb"], 0)


def _bwd_varlen(lib, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5, do=FAKE * 6, dq=FAKE * 7, dk=FAKE * 8,
             dv=FAKE * 9, cu=FAKE * 10, nseq=3, Hq=4, Hkv=2, T=1000, max_seqlen=600, d=128, causal=0, scale=0.088,
             ws=FAKE * 11, wsb=1 << 24)
    a.update(kw)
    return binding.fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"], a["dv"],
                                 a["cu"], a["nseq"], a["Hq"], a["Hkv"], a["T"], a["max_seqlen"], a["d"],
                                 a["causal"], a["scale"], a["ws"], a["wsb"], 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), binding.FA_ERR_INVALID_ARG),
    (dict(cu=0), binding.FA_ERR_INVALID_ARG),
    (dict(cu=FAKE * 6 + 2), binding.FA_ERR_INVALID_ARG),         # cu_seqlens not 4-byte aligned
    (dict(o=FAKE * 4 + 8), binding.FA_ERR_INVALID_ARG),          # misaligned
    (dict(ws=FAKE * 7 + 16), binding.FA_ERR_INVALID_ARG),        # workspace not 256-aligned
    (dict(wsb=100), binding.FA_ERR_INVALID_ARG),                 # workspace too small
    (dict(o=FAKE), binding.FA_ERR_INVALID_ARG),                  # output aliases q
    (dict(ws=FAKE * 6), binding.FA_ERR_INVALID_ARG),             # workspace aliases cu_seqlens
    (dict(Hq=3), binding.FA_ERR_INVALID_ARG),                    # Hq % Hkv
    (dict(nseq=-1), binding.FA_ERR_INVALID_ARG),
    (dict(max_seqlen=0), binding.FA_ERR_INVALID_ARG),
    (dict(max_seqlen=(1 << 20) + 1), binding.FA_ERR_UNSUPPORTED),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), binding.FA_ERR_INVALID_ARG),
    (dict(T=0), binding.FA_OK),                                  # empty problem: nothing to do
    (dict(nseq=0, T=0), binding.FA_OK),
])
def test_fwd_varlen_argument_validation(lib, kw, expect):
    assert _fwd_varlen(lib, **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(do=0), binding.FA_ERR_INVALID_ARG),
    (dict(cu=0), binding.FA_ERR_INVALID_ARG),
    (dict(wsb=1000), binding.FA_ERR_INVALID_ARG),                # workspace too small
    (dict(dk=FAKE * 7), binding.FA_ERR_INVALID_ARG),             # dk aliases dq
    (dict(dq=FAKE * 10), binding.FA_ERR_INVALID_ARG),            # dq overlaps cu_seqlens
    (dict(Hq=1), binding.FA_ERR_INVALID_ARG),                    # Hq % Hkv
    (dict(d=32), binding.FA_ERR_UNSUPPORTED),
    (dict(Hq=4096, Hkv=2, T=1 << 19, nseq=1), binding.FA_ERR_UNSUPPORTED),  # padded rows reach 2^31
    (dict(T=0, nseq=0), binding.FA_OK),
])
def test_bwd_varlen_argument_validation(lib, kw, expect):
    assert _bwd_varlen(lib, **kw) == expect


def test_pair_forward_argument_validation(lib):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, o=FAKE * 4, lse=FAKE * 5, B=1, Hq=2, Hkv=2, N=256, d=128, causal=0,
             scale=0.088)
    call = lambda **kw: binding.fa_fwd_pair(*[{**a, **kw}[n] for n in ("q", "k", "v", "o", "lse", "B", "Hq", "Hkv",  # noqa: E731
                                                                       "N", "d", "causal", "scale")], 0)
    assert call(d=64) == binding.FA_ERR_UNSUPPORTED
    assert call(d=256) == binding.FA_ERR_UNSUPPORTED
    assert call(q=0) == binding.FA_ERR_INVALID_ARG
    assert call(o=FAKE) == binding.FA_ERR_INVALID_ARG       # output aliases q
    assert call(Hq=3) == binding.FA_ERR_INVALID_ARG
    assert call(N=0) == binding.FA_OK
