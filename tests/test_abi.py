"""Host-side checks of the C ABI (no GPU): the library loads, exports every
entry point declared in include/hysparse.h, sizes workspaces, and rejects bad
arguments with the documented status before launching anything.  Pointers
here are fake device addresses: argument checking never dereferences them."""
import ctypes
import os
import re

import pytest

from hybrid_sparse_attention_tcgen05_b200 import _lib, build as hs_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hysparse.h")


@pytest.fixture(scope="module")
def L():
    hs_build.build()
    return _lib.lib()


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(hysparse_\w+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), f"{n} declared in hysparse.h but not exported"
    assert set(names) == set(_lib.EXPORTS)


def test_version_and_status_strings(L):
    assert L.hysparse_version().decode().startswith("hysparse-b200")
    seen = set()
    for code in range(7):
        s = L.hysparse_status_string(code).decode()
        assert s and s not in seen
        seen.add(s)
    assert L.hysparse_status_string(99).decode() == "unknown status"


def shape(B=1, Lq=64, Lkv=64, Hq=4, Hkv=1, d=64, dtype=_lib.HS_F32, scale=0.0):
    return _lib.HsShape(B, Lq, Lkv, Hq, Hkv, d, dtype, scale)


def ws_size(L, s, topk=8, window=16, n_sparse=1, row_chunk=0):
    return L.hysparse_workspace_size(ctypes.byref(s), topk, window, n_sparse, row_chunk)


def test_workspace_size(L):
    s = shape()
    n = ws_size(L, s)
    assert n >= 256 and n % 256 == 0
    # block scores chunk grows with the chunk
    assert ws_size(L, s, row_chunk=8) < ws_size(L, s, row_chunk=32) <= ws_size(L, s, row_chunk=0)
    for bad in (shape(Hq=3, Hkv=2), shape(Lq=65), shape(d=96), shape(dtype=7), shape(B=0),
                shape(dtype=_lib.HS_BF16, d=64), shape(Hq=64, Hkv=1)):
        assert ws_size(L, bad) == 0
    assert ws_size(L, s, topk=0) == 0
    assert ws_size(L, s, topk=4097) == 0
    assert ws_size(L, s, window=0) == 0


A = 0x7f0000000000        # fake, 16-byte aligned "device" addresses
P = lambda i: ctypes.c_void_p(A + 0x100000 * i)


def full(L, s, q=1, k=2, v=3, out=4, lse=5, scores=6, ld=None, rb=0, rc=None, ws=7, wsb=None):
    ld = s.Lkv if ld is None else ld
    rc = s.Lq if rc is None else rc
    wsb = ws_size(L, s) if wsb is None else wsb
    pp = lambda i: None if i is None else (ctypes.c_void_p(A + 0x100000 * i + 1) if i < 0 else P(i))
    return L.hysparse_full_attn_scores(ctypes.byref(s), pp(q), pp(k), pp(v), pp(out), pp(lse),
                                       pp(scores), ld, rb, rc, pp(ws), wsb, None)


def test_full_attn_scores_rejects(L):
    s = shape()
    assert full(L, s, q=None) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, k=-2) == _lib.HS_ERR_INVALID_ARG           # misaligned
    assert full(L, s, lse=None) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, ld=63) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, rb=60, rc=5) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, rb=-1, rc=5) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, rc=0) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, ws=None) == _lib.HS_ERR_INVALID_ARG
    assert full(L, s, wsb=16) == _lib.HS_ERR_WORKSPACE
    assert full(L, shape(d=96)) == _lib.HS_ERR_UNSUPPORTED
    assert full(L, shape(Hq=3, Hkv=2)) == _lib.HS_ERR_INVALID_ARG
    assert full(L, shape(Lq=65)) == _lib.HS_ERR_INVALID_ARG
    assert full(L, shape(scale=float("nan"))) == _lib.HS_ERR_INVALID_ARG
    assert L.hysparse_full_attn_scores(None, P(1), P(2), P(3), P(4), P(5), None, 0, 0, 1, P(7),
                                       1 << 20, None) == _lib.HS_ERR_INVALID_ARG


def test_topk_rejects(L):
    s = shape()
    f = lambda **kw: L.hysparse_topk(ctypes.byref(kw.get("s", s)), kw.get("sc", P(1)),
                                     kw.get("ld", 64), kw.get("rb", 0), kw.get("rc", 64),
                                     kw.get("k", 8), kw.get("idx", P(2)), None)
    assert f(sc=None) == _lib.HS_ERR_INVALID_ARG
    assert f(idx=ctypes.c_void_p(A + 4)) == _lib.HS_ERR_INVALID_ARG
    assert f(ld=10) == _lib.HS_ERR_INVALID_ARG
    assert f(k=0) == _lib.HS_ERR_INVALID_ARG
    assert f(k=4097) == _lib.HS_ERR_INVALID_ARG
    assert f(rb=1) == _lib.HS_ERR_INVALID_ARG


def test_sparse_attn_rejects(L):
    s = shape()
    wsb = ws_size(L, s)

    def f(**kw):
        return L.hysparse_sparse_attn(ctypes.byref(kw.get("s", s)), kw.get("q", P(1)), P(2), P(3),
                                      kw.get("idx", P(4)), kw.get("k", 8), kw.get("gate", P(5)),
                                      kw.get("w", 16), kw.get("out", P(6)), kw.get("og", None),
                                      None, kw.get("ws", P(7)), kw.get("wsb", wsb), None)
    assert f(q=None) == _lib.HS_ERR_INVALID_ARG
    assert f(idx=None) == _lib.HS_ERR_INVALID_ARG
    assert f(gate=None) == _lib.HS_ERR_INVALID_ARG
    assert f(out=None) == _lib.HS_ERR_INVALID_ARG
    assert f(og=ctypes.c_void_p(A + 8)) == _lib.HS_ERR_INVALID_ARG
    assert f(k=0) == _lib.HS_ERR_INVALID_ARG
    assert f(w=0) == _lib.HS_ERR_INVALID_ARG
    assert f(w=1025) == _lib.HS_ERR_INVALID_ARG
    assert f(ws=None) == _lib.HS_ERR_INVALID_ARG
    assert f(wsb=0) == _lib.HS_ERR_WORKSPACE
    assert f(s=shape(dtype=_lib.HS_BF16, d=64)) == _lib.HS_ERR_UNSUPPORTED


def test_sparse_attn_own_window_rejects(L):
    """The own window buffer must be aligned, hold 1 .. Lkv rows and reach
    back to the first key of the first query row's window."""
    def f(s=None, kw=P(8), vw=P(9), lwin=None, w=16, q=P(1), wsb=None):
        s = s or shape()
        lwin = s.Lkv if lwin is None else lwin
        wsb = ws_size(L, s) if wsb is None else wsb
        return L.hysparse_sparse_attn_own_window(ctypes.byref(s), q, P(2), P(3), kw, vw, lwin, P(4), 8, P(5), w,
                                                 P(6), None, None, P(7), wsb, None)
    assert f(kw=None) == _lib.HS_ERR_INVALID_ARG
    assert f(vw=None) == _lib.HS_ERR_INVALID_ARG
    assert f(vw=ctypes.c_void_p(A + 8)) == _lib.HS_ERR_INVALID_ARG
    assert f(lwin=0) == _lib.HS_ERR_INVALID_ARG
    assert f(lwin=65) == _lib.HS_ERR_INVALID_ARG
    assert f(lwin=63) == _lib.HS_ERR_INVALID_ARG           # prefill: row 0 sees key 0
    dec = shape(Lq=1, Lkv=64)
    assert f(s=dec, lwin=15) == _lib.HS_ERR_INVALID_ARG    # row 0 (position 63) sees keys 48 .. 63
    assert f(s=dec, lwin=15, w=15, q=None) == _lib.HS_ERR_INVALID_ARG
    assert f(w=0) == _lib.HS_ERR_INVALID_ARG
    assert f(q=None) == _lib.HS_ERR_INVALID_ARG
    assert f(wsb=0) == _lib.HS_ERR_WORKSPACE
    assert f(s=dec, lwin=16, wsb=0) == _lib.HS_ERR_WORKSPACE   # long enough: checks go on to the workspace


def test_block_rejects(L):
    s = shape()
    wsb = ws_size(L, s, n_sparse=2)
    PA = ctypes.c_void_p * 2
    qa, ga, oa = PA(A, A + 256), PA(A + 512, A + 768), PA(A + 1024, A + 1280)
    c = lambda x: ctypes.cast(x, ctypes.c_void_p)

    def f(**kw):
        return L.hysparse_block(ctypes.byref(s), P(1), P(2), P(3), P(4), None, kw.get("n", 2),
                                kw.get("qa", c(qa)), c(ga), c(oa), kw.get("k", 8), 16, None,
                                kw.get("chunk", 0), P(7), kw.get("wsb", wsb), None)
    assert f(qa=None) == _lib.HS_ERR_INVALID_ARG
    assert f(n=-1) == _lib.HS_ERR_INVALID_ARG
    assert f(k=0) == _lib.HS_ERR_INVALID_ARG
    assert f(wsb=wsb - 1) == _lib.HS_ERR_WORKSPACE
    bad = PA(A, A + 3)
    assert f(qa=c(bad)) == _lib.HS_ERR_INVALID_ARG
    # a smaller chunk needs less workspace
    assert f(chunk=8, wsb=ws_size(L, s, n_sparse=2, row_chunk=8) - 1) == _lib.HS_ERR_WORKSPACE


def test_block_own_window_rejects(L):
    """hysparse_block_own_window: every layer's window buffer present, aligned
    and reaching back to the first row's window, before anything runs."""
    s = shape()            # Lq = Lkv = 64: lwin must be 64
    wsb = ws_size(L, s, n_sparse=2)
    PA = ctypes.c_void_p * 2
    qa, ga, oa = PA(A, A + 256), PA(A + 512, A + 768), PA(A + 1024, A + 1280)
    kw, vw = PA(A + 2048, A + 4096), PA(A + 6144, A + 8192)
    c = lambda x: ctypes.cast(x, ctypes.c_void_p)

    def f(**a):
        return L.hysparse_block_own_window(ctypes.byref(s), P(1), P(2), P(3), P(4), None, 2, c(qa), c(ga),
                                           a.get("kw", c(kw)), a.get("vw", c(vw)), a.get("lwin", 64), c(oa), 8,
                                           16, None, 0, P(7), a.get("wsb", wsb), None)
    assert f(kw=None) == _lib.HS_ERR_INVALID_ARG
    assert f(vw=None) == _lib.HS_ERR_INVALID_ARG
    assert f(lwin=63) == _lib.HS_ERR_INVALID_ARG      # row 0 sees key 0
    assert f(lwin=65) == _lib.HS_ERR_INVALID_ARG
    assert f(lwin=0) == _lib.HS_ERR_INVALID_ARG
    assert f(kw=c(PA(A + 2048, A + 4100))) == _lib.HS_ERR_INVALID_ARG   # layer 1 misaligned
    assert f(wsb=wsb - 1) == _lib.HS_ERR_WORKSPACE      # valid window buffers: on to the workspace check


def test_block_varlen_rejects(L):
    """hysparse_block_varlen: decode shapes on the bf16 path only, a 4-byte
    aligned length array, and the workspace of the fixed-length block."""
    dec = shape(B=2, Lq=1, Lkv=300, Hq=8, Hkv=2, d=128, dtype=_lib.HS_BF16)
    wsb = ws_size(L, dec, n_sparse=2)
    PA = ctypes.c_void_p * 2
    qa, ga, oa = PA(A, A + 256), PA(A + 512, A + 768), PA(A + 1024, A + 1280)
    c = lambda x: ctypes.cast(x, ctypes.c_void_p)

    def f(**kw):
        s = kw.get("s", dec)
        return L.hysparse_block_varlen(ctypes.byref(s), kw.get("kvl", P(8)), P(1), P(2), P(3), P(4), None, 2,
                                       c(qa), c(ga), c(oa), kw.get("k", 8), 16, None, P(7),
                                       kw.get("wsb", wsb), None)
    assert f(kvl=None) == _lib.HS_ERR_INVALID_ARG
    assert f(kvl=ctypes.c_void_p(A + 0x100000 * 8 + 2)) == _lib.HS_ERR_INVALID_ARG     # misaligned
    assert f(s=shape(B=2, Lq=64, Lkv=300, Hq=8, Hkv=2, d=128, dtype=_lib.HS_BF16)) == _lib.HS_ERR_UNSUPPORTED
    assert f(s=shape(B=2, Lq=1, Lkv=300, Hq=8, Hkv=2, d=64)) == _lib.HS_ERR_UNSUPPORTED   # fp32 path
    assert f(k=0) == _lib.HS_ERR_INVALID_ARG
    assert f(wsb=wsb - 1) == _lib.HS_ERR_WORKSPACE


def test_block_paged_rejects(L):
    """hysparse_block_paged: a power-of-two page size, a table long enough for
    Lkv, a pool whose rows fit in int32, aligned lengths and table."""
    dec = shape(B=2, Lq=1, Lkv=300, Hq=8, Hkv=2, d=128, dtype=_lib.HS_BF16)
    wsb = ws_size(L, dec, n_sparse=2)
    PA = ctypes.c_void_p * 2
    qa, ga, oa = PA(A, A + 256), PA(A + 512, A + 768), PA(A + 1024, A + 1280)
    c = lambda x: ctypes.cast(x, ctypes.c_void_p)

    def f(**kw):
        s = kw.get("s", dec)
        return L.hysparse_block_paged(ctypes.byref(s), kw.get("kvl", P(8)), kw.get("tab", P(9)),
                                      kw.get("ps", 64), kw.get("mp", 5), kw.get("np", 100), P(1), P(2), P(3),
                                      P(4), None, 2, c(qa), c(ga), c(oa), 8, 16, None, P(7), wsb, None)
    assert f(tab=None) == _lib.HS_ERR_INVALID_ARG
    assert f(kvl=None) == _lib.HS_ERR_INVALID_ARG
    assert f(ps=48) == _lib.HS_ERR_INVALID_ARG                       # not a power of two
    assert f(ps=0) == _lib.HS_ERR_INVALID_ARG
    assert f(mp=4) == _lib.HS_ERR_INVALID_ARG                        # 4 * 64 < Lkv = 300
    assert f(np=0) == _lib.HS_ERR_INVALID_ARG
    assert f(ps=1 << 16, np=1 << 16) == _lib.HS_ERR_INVALID_ARG      # pool rows past int32
    assert f(tab=ctypes.c_void_p(A + 0x100000 * 9 + 2)) == _lib.HS_ERR_INVALID_ARG
    assert f(s=shape(B=2, Lq=64, Lkv=300, Hq=8, Hkv=2, d=128, dtype=_lib.HS_BF16)) == _lib.HS_ERR_UNSUPPORTED


def test_workspace_status_rejects_null(L):
    assert L.hysparse_workspace_status(None, None) == _lib.HS_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(L):
    import torch
    import hybrid_sparse_attention_tcgen05_b200 as hs
    q = torch.zeros(1, 4, 4, 64)
    with pytest.raises(ValueError):
        hs.full_attn_scores(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous())


NOALLOC_BYTES = 16 << 20


def noalloc_scratch_bytes(B, Lq, Lkv, Hq, decode):
    """Scratch of hysparse_full_attn_scores_noalloc as hysparse.h states it:
    256 + 8*B*Hq*Lq rounded up to 256, plus for decode-shaped calls
    4*B*Hq*Lkv + 520*B*Hq*ceil(Lkv/1024) + 768 rounded up to 256."""
    up = lambda x: (x + 255) // 256 * 256
    n = up(256 + 8 * B * Hq * Lq)
    if decode:
        n += up(4 * B * Hq * Lkv + 520 * B * Hq * ((Lkv + 1023) // 1024) + 768)
    return n


_NOALLOC_CHILD = r"""
import ctypes, sys
sys.path.insert(0, {root!r})
from hybrid_sparse_attention_tcgen05_b200 import _lib
L = _lib.lib()
A = 0x7f0000000000
P = lambda i: ctypes.c_void_p(A + (i << 32))
for B, Lq, Lkv, Hq, Hkv in {cases!r}:
    s = _lib.HsShape(B, Lq, Lkv, Hq, Hkv, 128, _lib.HS_BF16, 0.0)
    print(L.hysparse_full_attn_scores_noalloc(ctypes.byref(s), P(1), P(2), P(3), P(4), P(5), None, 0, 0, Lq,
                                              None))
"""


def test_noalloc_refuses_scratch_beyond_its_array():
    """The size check of the allocation-free entry point comes before any
    CUDA call.  Run in a child process that sees no GPU, so that a shape the
    check lets through stops at the first CUDA call (HS_ERR_CUDA) instead of
    launching anything on fake addresses.  Shapes on both sides of the 16 MiB
    array, prefill- and decode-shaped, follow the bound hysparse.h states."""
    import subprocess
    import sys
    cases = [(1, 65536, 65536, 64, 4),        # 8 B of statistics per (head, row): 32 MiB
             (1, 32000, 32000, 64, 4),        # 16.0 MB: fits
             (1, 32800, 32800, 64, 4),        # just over
             (64, 1, 32768, 32, 8),           # the 64 x 32k decode step: its logit stash alone is 256 MiB
             (2, 1, 1000, 8, 2),              # small decode: fits
             (4, 1, 28000, 32, 8),            # decode just under the array
             (4, 1, 30000, 32, 8)]            # and just over
    expect = []
    for B, Lq, Lkv, Hq, Hkv in cases:
        n = noalloc_scratch_bytes(B, Lq, Lkv, Hq, Lq == 1)
        expect.append(_lib.HS_ERR_WORKSPACE if n > NOALLOC_BYTES else _lib.HS_ERR_CUDA)
    assert _lib.HS_ERR_WORKSPACE in expect and _lib.HS_ERR_CUDA in expect
    hs_build.build()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", _NOALLOC_CHILD.format(root=ROOT, cases=cases)],
                         capture_output=True, text=True, env=env, timeout=120)
    assert res.returncode == 0, res.stderr
    got = [int(x) for x in res.stdout.split()]
    assert got == expect
