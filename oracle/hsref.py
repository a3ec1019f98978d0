"""ctypes front end of the fp64 C oracle in ``hsref.c``.

TEST INFRASTRUCTURE ONLY (tests, smoke check, the benchmark's CPU-baseline
leg).  Arguments are host tensors; the wrappers widen inputs to contiguous fp32
(exact for bf16 inputs) and return fp64 / int32 host tensors.  Every function
names the definition it follows in ``hsref.c``'s header.

Row lists: a "row" is a (batch b, query index i) pair, i in [0, Lq); its
causal position is pos = Lkv - Lq + i.  ``q_rows`` holds those rows' queries,
shape [nrows, Hq, d].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hsref.c")
_LIB = os.path.join(_HERE, "libhsref.so")
_lock = threading.Lock()
_libs = {}


def library_path() -> str:
    return _LIB


def build(force: bool = False, src: str = _SRC, lib: str = _LIB) -> str:
    """Compile ``src`` (default hsref.c) with gcc (-O2, OpenMP, IEEE
    arithmetic) into ``lib`` if it is missing or older than the source."""
    with _lock:
        if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
            tmp = lib + f".tmp{os.getpid()}"
            subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
                            "-o", tmp, src, "-lm"], check=True)
            os.replace(tmp, lib)
    return lib


_active = [None]


def use_library(path: Optional[str]) -> None:
    """Point the wrappers at another build of the oracle (None: the default).

    Used by the tests that plant a mistake in a copy of hsref.c and check that
    the pins catch it."""
    _active[0] = path


def _load():
    path = _active[0] or _LIB
    lib = _libs.get(path)
    if lib is None:
        if path == _LIB:
            build()
        lib = ctypes.CDLL(path)
        I, D, P, LL = ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_longlong
        lib.hsref_full_rows.argtypes = [I, I, I, I, I, I, D, P, P, P, P, P, I, P, P, P]
        lib.hsref_topk_rows.argtypes = [P, LL, P, I, I, P]
        lib.hsref_sparse_rows.argtypes = [I, I, I, I, I, I, D, P, P, P, P, P, I, P, I, P, I,
                                          P, P, P]
        lib.hsref_sparse_rows_own_window.argtypes = [I, I, I, I, I, I, D, P, P, P, P, P, I, P, P, I, P, I,
                                                     P, I, P, P, P]
        lib.hsref_block_rows.argtypes = [I, I, I, I, I, I, D, P, P, P, P, P, I, I, P, P, I, I,
                                         P, P, P]
        for f in ("hsref_full_rows", "hsref_topk_rows", "hsref_sparse_rows", "hsref_sparse_rows_own_window",
                  "hsref_block_rows", "hsref_max_threads"):
            getattr(lib, f).restype = I
        lib.hsref_set_threads.argtypes = [I]
        lib.hsref_set_threads.restype = None
        _libs[path] = lib
    return lib


def max_threads() -> int:
    return _load().hsref_max_threads()


def set_threads(n: int) -> None:
    _load().hsref_set_threads(int(n))


def _f32(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu", torch.float32).contiguous()


def _i32(x) -> torch.Tensor:
    return torch.as_tensor(x, dtype=torch.int32).contiguous()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(rc: int, what: str) -> None:
    if rc != 0:
        msg = {-1: "bad argument", -2: "malformed index list", -3: "out of memory"}.get(rc, "?")
        raise ValueError(f"{what}: oracle returned {rc} ({msg})")


def _rows(rows, B: int) -> Tuple[torch.Tensor, torch.Tensor]:
    rows = list(rows)
    rb = _i32([r[0] for r in rows])
    ri = _i32([r[1] for r in rows])
    return rb, ri


def full_rows(q_rows: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rows: Sequence[Tuple[int, int]],
              Lq: int, scale: float, want_scores: bool = True):
    """Full causal GQA attention + importance scores for the listed rows.

    q_rows [nrows,Hq,d]; k, v [B,Lkv,Hkv,d].  Returns (out [nrows,Hq,d] f64,
    lse [nrows,Hq] f64, scores [nrows,Hkv,Lkv] f64 or None).
    """
    B, Lkv, Hkv, d = k.shape
    nrows, Hq, _ = q_rows.shape
    qf, kf, vf = _f32(q_rows), _f32(k), _f32(v)
    rb, ri = _rows(rows, B)
    out = torch.empty(nrows, Hq, d, dtype=torch.float64)
    lse = torch.empty(nrows, Hq, dtype=torch.float64)
    sc = torch.empty(nrows, Hkv, Lkv, dtype=torch.float64) if want_scores else None
    rc = _load().hsref_full_rows(B, Lq, Lkv, Hq, Hkv, d, float(scale), _ptr(qf), _ptr(kf), _ptr(vf),
                                 _ptr(rb), _ptr(ri), nrows, _ptr(out), _ptr(lse), _ptr(sc))
    _check(rc, "hsref_full_rows")
    return out, lse, sc


def topk_rows(scores: torch.Tensor, n_valid, topk: int) -> torch.Tensor:
    """Top-k over score rows [..., ld]: row r uses its first n_valid[r] entries.

    Returns int32 [..., topk], ascending keys, -1 padded.  Any float dtype is
    widened exactly to fp64 before ranking.
    """
    shape = scores.shape
    ld = shape[-1]
    s2 = scores.detach().to("cpu", torch.float64).reshape(-1, ld).contiguous()
    nv = _i32(n_valid).reshape(-1)
    if nv.numel() != s2.shape[0]:
        raise ValueError("n_valid must give one count per score row")
    idx = torch.empty(s2.shape[0], topk, dtype=torch.int32)
    rc = _load().hsref_topk_rows(_ptr(s2), ld, _ptr(nv), s2.shape[0], int(topk), _ptr(idx))
    _check(rc, "hsref_topk_rows")
    return idx.reshape(*shape[:-1], topk)


def sparse_rows(q_rows: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rows, Lq: int, scale: float,
                idx_rows: torch.Tensor, gate_rows: torch.Tensor, window: int,
                k_win: Optional[torch.Tensor] = None, v_win: Optional[torch.Tensor] = None):
    """One sparse layer for the listed rows.

    idx_rows [nrows,Hkv,topk] int32; gate_rows [nrows,Hq] fp32 logits.
    k_win, v_win (optional, [B,Lwin,Hkv,d]): the layer's own window keys and
    values for the last Lwin positions (row r = position Lkv - Lwin + r); the
    window branch reads them instead of the shared cache.
    Returns (out, out_global, out_local), each [nrows,Hq,d] f64.
    """
    B, Lkv, Hkv, d = k.shape
    nrows, Hq, _ = q_rows.shape
    qf, kf, vf = _f32(q_rows), _f32(k), _f32(v)
    ix = idx_rows.detach().to("cpu", torch.int32).contiguous()
    gt = _f32(gate_rows)
    topk = ix.shape[-1]
    rb, ri = _rows(rows, B)
    out = torch.empty(nrows, Hq, d, dtype=torch.float64)
    og = torch.empty_like(out)
    ol = torch.empty_like(out)
    if k_win is not None:
        kwf, vwf = _f32(k_win), _f32(v_win)
        rc = _load().hsref_sparse_rows_own_window(B, Lq, Lkv, Hq, Hkv, d, float(scale), _ptr(qf), _ptr(kf),
                                                  _ptr(vf), _ptr(kwf), _ptr(vwf), int(kwf.shape[1]), _ptr(rb),
                                                  _ptr(ri), nrows, _ptr(ix), int(topk), _ptr(gt), int(window),
                                                  _ptr(out), _ptr(og), _ptr(ol))
        _check(rc, "hsref_sparse_rows_own_window")
        return out, og, ol
    rc = _load().hsref_sparse_rows(B, Lq, Lkv, Hq, Hkv, d, float(scale), _ptr(qf), _ptr(kf), _ptr(vf),
                                   _ptr(rb), _ptr(ri), nrows, _ptr(ix), int(topk), _ptr(gt),
                                   int(window), _ptr(out), _ptr(og), _ptr(ol))
    _check(rc, "hsref_sparse_rows")
    return out, og, ol


def block_rows(q_rows, k, v, rows, Lq: int, scale: float, q_sparse_rows, gate_rows, topk: int,
               window: int):
    """A whole hybrid block for the listed rows.

    q_sparse_rows [n_sparse,nrows,Hq,d]; gate_rows [n_sparse,nrows,Hq].
    Returns (out_full [nrows,Hq,d] f64, idx [nrows,Hkv,topk] int32,
    out_sparse [n_sparse,nrows,Hq,d] f64).
    """
    B, Lkv, Hkv, d = k.shape
    nrows, Hq, _ = q_rows.shape
    n_sparse = q_sparse_rows.shape[0]
    qf, kf, vf = _f32(q_rows), _f32(k), _f32(v)
    qs, gt = _f32(q_sparse_rows), _f32(gate_rows)
    rb, ri = _rows(rows, B)
    out_full = torch.empty(nrows, Hq, d, dtype=torch.float64)
    idx = torch.empty(nrows, Hkv, topk, dtype=torch.int32)
    out_sp = torch.empty(n_sparse, nrows, Hq, d, dtype=torch.float64)
    rc = _load().hsref_block_rows(B, Lq, Lkv, Hq, Hkv, d, float(scale), _ptr(qf), _ptr(kf), _ptr(vf),
                                  _ptr(rb), _ptr(ri), nrows, n_sparse, _ptr(qs), _ptr(gt), int(topk),
                                  int(window), _ptr(out_full), _ptr(idx), _ptr(out_sp))
    _check(rc, "hsref_block_rows")
    return out_full, idx, out_sp
