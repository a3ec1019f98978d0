"""HySparse hybrid-block attention for B200 (sm_100a).

A thin Python binding over libhysparse.so (C ABI in include/hysparse.h).  The
functions below only marshal torch tensors into pointers, sizes and the
current CUDA stream; every step of the hot path runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback: calls raise when the library
is missing or a tensor is not on a CUDA device.

Calls (same names as the C ABI, without the ``hysparse_`` prefix):

* ``full_attn_scores`` -- the full causal GQA layer: O, LSE and the
  group-summed importance scores of a chunk of query rows.
* ``topk`` -- per-row top-k of those scores (ties to the lower key index),
  ascending keys, -1 padded.
* ``sparse_attn`` -- one sparse layer: global branch over the top-k keys,
  causal 128-token window branch, sigmoid gate; reuses the full layer's K/V.
* ``block`` -- one full layer + top-k + N sparse layers.
"""
from __future__ import annotations

import ctypes
import math
from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import HysparseError, HsShape

__all__ = ["shape_of", "workspace_size", "alloc_workspace", "full_attn_scores", "topk",
           "sparse_attn", "block", "block_paged", "workspace_status", "version", "launch_count",
           "kv_cache_bytes", "HysparseError", "HsShape"]


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return _lib.HS_F32
    if t == torch.bfloat16:
        return _lib.HS_BF16
    raise TypeError(f"unsupported dtype {t}; use float32 or bfloat16")


def shape_of(q: torch.Tensor, k: torch.Tensor, scale: Optional[float] = None) -> HsShape:
    """hs_shape from q [B,Lq,Hq,d] and k [B,Lkv,Hkv,d]."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be 4-D: [B, L, H, d]")
    B, Lq, Hq, d = q.shape
    Bk, Lkv, Hkv, dk = k.shape
    if B != Bk or d != dk:
        raise ValueError("q and k disagree on batch or head dim")
    return HsShape(B, Lq, Lkv, Hq, Hkv, d, _dtype_code(q.dtype), float(scale or 0.0))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts: Optional[torch.Tensor]) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("hysparse runs on CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("hysparse needs contiguous tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on the same device")
    return dev


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def workspace_size(shape: HsShape, topk: int, window: int, n_sparse: int = 0, row_chunk: int = 0) -> int:
    n = _lib.lib().hysparse_workspace_size(ctypes.byref(shape), int(topk), int(window),
                                          int(n_sparse), int(row_chunk))
    if n == 0:
        raise HysparseError(_lib.HS_ERR_INVALID_ARG, "hysparse_workspace_size")
    return int(n)


def alloc_workspace(shape: HsShape, topk: int, window: int, n_sparse: int = 0, row_chunk: int = 0,
                    device=None) -> torch.Tensor:
    """A zeroed uint8 device workspace of the size the library asks for."""
    n = workspace_size(shape, topk, window, n_sparse, row_chunk)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def full_attn_scores(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, want_scores: bool = True,
                     row_begin: int = 0, row_count: Optional[int] = None,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     scores: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     scale: Optional[float] = None):
    """Full layer for query rows [row_begin, row_begin+row_count).

    Returns (out [B,Lq,Hq,d], lse [B,Hq,Lq] f32, scores [B,Hkv,row_count,Lkv]
    f32 or None).  Only the listed rows of out/lse are written.
    """
    dev = _need_cuda(q, k, v, out, lse, scores, ws)
    s = shape_of(q, k, scale)
    rc_ = s.Lq - row_begin if row_count is None else row_count
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(s.B, s.Hq, s.Lq, dtype=torch.float32, device=dev)
    if want_scores and scores is None:
        scores = torch.empty(s.B, s.Hkv, rc_, s.Lkv, dtype=torch.float32, device=dev)
    if not want_scores:
        scores = None
    if ws is None:
        ws = alloc_workspace(s, 1, 1, 0, rc_, dev)
    ld = scores.shape[-1] if scores is not None else 0
    st = _lib.lib().hysparse_full_attn_scores(
        ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(scores), ld,
        int(row_begin), int(rc_), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "hysparse_full_attn_scores")
    return out, lse, scores


def topk(q_shape: HsShape, scores: torch.Tensor, k_top: int, *, row_begin: int = 0,
         idx: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Top-k of a score chunk [B,Hkv,row_count,ld] into idx [B,Hkv,Lq,k_top]
    (rows row_begin .. row_begin+row_count-1 are written)."""
    dev = _need_cuda(scores, idx)
    s = q_shape
    if idx is None:
        idx = torch.empty(s.B, s.Hkv, s.Lq, k_top, dtype=torch.int32, device=dev)
    row_count = scores.shape[2]
    st = _lib.lib().hysparse_topk(ctypes.byref(s), _ptr(scores), scores.shape[-1], int(row_begin),
                                  int(row_count), int(k_top), _ptr(idx), _stream(dev))
    _lib.check(st, "hysparse_topk")
    return idx


def sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                gate_logit: torch.Tensor, window: int, *, want_branches: bool = False,
                out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                scale: Optional[float] = None, k_win: Optional[torch.Tensor] = None,
                v_win: Optional[torch.Tensor] = None):
    """One sparse layer.  Returns out, or (out, out_global, out_local) when
    want_branches.

    k_win / v_win ([B, lwin, Hkv, d], the layer's own window keys and values
    for cache positions Lkv - lwin .. Lkv - 1): the local branch reads them
    instead of k / v (hysparse_sparse_attn_own_window)."""
    dev = _need_cuda(q, k, v, idx, gate_logit, out, ws, k_win, v_win)
    if (k_win is None) != (v_win is None):
        raise ValueError("k_win and v_win go together")
    if idx.dtype != torch.int32 or gate_logit.dtype != torch.float32:
        raise TypeError("idx must be int32 and gate_logit float32")
    s = shape_of(q, k, scale)
    k_top = idx.shape[-1]
    if out is None:
        out = torch.empty_like(q)
    og = torch.empty_like(q) if want_branches else None
    ol = torch.empty_like(q) if want_branches else None
    if ws is None:
        ws = alloc_workspace(s, k_top, window, 1, 1, dev)
    if k_win is not None:
        lwin = k_win.shape[1]
        want = (k.shape[0], lwin) + tuple(k.shape[2:])
        for t in (k_win, v_win):
            if tuple(t.shape) != want or t.dtype != k.dtype or not t.is_contiguous():
                raise TypeError("k_win and v_win must be contiguous [B, lwin, Hkv, d] of k's dtype")
        st = _lib.lib().hysparse_sparse_attn_own_window(
            ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(k_win), _ptr(v_win), int(lwin), _ptr(idx),
            int(k_top), _ptr(gate_logit), int(window), _ptr(out), _ptr(og), _ptr(ol), _ptr(ws), ws.numel(),
            _stream(dev))
        _lib.check(st, "hysparse_sparse_attn_own_window")
        return (out, og, ol) if want_branches else out
    st = _lib.lib().hysparse_sparse_attn(
        ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), int(k_top), _ptr(gate_logit),
        int(window), _ptr(out), _ptr(og), _ptr(ol), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "hysparse_sparse_attn")
    return (out, og, ol) if want_branches else out


def block(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_sparse: Sequence[torch.Tensor],
          gate_logit: Sequence[torch.Tensor], k_top: int, window: int, *, row_chunk: int = 0,
          out_full: Optional[torch.Tensor] = None, out_sparse: Optional[List[torch.Tensor]] = None,
          idx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
          ws: Optional[torch.Tensor] = None, scale: Optional[float] = None,
          kv_len: Optional[torch.Tensor] = None, k_win: Optional[Sequence[torch.Tensor]] = None,
          v_win: Optional[Sequence[torch.Tensor]] = None):
    """One hybrid block.  Returns (out_full, lse, idx, [out_sparse_n]).

    kv_len (int32 [B] on the device, decode only): sequence b's cache is the
    first kv_len[b] rows of k[b] and v[b], its new query at position
    kv_len[b] - 1 (hysparse_block_varlen).

    k_win, v_win (one [B, lwin, Hkv, d] tensor per sparse layer, the same
    lwin for all): the layers' own window K/V for cache positions
    Lkv - lwin .. Lkv - 1, read by their window branches
    (hysparse_block_own_window)."""
    dev = _need_cuda(q, k, v, out_full, idx, lse, ws, kv_len, *q_sparse, *gate_logit, *(out_sparse or []),
                     *(k_win or []), *(v_win or []))
    s = shape_of(q, k, scale)
    n = len(q_sparse)
    if len(gate_logit) != n:
        raise ValueError("one gate tensor per sparse layer")
    if out_full is None:
        out_full = torch.empty_like(q)
    if out_sparse is None:
        out_sparse = [torch.empty_like(x) for x in q_sparse]
    if idx is None:
        idx = torch.empty(s.B, s.Hkv, s.Lq, k_top, dtype=torch.int32, device=dev)
    if lse is None:
        lse = torch.empty(s.B, s.Hq, s.Lq, dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(s, k_top, window, n, row_chunk, dev)
    PA = ctypes.c_void_p * max(n, 1)
    qa = PA(*[x.data_ptr() for x in q_sparse])
    ga = PA(*[x.data_ptr() for x in gate_logit])
    oa = PA(*[x.data_ptr() for x in out_sparse])
    if kv_len is not None:
        if kv_len.dtype != torch.int32 or kv_len.shape != (s.B,) or not kv_len.is_contiguous():
            raise TypeError("kv_len must be a contiguous int32 tensor of shape [B]")
        st = _lib.lib().hysparse_block_varlen(
            ctypes.byref(s), _ptr(kv_len), _ptr(q), _ptr(k), _ptr(v), _ptr(out_full), _ptr(lse), n,
            ctypes.cast(qa, ctypes.c_void_p), ctypes.cast(ga, ctypes.c_void_p),
            ctypes.cast(oa, ctypes.c_void_p), int(k_top), int(window), _ptr(idx),
            _ptr(ws), ws.numel(), _stream(dev))
        _lib.check(st, "hysparse_block_varlen")
        return out_full, lse, idx, out_sparse
    if k_win is not None or v_win is not None:
        if k_win is None or v_win is None or len(k_win) != n or len(v_win) != n:
            raise ValueError("one k_win and one v_win tensor per sparse layer")
        lwin = k_win[0].shape[1] if n else 0
        want = (k.shape[0], lwin) + tuple(k.shape[2:])
        for t in (*k_win, *v_win):
            if tuple(t.shape) != want or t.dtype != k.dtype:
                raise TypeError("k_win and v_win must be [B, lwin, Hkv, d] of k's dtype, one lwin for all layers")
        ka = PA(*[x.data_ptr() for x in k_win])
        va = PA(*[x.data_ptr() for x in v_win])
        st = _lib.lib().hysparse_block_own_window(
            ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(out_full), _ptr(lse), n,
            ctypes.cast(qa, ctypes.c_void_p), ctypes.cast(ga, ctypes.c_void_p), ctypes.cast(ka, ctypes.c_void_p),
            ctypes.cast(va, ctypes.c_void_p), int(lwin), ctypes.cast(oa, ctypes.c_void_p), int(k_top),
            int(window), _ptr(idx), int(row_chunk), _ptr(ws), ws.numel(), _stream(dev))
        _lib.check(st, "hysparse_block_own_window")
        return out_full, lse, idx, out_sparse
    st = _lib.lib().hysparse_block(
        ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(out_full), _ptr(lse), n,
        ctypes.cast(qa, ctypes.c_void_p), ctypes.cast(ga, ctypes.c_void_p),
        ctypes.cast(oa, ctypes.c_void_p), int(k_top), int(window), _ptr(idx), int(row_chunk),
        _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "hysparse_block")
    return out_full, lse, idx, out_sparse


def block_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, q_sparse: Sequence[torch.Tensor],
                gate_logit: Sequence[torch.Tensor], k_top: int, window: int, kv_len: torch.Tensor,
                block_table: torch.Tensor, *, max_len: Optional[int] = None,
                out_full: Optional[torch.Tensor] = None, out_sparse: Optional[List[torch.Tensor]] = None,
                idx: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, scale: Optional[float] = None):
    """One decode step over paged caches (hysparse_block_paged).

    q [B,1,Hq,d]; k_pages, v_pages [num_pages,page_size,Hkv,d]; kv_len int32
    [B]; block_table int32 [B,max_pages] (sequence b's key j is row
    j % page_size of page block_table[b, j // page_size]).  max_len: the
    longest cache a sequence may have (default max_pages * page_size).
    Returns (out_full, lse, idx, [out_sparse_n])."""
    dev = _need_cuda(q, k_pages, v_pages, kv_len, block_table, out_full, idx, lse, ws, *q_sparse, *gate_logit,
                     *(out_sparse or []))
    if k_pages.dim() != 4 or v_pages.shape != k_pages.shape or block_table.dim() != 2:
        raise ValueError("k_pages, v_pages: [num_pages, page_size, Hkv, d]; block_table: [B, max_pages]")
    if kv_len.dtype != torch.int32 or block_table.dtype != torch.int32:
        raise TypeError("kv_len and block_table must be int32")
    num_pages, page_size, Hkv, d = k_pages.shape
    B, Lq, Hq, dq = q.shape
    if Lq != 1 or dq != d or kv_len.shape != (B,) or block_table.shape[0] != B:
        raise ValueError("q [B,1,Hq,d], kv_len [B] and block_table [B, max_pages] must agree")
    max_pages = block_table.shape[1]
    Lkv = max_pages * page_size if max_len is None else int(max_len)
    s = HsShape(B, 1, Lkv, Hq, Hkv, d, _dtype_code(q.dtype), float(scale or 0.0))
    n = len(q_sparse)
    if len(gate_logit) != n:
        raise ValueError("one gate tensor per sparse layer")
    if out_full is None:
        out_full = torch.empty_like(q)
    if out_sparse is None:
        out_sparse = [torch.empty_like(x) for x in q_sparse]
    if idx is None:
        idx = torch.empty(B, Hkv, 1, k_top, dtype=torch.int32, device=dev)
    if lse is None:
        lse = torch.empty(B, Hq, 1, dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(s, k_top, window, n, 0, dev)
    PA = ctypes.c_void_p * max(n, 1)
    qa = PA(*[x.data_ptr() for x in q_sparse])
    ga = PA(*[x.data_ptr() for x in gate_logit])
    oa = PA(*[x.data_ptr() for x in out_sparse])
    st = _lib.lib().hysparse_block_paged(
        ctypes.byref(s), _ptr(kv_len), _ptr(block_table), int(page_size), int(max_pages), int(num_pages),
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(out_full), _ptr(lse), n,
        ctypes.cast(qa, ctypes.c_void_p), ctypes.cast(ga, ctypes.c_void_p), ctypes.cast(oa, ctypes.c_void_p),
        int(k_top), int(window), _ptr(idx), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "hysparse_block_paged")
    return out_full, lse, idx, out_sparse


def workspace_status(ws: torch.Tensor) -> int:
    """Synchronise, read and clear the workspace status word (0 = ok)."""
    dev = _need_cuda(ws)
    return int(_lib.lib().hysparse_workspace_status(_ptr(ws), _stream(dev)))


def probe_l2_read(buf: torch.Tensor, passes: int, mode: int, blocks: int, sink: torch.Tensor) -> None:
    """Enqueue one L2 read-bandwidth probe over the device buffer `buf`
    (mode 0 streaming, 1 random 256-byte rows; passes * buf bytes read);
    `sink` holds at least `blocks` int64 words.  Time it with CUDA events."""
    dev = _need_cuda(buf, sink)
    nbytes = buf.numel() * buf.element_size()
    st = _lib.lib().hysparse_probe_l2_read(_ptr(buf), nbytes, int(passes), int(mode), int(blocks), _ptr(sink),
                                           _stream(dev))
    _lib.check(st, "hysparse_probe_l2_read")


def kv_cache_bytes(B: int, Lkv: int, Hkv: int, d: int, elem_bytes: int, n_sparse: int, window: int,
                   own_window: bool = False, Lq: int = 1) -> dict:
    """KV-cache bytes one hybrid block keeps for a batch (HySparse abstract and
    write-up section 3.1: only the full layer writes a cache, which its sparse
    layers reuse; section 2.2: a sparse layer's local branch may keep its own
    sliding window).

    full: the full layer's K and V, 2 * B * Lkv * Hkv * d elements.
    sparse: 0 when the sparse layers read the shared cache; with own windows,
    each of the n_sparse layers keeps K and V for the rows its window branch
    reads while Lq new rows are processed, min(Lkv, window - 1 + Lq) per
    sequence (window rows for one decode step).
    dense_equivalent: the same 1 + n_sparse layers all with full caches.
    """
    per_row = 2 * B * Hkv * d * elem_bytes
    full = per_row * Lkv
    sparse = n_sparse * per_row * min(Lkv, window - 1 + Lq) if own_window else 0
    return {"full": full, "sparse": sparse, "total": full + sparse,
            "dense_equivalent": (1 + n_sparse) * full}


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.lib().hysparse_launch_count())


def version() -> str:
    return _lib.lib().hysparse_version().decode()
