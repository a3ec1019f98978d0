"""Seeded synthetic inputs for the HySparse hybrid block.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic (no attention, no scores, no selection).  Both the CUDA
path and the CPU oracle consume the tensors it returns, so the two sides see
the same bytes.

Workloads (HySparse: A Hybrid Sparse Attention Architecture with Oracle Token
Selection and KV Cache Sharing, abstract: 7B dense and 80B MoE models, 49
layers of which 5 are full attention; the intelliparadigm write-up, section
2.2: a 128-token local window; DeepSeek Sparse Attention as described in the
ultralytics glossary, "content-based patterns": 2048 selected keys):

* ``tiny``      B=1, L=512,   Hq=4,  Hkv=1, d=64,  fp32, 1 sparse layer, k=64
* ``prefill8k`` B=1, L=8192,  Hq=32, Hkv=8, d=128, bf16, 3 sparse layers, k=1024
* ``prefill32k``B=1, L=32768, Hq=32, Hkv=8, d=128, bf16, 3 sparse layers, k=2048
* ``decode``    B=64, 1 new token over a 32768-token cache, Hq=32, Hkv=8,
                d=128, bf16, 3 sparse layers, k=2048
* ``moe64k``    B=1, L=65536, Hq=64, Hkv=4, d=128, bf16, 9 sparse layers, k=2048

Value recipes:

* ``normal``: Q, K, V, every sparse layer's Q' ~ N(0, 1).
* ``shifted``: Q, K, V, Q' ~ N(0, 1)/sqrt(d); then, per (batch, KV head) g, a
  random unit direction u_g and round(0.02 * Lkv) random key positions (a
  random permutation's prefix) get +3*sigma*u_g added (sigma = 1/sqrt(d), the
  per-coordinate std), and the same +3*sigma*u_g is added to every query of
  group g in the full layer and in every sparse layer.  V is not shifted.
* Gate logits ~ N(0, 1), one per (batch, token, query head, sparse layer), fp32.

Draw order (fixed): Q_full, K, V, [u, shifted positions], then for each
sparse layer n: Q'_n, gate_n.  Values are drawn in fp32, scaled and shifted in
fp32, then rounded to bf16 where the workload is bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Lq: int
    Lkv: int
    Hq: int
    Hkv: int
    d: int
    dtype: str          # "f32" or "bf16"
    topk: int
    window: int
    n_sparse: int
    dist: str           # "normal" or "shifted"

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 512, 512, 4, 1, 64, "f32", 64, 128, 1, "normal"),
    "prefill8k": Workload("prefill8k", 1, 8192, 8192, 32, 8, 128, "bf16", 1024, 128, 3, "shifted"),
    "prefill32k": Workload("prefill32k", 1, 32768, 32768, 32, 8, 128, "bf16", 2048, 128, 3, "shifted"),
    "decode": Workload("decode", 64, 1, 32768, 32, 8, 128, "bf16", 2048, 128, 3, "normal"),
    "moe64k": Workload("moe64k", 1, 65536, 65536, 64, 4, 128, "bf16", 2048, 128, 9, "shifted"),
}

SHIFT_FRACTION = 0.02
SHIFT_SIGMAS = 3.0


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def make_inputs(w: Workload, seed: int = 0, device: str = "cpu") -> Dict[str, object]:
    """Draw one hybrid block's inputs for workload ``w``.

    Returns a dict with ``q`` [B,Lq,Hq,d], ``k`` and ``v`` [B,Lkv,Hkv,d]
    (the workload dtype), ``q_sparse`` (list of n_sparse tensors shaped like
    ``q``), ``gate`` (list of n_sparse fp32 tensors [B,Lq,Hq]) and, for the
    shifted recipe, ``shift_pos`` [B,Hkv,n_shift] (int64) for diagnostics.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    f32 = torch.float32
    B, Lq, Lkv, Hq, Hkv, d = w.B, w.Lq, w.Lkv, w.Hq, w.Hkv, w.d
    out_dtype = torch_dtype(w)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=f32)

    q = randn(B, Lq, Hq, d)
    k = randn(B, Lkv, Hkv, d)
    v = randn(B, Lkv, Hkv, d)
    shift = None
    shift_pos = None
    if w.dist == "shifted":
        sigma = 1.0 / math.sqrt(d)
        q.mul_(sigma)
        k.mul_(sigma)
        v.mul_(sigma)
        u = randn(B, Hkv, d)
        u = u / u.norm(dim=-1, keepdim=True)
        shift = (SHIFT_SIGMAS * sigma) * u                          # [B,Hkv,d]
        n_shift = int(round(SHIFT_FRACTION * Lkv))
        shift_pos = torch.empty(B, Hkv, n_shift, dtype=torch.int64, device=dev)
        for b in range(B):
            for h in range(Hkv):
                shift_pos[b, h] = torch.randperm(Lkv, generator=g, device=dev)[:n_shift]
        for b in range(B):
            for h in range(Hkv):
                k[b, shift_pos[b, h], h, :] += shift[b, h]
        q.add_(shift.repeat_interleave(w.G, dim=1)[:, None, :, :])
    elif w.dist != "normal":
        raise ValueError(f"unknown value recipe {w.dist!r}")

    q_sparse: List[torch.Tensor] = []
    gate: List[torch.Tensor] = []
    for _ in range(w.n_sparse):
        qs = randn(B, Lq, Hq, d)
        if shift is not None:
            qs.mul_(1.0 / math.sqrt(d))
            qs.add_(shift.repeat_interleave(w.G, dim=1)[:, None, :, :])
        q_sparse.append(qs.to(out_dtype))
        gate.append(randn(B, Lq, Hq))
    res = {
        "q": q.to(out_dtype),
        "k": k.to(out_dtype),
        "v": v.to(out_dtype),
        "q_sparse": q_sparse,
        "gate": gate,
    }
    if shift_pos is not None:
        res["shift_pos"] = shift_pos
    return res


def make_window_kv(w: Workload, lwin: int, seed: int = 0, device: str = "cpu"):
    """Draw one sparse layer's own window keys and values, [B,lwin,Hkv,d]
    each in the workload dtype, for cache positions Lkv - lwin .. Lkv - 1.

    Drawn from a generator of their own (so the block's other inputs are the
    same with or without them): standard normal for the "normal" recipe,
    normal with std 1/sqrt(d) for the "shifted" one (the scale of that
    recipe's unshifted keys and values).
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    sigma = 1.0 / math.sqrt(w.d) if w.dist == "shifted" else 1.0
    kw = torch.randn(w.B, lwin, w.Hkv, w.d, generator=g, device=dev, dtype=torch.float32) * sigma
    vw = torch.randn(w.B, lwin, w.Hkv, w.d, generator=g, device=dev, dtype=torch.float32) * sigma
    return kw.to(torch_dtype(w)), vw.to(torch_dtype(w))


def random_index_sets(B: int, Hkv: int, Lq: int, Lkv: int, topk: int, seed: int = 0) -> torch.Tensor:
    """Seeded index sets for a sparse layer, int32 [B,Hkv,Lq,topk] on the
    host: row i of (b, g) holds min(pos(i) + 1, topk) distinct keys drawn
    uniformly from [0, pos(i)], pos(i) = Lkv - Lq + i, in ascending order,
    padded with -1 (the layout a top-k selection writes)."""
    g = torch.Generator().manual_seed(seed)
    idx = torch.full((B, Hkv, Lq, topk), -1, dtype=torch.int32)
    for b in range(B):
        for h in range(Hkv):
            for i in range(Lq):
                n = Lkv - Lq + i + 1
                take = min(n, topk)
                if n <= 4 * topk:
                    pick = torch.randperm(n, generator=g)[:take]
                else:
                    pick = torch.unique(torch.randint(0, n, (2 * take,), generator=g))
                    while pick.numel() < take:
                        pick = torch.unique(torch.cat([pick, torch.randint(0, n, (take,), generator=g)]))
                    pick = pick[torch.randperm(pick.numel(), generator=g)[:take]]
                idx[b, h, i, :take] = pick.sort().values.to(torch.int32)
    return idx


def sample_rows(Lq: int, topk: int, window: int, n_random: int = 256, seed: int = 0,
                edge: int = 64) -> List[int]:
    """A seeded, sorted sample of query rows for checks at full size.

    Takes the first and last ``edge`` rows, the rows around the point where a
    row first has more causal keys than ``topk`` (topk-2 .. topk+1), the rows
    around the window edge (window-2 .. window+1), and ``n_random`` uniform
    random rows.
    """
    rows = set(range(min(edge, Lq)))
    rows.update(range(max(0, Lq - edge), Lq))
    for c in (topk, window):
        rows.update(r for r in range(c - 2, c + 2) if 0 <= r < Lq)
    g = torch.Generator().manual_seed(seed)
    if n_random > 0 and Lq > 0:
        rows.update(torch.randint(0, Lq, (n_random,), generator=g).tolist())
    return sorted(rows)


def to_oracle_f32(t: torch.Tensor) -> torch.Tensor:
    """Exact widening of a bf16/fp32 tensor to contiguous fp32 on the host."""
    return t.detach().to("cpu", torch.float32).contiguous()


def n_shift_keys(Lkv: int) -> int:
    return int(round(SHIFT_FRACTION * Lkv))


def workload(name: str, **override) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**override) if override else w


__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_window_kv", "random_index_sets", "sample_rows",
           "to_oracle_f32", "torch_dtype", "workload", "n_shift_keys"]
