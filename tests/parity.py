"""Shared helpers for the GPU-vs-oracle parity tests (test infrastructure).

Tolerances (HySparse hot-path contract): attention outputs max-abs error
<= 2e-2 for bf16 and <= 1e-4 for fp32; top-k sets bit-exact except for keys
whose oracle score lies within 1e-6 relative of the k-th oracle score.
Scores and LSE have no stated tolerance; the bounds below follow from fp32
arithmetic: an fp32 logit over d <= 128 products and a correctly-rounded-
ish exp2 give a few ulp (~1e-6 relative) per probability, so scores are
checked at 2e-5 relative to the row's largest score and LSE at 1e-4 absolute.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import torch

import oracle

OUT_TOL = {"f32": 1e-4, "bf16": 2e-2}
# Per-row relative L2 error gate, beside the absolute one.  On the shifted
# prefill workloads the outputs are ~1e-3 (nearly flat softmax over values of
# std 1/sqrt(d)), so the absolute bound alone would pass zeros; a row's error
# relative to its own norm does not.  bf16: the output's rounding (unit
# roundoff 2^-8, ~2.3e-3 rms relative) plus P rounded to bf16 before the PV
# product (~2.3e-3 rms relative of a random-sign sum) give ~3.3e-3; the gate
# is 1e-2.  fp32: a few ulp per term, ~1e-6; the gate is 1e-4.
REL_L2_TOL = {"f32": 1e-4, "bf16": 1e-2}
SCORE_RTOL = 2e-5
LSE_ATOL = 1e-4
TIE_BAND = 1e-6


def scale_of(d: int) -> float:
    return 1.0 / math.sqrt(d)


def rows_for(B: int, Lq: int, row_list: Sequence[int]) -> List[Tuple[int, int]]:
    return [(b, i) for b in range(B) for i in row_list]


def gather_rows(t: torch.Tensor, rows) -> torch.Tensor:
    """t [B,Lq,...] -> [nrows,...] on the host (fp32 widening is exact)."""
    b = torch.tensor([r[0] for r in rows], device=t.device)
    i = torch.tensor([r[1] for r in rows], device=t.device)
    return t[b, i].to("cpu")


def gather_idx_rows(idx: torch.Tensor, rows) -> torch.Tensor:
    """idx [B,Hkv,Lq,k] -> [nrows,Hkv,k] on the host."""
    b = torch.tensor([r[0] for r in rows], device=idx.device)
    i = torch.tensor([r[1] for r in rows], device=idx.device)
    return idx[b, :, i].to("cpu")


def max_abs(a: torch.Tensor, b: torch.Tensor) -> float:
    return float((a.double().cpu() - b.double().cpu()).abs().max()) if a.numel() else 0.0


def rel_l2(a: torch.Tensor, b: torch.Tensor) -> float:
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).norm() / max(float(b.norm()), 1e-300))


def row_rel_l2(got: torch.Tensor, ref: torch.Tensor) -> torch.Tensor:
    """Relative L2 error of every leading-index row ([R, ...] -> [R]); rows
    whose reference is exactly zero (an empty branch) give their absolute
    error norm."""
    a = got.double().cpu().reshape(got.shape[0], -1)
    b = ref.double().cpu().reshape(ref.shape[0], -1)
    nb = b.norm(dim=1)
    return (a - b).norm(dim=1) / torch.where(nb > 0, nb, torch.ones_like(nb))


WORST = {}


def check_out(name: str, got: torch.Tensor, ref: torch.Tensor, dtype: str) -> float:
    """max-abs error <= OUT_TOL (the contract's bound) and, per row, relative
    L2 error <= REL_L2_TOL.  Returns the worst row's relative L2 error (also
    kept in WORST under `name` and printed, so pytest -s shows it)."""
    err = max_abs(got, ref)
    rel = float(row_rel_l2(got, ref).max()) if got.numel() else 0.0
    WORST[name] = max(rel, WORST.get(name, 0.0))
    print(f"[parity] {name}: max abs {err:.3e}, worst row rel L2 {rel:.3e}")
    tol = OUT_TOL[dtype]
    assert err <= tol, f"{name}: max abs error {err:.3e} > {tol:.1e} (worst row rel L2 {rel:.2e})"
    rtol = REL_L2_TOL[dtype]
    assert rel <= rtol, f"{name}: worst row relative L2 error {rel:.3e} > {rtol:.0e} (max abs {err:.2e})"
    return rel


def check_topk(gpu_idx: torch.Tensor, ora_scores: torch.Tensor, n_valid: Sequence[int], topk: int) -> Dict[str, int]:
    """gpu_idx [R,k] int32 host; ora_scores [R,Lkv] f64 (oracle); n_valid[r]
    = pos+1.  The GPU set must equal the oracle's top-k except for keys inside
    the tie band around the k-th oracle score; the GPU list must also be
    well formed (ascending valid keys, then -1)."""
    ora_idx = oracle.topk_rows(ora_scores, n_valid, topk)
    stats = {"rows": 0, "band_rows": 0, "band_keys": 0}
    for r in range(gpu_idx.shape[0]):
        n = int(n_valid[r])
        g = gpu_idx[r].tolist()
        take = min(n, topk)
        assert all(x == -1 for x in g[take:]), f"row {r}: padding wrong"
        sel = g[:take]
        assert all(0 <= x < n for x in sel), f"row {r}: key out of range"
        assert all(sel[t] < sel[t + 1] for t in range(len(sel) - 1)), f"row {r}: not ascending"
        stats["rows"] += 1
        o = set(ora_idx[r, :take].tolist())
        gs = set(sel)
        if gs == o:
            continue
        s = ora_scores[r, :n].double()
        kth = float(torch.topk(s, take).values[-1])
        diff = gs.symmetric_difference(o)
        for j in diff:
            assert abs(float(s[j]) - kth) <= TIE_BAND * kth, \
                f"row {r}: key {j} score {float(s[j]):.9e} outside the tie band of k-th {kth:.9e}"
        stats["band_rows"] += 1
        stats["band_keys"] += len(diff)
    return stats


def check_scores(gpu_scores_rows: torch.Tensor, ora_scores: torch.Tensor, n_valid: Sequence[int]) -> float:
    """Relative (to the row max) score error over valid entries; returns the max."""
    worst = 0.0
    for r in range(ora_scores.shape[0]):
        n = int(n_valid[r])
        a = gpu_scores_rows[r, :n].double().cpu()
        b = ora_scores[r, :n].double()
        e = float((a - b).abs().max() / b.max())
        worst = max(worst, e)
    assert worst <= SCORE_RTOL, f"score error {worst:.3e} > {SCORE_RTOL:.0e}"
    return worst
