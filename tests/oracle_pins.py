"""Pins for the CPU oracle: each check ties one oracle function to something
other than itself -- a library routine for a special case (torch's fp64
scaled_dot_product_attention, softmax, logsumexp; numpy's stable argsort), a
closed form, an invariant, or brute force on tiny inputs.

Each ``pin_*`` function raises AssertionError when the oracle disagrees.  The
same functions run against mutated copies of the oracle (test_oracle_mutants)
to show that a plausible slip in any step is caught.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle

TOL = 1e-10


def _rand(*shape, seed=0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def _all_rows(B, Lq):
    return [(b, i) for b in range(B) for i in range(Lq)]


def _q_rows(q, rows):
    return torch.stack([q[b, i] for b, i in rows])


def _allowed(Lq, Lkv):
    """Boolean [Lq, Lkv]: key j is visible to query row i (bottom-right causal)."""
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lkv)[None, :]
    return j <= (Lkv - Lq + i)


def _sdpa(q, k, v, allowed, scale):
    """torch fp64 attention with an explicit boolean mask [B?,Lq,Lkv] or
    [Lq,Lkv] (True = attend).  q [B,Lq,Hq,d], k/v [B,Lkv,Hkv,d]."""
    B, Lq, Hq, d = q.shape
    G = Hq // k.shape[2]
    qq = q.double().permute(0, 2, 1, 3)
    kk = k.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vv = v.double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    if allowed.dim() == 2:
        allowed = allowed[None, None]
    return F.scaled_dot_product_attention(qq, kk, vv, attn_mask=allowed, scale=scale).permute(0, 2, 1, 3)


def _masked_logits(q, k, scale, allowed):
    B, Lq, Hq, d = q.shape
    G = Hq // k.shape[2]
    kk = k.double().repeat_interleave(G, dim=2)
    lg = torch.einsum("bihd,bjhd->bhij", q.double(), kk) * scale
    return lg.masked_fill(~allowed[None, None], float("-inf"))


SHAPES = [
    # B, Lq, Lkv, Hq, Hkv, d
    (2, 13, 13, 4, 2, 8),
    (1, 5, 17, 6, 3, 16),
    (3, 1, 11, 4, 1, 8),
    (1, 9, 9, 2, 2, 4),
]


def pin_full_matches_sdpa():
    """Full layer O and LSE equal torch's fp64 masked attention and logsumexp."""
    for si, (B, Lq, Lkv, Hq, Hkv, d) in enumerate(SHAPES):
        q, k, v = _rand(B, Lq, Hq, d, seed=si), _rand(B, Lkv, Hkv, d, seed=10 + si), _rand(B, Lkv, Hkv, d, seed=20 + si)
        scale = 1.0 / math.sqrt(d)
        rows = _all_rows(B, Lq)
        out, lse, _ = oracle.full_rows(_q_rows(q, rows), k, v, rows, Lq, scale, want_scores=False)
        allowed = _allowed(Lq, Lkv)
        ref = _sdpa(q, k, v, allowed, scale).reshape(B * Lq, Hq, d)
        assert torch.allclose(out, ref, atol=TOL, rtol=0), f"O mismatch shape {si}"
        lse_ref = torch.logsumexp(_masked_logits(q, k, scale, allowed), dim=-1)  # [B,Hq,Lq]
        assert torch.allclose(lse, lse_ref.permute(0, 2, 1).reshape(B * Lq, Hq), atol=TOL, rtol=0), \
            f"LSE mismatch shape {si}"


def pin_scores_match_softmax_group_sum():
    """Importance = sum over the group's heads of torch.softmax probabilities."""
    for si, (B, Lq, Lkv, Hq, Hkv, d) in enumerate(SHAPES):
        q, k, v = _rand(B, Lq, Hq, d, seed=30 + si), _rand(B, Lkv, Hkv, d, seed=40 + si), _rand(B, Lkv, Hkv, d, seed=50 + si)
        scale = 1.0 / math.sqrt(d)
        rows = _all_rows(B, Lq)
        _, _, sc = oracle.full_rows(_q_rows(q, rows), k, v, rows, Lq, scale)
        allowed = _allowed(Lq, Lkv)
        p = torch.softmax(_masked_logits(q, k, scale, allowed), dim=-1)       # [B,Hq,Lq,Lkv]
        G = Hq // Hkv
        ref = p.reshape(B, Hkv, G, Lq, Lkv).sum(2).permute(0, 2, 1, 3).reshape(B * Lq, Hkv, Lkv)
        assert torch.allclose(sc, ref, atol=TOL, rtol=0), f"score mismatch shape {si}"


def pin_scores_sum_to_group_size():
    """Each (row, KV head) importance row sums to G: the G softmax rows each sum to 1."""
    B, Lq, Lkv, Hq, Hkv, d = 2, 24, 40, 8, 2, 16
    q, k, v = _rand(B, Lq, Hq, d, seed=1), _rand(B, Lkv, Hkv, d, seed=2), _rand(B, Lkv, Hkv, d, seed=3)
    q = q * 3.0   # sharper softmax
    rows = _all_rows(B, Lq)
    _, _, sc = oracle.full_rows(_q_rows(q, rows), k, v, rows, Lq, 1.0 / math.sqrt(d))
    s = sc.sum(-1)
    assert torch.allclose(s, torch.full_like(s, Hq // Hkv), atol=1e-12, rtol=0)
    # entries past the causal position are zero
    for r, (b, i) in enumerate(rows):
        pos = Lkv - Lq + i
        assert torch.all(sc[r, :, pos + 1:] == 0)
        assert torch.all(sc[r, :, :pos + 1] > 0)


def pin_scores_closed_forms():
    """L=1: the single key gets score G.  Identical keys: every visible key
    gets G/(pos+1), and O equals that shared value row."""
    Hq, Hkv, d = 6, 2, 8
    G = Hq // Hkv
    q, k, v = _rand(1, 1, Hq, d, seed=4), _rand(1, 1, Hkv, d, seed=5), _rand(1, 1, Hkv, d, seed=6)
    out, lse, sc = oracle.full_rows(q[0], k, v, [(0, 0)], 1, 0.3)
    assert torch.all(sc == G)
    assert torch.allclose(out[0], v[0, 0].double().repeat_interleave(G, 0), atol=1e-15)
    L = 7
    q = _rand(1, L, Hq, d, seed=7)
    k = _rand(1, 1, Hkv, d, seed=8).expand(1, L, Hkv, d).contiguous()
    v = _rand(1, 1, Hkv, d, seed=9).expand(1, L, Hkv, d).contiguous()
    rows = _all_rows(1, L)
    out, lse, sc = oracle.full_rows(_q_rows(q, rows), k, v, rows, L, 0.5)
    for r, (_, i) in enumerate(rows):
        assert torch.allclose(sc[r, :, :i + 1], torch.full((Hkv, i + 1), G / (i + 1), dtype=torch.float64),
                              atol=1e-14, rtol=0)
        assert torch.allclose(out[r], v[0, 0].double().repeat_interleave(G, 0), atol=1e-14)


def _stable_topk(s: np.ndarray, n: int, k: int) -> np.ndarray:
    order = np.argsort(-s[:n], kind="stable")[:min(n, k)]
    res = np.full(k, -1, dtype=np.int64)
    res[:len(order)] = np.sort(order)
    return res


def pin_topk_matches_stable_argsort():
    """Top-k equals numpy's stable argsort of -score (stable = lower index
    first among equal scores), sorted ascending and -1 padded.  Rows include
    exact ties, rows shorter than k and an all-equal row."""
    rng = np.random.default_rng(0)
    L, k = 200, 37
    rows = []
    for r in range(40):
        s = rng.random(L)
        if r % 3 == 0:
            s = np.round(s * 8) / 8               # heavy exact ties
        if r % 7 == 0:
            s[:] = 0.25                            # all tied
        rows.append(s)
    S = torch.tensor(np.stack(rows))
    n_valid = [int(n) for n in rng.integers(1, L + 1, size=len(rows))]
    n_valid[1] = 5                                  # shorter than k
    n_valid[2] = k
    n_valid[3] = L
    got = oracle.topk_rows(S, n_valid, k).numpy()
    for r in range(len(rows)):
        np.testing.assert_array_equal(got[r], _stable_topk(rows[r], n_valid[r], k))


def pin_topk_bruteforce():
    """On tiny rows, enumerate every k-subset: exactly one subset T has every
    member ranked before every non-member under (-score, index); the oracle
    must return it."""
    rng = np.random.default_rng(1)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, 9))
        s = rng.integers(0, 4, size=n).astype(np.float64) / 4.0   # many ties
        got = oracle.topk_rows(torch.tensor(s)[None], [n], k).numpy()[0]
        m = min(n, k)
        winners = []
        for T in itertools.combinations(range(n), m):
            rest = [j for j in range(n) if j not in T]
            if all((s[a] > s[b]) or (s[a] == s[b] and a < b) for a in T for b in rest):
                winners.append(T)
        assert len(winners) == 1
        expect = list(winners[0]) + [-1] * (k - m)
        assert list(got) == expect, (s, k, got, expect)


def _sparse_case(seed, B=2, Lq=10, Lkv=16, Hq=4, Hkv=2, d=8):
    q = _rand(B, Lq, Hq, d, seed=seed)
    k = _rand(B, Lkv, Hkv, d, seed=seed + 1)
    v = _rand(B, Lkv, Hkv, d, seed=seed + 2)
    gate = _rand(B, Lq, Hq, seed=seed + 3)
    return q, k, v, gate


def _idx_from_sets(sets, topk):
    out = torch.full((len(sets), len(sets[0]), topk), -1, dtype=torch.int32)
    for r, per_g in enumerate(sets):
        for g, st in enumerate(per_g):
            st = sorted(st)
            out[r, g, :len(st)] = torch.tensor(st, dtype=torch.int32)
    return out


def pin_sparse_branches_vs_sdpa():
    """Global branch = torch attention masked to the index set; local branch =
    torch attention masked to the band pos-w+1 .. pos (w keys including the
    query's own position)."""
    B, Lq, Lkv, Hq, Hkv, d = 2, 10, 16, 4, 2, 8
    q, k, v, gate = _sparse_case(100, B, Lq, Lkv, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    rows = _all_rows(B, Lq)
    rng = np.random.default_rng(5)
    topk, window = 5, 3
    sets = []
    allowed_g = torch.zeros(B, Hkv, Lq, Lkv, dtype=torch.bool)
    for (b, i) in rows:
        pos = Lkv - Lq + i
        per_g = []
        for g in range(Hkv):
            st = rng.choice(pos + 1, size=min(topk, pos + 1), replace=False).tolist()
            per_g.append(st)
            allowed_g[b, g, i, st] = True
        sets.append(per_g)
    idx = _idx_from_sets(sets, topk)
    out, og, ol = oracle.sparse_rows(_q_rows(q, rows), k, v, rows, Lq, scale, idx,
                                     _q_rows(gate, rows), window)
    G = Hq // Hkv
    ref_g = _sdpa(q, k, v, allowed_g.repeat_interleave(G, dim=1), scale).reshape(B * Lq, Hq, d)
    assert torch.allclose(og, ref_g, atol=TOL, rtol=0), "global branch"
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lkv)[None, :]
    pos = Lkv - Lq + i
    band = (j <= pos) & (j >= pos - window + 1)
    ref_l = _sdpa(q, k, v, band, scale).reshape(B * Lq, Hq, d)
    assert torch.allclose(ol, ref_l, atol=TOL, rtol=0), "local branch"


def pin_own_window_branch_vs_sdpa():
    """Own-window variant (each sparse layer keeps its own K/V for its window):
    the local branch = torch attention over the band pos-w+1 .. pos with the
    layer's own keys and values placed at their positions, for a buffer that
    holds the whole sequence and for one that holds only its last Lwin
    positions; the global branch still reads the shared cache unchanged."""
    B, Lkv, Hq, Hkv, d = 2, 16, 4, 2, 8
    scale = 1.0 / math.sqrt(d)
    window, topk = 4, 5
    for Lq, Lwin in ((16, 16), (3, 6)):
        q, k, v, gate = _sparse_case(700 + Lq, B, Lq, Lkv, Hq, Hkv, d)
        kw = _rand(B, Lwin, Hkv, d, seed=710 + Lq)
        vw = _rand(B, Lwin, Hkv, d, seed=720 + Lq)
        rows = _all_rows(B, Lq)
        rng = np.random.default_rng(7)
        sets = [[rng.choice(Lkv - Lq + i + 1, size=min(topk, Lkv - Lq + i + 1), replace=False).tolist()
                 for _ in range(Hkv)] for (_, i) in rows]
        idx = _idx_from_sets(sets, topk)
        qr, gr = _q_rows(q, rows), _q_rows(gate, rows)
        out, og, ol = oracle.sparse_rows(qr, k, v, rows, Lq, scale, idx, gr, window, k_win=kw, v_win=vw)
        out0, og0, _ = oracle.sparse_rows(qr, k, v, rows, Lq, scale, idx, gr, window)
        assert torch.equal(og, og0), "global branch reads the shared cache"
        kfull = torch.zeros(B, Lkv, Hkv, d)
        vfull = torch.zeros(B, Lkv, Hkv, d)
        kfull[:, Lkv - Lwin:] = kw
        vfull[:, Lkv - Lwin:] = vw
        i = torch.arange(Lq)[:, None]
        j = torch.arange(Lkv)[None, :]
        pos = Lkv - Lq + i
        band = (j <= pos) & (j >= pos - window + 1)
        ref_l = _sdpa(q, kfull, vfull, band, scale).reshape(B * Lq, Hq, d)
        assert torch.allclose(ol, ref_l, atol=TOL, rtol=0), "own-window local branch"
        sg = torch.sigmoid(gr.double())[..., None]
        assert torch.allclose(out, sg * og + (1 - sg) * ol, atol=TOL, rtol=0), "gate"
        assert not torch.allclose(ol, _sdpa(q, k, v, band, scale).reshape(B * Lq, Hq, d))


def pin_sparse_reduces_to_full():
    """With k >= pos+1 the global branch is full causal attention; with a
    window >= Lkv the local branch is full causal attention."""
    B, Lq, Lkv, Hq, Hkv, d = 1, 12, 12, 4, 1, 8
    q, k, v, gate = _sparse_case(200, B, Lq, Lkv, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    rows = _all_rows(B, Lq)
    topk = Lkv
    sets = [[list(range(Lkv - Lq + i + 1)) for _ in range(Hkv)] for (_, i) in rows]
    idx = _idx_from_sets(sets, topk)
    _, og, ol = oracle.sparse_rows(_q_rows(q, rows), k, v, rows, Lq, scale, idx, _q_rows(gate, rows), Lkv)
    ref = _sdpa(q, k, v, _allowed(Lq, Lkv), scale).reshape(B * Lq, Hq, d)
    assert torch.allclose(og, ref, atol=TOL, rtol=0)
    assert torch.allclose(ol, ref, atol=TOL, rtol=0)


def pin_gate_limits():
    """gate logit -> -inf gives the local branch alone, +inf the global branch
    alone, 0 their mean (sigmoid(0) = 1/2)."""
    B, Lq, Lkv, Hq, Hkv, d = 1, 8, 8, 4, 2, 8
    q, k, v, _ = _sparse_case(300, B, Lq, Lkv, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    rows = _all_rows(B, Lq)
    sets = [[[0, Lkv - Lq + i] if Lkv - Lq + i > 0 else [0] for _ in range(Hkv)] for (_, i) in rows]
    idx = _idx_from_sets(sets, 2)
    qr = _q_rows(q, rows)
    for val, pick in ((-1e30, "l"), (1e30, "g"), (0.0, "mean")):
        gate = torch.full((len(rows), Hq), val)
        out, og, ol = oracle.sparse_rows(qr, k, v, rows, Lq, scale, idx, gate, 3)
        expect = {"l": ol, "g": og, "mean": 0.5 * (og + ol)}[pick]
        assert torch.allclose(out, expect, atol=1e-15, rtol=0), pick
        assert not torch.allclose(og, ol)


def pin_block_composes():
    """block_rows = full layer -> top-k -> each sparse layer, row by row."""
    B, Lq, Lkv, Hq, Hkv, d = 1, 20, 20, 4, 2, 8
    q, k, v, gate = _sparse_case(400, B, Lq, Lkv, Hq, Hkv, d)
    qs = torch.stack([_rand(B, Lq, Hq, d, seed=500 + n) for n in range(2)])
    gs = torch.stack([_rand(B, Lq, Hq, seed=600 + n) for n in range(2)])
    scale = 1.0 / math.sqrt(d)
    rows = _all_rows(B, Lq)
    topk, window = 6, 4
    of, idx, osp = oracle.block_rows(_q_rows(q, rows), k, v, rows, Lq, scale,
                                     torch.stack([_q_rows(qs[n], rows) for n in range(2)]),
                                     torch.stack([_q_rows(gs[n], rows) for n in range(2)]), topk, window)
    out, _, sc = oracle.full_rows(_q_rows(q, rows), k, v, rows, Lq, scale)
    assert torch.equal(of, out)
    n_valid = [[Lkv - Lq + i + 1] * Hkv for (_, i) in rows]
    idx2 = oracle.topk_rows(sc, n_valid, topk)
    assert torch.equal(idx, idx2)
    for n in range(2):
        o2, _, _ = oracle.sparse_rows(_q_rows(qs[n], rows), k, v, rows, Lq, scale, idx2,
                                      _q_rows(gs[n], rows), window)
        assert torch.equal(osp[n], o2)


ALL_PINS = [
    pin_full_matches_sdpa,
    pin_scores_match_softmax_group_sum,
    pin_scores_sum_to_group_size,
    pin_scores_closed_forms,
    pin_topk_matches_stable_argsort,
    pin_topk_bruteforce,
    pin_sparse_branches_vs_sdpa,
    pin_own_window_branch_vs_sdpa,
    pin_sparse_reduces_to_full,
    pin_gate_limits,
    pin_block_composes,
]
