"""The seeded input generator (no GPU): deterministic, the documented shapes
and dtypes, and the two value recipes as stated -- N(0, 1) draws, and the
shifted recipe (N(0, 1)/sqrt(d), 2 % of the keys of each (batch, KV head)
moved by 3 sigma along one unit direction that every query of the group also
carries; V not shifted).  Both the CUDA path and the oracle consume these
tensors, so the recipe is pinned here rather than trusted."""
import math

import pytest
import torch

from hybrid_sparse_attention_tcgen05_b200 import inputs as gen


def _small(name, **kw):
    base = dict(Lq=256, Lkv=256, n_sparse=2)
    if name == "decode":
        base = dict(B=2, Lq=1, Lkv=512, n_sparse=2)
    base.update(kw)
    return gen.workload(name, **base)


@pytest.mark.parametrize("name", sorted(gen.WORKLOADS))
def test_shapes_dtypes_and_determinism(name):
    w = _small(name)
    a = gen.make_inputs(w, seed=5)
    b = gen.make_inputs(w, seed=5)
    c = gen.make_inputs(w, seed=6)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    assert a["q"].shape == (w.B, w.Lq, w.Hq, w.d) and a["q"].dtype == dt
    for t in ("k", "v"):
        assert a[t].shape == (w.B, w.Lkv, w.Hkv, w.d) and a[t].dtype == dt
    assert len(a["q_sparse"]) == len(a["gate"]) == w.n_sparse
    for qs, gl in zip(a["q_sparse"], a["gate"]):
        assert qs.shape == a["q"].shape and qs.dtype == dt
        assert gl.shape == (w.B, w.Lq, w.Hq) and gl.dtype == torch.float32
    for t in ("q", "k", "v"):
        assert torch.equal(a[t], b[t])
        assert not torch.equal(a[t], c[t])
    for n in range(w.n_sparse):
        assert torch.equal(a["q_sparse"][n], b["q_sparse"][n]) and torch.equal(a["gate"][n], b["gate"][n])


def test_normal_recipe_moments():
    w = gen.workload("tiny").with_(Lq=1024, Lkv=1024, n_sparse=1)
    x = gen.make_inputs(w, seed=0)
    for t in (x["q"], x["k"], x["v"], x["q_sparse"][0], x["gate"][0]):
        t = t.float()
        n = t.numel()                     # bounds: 5 standard errors of the sample mean / std
        assert abs(t.mean().item()) < 5.0 / math.sqrt(n)
        assert abs(t.std().item() - 1.0) < 5.0 / math.sqrt(2 * n)
    assert "shift_pos" not in x


def test_shifted_recipe():
    w = gen.workload("prefill8k").with_(Lq=2048, Lkv=2048, n_sparse=1)
    x = gen.make_inputs(w, seed=1)
    sigma = 1.0 / math.sqrt(w.d)
    n_shift = gen.n_shift_keys(w.Lkv)
    assert n_shift == round(0.02 * w.Lkv)
    pos = x["shift_pos"]
    assert pos.shape == (w.B, w.Hkv, n_shift)
    q, k, v = (x[t].float() for t in ("q", "k", "v"))
    qs = x["q_sparse"][0].float()
    for b in range(w.B):
        for g in range(w.Hkv):
            p = pos[b, g]
            assert len(set(p.tolist())) == n_shift and int(p.min()) >= 0 and int(p.max()) < w.Lkv
            heads = slice(g * w.G, (g + 1) * w.G)
            # the group's queries carry +3 sigma u: their mean recovers u
            mq = q[b, :, heads, :].reshape(-1, w.d).mean(0)
            assert abs(mq.norm().item() / sigma - 3.0) < 0.1
            u = mq / mq.norm()
            # the sparse layers' queries carry the same direction
            ms = qs[b, :, heads, :].reshape(-1, w.d).mean(0)
            assert torch.dot(ms, u).item() / sigma == pytest.approx(3.0, abs=0.1)
            mask = torch.zeros(w.Lkv, dtype=torch.bool)
            mask[p] = True
            proj = k[b, :, g, :] @ u / sigma
            assert abs(proj[mask].mean().item() - 3.0) < 0.6
            assert abs(proj[~mask].mean().item()) < 0.1
            assert abs(k[b, ~mask, g, :].std().item() / sigma - 1.0) < 0.05
            vproj = v[b, :, g, :] @ u / sigma
            assert abs(vproj[mask].mean().item()) < 0.6      # V is not shifted
    for t in (q, k, v):
        assert abs(t.std().item() / sigma - 1.0) < 0.15


def test_sample_rows():
    rows = gen.sample_rows(4096, 1024, 128, n_random=50, seed=0, edge=16)
    assert rows == sorted(set(rows)) and rows[0] == 0 and rows[-1] == 4095
    for r in list(range(16)) + list(range(4080, 4096)) + [1022, 1023, 1024, 1025, 126, 127, 128, 129]:
        assert r in rows
    assert gen.sample_rows(4096, 1024, 128, n_random=50, seed=0, edge=16) == rows


def test_window_kv_and_index_sets():
    w = gen.Workload("t", 2, 50, 300, 8, 2, 128, "bf16", 40, 64, 1, "shifted")
    kw, vw = gen.make_window_kv(w, 113, seed=1)
    assert kw.shape == (2, 113, 2, 128) and vw.shape == kw.shape and kw.dtype == torch.bfloat16
    kw2, _ = gen.make_window_kv(w, 113, seed=1)
    assert torch.equal(kw, kw2)
    assert abs(float(kw.float().std()) * math.sqrt(128) - 1.0) < 0.05     # std 1/sqrt(d)
    # drawn apart from the block's other inputs: those are unchanged
    a = gen.make_inputs(w, seed=1)
    gen.make_window_kv(w, 113, seed=1)
    assert torch.equal(a["k"], gen.make_inputs(w, seed=1)["k"])
    for Lq, Lkv, topk in ((50, 300, 40), (3, 20000, 64)):
        idx = gen.random_index_sets(2, 2, Lq, Lkv, topk, seed=7)
        assert idx.dtype == torch.int32 and idx.shape == (2, 2, Lq, topk)
        assert torch.equal(idx, gen.random_index_sets(2, 2, Lq, Lkv, topk, seed=7))
        for b in range(2):
            for h in range(2):
                for i in range(Lq):
                    pos = Lkv - Lq + i
                    row = idx[b, h, i].tolist()
                    take = min(pos + 1, topk)
                    assert all(x == -1 for x in row[take:])
                    sel = row[:take]
                    assert all(0 <= x <= pos for x in sel) and sel == sorted(set(sel))


def test_kv_cache_bytes():
    import hybrid_sparse_attention_tcgen05_b200 as hs
    B, Lkv, Hkv, d, n, win = 2, 1000, 4, 128, 3, 128
    full = torch.empty(2, B, Lkv, Hkv, d, dtype=torch.bfloat16)
    ring = torch.empty(n, 2, B, win, Hkv, d, dtype=torch.bfloat16)
    r = hs.kv_cache_bytes(B, Lkv, Hkv, d, 2, n, win)
    assert r["full"] == full.nbytes and r["sparse"] == 0 and r["dense_equivalent"] == (1 + n) * full.nbytes
    r = hs.kv_cache_bytes(B, Lkv, Hkv, d, 2, n, win, own_window=True)
    assert r["sparse"] == ring.nbytes and r["total"] == full.nbytes + ring.nbytes
    # a prefill chunk of 64 rows needs window - 1 + 64 rows; never more than the cache
    assert hs.kv_cache_bytes(B, Lkv, Hkv, d, 2, n, win, True, Lq=64)["sparse"] == n * 2 * B * 191 * Hkv * d * 2
    assert hs.kv_cache_bytes(B, 100, Hkv, d, 2, n, win, True, Lq=100)["sparse"] == n * 2 * B * 100 * Hkv * d * 2
