"""Decode over caches of different lengths (hysparse_block_varlen) and over
paged caches (hysparse_block_paged) on the GPU: every sequence must get
exactly what a fixed-length decode over its own contiguous cache gives, and
match the oracle; lengths outside [1, Lkv] and pages outside the pool are
reported through the workspace status word without any read outside the
cache."""
import pytest
import torch

import oracle
import hybrid_sparse_attention_tcgen05_b200 as hs
from hybrid_sparse_attention_tcgen05_b200 import _lib, inputs as gen
from parity import check_out, check_topk, scale_of

pytestmark = pytest.mark.gpu
DEV = "cuda"

# one key; shorter than, equal to and one past the window; around the
# top-k size; around the 1024-key split-K chunks of the decode kernels; the
# whole buffer
LENS = [1, 7, 128, 129, 255, 256, 300, 1023, 1024, 1025, 2049, 2500]
LKV, TOPK, WINDOW = 2500, 256, 128


def _inputs(seed=5):
    w = gen.Workload("varlen", len(LENS), 1, LKV, 32, 8, 128, "bf16", TOPK, WINDOW, 2, "normal")
    return w, gen.make_inputs(w, seed=seed, device=DEV)


def _one(inp, b, L):
    return (inp["q"][b:b + 1], inp["k"][b:b + 1, :L].contiguous(), inp["v"][b:b + 1, :L].contiguous(),
            [x[b:b + 1] for x in inp["q_sparse"]], [x[b:b + 1] for x in inp["gate"]])


def test_varlen_decode_equals_fixed_length_per_sequence():
    w, inp = _inputs()
    kv_len = torch.tensor(LENS, dtype=torch.int32, device=DEV)
    shape = hs.shape_of(inp["q"], inp["k"])
    ws = hs.alloc_workspace(shape, TOPK, WINDOW, 2, 0, DEV)
    out, lse, idx, outs = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], TOPK, WINDOW,
                                   ws=ws, kv_len=kv_len)
    assert hs.workspace_status(ws) == _lib.HS_OK
    for b, L in enumerate(LENS):
        q1, k1, v1, qs1, g1 = _one(inp, b, L)
        o1, l1, i1, s1 = hs.block(q1, k1, v1, qs1, g1, TOPK, WINDOW)
        torch.cuda.synchronize()
        assert torch.equal(out[b:b + 1], o1), f"len {L}: full-layer output"
        assert torch.equal(lse[b:b + 1], l1), f"len {L}: LSE"
        assert torch.equal(idx[b:b + 1], i1), f"len {L}: index set"
        for n in range(w.n_sparse):
            assert torch.equal(outs[n][b:b + 1], s1[n]), f"len {L}: sparse layer {n}"


def test_varlen_decode_matches_oracle():
    w, inp = _inputs(seed=6)
    lens = torch.tensor(LENS, dtype=torch.int32, device=DEV)
    out, lse, idx, outs = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], TOPK, WINDOW,
                                   kv_len=lens)
    torch.cuda.synchronize()
    scale = scale_of(128)
    for b, L in enumerate(LENS):
        q1, k1, v1, qs1, g1 = (t if isinstance(t, list) else t.cpu() for t in _one(inp, b, L))
        o_out, o_lse, o_sc = oracle.full_rows(q1[0], k1, v1, [(0, 0)], 1, scale)
        check_out(f"len {L} full out", out[b].cpu(), o_out, "bf16")
        assert float((lse[b, :, 0].cpu().double() - o_lse[0]).abs().max()) <= 1e-4
        g_idx = idx[b, :, 0].cpu()
        check_topk(g_idx, o_sc.reshape(-1, L), [L] * w.Hkv, TOPK)
        for n in range(w.n_sparse):
            r_out, _, _ = oracle.sparse_rows(qs1[n][0].cpu(), k1, v1, [(0, 0)], 1, scale, g_idx[None],
                                             g1[n][0].cpu(), WINDOW)
            check_out(f"len {L} sparse{n} out", outs[n][b].cpu(), r_out, "bf16")


def test_varlen_lengths_outside_the_cache_are_reported():
    w, inp = _inputs(seed=7)
    bad = list(LENS)
    bad[0], bad[-1] = 0, LKV + 5
    kv_len = torch.tensor(bad, dtype=torch.int32, device=DEV)
    shape = hs.shape_of(inp["q"], inp["k"])
    ws = hs.alloc_workspace(shape, TOPK, WINDOW, 2, 0, DEV)
    out, lse, idx, outs = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], TOPK, WINDOW,
                                   ws=ws, kv_len=kv_len)
    assert hs.workspace_status(ws) == _lib.HS_ERR_INVALID_ARG
    # the rest of the batch is computed as usual and the context stays usable
    assert torch.isfinite(out.float()).all()
    good = torch.tensor(LENS, dtype=torch.int32, device=DEV)
    hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], TOPK, WINDOW, ws=ws, kv_len=good)
    assert hs.workspace_status(ws) == _lib.HS_OK


def _paged(k, v, lens, page_size, seed=9, spare=7):
    """Scatter the contiguous caches into shuffled pages: pools
    [num_pages, page_size, Hkv, d] and the block table [B, max_pages]."""
    B, Lkv, Hkv, d = k.shape
    max_pages = (Lkv + page_size - 1) // page_size
    need = [(L + page_size - 1) // page_size for L in lens]
    num_pages = sum(need) + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g).tolist()
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    kp = torch.zeros(num_pages, page_size, Hkv, d, dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    nxt = 0
    for b, L in enumerate(lens):
        for pg in range(need[b]):
            page = perm[nxt]
            nxt += 1
            table[b, pg] = page
            lo, hi = pg * page_size, min(L, (pg + 1) * page_size)
            kp[page, : hi - lo] = k[b, lo:hi]
            vp[page, : hi - lo] = v[b, lo:hi]
    return kp, vp, table.to(k.device)


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_paged_decode_equals_contiguous(page_size):
    w, inp = _inputs(seed=8)
    kv_len = torch.tensor(LENS, dtype=torch.int32, device=DEV)
    out, lse, idx, outs = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], TOPK, WINDOW,
                                   kv_len=kv_len)
    kp, vp, table = _paged(inp["k"], inp["v"], LENS, page_size)
    shape = hs.HsShape(w.B, 1, LKV, w.Hq, w.Hkv, w.d, 1, 0.0)
    ws = hs.alloc_workspace(shape, TOPK, WINDOW, 2, 0, DEV)
    po, pl, pi, ps = hs.block_paged(inp["q"], kp, vp, inp["q_sparse"], inp["gate"], TOPK, WINDOW, kv_len, table,
                                    max_len=LKV, ws=ws)
    assert hs.workspace_status(ws) == _lib.HS_OK
    assert torch.equal(po, out)
    assert torch.equal(pl, lse)
    assert torch.equal(pi, idx)
    for n in range(w.n_sparse):
        assert torch.equal(ps[n], outs[n])


def test_paged_page_outside_the_pool_is_reported():
    w, inp = _inputs(seed=9)
    kv_len = torch.tensor(LENS, dtype=torch.int32, device=DEV)
    kp, vp, table = _paged(inp["k"], inp["v"], LENS, 64)
    table[-1, 3] = kp.shape[0]            # a page covering valid keys of the last sequence
    shape = hs.HsShape(w.B, 1, LKV, w.Hq, w.Hkv, w.d, 1, 0.0)
    ws = hs.alloc_workspace(shape, TOPK, WINDOW, 2, 0, DEV)
    po, _, _, ps = hs.block_paged(inp["q"], kp, vp, inp["q_sparse"], inp["gate"], TOPK, WINDOW, kv_len, table,
                                  max_len=LKV, ws=ws)
    assert hs.workspace_status(ws) == _lib.HS_ERR_INVALID_INDEX
    assert torch.isfinite(po.float()).all()
    for x in ps:
        assert torch.isfinite(x.float()).all()
