"""Decode over caches of different lengths (hysparse_block_varlen) on the
GPU: every sequence must get exactly what a fixed-length decode over its own
cache gives, and match the oracle; lengths outside [1, Lkv] are reported
through the workspace status word without any read outside the cache."""
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
