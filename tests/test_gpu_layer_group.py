"""hysparse_block's sparse layers as one gather launch (the layers share the
index set and the cache: write-up section 3.1).  Every (item, layer) warp
runs the same code as a single-layer launch, so the block's sparse outputs
must equal the per-layer hysparse_sparse_attn calls on the block's own index
set bit for bit."""
from __future__ import annotations

import pytest
import torch

import hybrid_sparse_attention_tcgen05_b200 as hs
from hybrid_sparse_attention_tcgen05_b200 import inputs as gen

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _block_vs_layers(w, seed, kv_len=None):
    inp = gen.make_inputs(w, seed=seed, device=DEV)
    q, k, v = inp["q"], inp["k"], inp["v"]
    of, lse, idx, outs = hs.block(q, k, v, inp["q_sparse"], inp["gate"], w.topk, w.window, kv_len=kv_len)
    torch.cuda.synchronize()
    for n in range(w.n_sparse):
        if kv_len is None:
            ref = hs.sparse_attn(inp["q_sparse"][n], k, v, idx, inp["gate"][n], w.window)
        else:
            # one sequence at a time: sequence b's cache is its first kv_len[b] rows
            ref = torch.empty_like(outs[n])
            for b in range(w.B):
                L = int(kv_len[b])
                ref[b:b + 1] = hs.sparse_attn(inp["q_sparse"][n][b:b + 1], k[b:b + 1, :L].contiguous(),
                                              v[b:b + 1, :L].contiguous(), idx[b:b + 1], inp["gate"][n][b:b + 1],
                                              w.window)
        torch.cuda.synchronize()
        assert torch.equal(outs[n], ref), f"layer {n}"


@pytest.mark.parametrize("Hq,Hkv,n_sparse", [(32, 8, 3), (32, 2, 3), (16, 4, 5), (8, 8, 2)])
def test_decode_layer_group_equals_single_layers(Hq, Hkv, n_sparse, monkeypatch):
    monkeypatch.delenv("HYSPARSE_LAYER_GROUP", raising=False)
    w = gen.Workload("dec_group", 6, 1, 3000, Hq, Hkv, 128, "bf16", 256, 128, n_sparse, "normal")
    _block_vs_layers(w, seed=7)


def test_decode_layer_group_mixed_lengths(monkeypatch):
    monkeypatch.delenv("HYSPARSE_LAYER_GROUP", raising=False)
    w = gen.Workload("dec_group_vl", 5, 1, 2000, 32, 8, 128, "bf16", 300, 128, 3, "normal")
    kv_len = torch.tensor([1, 129, 700, 1999, 2000], dtype=torch.int32, device=DEV)
    _block_vs_layers(w, seed=8, kv_len=kv_len)


def test_prefill_layer_group_when_forced(monkeypatch):
    monkeypatch.setenv("HYSPARSE_LAYER_GROUP", "1")
    monkeypatch.setenv("HYSPARSE_SPARSE_PATH", "gather")
    w = gen.Workload("pre_group", 1, 700, 700, 32, 2, 128, "bf16", 100, 128, 3, "shifted")
    _block_vs_layers(w, seed=9)


def test_decode_layer_group_full_size(monkeypatch):
    """The decode workload itself (64 sequences, 32768-token caches, 32/8 heads,
    top-k 2048, 3 sparse layers): the grouped launch that the bench times
    equals the per-layer calls bit for bit."""
    monkeypatch.delenv("HYSPARSE_LAYER_GROUP", raising=False)
    _block_vs_layers(gen.workload("decode"), seed=10)
