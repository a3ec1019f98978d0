"""Host-side accounting, pinned to figures the pages print (no GPU).

* KV cache: the HySparse abstract's 80B MoE model has 49 layers of which 5
  are full attention, and its KV cache is "nearly 10x" smaller, because only
  the full layers store K/V and their sparse layers reuse it (write-up
  section 3.1).  The binding's kv_cache_bytes must give 49/5 = 9.8 for that
  layout, and a little less when every sparse layer keeps its own 128-token
  window (write-up section 2.2).
* Tile arithmetic: the sparse-attention glossary page builds a FlexAttention
  block mask for 8192 tokens (causal, a 1024-token window plus 4 sink tokens)
  and prints that 85.47 % of its 128 x 128 blocks hold no allowed pair.  A
  brute-force tile counter reproduces that figure, and then checks the
  causal tile count that the bench's dense-or-gather estimate and its
  executed-FLOP figure use, and the per-row key counts (k_eff, w_eff) of the
  roofline's algorithmic bytes.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import hybrid_sparse_attention_tcgen05_b200 as hs  # noqa: E402
from hybrid_sparse_attention_tcgen05_b200 import inputs as gen  # noqa: E402


def model_kv(seq, own_window, blocks=(9, 9, 9, 9, 8)):
    """KV bytes of the 49-layer model: 5 hybrid blocks of one full layer and
    blocks[n] sparse layers (44 sparse layers in all); the MoE workload's
    attention shape (4 KV heads, d = 128, bf16)."""
    tot = dense = 0
    for n in blocks:
        r = hs.kv_cache_bytes(1, seq, 4, 128, 2, n, 128, own_window=own_window)
        tot += r["total"]
        dense += r["dense_equivalent"]
    return tot, dense


def test_kv_cache_reduction_matches_the_abstract():
    blocks = (9, 9, 9, 9, 8)
    assert len(blocks) + sum(blocks) == 49        # 5 full layers, 44 sparse
    tot, dense = model_kv(65536, own_window=False)
    assert dense / tot == pytest.approx(49 / 5, rel=1e-12)     # "nearly 10x"
    # own 128-token windows in the 44 sparse layers: 5 + 44 * 128 / L layer-equivalents
    tot_w, dense_w = model_kv(65536, own_window=True)
    assert dense_w == dense
    assert dense_w / tot_w == pytest.approx(49 / (5 + 44 * 128 / 65536), rel=1e-12)
    assert 9.6 < dense_w / tot_w < 49 / 5


def nonempty_tiles(allowed, L, block=128):
    """Brute force: tiles (qb, kb) of an L x L mask that hold an allowed pair."""
    q = np.arange(L)[:, None]
    kv = np.arange(L)[None, :]
    m = allowed(q, kv)
    nb = L // block
    return m.reshape(nb, block, nb, block).any(axis=(1, 3))


def test_block_sparsity_of_the_glossary_mask():
    seq_len, window, sinks = 8192, 1024, 4

    def local_plus_sinks(q, kv):
        return (q >= kv) & ((q - kv <= window) | (kv < sinks))

    t = nonempty_tiles(local_plus_sinks, seq_len)
    assert round(100.0 * (1.0 - t.sum() / t.size), 2) == 85.47
    # the same count in closed form: 9 live diagonals and the sink column
    assert t.sum() == sum(64 - d for d in range(9)) + (64 - 9)


@pytest.mark.parametrize("Lq,Lkv", [(1024, 1024), (1000, 1000), (640, 2048), (129, 300), (64, 64), (200, 4097)])
def test_causal_tile_count(Lq, Lkv):
    block = 128
    off = Lkv - Lq
    rows = np.arange(((Lq + block - 1) // block) * block)[:, None]
    keys = np.arange(((Lkv + block - 1) // block) * block)[None, :]
    allowed = (rows < Lq) & (keys <= off + rows) & (keys < Lkv)
    nq, nk = rows.shape[0] // block, keys.shape[1] // block
    t = allowed.reshape(nq, block, nk, block).any(axis=(1, 3))
    assert bench.causal_tiles(Lq, Lkv, block) == int(t.sum())


@pytest.mark.parametrize("name", ["tiny", "prefill8k", "decode"])
def test_key_counts_of_the_roofline(name):
    w = gen.workload(name)
    pos = w.Lkv - w.Lq + np.arange(w.Lq)
    assert bench.sum_min(w, w.topk) == int(np.minimum(pos + 1, w.topk).sum())
    assert bench.sum_min(w, w.window) == int(np.minimum(pos + 1, w.window).sum())
    assert bench.pairs_causal(w) == int((pos + 1).sum())
