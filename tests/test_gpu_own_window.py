"""Sparse layers whose local branch reads the layer's own window K/V
(HySparse write-up, section 2.2: the global branch runs on the KV cache the
full layer shares; the local branch keeps its own sliding window), through
hysparse_sparse_attn_own_window, against the oracle on the same seeded
inputs.  The index sets are seeded host draws, so every oracle input is
independent of the CUDA path."""
from __future__ import annotations

import pytest
import torch

import oracle
import hybrid_sparse_attention_tcgen05_b200 as hs
from hybrid_sparse_attention_tcgen05_b200 import inputs as gen
from parity import check_out, gather_idx_rows, gather_rows, max_abs, rows_for, scale_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture
def sparse_path(request, monkeypatch):
    """"dense" or "gather" forces that sparse-layer path (an own window that
    the dense pipeline cannot read falls back to the gather by itself); None
    keeps the library's choice."""
    monkeypatch.delenv("HYSPARSE_SPARSE_PATH", raising=False)
    monkeypatch.delenv("HYSPARSE_GATHER_KERNEL", raising=False)
    if request.param is not None:
        monkeypatch.setenv("HYSPARSE_SPARSE_PATH", request.param)
    return request.param


def _setup(w: gen.Workload, lwin: int, seed: int):
    cpu = gen.make_inputs(w, seed=seed, device="cpu")
    kw, vw = gen.make_window_kv(w, lwin, seed=seed + 100)
    idx = gen.random_index_sets(w.B, w.Hkv, w.Lq, w.Lkv, w.topk, seed=seed + 200)
    return cpu, kw, vw, idx


def _check(w, cpu, kw, vw, idx, rows, got, tag):
    scale = scale_of(w.d)
    qsr = gather_rows(cpu["q_sparse"][0], rows)
    gtr = gather_rows(cpu["gate"][0], rows)
    ir = gather_idx_rows(idx, rows)
    r_out, r_og, r_ol = oracle.sparse_rows(qsr, cpu["k"], cpu["v"], rows, w.Lq, scale, ir, gtr, w.window,
                                           k_win=kw, v_win=vw)
    g_out, g_og, g_ol = got
    check_out(f"{tag} out", gather_rows(g_out, rows), r_out, w.dtype)
    check_out(f"{tag} global", gather_rows(g_og, rows), r_og, w.dtype)
    check_out(f"{tag} local", gather_rows(g_ol, rows), r_ol, w.dtype)
    # the local branch really changed: the shared-cache window gives another result
    _, _, s_ol = oracle.sparse_rows(qsr, cpu["k"], cpu["v"], rows, w.Lq, scale, ir, gtr, w.window)
    assert max_abs(s_ol, r_ol) > 10 * max_abs(gather_rows(g_ol, rows), r_ol)


def _run(w, cpu, kw, vw, idx):
    q = cpu["q_sparse"][0].to(DEV)
    out = hs.sparse_attn(q, cpu["k"].to(DEV), cpu["v"].to(DEV), idx.to(DEV), cpu["gate"][0].to(DEV), w.window,
                         want_branches=True, k_win=kw.to(DEV), v_win=vw.to(DEV))
    torch.cuda.synchronize()
    return out


# (name, B, Lq, Lkv, Hq, Hkv, d, dtype, topk, window, lwin): lwin None = Lkv
CASES = [
    ("prefill_g4", 1, 600, 600, 8, 2, 128, "bf16", 64, 128, None),     # dense pair pipeline or gather
    ("prefill_g3", 1, 400, 400, 6, 2, 128, "bf16", 64, 128, None),     # odd ratio: gather even when dense forced
    ("prefill_g16", 1, 300, 300, 16, 1, 128, "bf16", 48, 128, None),
    ("chunk_tail", 2, 64, 1000, 8, 2, 128, "bf16", 96, 128, 191),     # last 64 rows, buffer = window + 63
    ("chunk_longer", 1, 100, 700, 8, 4, 128, "bf16", 64, 200, 450),   # buffer longer than needed
    ("decode", 3, 1, 1000, 8, 2, 128, "bf16", 128, 128, 128),          # ring of exactly the window
    ("fp32_d64", 2, 150, 150, 4, 2, 64, "f32", 32, 48, None),
    ("fp32_tail", 1, 40, 300, 4, 1, 128, "f32", 32, 64, 103),
    ("fp32_decode", 2, 1, 300, 8, 2, 64, "f32", 64, 48, 48),
]


@pytest.mark.parametrize("sparse_path", [None, "dense", "gather"], indirect=True)
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_own_window_matches_oracle_all_rows(case, sparse_path):
    name, B, Lq, Lkv, Hq, Hkv, d, dt, topk, window, lwin = case
    if sparse_path == "dense" and (dt != "bf16" or Lq < 64):
        pytest.skip("no dense path for this shape")
    w = gen.Workload(name, B, Lq, Lkv, Hq, Hkv, d, dt, topk, window, 1, "shifted" if Lq > 1 else "normal")
    cpu, kw, vw, idx = _setup(w, lwin or Lkv, seed=11)
    got = _run(w, cpu, kw, vw, idx)
    _check(w, cpu, kw, vw, idx, rows_for(B, Lq, range(Lq)), got, f"{name}/{sparse_path or 'auto'}")


@pytest.mark.parametrize("sparse_path", [None, "dense", "gather"], indirect=True)
def test_own_window_equal_to_shared_cache_is_bit_identical(sparse_path):
    """k_win = k, v_win = v over the whole cache is the plain sparse layer."""
    w = gen.Workload("same", 1, 520, 520, 8, 2, 128, "bf16", 64, 128, 1, "shifted")
    cpu = gen.make_inputs(w, seed=4, device=DEV)
    idx = gen.random_index_sets(1, 2, 520, 520, 64, seed=5).to(DEV)
    q, k, v, gt = cpu["q_sparse"][0], cpu["k"], cpu["v"], cpu["gate"][0]
    a = hs.sparse_attn(q, k, v, idx, gt, w.window, want_branches=True)
    b = hs.sparse_attn(q, k, v, idx, gt, w.window, want_branches=True, k_win=k, v_win=v)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_own_window_full_size_decode_sampled():
    """A decode step with the decode workload's cache length (32K), heads and
    top-k, on 4 of its 64 sequences, with a window ring of 128 rows; every
    sequence checked."""
    w = gen.workload("decode", B=4, n_sparse=1)
    cpu, kw, vw, idx = _setup(w, 128, seed=21)
    got = _run(w, cpu, kw, vw, idx)
    _check(w, cpu, kw, vw, idx, rows_for(w.B, 1, [0]), got, "decode32k_own")


def test_own_window_rejects_short_buffer():
    w = gen.Workload("short", 1, 64, 1000, 8, 2, 128, "bf16", 64, 128, 1, "normal")
    cpu, kw, vw, idx = _setup(w, 190, seed=3)             # needs 64 + 127 = 191 rows
    with pytest.raises(hs._lib.HysparseError) as e:
        _run(w, cpu, kw, vw, idx)
    assert e.value.status == hs._lib.HS_ERR_INVALID_ARG


@pytest.mark.parametrize("sparse_path", ["dense", "gather"], indirect=True)
def test_own_window_full_size_prefill_sampled(sparse_path):
    """The prefill8k workload (8192 tokens, 32/8 heads, top-k 1024) with a
    whole-cache window buffer, on both sparse paths; sampled rows (both ends,
    the top-k and window edges, random rows) against the oracle."""
    w = gen.workload("prefill8k", n_sparse=1)
    cpu, kw, vw, idx = _setup(w, w.Lkv, seed=31)
    got = _run(w, cpu, kw, vw, idx)
    rows = rows_for(w.B, w.Lq, gen.sample_rows(w.Lq, w.topk, w.window, n_random=128, seed=31))
    _check(w, cpu, kw, vw, idx, rows, got, f"prefill8k_own/{sparse_path}")


# (name, B, Lq, Lkv, Hq, Hkv, topk, window, lwin, n_sparse, sparse_path)
BLOCK_CASES = [
    ("prefill_dense", 1, 600, 600, 8, 2, 64, 128, 600, 3, "dense"),
    ("prefill_gather", 1, 600, 600, 8, 2, 64, 128, 600, 3, "gather"),
    ("prefill_auto_g3", 1, 400, 400, 6, 2, 64, 128, 400, 2, None),
    ("chunk_tail", 2, 64, 1000, 8, 2, 96, 128, 191, 2, None),
    ("decode_ring", 4, 1, 2000, 32, 8, 256, 128, 128, 3, None),
]


@pytest.mark.parametrize("case", BLOCK_CASES, ids=[c[0] for c in BLOCK_CASES])
def test_block_own_window_equals_layer_calls(case, monkeypatch):
    """hysparse_block_own_window: the full layer and index set of the plain
    block, and every sparse layer equal to hysparse_sparse_attn_own_window on
    that index set, bit for bit."""
    name, B, Lq, Lkv, Hq, Hkv, topk, window, lwin, n_sparse, path = case
    monkeypatch.delenv("HYSPARSE_SPARSE_PATH", raising=False)
    if path is not None:
        monkeypatch.setenv("HYSPARSE_SPARSE_PATH", path)
    w = gen.Workload(name, B, Lq, Lkv, Hq, Hkv, 128, "bf16", topk, window, n_sparse,
                     "shifted" if Lq > 1 else "normal")
    inp = gen.make_inputs(w, seed=41, device=DEV)
    wins = [gen.make_window_kv(w, lwin, seed=500 + n, device=DEV) for n in range(n_sparse)]
    kw, vw = [x[0] for x in wins], [x[1] for x in wins]
    of, lse, idx, outs = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], topk, window,
                                  k_win=kw, v_win=vw)
    pf, plse, pidx, _ = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], topk, window)
    torch.cuda.synchronize()
    assert torch.equal(idx, pidx) and torch.equal(of, pf) and torch.equal(lse, plse)
    for n in range(n_sparse):
        ref = hs.sparse_attn(inp["q_sparse"][n], inp["k"], inp["v"], idx, inp["gate"][n], window,
                             k_win=kw[n], v_win=vw[n])
        torch.cuda.synchronize()
        assert torch.equal(outs[n], ref), f"layer {n}"
