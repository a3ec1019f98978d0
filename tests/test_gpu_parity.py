"""GPU (CUDA path, through the C ABI) against the CPU oracle on the same
seeded inputs.  Needs a B200; run with ``pytest -m gpu``."""
from __future__ import annotations

import pytest
import torch

import oracle
import hybrid_sparse_attention_tcgen05_b200 as hs
from hybrid_sparse_attention_tcgen05_b200 import inputs as gen
from parity import (check_out, check_scores, check_topk, gather_idx_rows, gather_rows, rows_for,
                    scale_of)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_stages(inp, w, row_chunk=None):
    """full_attn_scores (one chunk = all rows unless row_chunk) -> topk ->
    sparse layers, each through its own C-ABI call."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    shape = hs.shape_of(q, k)
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.Lq, w.topk, dtype=torch.int32, device=DEV)
    chunk = row_chunk or w.Lq
    scores_all = torch.empty(w.B, w.Hkv, w.Lq, w.Lkv, dtype=torch.float32, device=DEV) \
        if w.Lq * w.Lkv * w.B * w.Hkv <= (1 << 28) else None
    for r0 in range(0, w.Lq, chunk):
        rc = min(chunk, w.Lq - r0)
        _, _, sc = hs.full_attn_scores(q, k, v, row_begin=r0, row_count=rc, out=out, lse=lse)
        hs.topk(shape, sc, w.topk, row_begin=r0, idx=idx)
        if scores_all is not None:
            scores_all[:, :, r0:r0 + rc] = sc
    outs = [hs.sparse_attn(qs, k, v, idx, gt, w.window, want_branches=True)
            for qs, gt in zip(inp["q_sparse"], inp["gate"])]
    torch.cuda.synchronize()
    return out, lse, idx, scores_all, outs


def oracle_check_rows(inp, w, rows, out, lse, idx, scores_all, outs, check_own_idx=True):
    """Compare the listed rows against the oracle (full layer, scores, top-k,
    every sparse layer on the oracle's and on the GPU's own index sets)."""
    scale = scale_of(w.d)
    k_h, v_h = inp["k"].to("cpu"), inp["v"].to("cpu")
    qr = gather_rows(inp["q"], rows)
    o_out, o_lse, o_sc = oracle.full_rows(qr, k_h, v_h, rows, w.Lq, scale)
    check_out("full out", gather_rows(out, rows), o_out, w.dtype)
    b = torch.tensor([r[0] for r in rows])
    i = torch.tensor([r[1] for r in rows])
    g_lse = lse.to("cpu")[b, :, i]
    assert float((g_lse.double() - o_lse).abs().max()) <= 1e-4
    n_valid = [w.Lkv - w.Lq + r[1] + 1 for r in rows for _ in range(w.Hkv)]
    if scores_all is not None:
        g_sc = scores_all.to("cpu")[b, :, i].reshape(-1, w.Lkv)
        check_scores(g_sc, o_sc.reshape(-1, w.Lkv), n_valid)
    g_idx = gather_idx_rows(idx, rows)
    stats = check_topk(g_idx.reshape(-1, w.topk), o_sc.reshape(-1, w.Lkv), n_valid, w.topk)
    o_idx = oracle.topk_rows(o_sc.reshape(-1, w.Lkv), n_valid, w.topk).reshape(len(rows), w.Hkv, w.topk)
    for n, (qs, gt) in enumerate(zip(inp["q_sparse"], inp["gate"])):
        g_out, g_og, g_ol = outs[n]
        qsr, gtr = gather_rows(qs, rows), gather_rows(gt, rows)
        # on the GPU's own index sets
        r_out, r_og, r_ol = oracle.sparse_rows(qsr, k_h, v_h, rows, w.Lq, scale, g_idx, gtr, w.window)
        check_out(f"sparse{n} out (own idx)", gather_rows(g_out, rows), r_out, w.dtype)
        check_out(f"sparse{n} global (own idx)", gather_rows(g_og, rows), r_og, w.dtype)
        check_out(f"sparse{n} local", gather_rows(g_ol, rows), r_ol, w.dtype)
    return stats, o_idx


def check_sparse_on_oracle_idx(inp, w, rows, idx, o_idx, tag=""):
    """Run every sparse layer on the oracle's own index sets: the GPU index
    tensor with the sampled rows replaced by the oracle's sets (o_idx
    [nrows, Hkv, k]), one layer at a time, compared on those rows with the
    oracle's sparse layer over the same sets."""
    scale = scale_of(w.d)
    k_h, v_h = inp["k"].to("cpu"), inp["v"].to("cpu")
    b = torch.tensor([r[0] for r in rows], device=idx.device)
    i = torch.tensor([r[1] for r in rows], device=idx.device)
    idx_o = idx.clone()
    idx_o[b, :, i] = o_idx.to(idx.device, torch.int32)
    for n, (qs, gt) in enumerate(zip(inp["q_sparse"], inp["gate"])):
        g_out, g_og, g_ol = hs.sparse_attn(qs, inp["k"], inp["v"], idx_o, gt, w.window, want_branches=True)
        torch.cuda.synchronize()
        r_out, r_og, r_ol = oracle.sparse_rows(gather_rows(qs, rows), k_h, v_h, rows, w.Lq, scale, o_idx,
                                               gather_rows(gt, rows), w.window)
        check_out(f"{tag}sparse{n} out (oracle idx)", gather_rows(g_out, rows), r_out, w.dtype)
        check_out(f"{tag}sparse{n} global (oracle idx)", gather_rows(g_og, rows), r_og, w.dtype)
        check_out(f"{tag}sparse{n} local (oracle idx)", gather_rows(g_ol, rows), r_ol, w.dtype)
        del g_out, g_og, g_ol
    del idx_o


def sparse_on_indices(inp, w, idx_dev):
    return [hs.sparse_attn(qs, inp["k"], inp["v"], idx_dev, gt, w.window, want_branches=True)
            for qs, gt in zip(inp["q_sparse"], inp["gate"])]


# ---------------------------------------------------------------- tiny (fp32)

def _tiny_inputs():
    w = gen.WORKLOADS["tiny"]
    cpu = gen.make_inputs(w, seed=0, device="cpu")
    dev = {key: (val.to(DEV) if torch.is_tensor(val) else [x.to(DEV) for x in val])
           for key, val in cpu.items()}
    return w, dev


def test_tiny_all_rows():
    w, inp = _tiny_inputs()
    out, lse, idx, sc, outs = run_stages(inp, w)
    rows = rows_for(w.B, w.Lq, range(w.Lq))
    stats, o_idx = oracle_check_rows(inp, w, rows, out, lse, idx, sc, outs)
    # sparse layer on the oracle's index sets
    idx_o = torch.empty_like(idx)
    idx_o[0] = o_idx.permute(1, 0, 2).to(DEV)
    outs_o = sparse_on_indices(inp, w, idx_o)
    k_h, v_h = inp["k"].cpu(), inp["v"].cpu()
    for n, (qs, gt) in enumerate(zip(inp["q_sparse"], inp["gate"])):
        r_out, r_og, _ = oracle.sparse_rows(gather_rows(qs, rows), k_h, v_h, rows, w.Lq,
                                            scale_of(w.d), o_idx, gather_rows(gt, rows), w.window)
        check_out("sparse out (oracle idx)", gather_rows(outs_o[n][0], rows), r_out, w.dtype)
        check_out("sparse global (oracle idx)", gather_rows(outs_o[n][1], rows), r_og, w.dtype)


def test_tiny_block_matches_stages():
    w, inp = _tiny_inputs()
    out, lse, idx, _, outs = run_stages(inp, w)
    for chunk in (0, 100):
        of, lb, ib, ob = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], w.topk,
                                  w.window, row_chunk=chunk)
        torch.cuda.synchronize()
        assert torch.equal(ib, idx)
        assert torch.equal(of, out)
        assert torch.equal(lb, lse)
        for n in range(w.n_sparse):
            assert torch.equal(ob[n], outs[n][0])


def test_topk_stage_isolated_bit_exact():
    """The same fp32 score buffer through the GPU top-k and the oracle top-k:
    identical index lists, no tolerance band."""
    w, inp = _tiny_inputs()
    _, _, idx, sc, _ = run_stages(inp, w)
    n_valid = [w.Lkv - w.Lq + i + 1 for i in range(w.Lq)]
    o_idx = oracle.topk_rows(sc[0, 0].cpu(), n_valid, w.topk)
    assert torch.equal(idx[0, 0].cpu(), o_idx)


# Row lengths around which the top-k launch switches from rows cached in
# shared memory to rows read from global memory (and a few other lengths).
TOPK_BUCKET_EDGES = (9984, 25600)


@pytest.mark.parametrize("case", ["ties", "ties_unaligned", "all_equal", "zeros_and_denormals", "long_rows",
                                  "flat_narrow", "flat_long_unaligned", "many_rows_ties",
                                  "many_rows_ties_aligned", "rows_8192", "short_rows_between_long",
                                  "clustered", "clustered_wide", "unsampled_peaks", "uniform_8192"]
                         + [f"edge{e}" for e in TOPK_BUCKET_EDGES]
                         + [f"edge{e}_unaligned" for e in TOPK_BUCKET_EDGES])
@pytest.mark.parametrize("kernel", ["sampled", "block", "warp"])
def test_topk_synthetic_rows_bit_exact(case, kernel, monkeypatch):
    """Score rows built directly (not by the CUDA path), with exact ties,
    through every top-k kernel (sampled single pass / one CTA per row / one
    warp per row)."""
    monkeypatch.setenv("HYSPARSE_TOPK_PATH", kernel)
    g = torch.Generator().manual_seed(7)
    B, Hkv, Lq, Lkv, k = 2, 3, 37, 300, 29
    if case == "long_rows":
        Lq, Lkv, k = 5, 70000, 2048
    elif case.startswith("edge"):    # rows on both sides of a bucket edge
        e = int(case[4:].split("_")[0])
        B, Hkv, Lq, k = 1, 2, 40, 1000
        Lkv = e + 20 + (1 if case.endswith("unaligned") else 0)   # odd Lkv: rows not 16-byte aligned
    elif case == "flat_narrow":     # near-flat rows: every key in one coarse bin
        Lq, Lkv, k = 16, 20000, 1500
    elif case == "flat_long_unaligned":
        B, Hkv, Lq, Lkv, k = 1, 1, 6, 60001, 2048
    elif case == "ties_unaligned":
        Lkv = 301
    elif case == "many_rows_ties":   # enough rows for the one-warp-per-row kernel by default
        B, Hkv, Lq, Lkv, k = 1, 2, 2100, 2203, 150
    elif case == "many_rows_ties_aligned":   # 16-byte aligned rows, many per launch
        B, Hkv, Lq, Lkv, k = 1, 2, 2100, 2204, 150
    elif case == "rows_8192":        # the prefill8k row lengths at their longest
        B, Hkv, Lq, Lkv, k = 1, 2, 300, 8192, 1000
    elif case == "short_rows_between_long":   # rows with n <= k end every (b, g) block
        B, Hkv, Lq, Lkv, k = 2, 2, 1500, 1500, 700
    elif case.startswith("clustered"):   # the k-th key's bin holds more keys than the candidate list
        B, Hkv, Lq, Lkv, k = 1, 2, 2100, 3000, 900
    elif case == "unsampled_peaks":   # the largest keys all lie outside the sampled lines
        B, Hkv, Lq, Lkv, k = 1, 2, 64, 3000, 200
    elif case == "uniform_8192":      # distinct values: no ties, the sampled pass's common case
        B, Hkv, Lq, Lkv, k = 1, 2, 300, 8192, 1000
    s = torch.rand(B, Hkv, Lq, Lkv, generator=g)
    if case in ("ties", "ties_unaligned"):
        s = torch.round(s * 16) / 16
    elif case.startswith("many_rows_ties") or case in ("rows_8192", "short_rows_between_long"):
        s = torch.round(s * 512) / 512
    elif case == "all_equal":
        s[:] = 0.125
    elif case == "zeros_and_denormals":
        s = torch.where(s < 0.5, torch.zeros_like(s), s * 1e-39)
    elif case == "long_rows":
        s = torch.round(s * 4096) / 4096
    elif case.startswith("edge"):
        s = torch.round(s * 65536) / 65536
    elif case.startswith("flat"):
        s = (1.0 + 0.02 * s) / 8192.0
    elif case.startswith("clustered"):
        # 80 % of the keys within 2^9 (2^14) fp32 steps above 0.5, the rest uniform
        span = 2.0 ** (-15 if case == "clustered" else -10)
        c = 0.5 + span * torch.rand(s.shape, generator=g)
        s = torch.where(torch.rand(s.shape, generator=g) < 0.8, c, s)
    elif case == "unsampled_peaks":
        # the sampled select reads 32 lines of 32 keys starting at
        # floor((n - 32) q / 31); 1.5 k keys outside them get values above 1
        for i in range(Lq):
            n = Lkv - Lq + i + 1
            inside = torch.zeros(n, dtype=torch.bool)
            for q in range(32):
                st = (n - 32) * q // 31
                inside[st:st + 32] = True
            out = (~inside).nonzero().flatten()
            pick = out[torch.randperm(out.numel(), generator=g)[:3 * k // 2]]
            s[:, :, i, pick] += 1.0
    shape = hs.HsShape(B, Lq, Lkv, 4 * Hkv, Hkv, 128, 1, 0.0)
    idx = hs.topk(shape, s.to(DEV), k)
    n_valid = [Lkv - Lq + i + 1 for _ in range(B) for _ in range(Hkv) for i in range(Lq)]
    o_idx = oracle.topk_rows(s.reshape(-1, Lkv), n_valid, k).reshape(B, Hkv, Lq, k)
    assert torch.equal(idx.cpu(), o_idx)


@pytest.mark.parametrize("topk_path", ["sampled", "warp", "block"])
@pytest.mark.parametrize("Lkv", [1000, 8500])
def test_block_selection_mask_matches_stages(topk_path, Lkv, monkeypatch):
    """hysparse_block on the dense sparse path: with the one-warp-per-row
    top-k kernel the bitmask comes from the top-k pass itself, with the
    one-CTA-per-row kernel from a pass over the index lists; either way the
    outputs equal the stage calls' (whose sparse_attn builds the bitmask from
    the index lists)."""
    monkeypatch.setenv("HYSPARSE_SPARSE_PATH", "dense")
    monkeypatch.setenv("HYSPARSE_TOPK_PATH", topk_path)
    Lq = 1000 if Lkv == 1000 else 600     # the 8500 case: a row longer than 8192 keys
    w = gen.Workload("bf16_mask_block", 1, Lq, Lkv, 8, 2, 128, "bf16", 100, 64, 2, "shifted")
    inp = gen.make_inputs(w, seed=3, device=DEV)
    out, lse, idx, _, outs = run_stages(inp, w)
    of, lb, ib, ob = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"], w.topk, w.window)
    torch.cuda.synchronize()
    assert torch.equal(ib, idx)
    assert torch.equal(of, out)
    for n in range(w.n_sparse):
        assert torch.equal(ob[n], outs[n][0])


# ------------------------------------------------------------- shape sweep

SWEEP = [
    # name, B, Lq, Lkv, Hq, Hkv, d, dtype, topk, window, dist
    ("f32_ragged", 2, 77, 77, 4, 2, 64, "f32", 9, 5, "normal"),
    ("f32_chunked_prefix", 1, 40, 150, 8, 1, 128, "f32", 33, 16, "normal"),
    ("f32_decode", 3, 1, 300, 8, 2, 64, "f32", 64, 128, "normal"),
    ("f32_topk_ge_len", 1, 50, 50, 2, 2, 64, "f32", 64, 1, "normal"),
    ("bf16_small", 1, 300, 300, 8, 2, 128, "bf16", 64, 128, "shifted"),
    ("bf16_g16", 1, 200, 260, 32, 2, 128, "bf16", 100, 17, "shifted"),
    ("bf16_g1_ragged", 2, 129, 129, 2, 2, 128, "bf16", 1, 3, "normal"),
    ("bf16_decode", 4, 1, 1000, 32, 8, 128, "bf16", 128, 128, "normal"),
    ("bf16_decode_multichunk_g16", 3, 1, 2500, 32, 2, 128, "bf16", 200, 128, "normal"),
    ("bf16_decode_shifted_g4", 2, 1, 4097, 16, 4, 128, "bf16", 512, 128, "shifted"),
    ("bf16_window_ge_len", 1, 130, 130, 4, 1, 128, "bf16", 16, 1024, "shifted"),
    ("bf16_prefix_ragged", 2, 200, 333, 8, 2, 128, "bf16", 40, 100, "normal"),
    ("bf16_window_256", 1, 600, 600, 8, 4, 128, "bf16", 300, 256, "shifted"),
]


@pytest.fixture
def sparse_path(request, monkeypatch):
    """Force one sparse-layer kernel for the test: "dense" (dense-masked
    tcgen05 tiles), "gather" (warp-MMA row gather) or "gather_tc" (tcgen05
    row gather); None keeps the library's own choice."""
    monkeypatch.delenv("HYSPARSE_SPARSE_PATH", raising=False)
    monkeypatch.delenv("HYSPARSE_GATHER_KERNEL", raising=False)
    if request.param == "dense":
        monkeypatch.setenv("HYSPARSE_SPARSE_PATH", "dense")
    elif request.param in ("gather", "gather_tc"):
        monkeypatch.setenv("HYSPARSE_SPARSE_PATH", "gather")
        monkeypatch.setenv("HYSPARSE_GATHER_KERNEL", "tc" if request.param == "gather_tc" else "mma")
    return request.param


def _sweep_params():
    out = []
    for c in SWEEP:
        paths = [None]
        if c[7] == "bf16":
            paths = ["gather", "gather_tc"] + (["dense"] if c[2] >= 64 else [])
        for pth in paths:
            out.append(pytest.param(c, pth, id=f"{c[0]}-{pth or 'auto'}"))
    return out


@pytest.mark.parametrize("case,sparse_path", _sweep_params(), indirect=["sparse_path"])
def test_shape_sweep_all_rows(case, sparse_path):
    name, B, Lq, Lkv, Hq, Hkv, d, dt, topk, window, dist = case
    w = gen.Workload(name, B, Lq, Lkv, Hq, Hkv, d, dt, topk, window, 2, dist)
    cpu = gen.make_inputs(w, seed=3, device="cpu")
    inp = {key: (val.to(DEV) if torch.is_tensor(val) else [x.to(DEV) for x in val])
           for key, val in cpu.items()}
    out, lse, idx, sc, outs = run_stages(inp, w, row_chunk=max(1, Lq // 3))
    rows = rows_for(B, Lq, range(Lq))
    oracle_check_rows(inp, w, rows, out, lse, idx, sc, outs)


@pytest.mark.parametrize("sparse_path", ["dense", "gather", "gather_tc"], indirect=True)
def test_global_branch_far_below_unselected_keys(sparse_path):
    """Unselected keys whose logits sit ~200 (log2 units) above every selected
    key: a softmax reference taken over all keys would underflow every
    selected term to zero.  Both sparse kernels take the reference over the
    selected keys only and must give the exact global branch."""
    B, L, Hq, Hkv, d, topk, window = 1, 640, 8, 2, 128, 48, 32
    g = torch.Generator().manual_seed(11)
    k = torch.randn(B, L, Hkv, d, generator=g) / d ** 0.5
    v = torch.randn(B, L, Hkv, d, generator=g)
    qs = torch.randn(B, L, Hq, d, generator=g) / d ** 0.5
    trap = torch.arange(L) % 9 == 4                 # never selected, huge logits
    k[:, trap] = 0.0
    k[:, trap, :, 0] = 40.0
    qs[..., 0] = 40.0                               # q'.k = 1600 on trap keys
    gate = torch.randn(B, L, Hq, generator=g)
    idx = torch.full((B, Hkv, L, topk), -1, dtype=torch.int32)
    for gi in range(Hkv):
        for i in range(L):
            cand = torch.nonzero(~trap[: i + 1]).flatten()
            pick = cand[torch.randperm(len(cand), generator=g)[:topk]].sort().values
            idx[0, gi, i, : len(pick)] = pick.to(torch.int32)
    k, v, qs = (t.to(torch.bfloat16) for t in (k, v, qs))
    out, og, ol = hs.sparse_attn(qs.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), gate.to(DEV), window,
                                 want_branches=True)
    torch.cuda.synchronize()
    rows = rows_for(B, L, range(L))
    r_out, r_og, r_ol = oracle.sparse_rows(gather_rows(qs, rows), k, v, rows, L, scale_of(d),
                                           gather_idx_rows(idx, rows), gather_rows(gate, rows), window)
    check_out("global branch", gather_rows(og, rows), r_og, "bf16")
    check_out("local branch", gather_rows(ol, rows), r_ol, "bf16")
    check_out("out", gather_rows(out, rows), r_out, "bf16")


# ------------------------------------------------- full-size, sampled rows

FULL = [pytest.param("prefill8k", "gather", id="prefill8k-gather"),
        pytest.param("prefill8k", "dense", id="prefill8k-dense"),
        pytest.param("prefill32k", None, id="prefill32k-auto"),
        pytest.param("moe64k", None, id="moe64k-auto"),
        pytest.param("moe64k", "gather_tc", id="moe64k-gather_tc")]


@pytest.mark.parametrize("name,sparse_path", FULL, indirect=["sparse_path"])
def test_full_size_prefill_sampled_rows(name, sparse_path):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w, seed=0, device=DEV)
    chunk = 4096 if w.Lq > 8192 else w.Lq
    out, lse, idx, outs_list = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"],
                                        w.topk, w.window, row_chunk=chunk)[0:4]
    sp = [hs.sparse_attn(qs, inp["k"], inp["v"], idx, gt, w.window, want_branches=True)
          for qs, gt in zip(inp["q_sparse"], inp["gate"])]
    torch.cuda.synchronize()
    for n in range(w.n_sparse):
        assert torch.equal(sp[n][0], outs_list[n])
    n_rand = {"prefill8k": 96, "prefill32k": 48, "moe64k": 24}[name]
    rows = rows_for(w.B, w.Lq, gen.sample_rows(w.Lq, w.topk, w.window, n_random=n_rand, seed=0,
                                               edge=8))
    _, o_idx = oracle_check_rows(inp, w, rows, out, lse, idx, None, sp)
    del sp, outs_list
    # the same sparse kernels on the oracle's index sets for the sampled rows
    check_sparse_on_oracle_idx(inp, w, rows, idx, o_idx, tag=f"{name}: ")


@pytest.mark.parametrize("sparse_path", [None, "gather", "gather_tc"], indirect=True)
def test_full_size_decode_sampled_batches(sparse_path):
    w = gen.WORKLOADS["decode"]
    inp = gen.make_inputs(w, seed=0, device=DEV)
    out, lse, idx, outs_list = hs.block(inp["q"], inp["k"], inp["v"], inp["q_sparse"], inp["gate"],
                                        w.topk, w.window)
    sp = [hs.sparse_attn(qs, inp["k"], inp["v"], idx, gt, w.window, want_branches=True)
          for qs, gt in zip(inp["q_sparse"], inp["gate"])]
    torch.cuda.synchronize()
    picked = (0, 21, 42, 63)
    o_sets = []
    for b in picked:
        one = {"q": inp["q"][b:b + 1], "k": inp["k"][b:b + 1], "v": inp["v"][b:b + 1],
               "q_sparse": [x[b:b + 1] for x in inp["q_sparse"]],
               "gate": [x[b:b + 1] for x in inp["gate"]]}
        w1 = w.with_(B=1)
        _, o_idx = oracle_check_rows(one, w1, [(0, 0)], out[b:b + 1], lse[b:b + 1], idx[b:b + 1], None,
                                     [tuple(t[b:b + 1] for t in s) for s in sp])
        o_sets.append(o_idx[0])
    # the decode sparse kernels on the oracle's index sets of those sequences
    check_sparse_on_oracle_idx(inp, w, [(b, 0) for b in picked], idx, torch.stack(o_sets), tag="decode: ")
