"""The allocation-free full-layer entry point, called through the C ABI.

hysparse_full_attn_scores_noalloc serves callers that cannot allocate device
memory (a process whose memory pool is frozen, a plug-in host that only lends
its input and output buffers): its scratch lives in a fixed device array in
the library instead of a caller workspace.  It runs the same kernels as the
workspace entry point on the same inputs, so its results must be
bit-identical to that entry point's, on two calls in a row (the array keeps
the previous call's contents).  Shapes that need more scratch than the array
holds are refused before anything runs; that is checked without a GPU in
test_abi.py.

This file is collected last so that a failure here cannot hide any other
test's result in a run that stops at the first failure."""
import ctypes
import os

import pytest
import torch

import hybrid_sparse_attention_tcgen05_b200 as hs
from hybrid_sparse_attention_tcgen05_b200 import _lib, inputs as gen

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(shape, q, k, v, out, lse, scores, row_begin, row_count):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ld = scores.shape[-1] if scores is not None else 0
    return _lib.lib().hysparse_full_attn_scores_noalloc(
        ctypes.byref(shape), _p(q), _p(k), _p(v), _p(out), _p(lse), _p(scores), ld, row_begin,
        row_count, stream)


# (B, Lq, Lkv, Hq, Hkv, row_begin, row_count): prefill on the tensor-core
# path (whole and part of the rows), and a decode step (Lq = 1), whose split-K
# partials and logit stash also live in the array
CASES = [pytest.param(1, 1000, 1000, 8, 2, 0, 1000, id="prefill-all-rows"),
         pytest.param(1, 1000, 1000, 8, 2, 384, 500, id="prefill-row-chunk"),
         pytest.param(2, 1, 1000, 8, 2, 0, 1, id="decode")]


@pytest.mark.parametrize("B,Lq,Lkv,Hq,Hkv,row_begin,row_count", CASES)
def test_noalloc_matches_workspace_entry_point_twice(B, Lq, Lkv, Hq, Hkv, row_begin, row_count):
    w = gen.Workload("noalloc", B, Lq, Lkv, Hq, Hkv, 128, "bf16", 64, 128, 0,
                     "normal" if Lq == 1 else "shifted")
    inp = gen.make_inputs(w, seed=5, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    shape = hs.shape_of(q, k)
    ref_out, ref_lse, ref_sc = hs.full_attn_scores(q, k, v, row_begin=row_begin, row_count=row_count)
    torch.cuda.synchronize()
    rows = slice(row_begin, row_begin + row_count)
    pos = torch.arange(row_begin, row_begin + row_count, device="cuda") + (Lkv - Lq)
    valid = torch.arange(Lkv, device="cuda")[None, :] <= pos[:, None]      # causal entries
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, Lq), float("nan"), device="cuda")
        sc = torch.full((B, Hkv, row_count, Lkv), float("nan"), device="cuda")
        assert _call(shape, q, k, v, out, lse, sc, row_begin, row_count) == _lib.HS_OK
        torch.cuda.synchronize()
        assert torch.equal(out[:, rows], ref_out[:, rows])
        assert torch.equal(lse[:, :, rows], ref_lse[:, :, rows])
        for b in range(B):
            for g in range(Hkv):
                assert torch.equal(sc[b, g][valid], ref_sc[b, g][valid])


def test_noalloc_timeout_marks_lse_nan_and_next_call_is_exact():
    """The status word in the array cannot be read through the API, so a wait
    that gives up inside a kernel shows as NaN in the caller's lse rows; a
    following call with the normal bound gives the exact result again."""
    w = gen.Workload("noalloc_to", 1, 512, 512, 8, 2, 128, "bf16", 64, 128, 0, "shifted")
    inp = gen.make_inputs(w, seed=6, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    shape = hs.shape_of(q, k)
    ref_out, ref_lse, _ = hs.full_attn_scores(q, k, v)
    torch.cuda.synchronize()
    out = torch.empty_like(q)
    lse = torch.zeros(1, 8, 512, device="cuda")
    sc = torch.empty(1, 2, 512, 512, device="cuda")
    old = os.environ.get("HYSPARSE_WAIT_LIMIT_NS")
    os.environ["HYSPARSE_WAIT_LIMIT_NS"] = "0"
    try:
        assert _call(shape, q, k, v, out, lse, sc, 0, 512) == _lib.HS_OK
        torch.cuda.synchronize()
    finally:
        if old is None:
            del os.environ["HYSPARSE_WAIT_LIMIT_NS"]
        else:
            os.environ["HYSPARSE_WAIT_LIMIT_NS"] = old
    assert torch.isnan(lse).any()
    assert _call(shape, q, k, v, out, lse, sc, 0, 512) == _lib.HS_OK
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)
