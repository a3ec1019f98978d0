"""The allocation-free full-layer entry point, called through the C ABI.

hysparse_full_attn_scores_noalloc serves callers that cannot allocate device
memory (a process whose memory pool is frozen, a plug-in host that only lends
its input and output buffers): its scratch lives in a fixed device array in
the library instead of a caller workspace.  Its results must match the
workspace entry point's, on two calls in a row (the array keeps the previous
call's contents), and shapes that need more scratch than the array holds are
refused before anything runs.

This file is collected last so that a failure here cannot hide any other
test's result in a run that stops at the first failure."""
import ctypes

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


@pytest.mark.parametrize("row_begin,row_count", [(0, 1000), (384, 500)])
def test_noalloc_matches_workspace_entry_point_twice(row_begin, row_count):
    w = gen.Workload("noalloc", 1, 1000, 1000, 8, 2, 128, "bf16", 64, 128, 0, "shifted")
    inp = gen.make_inputs(w, seed=5, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    shape = hs.shape_of(q, k)
    ref_out, ref_lse, ref_sc = hs.full_attn_scores(q, k, v, row_begin=row_begin, row_count=row_count)
    torch.cuda.synchronize()
    rows = slice(row_begin, row_begin + row_count)
    pos = torch.arange(row_begin, row_begin + row_count, device="cuda")
    valid = torch.arange(w.Lkv, device="cuda")[None, :] <= pos[:, None]      # causal entries
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.B, w.Hq, w.Lq), float("nan"), device="cuda")
        sc = torch.full((w.B, w.Hkv, row_count, w.Lkv), float("nan"), device="cuda")
        assert _call(shape, q, k, v, out, lse, sc, row_begin, row_count) == _lib.HS_OK
        torch.cuda.synchronize()
        assert float((out[:, rows].float() - ref_out[:, rows].float()).abs().max()) <= 2e-2
        assert float((lse[:, :, rows] - ref_lse[:, :, rows]).abs().max()) <= 1e-4
        for g in range(w.Hkv):
            a, b = sc[0, g][valid], ref_sc[0, g][valid]
            assert float((a - b).abs().max() / b.max()) <= 2e-5


def test_noalloc_rejects_scratch_beyond_its_array():
    # 8 bytes of statistics per (batch, query head, row): 64 * 65536 * 8 B > 16 MiB
    shape = _lib.HsShape(1, 65536, 65536, 64, 4, 128, _lib.HS_BF16, 0.0)
    A = 0x7f0000000000
    P = lambda i: ctypes.c_void_p(A + (i << 32))
    rc = _lib.lib().hysparse_full_attn_scores_noalloc(ctypes.byref(shape), P(1), P(2), P(3), P(4), P(5),
                                                      None, 0, 0, 65536, None)
    assert rc == _lib.HS_ERR_WORKSPACE
