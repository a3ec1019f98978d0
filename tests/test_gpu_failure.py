"""Failure detection on the GPU without faulting it: every barrier wait in
the tensor-core kernels is bounded.  With the bound forced to zero the kernel
gives up at its first wait that is not already satisfied, drains its own
copies and MMAs, frees its tensor memory, records HS_ERR_TIMEOUT in the
workspace status word and returns; the context stays usable."""
import os

import pytest
import torch

import hybrid_sparse_attention_tcgen05_b200 as hs
from hybrid_sparse_attention_tcgen05_b200 import _lib, inputs as gen

pytestmark = pytest.mark.gpu


def test_zero_wait_limit_reports_timeout_and_context_survives():
    w = gen.Workload("t", 1, 512, 512, 8, 2, 128, "bf16", 64, 128, 0, "shifted")
    inp = gen.make_inputs(w, seed=1, device="cuda")
    shape = hs.shape_of(inp["q"], inp["k"])
    ws = hs.alloc_workspace(shape, 64, 128, 0, 0, "cuda")
    old = os.environ.get("HYSPARSE_WAIT_LIMIT_NS")
    os.environ["HYSPARSE_WAIT_LIMIT_NS"] = "0"
    try:
        _, lse_to, _ = hs.full_attn_scores(inp["q"], inp["k"], inp["v"], ws=ws)
        st = hs.workspace_status(ws)
    finally:
        if old is None:
            del os.environ["HYSPARSE_WAIT_LIMIT_NS"]
        else:
            os.environ["HYSPARSE_WAIT_LIMIT_NS"] = old
    assert st == _lib.HS_ERR_TIMEOUT
    assert torch.isnan(lse_to).any()      # the rows it gave up on are marked in the caller's lse
    # status word was cleared; a normal call now succeeds and reports OK
    out, lse, sc = hs.full_attn_scores(inp["q"], inp["k"], inp["v"], ws=ws)
    assert hs.workspace_status(ws) == _lib.HS_OK
    assert torch.isfinite(out.float()).all()


def test_invalid_index_is_reported_not_read():
    w = gen.Workload("t", 1, 64, 64, 4, 1, 128, "bf16", 8, 16, 1, "normal")
    inp = gen.make_inputs(w, seed=2, device="cuda")
    idx = torch.full((1, 1, 64, 8), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, :, 0] = 0
    idx[0, 0, 10, 1] = 1000000      # far outside the cache
    idx[0, 0, 11, 1] = 40           # beyond row 11's causal position
    shape = hs.shape_of(inp["q"], inp["k"])
    ws = hs.alloc_workspace(shape, 8, 16, 1, 0, "cuda")
    out = hs.sparse_attn(inp["q_sparse"][0], inp["k"], inp["v"], idx, inp["gate"][0], 16, ws=ws)
    assert hs.workspace_status(ws) == _lib.HS_ERR_INVALID_INDEX
    assert torch.isfinite(out.float()).all()
