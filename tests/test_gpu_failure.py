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
        hs.full_attn_scores(inp["q"], inp["k"], inp["v"], ws=ws)
        st = hs.workspace_status(ws)
    finally:
        if old is None:
            del os.environ["HYSPARSE_WAIT_LIMIT_NS"]
        else:
            os.environ["HYSPARSE_WAIT_LIMIT_NS"] = old
    assert st == _lib.HS_ERR_TIMEOUT
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


def test_polynomial_exp2_within_error_bound():
    """The FMA-pipe exponential the softmax kernels use for part of their
    elements (Remez degree-5 fit of 2^f after rounding x to an integer)
    against exact 2^x: relative error <= 3e-7 (the fit's fp32 bound is
    2.2e-7), exactly 0 below -125; the hardware ex2 is checked alongside."""
    import ctypes
    import numpy as np
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.linspace(-125.0, 12.0, 400001), torch.rand(100000, generator=g) * 30 - 20,
                   torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.999, -124.9999])]).float()
    xd = x.cuda()
    yp = torch.empty_like(xd)
    ym = torch.empty_like(xd)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _lib.lib().hysparse_selftest_exp2(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yp.data_ptr()),
                                          ctypes.c_void_p(ym.data_ptr()), xd.numel(), st)
    assert rc == _lib.HS_OK
    torch.cuda.synchronize()
    exact = np.exp2(x.double().numpy())
    rp = np.abs(yp.cpu().double().numpy() - exact) / exact
    rm = np.abs(ym.cpu().double().numpy() - exact) / exact
    assert rp.max() <= 3e-7, rp.max()
    assert rm.max() <= 5e-7, rm.max()
    xlow = torch.tensor([-126.0, -200.0, float("-inf")], device="cuda")
    ylow = torch.empty_like(xlow)
    ylm = torch.empty_like(xlow)
    _lib.lib().hysparse_selftest_exp2(ctypes.c_void_p(xlow.data_ptr()), ctypes.c_void_p(ylow.data_ptr()),
                                      ctypes.c_void_p(ylm.data_ptr()), 3, st)
    torch.cuda.synchronize()
    assert torch.all(ylow == 0)
