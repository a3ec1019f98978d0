"""CPU oracle against its pins (library special cases, closed forms,
invariants, brute force).  No GPU needed."""
import pytest
import torch

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    oracle.use_library(None)
    pin()


def test_malformed_index_lists_rejected():
    k = torch.randn(1, 8, 1, 4)
    v = torch.randn(1, 8, 1, 4)
    q = torch.randn(1, 1, 4)
    gate = torch.zeros(1, 1)
    rows = [(0, 7)]
    bad = [
        [3, 2, -1],      # not ascending
        [2, 2, -1],      # duplicate
        [1, -1, 4],      # key after padding
        [0, 9, -1],      # beyond the causal position (pos = 7)
        [-5, 1, 2],      # negative other than -1
    ]
    for lst in bad:
        idx = torch.tensor([[lst]], dtype=torch.int32)
        with pytest.raises(ValueError):
            oracle.sparse_rows(q, k, v, rows, 8, 0.5, idx, gate, 2)


def test_empty_global_set_is_zero():
    k = torch.randn(1, 8, 1, 4)
    v = torch.randn(1, 8, 1, 4)
    q = torch.randn(1, 1, 4)
    idx = torch.full((1, 1, 3), -1, dtype=torch.int32)
    out, og, ol = oracle.sparse_rows(q, k, v, [(0, 5)], 8, 0.5, idx, torch.zeros(1, 1), 2)
    assert torch.all(og == 0)
    assert torch.allclose(out, 0.5 * ol)


def test_bad_shapes_rejected():
    k = torch.randn(1, 8, 2, 4)
    with pytest.raises(ValueError):
        oracle.full_rows(torch.randn(1, 3, 4), k, k, [(0, 0)], 8, 0.5)   # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.full_rows(torch.randn(1, 4, 4), k, k, [(0, 9)], 8, 0.5)   # row out of range
    with pytest.raises(ValueError):
        oracle.full_rows(torch.randn(1, 4, 4), k, k, [(0, 0)], 9, 0.5)   # Lq > Lkv


def test_own_window_buffer_must_cover_every_window():
    """The own-window variant reads positions Lkv - Lwin .. Lkv - 1 only: a row
    whose window starts below that is an argument error, not a silent read."""
    k = torch.randn(1, 8, 1, 4)
    q = torch.randn(1, 1, 4)
    idx = torch.full((1, 1, 2), -1, dtype=torch.int32)
    kw = torch.randn(1, 3, 1, 4)
    # row 0 of Lq = 1: pos 7, window 3 -> keys 5..7, inside a 3-row tail buffer
    oracle.sparse_rows(q, k, k, [(0, 0)], 1, 0.5, idx, torch.zeros(1, 1), 3, k_win=kw, v_win=kw)
    with pytest.raises(ValueError):   # window 4 reaches key 4, below the buffer
        oracle.sparse_rows(q, k, k, [(0, 0)], 1, 0.5, idx, torch.zeros(1, 1), 4, k_win=kw, v_win=kw)
