"""The Python binding refuses, before any library call, caller tensors that would hand a
kernel memory of the wrong device, shape or type (no GPU needed: 'meta' tensors stand in for
another device)."""

import pytest
import torch

import exact_io_aware_77_b200 as fa


def _q():
    return torch.empty(1, 2, 8, 64, dtype=torch.bfloat16)


def test_like_checks():
    q = _q()
    fa._check_like(torch.empty_like(q), q, "out")
    fa._check_like(torch.empty(1, 8, 2, 64, dtype=torch.bfloat16).transpose(1, 2), q, "out")   # strided is fine
    for bad in (torch.empty(1, 2, 8, 64, dtype=torch.float16),              # dtype
                torch.empty(1, 2, 9, 64, dtype=torch.bfloat16),             # shape
                torch.empty(1, 2, 64, 8, dtype=torch.bfloat16).transpose(2, 3),   # d not contiguous
                torch.empty(1, 2, 8, 64, dtype=torch.bfloat16, device="meta")):   # device
        with pytest.raises(ValueError):
            fa._check_like(bad, q, "out")


def test_lse_checks():
    q = _q()
    fa._check_lse(torch.empty(1, 2, 8), q, 16)
    for bad in (torch.empty(1, 2, 8, dtype=torch.float64), torch.empty(1, 2, 9), torch.empty(2, 8).t(),
                torch.empty(1, 2, 8, device="meta")):
        with pytest.raises(ValueError):
            fa._check_lse(bad, q, 16)


def test_workspace_checks():
    q = _q()
    fa._check_workspace(torch.empty(100, dtype=torch.uint8), q)
    for bad in (torch.empty(100, dtype=torch.uint8, device="meta"), torch.empty(10, 10, dtype=torch.uint8).t()):
        with pytest.raises(ValueError):
            fa._check_workspace(bad, q)


def test_decode_workspace_size_argument_checks():
    for args in ((1, 8, 0, 1, 10, 64), (1, 8, 3, 1, 10, 64), (1, 8, 2, 11, 10, 64), (1, 8, 2, 1, 10, 96),
                 (0, 8, 2, 1, 10, 64)):
        with pytest.raises(ValueError):
            fa.decode_workspace_size(*args)
