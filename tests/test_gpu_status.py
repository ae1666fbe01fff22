"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies gives up, the status word reports it, and the context stays
usable (the next call runs and the status is clear again)."""
import pytest
import torch

from channel_decay_softmax_b200 import _lib as L
from channel_decay_softmax_b200 import api

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert L.wall_get_status() == L.WALL_OK
    L.wall_selftest_wait_timeout(2000)          # 2 ms limit
    assert L.wall_get_status() == L.WALL_ERR_TIMEOUT
    assert L.wall_get_status() == L.WALL_OK     # read-and-clear
    g = torch.randn(1, 64, 2, 64, device="cuda")
    P = api.prefix_cumsum(g)
    torch.cuda.synchronize()
    assert torch.isfinite(P).all()
    assert L.wall_get_status() == L.WALL_OK


def test_bad_cu_seqlens_reported_not_faulted():
    """A malformed cu_seqlens (decreasing, wrong end) is clamped by the
    kernels and reported through the status word."""
    g = torch.randn(1, 100, 2, 64, device="cuda")
    cu = torch.tensor([0, 60, 40, 120], dtype=torch.int32, device="cuda")
    api.prefix_cumsum(g, cu)
    torch.cuda.synchronize()
    assert L.wall_get_status() == L.WALL_ERR_INVALID_ARG
    assert L.wall_get_status() == L.WALL_OK
