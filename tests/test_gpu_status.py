"""Failure detection without a GPU fault: a bounded device wait on a barrier that
never completes returns SVDQ_ETIMEOUT and leaves the context usable."""

import pytest
import torch

import rank_bit_residual_b200 as rb
from tests.gpu_util import device

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    device()
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert rb.svdq_selftest_wait_timeout(1000) == rb.SVDQ_ETIMEOUT
    assert rb.svdq_check_status() == rb.SVDQ_OK          # the word was cleared
    x = torch.ones(1024, device=device())
    assert float((x * 2).sum()) == 2048.0                  # the context still works
