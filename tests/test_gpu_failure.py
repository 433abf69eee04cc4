"""Failure detection without a GPU fault: a bounded device wait that runs out."""

import pytest
import torch

from long_context_sparse_05_b200 import _lib as L

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert L.csa_device_error() == 0                 # clears any earlier state
    L.csa_selftest_bounded_wait(20000)               # 20 ms bound on a barrier nobody signals
    assert L.csa_device_error() == 4                 # CSA_ERR_TIMEOUT, read and cleared
    assert L.csa_device_error() == 0
    x = torch.arange(8, device="cuda") * 2           # the context is still usable
    torch.cuda.synchronize()
    assert int(x.sum()) == 56


def test_selftest_rejects_unbounded_limits():
    with pytest.raises(L.CsaError):
        L.csa_selftest_bounded_wait(0)
    with pytest.raises(L.CsaError):
        L.csa_selftest_bounded_wait(10 ** 7)
