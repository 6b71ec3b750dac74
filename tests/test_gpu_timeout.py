"""Failure detection without a fault: a device wait that nothing completes
gives up after its bounded limit and reports HISA_DEV_TIMEOUT, and the
context stays usable for the next call."""
import numpy as np
import pytest
import torch

from hisa_inputs import make_case
from tests.gpu_util import check_hisa, device_case, lib, run_hisa

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    h = lib()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    h.hisa_selftest_wait(status)
    torch.cuda.synchronize()
    assert int(status.item()) & h.HISA_DEV_TIMEOUT
    case = make_case(batch=1, L=2048, H=8, d=128, B=64, m=6, k=128, seed=21,
                     positions=np.array([2047, 700]))
    kv = device_case(case)
    check_hisa(case, run_hisa(case, kv))
    assert kv.status_bits() == 0
