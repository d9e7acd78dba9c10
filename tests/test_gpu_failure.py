"""Failure detection without a GPU fault: a device-side wait that can never
complete gives up after its bound, the kernel returns, the host reads
HCA_ERR_TIMEOUT from the status word, and the context keeps working."""
import time

import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from tests.helpers import rnd


@pytest.mark.gpu
def test_expired_wait_is_reported_and_the_context_survives(cuda):
    assert hb.device_status() == hb.HCA_OK          # clears any earlier state
    t0 = time.perf_counter()
    hb.selftest_wait(50_000_000)                     # 50 ms bound
    assert hb.device_status() == hb.HCA_ERR_TIMEOUT
    assert time.perf_counter() - t0 >= 0.04          # it really waited for its bound
    assert hb.device_status() == hb.HCA_OK           # reading clears the word
    # the context still runs real work
    x = rnd((256, 256), 1, 1)
    assert torch.isfinite(x @ x).all()
    hb.selftest_wait(1_000_000)
    assert hb.device_status() == hb.HCA_ERR_TIMEOUT


def test_selftest_rejects_out_of_range_limits():
    import ctypes
    hb.lib()
    rc = hb.lib().hca_selftest_wait(ctypes.c_ulonglong(10), None)
    assert rc == hb.HCA_ERR_INVALID and "limit_ns" in hb.last_error()
    rc = hb.lib().hca_selftest_wait(ctypes.c_ulonglong(3_000_000_000), None)
    assert rc == hb.HCA_ERR_INVALID
