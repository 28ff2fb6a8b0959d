"""Failure detection without a GPU fault: a device wait that nothing completes
gives up after its limit, reports XATTN_ETIMEOUT through the device error word,
and the context stays usable for ordinary work afterwards."""
import time

import pytest
import torch

import block_sparse_long_04_b200 as xa

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert xa.xattn_get_device_error() == xa.XATTN_OK
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    xa.xattn_selftest_wait_timeout(20_000_000, flag)        # 20 ms
    assert xa.xattn_get_device_error() == xa.XATTN_ETIMEOUT
    elapsed = time.perf_counter() - t0
    assert int(flag.item()) == 1
    assert 0.015 < elapsed < 5.0
    assert xa.xattn_get_device_error() == xa.XATTN_OK       # read clears the word
    # the context still runs kernels
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2
