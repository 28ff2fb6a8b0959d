"""The FMA-pipe base-2 exponential of the attention softmax against fp64 2^x
and its stated error bound (range reduction to [-1/2, 1/2] plus a fitted cubic;
the bound comes from the fit, checked here on the device's own arithmetic)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

xa = pytest.importorskip("block_sparse_long_04_b200")

REL_BOUND = 1.1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    assert xa.xattn_get_device_error() == xa.XATTN_OK


def _run(x_np):
    x = torch.from_numpy(x_np.astype(np.float32)).cuda()
    y = torch.empty_like(x)
    xa.xattn_selftest_exp2(x, y)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_relative_error_over_the_domain():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 127.0, 200001),
        rng.uniform(-30.0, 8.0, 400001),           # the softmax's range (x <= 8)
        np.arange(-126, 128, dtype=np.float64),     # integers: f = 0
        np.arange(-126, 127) + 0.5,                 # ties of the rounding
    ]).astype(np.float32)
    y = _run(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= REL_BOUND, (rel.max(), x[np.argmax(rel)])
    # the cubic has constant term 1: every integer power of two is exact
    ints = np.arange(-126, 128, dtype=np.float32)
    assert np.array_equal(_run(ints), np.exp2(ints.astype(np.float64)))


def test_zero_below_the_clamp_and_odd_length():
    x = np.array([-np.inf, -1e30, -1000.0, -127.0, -126.7, -126.2, 0.0], dtype=np.float32)
    y = _run(x)
    assert np.array_equal(y[:4], np.zeros(4))
    assert np.all(y[4:6] >= 0.0) and np.all(y[4:6] <= 2.0 ** -126)
    assert y[6] == 1.0
