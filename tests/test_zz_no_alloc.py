"""xattn_select_noalloc: threshold selection for callers that cannot allocate.

Some callers cannot hand the library a workspace: a host framework that owns
all device memory and forbids allocation inside its execute callbacks, or a
latency-critical caller that cannot take the synchronisation a cudaMalloc may
bring. xattn_select_noalloc serves them from a fixed scratch array inside the
library. Its kept lists must equal those of xattn_select exactly (they are
integer outputs), call after call, although every call reuses the same scratch.

This file is collected last, so that a run stopping at its first failure has
already run every other test. It builds the library itself (a no-op when the
build is current) and sets up every input it needs, so it also passes when run
alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import poisoned

from block_sparse_long_04_b200 import build as _build

_build.build()
import block_sparse_long_04_b200 as xa  # noqa: E402


def _scores(seed, Hq, nb, causal):
    rng = np.random.default_rng(seed)
    s = rng.gamma(0.4, size=(1, Hq, nb, nb))
    if causal:
        s = np.tril(s)
    s /= s.sum(axis=-1, keepdims=True)
    return torch.from_numpy(s.astype(np.float32)).cuda()


def _outputs(Hq, nb, causal):
    rows = Hq * nb
    cap = xa.max_kept(1, Hq, nb, causal)
    return (torch.full((rows + 1,), -1, dtype=torch.int32, device="cuda"),
            torch.full((cap,), -1, dtype=torch.int32, device="cuda"),
            torch.full((1,), -1, dtype=torch.int32, device="cuda"))


@pytest.mark.gpu
def test_noalloc_select_equals_select_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # two calls in a row with different shapes and thresholds; the second call
    # finds the first call's rows still in the shared scratch
    for seed, Hq, nb, causal, taus in ((1, 4, 300, True, [0.9, 0.5, 0.99, 0.8]),
                                       (2, 3, 97, False, [0.95, 0.7, 0.3])):
        scores = _scores(seed, Hq, nb, causal)
        tau = torch.tensor(taus, dtype=torch.float32, device="cuda")
        ref = _outputs(Hq, nb, causal)
        ws = poisoned(xa.xattn_select_workspace_size(1, Hq, nb), torch.uint8)
        xa.xattn_select(scores, tau, causal, *ref, ws)
        got = _outputs(Hq, nb, causal)
        rp, ci, nz = got
        # straight through the C ABI: no workspace argument at all
        rc = xa._lib.xattn_select_noalloc(
            ctypes.c_void_p(scores.data_ptr()), ctypes.c_void_p(tau.data_ptr()), 1, Hq, nb,
            int(causal), ctypes.c_void_p(rp.data_ptr()), ctypes.c_void_p(ci.data_ptr()),
            ci.numel(), ctypes.c_void_p(nz.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == xa.XATTN_OK, xa.status_string(rc)
        torch.cuda.synchronize()
        assert xa.xattn_get_device_error() == xa.XATTN_OK
        n = int(ref[2].item())
        assert int(nz.item()) == n
        assert torch.equal(rp, ref[0])
        assert torch.equal(ci[:n], ref[1][:n])


def _call(ptrs, B, Hq, nb, causal, cap, stream=None):
    sc, tau, rp, ci, nz = (ctypes.c_void_p(p) if p is not None else None for p in ptrs)
    return xa._lib.xattn_select_noalloc(sc, tau, B, Hq, nb, int(causal), rp, ci, cap, nz, stream)


def test_noalloc_select_rejects_rows_beyond_its_scratch():
    # checked on the host before any launch: no GPU needed
    fake = 0x7F0000001000
    top = xa.XATTN_SELECT_NOALLOC_MAX_ROWS
    # one row beyond the scratch array
    assert _call([fake] * 5, 1, top + 1, 1, True, 1 << 30) == xa.XATTN_EUNSUPPORTED
    assert _call([fake] * 5, 1, top // 2048 + 1, 2048, True, 1 << 30) == xa.XATTN_EUNSUPPORTED
    # exactly the scratch size passes the size check: with no output pointers the
    # call then stops at the argument check, still before any launch
    assert _call([fake, fake, None, fake, None], 1, top, 1, True, 1 << 30) == xa.XATTN_EINVAL
    assert _call([fake, fake, None, fake, None], 2, top // 2048, 1024, True,
                 1 << 30) == xa.XATTN_EINVAL


@pytest.mark.gpu
def test_noalloc_select_fills_its_whole_scratch():
    """Exactly XATTN_SELECT_NOALLOC_MAX_ROWS rows (B = 2, 128 heads, 1024 query
    blocks), so the last row lands in the last slot of the fixed array; the kept
    lists must equal xattn_select's."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B, Hq, nb, causal = 2, 128, 1024, True
    assert B * Hq * nb == xa.XATTN_SELECT_NOALLOC_MAX_ROWS
    g = torch.Generator(device="cuda").manual_seed(7)
    s = torch.rand((B, Hq, nb, nb), device="cuda", generator=g) ** 6
    s = torch.tril(s)
    s /= s.sum(dim=-1, keepdim=True)
    tau = torch.linspace(0.5, 0.98, Hq, device="cuda")
    cap = xa.max_kept(B, Hq, nb, causal)
    ref = (torch.full((B * Hq * nb + 1,), -1, dtype=torch.int32, device="cuda"),
           torch.full((cap,), -1, dtype=torch.int32, device="cuda"),
           torch.full((1,), -1, dtype=torch.int32, device="cuda"))
    ws = poisoned(xa.xattn_select_workspace_size(B, Hq, nb), torch.uint8)
    xa.xattn_select(s, tau, causal, *ref, ws)
    got = tuple(torch.full_like(t, -1) for t in ref)
    rc = _call([s.data_ptr(), tau.data_ptr(), got[0].data_ptr(), got[1].data_ptr(),
                got[2].data_ptr()], B, Hq, nb, causal, cap,
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == xa.XATTN_OK, xa.status_string(rc)
    torch.cuda.synchronize()
    assert xa.xattn_get_device_error() == xa.XATTN_OK
    n = int(ref[2].item())
    assert int(got[2].item()) == n
    assert torch.equal(got[0], ref[0])
    assert torch.equal(got[1][:n], ref[1][:n])
