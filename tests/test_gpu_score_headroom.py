"""Scoring rows whose logits grow (or fall) far from those of their first block.

The scoring epilogue sums each half row of the strided antidiagonal logits
against one reference: its first visible key block's maximum, raised (with the
running sum rescaled) only when a later block exceeds it by more than 2^64
(XAttention summary, Approach: row softmax, then block summation). These cases
put one key per chosen block far above (or below) the rest, so that rows see
growth within that headroom, beyond it, beyond the fp32 range of an exponential,
and a first block far above everything after it, and compare every block score
with the fp64 oracle and every row sum with 1.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import synthetic as sy
from tests import parity as P
from tests.gpu_util import poisoned, to_dev

pytestmark = pytest.mark.gpu

xa = pytest.importorskip("block_sparse_long_04_b200")

LOG2E = 1.0 / math.log(2.0)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()
    yield
    assert xa.xattn_get_device_error() == xa.XATTN_OK


def _inputs(M, C, Hq, S, boost_log2, heavy_blocks, seed):
    """Q, K ~ N(0,1); every query gets +a*u and one key in each heavy block gets
    +beta*u. A reshaped query row then meets that key in exactly one term of its
    dot product with the reshaped key row that holds it, which lifts that logit
    by about boost_log2 (base 2, with the default scale 1/sqrt(S*C))."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, Hq, M, C)).astype(np.float32)
    k = rng.standard_normal((1, 1, M, C)).astype(np.float32)
    u = rng.standard_normal(C)
    u = (u / np.linalg.norm(u)).astype(np.float32)
    a = 4.0
    beta = boost_log2 * math.sqrt(S * C) / (a * LOG2E)
    q += a * u
    for c in heavy_blocks:
        k[0, 0, c * 128 + 37] += beta * u
    return tuple(sy.bf16_round(x) for x in (q, k))


CASES = [
    # M, C, stride, causal, boost (log2 units), heavy key blocks
    (1024, 128, 8, True, 40.0, [2, 5]),     # within the headroom: no rescale
    (1024, 128, 8, True, 100.0, [2, 5]),    # beyond it: rows r >= 2 rescale once or twice
    (1024, 64, 4, False, 100.0, [6]),
    (1024, 128, 8, True, 200.0, [3]),       # beyond the fp32 range of one exponential
    (1024, 128, 8, True, 100.0, [0]),       # the first block far above every later one
    (1024, 64, 16, True, -80.0, [4]),       # a few keys far below the rest
    (2048, 128, 32, False, 150.0, [1, 9]),  # four reshaped columns per block
]


@pytest.mark.parametrize("M,C,S,causal,boost,heavy", CASES)
def test_scores_far_from_first_block(M, C, S, causal, boost, heavy):
    Hq = 2
    Qb, Kb = _inputs(M, C, Hq, S, boost, heavy, seed=23)
    Q, K = to_dev(Qb), to_dev(Kb)
    nb = M // 128
    scores = torch.full((1, Hq, nb, nb), float("nan"), device="cuda")
    ws = poisoned(xa.xattn_score_workspace_size(1, Hq, M, S, causal), torch.uint8)
    scale = orc.default_score_scale(S, C)
    xa.xattn_score(Q, K, S, causal, scale, scores, ws)
    got = scores.cpu().numpy()
    ref = orc.layer_block_scores(Qb, Kb, 1, S, 128, scale, causal)
    for h in range(Hq):
        P.assert_scores_close(got[0, h], ref[(0, h)], f"scores head {h}")
        np.testing.assert_allclose(got[0, h].sum(axis=1), 1.0, atol=1e-4)
    assert xa.xattn_get_device_error() == xa.XATTN_OK
