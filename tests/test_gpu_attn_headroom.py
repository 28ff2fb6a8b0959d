"""Attention rows whose logits grow far beyond those of their first kept block.

The attention kernel exponentiates every block of a row against one reference,
the maximum over the row's first kept block (FlashAttention-style online
softmax, XAttention summary, Approach, with the rescaling folded into a fixed
reference). Rows whose later blocks exceed it by more than the kernel's headroom
are computed a second time against their true maximum. These cases put a few
keys with very large (or very small) logits in later blocks and compare the
output and log-sum-exp with the fp64 oracle: growth within the headroom (one
pass, P far above 1), growth beyond it (second pass), and a first block far
above the rest (P far below 1).
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import synthetic as sy
from tests import parity as P
from tests.gpu_util import bf16_to_np, poisoned, poisoned_like, to_dev

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


def _inputs(M, C, Hq, boost_log2, heavy_blocks, seed):
    """Q, K, V ~ N(0,1); every query gets +a*u and one key per heavy block gets
    +beta*u, so that key's logit sits about boost_log2 (base 2, scaled) above
    the noise."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, Hq, M, C)).astype(np.float32)
    k = rng.standard_normal((1, 1, M, C)).astype(np.float32)
    v = rng.standard_normal((1, 1, M, C)).astype(np.float32)
    u = rng.standard_normal(C)
    u = (u / np.linalg.norm(u)).astype(np.float32)
    a = 4.0
    beta = boost_log2 * math.sqrt(C) / (a * LOG2E)
    q += a * u
    for c in heavy_blocks:
        k[0, 0, c * 128 + 7] += beta * u
    return tuple(sy.bf16_round(x) for x in (q, k, v))


CASES = [
    # C, causal, boost (log2 units), heavy key blocks
    (64, True, 18.0, [2, 5]),       # within the headroom: one pass, P up to ~2^18
    (128, False, 18.0, [3]),
    (64, True, 40.0, [1, 4, 6]),    # beyond it: the tiles of rows r >= 1 run twice
    (128, False, 40.0, [6]),        # every row's first block (block 0) is far below
    (64, True, 200.0, [2, 5]),      # beyond fp32 range of 2^(x - m_ref): only the
    (128, False, 200.0, [6]),       # second pass can produce finite results
    (128, True, 40.0, [0]),         # the first block holds the largest logit
    (128, True, 200.0, [0]),
    (64, False, -30.0, [3]),        # a few keys far below the rest
]


@pytest.mark.parametrize("C,causal,boost,heavy", CASES)
def test_dense_attention_far_from_first_block(C, causal, boost, heavy):
    M, Hq = 1024, 2
    Qb, Kb, Vb = _inputs(M, C, Hq, boost, heavy, seed=17)
    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    O = poisoned_like(Q)
    lse = poisoned((1, Hq, M))
    scale = 1 / math.sqrt(C)
    xa.xattn_dense_attn(Q, K, V, causal, scale, O, lse)
    got, gl = bf16_to_np(O), lse.cpu().numpy()
    k, v = orc.bf16_to_f64(Kb[0, 0]), orc.bf16_to_f64(Vb[0, 0])
    for h in range(Hq):
        o, l = orc.dense_attention(orc.bf16_to_f64(Qb[0, h]), k, v, causal, scale)
        P.assert_outputs_close(got[0, h], o, f"O head {h}")
        np.testing.assert_allclose(gl[0, h], l, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("C,causal,boost,heavy", CASES)
def test_sparse_attention_far_from_first_block(C, causal, boost, heavy):
    """Shuffled lists: the first kept block of a row is a random one of them."""
    M, Hq = 1024, 2
    nb = M // 128
    Qb, Kb, Vb = _inputs(M, C, Hq, boost, heavy, seed=23)
    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    rng = np.random.default_rng(29)
    kept, rows, ptr = {}, [], [0]
    for h in range(Hq):
        for r in range(nb):
            n = r + 1 if causal else nb
            pick = set(rng.choice(n, size=max(1, (2 * n) // 3), replace=False).tolist()) | {r}
            pick |= {c for c in heavy if c < n}
            lst = rng.permutation(sorted(pick)).tolist()
            kept.setdefault(h, {})[r] = sorted(pick)
            rows.extend(lst)
            ptr.append(len(rows))
    rp = torch.tensor(ptr, dtype=torch.int32, device="cuda")
    ci = torch.tensor(rows, dtype=torch.int32, device="cuda")
    O = poisoned_like(Q)
    lse = poisoned((1, Hq, M))
    scale = 1 / math.sqrt(C)
    xa.xattn_sparse_attn(Q, K, V, rp, ci, causal, scale, O, lse)
    got, gl = bf16_to_np(O), lse.cpu().numpy()
    k, v = orc.bf16_to_f64(Kb[0, 0]), orc.bf16_to_f64(Vb[0, 0])
    for h in range(Hq):
        o, l = orc.block_sparse_attention(orc.bf16_to_f64(Qb[0, h]), k, v, kept[h], 128, causal,
                                          scale)
        P.assert_outputs_close(got[0, h], o, f"O head {h}")
        np.testing.assert_allclose(gl[0, h], l, rtol=1e-4, atol=1e-4)
