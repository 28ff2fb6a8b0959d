"""Full-size parity on every workload, in the launch configuration bench.py times.

The whole layer runs on the GPU through the public API (xattn_prefill on the
Buffers the bench uses). The oracle then recomputes a sample of rows one by one:
for three query heads from different KV groups, the first, second, middle and last
query blocks plus two drawn at random. On those rows: every block score, the kept
list (mask-exception rules of tests/parity.py), and every output element, once
with the GPU's own kept lists and once with the oracle's.
Properties that hold at any size are checked on the whole layer: CSR structure,
every diagonal present, score rows summing to 1, and nnz.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import synthetic as sy
from tests import parity as P
from tests.gpu_util import bf16_to_np, to_dev

pytestmark = pytest.mark.gpu

xa = pytest.importorskip("block_sparse_long_04_b200")

FULL = [("tiny_1h_2k", None), ("llama8b_gqa_32k", None), ("llama8b_gqa_128k", 4),
        ("llama8b_gqa_128k", 8), ("llama8b_gqa_128k", 16), ("llama8b_gqa_256k", None),
        ("video_dit_118k", None)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield


def _sample(w, seed=5):
    rng = np.random.default_rng(seed)
    heads = sorted({0, min(w.Hq - 1, w.Hq // 2 + 1), w.Hq - 1})
    nb = w.nb
    rows = sorted({0, min(1, nb - 1), nb // 2, nb - 1, *rng.integers(0, nb, 2).tolist()})
    return heads, rows


@pytest.mark.parametrize("name,stride", FULL)
def test_full_size_sampled_rows(name, stride):
    w = sy.workload(name)
    if stride:
        w = w.with_(stride=stride)
    Qb, Kb, Vb = sy.layer_inputs(w)
    tau = sy.tau_vector(w)
    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    bufs = xa.Buffers.allocate(w.B, w.Hq, w.M, w.C, w.stride, w.causal)
    xa.xattn_prefill(Q, K, V, torch.from_numpy(tau).cuda(), w.stride, w.causal, bufs)
    torch.cuda.synchronize()
    assert xa.xattn_get_device_error() == xa.XATTN_OK
    nb, grp = w.nb, w.group

    # properties of the whole layer
    rs = bufs.scores.sum(dim=-1)
    assert torch.allclose(rs, torch.ones_like(rs), atol=1e-3), float((rs - 1).abs().max())
    row_ptr = bufs.row_ptr.cpu().numpy().astype(np.int64)
    col = bufs.col_idx.cpu().numpy()
    nnz = int(bufs.nnz.item())
    assert row_ptr[0] == 0 and row_ptr[-1] == nnz and (np.diff(row_ptr) >= 1).all()
    rows_all = np.repeat(np.arange(w.B * w.Hq * nb) % nb, np.diff(row_ptr))
    cols = col[:nnz].astype(np.int64)
    assert (cols >= 0).all() and (cols < nb).all()
    if w.causal:
        assert (cols <= rows_all).all()
    diag = np.zeros(w.B * w.Hq * nb, bool)
    is_diag = cols == rows_all
    diag[np.repeat(np.arange(w.B * w.Hq * nb), np.diff(row_ptr))[is_diag]] = True
    assert diag.all(), "a row lost its diagonal block"
    same_row = np.repeat(np.arange(w.B * w.Hq * nb), np.diff(row_ptr))
    inc = np.diff(cols)[np.diff(same_row) == 0]
    assert (inc > 0).all(), "kept lists must be ascending and unique"

    # sampled rows against the oracle
    heads, rows = _sample(w)
    sig, sa = orc.default_score_scale(w.stride, w.C), 1 / math.sqrt(w.C)
    got_s = bufs.scores.cpu().numpy()
    got_o = bf16_to_np(bufs.O)
    log, fails = [], []
    ok_lists = {}
    for h in heads:
        q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // grp], Vb[0, h // grp]))
        ref = orc.block_scores(q, k, w.stride, w.block, sig, w.causal, rows=rows)
        gk, okk = {}, {}
        for r in rows:
            P.assert_scores_close(got_s[0, h, r], ref[r], f"{name} scores h{h} r{r}")
            gk[r] = col[row_ptr[h * nb + r]:row_ptr[h * nb + r + 1]].astype(np.int64)
            e, f = P.compare_row_mask(gk[r], ref[r], r, float(tau[h]), w.causal)
            log += e
            fails += f
            okk[r] = orc.select_row(ref[r], r, float(tau[h]), w.causal)
        ok_lists[h] = okk
        o, _ = orc.block_sparse_attention(q, k, v, gk, w.block, w.causal, sa, rows=rows)
        for i, r in enumerate(rows):
            P.assert_outputs_close(got_o[0, h, r * 128:(r + 1) * 128], o[i * 128:(i + 1) * 128],
                                   f"{name} O h{h} r{r}")
    assert not fails, fails[:5]
    print(f"{name} S={w.stride}: nnz={nnz} density={nnz / xa.max_kept(1, w.Hq, nb, w.causal):.4f} "
          f"mask exceptions on sampled rows={len(log)}")

    # outputs given the oracle's kept lists on the sampled rows
    lists = [col[row_ptr[i]:row_ptr[i + 1]] for i in range(w.B * w.Hq * nb)]
    for h in heads:
        for r in rows:
            lists[h * nb + r] = ok_lists[h][r].astype(np.int32)
    rp2 = np.zeros(len(lists) + 1, np.int64)
    rp2[1:] = np.cumsum([len(x) for x in lists])
    O2 = torch.empty_like(Q)
    xa.xattn_sparse_attn(Q, K, V, torch.from_numpy(rp2.astype(np.int32)).cuda(),
                         torch.from_numpy(np.concatenate(lists).astype(np.int32)).cuda(),
                         w.causal, sa, O2)
    got2 = bf16_to_np(O2)
    for h in heads:
        q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // grp], Vb[0, h // grp]))
        o, _ = orc.block_sparse_attention(q, k, v, ok_lists[h], w.block, w.causal, sa, rows=rows)
        for i, r in enumerate(rows):
            P.assert_outputs_close(got2[0, h, r * 128:(r + 1) * 128], o[i * 128:(i + 1) * 128],
                                   f"{name} O (oracle mask) h{h} r{r}")


@pytest.mark.parametrize("name", ["llama8b_gqa_128k", "video_dit_118k"])
def test_full_size_fused_score_select_is_bit_identical(name):
    """The fused score+select entry point at full size: scores and kept lists
    bit-identical to the two separate calls the bench times."""
    w = sy.workload(name)
    Qb, Kb, _ = sy.layer_inputs(w)
    Q, K = to_dev(Qb), to_dev(Kb)
    tau = torch.from_numpy(sy.tau_vector(w)).cuda()
    ss = xa.default_score_scale(w.stride, w.C)
    a = xa.Buffers.allocate(w.B, w.Hq, w.M, w.C, w.stride, w.causal)
    xa.xattn_score(Q, K, w.stride, w.causal, ss, a.scores, a.score_ws)
    xa.xattn_select(a.scores, tau, w.causal, a.row_ptr, a.col_idx, a.nnz, a.select_ws)
    f = xa.Buffers.allocate(w.B, w.Hq, w.M, w.C, w.stride, w.causal)
    xa.xattn_score_select(Q, K, tau, xa.XATTN_SELECT_THRESHOLD, w.stride, w.causal, ss, f.scores,
                          f.row_ptr, f.col_idx, f.nnz, f.score_ws)
    torch.cuda.synchronize()
    assert xa.xattn_get_device_error() == xa.XATTN_OK
    n = int(a.nnz.item())
    assert int(f.nnz.item()) == n
    assert torch.equal(a.scores, f.scores)
    assert torch.equal(a.row_ptr, f.row_ptr)
    assert torch.equal(a.col_idx[:n], f.col_idx[:n])
