"""Full-size parity on every workload, in the launch configuration bench.py times.

The whole layer runs on the GPU through the public API (xattn_prefill on the
Buffers the bench uses), and once more through the fused xattn_score_select, all
outputs poisoned beforehand. Then:
- masks, complete: for every query block of the "complete" heads (every head up
  to 32K tokens; longer layers one query head per KV group, each at a different
  position inside its group), every block score against the oracle and the kept
  list of both the two-call and the fused path against the oracle's selection on
  its own scores (mask-exception rules of tests/parity.py, every exception logged
  with config, head, row, block, margin and kind, and summarised per config at
  the end of the pytest run);
- outputs, sampled: for three query heads from different KV groups, the first,
  second, middle and last query blocks plus two drawn at random, every output
  element, once with the GPU's own kept lists and once with the oracle's;
- the whole layer: CSR structure, every diagonal present, score rows summing to
  1, nnz, and the fused path bit-identical to the two calls.
The oracle's per-head scoring runs in a pool of spawned worker processes (spawn,
not fork: the parent already holds a CUDA context).
"""
import concurrent.futures as cf
import math
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import oracle as orc
import synthetic as sy
from tests import parity as P
from tests.gpu_util import bf16_to_np, poison_buffers, poisoned_like, to_dev

pytestmark = pytest.mark.gpu

xa = pytest.importorskip("block_sparse_long_04_b200")

FULL = [("tiny_1h_2k", None), ("llama8b_gqa_32k", None), ("llama8b_gqa_128k", 4),
        ("llama8b_gqa_128k", 8), ("llama8b_gqa_128k", 16), ("llama8b_gqa_256k", None),
        ("video_dit_118k", None)]


def _alloc_poisoned(*a, **kw):
    return poison_buffers(xa.Buffers.allocate(*a, **kw))


@pytest.fixture(scope="module")
def pool():
    cores = len(os.sched_getaffinity(0))
    nproc = max(1, min(8, cores // 2))
    old = os.environ.get("OPENBLAS_NUM_THREADS")
    os.environ["OPENBLAS_NUM_THREADS"] = str(max(1, cores // nproc))
    ex = cf.ProcessPoolExecutor(nproc, mp_context=mp.get_context("spawn"))
    if old is None:
        os.environ.pop("OPENBLAS_NUM_THREADS")
    else:
        os.environ["OPENBLAS_NUM_THREADS"] = old
    yield ex
    ex.shutdown()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield


def complete_heads(w):
    """Heads whose every query block is checked against the oracle."""
    if w.M <= 32768:
        return list(range(w.Hq))
    if w.group > 1:
        return [kv * w.group + (kv % w.group) for kv in range(w.Hkv)]
    return list(range(w.Hq))


def _sample(w, seed=5):
    rng = np.random.default_rng(seed)
    heads = sorted({0, min(w.Hq - 1, w.Hq // 2 + 1), w.Hq - 1})
    nb = w.nb
    rows = sorted({0, min(1, nb - 1), nb // 2, nb - 1, *rng.integers(0, nb, 2).tolist()})
    return heads, rows


def _check_layer_structure(bufs, w):
    nb = w.nb
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
    return row_ptr, col, nnz


@pytest.mark.parametrize("name,stride", FULL)
def test_full_size_layer(name, stride, pool):
    w = sy.workload(name)
    if stride:
        w = w.with_(stride=stride)
    Qb, Kb, Vb = sy.layer_inputs(w)
    tau = sy.tau_vector(w)
    heads_full = complete_heads(w)
    nb, grp = w.nb, w.group
    # the oracle's complete scores of the checked heads, computed while the GPU runs
    jobs = {h: pool.submit(P.oracle_head_scores, (Qb[0, h], Kb[0, h // grp], w.stride, w.block,
                                                  w.causal)) for h in heads_full}

    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    tau_d = torch.from_numpy(tau).cuda()
    bufs = _alloc_poisoned(w.B, w.Hq, w.M, w.C, w.stride, w.causal)
    xa.xattn_prefill(Q, K, V, tau_d, w.stride, w.causal, bufs)
    fused = _alloc_poisoned(w.B, w.Hq, w.M, w.C, w.stride, w.causal)
    xa.xattn_score_select(Q, K, tau_d, xa.XATTN_SELECT_THRESHOLD, w.stride, w.causal,
                          xa.default_score_scale(w.stride, w.C), fused.scores, fused.row_ptr,
                          fused.col_idx, fused.nnz, fused.score_ws)
    torch.cuda.synchronize()
    assert xa.xattn_get_device_error() == xa.XATTN_OK

    row_ptr, col, nnz = _check_layer_structure(bufs, w)
    frp, fcol, fnnz = _check_layer_structure(fused, w)
    # the fused path: bit-identical scores and lists
    assert torch.equal(bufs.scores, fused.scores)
    assert fnnz == nnz and np.array_equal(frp, row_ptr) and np.array_equal(fcol[:nnz], col[:nnz])

    # complete masks of the checked heads, both paths, against the oracle
    got_s = bufs.scores.cpu().numpy()
    fails = []
    n_exc = 0
    ref_scores = {}
    for h in heads_full:
        ref = jobs[h].result()
        ref_scores[h] = ref
        P.assert_scores_close(got_s[0, h], ref, f"{name} S={w.stride} scores h{h}")
        for path, (rp_, ci_) in (("two-call", (row_ptr, col)), ("fused", (frp, fcol))):
            for r in range(nb):
                gk = ci_[rp_[h * nb + r]:rp_[h * nb + r + 1]].astype(np.int64)
                e, f = P.compare_row_mask(gk, ref[r], r, float(tau[h]), w.causal)
                for x in e:
                    P.log_exception(f"{name} S={w.stride} {path}", h, x)
                n_exc += len(e)
                fails += [(path, h) + tuple(x) for x in f]
    assert not fails, fails[:5]
    dens = nnz / xa.max_kept(1, w.Hq, nb, w.causal)
    P.report(f"{name} S={w.stride}: complete masks of {len(heads_full)}/{w.Hq} heads x {nb} "
             f"query blocks (two-call and fused) vs oracle: {n_exc} logged exceptions; "
             f"nnz={nnz} density={dens:.4f}")

    # outputs on sampled rows: the GPU's kept lists, then the oracle's
    heads, rows = _sample(w)
    sa = 1 / math.sqrt(w.C)
    sig = orc.default_score_scale(w.stride, w.C)
    got_o = bf16_to_np(bufs.O)
    ok_lists = {}
    for h in heads:
        q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // grp], Vb[0, h // grp]))
        ref = ref_scores[h] if h in ref_scores else \
            orc.block_scores(q, k, w.stride, w.block, sig, w.causal, rows=rows)
        gk = {}
        for r in rows:
            P.assert_scores_close(got_s[0, h, r], ref[r], f"{name} scores h{h} r{r}")
            gk[r] = col[row_ptr[h * nb + r]:row_ptr[h * nb + r + 1]].astype(np.int64)
        ok_lists[h] = {r: orc.select_row(ref[r], r, float(tau[h]), w.causal) for r in rows}
        o, _ = orc.block_sparse_attention(q, k, v, gk, w.block, w.causal, sa, rows=rows)
        for i, r in enumerate(rows):
            P.assert_outputs_close(got_o[0, h, r * 128:(r + 1) * 128], o[i * 128:(i + 1) * 128],
                                   f"{name} O h{h} r{r}")

    lists = [col[row_ptr[i]:row_ptr[i + 1]] for i in range(w.B * w.Hq * nb)]
    for h in heads:
        for r in rows:
            lists[h * nb + r] = ok_lists[h][r].astype(np.int32)
    rp2 = np.zeros(len(lists) + 1, np.int64)
    rp2[1:] = np.cumsum([len(x) for x in lists])
    O2 = poisoned_like(Q)
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
    assert xa.xattn_get_device_error() == xa.XATTN_OK
