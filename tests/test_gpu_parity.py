"""Parity of the CUDA path (through the C ABI) with the CPU fp64 oracle.

Small cases are compared element by element (every score, every mask row, every
output element); they span several 128-row score tiles with a ragged last tile,
all supported strides, both head dims, GQA, causal and non-causal. Tolerances and
mask-exception rules are in tests/parity.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import synthetic as sy
from tests import parity as P
from tests.gpu_util import (bf16_to_np, csr_to_dict, device_inputs, dict_to_csr, poison_buffers,
                            poisoned, poisoned_like, small_workload)

pytestmark = pytest.mark.gpu

xa = pytest.importorskip("block_sparse_long_04_b200")


def _alloc_poisoned(*a, **kw):
    return poison_buffers(xa.Buffers.allocate(*a, **kw))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()
    yield
    assert xa.xattn_get_device_error() == xa.XATTN_OK


def _oracle_scores(Qb, Kb, w, heads=None, rows=None, scale=None):
    s = orc.default_score_scale(w.stride, w.C) if scale is None else scale
    return orc.layer_block_scores(Qb, Kb, w.Hkv, w.stride, w.block, s, w.causal, heads, rows)


SCORE_CASES = [
    # M, C, Hq, Hkv, stride, causal
    (2048, 64, 1, 1, 8, True),      # the tiny single-head workload's shape
    (1152, 128, 4, 2, 8, True),     # M/S = 144: two score tiles, ragged tail
    (1152, 64, 2, 1, 4, False),
    (640, 128, 2, 2, 16, True),     # M/S = 40: one partial tile
    (1024, 64, 1, 1, 1, True),      # stride 1: plain attention mass per block
    (1024, 128, 2, 1, 2, False),
    (128, 128, 1, 1, 8, True),      # a single block
    (256, 64, 1, 1, 16, False),
    (4096, 128, 8, 2, 8, True),     # several tiles in both directions
    (3200, 128, 4, 4, 4, True),     # M/S = 800: 7 tiles, ragged
    (8320, 128, 2, 2, 32, False),   # M/S = 260: 3 tiles, ragged; 4 columns per block
    (4096, 64, 2, 1, 32, True),
    (16512, 128, 2, 1, 64, True),   # M/S = 258: 3 tiles, ragged; 2 columns per block
    (2048, 64, 1, 1, 64, False),    # M/S = 32: one partial tile
]


@pytest.mark.parametrize("M,C,Hq,Hkv,S,causal", SCORE_CASES)
def test_scores_match_oracle(M, C, Hq, Hkv, S, causal):
    w = small_workload(M, C, Hq, Hkv, S, causal)
    (Qb, Kb, _), (Q, K, _) = device_inputs(w)
    nb = M // 128
    scores = torch.full((1, Hq, nb, nb), float("nan"), device="cuda")
    ws = poisoned(xa.xattn_score_workspace_size(1, Hq, M, S, causal), torch.uint8)
    xa.xattn_score(Q, K, S, causal, orc.default_score_scale(S, C), scores, ws)
    got = scores.cpu().numpy()
    ref = _oracle_scores(Qb, Kb, w)
    for h in range(Hq):
        P.assert_scores_close(got[0, h], ref[(0, h)], f"scores head {h}")
        np.testing.assert_allclose(got[0, h].sum(axis=1), 1.0, atol=1e-4)


def test_score_scale_is_honoured():
    w = small_workload(1024, 128, 2, 1, 8, True)
    (Qb, Kb, _), (Q, K, _) = device_inputs(w)
    nb = 8
    scores = poisoned((1, 2, nb, nb))
    ws = poisoned(xa.xattn_score_workspace_size(1, 2, 1024, 8, True), torch.uint8)
    for sc in (1.0 / 128, 1.0 / math.sqrt(128)):
        xa.xattn_score(Q, K, 8, True, sc, scores, ws)
        ref = _oracle_scores(Qb, Kb, w, scale=sc)
        for h in range(2):
            P.assert_scores_close(scores.cpu().numpy()[0, h], ref[(0, h)])


def _run_select(scores_np, tau, causal, cap=None):
    B, Hq, nb, _ = scores_np.shape
    sc = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).cuda()
    t = torch.from_numpy(np.asarray(tau, np.float32)).cuda()
    cap = xa.max_kept(B, Hq, nb, causal) if cap is None else cap
    row_ptr = torch.full((B * Hq * nb + 1,), -7, dtype=torch.int32, device="cuda")
    col = torch.full((max(1, cap),), -7, dtype=torch.int32, device="cuda")
    nnz = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = poisoned(xa.xattn_select_workspace_size(B, Hq, nb), torch.uint8)
    xa.xattn_select(sc, t, causal, row_ptr, col, nnz, ws)
    return row_ptr.cpu().numpy(), col.cpu().numpy(), int(nnz.item())


def _check_masks(row_ptr, col, scores_ref, tau, causal, Hq, nb, log):
    fails = []
    for h in range(Hq):
        for r in range(nb):
            gcols = col[row_ptr[h * nb + r]:row_ptr[h * nb + r + 1]]
            exc, f = P.compare_row_mask(gcols, scores_ref[h][r], r, float(tau[h]), causal)
            for x in exc:
                P.log_exception(f"selection nb={nb} causal={causal}", h, x)
            log += exc
            fails += f
    return fails


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nb", [1, 2, 17, 300, 1024])
def test_selection_matches_oracle_on_same_scores(causal, nb):
    """The selection kernel alone: fed the oracle's scores (rounded to fp32)."""
    rng = np.random.default_rng(nb + causal)
    Hq = 3
    s = rng.gamma(0.3, size=(1, Hq, nb, nb))
    if causal:
        s = np.tril(s)
    s = (s / s.sum(axis=-1, keepdims=True)).astype(np.float32)
    s64 = s.astype(np.float64)
    tau = np.array([0.9, 0.5, 0.99], np.float32)
    row_ptr, col, nnz = _run_select(s, tau, causal)
    assert row_ptr[0] == 0 and nnz == row_ptr[-1]
    log = []
    fails = _check_masks(row_ptr, col, s64[0], tau.astype(np.float64), causal, Hq, nb, log)
    assert not fails, fails[:5]
    assert len(log) <= max(2, Hq * nb // 100), log[:10]


def test_selection_special_taus_and_ties():
    nb = 64
    s = np.full((1, 2, nb, nb), 1.0 / nb, np.float32)     # all tied, non-causal
    # tau = 1 keeps everything; tau small keeps block 0 (smallest index) + diagonal
    row_ptr, col, nnz = _run_select(s, [1.0, 1e-6], False)
    for r in range(nb):
        assert col[row_ptr[r]:row_ptr[r + 1]].tolist() == list(range(nb))
        want = sorted({0, r})
        assert col[row_ptr[nb + r]:row_ptr[nb + r + 1]].tolist() == want
    assert nnz == nb * nb + sum(len({0, r}) for r in range(nb))


def test_selection_cut_inside_a_tie_group():
    """Every candidate has the same score: the cut falls inside one tie group
    (the radix search resolves all 32 rank bits, then counts in index order)."""
    for nb, causal in ((64, False), (300, True)):
        s = np.full((1, 3, nb, nb), 1.0, np.float64)
        if causal:
            s = np.tril(s)
        s /= s.sum(-1, keepdims=True)
        s = s.astype(np.float32)
        tau = np.array([0.51, 0.26, 0.999], np.float32)
        row_ptr, col, nnz = _run_select(s, tau, causal)
        for h in range(3):
            for r in range(nb):
                got = col[row_ptr[h * nb + r]:row_ptr[h * nb + r + 1]]
                want = orc.select_row(s[0, h, r].astype(np.float64), r, float(tau[h]), causal)
                assert got.tolist() == want.tolist(), (nb, h, r)


def test_selection_rows_with_negative_and_infinite_scores():
    """Rows holding a negative or an infinite score (never produced by the scoring
    kernel) take the full-sort path; the threshold and Top-K rules still follow
    the descending order exactly."""
    rng = np.random.default_rng(3)
    nb, Hq = 40, 2
    s = rng.gamma(0.5, size=(1, Hq, nb, nb))
    s /= s.sum(-1, keepdims=True)
    s[0, 0, 5, [1, 7, 30]] = [-0.25, -0.5, -0.125]      # negative entries
    s[0, 1, 9, 3] = np.inf                               # an infinite entry
    s[0, 1, 11, :] = -s[0, 1, 11, :]                     # a row of negatives only
    s = s.astype(np.float32)
    tau = np.array([0.6, 0.8], np.float32)
    row_ptr, col, nnz = _run_select(s, tau, False)
    for h in range(Hq):
        for r in range(nb):
            got = col[row_ptr[h * nb + r]:row_ptr[h * nb + r + 1]]
            want = orc.select_row(s[0, h, r].astype(np.float64), r, float(tau[h]), False)
            assert got.tolist() == want.tolist(), (h, r, got, want)


def test_selection_capacity_error_is_reported():
    nb = 32
    s = np.tril(np.ones((1, 1, nb, nb), np.float32))
    s /= s.sum(-1, keepdims=True)
    row_ptr, col, nnz = _run_select(s, [1.0], True, cap=10)
    assert nnz == nb * (nb + 1) // 2
    assert (row_ptr == 0).all()
    assert (col == -7).all()                    # nothing written
    assert xa.xattn_get_device_error() == xa.XATTN_ECAPACITY
    assert xa.xattn_get_device_error() == xa.XATTN_OK   # read clears it


ATTN_CASES = [
    # M, C, Hq, Hkv, causal
    (1024, 64, 1, 1, True),
    (1024, 128, 4, 2, True),
    (1536, 128, 2, 1, False),
    (128, 64, 2, 2, True),
    (2048, 128, 8, 8, False),
    (1152, 128, 2, 1, True),     # odd block count: the last query block has no partner
    (1408, 64, 2, 2, False),
]


@pytest.mark.parametrize("M,C,Hq,Hkv,causal", ATTN_CASES)
def test_sparse_attention_on_oracle_mask(M, C, Hq, Hkv, causal):
    """The attention kernel alone: run on the oracle's kept lists."""
    w = small_workload(M, C, Hq, Hkv, 8, causal)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    nb = M // 128
    sc = _oracle_scores(Qb, Kb, w)
    kept = orc.layer_select(sc, np.full(Hq, 0.7), causal)
    row_ptr, col = dict_to_csr(kept, 1, Hq, nb)
    O = poisoned_like(Q)
    lse = poisoned((1, Hq, M))
    xa.xattn_sparse_attn(Q, K, V, row_ptr, col, causal, 1 / math.sqrt(C), O, lse)
    ref = orc.layer_sparse_attention(Qb, Kb, Vb, Hkv, kept, 128, causal, 1 / math.sqrt(C))
    got, glse = bf16_to_np(O), lse.cpu().numpy()
    for h in range(Hq):
        P.assert_outputs_close(got[0, h], ref[(0, h)][0], f"O head {h}")
        np.testing.assert_allclose(glse[0, h], ref[(0, h)][1], rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("M,C,Hq,Hkv,causal", ATTN_CASES)
def test_dense_attention_matches_oracle(M, C, Hq, Hkv, causal):
    w = small_workload(M, C, Hq, Hkv, 8, causal)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    O = poisoned_like(Q)
    lse = poisoned((1, Hq, M))
    xa.xattn_dense_attn(Q, K, V, causal, 1 / math.sqrt(C), O, lse)
    got = bf16_to_np(O)
    grp = Hq // Hkv
    for h in range(Hq):
        q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // grp], Vb[0, h // grp]))
        o, l = orc.dense_attention(q, k, v, causal, 1 / math.sqrt(C))
        P.assert_outputs_close(got[0, h], o, f"dense O head {h}")
        np.testing.assert_allclose(lse.cpu().numpy()[0, h], l, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("C", [64, 128])
def test_attention_skips_invalid_entries_and_empty_rows(C):
    """Invalid entries are skipped, an empty row gives O = 0 and lse = -inf. At
    C = 128 the query blocks run in pairs over the union of their lists, so this
    also covers a pair whose two lists are empty / disjoint / nested."""
    M, Hq = 512, 1
    w = small_workload(M, C, Hq, 1, 8, True)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    nb = 4
    # row 0: empty; row 1: {1}; row 2: {-1, 0, 2, 3(>r), 99}; row 3: {0, 3}
    lists = [[], [1], [-1, 0, 2, 3, 99], [0, 3]]
    rp = torch.tensor(np.concatenate([[0], np.cumsum([len(x) for x in lists])]), dtype=torch.int32,
                      device="cuda")
    ci = torch.tensor(sum(lists, []), dtype=torch.int32, device="cuda")
    O = poisoned_like(Q)
    lse = poisoned((1, Hq, M))
    xa.xattn_sparse_attn(Q, K, V, rp, ci, True, 0.125, O, lse)
    got, gl = bf16_to_np(O)[0, 0], lse.cpu().numpy()[0, 0]
    assert (got[:128] == 0).all() and np.isneginf(gl[:128]).all()
    kept = {1: [1], 2: [0, 2], 3: [0, 3]}
    q, k, v = (orc.bf16_to_f64(x[0, 0]) for x in (Qb, Kb, Vb))
    o, l = orc.block_sparse_attention(q, k, v, kept, 128, True, 0.125, rows=[1, 2, 3])
    P.assert_outputs_close(got[128:], o)
    np.testing.assert_allclose(gl[128:], l, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("causal", [True, False])
def test_sparse_attention_list_order_does_not_matter(causal):
    """Kept lists in descending or shuffled order: every entry of each row is
    still attended exactly once (the two query blocks of a CTA merge their lists
    step by step, which must not depend on the lists being ascending)."""
    M, C, Hq, Hkv = 1280, 128, 2, 1
    w = small_workload(M, C, Hq, Hkv, 8, causal)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    nb = M // 128
    rng = np.random.default_rng(11)
    kept = {}
    for h in range(Hq):
        for r in range(nb):
            n = r + 1 if causal else nb
            pick = sorted(set(rng.choice(n, size=max(1, n // 2), replace=False).tolist()) | {r})
            kept.setdefault((0, h), {})[r] = pick
    rows, ptr = [], [0]
    for h in range(Hq):
        for r in range(nb):
            lst = list(kept[(0, h)][r])
            mode = (r + h) % 3
            if mode == 1:
                lst = lst[::-1]
            elif mode == 2:
                lst = rng.permutation(lst).tolist()
            rows.extend(lst)
            ptr.append(len(rows))
    rp = torch.tensor(ptr, dtype=torch.int32, device="cuda")
    ci = torch.tensor(rows, dtype=torch.int32, device="cuda")
    O = poisoned_like(Q)
    xa.xattn_sparse_attn(Q, K, V, rp, ci, causal, 1 / math.sqrt(C), O)
    got = bf16_to_np(O)
    grp = Hq // Hkv
    for h in range(Hq):
        q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // grp], Vb[0, h // grp]))
        o, _ = orc.block_sparse_attention(q, k, v, kept[(0, h)], 128, causal, 1 / math.sqrt(C))
        P.assert_outputs_close(got[0, h], o, f"O head {h}")


def _pipeline(w, Q, K, V, tau, with_lse=False):
    bufs = _alloc_poisoned(w.B, w.Hq, w.M, w.C, w.stride, w.causal, with_lse=with_lse)
    t = torch.from_numpy(np.asarray(tau, np.float32)).cuda()
    xa.xattn_prefill(Q, K, V, t, w.stride, w.causal, bufs)
    torch.cuda.synchronize()
    return bufs


@pytest.mark.parametrize("name,kw", [
    ("tiny_1h_2k", dict()),                                             # the full tiny workload
    ("llama8b_gqa_32k", dict(M=2048, stride=4, Hq=4, Hkv=2)),
    ("video_dit_118k", dict(M=4096, Hq=3, Hkv=3, frame_tokens=1024)),   # non-causal
    ("llama8b_gqa_256k", dict(M=1536, stride=16, Hq=4, Hkv=2)),         # per-head tau
])
def test_pipeline_end_to_end_small(name, kw):
    """score -> select -> attend on small sizes: every mask row and output element."""
    w = sy.workload(name, **kw)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    tau = sy.tau_vector(w)
    bufs = _pipeline(w, Q, K, V, tau)
    nb = w.nb
    ref_s = _oracle_scores(Qb, Kb, w)
    got_s = bufs.scores.cpu().numpy()
    row_ptr, col = bufs.row_ptr.cpu().numpy(), bufs.col_idx.cpu().numpy()
    log, fails = [], []
    for h in range(w.Hq):
        P.assert_scores_close(got_s[0, h], ref_s[(0, h)], f"scores head {h}")
        for r in range(nb):
            gcols = col[row_ptr[h * nb + r]:row_ptr[h * nb + r + 1]]
            e, f = P.compare_row_mask(gcols, ref_s[(0, h)][r], r, float(tau[h]), w.causal)
            for x in e:
                P.log_exception(f"pipeline {name} M={w.M} S={w.stride}", h, x)
            log += e
            fails += f
    assert not fails, fails[:5]
    assert int(bufs.nnz.item()) == row_ptr[-1]
    # outputs with the GPU's own mask, and with the oracle's mask
    gk = {(0, h): csr_to_dict(row_ptr, col, h, nb) for h in range(w.Hq)}
    ok = orc.layer_select(ref_s, tau, w.causal)
    scale = 1 / math.sqrt(w.C)
    got_o = bf16_to_np(bufs.O)
    ref_gk = orc.layer_sparse_attention(Qb, Kb, Vb, w.Hkv, gk, 128, w.causal, scale)
    for h in range(w.Hq):
        P.assert_outputs_close(got_o[0, h], ref_gk[(0, h)][0], f"O (gpu mask) head {h}")
    rp2, col2 = dict_to_csr(ok, 1, w.Hq, nb)
    O2 = poisoned_like(Q)
    xa.xattn_sparse_attn(Q, K, V, rp2, col2, w.causal, scale, O2)
    ref_ok = orc.layer_sparse_attention(Qb, Kb, Vb, w.Hkv, ok, 128, w.causal, scale)
    got2 = bf16_to_np(O2)
    for h in range(w.Hq):
        P.assert_outputs_close(got2[0, h], ref_ok[(0, h)][0], f"O (oracle mask) head {h}")


def test_tau_one_equals_dense():
    w = small_workload(1024, 128, 2, 1, 8, True)
    (_, _, _), (Q, K, V) = device_inputs(w)
    bufs = _pipeline(w, Q, K, V, [1.0, 1.0])
    O = poisoned_like(Q)
    xa.xattn_dense_attn(Q, K, V, True, 1 / math.sqrt(128), O)
    assert torch.equal(O, bufs.O)
    assert int(bufs.nnz.item()) == 2 * 8 * 9 // 2


def test_repeatable_bits():
    w = small_workload(2048, 128, 4, 2, 8, True)
    (_, _, _), (Q, K, V) = device_inputs(w)
    tau = [0.9] * 4
    a = _pipeline(w, Q, K, V, tau)
    b = _pipeline(w, Q, K, V, tau)
    assert torch.equal(a.scores, b.scores) and torch.equal(a.O, b.O)
    assert torch.equal(a.row_ptr, b.row_ptr)


def test_empty_problem_is_a_no_op():
    Q = poisoned((1, 2, 0, 128), torch.bfloat16)
    O = poisoned_like(Q)
    xa.xattn_dense_attn(Q, Q[:, :1], Q[:, :1], True, 0.1, O)
    scores = poisoned((1, 2, 0, 0))
    ws = poisoned(16, torch.uint8)
    xa.xattn_score(Q, Q[:, :1], 8, True, 0.1, scores, ws)
    assert xa.xattn_get_device_error() == xa.XATTN_OK


@pytest.mark.parametrize("causal", [True, False])
def test_batch_of_two_layers(causal):
    """B = 2: every kernel indexes (batch, head) rows, KV heads and CSR rows by
    batch; each batch element must match the oracle on its own inputs."""
    w = small_workload(1536, 128, 4, 2, 8, causal).with_(B=2)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    tau = np.array([0.9, 0.8, 0.95, 0.7], np.float32)
    bufs = _pipeline(w, Q, K, V, tau, with_lse=True)
    nb = w.nb
    ref_s = _oracle_scores(Qb, Kb, w)
    got_s = bufs.scores.cpu().numpy()
    row_ptr, col = bufs.row_ptr.cpu().numpy(), bufs.col_idx.cpu().numpy()
    fails = []
    kept_gpu = {}
    for b in range(2):
        for h in range(w.Hq):
            P.assert_scores_close(got_s[b, h], ref_s[(b, h)], f"scores b{b} h{h}")
            bh = b * w.Hq + h
            kept_gpu[(b, h)] = csr_to_dict(row_ptr, col, bh, nb)
            for r in range(nb):
                _, f = P.compare_row_mask(kept_gpu[(b, h)][r], ref_s[(b, h)][r], r, float(tau[h]),
                                          causal)
                fails += f
    assert not fails, fails[:5]
    ref_o = orc.layer_sparse_attention(Qb, Kb, Vb, w.Hkv, kept_gpu, 128, causal, 1 / math.sqrt(w.C))
    got_o = bf16_to_np(bufs.O)
    got_l = bufs.lse.cpu().numpy()
    for (b, h), (o, l) in ref_o.items():
        P.assert_outputs_close(got_o[b, h], o, f"O b{b} h{h}")
        np.testing.assert_allclose(got_l[b, h], l, rtol=1e-4, atol=1e-4)
