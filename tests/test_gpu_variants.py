"""GPU parity of the ablation variants the pages compare against: diagonal-pattern
scoring, and Top-K / fixed-ratio block selection (XAttention summary, "Measured
effects" table; DuSA rebuttal, Response to Q2); the fused score+select entry point;
and GQA-shared kept lists, a variant the pages do not define."""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from tests import parity as P
from tests.gpu_util import (bf16_to_np, csr_to_dict, device_inputs, dict_to_csr, poisoned,
                            poisoned_like, small_workload)

pytestmark = pytest.mark.gpu

xa = pytest.importorskip("block_sparse_long_04_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    assert xa.xattn_get_device_error() == xa.XATTN_OK


@pytest.mark.parametrize("M,C,Hq,Hkv,S,causal", [
    (2048, 64, 1, 1, 8, True),
    (1152, 128, 4, 2, 8, True),
    (1024, 128, 2, 1, 4, False),
    (640, 64, 2, 2, 16, True),
    (8320, 128, 2, 1, 64, True),
])
def test_diagonal_pattern_scores(M, C, Hq, Hkv, S, causal):
    w = small_workload(M, C, Hq, Hkv, S, causal)
    (Qb, Kb, _), (Q, K, _) = device_inputs(w)
    nb = M // 128
    sig = orc.default_score_scale(S, C)
    scores = poisoned((1, Hq, nb, nb))
    ws = poisoned(xa.xattn_score_workspace_size(1, Hq, M, S, causal), torch.uint8)
    xa.xattn_score_ex(Q, K, S, causal, xa.XATTN_PATTERN_DIAGONAL, sig, scores, ws)
    diag = scores.cpu().numpy()
    ref = orc.layer_block_scores(Qb, Kb, Hkv, S, 128, sig, causal, antidiagonal=False)
    for h in range(Hq):
        P.assert_scores_close(diag[0, h], ref[(0, h)], f"diagonal scores head {h}")
    # and the antidiagonal pattern through the same entry point is xattn_score
    anti = poisoned_like(scores)
    xa.xattn_score_ex(Q, K, S, causal, xa.XATTN_PATTERN_ANTIDIAGONAL, sig, anti, ws)
    base = poisoned_like(scores)
    xa.xattn_score(Q, K, S, causal, sig, base, ws)
    assert torch.equal(anti, base)
    if M >= 1024:
        assert not torch.allclose(anti, scores)


def _select_ex(scores_np, param, rule, causal):
    B, Hq, nb, _ = scores_np.shape
    sc = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).cuda()
    pr = torch.tensor(param, dtype=torch.float32, device="cuda")
    row_ptr = poisoned(B * Hq * nb + 1, torch.int32)
    col = poisoned(xa.max_kept(B, Hq, nb, causal), torch.int32)
    nnz = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = poisoned(xa.xattn_select_workspace_size(B, Hq, nb), torch.uint8)
    xa.xattn_select_ex(sc, pr, rule, causal, row_ptr, col, nnz, ws)
    return row_ptr.cpu().numpy(), col.cpu().numpy(), int(nnz.item())


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nb", [1, 5, 64, 333])
def test_topk_and_ratio_selection_exact(causal, nb):
    """Top-K and ratio depend on the ranking only: bit-exact against the oracle
    given the same fp32 scores (ties included)."""
    rng = np.random.default_rng(nb * 3 + causal)
    Hq = 3
    s = rng.gamma(0.3, size=(1, Hq, nb, nb))
    s[0, 2] = np.round(s[0, 2] * 4) / 4          # head 2: many exact ties
    if causal:
        s = np.tril(s)
    s = (s / np.maximum(s.sum(-1, keepdims=True), 1e-30)).astype(np.float32)
    s64 = s.astype(np.float64)
    for rule, param, fn in ((xa.XATTN_SELECT_TOPK, [1.0, 7.5, 3.0], orc.select_row_topk),
                            (xa.XATTN_SELECT_RATIO, [0.1, 0.33, 1.0], orc.select_row_ratio)):
        rp, col, nnz = _select_ex(s, param, rule, causal)
        assert nnz == rp[-1]
        for h in range(Hq):
            p = np.float32(param[h])
            for r in range(nb):
                want = fn(s64[0, h, r], r, int(np.floor(p)) if rule == xa.XATTN_SELECT_TOPK
                          else float(p), causal)
                got = col[rp[h * nb + r]:rp[h * nb + r + 1]]
                np.testing.assert_array_equal(got, want, err_msg=f"rule {rule} h{h} r{r}")


def test_threshold_rule_equals_select():
    rng = np.random.default_rng(1)
    nb, Hq = 200, 2
    s = np.tril(rng.gamma(0.3, size=(1, Hq, nb, nb)))
    s = (s / s.sum(-1, keepdims=True)).astype(np.float32)
    a = _select_ex(s, [0.9, 0.6], xa.XATTN_SELECT_THRESHOLD, True)
    sc = torch.from_numpy(s).cuda()
    tau = torch.tensor([0.9, 0.6], device="cuda")
    row_ptr = poisoned(Hq * nb + 1, torch.int32)
    col = poisoned(xa.max_kept(1, Hq, nb, True), torch.int32)
    nnz = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = poisoned(xa.xattn_select_workspace_size(1, Hq, nb), torch.uint8)
    xa.xattn_select(sc, tau, True, row_ptr, col, nnz, ws)
    n = int(nnz.item())
    assert a[2] == n
    np.testing.assert_array_equal(a[0], row_ptr.cpu().numpy())
    np.testing.assert_array_equal(a[1][:n], col.cpu().numpy()[:n])


@pytest.mark.parametrize("M,C,Hq,Hkv,S,causal,B", [
    (2048, 64, 1, 1, 8, True, 1),
    (1152, 128, 4, 2, 8, True, 2),      # ragged score tile, two batch elements
    (1024, 128, 2, 1, 4, False, 1),
    (4096, 128, 4, 2, 16, True, 1),
])
def test_fused_score_select_equals_two_calls_and_oracle(M, C, Hq, Hkv, S, causal, B):
    w = small_workload(M, C, Hq, Hkv, S, causal).with_(B=B)
    (Qb, Kb, _), (Q, K, _) = device_inputs(w)
    nb = M // 128
    sig = orc.default_score_scale(S, C)
    ref_s = orc.layer_block_scores(Qb, Kb, Hkv, S, 128, sig, causal)
    rules = ((xa.XATTN_SELECT_THRESHOLD, [0.9, 0.7, 0.95, 0.6][:Hq]),
             (xa.XATTN_SELECT_TOPK, [3.0, 1.0, 5.0, 2.0][:Hq]),
             (xa.XATTN_SELECT_RATIO, [0.25, 0.5, 0.1, 1.0][:Hq]))
    cap = xa.max_kept(B, Hq, nb, causal)
    for rule, prm in rules:
        param = torch.tensor(prm, dtype=torch.float32, device="cuda")
        # reference: the two separate calls
        sc1 = poisoned((B, Hq, nb, nb))
        ws1 = poisoned(xa.xattn_score_workspace_size(B, Hq, M, S, causal), torch.uint8)
        xa.xattn_score(Q, K, S, causal, sig, sc1, ws1)
        rp1 = poisoned(B * Hq * nb + 1, torch.int32)
        ci1 = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        nz1 = torch.zeros(1, dtype=torch.int32, device="cuda")
        wss = poisoned(xa.xattn_select_workspace_size(B, Hq, nb), torch.uint8)
        xa.xattn_select_ex(sc1, param, rule, causal, rp1, ci1, nz1, wss)
        # fused
        sc2 = poisoned_like(sc1)
        rp2 = poisoned_like(rp1)
        ci2 = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        nz2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws2 = poisoned(xa.xattn_score_select_workspace_size(B, Hq, M, S, causal), torch.uint8)
        xa.xattn_score_select(Q, K, param, rule, S, causal, sig, sc2, rp2, ci2, nz2, ws2)
        torch.cuda.synchronize()
        n = int(nz1.item())
        assert torch.equal(sc1, sc2)
        assert int(nz2.item()) == n and torch.equal(rp1, rp2)
        assert torch.equal(ci1[:n], ci2[:n])
        # the fused lists against the oracle: the threshold rule on the oracle's own
        # scores (mask-exception rules), Top-K / ratio (ranking only) exactly on the
        # scores the GPU ranked
        rp, ci = rp2.cpu().numpy(), ci2.cpu().numpy()
        got_s = sc2.cpu().numpy().astype(np.float64)
        fails = []
        for b in range(B):
            for h in range(Hq):
                bh = b * Hq + h
                for r in range(nb):
                    gk = ci[rp[bh * nb + r]:rp[bh * nb + r + 1]]
                    if rule == xa.XATTN_SELECT_THRESHOLD:
                        e, f = P.compare_row_mask(gk, ref_s[(b, h)][r], r, float(np.float32(prm[h])),
                                                  causal)
                        for x in e:
                            P.log_exception(f"fused M={M} S={S} B={B}", h, x)
                        fails += f
                    elif rule == xa.XATTN_SELECT_TOPK:
                        want = orc.select_row_topk(got_s[b, h, r], r, int(prm[h]), causal)
                        assert gk.tolist() == want.tolist(), (b, h, r)
                    else:
                        want = orc.select_row_ratio(got_s[b, h, r], r, float(np.float32(prm[h])),
                                                    causal)
                        assert gk.tolist() == want.tolist(), (b, h, r)
        assert not fails, fails[:5]


def _select_group(scores_np, param, rule, Hkv, causal):
    B, Hq, nb, _ = scores_np.shape
    sc = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).cuda()
    pr = torch.tensor(param, dtype=torch.float32, device="cuda")
    row_ptr = poisoned(B * Hkv * nb + 1, torch.int32)
    col = torch.full((xa.max_kept(B, Hkv, nb, causal),), -7, dtype=torch.int32, device="cuda")
    nnz = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = poisoned(xa.xattn_select_group_workspace_size(B, Hq, Hkv, nb), torch.uint8)
    xa.xattn_select_group(sc, pr, rule, Hkv, causal, row_ptr, col, nnz, ws)
    return row_ptr.cpu().numpy(), col.cpu().numpy(), int(nnz.item())


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nb,B", [(1, 1), (17, 1), (300, 2)])
def test_group_selection_is_the_union_of_the_heads(causal, nb, B):
    """GQA-shared lists (a variant): with Top-K (ranking only) bit-exact against
    the oracle's union; with the threshold rule, exactly the union of the lists
    the per-head entry point returns on the same scores."""
    Hq, Hkv = 4, 2
    rng = np.random.default_rng(nb * 7 + B + causal)
    s = rng.gamma(0.3, size=(B, Hq, nb, nb))
    if causal:
        s = np.tril(s)
    s = (s / s.sum(-1, keepdims=True)).astype(np.float32)
    s64 = s.astype(np.float64)
    k_param = [3.0, 1.0, 5.0, 2.0]
    rp, col, nnz = _select_group(s, k_param, xa.XATTN_SELECT_TOPK, Hkv, causal)
    assert rp[0] == 0 and rp[-1] == nnz
    kept = {(b, h): {r: orc.select_row_topk(s64[b, h, r], r, int(k_param[h]), causal)
                     for r in range(nb)} for b in range(B) for h in range(Hq)}
    union = orc.layer_select_group(kept, Hq, Hkv)
    for b in range(B):
        for kvh in range(Hkv):
            got = csr_to_dict(rp, col, b * Hkv + kvh, nb)
            for r in range(nb):
                assert got[r].tolist() == union[(b, kvh)][r].tolist(), (b, kvh, r)
    tau = [0.9, 0.6, 0.95, 0.8]
    rp, col, nnz = _select_group(s, tau, xa.XATTN_SELECT_THRESHOLD, Hkv, causal)
    hrp, hcol, _ = _select_ex(s, tau, xa.XATTN_SELECT_THRESHOLD, causal)
    per_head = {(b, h): csr_to_dict(hrp, hcol, b * Hq + h, nb) for b in range(B) for h in range(Hq)}
    union = orc.layer_select_group(per_head, Hq, Hkv)
    for b in range(B):
        for kvh in range(Hkv):
            got = csr_to_dict(rp, col, b * Hkv + kvh, nb)
            for r in range(nb):
                assert got[r].tolist() == union[(b, kvh)][r].tolist(), (b, kvh, r)
    assert nnz == sum(len(v[r]) for v in union.values() for r in range(nb))


@pytest.mark.parametrize("M,C,Hq,Hkv,causal", [
    (1536, 128, 4, 2, True),
    (1152, 64, 4, 1, False),
])
def test_group_attention_matches_oracle(M, C, Hq, Hkv, causal):
    """Attention over GQA-shared lists: every head of a group attends over the
    group's union list."""
    w = small_workload(M, C, Hq, Hkv, 8, causal)
    (Qb, Kb, Vb), (Q, K, V) = device_inputs(w)
    nb = M // 128
    sig = orc.default_score_scale(8, C)
    sc = orc.layer_block_scores(Qb, Kb, Hkv, 8, 128, sig, causal)
    kept = orc.layer_select(sc, np.full(Hq, 0.7), causal)
    union = orc.layer_select_group(kept, Hq, Hkv)
    row_ptr, col = dict_to_csr(union, 1, Hkv, nb)
    O = poisoned_like(Q)
    lse = poisoned((1, Hq, M))
    xa.xattn_sparse_attn_group(Q, K, V, row_ptr, col, causal, 1 / math.sqrt(C), O, lse)
    grp = Hq // Hkv
    by_head = {(0, h): union[(0, h // grp)] for h in range(Hq)}
    ref = orc.layer_sparse_attention(Qb, Kb, Vb, Hkv, by_head, 128, causal, 1 / math.sqrt(C))
    got, glse = bf16_to_np(O), lse.cpu().numpy()
    for h in range(Hq):
        P.assert_outputs_close(got[0, h], ref[(0, h)][0], f"O head {h}")
        np.testing.assert_allclose(glse[0, h], ref[(0, h)][1], rtol=1e-4, atol=1e-4)


def test_group_selection_capacity_error_is_reported():
    """A col_idx too small for the shared lists: nnz written, every list
    withdrawn (row_ptr zero), nothing written to col_idx, ECAPACITY raised."""
    B, Hq, Hkv, nb = 1, 4, 2, 24
    s = np.tril(np.ones((B, Hq, nb, nb), np.float32))
    s /= s.sum(-1, keepdims=True)
    sc = torch.from_numpy(s).cuda()
    pr = torch.ones(Hq, dtype=torch.float32, device="cuda")
    row_ptr = poisoned(B * Hkv * nb + 1, torch.int32)
    col = torch.full((10,), -7, dtype=torch.int32, device="cuda")
    nnz = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = poisoned(xa.xattn_select_group_workspace_size(B, Hq, Hkv, nb), torch.uint8)
    xa.xattn_select_group(sc, pr, xa.XATTN_SELECT_THRESHOLD, Hkv, True, row_ptr, col, nnz, ws)
    torch.cuda.synchronize()
    assert int(nnz.item()) == B * Hkv * nb * (nb + 1) // 2
    assert (row_ptr == 0).all() and (col == -7).all()
    assert xa.xattn_get_device_error() == xa.XATTN_ECAPACITY
    assert xa.xattn_get_device_error() == xa.XATTN_OK
