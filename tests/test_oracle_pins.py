"""Pins for the CPU fp64 oracle, each against something other than the oracle itself.

Pins: the hand-worked fixture in tests/golden; the geometry of the antidiagonal
(XAttention abstract: lower-left to upper-right) on one-hot inputs; brute-force
antidiagonal walks over an explicitly looped q k^T; closed forms for Q = 0; the
stride-1 special case, which is the textbook softmax attention mass per block;
brute-force search over all subsets for the minimal-set selection; and the
textbook attention (torch fp64 scaled_dot_product_attention) for the sparse
attention with every block kept. The last tests plant mistakes in the oracle
(on the CPU) and check that the pins above catch them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax as sp_softmax, logsumexp

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "reshape_and_tiny_example.json")


def _rand(shape, seed, ints=False):
    rng = np.random.default_rng(seed)
    if ints:
        return rng.integers(-3, 4, size=shape).astype(np.float64)
    return rng.standard_normal(shape)


# ----------------------------------------------------------------- golden
def test_golden_reshape_shapes():
    g = json.load(open(GOLDEN))["reshape_shapes"]
    for c in g["cases"]:
        M, C, S = c["M"], c["C"], c["stride"]
        q = np.zeros((M, C), np.float32)
        qv, kv = orc.strided_views(q, q, S)
        assert [c["B"], c["H"], *qv.shape] == c["reshaped"]
        assert [c["B"], c["H"], *kv.shape] == c["reshaped"]


def test_golden_tiny_example():
    g = json.load(open(GOLDEN))["tiny_example"]
    q = np.array(g["q"], float)[:, None]
    k = np.array(g["k"], float)[:, None]
    S, b = g["stride"], g["block"]
    X = orc.antidiagonal_logits(q, k, S, 1.0, causal=False)
    np.testing.assert_array_equal(X, np.array(g["X_antidiagonal"], float))
    Xd = orc.antidiagonal_logits(q, k, S, 1.0, causal=False, antidiagonal=False)
    np.testing.assert_array_equal(Xd, np.array(g["X_diagonal"], float))
    ev = lambda s: eval(s, {"exp": math.exp})  # closed forms written in the fixture
    sc = orc.block_scores(q, k, S, b, 1.0, causal=True)
    want = np.array([[ev(x) for x in row] for row in g["scores_causal_closed_form"]])
    np.testing.assert_allclose(sc, want, rtol=1e-14, atol=1e-300)
    sn = orc.block_scores(q, k, S, b, 1.0, causal=False)
    np.testing.assert_allclose(sn[0], [ev(x) for x in g["scores_noncausal_row0_closed_form"]],
                               rtol=1e-14)
    kc = orc.select_blocks(sc, g["tau"], causal=True)
    assert [list(kc[r]) for r in range(2)] == g["kept_causal"]
    kn = orc.select_blocks(sn, g["tau"], causal=False)
    assert [list(kn[r]) for r in range(2)] == g["kept_noncausal"]


# ------------------------------------------------------- a1 + a2 geometry
@pytest.mark.parametrize("S", [2, 4])
@pytest.mark.parametrize("antidiagonal", [True, False])
def test_one_hot_lights_the_right_tile_entry(S, antidiagonal):
    """q = E, k = I gives q k^T = E; a one at (a, b) must reach X[a//S, b//S] iff
    (a, b) lies on the antidiagonal of its S x S tile, i.e. local row + local col
    = S-1 (lower-left (S-1, 0) to upper-right (0, S-1)); for the diagonal variant
    iff local row = local col."""
    M = 4 * S
    eye = np.eye(M)
    for a in range(M):
        for bcol in range(M):
            E = np.zeros((M, M))
            E[a, bcol] = 1.0
            X = orc.antidiagonal_logits(E, eye, S, 1.0, causal=False, antidiagonal=antidiagonal)
            lr, lc = a % S, bcol % S
            on = (lr + lc == S - 1) if antidiagonal else (lr == lc)
            want = np.zeros((M // S, M // S))
            if on:
                want[a // S, bcol // S] = 1.0
            np.testing.assert_array_equal(X, want)


@pytest.mark.parametrize("S", [2, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_antidiagonal_bruteforce_walk(S, causal):
    M, C = 4 * S, 3
    q = _rand((M, C), 10 + S, ints=True)
    k = _rand((M, C), 20 + S, ints=True)
    A = [[sum(q[i, d] * k[j, d] for d in range(C)) for j in range(M)] for i in range(M)]
    X = orc.antidiagonal_logits(q, k, S, 1.0, causal=causal)
    r = M // S
    for ip in range(r):
        for jp in range(r):
            if causal and jp > ip:
                assert X[ip, jp] == -np.inf
                continue
            row, col, tot = ip * S + S - 1, jp * S, 0.0
            for _ in range(S):               # walk up and to the right
                tot += A[row][col]
                row, col = row - 1, col + 1
            assert X[ip, jp] == tot


def test_scale_multiplies_logits():
    q, k = _rand((32, 4), 1), _rand((32, 4), 2)
    X1 = orc.antidiagonal_logits(q, k, 4, 1.0, causal=False)
    X3 = orc.antidiagonal_logits(q, k, 4, 0.37, causal=False)
    np.testing.assert_allclose(X3, 0.37 * X1, rtol=1e-15)


# ------------------------------------------------------------- a3 + a4
@pytest.mark.parametrize("S,b", [(2, 8), (4, 16), (8, 32), (4, 4), (1, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_block_rows_sum_to_one(S, b, causal):
    M, C = 8 * b, 8
    q, k = _rand((M, C), 3), _rand((M, C), 4)
    s = orc.block_scores(q, k, S, b, 0.7, causal)
    np.testing.assert_allclose(s.sum(axis=1), 1.0, atol=1e-12)
    assert (s >= 0).all()
    if causal:
        assert np.all(s[np.triu_indices(M // b, 1)] == 0.0)


@pytest.mark.parametrize("S,b", [(2, 8), (4, 16), (8, 32)])
def test_zero_query_closed_forms(S, b):
    """Q = 0 makes every visible logit equal. Non-causal: every score is 1/nb.
    Causal: reshaped row i' sees i'+1 columns, n_c(i') of them in block c, so
    score[r, c] = (1/g) * sum_{i' in r} n_c(i')/(i'+1)."""
    M, C = 6 * b, 5
    q = np.zeros((M, C))
    k = _rand((M, C), 5)
    nb, g = M // b, b // S
    s = orc.block_scores(q, k, S, b, 1.0, causal=False)
    np.testing.assert_allclose(s, np.full((nb, nb), 1.0 / nb), rtol=1e-13)
    s = orc.block_scores(q, k, S, b, 1.0, causal=True)
    want = np.zeros((nb, nb))
    for r in range(nb):
        for ip in range(r * g, (r + 1) * g):
            for c in range(nb):
                n_c = max(0, min(ip + 1, (c + 1) * g) - c * g)
                want[r, c] += n_c / (ip + 1) / g
    np.testing.assert_allclose(s, want, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_stride_one_is_textbook_block_mass(causal):
    """With stride 1 the reshape is the identity, so the scores must be the usual
    softmax attention probabilities summed over each b x b block and averaged
    over the block's b rows (scipy softmax on the full logit matrix)."""
    M, C, b = 96, 16, 16
    q, k = _rand((M, C), 6), _rand((M, C), 7)
    scale = 1 / math.sqrt(C)
    L = scale * np.einsum("id,jd->ij", q, k)
    if causal:
        L = np.where(np.tril(np.ones((M, M), bool)), L, -np.inf)
    P = sp_softmax(L, axis=1)
    nb = M // b
    want = P.reshape(nb, b, nb, b).sum(axis=(1, 3)) / b
    s = orc.block_scores(q, k, 1, b, scale, causal)
    np.testing.assert_allclose(s, want, rtol=1e-12, atol=1e-15)


def test_row_subset_matches_full():
    M, C, S, b = 256, 8, 4, 32
    q, k = _rand((M, C), 8), _rand((M, C), 9)
    full = orc.block_scores(q, k, S, b, 0.3, True)
    part = orc.block_scores(q, k, S, b, 0.3, True, rows=[0, 3, 7])
    for r in (0, 3, 7):
        np.testing.assert_allclose(part[r], full[r], rtol=1e-14)
    assert np.isnan(part[1]).all()


# ------------------------------------------------------------------- a5
def _brute_min_sets(row, cand, tau):
    """All minimal-cardinality subsets of cand with mass >= tau."""
    for n in range(1, len(cand) + 1):
        hits = [set(T) for T in itertools.combinations(cand, n) if sum(row[list(T)]) >= tau]
        if hits:
            return n, hits
    return len(cand), [set(cand)]


@pytest.mark.parametrize("seed", range(40))
def test_selection_is_a_minimal_set(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(2, 11))
    causal = bool(seed % 2)
    r = int(rng.integers(0, nb))
    row = rng.gamma(0.5, size=nb)
    if causal:
        row[r + 1:] = 0.0
    row /= row.sum()
    tau = float(rng.uniform(0.05, 0.99))
    kept = set(orc.select_row(row, r, tau, causal).tolist())
    cand = list(range(r + 1)) if causal else list(range(nb))
    n, hits = _brute_min_sets(row, cand, tau)
    # the threshold set is `kept` itself, or `kept` without the forced diagonal
    T = kept if kept in hits else kept - {r}
    assert T in hits and len(T) == n
    best = max(sum(row[list(H)]) for H in hits)
    assert math.isclose(sum(row[list(T)]), best, rel_tol=1e-12)
    assert r in kept and kept <= set(cand)


def test_selection_special_cases():
    row = np.array([0.1, 0.4, 0.2, 0.3])
    # tau = 1 keeps all candidates
    assert orc.select_row(row, 3, 1.0, True).tolist() == [0, 1, 2, 3]
    assert orc.select_row(row, 1, 1.0, True).tolist() == [0, 1]
    # tau -> 0+ keeps the arg-max plus the diagonal
    assert orc.select_row(row, 0, 1e-9, False).tolist() == [0, 1]
    assert orc.select_row(row, 1, 1e-9, False).tolist() == [1]
    # ties go to the smaller index
    tie = np.array([0.3, 0.3, 0.2, 0.2])
    assert orc.select_row(tie, 3, 0.25, False).tolist() == [0, 3]
    assert orc.select_row(tie, 0, 0.55, False).tolist() == [0, 1]
    # reaching tau exactly stops the prefix (>=)
    exact = np.array([0.5, 0.25, 0.25])
    assert orc.select_row(exact, 0, 0.75, False).tolist() == [0, 1]


@pytest.mark.parametrize("seed", range(30))
def test_topk_and_ratio_keep_the_heaviest_k(seed):
    """Brute force over all k-subsets: the Top-K set has the largest mass among
    sets of its size, and the ratio rule keeps ceil(ratio * candidates)."""
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(2, 10))
    causal = bool(seed % 2)
    r = int(rng.integers(0, nb))
    row = rng.gamma(0.5, size=nb)
    if causal:
        row[r + 1:] = 0.0
    row /= row.sum()
    cand = list(range(r + 1)) if causal else list(range(nb))
    k = int(rng.integers(1, len(cand) + 2))
    kept = set(orc.select_row_topk(row, r, k, causal).tolist())
    n = min(k, len(cand))
    T = kept if len(kept) == n else kept - {r}
    assert len(T) == n and T <= set(cand) and r in kept
    best = max(sum(row[list(H)]) for H in itertools.combinations(cand, n))
    assert math.isclose(sum(row[list(T)]), best, rel_tol=1e-12)
    ratio = float(rng.uniform(0.01, 1.0))
    kr = set(orc.select_row_ratio(row, r, ratio, causal).tolist())
    nr = math.ceil(ratio * len(cand))
    assert len(kr - {r}) in (nr, nr - 1) and len(kr) in (nr, nr + 1)


def test_topk_ratio_special_cases():
    row = np.array([0.1, 0.4, 0.2, 0.3])
    assert orc.select_row_topk(row, 0, 1, False).tolist() == [0, 1]
    assert orc.select_row_topk(row, 3, 2, False).tolist() == [1, 3]
    assert orc.select_row_topk(row, 3, 99, False).tolist() == [0, 1, 2, 3]
    assert orc.select_row_topk(row, 2, 0, True).tolist() == [1, 2]      # at least one
    assert orc.select_row_ratio(row, 0, 0.5, False).tolist() == [0, 1, 3]
    assert orc.select_row_ratio(row, 0, 1.0, False).tolist() == [0, 1, 2, 3]
    assert orc.ratio_count(1e-9, 5) == 1 and orc.ratio_count(0.2, 10) == 2
    tie = np.array([0.25, 0.25, 0.25, 0.25])
    assert orc.select_row_topk(tie, 3, 2, False).tolist() == [0, 1, 3]


def test_margins_agree_with_selection():
    rng = np.random.default_rng(3)
    for _ in range(50):
        nb = 12
        row = rng.dirichlet(np.full(nb, 0.3))
        r = int(rng.integers(0, nb))
        tau = float(rng.uniform(0.1, 0.95))
        margin, pos = orc.selection_margins(row, r, tau, causal=False)
        by_margin = set(np.nonzero(margin < 0)[0].tolist()) | {r}
        assert by_margin == set(orc.select_row(row, r, tau, False).tolist())


def test_csr():
    rp, ci = orc.to_csr([np.array([0]), np.array([0, 1]), np.array([2])])
    assert rp.tolist() == [0, 1, 3, 4] and ci.tolist() == [0, 0, 1, 2]
    assert rp.dtype == np.int32 and ci.dtype == np.int32


# ------------------------------------------------------------------- a6
def _sdpa(q, k, v, causal, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=causal, scale=scale)
    return o[0, 0].numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_all_blocks_kept_is_textbook_attention(causal):
    M, C, b = 128, 16, 16
    q, k, v = _rand((M, C), 11), _rand((M, C), 12), _rand((M, C), 13)
    scale = 1 / math.sqrt(C)
    nb = M // b
    sc = orc.block_scores(q, k, 4, b, 0.5, causal)
    kept = orc.select_blocks(sc, 1.0, causal)       # tau = 1 keeps every candidate
    O, lse = orc.block_sparse_attention(q, k, v, kept, b, causal, scale)
    np.testing.assert_allclose(O, _sdpa(q, k, v, causal, scale), atol=1e-12)
    L = scale * q @ k.T
    if causal:
        L = np.where(np.tril(np.ones((M, M), bool)), L, -np.inf)
    np.testing.assert_allclose(lse, logsumexp(L, axis=1), rtol=1e-13)
    Od, _ = orc.dense_attention(q, k, v, causal, scale, block=b)
    np.testing.assert_allclose(Od, O, atol=1e-13)
    assert all(len(kept[r]) == (r + 1 if causal else nb) for r in range(nb))


def test_one_block_per_row_is_attention_on_that_block():
    M, C, b = 96, 8, 16
    q, k, v = _rand((M, C), 14), _rand((M, C), 15), _rand((M, C), 16)
    scale = 0.3
    nb = M // b
    rng = np.random.default_rng(0)
    for causal in (False, True):
        kept = {}
        for r in range(nb):
            kept[r] = np.array([r if causal and r == 0 else int(rng.integers(0, r + 1 if causal else nb))])
        O, _ = orc.block_sparse_attention(q, k, v, kept, b, causal, scale)
        for r in range(nb):
            c = int(kept[r][0])
            ks, vs = k[c * b:(c + 1) * b], v[c * b:(c + 1) * b]
            want = _sdpa(q[r * b:(r + 1) * b], ks, vs, causal and c == r, scale)
            np.testing.assert_allclose(O[r * b:(r + 1) * b], want, atol=1e-12)


def test_unit_values_give_unit_output():
    M, C, b = 64, 8, 16
    q, k = 3 * _rand((M, C), 17), 3 * _rand((M, C), 18)
    v = np.ones((M, C))
    kept = {0: np.array([0]), 1: np.array([1]), 2: np.array([0, 2]), 3: np.array([1, 2, 3])}
    O, _ = orc.block_sparse_attention(q, k, v, kept, b, True, 1.0)
    np.testing.assert_allclose(O, 1.0, rtol=1e-14)


def test_bf16_widening_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F], np.uint16)
    want = [1.0, -1.0, 3.140625, 2.0 ** -133, 3.3895313892515355e38]
    np.testing.assert_array_equal(orc.bf16_to_f64(bits), want)


# ------------------------------------------- planted mistakes must be caught
def test_planted_forward_query_view_is_caught(monkeypatch):
    """Dropping the row reversal turns antidiagonals into diagonals; the one-hot
    geometry pin must fail."""
    real = orc.strided_views
    monkeypatch.setattr(orc.xattn_oracle, "strided_views",
                        lambda q, k, s, antidiagonal=True: real(q, k, s, False))
    with pytest.raises(AssertionError):
        test_one_hot_lights_the_right_tile_entry(4, True)


def test_planted_missing_normalisation_is_caught(monkeypatch):
    """Summing block mass without the 1/g factor breaks the row-sum pin."""
    real = orc.xattn_oracle.block_scores

    def wrong(q, k, stride, block, *a, **kw):
        return real(q, k, stride, block, *a, **kw) * (block // stride)
    monkeypatch.setattr(orc, "block_scores", wrong)
    with pytest.raises(AssertionError):
        test_block_rows_sum_to_one(4, 16, True)


def test_planted_wrong_tie_break_is_caught(monkeypatch):
    """Ascending instead of descending order breaks the minimal-set pin."""
    monkeypatch.setattr(orc.xattn_oracle, "_greedy_order",
                        lambda row, cand: cand[np.lexsort((cand, row[cand]))])
    with pytest.raises(AssertionError):
        for seed in range(40):
            test_selection_is_a_minimal_set(seed)


def test_group_union_hand_example_and_threshold_mass():
    """GQA-shared selection: a hand-worked union, and every member head still
    covers its own threshold mass over the shared list (checked on the scores,
    independently of how the union is formed)."""
    got = orc.select_group_union([{0: np.array([0]), 3: np.array([0, 3])},
                                  {0: np.array([0]), 3: np.array([1, 3])},
                                  {0: np.array([0]), 3: np.array([3])}])
    assert got[0].tolist() == [0] and got[3].tolist() == [0, 1, 3]
    rng = np.random.default_rng(5)
    nb, G = 9, 4
    for causal in (True, False):
        scores = [rng.gamma(0.4, size=(nb, nb)) for _ in range(G)]
        if causal:
            scores = [np.tril(x) for x in scores]
        scores = [x / x.sum(axis=1, keepdims=True) for x in scores]
        taus = [0.5, 0.7, 0.9, 0.95]
        kept = [orc.select_blocks(scores[i], taus[i], causal) for i in range(G)]
        union = orc.select_group_union(kept)
        for r in range(nb):
            u = union[r].tolist()
            assert u == sorted(set(u)) and r in u
            assert all(0 <= c <= (r if causal else nb - 1) for c in u)
            for i in range(G):
                assert scores[i][r, u].sum() >= taus[i] - 1e-12
                assert set(kept[i][r].tolist()) <= set(u)
            # no block that no member kept
            assert set(u) <= set().union(*(set(kept[i][r].tolist()) for i in range(G)))
        # a group of one is the head's own selection
        solo = orc.select_group_union([kept[0]])
        assert all(solo[r].tolist() == kept[0][r].tolist() for r in range(nb))


def test_layer_group_maps_heads_to_their_kv_head():
    kept = {(0, h): {0: np.array([0]), 1: np.array([h % 2, 1])} for h in range(4)}
    g = orc.layer_select_group(kept, Hq=4, Hkv=2)
    assert sorted(g) == [(0, 0), (0, 1)]
    assert g[(0, 0)][1].tolist() == [0, 1] and g[(0, 1)][1].tolist() == [0, 1]
    kept[(0, 2)][1] = np.array([1])
    kept[(0, 3)][1] = np.array([1])
    assert orc.layer_select_group(kept, Hq=4, Hkv=2)[(0, 1)][1].tolist() == [1]


# ------------------------------------------------ layer wrappers (GQA, per-head tau)
# Query head -> KV head for Hq = 4 query heads sharing Hkv = 2 KV heads, written out
# by hand: heads 0 and 1 read KV head 0, heads 2 and 3 read KV head 1 (the GQA head
# sharing of the Llama-shaped workloads; each query head keeps its own threshold,
# XAttention summary, "Approach").
_GQA_KV_OF = {0: 0, 1: 0, 2: 1, 3: 1}
_GQA_TAU = np.array([0.35, 0.6, 0.85, 0.97])


def _gqa_layer(seed=21, B=2, M=96, C=8):
    import synthetic as sy
    rng = np.random.default_rng(seed)
    # KV heads differ strongly (their own scale and offset), so a wrong head mapping
    # moves every score, kept list and output
    Q = rng.standard_normal((B, 4, M, C)).astype(np.float32)
    K = rng.standard_normal((B, 2, M, C)).astype(np.float32)
    V = rng.standard_normal((B, 2, M, C)).astype(np.float32)
    K[:, 1] = 2.5 * K[:, 1] + 1.0
    V[:, 1] = V[:, 1] - 3.0
    return sy.bf16_round(Q), sy.bf16_round(K), sy.bf16_round(V)


@pytest.mark.parametrize("causal", [True, False])
def test_layer_wrappers_map_query_heads_and_taus(causal):
    """layer_block_scores / layer_select / layer_sparse_attention on a B = 2,
    Hq = 4, Hkv = 2 layer equal the single-head functions called on hand-sliced
    (q of head h, k and v of KV head _GQA_KV_OF[h]) with that head's own tau."""
    S, b = 4, 16
    Qb, Kb, Vb = _gqa_layer()
    B = Qb.shape[0]
    sig, sa = 0.3, 0.25
    scores = orc.layer_block_scores(Qb, Kb, 2, S, b, sig, causal)
    kept = orc.layer_select(scores, _GQA_TAU, causal)
    outs = orc.layer_sparse_attention(Qb, Kb, Vb, 2, kept, b, causal, sa)
    assert sorted(scores) == [(bb, h) for bb in range(B) for h in range(4)]
    for bb in range(B):
        for h in range(4):
            kv = _GQA_KV_OF[h]
            q = orc.bf16_to_f64(Qb[bb, h])
            k = orc.bf16_to_f64(Kb[bb, kv])
            v = orc.bf16_to_f64(Vb[bb, kv])
            want_s = orc.block_scores(q, k, S, b, sig, causal)
            np.testing.assert_array_equal(scores[(bb, h)], want_s)
            want_k = orc.select_blocks(want_s, float(_GQA_TAU[h]), causal)
            assert {r: x.tolist() for r, x in kept[(bb, h)].items()} == \
                {r: x.tolist() for r, x in want_k.items()}
            want_o, want_l = orc.block_sparse_attention(q, k, v, want_k, b, causal, sa)
            np.testing.assert_array_equal(outs[(bb, h)][0], want_o)
            np.testing.assert_array_equal(outs[(bb, h)][1], want_l)


def _wrong_kv_mapping(Qb, Kb, Hkv, stride, block, sigma, causal, heads=None, rows=None,
                      antidiagonal=True):
    """A plausible slip: query head h read KV head h % Hkv instead of its group's."""
    B, Hq = Qb.shape[:2]
    heads = [(bb, h) for bb in range(B) for h in range(Hq)] if heads is None else heads
    return {(bb, h): orc.block_scores(orc.bf16_to_f64(Qb[bb, h]), orc.bf16_to_f64(Kb[bb, h % Hkv]),
                                      stride, block, sigma, causal, rows, antidiagonal)
            for (bb, h) in heads}


def test_planted_wrong_kv_head_mapping_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "layer_block_scores", _wrong_kv_mapping)
    with pytest.raises(AssertionError):
        test_layer_wrappers_map_query_heads_and_taus(True)


def test_planted_group_tau_is_caught(monkeypatch):
    """A plausible slip: every head of a group used the group's tau[h // grp]."""
    def wrong(scores_by_head, tau, causal, rows=None):
        return {(bb, h): orc.select_blocks(s, float(tau[h // 2]), causal, rows)
                for (bb, h), s in scores_by_head.items()}
    monkeypatch.setattr(orc, "layer_select", wrong)
    with pytest.raises(AssertionError):
        test_layer_wrappers_map_query_heads_and_taus(True)


def test_planted_wrong_attention_kv_head_is_caught(monkeypatch):
    """A plausible slip in the attention wrapper: V taken from KV head h % Hkv."""
    def wrong(Qb, Kb, Vb, Hkv, kept_by_head, block, causal, scale, rows=None):
        grp = Qb.shape[1] // Hkv
        return {(bb, h): orc.block_sparse_attention(
            orc.bf16_to_f64(Qb[bb, h]), orc.bf16_to_f64(Kb[bb, h // grp]),
            orc.bf16_to_f64(Vb[bb, h % Hkv]), kept, block, causal, scale, rows)
            for (bb, h), kept in kept_by_head.items()}
    monkeypatch.setattr(orc, "layer_sparse_attention", wrong)
    with pytest.raises(AssertionError):
        test_layer_wrappers_map_query_heads_and_taus(False)
