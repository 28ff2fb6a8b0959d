"""Comparison rules between the CUDA path and the CPU oracle (test helpers).

Floating-point tolerances (derived from the arithmetic; see the parity tests):
- block scores: |gpu - oracle| <= SCORE_ATOL + SCORE_RTOL * oracle. The GPU forms
  each logit as an fp32 sum of S*C exact bf16 products (relative error ~1e-6),
  then base-2 exp/log in fp32 with hardware ex2/lg2 (~2^-22 relative each), so a
  block score carries a relative error of a few 1e-6; 2e-4 leaves two orders of
  magnitude of headroom while still catching any dropped term or wrong index
  (which moves scores by O(1) relative).
- attention outputs: max-abs <= 2e-2 and mean-abs <= 2e-3 (bf16 inputs, fp32
  accumulation, bf16 output).
- masks: bit-exact, except (a) entries whose cumulative-mass margin to tau is
  below 1e-4, and (b) pairs of blocks that the two sides order differently at
  the cut because their scores are equal within twice the score tolerance
  (several minimal sets are then equally correct). Every exception is logged.
"""
from __future__ import annotations

import numpy as np

import oracle as orc

SCORE_ATOL = 1e-6
SCORE_RTOL = 2e-4
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
MASK_MARGIN = 1e-4


def score_tol(ref):
    return SCORE_ATOL + SCORE_RTOL * np.abs(ref)


def assert_scores_close(gpu: np.ndarray, ref: np.ndarray, what: str = "scores"):
    err = np.abs(gpu.astype(np.float64) - ref)
    bad = err > score_tol(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} entries out of tolerance; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]!r} oracle={ref[tuple(i)]!r}")
    return float(err.max()) if err.size else 0.0


def csr_rows(row_ptr: np.ndarray, col_idx: np.ndarray, row: int) -> np.ndarray:
    return col_idx[row_ptr[row]:row_ptr[row + 1]]


def compare_row_mask(gpu_cols, oracle_row_scores, r: int, tau: float, causal: bool):
    """Returns (exceptions, failures) for one query-block row.

    gpu_cols: the GPU's kept list for the row (must be ascending, unique).
    """
    failures, exceptions = [], []
    g = np.asarray(gpu_cols, dtype=np.int64)
    if g.size and (np.any(np.diff(g) <= 0)):
        failures.append(("not ascending/unique", r, g.tolist()))
    nb = oracle_row_scores.shape[0]
    hi = r + 1 if causal else nb
    if g.size and (g.min() < 0 or g.max() >= hi):
        failures.append(("out of range", r, g.tolist()))
    if r not in set(g.tolist()):
        failures.append(("diagonal missing", r))
    ref = set(orc.select_row(oracle_row_scores, r, tau, causal).tolist())
    got = set(g.tolist())
    only_ref, only_gpu = sorted(ref - got), sorted(got - ref)
    if not only_ref and not only_gpu:
        return exceptions, failures
    margin, _ = orc.selection_margins(oracle_row_scores, r, tau, causal)
    s = oracle_row_scores
    # (b) pair near-equal scores that crossed the cut in opposite directions
    unmatched_ref = list(only_ref)
    unmatched_gpu = []
    for c in only_gpu:
        tol = 2 * score_tol(s[c])
        hit = next((a for a in unmatched_ref if abs(s[a] - s[c]) <= tol), None)
        if hit is not None:
            unmatched_ref.remove(hit)
            exceptions.append(("tie", r, int(hit), int(c), float(s[hit] - s[c])))
        else:
            unmatched_gpu.append(c)
    # (a) the cumulative-mass margin rule
    for c in unmatched_ref + unmatched_gpu:
        if abs(margin[c]) < MASK_MARGIN:
            exceptions.append(("margin", r, int(c), float(margin[c])))
        else:
            failures.append(("mask", r, int(c), float(margin[c]),
                             "oracle keeps" if c in ref else "gpu keeps"))
    return exceptions, failures


def assert_outputs_close(gpu: np.ndarray, ref: np.ndarray, what: str = "O"):
    err = np.abs(gpu.astype(np.float64) - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, \
        f"{what}: max-abs {mx:.3e} (<= {OUT_MAX_ABS}), mean-abs {mean:.3e} (<= {OUT_MEAN_ABS})"
    return mx, mean


def oracle_head_scores(args):
    """The oracle's complete [nb, nb] block scores of one head, from bf16 bits
    (a top-level function, so that a spawned worker process can run it)."""
    qb, kb, stride, block, causal = args
    q, k = orc.bf16_to_f64(qb), orc.bf16_to_f64(kb)
    return orc.block_scores(q, k, stride, block, orc.default_score_scale(stride, q.shape[1]),
                            causal)


# Lines printed at the end of the pytest run (tests/conftest.py): every mask
# exception of the full-size runs, and one summary line per configuration.
REPORT: list = []


def log_exception(config: str, head: int, exc) -> None:
    """One mask exception from compare_row_mask: ("margin", r, c, margin) or
    ("tie", r, c_oracle, c_gpu, score difference)."""
    kind, r = exc[0], exc[1]
    if kind == "margin":
        REPORT.append(f"mask exception [{config}] head={head} row={r} block={exc[2]} "
                      f"margin={exc[3]:+.3e} kind=margin")
    else:
        REPORT.append(f"mask exception [{config}] head={head} row={r} block={exc[2]}/{exc[3]} "
                      f"score_diff={exc[4]:+.3e} kind=tie")


def report(line: str) -> None:
    REPORT.append(line)
