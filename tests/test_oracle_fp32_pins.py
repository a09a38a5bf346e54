"""Pins of the oracle's single-precision decision mode (no GPU).

The GPU's chunk lists are compared with ``oracle.plan(..., fp32=True)``: the
pooled means, the pooled scores and the CDF prefix decided in float, the
precision the selection kernels use. That mode needs pins of its own, apart
from the fp64 mode's, so that a mistake shared by it and a kernel cannot pass:

* the float scores against numpy's float64 matmul times the scale;
* the float selection against the fp64 selection of the same rows, row by row,
  where every row that differs must be an fp64 tie (scores within 1e-5
  relative) or sit at the CDF threshold (cumulative mass within 1e-5 of p), and
  every row, differing or not, must be a valid top set and CDF count under the
  fp64 scores (numpy softmax and sorting, tests/parity.py);
* hand-built rows whose answers follow from the rule as the pages state it
  ("LongCat-Video Technical Report", section "Block Sparse Attention (BSA)",
  CDF-p: keep chunks from the highest pooled score down until their softmax
  mass reaches p): an exactly representable flat row where "reaches"
  (cumulative >= p) and "exceeds" (> p) give different counts, a cap whose
  product with the candidate count lies just below an integer, and rows whose
  scores overflow or underflow float unless the row maximum is subtracted.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import TIE_REL, cdf_count_ok, compare_csr, rows_of, valid_topk_set

W = synth.WORKLOADS["tiny"]

CASES = {
    "tiny": W,
    "ragged_partial": W.with_(heads=2, T=6, H=10, W=20, d=64, topk=5),
    "ragged135": W.with_(heads=2, T=12, H=20, W=72, d=128, topk=9),
    "causal_cdf_small": W.with_(B=2, heads=2, T=16, H=16, W=32, d=128, mode="cdf", cdf_p=0.9,
                                cdf_cap_frac=0.25, t_cond=8),
    "cdf_nocap": W.with_(heads=2, T=8, H=16, W=32, d=64, mode="cdf", cdf_p=0.5,
                         cdf_cap_frac=1.0),
    "topk_cdf_small": W.with_(heads=2, T=8, H=16, W=32, d=128, mode="topk_cdf", topk=6,
                              cdf_p=0.2, cdf_cap_frac=0.5),
    "partial_causal_cdf": W.with_(B=2, heads=2, T=10, H=13, W=28, d=128, mode="cdf",
                                  cdf_p=0.9, cdf_cap_frac=0.25, t_cond=4),
}


def test_scores_fp32_equal_float64_matmul_times_scale():
    rng = np.random.default_rng(21)
    qp = rng.standard_normal((2, 3, 7, 64)).astype(np.float32).astype(np.float64)
    kp = rng.standard_normal((2, 3, 11, 64)).astype(np.float32).astype(np.float64)
    scale = 0.3
    s = oracle.scores(qp, kp, scale, fp32=True)
    assert np.all(s.astype(np.float32).astype(np.float64) == s)   # float-valued
    ref = np.einsum("bhid,bhmd->bhim", qp, kp) * scale
    bound = np.einsum("bhid,bhmd->bhim", np.abs(qp), np.abs(kp)) * scale
    assert np.all(np.abs(s - ref) <= 1e-5 * bound + 1e-30)
    # the scale is applied (not 1) and the operands are not transposed
    assert np.abs(s - ref / scale).max() > 1.0
    qk_sq = oracle.scores(qp[:, :, :7], kp[:, :, :7], scale, fp32=True)
    assert not np.allclose(qk_sq, np.swapaxes(qk_sq, -1, -2))


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp32_selection_agrees_with_fp64_up_to_ties(name):
    wl = CASES[name]
    q, k, _ = synth.make_qkv(wl)
    scale = 1.0 / math.sqrt(wl.d)
    args = (q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p, wl.cdf_cap_frac,
            wl.t_cond)
    rp32, ci32, _ = oracle.plan(*args, fp32=True)
    rp64, ci64, S64 = oracle.plan(*args, fp32=False)
    S64 = S64.reshape(-1, wl.Nc, wl.Nc)
    # rows that differ are ties or threshold cases under the fp64 scores
    n_checked, n_diff = compare_csr(rp32, ci32, rp64, ci64, S64, wl.Nc, wl.n_cond, wl.mode,
                                    wl.cdf_p, wl.cdf_cap_frac, topk=wl.topk)
    assert n_checked == wl.rows and n_diff <= max(1, wl.rows // 100)
    # and every float row is a valid selection under the fp64 scores
    for r, sel in enumerate(rows_of(rp32, ci32)):
        i = r % wl.Nc
        cand = np.arange(wl.n_cond if (wl.n_cond > 0 and i < wl.n_cond) else wl.Nc)
        s64 = S64[r // wl.Nc, i]
        assert valid_topk_set(sel, s64, cand), r
        if wl.mode == "topk":
            assert len(sel) == min(wl.topk, len(cand)), r
        else:
            k = wl.topk if wl.mode == "topk_cdf" else None
            assert cdf_count_ok(len(sel), s64, cand, wl.cdf_p, wl.cdf_cap_frac, k), r


@pytest.mark.parametrize("fp32", [False, True])
def test_cdf_reaching_p_is_inclusive(fp32):
    """A flat row of 8 chunks: each softmax mass is exactly 1/8 (also in float),
    so the prefix mass reaches p = 0.5 after exactly 4 chunks. A strict
    comparison would keep 5."""
    T, H, W_ = 4, 8, 32                                 # 8 chunks
    S = np.zeros((1, 1, 8, 8))
    rp, ci = oracle.select(S, T, H, W_, mode="cdf", cdf_p=0.5, cap_frac=1.0, fp32=fp32)
    assert list(np.diff(rp)) == [4] * 8
    assert all(list(ci[rp[r]:rp[r + 1]]) == [0, 1, 2, 3] for r in range(8))
    rp, ci = oracle.select(S, T, H, W_, mode="cdf", cdf_p=0.375, cap_frac=1.0, fp32=fp32)
    assert list(np.diff(rp)) == [3] * 8                 # 3/8 is exact as well


@pytest.mark.parametrize("fp32", [False, True])
def test_cdf_cap_is_the_floor_of_the_exact_product(fp32):
    """cap = max(1, floor(cap_frac * |A(i)|)) with the product taken exactly (in
    double). The library receives the fraction as a float: float(0.7) is
    0.699999988..., so 10 candidates give a cap of 6; a product rounded to
    float would give 7.0 and a cap of 7."""
    T, H, W_ = 4, 4, 80                                 # 1 x 1 x 10 chunks
    cap_frac = float(np.float32(0.7))
    assert cap_frac * 10 < 7.0 and float(np.float32(cap_frac) * np.float32(10)) == 7.0
    S = np.zeros((1, 1, 10, 10))
    rp, _ = oracle.select(S, T, H, W_, mode="cdf", cdf_p=1.0, cap_frac=cap_frac, fp32=fp32)
    assert list(np.diff(rp)) == [6] * 10
    rp, _ = oracle.select(S, T, H, W_, mode="cdf", cdf_p=0.9, cap_frac=0.05, fp32=fp32)
    assert list(np.diff(rp)) == [1] * 10                # floor(0.5) = 0 -> the floor of 1


@pytest.mark.parametrize("fp32", [False, True])
def test_cdf_rows_far_outside_the_float_exponent_range(fp32):
    """Scores of +-200: exp overflows (or underflows to zero) in float unless the
    row maximum is subtracted first. The softmax is unchanged by the shift."""
    T, H, W_ = 4, 8, 32                                 # 8 chunks
    S = np.zeros((1, 1, 8, 8))
    S[0, 0, :, 5] = 200.0                               # one dominant chunk per row
    rp, ci = oracle.select(S, T, H, W_, mode="cdf", cdf_p=0.9, cap_frac=1.0, fp32=fp32)
    assert list(np.diff(rp)) == [1] * 8 and list(ci) == [5] * 8
    S = np.full((1, 1, 8, 8), -200.0)                   # flat, far below zero
    rp, ci = oracle.select(S, T, H, W_, mode="cdf", cdf_p=0.5, cap_frac=1.0, fp32=fp32)
    assert list(np.diff(rp)) == [4] * 8
    S = np.full((1, 1, 8, 8), 150.0)                    # flat, far above zero
    S[0, 0, :, 2] = 150.0 + math.log(4.0)               # mass 4/11 on chunk 2
    rp, ci = oracle.select(S, T, H, W_, mode="cdf", cdf_p=0.5, cap_frac=1.0, fp32=fp32)
    # 4/11 + 1/11 < 0.5 <= 4/11 + 2/11: chunk 2 and the two lowest-index others
    assert list(np.diff(rp)) == [3] * 8
    assert all(list(ci[rp[r]:rp[r + 1]]) == [0, 1, 2] for r in range(8))


def test_fp32_threshold_rows_are_within_the_tie_bar():
    """Random CDF rows, fp32 against fp64: every count that differs sits where
    the fp64 prefix mass is within TIE_REL of p (the parity bar's reading of a
    threshold tie), never elsewhere."""
    rng = np.random.default_rng(4)
    T, H, W_ = 8, 16, 32                                # 32 chunks
    S = rng.standard_normal((1, 8, 32, 32)) * 2.0
    for p in (0.3, 0.6, 0.9):
        rp32, _ = oracle.select(S, T, H, W_, mode="cdf", cdf_p=p, cap_frac=1.0, fp32=True)
        rp64, _ = oracle.select(S, T, H, W_, mode="cdf", cdf_p=p, cap_frac=1.0, fp32=False)
        for r in np.nonzero(np.diff(rp32) != np.diff(rp64))[0]:
            row = S.reshape(-1, 32)[r]
            w = np.exp(row - row.max())
            mass = np.cumsum(np.sort(w / w.sum())[::-1])
            c = min(np.diff(rp32)[r], np.diff(rp64)[r])
            assert abs(mass[c - 1] - p) <= TIE_REL * p, (p, r)
