"""Comparison rules shared by the GPU parity tests.

Selection: the GPU's chunk lists must equal the oracle's (decided in fp32, the
kernel's precision) except where pooled scores tie within 1e-5 relative (or,
for CDF, where the cumulative mass sits within 1e-5 of p); every GPU row, equal
or not, must also be a valid selection under the oracle's fp64 scores.

Attention: GPU bf16 output vs the fp64 oracle evaluated on the GPU's own CSR,
max-abs <= 2e-2 and mean-abs <= 2e-3 (fp32 accumulation, bf16 inputs,
bf16-rounded softmax numerators and output).
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-5
ATT_MAX_ABS = 2e-2
ATT_MEAN_ABS = 2e-3


def rows_of(row_ptr, col_idx):
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx)
    return [ci[rp[r]:rp[r + 1]] for r in range(len(rp) - 1)]


def _candidates(i, Nk, n_cond, n_cond_k=None):
    """Key chunks a query chunk i may select: the condition key chunks for a
    condition query chunk, all Nk otherwise."""
    n_cond_k = n_cond if n_cond_k is None else n_cond_k
    return np.arange(n_cond_k if (n_cond > 0 and i < n_cond) else Nk)


def _tied(a, b):
    return abs(a - b) <= TIE_REL * max(abs(a), abs(b), 1e-30)


def valid_topk_set(sel, s64, cand):
    """sel is a top-|sel| subset of cand under s64 up to ties within TIE_REL."""
    sel = np.asarray(sel)
    if len(sel) != len(np.unique(sel)) or not np.all(np.diff(sel) > 0):
        return False
    if not np.all(np.isin(sel, cand)):
        return False
    rest = np.setdiff1d(cand, sel)
    if len(rest) == 0:
        return True
    lo = s64[sel].min()
    hi = s64[rest].max()
    return lo >= hi or _tied(lo, hi)


def cdf_count_ok(count, s64, cand, p, cap_frac, k=None):
    """count is the CDF count of this row (bounded by k in the combination
    mode) up to mass ties within TIE_REL."""
    s = s64[cand]
    w = np.exp(s - s.max())
    w /= w.sum()
    mass = np.cumsum(np.sort(w)[::-1])
    cap = max(1, int(np.floor(cap_frac * len(cand))))
    if k is not None:
        cap = min(cap, k)
    mstar = int(np.searchsorted(mass, p, side="left")) + 1  # first prefix with mass >= p
    mstar = min(mstar, len(cand))
    if count == min(mstar, cap):
        return True
    if count > cap or count < 1:
        return False
    # near-threshold prefixes: the mass after count-1 or count chunks is within tol of p
    near = lambda c: 1 <= c <= len(cand) and abs(mass[c - 1] - p) <= TIE_REL * p
    return (near(count) or near(count - 1) or near(mstar) or near(mstar - 1)) and \
        abs(count - min(mstar, cap)) <= 1


def compare_csr(gpu_rp, gpu_ci, ora_rp, ora_ci, S64, Nc, n_cond, mode, p=0.9, cap_frac=0.25,
                rows=None, topk=None, Nk=None, n_cond_k=None):
    """Returns (n_rows_checked, n_rows_differing); asserts validity of every row.
    Rows are (batch, head, query chunk) with Nc query chunks per head; columns are
    key chunks (Nk of them, Nc unless key chunks are larger)."""
    Nk = Nc if Nk is None else Nk
    S64 = np.asarray(S64).reshape(-1, Nc, Nk)
    g_rows, o_rows = rows_of(gpu_rp, gpu_ci), rows_of(ora_rp, ora_ci)
    assert len(g_rows) == len(o_rows)
    idx = range(len(g_rows)) if rows is None else rows
    ndiff = 0
    for r in idx:
        g, o = g_rows[r], o_rows[r]
        same = len(g) == len(o) and np.array_equal(g, o)
        ndiff += not same
        # every row, equal to the oracle's or not, must be a valid selection under the
        # fp64 scores, so a mistake shared by the kernel and the oracle's float mode fails
        i = r % Nc
        s64 = S64[r // Nc, i]
        cand = _candidates(i, Nk, n_cond, n_cond_k)
        assert valid_topk_set(g, s64, cand), f"row {r}: gpu {g} vs oracle {o} not a tie"
        if mode == "topk":
            assert len(g) == min(topk, len(cand)) if topk else len(g) == len(o), \
                f"row {r}: count {len(g)} vs {len(o)}"
        else:
            k = topk if mode == "topk_cdf" else None
            assert cdf_count_ok(len(g), s64, cand, p, cap_frac, k), \
                f"row {r}: cdf count {len(g)} vs oracle {len(o)}"
    return len(idx), ndiff


def compare_attention(gpu_out_rows, ora_out_rows):
    """max-abs and mean-abs error over the existing query slots (the oracle marks
    slots of partial edge chunks past the grid with NaN)."""
    g = np.asarray(gpu_out_rows, dtype=np.float64)
    o = np.asarray(ora_out_rows, dtype=np.float64)
    live = ~np.isnan(o)
    assert np.array_equal(live, ~np.isnan(g)), "existing slots differ"
    err = np.abs(g[live] - o[live])
    return float(err.max()), float(err.mean())
