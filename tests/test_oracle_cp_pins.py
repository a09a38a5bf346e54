"""Pins of the oracle's context-parallel merge ("LongCat-Video Technical
Report", "Block Sparse Attention (BSA)", ring block sparse attention: partial
results over key partitions combined with an online softmax). The merge of the
attention over two disjoint sets of selected key chunks must equal the
attention over their union (the oracle's attend, itself pinned against
numpy and dense attention), and it must be associative and commutative."""
import math

import numpy as np

import oracle
import synth


def split_csr(rp, ci, pred):
    """Rows of a CSR split by a predicate on the column index."""
    a_rows, b_rows = [], []
    for r in range(len(rp) - 1):
        cols = ci[rp[r]:rp[r + 1]]
        a_rows.append(cols[pred(cols)])
        b_rows.append(cols[~pred(cols)])
    mk = lambda rows: (np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32),  # noqa: E731
                       np.concatenate(rows).astype(np.int32) if rows else np.zeros(0, np.int32))
    return mk(a_rows), mk(b_rows)


def test_merge_of_disjoint_key_sets_is_attention_over_union():
    wl = synth.WORKLOADS["tiny"].with_(T=16, H=8, W=16, heads=2, d=32)   # 16 chunks
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, "topk", 6)
    rows = np.arange(wl.rows)
    full_o, full_l = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    for split in (8, 4, 12, 1):    # key chunks below `split` vs the rest
        (ra, ca), (rb, cb) = split_csr(rp, ci, lambda c: c < split)
        oa, la = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, ra, ca, rows)
        ob, lb = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rb, cb, rows)
        if split == 1:              # most rows do not keep chunk 0: empty first part
            assert np.isneginf(la).any()
        mo, ml = oracle.lse_merge(oa, la, ob, lb)
        np.testing.assert_allclose(mo, full_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(ml, full_l, rtol=0, atol=1e-12)


def test_merge_is_commutative_associative_and_keeps_empty_parts():
    rng = np.random.default_rng(3)
    n, d = 40, 8
    parts = [(rng.normal(size=(n, d)), rng.normal(size=n) * 3) for _ in range(3)]
    parts[1][1][:5] = -np.inf                      # empty partition for some queries
    (o0, l0), (o1, l1), (o2, l2) = parts
    ab, lab = oracle.lse_merge(o0, l0, o1, l1)
    ba, lba = oracle.lse_merge(o1, l1, o0, l0)
    np.testing.assert_allclose(ab, ba, atol=1e-12)
    np.testing.assert_allclose(lab, lba, atol=1e-12)
    left, ll = oracle.lse_merge(*oracle.lse_merge(o0, l0, o1, l1), o2, l2)
    right, lr = oracle.lse_merge(o0, l0, *oracle.lse_merge(o1, l1, o2, l2))
    np.testing.assert_allclose(left, right, atol=1e-12)
    np.testing.assert_allclose(ll, lr, atol=1e-12)
    # log-sum-exp closed form
    np.testing.assert_allclose(ll, np.logaddexp(np.logaddexp(l0, l1), l2), atol=1e-12)
    # empty second part leaves the first unchanged; both empty stays empty
    e = np.full(n, -np.inf)
    m, lm = oracle.lse_merge(o0, l0, o1, e)
    assert np.array_equal(m, o0) and np.array_equal(lm, l0)
    m, lm = oracle.lse_merge(np.zeros((n, d)), e, o1, e)
    assert not m.any() and np.all(np.isneginf(lm))


def _rows_to_tokens(x_rows, T, H, W, B, heads, nc):
    """[B*heads*nc, 128, ...] chunk rows -> [B, heads, N, ...] THW tokens."""
    N = T * H * W
    out = np.zeros((B * heads, N) + x_rows.shape[2:], dtype=np.float64)
    for c in range(nc):
        tok = oracle.chunk_tokens(T, H, W, c)
        ok = tok >= 0
        for bh in range(B * heads):
            out[bh, tok[ok]] = x_rows[bh * nc + c][ok]
    return out.reshape((B, heads, N) + x_rows.shape[2:])


def _backward_case(wl, topk):
    q, k, v = synth.make_qkv(wl)
    dout = synth.make_dout(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, "topk", topk)
    nc = oracle.num_chunks(wl.T, wl.H, wl.W)
    rows = np.arange(wl.B * wl.heads * nc)
    o, l = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    out = _rows_to_tokens(o, wl.T, wl.H, wl.W, wl.B, wl.heads, nc)
    lse = _rows_to_tokens(l, wl.T, wl.H, wl.W, wl.B, wl.heads, nc)
    full = oracle.attend_bwd(q, k, v, dout, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    return q, k, v, dout, out, lse, scale, rp, ci, rows, full


def test_backward_over_key_partitions_sums_to_full_backward():
    """Ring block sparse attention splits every query's keys across ranks; the
    gradient terms of the chain rule are sums over keys, so the contributions
    of disjoint key partitions (each weighted with the whole softmax: the full
    log-sum-exp and output) must add up to the backward of the unsplit
    attention (attend_bwd, pinned by finite differences). A partition that used
    its own softmax instead of the whole one fails this."""
    for wl, topk in ((synth.WORKLOADS["tiny"].with_(T=16, H=8, W=16, heads=2, d=32), 6),
                     (synth.WORKLOADS["tiny"].with_(T=10, H=6, W=13, heads=1, d=16), 5)):
        q, k, v, dout, out, lse, scale, rp, ci, rows, (fq, fk, fv) = _backward_case(wl, topk)
        nc = oracle.num_chunks(wl.T, wl.H, wl.W)
        for split in (nc // 2, 1, nc - 1):
            (ra, ca), (rb, cb) = split_csr(rp, ci, lambda c: c < split)
            aq, ak, av = oracle.attend_bwd_part(q, k, v, dout, out, lse, wl.T, wl.H, wl.W, scale,
                                                ra, ca, rows)
            bq, bk, bv = oracle.attend_bwd_part(q, k, v, dout, out, lse, wl.T, wl.H, wl.W, scale,
                                                rb, cb, rows)
            np.testing.assert_allclose(aq + bq, fq, rtol=0, atol=1e-11 * np.nanmax(np.abs(fq)))
            np.testing.assert_allclose(ak + bk, fk, rtol=0, atol=1e-11 * np.abs(fk).max())
            np.testing.assert_allclose(av + bv, fv, rtol=0, atol=1e-11 * np.abs(fv).max())
            # query slots past the grid edge carry no gradient in either
            assert np.array_equal(np.isnan(aq), np.isnan(fq))


def test_backward_of_the_whole_key_set_and_of_an_empty_one():
    wl = synth.WORKLOADS["tiny"].with_(T=8, H=8, W=16, heads=2, d=32)
    q, k, v, dout, out, lse, scale, rp, ci, rows, (fq, fk, fv) = _backward_case(wl, 3)
    aq, ak, av = oracle.attend_bwd_part(q, k, v, dout, out, lse, wl.T, wl.H, wl.W, scale, rp, ci,
                                        rows)
    np.testing.assert_allclose(aq, fq, rtol=0, atol=1e-11 * np.abs(fq).max())
    np.testing.assert_allclose(ak, fk, rtol=0, atol=1e-11 * np.abs(fk).max())
    np.testing.assert_allclose(av, fv, rtol=0, atol=1e-11 * np.abs(fv).max())
    empty_rp = np.zeros_like(rp)
    eq, ek, ev = oracle.attend_bwd_part(q, k, v, dout, out, lse, wl.T, wl.H, wl.W, scale, empty_rp,
                                        np.zeros(0, np.int32), rows)
    assert not eq.any() and not ek.any() and not ev.any()
