"""Pins of the oracle with key chunks larger than the (4,4,8) query chunk
("LongCat-Video Technical Report", "Block Sparse Attention (BSA)": the
robustness study varies the key-block token count up to 1024 with query
blocks of 64-128 tokens; "LongCat-Video Technical Report #", "开源实现": a
general forward kernel for key chunks above 128 tokens). Key chunks here are
multiples of (4,4,8) per axis, so each one is a set of (4,4,8) boxes; the
expectations are built with numpy from a padded iota grid."""
import math

import numpy as np
import pytest

import oracle
import synth

from test_oracle_pins import bf, _bruteforce_cdf  # noqa: F401

SHAPES = [(4, 8, 8), (8, 4, 8), (4, 4, 16), (8, 8, 16)]


def padded_map(T, H, W, chunk):
    st, sh, sw = chunk
    Tp, Hp, Wp = -(-T // st) * st, -(-H // sh) * sh, -(-W // sw) * sw
    iota = np.full((Tp, Hp, Wp), -1, dtype=np.int64)
    iota[:T, :H, :W] = np.arange(T * H * W).reshape(T, H, W)
    v = iota.reshape(Tp // st, st, Hp // sh, sh, Wp // sw, sw).transpose(0, 2, 4, 1, 3, 5)
    return v.reshape(-1, st * sh * sw)


def case(T, H, W, heads=2, d=32, t_cond=0):
    wl = synth.WORKLOADS["tiny"].with_(T=T, H=H, W=W, heads=heads, d=d, t_cond=t_cond)
    return (wl,) + synth.make_qkv(wl)


@pytest.mark.parametrize("chunk", SHAPES)
@pytest.mark.parametrize("grid", [(8, 16, 32), (10, 13, 37)])
def test_key_chunk_token_map_and_pool(chunk, grid):
    T, H, W = grid
    tm = padded_map(T, H, W, chunk)
    assert oracle.num_chunks(T, H, W, chunk) == tm.shape[0]
    for c in range(tm.shape[0]):
        assert np.array_equal(oracle.chunk_tokens(T, H, W, c, chunk), tm[c])
    wl, q, k, v = case(T, H, W)
    p = oracle.pool(k, T, H, W, chunk=chunk)
    kf = bf(k)
    for c in range(tm.shape[0]):
        ok = tm[c] >= 0
        np.testing.assert_allclose(p[:, :, c], kf[:, :, tm[c][ok]].mean(2), rtol=0, atol=1e-12)


@pytest.mark.parametrize("chunk", SHAPES[:3])
def test_key_chunk_selection_is_lexsort_topk_and_causal(chunk):
    T, H, W = 16, 16, 32
    wl, q, k, v = case(T, H, W, t_cond=8)
    scale = 1 / math.sqrt(wl.d)
    S = oracle.scores(oracle.pool(q, T, H, W), oracle.pool(k, T, H, W, chunk=chunk), scale)
    rp, ci = oracle.select(S, T, H, W, "topk", 3, t_cond=8, kchunk=chunk)
    Nq, Nk = S.shape[2], S.shape[3]
    qm, km = padded_map(T, H, W, (4, 4, 8)), padded_map(T, H, W, chunk)
    HW = H * W
    for bh in range(wl.heads):
        for i in range(Nq):
            q_cond = qm[i][qm[i] >= 0].max() // HW < 8           # every frame below t_cond
            cand = np.array([m for m in range(Nk)
                             if not q_cond or km[m][km[m] >= 0].max() // HW < 8])
            row = S[0, bh, i]
            order = cand[np.lexsort((cand, -row[cand]))]
            expect = np.sort(order[:min(3, len(cand))])
            r = bh * Nq + i
            assert np.array_equal(ci[rp[r]:rp[r + 1]], expect), (bh, i)


def masked_attention(q, k, v, T, H, W, chunk, rp, ci, scale, heads):
    qm, km = padded_map(T, H, W, (4, 4, 8)), padded_map(T, H, W, chunk)
    N = T * H * W
    q_of, k_of = np.empty(N, dtype=np.int64), np.empty(N, dtype=np.int64)
    for c in range(qm.shape[0]):
        q_of[qm[c][qm[c] >= 0]] = c
    for c in range(km.shape[0]):
        k_of[km[c][km[c] >= 0]] = c
    Nq, Nk = qm.shape[0], km.shape[0]
    qf, kf, vf = bf(q)[0], bf(k)[0], bf(v)[0]
    out = []
    for h in range(heads):
        M = np.zeros((Nq, Nk), dtype=bool)
        for i in range(Nq):
            M[i, ci[rp[h * Nq + i]:rp[h * Nq + i + 1]]] = True
        allowed = M[q_of][:, k_of]
        s = np.where(allowed, qf[h] @ kf[h].T * scale, -np.inf)
        s -= s.max(1, keepdims=True)
        w = np.exp(s)
        w /= w.sum(1, keepdims=True)
        out.append(w @ vf[h])
    return np.stack(out), qm


@pytest.mark.parametrize("chunk", SHAPES)
def test_attention_over_key_chunks_equals_token_masked_softmax(chunk):
    T, H, W = 8, 12, 40
    wl, q, k, v = case(T, H, W)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, S = oracle.plan(q, k, T, H, W, scale, "topk", 2, kchunk=chunk)
    Nq = S.shape[2]
    rows = np.arange(wl.heads * Nq)
    out, _ = oracle.attend(q, k, v, T, H, W, scale, rp, ci, rows, kchunk=chunk)
    ref, qm = masked_attention(q, k, v, T, H, W, chunk, rp, ci, scale, wl.heads)
    for r in rows:
        h, i = divmod(r, Nq)
        ok = qm[i] >= 0
        np.testing.assert_allclose(out[r][ok], ref[h][qm[i][ok]], rtol=0, atol=1e-12)


def expand_to_boxes(rp, ci, T, H, W, chunk):
    """Key-chunk CSR -> CSR over the (4,4,8) boxes each selected key chunk covers."""
    km = padded_map(T, H, W, chunk)
    bm = padded_map(T, H, W, (4, 4, 8))
    box_of = {}
    for b in range(bm.shape[0]):
        for tok in bm[b][bm[b] >= 0]:
            box_of[tok] = b
    boxes = [sorted({box_of[t] for t in km[c][km[c] >= 0]}) for c in range(km.shape[0])]
    rows = [sum((boxes[c] for c in ci[rp[r]:rp[r + 1]]), []) for r in range(len(rp) - 1)]
    erp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    eci = np.array(sum(rows, []), dtype=np.int32)
    return erp, eci


@pytest.mark.parametrize("chunk", SHAPES)
def test_key_chunk_attention_equals_box_expansion(chunk):
    """Attending over key chunks is attending over the (4,4,8) boxes they cover:
    the reduction the CUDA path uses."""
    T, H, W = 10, 13, 37
    wl, q, k, v = case(T, H, W)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, S = oracle.plan(q, k, T, H, W, scale, "topk", 2, kchunk=chunk)
    rows = np.arange(wl.heads * S.shape[2])
    out, lse = oracle.attend(q, k, v, T, H, W, scale, rp, ci, rows, kchunk=chunk)
    erp, eci = expand_to_boxes(rp, ci, T, H, W, chunk)
    out2, lse2 = oracle.attend(q, k, v, T, H, W, scale, erp, eci, rows)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)
    g = synth.make_dout(wl)
    a = oracle.attend_bwd(q, k, v, g, T, H, W, scale, rp, ci, rows, kchunk=chunk)
    b = oracle.attend_bwd(q, k, v, g, T, H, W, scale, erp, eci, rows)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)
