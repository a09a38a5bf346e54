"""Pins of the oracle with 64-token chunks (no GPU).

"LongCat-Video Technical Report", section "Block Sparse Attention (BSA)",
block-size robustness: query blocks of 64 or 128 tokens and key blocks from 64
to 1024 tokens; the blocks of its partitioning are t = h = w = 4, i.e. (4,4,4)
blocks of 64 tokens. The oracle takes the query chunk shape as a parameter of
selection and attention; these tests tie that generalisation to numpy
reshapes, sorts and a token-level masked softmax, to dense attention when
every chunk is kept, and to hand-built block-causal candidate sets. The
backward (gradients over 64-token query chunks) is tied to torch float64
autograd of the token-masked dense attention and to the (4,4,8) backward.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

Q64 = (4, 4, 4)
W0 = synth.WORKLOADS["tiny"]


def bf(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64)


def block64_view(x, T, H, W):
    B, Hh, N, d = x.shape
    return x.reshape(B, Hh, T // 4, 4, H // 4, 4, W // 4, 4, d)


def numpy_rearrange64(x, T, H, W):
    """[B,Hh,N,d] -> [B,Hh,Nc,64,d]: chunks in (t,h,w) order, tokens in (t,h,w) order."""
    B, Hh, N, d = x.shape
    v = block64_view(x, T, H, W).transpose(0, 1, 2, 4, 6, 3, 5, 7, 8)
    return v.reshape(B, Hh, N // 64, 64, d)


def test_token_map_of_64_token_chunks_equals_numpy_reshape():
    T, H, W = 8, 8, 16
    iota = np.arange(T * H * W).reshape(1, 1, -1, 1)
    tok = numpy_rearrange64(iota, T, H, W)[0, 0, :, :, 0]       # [chunk, local] -> token
    assert oracle.num_chunks(T, H, W, Q64) == 2 * 2 * 4
    for c in range(tok.shape[0]):
        np.testing.assert_array_equal(oracle.chunk_tokens(T, H, W, c, Q64), tok[c])


def test_token_map_of_partial_64_token_chunks():
    """W = 10: the last chunk column covers w = 8, 9 only; its slots lw = 2, 3 do
    not exist."""
    T, H, W = 4, 4, 10
    assert oracle.num_chunks(T, H, W, Q64) == 3
    toks = oracle.chunk_tokens(T, H, W, 2, Q64)
    for l in range(64):
        lt, lh, lw = l // 16, (l // 4) % 4, l % 4
        want = (lt * H + lh) * W + 8 + lw if lw < 2 else -1
        assert toks[l] == want, l


def test_pool_of_64_token_chunks_equals_numpy_block_mean():
    wl = W0.with_(T=8, H=8, W=16, heads=2)
    q, _, _ = synth.make_qkv(wl)
    p = oracle.pool(q, wl.T, wl.H, wl.W, chunk=Q64)
    ref = bf(block64_view(q, wl.T, wl.H, wl.W)).mean(axis=(3, 5, 7))
    np.testing.assert_allclose(p, ref.reshape(p.shape), rtol=0, atol=1e-14)


def test_topk_with_64_token_query_chunks_equals_lexsort():
    rng = np.random.default_rng(3)
    T, H, W = 8, 8, 16                                  # 16 chunks of 64 tokens
    S = rng.standard_normal((1, 2, 16, 16))
    S[0, 1, 4, [2, 7]] = S[0, 1, 4, 11]                 # exact ties
    for k in (1, 3, 16):
        rp, ci = oracle.select(S, T, H, W, "topk", k, kchunk=Q64, qchunk=Q64)
        flat = S.reshape(-1, 16)
        for r in range(flat.shape[0]):
            order = np.lexsort((np.arange(16), -flat[r]))
            assert list(ci[rp[r]:rp[r + 1]]) == sorted(order[:k].tolist())


def test_block_causal_candidates_of_64_token_chunks():
    """T = 8, H = 8, W = 16, t_cond = 4: with (4,4,4) chunks a block of 4 frames
    holds 2 x 4 = 8 chunks, so chunks 0..7 are the condition chunks."""
    T, H, W = 8, 8, 16
    S = np.zeros((1, 1, 16, 16))
    S[0, 0, :, 8:] = 5.0                                # noisy key chunks score highest
    S[0, 0, :, 3] = 1.0
    rp, ci = oracle.select(S, T, H, W, "topk", 2, t_cond=4, kchunk=Q64, qchunk=Q64)
    rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(16)]
    for i in range(8):                                  # condition rows: best is 3, then 0
        assert rows[i] == [0, 3]
    for i in range(8, 16):                              # noisy rows: 8 and 9 (ties to lower)
        assert rows[i] == [8, 9]


@pytest.mark.parametrize("kchunk", [Q64, (4, 4, 8)])
def test_attention_of_64_token_query_chunks_equals_numpy_masked_softmax(kchunk):
    """The chunk mask lifted to tokens with numpy reshapes, then a masked dense
    softmax, for 64-token query chunks and 64- or 128-token key chunks."""
    wl = W0.with_(T=8, H=8, W=16, heads=1)
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, "topk", 3, kchunk=kchunk, qchunk=Q64)
    nq = oracle.num_chunks(wl.T, wl.H, wl.W, Q64)
    nk = oracle.num_chunks(wl.T, wl.H, wl.W, kchunk)
    out, lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, np.arange(nq),
                             kchunk=kchunk, qchunk=Q64)
    assert out.shape == (nq, 64, wl.d)
    iota = np.arange(wl.N).reshape(1, 1, -1, 1)
    qtok = numpy_rearrange64(iota, wl.T, wl.H, wl.W)[0, 0, :, :, 0]
    kt, kh, kw = kchunk
    kv = iota.reshape(wl.T // kt, kt, wl.H // kh, kh, wl.W // kw, kw)
    ktok = kv.transpose(0, 2, 4, 1, 3, 5).reshape(nk, -1)
    kchunk_of = np.empty(wl.N, dtype=np.int64)
    kchunk_of[ktok.reshape(-1)] = np.repeat(np.arange(nk), ktok.shape[1])
    M = np.zeros((nq, nk), dtype=bool)
    for i in range(nq):
        M[i, ci[rp[i]:rp[i + 1]]] = True
    qchunk_of = np.empty(wl.N, dtype=np.int64)
    qchunk_of[qtok.reshape(-1)] = np.repeat(np.arange(nq), 64)
    tokmask = M[qchunk_of][:, kchunk_of]
    s = bf(q)[0, 0] @ bf(k)[0, 0].T * scale
    s = np.where(tokmask, s, -np.inf)
    mx = s.max(-1, keepdims=True)
    w = np.exp(s - mx)
    ref = (w / w.sum(-1, keepdims=True)) @ bf(v)[0, 0]
    np.testing.assert_allclose(out, ref[qtok], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, (mx[:, 0] + np.log(w.sum(-1)))[qtok], rtol=0, atol=1e-12)


def test_all_64_token_chunks_equals_dense():
    wl = W0.with_(T=8, H=8, W=12, heads=2)              # partial chunk column (w = 8..11)
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    nq = oracle.num_chunks(wl.T, wl.H, wl.W, Q64)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, "topk", nq, kchunk=Q64, qchunk=Q64)
    rows = np.arange(2 * nq)
    out, lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows, kchunk=Q64,
                             qchunk=Q64)
    qtok = np.concatenate([(r // nq) * wl.N + oracle.chunk_tokens(wl.T, wl.H, wl.W, r % nq, Q64)
                           for r in rows])
    ref, ref_lse = oracle.dense(q, k, v, wl.T, wl.H, wl.W, scale, qtok)
    np.testing.assert_allclose(out.reshape(-1, wl.d), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), ref_lse, rtol=0, atol=1e-12)


def test_64_token_query_rows_are_the_halves_of_128_token_rows_when_keys_agree():
    """A (4,4,8) query chunk is two (4,4,4) chunks side by side in w. Given the
    same key chunks, their outputs are the two halves (lw < 4, lw >= 4) of the
    (4,4,8) chunk's output."""
    wl = W0.with_(T=8, H=8, W=16, heads=1)
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    rp8 = np.array([0, 2, 4, 6, 8], dtype=np.int32)                 # 4 chunks of 128
    ci8 = np.array([0, 3, 1, 2, 0, 2, 1, 3], dtype=np.int32)
    out8, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp8, ci8, np.arange(4))
    # the same selection written for the 8 query chunks of 64 tokens: chunk 2c, 2c+1
    # of the (4,4,4) grid are the w-halves of chunk c of the (4,4,8) grid
    rp4 = np.arange(0, 17, 2, dtype=np.int32)
    ci4 = np.repeat(ci8.reshape(4, 2), 2, axis=0).reshape(-1).astype(np.int32)
    out4, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp4, ci4, np.arange(8),
                            kchunk=(4, 4, 8), qchunk=Q64)
    lw = np.arange(128) % 8
    for c in range(4):
        np.testing.assert_allclose(out4[2 * c], out8[c][lw < 4], rtol=0, atol=1e-12)
        np.testing.assert_allclose(out4[2 * c + 1], out8[c][lw >= 4], rtol=0, atol=1e-12)


def _q64_maps(wl, kchunk):
    """Token index of every (chunk, slot) for (4,4,4) query chunks and the given
    key chunks, from numpy reshapes, and the inverse (token -> chunk) maps."""
    iota = np.arange(wl.N).reshape(1, 1, -1, 1)
    qtok = numpy_rearrange64(iota, wl.T, wl.H, wl.W)[0, 0, :, :, 0]
    kt, kh, kw = kchunk
    kv = iota.reshape(wl.T // kt, kt, wl.H // kh, kh, wl.W // kw, kw)
    ktok = kv.transpose(0, 2, 4, 1, 3, 5).reshape(-1, kt * kh * kw)
    qchunk_of = np.empty(wl.N, dtype=np.int64)
    qchunk_of[qtok.reshape(-1)] = np.repeat(np.arange(qtok.shape[0]), qtok.shape[1])
    kchunk_of = np.empty(wl.N, dtype=np.int64)
    kchunk_of[ktok.reshape(-1)] = np.repeat(np.arange(ktok.shape[0]), ktok.shape[1])
    return qtok, qchunk_of, kchunk_of


@pytest.mark.parametrize("kchunk", [Q64, (4, 4, 8)])
def test_backward_of_64_token_query_chunks_equals_torch_autograd(kchunk):
    """The oracle's gradients with (4,4,4) query chunks against torch float64
    autograd of the dense softmax attention under the chunk mask lifted to
    tokens with numpy reshapes; one query chunk selects nothing (its queries
    have no output and no gradient)."""
    wl = W0.with_(T=8, H=8, W=16, heads=1, d=32)
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    scale = 0.3
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, "topk", 3, kchunk=kchunk, qchunk=Q64)
    nq = oracle.num_chunks(wl.T, wl.H, wl.W, Q64)
    nk = oracle.num_chunks(wl.T, wl.H, wl.W, kchunk)
    lists = [list(ci[rp[i]:rp[i + 1]]) for i in range(nq)]
    lists[5] = []                                            # an empty row
    rp = np.concatenate([[0], np.cumsum([len(r) for r in lists])]).astype(np.int32)
    ci = np.array([c for r in lists for c in r], dtype=np.int32)
    dq_rows, dk, dv = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp, ci,
                                        np.arange(nq), kchunk=kchunk, qchunk=Q64)
    assert dq_rows.shape == (nq, 64, wl.d)
    qtok, qchunk_of, kchunk_of = _q64_maps(wl, kchunk)
    dq = np.zeros((wl.N, wl.d))
    for i in range(nq):
        dq[qtok[i]] = dq_rows[i]
    M = np.zeros((nq, nk), dtype=bool)
    for i in range(nq):
        M[i, lists[i]] = True
    tm = torch.from_numpy(M[qchunk_of][:, kchunk_of])
    Q, K, V = (torch.tensor(bf(x)[0, 0], dtype=torch.float64, requires_grad=True)
               for x in (q, k, v))
    G = torch.tensor(bf(g)[0, 0], dtype=torch.float64)
    live = tm.any(-1)
    s = (Q @ K.T) * scale
    s = s.masked_fill(~tm, float("-inf"))
    s = torch.where(live[:, None], s, torch.zeros_like(s))
    w = torch.softmax(s, -1) * live[:, None]
    (G * (w @ V)).sum().backward()
    np.testing.assert_allclose(dq, Q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk[0, 0], K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv[0, 0], V.grad.numpy(), rtol=0, atol=1e-12)
    assert np.all(dq[qtok[5]] == 0) and np.abs(dq).max() > 1e-3 and np.abs(dk).max() > 1e-3


def test_backward_of_64_token_rows_equals_128_token_rows_when_keys_agree():
    """Selections written for the 8 query chunks of (4,4,4) that give both
    w-halves of every (4,4,8) chunk the same keys: dQ of each 64-token chunk is
    the matching half of the (4,4,8) chunk's dQ, and dK, dV are the same."""
    wl = W0.with_(T=8, H=8, W=16, heads=1)
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    scale = 1 / math.sqrt(wl.d)
    rp8 = np.array([0, 2, 4, 6, 8], dtype=np.int32)
    ci8 = np.array([0, 3, 1, 2, 0, 2, 1, 3], dtype=np.int32)
    dq8, dk8, dv8 = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp8, ci8, np.arange(4))
    rp4 = np.arange(0, 17, 2, dtype=np.int32)
    ci4 = np.repeat(ci8.reshape(4, 2), 2, axis=0).reshape(-1).astype(np.int32)
    dq4, dk4, dv4 = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp4, ci4, np.arange(8),
                                      kchunk=(4, 4, 8), qchunk=Q64)
    lw = np.arange(128) % 8
    for c in range(4):
        np.testing.assert_allclose(dq4[2 * c], dq8[c][lw < 4], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dq4[2 * c + 1], dq8[c][lw >= 4], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk4, dk8, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv4, dv8, rtol=0, atol=1e-12)
