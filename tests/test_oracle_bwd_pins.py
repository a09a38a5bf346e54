"""Pins of the oracle's backward (gradients of the block-sparse attention) on
the CPU, against things other than itself: torch autograd of a token-masked
dense softmax attention in float64 (a library routine the oracle does not
use), central finite differences of a numpy forward, and closed forms /
invariants of the softmax gradient."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

from test_oracle_pins import bf, chunk_const_tensor, numpy_rearrange


def tiny_case(heads=2, d=32, T=8, H=8, W=16):
    wl = synth.WORKLOADS["tiny"].with_(heads=heads, d=d, T=T, H=H, W=W)
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    return wl, q, k, v, g


def hand_csr(Nc, heads):
    """Rows of varied length per head, one of them empty, columns unsorted-free."""
    rows = []
    for h in range(heads):
        for i in range(Nc):
            if i == 3:
                rows.append([])                                   # empty row
            else:
                rows.append(sorted({i, (i * 3 + h) % Nc, (i + 5) % Nc}))
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate([np.array(r, dtype=np.int32) for r in rows]).astype(np.int32)
    return rp, ci


def token_maps(T, H, W):
    N = T * H * W
    iota = np.arange(N).reshape(1, 1, N, 1).astype(np.int64)
    tok_of = numpy_rearrange(iota, T, H, W).reshape(N // 128, 128)
    chunk_of = np.empty(N, dtype=np.int64)
    chunk_of[tok_of.reshape(-1)] = np.repeat(np.arange(N // 128), 128)
    return tok_of, chunk_of


def token_mask(rp, ci, Nc, heads, chunk_of):
    """[heads, N, N] boolean: key token allowed for query token (numpy lift of the CSR)."""
    M = np.zeros((heads, Nc, Nc), dtype=bool)
    for h in range(heads):
        for i in range(Nc):
            r = h * Nc + i
            M[h, i, ci[rp[r]:rp[r + 1]]] = True
    return M[:, chunk_of][:, :, chunk_of]


def numpy_loss(qf, kf, vf, gf, tm, scale):
    """sum(dO * O) with O the token-masked softmax attention (empty rows give O = 0)."""
    total = 0.0
    for h in range(qf.shape[0]):
        s = qf[h] @ kf[h].T * scale
        s = np.where(tm[h], s, -np.inf)
        live = tm[h].any(1)
        s = s[live]
        s -= s.max(-1, keepdims=True)
        w = np.exp(s)
        w /= w.sum(-1, keepdims=True)
        total += float(np.sum(gf[h][live] * (w @ vf[h])))
    return total


def oracle_grads(wl, q, k, v, g, rp, ci, scale):
    rows = np.arange(wl.rows)
    dq_rows, dk, dv = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    tok_of, _ = token_maps(wl.T, wl.H, wl.W)
    dq = np.zeros((wl.B * wl.heads, wl.N, wl.d))
    for r in rows:
        dq[r // wl.Nc][tok_of[r % wl.Nc]] = dq_rows[r]
    return dq.reshape(q.shape), dk, dv


def test_bwd_equals_torch_autograd_of_token_masked_attention():
    wl, q, k, v, g = tiny_case()
    scale = 1 / math.sqrt(wl.d)
    rp, ci = hand_csr(wl.Nc, wl.heads)
    dq, dk, dv = oracle_grads(wl, q, k, v, g, rp, ci, scale)
    _, chunk_of = token_maps(wl.T, wl.H, wl.W)
    tm = torch.from_numpy(token_mask(rp, ci, wl.Nc, wl.heads, chunk_of))
    Q, K, V = (torch.tensor(bf(x)[0], dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    G = torch.tensor(bf(g)[0], dtype=torch.float64)
    live = tm.any(-1)                                            # [heads, N]
    s = torch.einsum("hnd,hmd->hnm", Q, K) * scale
    s = s.masked_fill(~tm, float("-inf"))
    s = torch.where(live[..., None], s, torch.zeros_like(s))     # empty rows: no -inf row
    w = torch.softmax(s, -1) * live[..., None]                   # and no output
    loss = (G * torch.einsum("hnm,hmd->hnd", w, V)).sum()
    loss.backward()
    np.testing.assert_allclose(dq[0], Q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk[0], K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv[0], V.grad.numpy(), rtol=0, atol=1e-12)
    assert np.abs(dq[0]).max() > 1e-3 and np.abs(dk[0]).max() > 1e-3


def test_bwd_central_finite_differences():
    wl, q, k, v, g = tiny_case(heads=1, d=16, T=4, H=8, W=16)   # 4 chunks, 512 tokens
    scale = 0.4
    rp = np.array([0, 2, 3, 3, 6], dtype=np.int32)              # rows {0,2}, {1}, {}, {0,1,3}
    ci = np.array([0, 2, 1, 0, 1, 3], dtype=np.int32)
    dq, dk, dv = oracle_grads(wl, q, k, v, g, rp, ci, scale)
    _, chunk_of = token_maps(wl.T, wl.H, wl.W)
    tm = token_mask(rp, ci, wl.Nc, 1, chunk_of)
    X = [bf(x)[0].copy() for x in (q, k, v)]
    gf = bf(g)[0]
    rng = np.random.default_rng(7)
    eps = 1e-5
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(12):
            n, c = int(rng.integers(0, wl.N)), int(rng.integers(0, wl.d))
            Xp = [x.copy() for x in X]
            Xm = [x.copy() for x in X]
            Xp[which][0, n, c] += eps
            Xm[which][0, n, c] -= eps
            fd = (numpy_loss(*Xp, gf, tm, scale) - numpy_loss(*Xm, gf, tm, scale)) / (2 * eps)
            assert abs(fd - grad[0, 0, n, c]) <= 1e-7 * (1 + abs(fd)), (which, n, c, fd,
                                                                         grad[0, 0, n, c])


def test_bwd_invariants_sum_dk_zero_and_sum_dv_equals_live_dout():
    """sum_j dS[q,j] = 0 for every query, so dK summed over keys vanishes; the
    weights of a query sum to 1, so dV summed over keys equals dO summed over
    the queries whose row is not empty."""
    wl = synth.WORKLOADS["tiny"].with_(T=8, H=16, W=32, heads=2, d=64)
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, mode="topk", topk=5)
    dq, dk, dv = oracle_grads(wl, q, k, v, g, rp, ci, scale)
    gf = bf(g)
    for h in range(wl.heads):
        np.testing.assert_allclose(dk[0, h].sum(0), 0.0, rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[0, h].sum(0), gf[0, h].sum(0), rtol=0, atol=1e-10)
    assert np.abs(dk).max() > 1e-3
    # zero upstream gradient -> zero gradients
    z = np.zeros_like(g)
    dq0, dk0, dv0 = oracle_grads(wl, q, k, v, z, rp, ci, scale)
    assert not dq0.any() and not dk0.any() and not dv0.any()


def test_bwd_single_chunk_constant_value_has_no_qk_gradient():
    """One selected chunk with chunk-constant V: O is that constant whatever Q
    and K are, so dQ = dK = 0, and dV of a key is sum_q P[q,j] dO[q]."""
    wl = synth.WORKLOADS["tiny"].with_(heads=1, d=16)
    q, k, _ = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    v = chunk_const_tensor(wl.T, wl.H, wl.W, wl.d,
                           [np.full(wl.d, c, np.float32) for c in (0.5, -1.25, 2.0, 3.0)])
    scale = 1 / math.sqrt(wl.d)
    rp = np.array([0, 1, 2, 3, 4], dtype=np.int32)
    ci = np.array([2, 0, 3, 1], dtype=np.int32)
    dq, dk, dv = oracle_grads(wl, q, k, v, g, rp, ci, scale)
    np.testing.assert_allclose(dq, 0.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, rtol=0, atol=1e-12)
    # softmax weights of query chunk i over chunk ci[i], from numpy
    tok_of, _ = token_maps(wl.T, wl.H, wl.W)
    qf, kf, gf = bf(q)[0, 0], bf(k)[0, 0], bf(g)[0, 0]
    for i in range(4):
        qt, kt = tok_of[i], tok_of[ci[i]]
        s = qf[qt] @ kf[kt].T * scale
        w = np.exp(s - s.max(1, keepdims=True))
        w /= w.sum(1, keepdims=True)
        np.testing.assert_allclose(dv[0, 0][kt], w.T @ gf[qt], rtol=0, atol=1e-12)


def test_bwd_rows_listed_separately_add_up():
    """dK/dV of a set of rows is the sum of the per-row contributions."""
    wl, q, k, v, g = tiny_case(heads=1)
    scale = 1 / math.sqrt(wl.d)
    rp, ci = hand_csr(wl.Nc, 1)
    _, dk_all, dv_all = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp, ci,
                                          np.arange(wl.Nc))
    dk_sum, dv_sum = np.zeros_like(dk_all), np.zeros_like(dv_all)
    for r in range(wl.Nc):
        _, dk_r, dv_r = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp, ci, [r])
        dk_sum += dk_r
        dv_sum += dv_r
    np.testing.assert_allclose(dk_sum, dk_all, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv_sum, dv_all, rtol=0, atol=1e-13)
