"""Pins of the oracle on grids whose T, H, W are not multiples of the (4,4,8)
chunk shape ("LongCat-Video Technical Report", "Block Sparse Attention (BSA)":
blocks per axis by ceiling division, so edge chunks are partial). Each check
builds its expectation with numpy from a padded iota grid, independent of the
oracle's own index arithmetic."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

from test_oracle_pins import bf

GRIDS = [(6, 10, 20), (5, 8, 16), (4, 7, 9), (24, 45, 8)]


def padded_token_map(T, H, W):
    """[chunk, local] -> token index or -1, via a padded iota and numpy reshapes."""
    Tp, Hp, Wp = -(-T // 4) * 4, -(-H // 4) * 4, -(-W // 8) * 8
    iota = np.full((Tp, Hp, Wp), -1, dtype=np.int64)
    iota[:T, :H, :W] = np.arange(T * H * W).reshape(T, H, W)
    v = iota.reshape(Tp // 4, 4, Hp // 4, 4, Wp // 8, 8).transpose(0, 2, 4, 1, 3, 5)
    return v.reshape(-1, 128)


def case(T, H, W, heads=2, d=32):
    wl = synth.WORKLOADS["tiny"].with_(T=T, H=H, W=W, heads=heads, d=d)
    q, k, v = synth.make_qkv(wl)
    return wl, q, k, v


@pytest.mark.parametrize("grid", GRIDS)
def test_token_map_and_chunk_count(grid):
    T, H, W = grid
    tm = padded_token_map(T, H, W)
    assert oracle.num_chunks(T, H, W) == tm.shape[0]
    for c in range(tm.shape[0]):
        assert np.array_equal(oracle.chunk_tokens(T, H, W, c), tm[c]), c
    # every token appears exactly once
    got = tm[tm >= 0]
    assert np.array_equal(np.sort(got), np.arange(T * H * W))


@pytest.mark.parametrize("grid", GRIDS[:3])
def test_rearrange_and_pool_partial(grid):
    T, H, W = grid
    wl, q, _, _ = case(T, H, W)
    tm = padded_token_map(T, H, W)
    r = oracle.rearrange(q, T, H, W)
    for c in range(tm.shape[0]):
        ok = tm[c] >= 0
        assert np.array_equal(r[:, :, c][:, :, ok], q[:, :, tm[c][ok]])
        assert not r[:, :, c][:, :, ~ok].any()
    p = oracle.pool(q, T, H, W)
    qf = bf(q)
    for c in range(tm.shape[0]):
        ok = tm[c] >= 0
        np.testing.assert_allclose(p[:, :, c], qf[:, :, tm[c][ok]].mean(2), rtol=0, atol=1e-12)


def masked_attention_numpy(q, k, v, tm, rp, ci, scale, heads, Nc):
    """Token-level masked softmax: a key token is allowed for a query token when
    the key's chunk is in the query chunk's CSR row."""
    qf, kf, vf = bf(q)[0], bf(k)[0], bf(v)[0]
    N = qf.shape[1]
    chunk_of = np.empty(N, dtype=np.int64)
    for c in range(tm.shape[0]):
        chunk_of[tm[c][tm[c] >= 0]] = c
    out = np.full((heads, N, qf.shape[2]), np.nan)
    for h in range(heads):
        M = np.zeros((Nc, Nc), dtype=bool)
        for i in range(Nc):
            M[i, ci[rp[h * Nc + i]:rp[h * Nc + i + 1]]] = True
        allowed = M[chunk_of][:, chunk_of]
        s = np.where(allowed, qf[h] @ kf[h].T * scale, -np.inf)
        live = allowed.any(1)
        s = s[live] - s[live].max(1, keepdims=True)
        w = np.exp(s)
        w /= w.sum(1, keepdims=True)
        out[h][live] = w @ vf[h]
        out[h][~live] = 0.0
    return out


@pytest.mark.parametrize("grid", GRIDS[:3])
def test_sparse_attention_partial_equals_token_masked_softmax(grid):
    T, H, W = grid
    wl, q, k, v = case(T, H, W)
    scale = 1 / math.sqrt(wl.d)
    Nc = wl.Nc
    rp, ci, _ = oracle.plan(q, k, T, H, W, scale, mode="topk", topk=max(1, Nc // 3))
    out, lse = oracle.attend(q, k, v, T, H, W, scale, rp, ci, np.arange(wl.heads * Nc))
    ref = masked_attention_numpy(q, k, v, padded_token_map(T, H, W), rp, ci, scale, wl.heads, Nc)
    tm = padded_token_map(T, H, W)
    for r in range(wl.heads * Nc):
        h, c = divmod(r, Nc)
        ok = tm[c] >= 0
        np.testing.assert_allclose(out[r][ok], ref[h][tm[c][ok]], rtol=0, atol=1e-12)
        assert np.all(np.isnan(out[r][~ok])) and np.all(np.isnan(lse[r][~ok]))


@pytest.mark.parametrize("grid", GRIDS[:3])
def test_all_chunks_partial_equals_dense(grid):
    T, H, W = grid
    wl, q, k, v = case(T, H, W)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, T, H, W, scale, mode="topk", topk=wl.Nc)
    tm = padded_token_map(T, H, W)
    rows = np.arange(wl.heads * wl.Nc)
    out, lse = oracle.attend(q, k, v, T, H, W, scale, rp, ci, rows)
    for r in rows:
        h, c = divmod(r, wl.Nc)
        ok = tm[c] >= 0
        ref, ref_lse = oracle.dense(q, k, v, T, H, W, scale, h * wl.N + tm[c][ok])
        np.testing.assert_allclose(out[r][ok], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[r][ok], ref_lse, rtol=0, atol=1e-12)


def test_backward_partial_equals_torch_autograd():
    T, H, W = 6, 10, 20
    wl, q, k, v = case(T, H, W, heads=1, d=16)
    g = synth.make_dout(wl)
    scale = 0.3
    Nc = wl.Nc
    rp, ci, _ = oracle.plan(q, k, T, H, W, scale, mode="topk", topk=3)
    rows = np.arange(Nc)
    dq_rows, dk, dv = oracle.attend_bwd(q, k, v, g, T, H, W, scale, rp, ci, rows)
    tm = padded_token_map(T, H, W)
    chunk_of = np.empty(wl.N, dtype=np.int64)
    for c in range(Nc):
        chunk_of[tm[c][tm[c] >= 0]] = c
    M = np.zeros((Nc, Nc), dtype=bool)
    for i in range(Nc):
        M[i, ci[rp[i]:rp[i + 1]]] = True
    allowed = torch.from_numpy(M[chunk_of][:, chunk_of])
    Q, K, V = (torch.tensor(bf(x)[0, 0], dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    G = torch.tensor(bf(g)[0, 0], dtype=torch.float64)
    s = (Q @ K.T * scale).masked_fill(~allowed, float("-inf"))
    loss = (G * (torch.softmax(s, -1) @ V)).sum()
    loss.backward()
    for r in rows:
        ok = tm[r] >= 0
        np.testing.assert_allclose(dq_rows[r][ok], Q.grad.numpy()[tm[r][ok]], rtol=0, atol=1e-12)
        assert np.all(np.isnan(dq_rows[r][~ok]))
    np.testing.assert_allclose(dk[0, 0], K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv[0, 0], V.grad.numpy(), rtol=0, atol=1e-12)
