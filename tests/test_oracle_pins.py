"""Pins of the CPU oracle against things other than itself (no GPU).

Each test ties one oracle function to a hand-derived fixture (tests/golden), a
library routine (numpy reshape / sort / matmul), brute force on tiny inputs, a
closed form or an invariant, so that a dropped term, a wrong index or a
transposed operand in the oracle fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_to_bf16_bits(a):
    """Round float32 to bf16 (RNE) bit patterns -- used only to build inputs."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64)


def block_view(x, T, H, W):
    """[B,Hh,N,d] -> [B,Hh,NT,4,NH,4,NW,8,d] with numpy's reshape."""
    B, Hh, N, d = x.shape
    return x.reshape(B, Hh, T // 4, 4, H // 4, 4, W // 8, 8, d)


def numpy_rearrange(x, T, H, W):
    B, Hh, N, d = x.shape
    v = block_view(x, T, H, W).transpose(0, 1, 2, 4, 6, 3, 5, 7, 8)
    return v.reshape(B, Hh, N // 128, 128, d)


def chunk_const_tensor(T, H, W, d, values):
    """A [1,1,N,d] float tensor whose tokens in chunk c all equal values[c] (a d-vector)."""
    x = np.zeros((1, 1, T, H, W, d), dtype=np.float32)
    NH, NW = H // 4, W // 8
    for c, vec in enumerate(values):
        ct, ch, cw = c // (NH * NW), (c // NW) % NH, c % NW
        x[0, 0, ct * 4:(ct + 1) * 4, ch * 4:(ch + 1) * 4, cw * 8:(cw + 1) * 8, :] = vec
    return f32_to_bf16_bits(x.reshape(1, 1, T * H * W, d))


# ---------------------------------------------------------------- chunking

def test_chunk_index_hand_fixture():
    rows = []
    with open(os.path.join(GOLDEN, "chunk_index_hand.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    assert len(rows) >= 10
    for T, H, W, t, h, w, c, l in rows:
        assert oracle.token_of(T, H, W, c, l) == (t * H + h) * W + w, (t, h, w, c, l)


def test_rearrange_equals_numpy_block_transpose():
    wl = synth.WORKLOADS["tiny"].with_(T=8, H=8, W=16, heads=3)
    q, _, _ = synth.make_qkv(wl)
    got = oracle.rearrange(q, wl.T, wl.H, wl.W)
    np.testing.assert_array_equal(got, numpy_rearrange(q, wl.T, wl.H, wl.W))
    # and it is a permutation of each head's tokens
    np.testing.assert_array_equal(np.sort(got[0, 1].reshape(-1), kind="stable"),
                                  np.sort(q[0, 1].reshape(-1), kind="stable"))


# ---------------------------------------------------------------- pooling

def test_pool_chunk_id_hand():
    T, H, W, d = 8, 8, 16, 64
    x = chunk_const_tensor(T, H, W, d, [np.full(d, c, np.float32) for c in range(8)])
    p = oracle.pool(x, T, H, W)
    for c in range(8):
        assert np.all(p[0, 0, c] == c)


def test_pool_equals_numpy_block_mean_and_sum_invariant():
    wl = synth.WORKLOADS["tiny"].with_(T=8, H=8, W=16, heads=2)
    q, _, _ = synth.make_qkv(wl)
    p = oracle.pool(q, wl.T, wl.H, wl.W)
    ref = bf(block_view(q, wl.T, wl.H, wl.W)).mean(axis=(3, 5, 7))  # [B,Hh,NT,NH,NW,d]
    np.testing.assert_allclose(p, ref.reshape(p.shape), rtol=0, atol=1e-14)
    np.testing.assert_allclose(p.sum(axis=2) * 128, bf(q).sum(axis=2), rtol=1e-12, atol=1e-10)


def test_pool_fp32_mode_close_to_fp64():
    wl = synth.WORKLOADS["tiny"]
    q, _, _ = synth.make_qkv(wl)
    p64 = oracle.pool(q, wl.T, wl.H, wl.W)
    p32 = oracle.pool(q, wl.T, wl.H, wl.W, fp32=True)
    assert np.all(p32.astype(np.float32).astype(np.float64) == p32)
    np.testing.assert_allclose(p32, p64, rtol=0, atol=1e-6)


# ---------------------------------------------------------------- scores

def test_scores_equal_matmul():
    rng = np.random.default_rng(1)
    qp = rng.standard_normal((2, 3, 5, 16))
    kp = rng.standard_normal((2, 3, 5, 16))
    s = oracle.scores(qp, kp, 0.25)
    np.testing.assert_allclose(s, np.einsum("bhid,bhmd->bhim", qp, kp) * 0.25, rtol=1e-13,
                               atol=1e-13)
    # not symmetric in general: a transposed operand would be caught
    assert not np.allclose(s, np.swapaxes(s, -1, -2))


# ---------------------------------------------------------------- top-k

def _parse_topk_fixture():
    cases = {}
    with open(os.path.join(GOLDEN, "topk_hand.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, rows = line.split(":")
            name, kk = head.split()
            k = int(kk.split("=")[1])
            cases[(name, k)] = [[int(x) for x in r.split()] for r in rows.split("|")]
    return cases


def _hand_case(name):
    d = 64
    e = np.eye(d, dtype=np.float32)
    if name == "onehot":
        qv = [e[i] for i in (0, 1, 2, 3)]
        kv = [e[m] for m in (2, 0, 3, 1)]
    elif name == "graded":
        qv = [e[0]] * 4
        kv = [a * e[0] for a in (0.5, 2.0, 1.0, 0.25)]
    elif name == "negated":
        qv = [-e[0]] * 4
        kv = [a * e[0] for a in (0.5, 2.0, 1.0, 0.25)]
    elif name == "ties":
        qv = [e[0]] * 4
        kv = [e[0]] * 4
    else:
        raise KeyError(name)
    return chunk_const_tensor(4, 8, 16, d, qv), chunk_const_tensor(4, 8, 16, d, kv)


@pytest.mark.parametrize("case", sorted(_parse_topk_fixture()))
def test_topk_hand_fixture(case):
    name, k = case
    expected = _parse_topk_fixture()[case]
    q, kk = _hand_case(name)
    rp, ci, _ = oracle.plan(q, kk, 4, 8, 16, 1 / 8, mode="topk", topk=k)
    assert list(rp) == [0, k, 2 * k, 3 * k, 4 * k]
    got = [list(ci[rp[i]:rp[i + 1]]) for i in range(4)]
    assert got == expected


def test_topk_equals_lexsort_selection():
    rng = np.random.default_rng(7)
    T, H, W = 8, 16, 32  # 32 chunks
    S = rng.standard_normal((2, 2, 32, 32))
    S[0, 0, 3, 5] = S[0, 0, 3, 9] = S[0, 0, 3, 1]  # exact ties
    for k in (1, 5, 17, 32):
        rp, ci = oracle.select(S, T, H, W, mode="topk", topk=k)
        flat = S.reshape(-1, 32)
        for r in range(flat.shape[0]):
            order = np.lexsort((np.arange(32), -flat[r]))  # score desc, index asc
            assert list(ci[rp[r]:rp[r + 1]]) == sorted(order[:k].tolist())


def test_topk_clamped_to_candidates_and_structure():
    rng = np.random.default_rng(3)
    S = rng.standard_normal((1, 1, 8, 8))
    rp, ci = oracle.select(S, 8, 8, 16, mode="topk", topk=50)
    assert list(np.diff(rp)) == [8] * 8
    assert all(list(ci[rp[r]:rp[r + 1]]) == list(range(8)) for r in range(8))


# ---------------------------------------------------------------- CDF

def _bruteforce_cdf(row_scores, cand, p, cap_frac):
    """Smallest subset size reaching mass >= p (all subsets enumerated)."""
    s = np.array([row_scores[m] for m in cand])
    w = np.exp(s - s.max())
    w /= w.sum()
    n = len(cand)
    best = n
    for size in range(1, n + 1):
        if any(w[list(sub)].sum() >= p for sub in itertools.combinations(range(n), size)):
            best = size
            break
    cap = max(1, math.floor(cap_frac * n))
    return min(best, cap)


@pytest.mark.parametrize("p,cap_frac", [(0.9, 1.0), (0.5, 1.0), (0.9, 0.25), (0.7, 0.5)])
def test_cdf_bruteforce_minimal_subset(p, cap_frac):
    rng = np.random.default_rng(11)
    T, H, W = 4, 8, 32  # 8 chunks
    S = rng.standard_normal((1, 3, 8, 8)) * 1.5
    rp, ci = oracle.select(S, T, H, W, mode="cdf", cdf_p=p, cap_frac=cap_frac)
    flat = S.reshape(-1, 8)
    for r in range(flat.shape[0]):
        cnt = _bruteforce_cdf(flat[r], list(range(8)), p, cap_frac)
        got = list(ci[rp[r]:rp[r + 1]])
        assert len(got) == cnt
        order = np.lexsort((np.arange(8), -flat[r]))
        assert got == sorted(order[:cnt].tolist())


@pytest.mark.parametrize("k,p", [(2, 0.5), (4, 0.3), (6, 0.9), (1, 0.05)])
def test_topk_cdf_combination_is_the_intersection(k, p):
    """Combination mode keeps the chunks both rules keep: the lexsort top-k set
    intersected with the brute-force minimal CDF set."""
    rng = np.random.default_rng(5 + k)
    Nc = 8
    S = rng.normal(size=(1, 1, Nc, Nc)) * 1.5
    S[0, 0, 3, :4] = S[0, 0, 3, 4]                    # a row with ties
    T, H, W = 4, 8, 32                                  # 1 x 2 x 4 = 8 chunks
    rp, ci = oracle.select(S, T, H, W, mode="topk_cdf", topk=k, cdf_p=p, cap_frac=1.0)
    for i in range(Nc):
        row = S[0, 0, i]
        order = np.lexsort((np.arange(Nc), -row))      # score desc, index asc
        topk_set = set(order[:min(k, Nc)].tolist())
        cdf_set = set(order[:_bruteforce_cdf(row, np.arange(Nc), p, 1.0)].tolist())
        assert set(ci[rp[i]:rp[i + 1]].tolist()) == (topk_set & cdf_set), i


def test_cdf_special_cases():
    T, H, W = 4, 8, 32
    rng = np.random.default_rng(5)
    S = rng.standard_normal((1, 1, 8, 8))
    rp, ci = oracle.select(S, T, H, W, mode="cdf", cdf_p=1.0, cap_frac=1.0)
    assert list(np.diff(rp)) == [8] * 8           # p = 1, no cap -> every candidate
    S2 = np.zeros((1, 1, 8, 8))
    S2[0, 0, :, 6] = 60.0                          # one dominant chunk per row
    rp, ci = oracle.select(S2, T, H, W, mode="cdf", cdf_p=0.9, cap_frac=1.0)
    assert list(np.diff(rp)) == [1] * 8 and list(ci) == [6] * 8
    S3 = np.zeros((1, 1, 8, 8))                    # flat row: mass grows 1/8 per chunk
    rp, ci = oracle.select(S3, T, H, W, mode="cdf", cdf_p=0.5, cap_frac=1.0)
    assert list(np.diff(rp)) == [4] * 8 and list(ci[:4]) == [0, 1, 2, 3]


def test_cdf_minimality_invariant_random():
    rng = np.random.default_rng(9)
    T, H, W = 8, 16, 32
    S = rng.standard_normal((1, 2, 32, 32)) * 2
    rp, ci = oracle.select(S, T, H, W, mode="cdf", cdf_p=0.9, cap_frac=0.25)
    flat = S.reshape(-1, 32)
    for r in range(flat.shape[0]):
        got = ci[rp[r]:rp[r + 1]]
        w = np.exp(flat[r] - flat[r].max())
        w /= w.sum()
        mass = np.sort(w)[::-1]
        cnt = len(got)
        assert 1 <= cnt <= 8
        if cnt < 8:  # cap not binding: minimal prefix reaching 0.9
            assert mass[:cnt].sum() >= 0.9 and mass[:cnt - 1].sum() < 0.9
        else:  # cap binding (or exactly reached): 7 chunks were not enough
            assert mass[:7].sum() < 0.9


# ---------------------------------------------------------------- block-causal selection

def test_block_causal_candidates():
    T, H, W = 8, 8, 16  # 8 chunks; chunks 0..3 have frames 0..3
    S = np.zeros((1, 1, 8, 8))
    S[0, 0, :, 4:] = 5.0   # noisy key chunks score highest for every query chunk
    S[0, 0, :, 2] = 1.0
    rp, ci = oracle.select(S, T, H, W, mode="topk", topk=2, t_cond=4)
    rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(8)]
    for i in range(4):      # condition query chunks: only chunks 0..3, best is 2 then 0
        assert rows[i] == [0, 2]
    for i in range(4, 8):   # noisy query chunks: all candidates, best are 4 and 5
        assert rows[i] == [4, 5]
    rp, ci = oracle.select(S, T, H, W, mode="cdf", cdf_p=0.9, cap_frac=1.0, t_cond=4)
    for i in range(4):
        assert all(c < 4 for c in ci[rp[i]:rp[i + 1]])


# ---------------------------------------------------------------- attention

def _dense_numpy(q, k, v, scale, n_keys=None):
    qf, kf, vf = bf(q), bf(k), bf(v)
    if n_keys is not None:
        kf, vf = kf[:, :, :n_keys], vf[:, :, :n_keys]
    s = np.einsum("bhnd,bhmd->bhnm", qf, kf) * scale
    s -= s.max(-1, keepdims=True)
    w = np.exp(s)
    w /= w.sum(-1, keepdims=True)
    return np.einsum("bhnm,bhmd->bhnd", w, vf)


def test_dense_equals_numpy_softmax():
    wl = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    ids = np.arange(0, 2 * wl.N, 37)
    out, lse = oracle.dense(q, k, v, wl.T, wl.H, wl.W, scale, ids)
    ref = _dense_numpy(q, k, v, scale).reshape(-1, wl.d)[ids]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    s = np.einsum("nd,nmd->nm", bf(q).reshape(-1, wl.d)[ids],
                  bf(k).reshape(2, wl.N, wl.d)[ids // wl.N]) * scale
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(-1)), rtol=0, atol=1e-12)


def test_dense_block_causal_equals_numpy_masked():
    wl = synth.WORKLOADS["tiny"].with_(T=8, t_cond=4)
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    HW = wl.H * wl.W
    cond_ids = np.arange(0, 4 * HW, 13)             # head 0 queries in condition frames
    noisy_ids = np.arange(4 * HW, wl.N, 17)
    out_c, _ = oracle.dense(q, k, v, wl.T, wl.H, wl.W, scale, cond_ids, t_cond=4)
    out_n, _ = oracle.dense(q, k, v, wl.T, wl.H, wl.W, scale, noisy_ids, t_cond=4)
    ref_c = _dense_numpy(q, k, v, scale, n_keys=4 * HW)[0, 0][cond_ids]
    ref_n = _dense_numpy(q, k, v, scale)[0, 0][noisy_ids]
    np.testing.assert_allclose(out_c, ref_c, atol=1e-12, rtol=0)
    np.testing.assert_allclose(out_n, ref_n, atol=1e-12, rtol=0)


@pytest.mark.parametrize("grid", [(4, 8, 16, 64), (8, 16, 32, 64)])
def test_sparse_with_all_chunks_equals_dense(grid):
    T, H, W, d = grid
    wl = synth.WORKLOADS["tiny"].with_(T=T, H=H, W=W, d=d)
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(d)
    rp, ci, _ = oracle.plan(q, k, T, H, W, scale, mode="topk", topk=wl.Nc)
    rows = np.arange(wl.rows) if wl.rows <= 8 else np.arange(0, wl.rows, 5)
    out, lse = oracle.attend(q, k, v, T, H, W, scale, rp, ci, rows)
    qtok = np.concatenate([(r // wl.Nc) * wl.N + oracle.chunk_tokens(T, H, W, r % wl.Nc)
                           for r in rows])
    ref, ref_lse = oracle.dense(q, k, v, T, H, W, scale, qtok)
    np.testing.assert_allclose(out.reshape(-1, d), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), ref_lse, rtol=0, atol=1e-12)


def test_sparse_equals_numpy_token_masked_softmax():
    """Chunk mask lifted to tokens with numpy, then a masked dense softmax."""
    wl = synth.WORKLOADS["tiny"].with_(T=8, H=8, W=16, heads=1)  # 8 chunks
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, mode="topk", topk=3)
    out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, np.arange(8))
    # chunk id of every token via numpy reshape of an iota
    iota = np.arange(wl.N).reshape(1, 1, wl.N, 1).astype(np.int64)
    tok_of = numpy_rearrange(iota, wl.T, wl.H, wl.W).reshape(8, 128)  # [chunk, local] -> token
    chunk_of = np.empty(wl.N, dtype=np.int64)
    chunk_of[tok_of.reshape(-1)] = np.repeat(np.arange(8), 128)
    M = np.zeros((8, 8), dtype=bool)
    for i in range(8):
        M[i, ci[rp[i]:rp[i + 1]]] = True
    tokmask = M[chunk_of][:, chunk_of]                 # [query token, key token]
    s = bf(q)[0, 0] @ bf(k)[0, 0].T * scale
    s = np.where(tokmask, s, -np.inf)
    s -= s.max(-1, keepdims=True)
    w = np.exp(s)
    w /= w.sum(-1, keepdims=True)
    ref = (w @ bf(v)[0, 0])[tok_of]                    # [chunk, local, d]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_convexity_and_unit_weights():
    wl = synth.WORKLOADS["tiny"].with_(T=8, H=8, W=16)
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, mode="topk", topk=3)
    rows = np.arange(wl.rows)
    out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    vf = bf(v).reshape(wl.B * wl.heads, wl.N, wl.d)
    for r in rows:
        keys = np.concatenate([oracle.chunk_tokens(wl.T, wl.H, wl.W, c)
                               for c in ci[rp[r]:rp[r + 1]]])
        vv = vf[r // wl.Nc][keys]
        assert np.all(out[r] >= vv.min(0) - 1e-12) and np.all(out[r] <= vv.max(0) + 1e-12)
    ones = np.full_like(v, 0x3F80)  # bf16 1.0
    out1, _ = oracle.attend(q, k, ones, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    np.testing.assert_allclose(out1, 1.0, rtol=0, atol=1e-14)


def test_zero_keys_closed_form():
    """K = 0: every logit is 0, so O = mean of the selected V rows, LSE = log(#keys)."""
    wl = synth.WORKLOADS["tiny"]
    q, _, v = synth.make_qkv(wl)
    k = np.zeros_like(q)
    rp = np.array([0, 2, 3, 3, 4, 4, 4, 4, 4], dtype=np.int32)  # rows with 2,1,0,1,0.. chunks
    ci = np.array([1, 3, 0, 2], dtype=np.int32)
    out, lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, 0.125, rp, ci, np.arange(8))
    vf = bf(v).reshape(2, wl.N, wl.d)
    for r in range(8):
        chunks = ci[rp[r]:rp[r + 1]]
        if len(chunks) == 0:
            assert np.all(out[r] == 0) and np.all(np.isneginf(lse[r]))
            continue
        keys = np.concatenate([oracle.chunk_tokens(wl.T, wl.H, wl.W, c) for c in chunks])
        np.testing.assert_allclose(out[r], np.broadcast_to(vf[r // 4][keys].mean(0), out[r].shape),
                                   rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[r], math.log(128 * len(chunks)), rtol=0, atol=1e-14)


def test_single_chunk_constant_value():
    wl = synth.WORKLOADS["tiny"].with_(heads=1)
    q, k, _ = synth.make_qkv(wl)
    consts = [0.5, -1.25, 2.0, 3.0]
    v = chunk_const_tensor(wl.T, wl.H, wl.W, wl.d, [np.full(wl.d, c, np.float32) for c in consts])
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, mode="topk", topk=1)
    out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, np.arange(4))
    for r in range(4):
        np.testing.assert_allclose(out[r], consts[ci[r]], rtol=0, atol=1e-14)


def test_block_causal_condition_outputs_ignore_noisy_tokens():
    wl = synth.WORKLOADS["tiny"].with_(T=8, t_cond=4, mode="cdf")
    q, k, v = synth.make_qkv(wl)
    scale = 1 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, mode="topk", topk=2, t_cond=4)
    rows = np.arange(wl.rows)
    out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    k2, v2 = k.copy(), v.copy()
    HW = wl.H * wl.W
    rng = np.random.default_rng(0)
    k2[:, :, 4 * HW:] = rng.integers(0, 0x3F00, size=k2[:, :, 4 * HW:].shape, dtype=np.uint16)
    v2[:, :, 4 * HW:] = rng.integers(0, 0x3F00, size=v2[:, :, 4 * HW:].shape, dtype=np.uint16)
    rp2, ci2, _ = oracle.plan(q, k2, wl.T, wl.H, wl.W, scale, mode="topk", topk=2, t_cond=4)
    out2, _ = oracle.attend(q, k2, v2, wl.T, wl.H, wl.W, scale, rp2, ci2, rows)
    cond_rows = [r for r in rows if (r % wl.Nc) < wl.n_cond]
    assert cond_rows
    for r in cond_rows:
        assert np.array_equal(out[r], out2[r])
        assert list(ci[rp[r]:rp[r + 1]]) == list(ci2[rp2[r]:rp2[r + 1]])
