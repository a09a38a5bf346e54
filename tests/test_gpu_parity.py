"""GPU parity: every stage of the CUDA path against the CPU oracle on the same
seeded inputs (marked gpu; needs a B200).

Bars (from the method's targets): rearrangement bit-exact; pooled means within
1e-6 absolute of fp64; pooled scores within 1e-5 relative; chunk selection
bit-exact except near-ties within 1e-5 relative (tests/parity.py); attention
max-abs <= 2e-2 and mean-abs <= 2e-3 against the fp64 oracle evaluated on the
GPU's own CSR (so selection and attention errors stay separate).
"""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import ATT_MAX_ABS, ATT_MEAN_ABS, compare_attention, compare_csr, rows_of

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_sparse_attention_13_b200 as bsa  # noqa: E402

W = synth.WORKLOADS

# small cases that span several score tiles, a ragged tail and both head dims
SMALL = {
    "tiny": W["tiny"],
    "ragged60_d64": W["tiny"].with_(name="ragged60_d64", heads=3, T=8, H=24, W=40, d=64, topk=5),
    "ragged135_d128": W["tiny"].with_(name="ragged135_d128", heads=2, T=12, H=20, W=72, d=128,
                                      topk=9),
    "causal_topk": W["tiny"].with_(name="causal_topk", heads=2, T=16, H=16, W=32, d=128, topk=6,
                                   t_cond=8),
    "causal_cdf_small": W["tiny"].with_(name="causal_cdf_small", B=2, heads=2, T=16, H=16, W=32,
                                        d=128, mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25,
                                        t_cond=8),
    "cdf_nocap": W["tiny"].with_(name="cdf_nocap", heads=2, T=8, H=16, W=32, d=64, mode="cdf",
                                 cdf_p=0.5, cdf_cap_frac=1.0),
    # combination mode where each rule binds on some rows: CDF counts 3-12 against k = 5 or 6
    "topk_cdf_small": W["tiny"].with_(name="topk_cdf_small", heads=2, T=8, H=16, W=32, d=128,
                                      mode="topk_cdf", topk=6, cdf_p=0.2, cdf_cap_frac=0.5),
    # key chunks larger than the query chunk (256, 512, 1024 tokens), incl. partial ones
    "kchunk_256": W["tiny"].with_(name="kchunk_256", heads=2, T=8, H=16, W=32, d=64, topk=3,
                                  kchunk=(4, 8, 8)),
    "kchunk_512_partial": W["tiny"].with_(name="kchunk_512_partial", heads=2, T=10, H=13, W=37,
                                          d=128, topk=3, kchunk=(8, 8, 8)),
    "kchunk_1024_causal_cdf": W["tiny"].with_(name="kchunk_1024_causal_cdf", B=2, heads=2, T=16,
                                              H=16, W=64, d=64, mode="cdf", cdf_p=0.9,
                                              cdf_cap_frac=0.5, t_cond=8, kchunk=(8, 8, 16)),
    # partial edge chunks: grids that are not multiples of (4, 4, 8)
    "partial_topk": W["tiny"].with_(name="partial_topk", heads=2, T=6, H=10, W=20, d=64, topk=5),
    "partial_causal_cdf": W["tiny"].with_(name="partial_causal_cdf", B=2, heads=2, T=10, H=13,
                                          W=28, d=128, mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25,
                                          t_cond=4),
    "causal_topk_cdf": W["tiny"].with_(name="causal_topk_cdf", B=2, heads=2, T=16, H=16, W=32,
                                       d=64, mode="topk_cdf", topk=5, cdf_p=0.2,
                                       cdf_cap_frac=0.25, t_cond=8),
    # a softmax scale other than 1/sqrt(d): sharper (CDF counts and the attention's
    # softmax both change) and flatter than the default
    "scale_sharp_cdf": W["tiny"].with_(name="scale_sharp_cdf", B=2, heads=2, T=16, H=16, W=32,
                                       d=128, mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25,
                                       t_cond=8, scale=0.3),
    "scale_flat_topk": W["tiny"].with_(name="scale_flat_topk", heads=2, T=8, H=16, W=32, d=64,
                                       topk=5, scale=0.02),
    # 64-token query and key chunks (4,4,4): the kernel's tile is a (4,4,8) box of two
    # query chunks over the union of their key boxes, masked per quadrant
    "q64_k64": W["tiny"].with_(name="q64_k64", heads=2, T=8, H=16, W=32, d=128, topk=6,
                               qchunk=(4, 4, 4), kchunk=(4, 4, 4)),
    "q64_k128": W["tiny"].with_(name="q64_k128", heads=2, T=8, H=16, W=32, d=64, topk=4,
                                qchunk=(4, 4, 4), kchunk=(4, 4, 8)),
    # W = 20: the last box holds one query chunk; block-causal CDF
    "q64_odd_w_causal_cdf": W["tiny"].with_(name="q64_odd_w_causal_cdf", B=2, heads=2, T=12,
                                            H=16, W=20, d=128, mode="cdf", cdf_p=0.9,
                                            cdf_cap_frac=0.25, t_cond=4, qchunk=(4, 4, 4),
                                            kchunk=(4, 4, 4)),
    # partial chunks in h and w (H = 13, W = 30: the last chunk column holds 2 tokens)
    "q64_partial_topk_cdf": W["tiny"].with_(name="q64_partial_topk_cdf", heads=2, T=10, H=13,
                                            W=30, d=64, mode="topk_cdf", topk=7, cdf_p=0.3,
                                            cdf_cap_frac=0.5, qchunk=(4, 4, 4),
                                            kchunk=(4, 4, 4)),
}


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()


def host_f32(t):
    return t.float().cpu().numpy()


def run_gpu(wl, q, k, v):
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    qd, kd, vd = dev(q), dev(k), dev(v)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    out = torch.empty_like(qd)
    lse = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
    status = bsa.bsa_read_status(pl.workspace)
    rp = pl.row_ptr.cpu().numpy()
    ci = pl.col_idx[: int(rp[-1])].cpu().numpy()
    return rp, ci, out, lse, status


def gather_rows(x_bhnd, wl, rows):
    """[B,Hh,N,d] (numpy) -> [len(rows), slots, d] in chunk-local order (slots: the
    query chunk's tokens, 128 or 64); NaN for the slots of a partial edge chunk past
    the grid."""
    flat = x_bhnd.reshape(wl.B * wl.heads, wl.N, -1)
    qc = tuple(getattr(wl, "qchunk", (4, 4, 8)))
    out = np.full((len(rows), qc[0] * qc[1] * qc[2], flat.shape[-1]), np.nan)
    for n, r in enumerate(rows):
        tok = oracle.chunk_tokens(wl.T, wl.H, wl.W, r % wl.Nc, qc)
        ok = tok >= 0
        out[n][ok] = flat[r // wl.Nc][tok[ok]]
    return out


def boxes_to_key_chunks(rp, ci, wl):
    """The GPU's CSR over (4,4,8) boxes -> the key chunks they came from (the boxes of
    one key chunk are listed consecutively)."""
    mt, mh, mw = wl.kchunk[0] // 4, wl.kchunk[1] // 4, wl.kchunk[2] // 8
    NH, NW = wl.NH, wl.NW
    NkH, NkW = -(-wl.H // wl.kchunk[1]), -(-wl.W // wl.kchunk[2])
    b = np.asarray(ci, dtype=np.int64)
    key = ((b // (NH * NW)) // mt * NkH + (b // NW) % NH // mh) * NkW + (b % NW) // mw
    rows = []
    for r in range(len(rp) - 1):
        kr = key[rp[r]:rp[r + 1]]
        keep = np.ones(len(kr), dtype=bool)
        keep[1:] = kr[1:] != kr[:-1]
        rows.append(kr[keep])
    krp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    return krp, (np.concatenate(rows) if rows else np.zeros(0)).astype(np.int32)


def check_case(wl, rows=None, qkv=None):
    q, k, v = synth.make_qkv(wl) if qkv is None else qkv
    scale = wl.softmax_scale
    rp, ci, out, lse, status = run_gpu(wl, q, k, v)
    assert status == bsa.BSA_OK, bsa.status_string(status)
    kchunk, qchunk = tuple(wl.kchunk), tuple(wl.qchunk)
    q64 = qchunk == (4, 4, 4)
    # selection: oracle decides in fp32 (the kernel's precision); ties judged in fp64
    o_rp, o_ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                                wl.cdf_cap_frac, wl.t_cond, fp32=True, kchunk=kchunk,
                                qchunk=qchunk)
    S64 = oracle.scores(oracle.pool(q, wl.T, wl.H, wl.W, chunk=qchunk),
                        oracle.pool(k, wl.T, wl.H, wl.W, chunk=kchunk), scale)
    # the plan's CSR lists key chunks, except with larger key chunks of 128-token query
    # chunks, where it lists the (4,4,8) boxes they cover
    direct = kchunk == (4, 4, 8) or q64
    g_rp, g_ci = (rp, ci) if direct else boxes_to_key_chunks(rp, ci, wl)
    n_checked, n_diff = compare_csr(g_rp, g_ci, o_rp, o_ci, S64, wl.Nc, wl.n_cond, wl.mode,
                                    wl.cdf_p, wl.cdf_cap_frac, topk=wl.topk, Nk=wl.Nk,
                                    n_cond_k=wl.n_cond_k)
    assert n_diff <= max(1, n_checked // 100), f"{n_diff} of {n_checked} rows differ (ties)"
    # attention on the GPU's own CSR
    if rows is None:
        rows = np.arange(wl.rows)
    o_out, o_lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows,
                                 **(dict(kchunk=kchunk, qchunk=qchunk) if q64 else {}))
    g_out = gather_rows(host_f32(out), wl, rows)
    mx, mean = compare_attention(g_out, o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    g_lse = gather_rows(lse.cpu().numpy()[..., None], wl, rows)[..., 0]
    np.testing.assert_allclose(g_lse, o_lse, rtol=0, atol=2e-3)
    return dict(rows_diff=n_diff, max_abs=mx, mean_abs=mean)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_cases_all_rows(name):
    check_case(SMALL[name])


def _f32_to_bf16_bits(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_long_rows_divergent_rescale():
    """Rows of 180 chunks where K grows with the chunk index, so every query
    row's running max jumps by more than 2^8 at its own chunk: the lazy O
    rescale is needed by some rows of a warp and not by others."""
    wl = W["tiny"].with_(name="long_rows", heads=2, T=16, H=32, W=56, d=128, topk=180)
    q, k, v = synth.make_qkv(wl)
    kf = synth.bf16_bits_to_f32(k).reshape(wl.B, wl.heads, wl.T // 4, 4, wl.H // 4, 4,
                                           wl.W // 8, 8, wl.d).copy()
    NH, NW = wl.H // 4, wl.W // 8
    for ct in range(wl.T // 4):
        for ch in range(NH):
            for cw in range(NW):
                c = (ct * NH + ch) * NW + cw
                kf[:, :, ct, :, ch, :, cw] *= 0.5 + 4.0 * c / wl.Nc
    k2 = _f32_to_bf16_bits(kf.reshape(k.shape))
    check_case(wl, rows=np.arange(0, wl.rows, 19), qkv=(q, k2, v))


def test_rows_longer_than_the_staged_chunk_list():
    """Rows of 420 chunks: the forward kernel stages the first 384 chunk indices
    of a row in shared memory and reads the rest from col_idx."""
    wl = W["720p"].with_(name="long_rows_420", heads=1, topk=420)
    check_case(wl, rows=np.arange(0, wl.rows, 97))


@pytest.mark.parametrize("case", ["cdf_noisy_only", "topk_part_condition"])
def test_kv_cached_step_equals_rows_of_the_full_computation(case):
    """q_begin: only query chunks from frame q_begin on are computed (the
    KV-cached video-continuation step). Their CSR rows and outputs must equal
    those rows of the full block-causal computation; skipped queries are not
    read (they hold NaN here) and their outputs are not written."""
    if case == "cdf_noisy_only":
        wl = SMALL["causal_cdf_small"].with_(q_begin=8)
    else:
        wl = SMALL["causal_topk"].with_(q_begin=4, topk=20)
    full = wl.with_(q_begin=0)
    q, k, v = synth.make_qkv(wl)
    HW = wl.H * wl.W
    q_nan = q.copy()
    q_nan[:, :, : wl.q_begin * HW] = 0x7FC0          # bf16 NaN in the skipped query frames
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    qd, kd, vd = dev(q_nan), dev(k), dev(v)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    out = torch.full_like(qd, 3.0)
    lse = torch.full((wl.B, wl.heads, wl.N), 5.0, dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    rp = pl.row_ptr.cpu().numpy()
    ci = pl.col_idx[: int(rp[-1])].cpu().numpy()
    assert len(rp) == wl.rows + 1
    scale = wl.softmax_scale
    o_rp, o_ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                                wl.cdf_cap_frac, wl.t_cond, fp32=True)
    # place the GPU's rows at their positions in the full plan (the oracle's rows elsewhere)
    # and judge the selection with the same tie rules as the full computation
    full_rows = np.array([(r // wl.Nq) * wl.Nc + wl.q_skip + r % wl.Nq for r in range(wl.rows)])
    merged = rows_of(o_rp, o_ci)
    for r, g in enumerate(rows_of(rp, ci)):
        merged[full_rows[r]] = g
    m_rp = np.concatenate([[0], np.cumsum([len(x) for x in merged])]).astype(np.int32)
    m_ci = np.concatenate(merged).astype(np.int32)
    S64 = oracle.scores(oracle.pool(q, wl.T, wl.H, wl.W), oracle.pool(k, wl.T, wl.H, wl.W), scale)
    n_checked, n_diff = compare_csr(m_rp, m_ci, o_rp, o_ci, S64, wl.Nc, wl.n_cond, wl.mode,
                                    wl.cdf_p, wl.cdf_cap_frac, rows=full_rows)
    assert n_diff <= max(1, wl.rows // 100), f"{n_diff} of {wl.rows} rows differ (ties)"
    o_out, o_lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, m_rp, m_ci, full_rows)
    g_out = gather_rows(host_f32(out), full, full_rows)
    mx, mean = compare_attention(g_out, o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    g_lse = gather_rows(lse.cpu().numpy()[..., None], full, full_rows)[..., 0]
    np.testing.assert_allclose(g_lse, o_lse, rtol=0, atol=2e-3)
    # skipped query frames: outputs untouched
    assert torch.all(out[:, :, : wl.q_begin * HW] == 3.0)
    assert torch.all(lse[:, :, : wl.q_begin * HW] == 5.0)


def test_rearrange_bit_exact_and_inverse():
    for wl in (SMALL["ragged60_d64"], SMALL["ragged135_d128"]):
        q, _, _ = synth.make_qkv(wl)
        p = bsa.params_for(wl)
        x = dev(q)
        blk = torch.empty_like(x)
        bsa.bsa_rearrange(p, x, blk)
        back = torch.empty_like(x)
        bsa.bsa_rearrange(p, blk, back, inverse=True)
        torch.cuda.synchronize()
        got = blk.view(torch.int16).cpu().numpy().view(np.uint16).reshape(
            wl.B, wl.heads, wl.Nc, 128, wl.d)
        np.testing.assert_array_equal(got, oracle.rearrange(q, wl.T, wl.H, wl.W))
        assert torch.equal(back.view(torch.int16), x.view(torch.int16))


def test_pool_and_scores_match_oracle():
    wl = SMALL["ragged135_d128"]
    q, k, _ = synth.make_qkv(wl)
    p = bsa.params_for(wl)
    qp = torch.empty((wl.B, wl.heads, wl.Nc, wl.d), dtype=torch.float32, device="cuda")
    kp = torch.empty_like(qp)
    bsa.bsa_pool(p, dev(q), qp)
    bsa.bsa_pool(p, dev(k), kp)
    S = torch.empty((wl.B, wl.heads, wl.Nc, wl.Nc), dtype=torch.float32, device="cuda")
    bsa.bsa_scores(p, qp, kp, S)
    torch.cuda.synchronize()
    np.testing.assert_allclose(qp.cpu().numpy(), oracle.pool(q, wl.T, wl.H, wl.W), rtol=0,
                               atol=1e-6)
    scale = 1 / math.sqrt(wl.d)
    S_or = oracle.scores(qp.cpu().numpy().astype(np.float64),
                         kp.cpu().numpy().astype(np.float64), scale)
    err = np.abs(S.cpu().numpy() - S_or)
    assert err.max() <= 1e-5 * np.abs(S_or).max()


def test_all_chunks_equals_dense_oracle():
    wl = W["tiny"].with_(T=8, H=16, W=32, d=64, heads=2)  # 32 chunks
    wl = wl.with_(topk=wl.Nc)
    q, k, v = synth.make_qkv(wl)
    rp, ci, out, lse, status = run_gpu(wl, q, k, v)
    assert status == bsa.BSA_OK
    assert np.all(np.diff(rp) == wl.Nc)
    ids = np.arange(0, wl.B * wl.heads * wl.N, 7)
    ref, ref_lse = oracle.dense(q, k, v, wl.T, wl.H, wl.W, 1 / math.sqrt(wl.d), ids)
    got = host_f32(out).reshape(-1, wl.d)[ids]
    assert np.abs(got - ref).max() <= ATT_MAX_ABS and np.abs(got - ref).mean() <= ATT_MEAN_ABS
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1)[ids], ref_lse, atol=2e-3, rtol=0)


def test_caller_csr_empty_and_out_of_range_rows():
    wl = W["tiny"]  # 8 rows of 4 chunks
    q, k, v = synth.make_qkv(wl)
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    # rows: [0,3] [] [1] [2,3] [3,7] [] [0,1] [2]; chunk 7 does not exist (Nc = 4)
    rp = np.array([0, 2, 2, 3, 5, 7, 7, 9, 10], dtype=np.int32)
    ci = np.array([0, 3, 1, 2, 3, 3, 7, 0, 1, 2], dtype=np.int32)
    qd, kd, vd = dev(q), dev(k), dev(v)
    out = torch.full_like(qd, 7.0)
    lse = torch.zeros((1, 2, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                    pl.workspace, out, lse)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_ERR_DEVICE_BAD_INDEX
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK  # cleared by the read
    g = host_f32(out)
    g_lse = lse.cpu().numpy()[..., None]
    # the out-of-range chunk is skipped: row 4 attends to chunk 3 only
    rp_o = np.array([0, 2, 2, 3, 5, 6, 6, 8, 9], dtype=np.int32)
    ci_o = np.array([0, 3, 1, 2, 3, 3, 0, 1, 2], dtype=np.int32)
    good = [0, 2, 3, 4, 6, 7]
    o_out, o_lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, 1 / math.sqrt(wl.d), rp_o, ci_o, good)
    mx, mean = compare_attention(gather_rows(g, wl, good), o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS
    np.testing.assert_allclose(gather_rows(g_lse, wl, good)[..., 0], o_lse, rtol=0, atol=2e-3)
    for r in (1, 5):  # empty rows: zeros and lse = -inf
        assert np.all(gather_rows(g, wl, [r]) == 0)
        assert np.all(np.isneginf(gather_rows(g_lse, wl, [r])))


def test_row_ptr_out_of_range_is_rejected_not_read():
    wl = W["tiny"]
    q, k, v = synth.make_qkv(wl)
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    rp = torch.tensor([0, 2, 4, 6, 8, 1 << 30, 12, 14, 16], dtype=torch.int32, device="cuda")
    ci = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = torch.empty_like(dev(q))
    bsa.bsa_forward(p, dev(q), dev(k), dev(v), rp, ci, pl.workspace, out)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_ERR_DEVICE_BAD_INDEX


def test_deterministic():
    wl = SMALL["causal_cdf_small"]
    q, k, v = synth.make_qkv(wl)
    a = run_gpu(wl, q, k, v)
    b = run_gpu(wl, q, k, v)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert torch.equal(a[2].view(torch.int16), b[2].view(torch.int16))


def test_bounded_wait_selftest_reports_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    bsa.bsa_selftest_timeout(ws, 20_000_000)  # 20 ms
    assert bsa.bsa_read_status(ws) == bsa.BSA_ERR_DEVICE_TIMEOUT
    check_case(SMALL["tiny"])  # the context is still usable


def status_words(ws):
    """The first 16 uint32 words of a workspace's status block."""
    return ws[:64].cpu().numpy().view(np.uint32).copy()


def check_timeout_record(ws):
    """The record of the first expired wait, then its clearing by bsa_read_status."""
    w = status_words(ws)
    assert w[1] >= 1 and w[2] == 1, w[:6]          # expired waits; a site was recorded
    assert w[3] // 1_000_000 in (1, 2, 3), w[3]     # role: producer, MMA issuer or warps
    assert bsa.bsa_read_status(ws) == bsa.BSA_ERR_DEVICE_TIMEOUT
    assert not status_words(ws)[:6].any()
    return w


def test_forward_kernel_abort_path_reports_timeout():
    """The forward kernel's own bounded waits: with debug bit 0 the MMA warp
    withholds the first S-ready signal of tile 0, so that tile's softmax warps
    (and then every role) wait until the 20 ms limit, record the timeout, drain
    their copies and products, free TMEM and return; with bit 1 every CTA
    counts itself on the way out. The status must say DEVICE_TIMEOUT, every CTA
    must have returned, and the next calls must work."""
    wl = SMALL["tiny"]
    q, k, v = synth.make_qkv(wl)
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    qd, kd, vd = dev(q), dev(k), dev(v)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    out = torch.zeros_like(qd)
    bsa.bsa_forward_ex(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out,
                       timeout_ns=20_000_000, debug_flags=3)
    w = check_timeout_record(pl.workspace)
    ctas = (wl.rows + 1) // 2                       # two query chunks per CTA
    assert w[8] == ctas and w[4] < ctas, (w[8], w[4])
    # the same buffers give the right result on the next call, and so does a fresh case
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    rp = pl.row_ptr.cpu().numpy()
    ci = pl.col_idx[: int(rp[-1])].cpu().numpy()
    rows = np.arange(wl.rows)
    o_out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, wl.softmax_scale, rp, ci, rows)
    mx, mean = compare_attention(gather_rows(host_f32(out), wl, rows), o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    check_case(SMALL["causal_cdf_small"])


# ------------------------------------------------------------------ full-size workloads

def _sample_rows(wl, per_head, seed=0):
    rng = np.random.default_rng(seed)
    rows = []
    for bh in range(wl.B * wl.heads):
        rows.extend(bh * wl.Nc + rng.choice(wl.Nc, size=min(per_head, wl.Nc), replace=False))
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name,per_head", [("480p", 224), ("720p", 64), ("long", 16),
                                           ("causal_cdf", 16), ("720p_r8", 4),
                                           ("720p_topk_cdf", 4), ("720p_real", 4),
                                           ("480p_real", 4), ("720p_k512", 4),
                                           ("720p_q64", 16)])
def test_full_size_workloads(name, per_head):
    wl = W[name]
    check_case(wl, rows=_sample_rows(wl, per_head))


def test_64_token_chunks_caller_csr_with_an_empty_half():
    """A caller CSR where one of the two query chunks of a box selects nothing: its
    rows are zeros with LSE -inf while its neighbour's rows are exact."""
    wl = SMALL["q64_k64"].with_(heads=1)
    q, k, v = synth.make_qkv(wl)
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    nc = wl.Nc                                  # 2 x 4 x 8 = 64 query chunks
    rows = [[] if i % 3 == 1 else sorted({(i * 7) % nc, (i * 5 + 3) % nc, i}) for i in range(nc)]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate([np.array(r, dtype=np.int32) for r in rows]).astype(np.int32)
    qd, kd, vd = dev(q), dev(k), dev(v)
    out = torch.full_like(qd, 7.0)
    lse = torch.zeros((1, 1, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                    pl.workspace, out, lse)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    full = [i for i in range(nc) if rows[i]]
    o_out, o_lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, wl.softmax_scale, rp, ci, full,
                                 kchunk=(4, 4, 4), qchunk=(4, 4, 4))
    mx, mean = compare_attention(gather_rows(host_f32(out), wl, full), o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    g_lse = gather_rows(lse.cpu().numpy()[..., None], wl, full)[..., 0]
    np.testing.assert_allclose(g_lse, o_lse, rtol=0, atol=2e-3)
    empty = [i for i in range(nc) if not rows[i]]
    assert np.all(gather_rows(host_f32(out), wl, empty) == 0)
    assert np.all(np.isneginf(gather_rows(lse.cpu().numpy()[..., None], wl, empty)))
    # the union of a box's rows does not depend on the order of their entries:
    # a shuffled row and a repeated entry give the same output bit for bit
    ci_shuf = ci.copy()
    ci_shuf[0], ci_shuf[1] = ci[1], ci[0]
    ci_shuf[rp[2]] = ci_shuf[rp[2] + 1]
    out2 = torch.full_like(qd, 7.0)
    bsa.bsa_forward(p, qd, kd, vd, torch.from_numpy(rp).cuda(), torch.from_numpy(ci_shuf).cuda(),
                    pl.workspace, out2)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    ref_rows = [r for r in range(nc) if set(rows[r]) == set(ci_shuf[rp[r]:rp[r + 1]])]
    assert 0 in ref_rows
    g1, g2 = gather_rows(host_f32(out), wl, ref_rows), gather_rows(host_f32(out2), wl, ref_rows)
    assert np.array_equal(np.nan_to_num(g1), np.nan_to_num(g2))


@pytest.mark.parametrize("name", ["causal_cdf_small", "q64_k64", "scale_sharp_cdf"])
def test_one_call_api_equals_plan_and_forward(name):
    """block_sparse_attention (plan + forward in one call) gives the explicit
    calls' output bit for bit."""
    wl = SMALL[name]
    q, k, v = synth.make_qkv(wl)
    rp, ci, out, lse, status = run_gpu(wl, q, k, v)
    assert status == bsa.BSA_OK
    o1, l1 = bsa.block_sparse_attention(dev(q), dev(k), dev(v), topk=wl.topk or None,
                                        mode=wl.mode, cdf_p=wl.cdf_p,
                                        cdf_cap_frac=wl.cdf_cap_frac, t_cond=wl.t_cond,
                                        grid=(wl.T, wl.H, wl.W), want_lse=True,
                                        chunk=tuple(wl.qchunk), kchunk=tuple(wl.kchunk),
                                        scale=wl.scale)
    assert torch.equal(o1.view(torch.int16), out.view(torch.int16))
    assert torch.equal(l1, lse)


def test_grid_of_1920_chunks():
    """A grid near the library's limit of 2,048 chunks per (batch, head):
    64 x 48 x 80 latent tokens, 1,920 chunks, k = 120 (93.75 % sparse). Its
    rows take the selector's widest instantiation (64 keys per lane)."""
    wl = W["720p"].with_(name="grid1920", heads=1, T=64, topk=120)
    assert 1792 < wl.Nc <= 2048
    check_case(wl, rows=_sample_rows(wl, 32))
