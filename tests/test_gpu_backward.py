"""GPU parity of the backward (dQ, dK, dV) against the fp64 oracle, through
the C ABI. The oracle runs on the GPU's own CSR with its own exact forward
(P, O, D in fp64); the GPU recomputes P from its bf16-path LSE and takes D
from its bf16 output, so the bars below absorb bf16 rounding of P, dS and the
outputs (relative to the gradients' own scale)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import ATT_MAX_ABS, ATT_MEAN_ABS, compare_attention, rows_of
from test_gpu_parity import SMALL, W, check_timeout_record, dev, gather_rows, host_f32

pytestmark = pytest.mark.gpu

import block_sparse_attention_13_b200 as bsa  # noqa: E402

# bars: max |gpu - ref| / max |ref| and mean |gpu - ref| / mean |ref|, per tensor.
# Rounding the gradients to bf16 alone costs up to 2^-9 (0.2 %) of an element;
# P and dS enter the products as bf16 (2^-9 each) and D comes from the bf16
# output. dQ = scale * sum_j dS_j K_j cancels (sum_j dS_j = 0) while the
# rounding of dS adds up over the row's keys, so its relative error grows with
# the row length. Measured: small grids at most 0.5 % max / 0.3 % mean; the
# 720p grid (5,760 keys per row) 1.04 % / 0.48 % for dQ. Bars: twice that.
BWD_MAX_REL = 2e-2
BWD_MEAN_REL = 1e-2


def rel_errors(g, o):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    live = ~np.isnan(o)            # slots of partial edge chunks past the grid: NaN
    g, o = g[live], o[live]
    err = np.abs(g - o)
    return float(err.max() / max(np.abs(o).max(), 1e-30)), \
        float(err.mean() / max(np.abs(o).mean(), 1e-30))


def gpu_fwd_bwd(wl, q, k, v, g, csr=None, sentinel=None):
    """Plan (or the caller's CSR), forward with LSE, backward. Returns host
    CSR, device out/lse/dq/dk/dv and the two status codes."""
    p = bsa.params_for(wl)
    qd, kd, vd, gd = dev(q), dev(k), dev(v), dev(g)
    if csr is None:
        pl = bsa.allocate(p)
        bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    else:
        pl = bsa.allocate(p)
        rp, ci = csr
        pl.row_ptr.copy_(torch.from_numpy(np.asarray(rp, dtype=np.int32)))
        pl.col_idx = torch.from_numpy(np.asarray(ci, dtype=np.int32).copy()).cuda() \
            if len(ci) else torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(qd)
    lse = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
    st_f = bsa.bsa_read_status(pl.workspace)
    ws = bsa.backward_workspace(p)
    fill = float("nan") if sentinel is None else sentinel
    dq, dk, dv = (torch.full_like(qd, fill) for _ in range(3))
    bsa.bsa_backward(p, qd, kd, vd, out, lse, gd, pl.row_ptr, pl.col_idx, ws, dq, dk, dv)
    st_b = bsa.bsa_read_status(ws)
    rp = pl.row_ptr.cpu().numpy()
    ci = pl.col_idx[: int(rp[-1])].cpu().numpy()
    return rp, ci, out, lse, dq, dk, dv, st_f, st_b


def check_bwd(wl, csr=None):
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    scale = wl.softmax_scale
    rp, ci, out, lse, dq, dk, dv, st_f, st_b = gpu_fwd_bwd(wl, q, k, v, g, csr)
    assert st_f == bsa.BSA_OK and st_b == bsa.BSA_OK, (st_f, st_b)
    rows = np.arange(wl.rows)
    # 64-token query chunks: the plan's CSR is over the chunks themselves (the library
    # builds the box CSR inside the forward and backward); otherwise it is over boxes
    shapes = dict(kchunk=tuple(wl.kchunk), qchunk=tuple(wl.qchunk)) \
        if tuple(wl.qchunk) == (4, 4, 4) else {}
    o_dq, o_dk, o_dv = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, rp, ci, rows,
                                         **shapes)
    errs = {
        "dq": rel_errors(gather_rows(host_f32(dq), wl, rows), o_dq),
        "dk": rel_errors(host_f32(dk), o_dk),
        "dv": rel_errors(host_f32(dv), o_dv),
    }
    for name, (mx, mean) in errs.items():
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (name, errs)
    return errs


@pytest.mark.parametrize("name", sorted(SMALL))
def test_backward_small_cases(name):
    check_bwd(SMALL[name])


@pytest.mark.parametrize("name,flags", [("tiny", 1), ("tiny", 2), ("q64_k64", 3)])
def test_backward_kernel_abort_paths_report_timeout(name, flags):
    """The backward kernels' own bounded waits: debug bit 0 makes the dQ
    kernel's MMA thread, bit 1 the dK/dV kernel's, withhold its first
    S-ready signal, so that kernel's exponential warps (and then every role)
    wait until the 20 ms limit, record the timeout, and the CTA waits for its
    copies and products in flight before freeing TMEM and returning. The status
    must say DEVICE_TIMEOUT, and the next call on the same buffers must give
    the right gradients."""
    wl = SMALL[name]
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    p = bsa.params_for(wl)
    qd, kd, vd, gd = dev(q), dev(k), dev(v), dev(g)
    pl = bsa.allocate(p)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    out = torch.empty_like(qd)
    lse = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    ws = bsa.backward_workspace(p)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    args = (p, qd, kd, vd, out, lse, gd, pl.row_ptr, pl.col_idx, ws, dq, dk, dv)
    bsa.bsa_backward_ex(*args, timeout_ns=20_000_000, debug_flags=flags)
    check_timeout_record(ws)
    bsa.bsa_backward(*args)
    assert bsa.bsa_read_status(ws) == bsa.BSA_OK
    rp = pl.row_ptr.cpu().numpy()
    ci = pl.col_idx[: int(rp[-1])].cpu().numpy()
    rows = np.arange(wl.rows)
    shapes = dict(kchunk=tuple(wl.kchunk), qchunk=tuple(wl.qchunk)) \
        if tuple(wl.qchunk) == (4, 4, 4) else {}
    refs = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, wl.softmax_scale, rp, ci, rows,
                             **shapes)
    gots = (gather_rows(host_f32(dq), wl, rows), host_f32(dk), host_f32(dv))
    for nm, got, ref in zip(("dq", "dk", "dv"), gots, refs):
        mx, mean = rel_errors(got, ref)
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (nm, mx, mean)


def test_64_token_chunks_with_masked_quadrants_of_huge_logits():
    """64-token chunks whose box partner selected a key chunk they did not: the
    kernels compute those quadrants of the (4,4,8) box tile and must keep them
    out of every result. Key chunk 11 of head 0 has K scaled by 64 (exact in
    bf16), so its logits reach about +-200 and exp() of them overflows fp32: a
    masked logit that entered the row max would underflow the row's kept
    weights to 0, and one that reached an exponential before the mask would
    give inf * 0 = NaN. Query chunk 20 keeps 10 (the other half of 11's box)
    while 21 keeps 11; 36 keeps neither while 37 keeps 11; 45 and 44 keep 11
    together with the rest of their own selection. Forward O and LSE must match
    the oracle on every row and every gradient must be finite. The gradient
    bars: the usual ones wherever the hot chunk is not attended (every masked
    quadrant is there); where it is, only the max bar against the tensor's own
    largest gradient. Those rows put nearly all their weight on the hot keys,
    so their exact dS, and hence dQ and the hot keys' dK, cancel to near zero,
    while D = sum(dO * O) comes from the bf16 output: its 2^-9 rounding, times
    K scaled by 64, is then most of what is left."""
    wl = SMALL["q64_k64"]
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    hot, partner = 11, 10                                 # key chunks sharing one (4,4,8) box
    toks = oracle.chunk_tokens(wl.T, wl.H, wl.W, hot, (4, 4, 4))
    kf = (k[0, 0, toks].astype(np.uint32) << 16).view(np.float32) * np.float32(64.0)
    k = k.copy()
    k[0, 0, toks] = (kf.view(np.uint32) >> 16).astype(np.uint16)  # exact: a power of two
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, wl.softmax_scale, wl.mode, wl.topk,
                            kchunk=tuple(wl.kchunk), qchunk=tuple(wl.qchunk))
    lists = [set(ci[rp[r]:rp[r + 1]]) for r in range(wl.rows)]
    for r, add, drop in ((20, {partner}, {hot}), (21, {hot}, set()), (36, set(), {hot, partner}),
                         (37, {hot}, set()), (44, {hot}, set()), (45, {hot}, set())):
        lists[r] = (lists[r] - drop) | add
    rp2 = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int32)
    ci2 = np.array([c for x in lists for c in sorted(x)], dtype=np.int32)
    rows = np.arange(wl.rows)
    shapes = dict(kchunk=tuple(wl.kchunk), qchunk=tuple(wl.qchunk))
    _, _, out, lse, dq, dk, dv, st_f, st_b = gpu_fwd_bwd(wl, q, k, v, g, csr=(rp2, ci2))
    assert st_f == bsa.BSA_OK and st_b == bsa.BSA_OK, (st_f, st_b)
    o_out, o_lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, wl.softmax_scale, rp2, ci2, rows,
                                 **shapes)
    mx, mean = compare_attention(gather_rows(host_f32(out), wl, rows), o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    g_lse = gather_rows(lse.cpu().numpy()[..., None], wl, rows)[..., 0]
    # LSE: the forward's bar, plus fp32 accumulation of logits that are 64 times larger
    np.testing.assert_array_less(np.abs(g_lse - o_lse), 2e-3 + 2e-5 * np.abs(o_lse))
    assert np.abs(o_lse).max() > 50                       # the hot chunk's logits are in play
    refs = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, wl.softmax_scale, rp2, ci2, rows,
                             **shapes)
    gots = (gather_rows(host_f32(dq), wl, rows), host_f32(dk), host_f32(dv))
    hot_rows = np.array([r < wl.Nc and hot in lists[r] for r in range(wl.rows)])  # head 0
    hot_keys = np.zeros((wl.B, wl.heads, wl.N), dtype=bool)
    hot_keys[0, 0, toks] = True
    for nm, got, ref, sel in zip(("dq", "dk", "dv"), gots, refs, (hot_rows, hot_keys, hot_keys)):
        assert np.isfinite(got[~np.isnan(ref)]).all(), nm
        mx, mean = rel_errors(got[~sel], ref[~sel])
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (nm, "elsewhere", mx, mean)
        err = np.abs(got[sel] - ref[sel])
        assert np.nanmax(err) <= BWD_MAX_REL * np.nanmax(np.abs(ref)), (nm, "hot")


def test_backward_64_token_chunks_with_an_empty_chunk_and_unselected_halves():
    """64-token query chunks with a caller CSR: one query chunk selects nothing
    (its queries have no output: dQ exactly 0) and some 64-token key chunks no
    query chunk selects (dK, dV exactly 0), beside chunks whose box partner
    selected different keys."""
    wl = SMALL["q64_k64"]
    q, k, v = synth.make_qkv(wl)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, wl.softmax_scale, wl.mode, wl.topk,
                            kchunk=tuple(wl.kchunk), qchunk=tuple(wl.qchunk))
    lists = [list(ci[rp[r]:rp[r + 1]]) for r in range(wl.rows)]
    lists[3] = []                                        # head 0, chunk 3: no keys
    unused = {5, 6}                                      # key chunks 5, 6 of head 0: never kept
    lists = [[c for c in row if not (r < wl.Nc and c in unused)] for r, row in enumerate(lists)]
    rp2 = np.concatenate([[0], np.cumsum([len(r) for r in lists])]).astype(np.int32)
    ci2 = np.array([c for row in lists for c in row], dtype=np.int32)
    check_bwd(wl, csr=(rp2, ci2))
    g = synth.make_dout(wl)
    _, _, _, _, dq, dk, dv, _, _ = gpu_fwd_bwd(wl, q, k, v, g, csr=(rp2, ci2))
    dqh = gather_rows(host_f32(dq), wl, np.array([3]))
    assert np.all(dqh == 0)
    for c in unused:
        toks = oracle.chunk_tokens(wl.T, wl.H, wl.W, c, tuple(wl.kchunk))
        toks = toks[toks >= 0]
        assert np.all(host_f32(dk)[0, 0][toks] == 0) and np.all(host_f32(dv)[0, 0][toks] == 0)


def test_backward_all_chunks_selected():
    wl = W["tiny"].with_(T=8, H=16, W=32, d=128, heads=2)
    check_bwd(wl.with_(topk=wl.Nc))


def test_backward_empty_rows_and_unselected_key_chunks():
    """Caller CSR with empty rows and key chunks that no row selects: the dQ of
    an empty row and the dK/dV of an unselected chunk are exact zeros."""
    wl = W["tiny"].with_(T=8, H=16, W=32, d=64, heads=2)   # 32 chunks per head
    rng = np.random.default_rng(3)
    rows = []
    for r in range(wl.rows):
        if r % 7 == 3:
            rows.append([])
        else:
            rows.append(sorted(rng.choice(np.arange(0, wl.Nc, 2), size=int(rng.integers(1, 6)),
                                          replace=False)))   # odd chunks never selected
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    ci = np.concatenate([np.asarray(x, dtype=np.int32) for x in rows])
    check_bwd(wl, csr=(rp, ci))
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    _, _, _, _, dq, dk, dv, _, st_b = gpu_fwd_bwd(wl, q, k, v, g, csr=(rp, ci))
    assert st_b == bsa.BSA_OK
    for r in range(wl.rows):
        if not rows[r]:
            toks = oracle.chunk_tokens(wl.T, wl.H, wl.W, r % wl.Nc)
            assert torch.all(dq.view(-1, wl.N, wl.d)[r // wl.Nc, toks] == 0)
    for c in range(1, wl.Nc, 2):
        toks = oracle.chunk_tokens(wl.T, wl.H, wl.W, c)
        assert torch.all(dk.view(-1, wl.N, wl.d)[:, toks] == 0)
        assert torch.all(dv.view(-1, wl.N, wl.d)[:, toks] == 0)


def test_backward_duplicate_chunk_in_row_is_reported():
    wl = W["tiny"].with_(T=8, H=16, W=32, d=64, heads=1)
    rows = [[c, (c + 1) % wl.Nc] for c in range(wl.Nc)]
    rows[5] = [2, 2, 9]                                        # duplicate entry
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    ci = np.concatenate([np.asarray(x, dtype=np.int32) for x in rows])
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    *_, st_b = gpu_fwd_bwd(wl, q, k, v, g, csr=(rp, ci))
    assert st_b == bsa.BSA_ERR_DEVICE_BAD_INDEX


def test_backward_kv_cached_rows():
    """q_begin: the backward of the computed rows only. dQ of skipped query
    frames is not written; dK/dV hold the contributions of the computed rows."""
    wl = SMALL["causal_cdf_small"].with_(q_begin=8)
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    scale = 1.0 / math.sqrt(wl.d)
    rp, ci, out, lse, dq, dk, dv, st_f, st_b = gpu_fwd_bwd(wl, q, k, v, g, sentinel=7.0)
    assert st_f == bsa.BSA_OK and st_b == bsa.BSA_OK
    full = wl.with_(q_begin=0)
    full_rows = np.array([(r // wl.Nq) * wl.Nc + wl.q_skip + r % wl.Nq for r in range(wl.rows)])
    merged = [np.zeros(0, dtype=np.int32)] * (wl.B * wl.heads * wl.Nc)
    for r, x in enumerate(rows_of(rp, ci)):
        merged[full_rows[r]] = x
    m_rp = np.concatenate([[0], np.cumsum([len(x) for x in merged])]).astype(np.int32)
    m_ci = np.concatenate(merged).astype(np.int32)
    o_dq, o_dk, o_dv = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, m_rp, m_ci,
                                         full_rows)
    for name, (gx, ox) in {"dq": (gather_rows(host_f32(dq), full, full_rows), o_dq),
                           "dk": (host_f32(dk), o_dk), "dv": (host_f32(dv), o_dv)}.items():
        mx, mean = rel_errors(gx, ox)
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (name, mx, mean)
    HW = wl.H * wl.W
    assert torch.all(dq[:, :, : wl.q_begin * HW] == 7.0)


@pytest.mark.parametrize("name", ["ragged135_d128", "q64_k128"])
def test_autograd_op_matches_the_c_abi_calls(name):
    """block_sparse_attention_train (torch.autograd) runs the same plan, forward and
    backward as the direct C-ABI calls: outputs and gradients bit for bit (also with
    64-token query chunks)."""
    from block_sparse_attention_13_b200.autograd import block_sparse_attention_train
    wl = SMALL[name]
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    rp, ci, out, lse, dq, dk, dv, st_f, st_b = gpu_fwd_bwd(wl, q, k, v, g)
    assert st_f == bsa.BSA_OK and st_b == bsa.BSA_OK
    qt, kt, vt = (dev(x).requires_grad_(True) for x in (q, k, v))
    o = block_sparse_attention_train(qt, kt, vt, (wl.T, wl.H, wl.W), topk=wl.topk, mode=wl.mode,
                                     cdf_p=wl.cdf_p, cdf_cap_frac=wl.cdf_cap_frac,
                                     t_cond=wl.t_cond, chunk=tuple(wl.qchunk),
                                     kchunk=tuple(wl.kchunk))
    o.backward(dev(g))
    for a, b in ((o.detach(), out), (qt.grad, dq), (kt.grad, dk), (vt.grad, dv)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_backward_deterministic():
    wl = SMALL["ragged135_d128"]
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    a = gpu_fwd_bwd(wl, q, k, v, g)
    b = gpu_fwd_bwd(wl, q, k, v, g)
    for x, y in zip(a[4:7], b[4:7]):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


@pytest.mark.parametrize("name", ["720p", "720p_real", "720p_q64"])
def test_backward_full_size_720p_sampled(name):
    """Full 720p grids, 32 heads, in the launch configuration of the benchmark
    (720p_real has partial edge chunks, 720p_q64 64-token query and key chunks):
    dQ of sampled rows and dK/dV of a sampled key chunk of (batch 0, head 0)
    against the oracle, plus the invariants sum(dK) = 0 and sum(dV) = sum(dO)
    per head (every row is non-empty under top-k)."""
    wl = W[name]
    q64 = tuple(wl.qchunk) == (4, 4, 4)
    shapes = dict(kchunk=tuple(wl.kchunk), qchunk=tuple(wl.qchunk)) if q64 else {}
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    scale = 1.0 / math.sqrt(wl.d)
    rp, ci, out, lse, dq, dk, dv, st_f, st_b = gpu_fwd_bwd(wl, q, k, v, g)
    assert st_f == bsa.BSA_OK and st_b == bsa.BSA_OK
    # invariants on every head, from the GPU's bf16 gradients
    dkf = dk.float().view(wl.heads, wl.N, wl.d)
    dvf = dv.float().view(wl.heads, wl.N, wl.d)
    gf = torch.from_numpy(synth.bf16_bits_to_f32(g)).cuda().view(wl.heads, wl.N, wl.d)
    sk = dkf.sum(1).abs().max() / dkf.abs().sum(1).max()
    sv = (dvf.sum(1) - gf.sum(1)).abs().max() / gf.abs().sum(1).max()
    assert sk < 1e-3 and sv < 1e-3, (float(sk), float(sv))
    # oracle on (batch 0, head 0)
    q0, k0, v0, g0 = (x[:, :1] for x in (q, k, v, g))
    rp0 = rp[: wl.Nc + 1]
    ci0 = ci[: int(rp0[-1])]
    rng = np.random.default_rng(11)
    sample_rows = np.sort(rng.choice(wl.Nc, size=3, replace=False))
    col = int(ci0[int(rng.integers(0, len(ci0)))])
    col_rows = np.array([r for r in range(wl.Nc) if col in ci0[rp0[r]:rp0[r + 1]]])
    rows = np.unique(np.concatenate([sample_rows, col_rows]))
    w1 = wl.with_(heads=1)
    o_dq, o_dk, o_dv = oracle.attend_bwd(q0, k0, v0, g0, wl.T, wl.H, wl.W, scale, rp0, ci0, rows,
                                         **shapes)
    sel = np.isin(rows, sample_rows)
    mx, mean = rel_errors(gather_rows(host_f32(dq[:, :1]), w1, sample_rows), o_dq[sel])
    assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, ("dq", mx, mean)
    toks = oracle.chunk_tokens(wl.T, wl.H, wl.W, col, *([tuple(wl.kchunk)] if q64 else []))
    toks = toks[toks >= 0]
    for name, gx, ox in (("dk", dk, o_dk), ("dv", dv, o_dv)):
        mx, mean = rel_errors(host_f32(gx[0, 0, toks]), ox[0, 0, toks])
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (name, col, mx, mean)
