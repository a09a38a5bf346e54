"""GPU checks of the context-parallel (ring) path on one device: the ranks of a
group of 2 or 4 are run one after the other through the same driver, with a
communicator that hands each rank what the real all-gather and ring shifts
would deliver. Every device step runs through the C ABI; the result of each
rank must equal the rows of the unsplit computation (selection exactly, the
attention within the rounding of the bf16 partial results) and the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import ATT_MAX_ABS, ATT_MEAN_ABS, compare_attention
from test_gpu_parity import dev, gather_rows, host_f32

pytestmark = pytest.mark.gpu

import block_sparse_attention_13_b200 as bsa  # noqa: E402
from block_sparse_attention_13_b200.context_parallel import (CudaOps, ring_backward,  # noqa: E402
                                                            ring_backward_partials, ring_forward)
from test_gpu_backward import BWD_MAX_REL, BWD_MEAN_REL, rel_errors  # noqa: E402


class SimComm:
    """What rank `rank` of a `world`-rank group receives: the stacked pooled keys
    of all shards, and at ring step s the K/V shard of rank (rank - s - 1)."""

    def __init__(self, rank, world, kp_all, k_shards, v_shards):
        self.rank, self.world = rank, world
        self.kp_all, self.k, self.v = kp_all, k_shards, v_shards
        self.step = 0

    def all_gather(self, x):
        assert torch.equal(x, self.kp_all[self.rank])
        return self.kp_all

    def start_shift(self, tensors):
        self.step += 1
        return (self.rank - self.step) % self.world

    def finish_shift(self, j):
        return [self.k[j], self.v[j]]

    def reduce_scatter(self, x):
        # only a one-rank group can be answered without the other ranks' buffers
        assert self.world == 1
        return x[0].clone()


def shard(x, world, frames, HW):
    return [x[:, :, r * frames * HW:(r + 1) * frames * HW].contiguous() for r in range(world)]


CASES = {
    "w2_topk": (synth.WORKLOADS["tiny"].with_(heads=2, T=16, H=16, W=32, d=128, topk=6), 2),
    "w4_topk": (synth.WORKLOADS["tiny"].with_(heads=2, T=16, H=16, W=32, d=64, topk=9), 4),
    "w2_causal_cdf": (synth.WORKLOADS["tiny"].with_(B=2, heads=2, T=16, H=16, W=32, d=128,
                                                    mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25,
                                                    t_cond=8), 2),
    "w2_partial": (synth.WORKLOADS["tiny"].with_(heads=2, T=8, H=13, W=37, d=128, topk=5), 2),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_ring_forward_equals_unsplit(name):
    wl, world = CASES[name]
    q, k, v = synth.make_qkv(wl)
    HW = wl.H * wl.W
    T_l = wl.T // world
    qd, kd, vd = dev(q), dev(k), dev(v)
    # the unsplit computation
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    out_g = torch.empty_like(qd)
    lse_g = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out_g, lse_g)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    g_rp = pl.row_ptr.cpu().numpy()
    g_ci = pl.col_idx[: int(g_rp[-1])].cpu().numpy()
    # per-rank shards and the pooled keys the all-gather would deliver
    qs, ks, vs = (shard(x, world, T_l, HW) for x in (qd, kd, vd))
    ops = CudaOps()
    p_local = bsa.make_params(wl.B, wl.heads, T_l, wl.H, wl.W, wl.d, wl.mode, wl.topk)
    kp_all = torch.stack([ops.pool(p_local, ks[r]) for r in range(world)])
    nc_l = wl.Nc // world
    scale = 1.0 / math.sqrt(wl.d)
    for r in range(world):
        comm = SimComm(r, world, kp_all, ks, vs)
        probe = CudaOps()
        out, lse = ring_forward(qs[r], ks[r], vs[r], (T_l, wl.H, wl.W), wl.topk, wl.mode,
                                wl.cdf_p, wl.cdf_cap_frac, wl.t_cond, comm=comm, ops=probe)
        # selection: this rank's rows of the unsplit plan, exactly
        p_rank = bsa.make_params(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, wl.mode, wl.topk,
                                 wl.cdf_p, wl.cdf_cap_frac, wl.t_cond, q_begin=r * T_l,
                                 q_end=(r + 1) * T_l)
        rp, ci = CudaOps().select_pooled(p_rank, ops.pool(p_local, qs[r]), kp_all, nc_l)
        rp, ci = rp.cpu().numpy(), ci.cpu().numpy()
        for bh in range(wl.B * wl.heads):
            for i in range(nc_l):
                row = bh * nc_l + i
                grow = bh * wl.Nc + r * nc_l + i
                assert np.array_equal(ci[rp[row]:rp[row + 1]], g_ci[g_rp[grow]:g_rp[grow + 1]])
        # attention: the unsplit result for these frames. The partial outputs stay in
        # fp32 through the merges and are rounded to bf16 once, as the unsplit call's
        # output is. What differs is the bf16 rounding of the softmax numerators P,
        # taken against each shard's own running max instead of the whole row's, so
        # the ring must be as accurate as the unsplit call against the fp64 oracle
        # (below); here, close to it element by element
        sl = slice(r * T_l * HW, (r + 1) * T_l * HW)
        diff = (out.float() - out_g[:, :, sl].float()).abs()
        assert float(diff.max()) <= ATT_MAX_ABS / 2 and float(diff.mean()) <= ATT_MEAN_ABS / 4, \
            (float(diff.max()), float(diff.mean()))
        np.testing.assert_allclose(lse.cpu().numpy(), lse_g[:, :, sl].cpu().numpy(), rtol=0,
                                   atol=1e-4)
        # and the oracle, on the unsplit CSR rows of this rank
        rows = np.array([bh * wl.Nc + r * nc_l + i for bh in range(wl.B * wl.heads)
                         for i in range(nc_l)])
        o_out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, g_rp, g_ci, rows)
        full = torch.zeros_like(out_g)
        full[:, :, sl] = out
        mx, mean = compare_attention(gather_rows(host_f32(full), wl, rows), o_out)
        assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
        # as accurate as the unsplit call on these rows (measured: max within 2 %, mean
        # within 0.1 %; with bf16 partials merged in bf16 the ring was 1.5-2.7x worse)
        mx_u, mean_u = compare_attention(gather_rows(host_f32(out_g), wl, rows), o_out)
        assert mx <= 1.1 * mx_u and mean <= 1.02 * mean_u, (mx, mx_u, mean, mean_u)


def test_csr_slice_and_merge_units():
    """bsa_csr_slice keeps [lo, hi) re-indexed in row order; bsa_lse_merge of a
    split selection equals the forward over the whole selection."""
    wl = synth.WORKLOADS["tiny"].with_(heads=2, T=8, H=16, W=32, d=64, topk=7)
    q, k, v = synth.make_qkv(wl)
    qd, kd, vd = dev(q), dev(k), dev(v)
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    ops = CudaOps()
    rp_h = pl.row_ptr.cpu().numpy()
    ci_h = pl.col_idx[: int(rp_h[-1])].cpu().numpy()
    outs = []
    for lo, hi in ((0, 13), (13, 32)):
        srp, sci = ops.slice(pl.row_ptr, pl.col_idx, lo, hi)
        srp_h, sci_h = srp.cpu().numpy(), sci.cpu().numpy()
        for r in range(wl.rows):
            row = ci_h[rp_h[r]:rp_h[r + 1]]
            assert np.array_equal(sci_h[srp_h[r]:srp_h[r + 1]], row[(row >= lo) & (row < hi)] - lo)
        # attention over the slice: shift the key ids back by running on the whole grid
        back = torch.from_numpy(sci_h[: srp_h[-1]] + lo).cuda() if srp_h[-1] else \
            torch.zeros(1, dtype=torch.int32, device="cuda")
        outs.append(ops.forward(p, qd, kd, vd, srp, back.to(torch.int32)))
    (o, l), (o2, l2) = outs
    assert o.dtype == torch.float32 and o2.dtype == torch.float32   # fp32 partial results
    ops.merge(p, o, l, o2, l2)
    of, lf = ops.forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx)
    ops.check()
    # fp32 against fp32: only the bf16 rounding of P against different running maxima
    diff = (o - of).abs()
    assert float(diff.max()) <= 2e-3 and float(diff.mean()) <= 1e-4, \
        (float(diff.max()), float(diff.mean()))
    torch.testing.assert_close(l, lf, rtol=0, atol=1e-4)
    # and the merged fp32 result against the oracle
    rows = np.arange(wl.rows)
    o_out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, 1 / math.sqrt(wl.d), rp_h, ci_h, rows)
    mx, mean = compare_attention(gather_rows(o.cpu().numpy(), wl, rows), o_out)
    assert mx <= ATT_MAX_ABS / 4 and mean <= ATT_MEAN_ABS / 4, (mx, mean)


def _unsplit_backward(wl, qd, kd, vd, gd):
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    bsa.bsa_plan(p, qd, kd, pl.workspace, pl.row_ptr, pl.col_idx)
    out = torch.empty_like(qd)
    lse = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_forward(p, qd, kd, vd, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
    ws = bsa.backward_workspace(p)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    bsa.bsa_backward(p, qd, kd, vd, out, lse, gd, pl.row_ptr, pl.col_idx, ws, dq, dk, dv)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    assert bsa.bsa_read_status(ws) == bsa.BSA_OK
    rp = pl.row_ptr.cpu().numpy()
    return rp, pl.col_idx[: int(rp[-1])].cpu().numpy(), dq, dk, dv


@pytest.mark.parametrize("name", sorted(CASES))
def test_ring_backward_equals_unsplit(name):
    """Each rank's ring backward, run one rank after another with the K/V shards
    each step would deliver, and the dK/dV contributions summed over the ranks as
    the reduce-scatter would: the gradients must match the unsplit backward and
    the oracle within the backward bars (the shard contributions are rounded to
    bf16 before their fp32 sum)."""
    wl, world = CASES[name]
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    HW = wl.H * wl.W
    T_l = wl.T // world
    qd, kd, vd, gd = dev(q), dev(k), dev(v), dev(g)
    g_rp, g_ci, dq_g, dk_g, dv_g = _unsplit_backward(wl, qd, kd, vd, gd)
    qs, ks, vs, gs = (shard(x, world, T_l, HW) for x in (qd, kd, vd, gd))
    ops = CudaOps()
    p_local = bsa.make_params(wl.B, wl.heads, T_l, wl.H, wl.W, wl.d, wl.mode, wl.topk)
    kp_all = torch.stack([ops.pool(p_local, ks[r]) for r in range(world)])
    grid = (T_l, wl.H, wl.W)
    dq_full = torch.empty_like(qd)
    parts = []
    for r in range(world):
        out, lse, rp, ci = ring_forward(qs[r], ks[r], vs[r], grid, wl.topk, wl.mode, wl.cdf_p,
                                        wl.cdf_cap_frac, wl.t_cond,
                                        comm=SimComm(r, world, kp_all, ks, vs), ops=CudaOps(),
                                        return_csr=True)
        bops = CudaOps()
        dq_acc, dkv = ring_backward_partials(qs[r], ks[r], vs[r], out, lse, gs[r], rp, ci, grid,
                                             comm=SimComm(r, world, kp_all, ks, vs), ops=bops)
        bops.check()
        dq_full[:, :, r * T_l * HW:(r + 1) * T_l * HW] = bops.finalize(p_local, dq_acc)
        parts.append(dkv)
    dk_full, dv_full = torch.empty_like(kd), torch.empty_like(vd)
    for j in range(world):
        sl = slice(j * T_l * HW, (j + 1) * T_l * HW)
        dk_full[:, :, sl] = ops.finalize(p_local, sum(pt[0, j] for pt in parts).contiguous())
        dv_full[:, :, sl] = ops.finalize(p_local, sum(pt[1, j] for pt in parts).contiguous())
    rows = np.arange(wl.rows)
    scale = 1.0 / math.sqrt(wl.d)
    o_dq, o_dk, o_dv = oracle.attend_bwd(q, k, v, g, wl.T, wl.H, wl.W, scale, g_rp, g_ci, rows)
    errs = {"dq": rel_errors(gather_rows(host_f32(dq_full), wl, rows), o_dq),
            "dk": rel_errors(host_f32(dk_full), o_dk),
            "dv": rel_errors(host_f32(dv_full), o_dv)}
    for nm, (mx, mean) in errs.items():
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (nm, errs)
    # and against the unsplit GPU backward, within the same bars
    ref = {"dq": gather_rows(host_f32(dq_g), wl, rows), "dk": host_f32(dk_g),
           "dv": host_f32(dv_g)}
    got = {"dq": gather_rows(host_f32(dq_full), wl, rows), "dk": host_f32(dk_full),
           "dv": host_f32(dv_full)}
    for nm in ref:
        mx, mean = rel_errors(got[nm], ref[nm])
        assert mx <= BWD_MAX_REL and mean <= BWD_MEAN_REL, (nm, mx, mean)


def test_ring_backward_one_rank_is_the_backward():
    """A group of one: ring_backward (forward CSR, one shard, reduce-scatter of
    one) must give the unsplit backward up to the fp32 round trip, i.e. exactly."""
    wl = synth.WORKLOADS["tiny"].with_(heads=2, T=8, H=13, W=37, d=128, topk=5)
    q, k, v = synth.make_qkv(wl)
    g = synth.make_dout(wl)
    qd, kd, vd, gd = dev(q), dev(k), dev(v), dev(g)
    _, _, dq_g, dk_g, dv_g = _unsplit_backward(wl, qd, kd, vd, gd)
    ops = CudaOps()
    p = bsa.make_params(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, wl.mode, wl.topk)
    kp_all = torch.stack([ops.pool(p, kd)])
    comm = SimComm(0, 1, kp_all, [kd], [vd])
    out, lse, rp, ci = ring_forward(qd, kd, vd, (wl.T, wl.H, wl.W), wl.topk, comm=comm, ops=ops,
                                    return_csr=True)
    dq, dk, dv = ring_backward(qd, kd, vd, out, lse, gd, rp, ci, (wl.T, wl.H, wl.W),
                               comm=SimComm(0, 1, kp_all, [kd], [vd]), ops=CudaOps())
    # bf16 -> fp32 -> bf16 is the identity
    for a, b in ((dq, dq_g), (dk, dk_g), (dv, dv_g)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_grad_accumulate_and_finalize_units():
    """The fp32 accumulation of bf16 parts equals the fp32 sums taken in the same
    order (bf16 widens exactly), and the final rounding is round-to-nearest-even
    (torch's bf16 cast)."""
    wl = synth.WORKLOADS["tiny"].with_(heads=2, T=4, H=4, W=8, d=64)
    p = bsa.make_params(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, "topk", 1)
    shape = (wl.B, wl.heads, wl.N, wl.d)
    gen = torch.Generator(device="cpu").manual_seed(5)
    parts = [torch.randn(shape, generator=gen).to(torch.bfloat16).cuda() for _ in range(3)]
    acc = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    bsa.bsa_grad_accumulate(p, parts[0], acc, overwrite=True)
    for x in parts[1:]:
        bsa.bsa_grad_accumulate(p, x, acc, overwrite=False)
    ref = parts[0].float() + parts[1].float() + parts[2].float()
    assert torch.equal(acc, ref)
    acc2 = torch.randn(shape, generator=gen).cuda() * 3
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    bsa.bsa_grad_finalize(p, acc2, out)
    assert torch.equal(out.view(torch.int16), acc2.to(torch.bfloat16).view(torch.int16))
