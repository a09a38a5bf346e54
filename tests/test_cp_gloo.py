"""The context-parallel ring driver on CPU ranks (gloo, world size 2 and 4).

Real ranks exchange the pooled keys (all-gather) and the K/V shards (ring
send/receive) over gloo; their device steps are replaced by an oracle-backed
op set, so what is checked here is the host logic of the ring: the shard
layout of the gathered keys, each rank's row range, which shard is held at
which step, the re-indexing of the selection to it, and the merge order. Each
rank's merged result must equal its rows of the oracle's unsplit computation.
"""
import math
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(x):
    return x.view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    """The ring driver's device steps, done by the oracle on CPU tensors."""

    def __init__(self, wl, world):
        self.wl, self.world = wl, world

    def pool(self, p, x):
        return torch.from_numpy(oracle.pool(_bits(x), p.T, p.H, p.W))

    def select_pooled(self, p, qp, kp_all, kshard):
        wl = self.wl
        w = kp_all.shape[0]
        kp = kp_all.permute(1, 2, 0, 3, 4).reshape(wl.B, wl.heads, w * kshard, wl.d).numpy()
        S = oracle.scores(qp.numpy(), kp, 1.0 / math.sqrt(wl.d))
        # rows of this rank inside a score matrix of the whole grid (block-causal
        # decisions depend on the global query chunk index)
        nc = wl.Nc
        lo = (p.q_begin // 4) * wl.NH * wl.NW
        full = np.zeros((wl.B, wl.heads, nc, nc))
        full[:, :, lo:lo + qp.shape[2]] = S
        rp, ci = oracle.select(full, wl.T, wl.H, wl.W, wl.mode, wl.topk, wl.cdf_p,
                               wl.cdf_cap_frac, wl.t_cond)
        rows = [ci[rp[bh * nc + i]:rp[bh * nc + i + 1]] for bh in range(wl.B * wl.heads)
                for i in range(lo, lo + qp.shape[2])]
        return (torch.from_numpy(np.concatenate([[0], np.cumsum([len(x) for x in rows])])
                                 .astype(np.int32)),
                torch.from_numpy(np.concatenate(rows).astype(np.int32)))

    def slice(self, rp, ci, lo, hi):
        rp, ci = rp.numpy(), ci.numpy()
        rows = [ci[rp[r]:rp[r + 1]] for r in range(len(rp) - 1)]
        rows = [x[(x >= lo) & (x < hi)] - lo for x in rows]
        return (torch.from_numpy(np.concatenate([[0], np.cumsum([len(x) for x in rows])])
                                 .astype(np.int32)),
                torch.from_numpy(np.concatenate(rows).astype(np.int32)))

    def forward(self, p, q, k, v, rp, ci):
        T, H, W = p.T, p.H, p.W
        nc = oracle.num_chunks(T, H, W)
        rows = np.arange(p.B * p.heads * nc)
        o, lse = oracle.attend(_bits(q), _bits(k), _bits(v), T, H, W, 1.0 / math.sqrt(p.d),
                               rp.numpy(), ci.numpy(), rows)
        N = T * H * W
        out = np.zeros((p.B * p.heads, N, p.d))
        ls = np.zeros((p.B * p.heads, N))
        for r in rows:
            tok = oracle.chunk_tokens(T, H, W, r % nc)
            ok = tok >= 0
            out[r // nc][tok[ok]] = o[r][ok]
            ls[r // nc][tok[ok]] = lse[r][ok]
        return (torch.from_numpy(out.reshape(p.B, p.heads, N, p.d)),
                torch.from_numpy(ls.reshape(p.B, p.heads, N)))

    def merge(self, p, out, lse, o2, l2):
        m, lm = oracle.lse_merge(out.numpy(), lse.numpy(), o2.numpy(), l2.numpy())
        out.copy_(torch.from_numpy(m))
        lse.copy_(torch.from_numpy(lm))

    def backward(self, p, q, k, v, out, lse, dout, rp, ci):
        T, H, W = p.T, p.H, p.W
        nc = oracle.num_chunks(T, H, W)
        rows = np.arange(p.B * p.heads * nc)
        dq_rows, dk, dv = oracle.attend_bwd_part(_bits(q), _bits(k), _bits(v), _bits(dout),
                                                 out.numpy(), lse.numpy(), T, H, W,
                                                 1.0 / math.sqrt(p.d), rp.numpy(), ci.numpy(),
                                                 rows)
        N = T * H * W
        dq = np.zeros((p.B * p.heads, N, p.d))
        for r in rows:
            tok = oracle.chunk_tokens(T, H, W, r % nc)
            ok = tok >= 0
            dq[r // nc][tok[ok]] = dq_rows[r][ok]
        return (torch.from_numpy(dq.reshape(p.B, p.heads, N, p.d)), torch.from_numpy(dk),
                torch.from_numpy(dv))

    def accumulate(self, p, part, acc, overwrite):
        if overwrite:
            acc.copy_(part)
        else:
            acc.add_(part.to(acc.dtype))

    def finalize(self, p, acc):
        return acc.double()

    def check(self):
        pass


WORKLOADS = {
    "topk": synth.WORKLOADS["tiny"].with_(heads=2, T=16, H=8, W=16, d=16, topk=3),
    "causal_cdf": synth.WORKLOADS["tiny"].with_(B=2, heads=1, T=16, H=8, W=16, d=16, mode="cdf",
                                                cdf_p=0.9, cdf_cap_frac=0.5, t_cond=8),
}


def _worker(rank, world, port, name, result_dir, backward=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from block_sparse_attention_13_b200.context_parallel import TorchComm, ring_forward
        wl = WORKLOADS[name]
        q, k, v = synth.make_qkv(wl)
        HW = wl.H * wl.W
        T_l = wl.T // world
        sl = slice(rank * T_l * HW, (rank + 1) * T_l * HW)
        qs, ks, vs = (torch.from_numpy(x[:, :, sl].copy()).view(torch.bfloat16) for x in (q, k, v))
        comm, ops = TorchComm(), OracleOps(wl, world)
        out, lse, rp, ci = ring_forward(qs, ks, vs, (T_l, wl.H, wl.W), wl.topk, wl.mode,
                                        wl.cdf_p, wl.cdf_cap_frac, wl.t_cond, comm=comm, ops=ops,
                                        return_csr=True)
        np.save(os.path.join(result_dir, f"out{rank}.npy"), out.numpy())
        np.save(os.path.join(result_dir, f"lse{rank}.npy"), lse.numpy())
        if backward:
            from block_sparse_attention_13_b200.context_parallel import ring_backward
            dout = torch.from_numpy(synth.make_dout(wl)[:, :, sl].copy()).view(torch.bfloat16)
            dq, dk, dv = ring_backward(qs, ks, vs, out, lse, dout, rp, ci, (T_l, wl.H, wl.W),
                                       comm=comm, ops=ops)
            for nm, x in (("dq", dq), ("dk", dk), ("dv", dv)):
                np.save(os.path.join(result_dir, f"{nm}{rank}.npy"), x.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world", [("topk", 2), ("topk", 4), ("causal_cdf", 2)])
def test_ring_forward_on_gloo_ranks(tmp_path, name, world):
    mp.spawn(_worker, args=(world, _free_port(), name, str(tmp_path)), nprocs=world, join=True)
    wl = WORKLOADS[name]
    q, k, v = synth.make_qkv(wl)
    scale = 1.0 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                            wl.cdf_cap_frac, wl.t_cond)
    rows = np.arange(wl.rows)
    o, lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    full = np.zeros((wl.B * wl.heads, wl.N, wl.d))
    full_l = np.zeros((wl.B * wl.heads, wl.N))
    for r in rows:
        tok = oracle.chunk_tokens(wl.T, wl.H, wl.W, r % wl.Nc)
        full[r // wl.Nc][tok] = o[r]
        full_l[r // wl.Nc][tok] = lse[r]
    HW = wl.H * wl.W
    T_l = wl.T // world
    for rank in range(world):
        sl = slice(rank * T_l * HW, (rank + 1) * T_l * HW)
        got = np.load(tmp_path / f"out{rank}.npy").reshape(wl.B * wl.heads, -1, wl.d)
        got_l = np.load(tmp_path / f"lse{rank}.npy").reshape(wl.B * wl.heads, -1)
        np.testing.assert_allclose(got, full[:, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got_l, full_l[:, sl], rtol=0, atol=1e-12)


@pytest.mark.parametrize("name,world", [("topk", 2), ("topk", 4), ("causal_cdf", 2)])
def test_ring_backward_on_gloo_ranks(tmp_path, name, world):
    """dQ of each rank's queries and dK, dV of each rank's shard must equal the
    rows of the unsplit oracle backward: the shard contributions weighted with
    the merged softmax, dQ summed over the ring's steps and dK/dV over the
    ranks by the reduce-scatter."""
    mp.spawn(_worker, args=(world, _free_port(), name, str(tmp_path), True), nprocs=world,
             join=True)
    wl = WORKLOADS[name]
    q, k, v = synth.make_qkv(wl)
    dout = synth.make_dout(wl)
    scale = 1.0 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                            wl.cdf_cap_frac, wl.t_cond)
    rows = np.arange(wl.rows)
    dq_rows, dk, dv = oracle.attend_bwd(q, k, v, dout, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    dq = np.zeros((wl.B * wl.heads, wl.N, wl.d))
    for r in rows:
        tok = oracle.chunk_tokens(wl.T, wl.H, wl.W, r % wl.Nc)
        dq[r // wl.Nc][tok] = dq_rows[r]
    full = {"dq": dq, "dk": dk.reshape(wl.B * wl.heads, wl.N, wl.d),
            "dv": dv.reshape(wl.B * wl.heads, wl.N, wl.d)}
    HW = wl.H * wl.W
    T_l = wl.T // world
    for rank in range(world):
        sl = slice(rank * T_l * HW, (rank + 1) * T_l * HW)
        for nm in ("dq", "dk", "dv"):
            got = np.load(tmp_path / f"{nm}{rank}.npy").reshape(wl.B * wl.heads, -1, wl.d)
            ref = full[nm][:, sl]
            # fp32 accumulators of fp64 contributions
            np.testing.assert_allclose(got, ref, rtol=0, atol=2e-6 * np.abs(full[nm]).max())
