"""Multi-rank host logic on CPU (gloo, world size 2 and 3).

The operator shards with no exchange. By default the heads of the one call are
split across the ranks; with replicas each rank runs its own problem (its own
batch element). Only the timing is reduced over ranks. The ranks here run the
CPU oracle as a stand-in for their GPU step, so this needs no GPU.
"""
import math
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        wl = synth.WORKLOADS["tiny"]
        q, k, v = synth.make_qkv(wl, batch_offset=bench.shard_batch_offset(rank, wl))
        scale = 1 / math.sqrt(wl.d)
        rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, "topk", wl.topk)
        out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, np.arange(wl.rows))
        step_ms = 10.0 + 5.0 * rank               # a rank-dependent step time
        flops = bench.exec_flops(wl, int(rp[-1]))
        t_max = bench.reduce_over_ranks(step_ms, "max", world, "cpu")
        f_sum = bench.reduce_over_ranks(flops, "sum", world, "cpu")
        np.savez(os.path.join(result_dir, f"r{rank}.npz"), out=out, q=q, t_max=t_max,
                 f_sum=f_sum, flops=flops)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_shard_independent_problems(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r = [np.load(tmp_path / f"r{i}.npz") for i in range(world)]
    # timing: max over ranks; work: sum over ranks
    assert all(float(x["t_max"]) == 15.0 for x in r)
    assert all(float(x["f_sum"]) == float(r[0]["flops"]) + float(r[1]["flops"]) for x in r)
    # the ranks drew different problems ...
    assert not np.array_equal(r[0]["q"], r[1]["q"])
    # ... which are exactly the batch elements of one B=2 problem
    wl2 = synth.WORKLOADS["tiny"].with_(B=2)
    q2, k2, v2 = synth.make_qkv(wl2)
    scale = 1 / math.sqrt(wl2.d)
    rp, ci, _ = oracle.plan(q2, k2, wl2.T, wl2.H, wl2.W, scale, "topk", wl2.topk)
    out2, _ = oracle.attend(q2, k2, v2, wl2.T, wl2.H, wl2.W, scale, rp, ci, np.arange(wl2.rows))
    per_rank = wl2.rows // world
    for i in range(world):
        np.testing.assert_array_equal(r[i]["q"][0], q2[i])
        np.testing.assert_array_equal(r[i]["out"], out2[i * per_rank:(i + 1) * per_rank])


def _head_worker(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        full = synth.WORKLOADS["tiny"].with_(heads=5, T=8, mode="cdf", t_cond=4)
        wl, b_off, h_off = bench.rank_problem(full, rank, world, "heads")
        q, k, v = synth.make_qkv(wl, batch_offset=b_off, head_offset=h_off)
        scale = 1 / math.sqrt(wl.d)
        rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                                wl.cdf_cap_frac, wl.t_cond)
        out, lse = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, np.arange(wl.rows))
        # gather every rank's heads (the caller's optional all-gather of O over heads)
        parts = [None] * world
        dist.all_gather_object(parts, (h_off, out, lse))
        np.savez(os.path.join(result_dir, f"h{rank}.npz"),
                 offsets=np.array([p[0] for p in parts]),
                 out=np.concatenate([p[1] for p in sorted(parts, key=lambda x: x[0])]),
                 lse=np.concatenate([p[2] for p in sorted(parts, key=lambda x: x[0])]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_head_split_shards_concatenate_to_the_unsplit_call(tmp_path, world):
    """5 heads over 2 or 3 ranks (uneven shards): every rank draws exactly its
    heads of the one problem, and the shards' outputs, in head order, equal the
    oracle's output of the unsplit call."""
    mp.start_processes(_head_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    full = synth.WORKLOADS["tiny"].with_(heads=5, T=8, mode="cdf", t_cond=4)
    q, k, v = synth.make_qkv(full)
    scale = 1 / math.sqrt(full.d)
    rp, ci, _ = oracle.plan(q, k, full.T, full.H, full.W, scale, full.mode, full.topk,
                            full.cdf_p, full.cdf_cap_frac, full.t_cond)
    out, lse = oracle.attend(q, k, v, full.T, full.H, full.W, scale, rp, ci,
                             np.arange(full.rows))
    for r in range(world):
        got = np.load(tmp_path / f"h{r}.npz")
        assert list(got["offsets"]) == [bench.shard_heads(i, world, 5)[0] for i in range(world)]
        np.testing.assert_array_equal(got["out"], out)
        np.testing.assert_array_equal(got["lse"], lse)


def test_shard_heads_covers_every_head_once():
    for heads in (1, 5, 32):
        for world in range(1, heads + 1):
            spans = [bench.shard_heads(r, world, heads) for r in range(world)]
            assert spans[0][0] == 0 and all(n >= 1 for _, n in spans)
            assert all(spans[i][0] + spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            assert spans[-1][0] + spans[-1][1] == heads
            assert max(n for _, n in spans) - min(n for _, n in spans) <= 1
