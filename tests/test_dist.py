"""Multi-rank host logic on CPU (gloo, world size 2).

The operator shards with no exchange: each rank runs its own problem (its own
batch element) and only the timing is reduced over ranks. The ranks here run
the CPU oracle as a stand-in for their GPU step, so this needs no GPU.
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
