#!/usr/bin/env python
"""Benchmark of the 3D block sparse attention hot path on B200.

One step = bsa_plan (chunk gather + mean-pool, pooled scores, selection into
CSR) + bsa_forward (block-sparse attention) over one synthetic batch of the
chosen workload (default: the 720p-like refinement grid, 93.75% sparse),
inputs resident in HBM. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 720p]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

Multi-GPU: one process per GPU (torchrun). By default the heads of the one
call are split across the ranks (every (batch, head) pair is an independent
problem for pooling, selection and attention, so there is no collective on the
data path; strong scaling: the total work is the same for every N). With
--partition replicas every rank runs its own copy of the problem (its own batch
element; weak scaling). Timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BSA fwd ms/call and executed TFLOPS (% of bf16 peak) at 720p grid, 93.75% sparse"
UNIT = "TFLOP/s"
KERNEL_SRC = os.path.join(ROOT, "block_sparse_attention_13_b200", "csrc", "bsa_attn.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "bsa_fwd_traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="720p")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller cases for profiling)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-group", type=int, default=2,
                    help="(batch, head) pairs per group of the host-buffer pipeline")
    ap.add_argument("--e2e-streams", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--backward", action="store_true",
                    help="time bsa_backward (dQ, dK, dV) on the same plan (the default)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward timing")
    ap.add_argument("--bwd-steps", type=int, default=10)
    ap.add_argument("--partition", default="heads", choices=["heads", "replicas"],
                    help="N > 1: split the heads of the one call (default) or run replicas")
    ap.add_argument("--per-config", default="480p,long,causal_cdf,720p_q64",
                    help="other workloads timed after the main one (N = 1; '' for none)")
    ap.add_argument("--per-config-steps", type=int, default=10)
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk.get("bf16_tflops", 1590.0), pk.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for f in sorted(os.listdir(os.path.dirname(KERNEL_SRC))):
        if f in ("bsa_attn.cu", "bsa_ptx.cuh", "bsa_internal.cuh"):   # the kernel's sources
            with open(os.path.join(os.path.dirname(KERNEL_SRC), f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(wl):
    """DRAM bytes per forward launch of workload `wl` from a committed ncu
    capture, if the kernel source is unchanged since that capture. The record
    is for the named workload's whole call; a rank's launch over part of its
    (batch, head) pairs moves that share of it (each pair reads its own Q, K,
    V and writes its own O)."""
    import synth
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f)
    ent = rec.get(wl.name)
    if not ent or ent.get("kernel_hash") != kernel_hash():
        return None
    full = synth.WORKLOADS[wl.name]
    return ent["bytes_per_launch"] * (wl.B * wl.heads) / (full.B * full.heads)


def exec_flops(wl, nnz):
    """Attention FLOPs of the kept chunk pairs: QK^T and PV over the query chunk's
    and the key chunk's tokens. With 128-token query chunks the plan's CSR lists
    (4,4,8) boxes (128 x 128 per entry); with 64-token query chunks it lists key
    chunks of 64 or 128 tokens."""
    qc = tuple(getattr(wl, "qchunk", (4, 4, 8)))
    if qc == (4, 4, 8):
        return 4.0 * wl.d * 128 * 128 * nnz
    kc = tuple(wl.kchunk)
    return 4.0 * wl.d * (qc[0] * qc[1] * qc[2]) * (kc[0] * kc[1] * kc[2]) * nnz


def sparsity(wl, nnz):
    """1 - (attended query-key pairs) / (all query-key pairs of the computed rows)."""
    qc = tuple(getattr(wl, "qchunk", (4, 4, 8)))
    qn = qc[0] * qc[1] * qc[2]
    return 1.0 - exec_flops(wl, nnz) / (4.0 * wl.d * wl.rows * qn * wl.N)


def q64_box_entries(wl, row_ptr, col_idx):
    """64-token query chunks: the (query box, key box) pairs the kernel computes
    (each a 128 x 128 tile), i.e. the union over a box's two query chunks."""
    import numpy as np
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx[: rp[-1]], dtype=np.int64)
    NH, NW, NWq = wl.NH, wl.NW, wl.NWq
    rows = np.repeat(np.arange(len(rp) - 1), np.diff(rp))
    bh, q = rows // wl.Nc, rows % wl.Nc
    qbox = bh * (wl.Nc // NWq * NW) + (q // NWq) * NW + (q % NWq) // 2
    if tuple(wl.kchunk) == (4, 4, 4):
        kbox = (ci // NWq) * NW + (ci % NWq) // 2
    else:
        kbox = ci
    return int(np.unique(qbox * (1 << 20) + kbox).size)


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"bsa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self, t_begin=None, t_end=None):
        """Median SM clock and throttle reasons over the samples taken between
        host times t_begin and t_end (seconds since the epoch)."""
        import datetime
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    clk, cmax = float(parts[2]), float(parts[3])
                except ValueError:
                    continue
                if t_begin is not None and not (t_begin <= ts <= t_end):
                    continue
                sm.append(clk)
                mx.append(cmax)
                for nm, val in zip(names, parts[6:10]):
                    if val.lower() == "active":
                        reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------- CPU oracle leg

def cpu_oracle_sample(wl, q, k, v, target_s):
    """Time the oracle (as it stands) on a bounded sample and extrapolate the
    full step: plan on one head, attention on a seeded sample of query chunks."""
    import numpy as np
    import oracle

    scale = 1.0 / math.sqrt(wl.d)
    qh, kh = q[:1, :1], k[:1, :1]
    t0 = time.perf_counter()
    rp, ci, _ = oracle.plan(qh, kh, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                            wl.cdf_cap_frac, min(wl.t_cond, wl.T))
    t_plan_head = time.perf_counter() - t0
    # attention rows of head 0, grown until the sample takes ~target_s
    rng = np.random.default_rng(0)
    order = wl.q_skip + rng.permutation(wl.Nq)   # only the computed query chunks
    n, t_att, done = 4, 0.0, 0
    while True:
        rows = np.sort(order[done:done + n])
        t0 = time.perf_counter()
        oracle.attend(qh, kh, v[:1, :1], wl.T, wl.H, wl.W, scale, rp, ci, rows, want_lse=False)
        t_att += time.perf_counter() - t0
        done += len(rows)
        if t_att + t_plan_head >= target_s or done >= wl.Nq:
            break
        n = min(wl.Nq - done, max(4, int(n * 2)))
    sample_nnz = int(sum(rp[r + 1] - rp[r] for r in order[:done]))
    t_per_chunk_pair = t_att / max(sample_nnz, 1)
    # head 0's selection size over the computed rows as the estimate
    full_nnz = int(rp[-1] - rp[wl.q_skip]) * wl.B * wl.heads
    t_full = t_plan_head * wl.B * wl.heads + t_per_chunk_pair * full_nnz
    value = exec_flops(wl, full_nnz) / t_full / 1e12
    return {
        "value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
        "sample": (f"plan on 1 of {wl.B * wl.heads} (batch,head) pairs + attention on {done} of "
                   f"{wl.rows} query chunks; full step extrapolated linearly "
                   f"({t_full:.1f} s)"),
        "sample_seconds": round(t_plan_head + t_att, 2),
        "est_full_step_s": t_full,
    }


def run_reference(args, wl, rank, world):
    """The oracle as it stands, on the host cores. Each timed step is one
    bounded sample of the workload (plan on one (batch, head) pair, attention
    on a growing set of that head's query chunks); the line reports what ran:
    `steps` samples of `ms_per_step` wall time each, and the throughput the
    sample extrapolates to for the full workload (`extrapolated`)."""
    if rank != 0:
        return 0
    import synth
    q, k, v = synth.make_qkv(wl.with_(B=1, heads=1))
    per_step = max(1.0, min(args.cpu_seconds, 100.0 / max(1, args.steps + args.warmup)))
    vals, secs = [], []
    cb = None
    t_run0 = time.perf_counter()
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cb = cpu_oracle_sample(wl, q, k, v, per_step)
        if s >= args.warmup:
            vals.append(cb["value"])
            secs.append(time.perf_counter() - t0)
    value = statistics.median(vals)
    cb["value"] = value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": len(secs), "warmup": args.warmup,
        "ms_per_step": statistics.mean(secs) * 1e3, "higher_is_better": True,
        "extrapolated": True, "est_full_step_s": cb["est_full_step_s"],
        "wall_s": time.perf_counter() - t_run0,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world, "oracle"),
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, world, parallelism):
    return {"workload": wl.name, "B": wl.B, "heads": wl.heads, "grid_thw": [wl.T, wl.H, wl.W],
            "d": wl.d, "chunk_thw": list(getattr(wl, "qchunk", (4, 4, 8))),
            "key_chunk_thw": list(getattr(wl, "kchunk", (4, 4, 8))), "mode": wl.mode,
            "topk": wl.topk if wl.mode != "cdf" else None,
            "cdf_p": wl.cdf_p if wl.mode != "topk" else None,
            "t_cond": wl.t_cond, "q_begin": wl.q_begin, "parallelism": parallelism,
            "l2": "inputs larger than L2 (Q+K+V per step "
                  f"{3 * wl.B * wl.heads * wl.N * wl.d * 2 / 1e9:.2f} GB)"}


# ---------------------------------------------------------------------- backward

def time_backward(args, wl, p, pl, q, k, v, stream, peak_tf, batch_offset=0, head_offset=0):
    """bsa_backward on the plan of the timed forward: forward once with LSE,
    then K timed backward calls (events on the launching stream). Algorithmic
    FLOPs are the five products of the gradient (S, dP, dV, dS K, dS^T Q:
    2.5x the forward's); the kernels execute seven (S and dP are recomputed
    once for dQ and once for dK/dV)."""
    import torch
    import synth
    import block_sparse_attention_13_b200 as bsa
    g_np = synth.make_dout(wl, batch_offset=batch_offset, head_offset=head_offset)
    dout = torch.from_numpy(g_np).view(torch.bfloat16).to("cuda")
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    bsa.bsa_plan(p, q, k, pl.workspace, pl.row_ptr, pl.col_idx)
    bsa.bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
    ws = bsa.backward_workspace(p)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def bwd():
        bsa.bsa_backward(p, q, k, v, out, lse, dout, pl.row_ptr, pl.col_idx, ws, dq, dk, dv)

    for _ in range(max(3, args.warmup)):
        bwd()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.bwd_steps)]
    for a, b in evs:
        a.record(stream)
        bwd()
        b.record(stream)
    torch.cuda.synchronize()
    rc = bsa.bsa_read_status(ws)
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    nnz = int(pl.row_ptr[-1].item())
    alg = 2.5 * exec_flops(wl, nnz)
    executed = 3.5 * exec_flops(wl, nnz)
    return {"bwd_ms": ms, "steps": args.bwd_steps, "algorithmic_flops": alg,
            "executed_flops": executed, "alg_tflops": alg / ms / 1e9,
            "exec_tflops": executed / ms / 1e9, "exec_frac": executed / ms / 1e9 / peak_tf,
            # prep, CSR->CSC (scatter, count, scan, emit), dQ, dK/dV
            "launches_per_call": 7, "device_status": bsa.status_string(rc)}


# ---------------------------------------------------------------------- other workloads

def time_config(wl, steps, peak_tf, stream):
    """plan + forward on another workload (inputs resident, larger than L2):
    CUDA events per kernel group on the launching stream, `steps` timed steps
    after 3 warm-up steps."""
    import torch
    import synth
    import block_sparse_attention_13_b200 as bsa
    host = synth.make_qkv(wl)
    q, k, v = (torch.from_numpy(a).view(torch.bfloat16).to("cuda") for a in host)
    del host
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    out = torch.empty_like(q)
    for _ in range(3):
        bsa.bsa_plan(p, q, k, pl.workspace, pl.row_ptr, pl.col_idx)
        bsa.bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        e[0].record(stream)
        bsa.bsa_plan(p, q, k, pl.workspace, pl.row_ptr, pl.col_idx)
        e[1].record(stream)
        bsa.bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out)
        e[2].record(stream)
    torch.cuda.synchronize()
    rc = bsa.bsa_read_status(pl.workspace)
    nnz = int(pl.row_ptr[-1].item())
    plan_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    fwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    tf = exec_flops(wl, nnz) / fwd_ms / 1e9
    res = {"plan_ms": plan_ms, "fwd_ms": fwd_ms, "step_ms": plan_ms + fwd_ms,
           "fwd_exec_tflops": tf, "frac": tf / peak_tf, "nnz": nnz,
           "sparsity": sparsity(wl, nnz), "steps": steps,
           "config": workload_config(wl, 1, "single"), "device_status": bsa.status_string(rc)}
    if tuple(wl.qchunk) != (4, 4, 8):
        # the kernel's tiles: (query box, key box) pairs of the two chunks' union
        n_box = q64_box_entries(wl, pl.row_ptr.cpu().numpy(), pl.col_idx.cpu().numpy())
        tile_tf = 4.0 * wl.d * 128 * 128 * n_box / fwd_ms / 1e9
        res.update({"fwd_exec_tflops_note": "algorithmic: 4*d*64*64 per kept chunk pair",
                    "box_tiles": n_box, "tile_tflops": tile_tf, "tile_frac": tile_tf / peak_tf,
                    "useful_share_of_tiles": exec_flops(wl, nnz) / (4.0 * wl.d * 128 * 128 *
                                                                    n_box)})
        # the backward over the same box tiles: 7 products of 2*d*128*128 FLOP per
        # (query box, key box) pair executed; 5 per kept chunk pair are the gradient's
        dout = torch.from_numpy(synth.make_dout(wl)).view(torch.bfloat16).to("cuda")
        lse = torch.empty((wl.B, wl.heads, wl.N), dtype=torch.float32, device="cuda")
        bsa.bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
        ws = bsa.backward_workspace(p)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def bwd():
            bsa.bsa_backward(p, q, k, v, out, lse, dout, pl.row_ptr, pl.col_idx, ws, dq, dk, dv)

        for _ in range(3):
            bwd()
        torch.cuda.synchronize()
        bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for a, b in bev:
            a.record(stream)
            bwd()
            b.record(stream)
        torch.cuda.synchronize()
        bwd_ms = statistics.mean(a.elapsed_time(b) for a, b in bev)
        bwd_tile_tf = 3.5 * 4.0 * wl.d * 128 * 128 * n_box / bwd_ms / 1e9
        res["backward"] = {"bwd_ms": bwd_ms, "steps": steps,
                           "alg_tflops": 2.5 * exec_flops(wl, nnz) / bwd_ms / 1e9,
                           "tile_tflops": bwd_tile_tf, "tile_frac": bwd_tile_tf / peak_tf,
                           "device_status": bsa.status_string(bsa.bsa_read_status(ws))}
        del dout, lse, ws, dq, dk, dv
    del q, k, v, out, pl
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------- ranks

def shard_batch_offset(rank, wl):
    """Batch index of this rank's first element when every rank runs its own
    independent replica of the problem (weak scaling, no data exchange)."""
    return rank * wl.B


def shard_heads(rank, world, heads):
    """Heads [h0, h0 + n) of the call that this rank computes: the heads split as
    evenly as possible, the first `heads % world` ranks taking one more. Every
    (batch, head) pair is an independent problem for pooling, selection and
    attention, so the ranks exchange nothing."""
    base, extra = divmod(heads, world)
    n = base + (1 if rank < extra else 0)
    h0 = rank * base + min(rank, extra)
    return h0, n


def rank_problem(wl, rank, world, partition):
    """(this rank's workload, batch offset, head offset) of its inputs."""
    if partition == "heads" and world > 1:
        h0, n = shard_heads(rank, world, wl.heads)
        if n == 0:
            raise ValueError(f"{world} ranks for {wl.heads} heads: rank {rank} has none")
        return wl.with_(heads=n), 0, h0
    return wl, shard_batch_offset(rank, wl), 0


def parallelism_of(partition, world):
    if world == 1:
        return "single"
    return f"heads/{world}" if partition == "heads" else f"replicas{world}"


def reduce_over_ranks(value, op, world, device):
    """MAX or SUM of a scalar over ranks (plumbing for the timing only)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------- GPU leg

def main():
    args = parse()
    import synth
    wl = synth.WORKLOADS[args.workload]
    if args.heads:
        wl = wl.with_(heads=args.heads, name=f"{wl.name}_h{args.heads}")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, wl, rank, world)

    import torch
    import torch.distributed as dist
    import block_sparse_attention_13_b200 as bsa

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_over_ranks(x, "max", world, "cuda")

    def sum_over_ranks(x):
        return reduce_over_ranks(x, "sum", world, "cuda")

    # inputs: this rank's part of the call (its heads) or its own replica, pinned host +
    # device copies
    wl_full = wl
    wl, b_off, h_off = rank_problem(wl_full, rank, world, args.partition)
    q_np, k_np, v_np = synth.make_qkv(wl, batch_offset=b_off, head_offset=h_off)
    host = [torch.from_numpy(a).view(torch.bfloat16).pin_memory() for a in (q_np, k_np, v_np)]
    q, k, v = (h.to("cuda", non_blocking=False) for h in host)
    p = bsa.params_for(wl)
    pl = bsa.allocate(p)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def step():
        bsa.bsa_plan(p, q, k, pl.workspace, pl.row_ptr, pl.col_idx)
        bsa.bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    rc = bsa.bsa_read_status(pl.workspace)
    if rc != bsa.BSA_OK:
        print(json.dumps({"error": f"device status {bsa.status_string(rc)}"}), flush=True)
        return 1
    nnz = int(pl.row_ptr[-1].item())
    flops = exec_flops(wl, nnz)

    # ---- timed region: K steps, per-kernel events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.5)  # let the sampler start before the timed region
        host_t0 = time.time()
        t_start.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            bsa.bsa_plan(p, q, k, pl.workspace, pl.row_ptr, pl.col_idx)
            ev[s][1].record(stream)
            bsa.bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out)
            ev[s][2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        host_t1 = time.time()
        barrier()
    clocks = clk.summary(host_t0, host_t1)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end))
    plan_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    fwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    ms_per_step = total_ms / args.steps
    rc = bsa.bsa_read_status(pl.workspace)
    launches_per_step = 4 if wl.mode == "topk" else 6   # pool, scores, select(+scan, compact), fwd
    total_flops = sum_over_ranks(flops * args.steps)
    value = total_flops / (total_ms / 1e3) / 1e12

    # ---- end to end with host buffers (pinned) through the C ABI's host-buffer entry
    # (bsa_forward_host, via HostForward): per step H2D of q, k, v, plan, forward and D2H
    # of the output, in groups of (batch, head) pairs whose copies overlap the other
    # groups' kernels
    from block_sparse_attention_13_b200.host import HostForward
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hf = HostForward(p, group=args.e2e_group, streams=args.e2e_streams)
    hf(host[0], host[1], host[2], out_host)          # warm-up
    torch.cuda.synchronize()
    hf.check()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e_s.record(stream)
    for _ in range(max(args.e2e_steps, 1)):
        hf(host[0], host[1], host[2], out_host)
    e_e.record(stream)
    torch.cuda.synchronize()
    hf.check()
    barrier()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e)) / max(args.e2e_steps, 1)
    e2e_value = sum_over_ranks(flops) / (e2e_ms / 1e3) / 1e12
    h2d = sum(h.numel() * h.element_size() for h in host)
    d2h = out_host.numel() * out_host.element_size()

    # ---- dense comparator at the same shape (torch SDPA as dispatched)
    dense = None
    if not args.no_dense and rank == 0 and wl.t_cond == 0:
        import torch.nn.functional as F
        F.scaled_dot_product_attention(q, k, v)
        torch.cuda.synchronize()
        ts = []
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            F.scaled_dot_product_attention(q, k, v)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        dense_ms = statistics.median(ts)
        dense = {"sdpa_ms": dense_ms, "bsa_step_ms": ms_per_step,
                 "speedup": dense_ms / ms_per_step,
                 "dense_tflops": 4.0 * wl.B * wl.heads * wl.N * wl.N * wl.d / dense_ms / 1e9}

    peak_tf, peak_hbm, peak_src = load_peaks()
    fwd_tflops = flops / (fwd_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "achieved": fwd_tflops, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": fwd_tflops / peak_tf, "traffic": load_traffic(wl),
                "kernel": "bsa_fwd_kernel", "peak_source": f"{peak_src} bf16 (burst)",
                "algorithmic_flops_per_launch": flops}

    bwd = None
    if not args.no_backward:
        bwd = time_backward(args, wl, p, pl, q, k, v, stream, peak_tf, b_off, h_off)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(wl, q_np, k_np, v_np, args.cpu_seconds)

    per_config = None
    if world == 1 and args.per_config:
        per_config = {}
        del hf, out_host
        for name in [x for x in args.per_config.split(",") if x]:
            per_config[name] = time_config(synth.WORKLOADS[name], args.per_config_steps,
                                           peak_tf, stream)

    # the whole job's dense-equivalent work (every rank reaches this collective)
    dense_equiv = sum_over_ranks(4.0 * wl.B * wl.heads * wl.Nq * 128 * wl.N * wl.d)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "strong" if (args.partition == "heads" and world > 1) else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(wl_full, world, parallelism_of(args.partition, world)),
            "plan_ms": plan_ms, "fwd_ms": fwd_ms, "fwd_exec_tflops": fwd_tflops,
            "nnz": nnz, "sparsity": sparsity(wl, nnz),
            "dense_equiv_tflops": dense_equiv / ms_per_step / 1e9,
            "dense": dense, "roofline": roofline, "cpu_baseline": cpu, "backward": bwd,
            "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "bsa_forward_host (C ABI, via HostForward; pinned host q, k, v "
                           "-> out)",
                    "group": args.e2e_group, "streams": args.e2e_streams},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks, "device_status": bsa.status_string(rc),
            "per_config": per_config,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if rc == bsa.BSA_OK else 1


if __name__ == "__main__":
    sys.exit(main())
