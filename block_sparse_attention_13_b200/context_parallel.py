"""Context-parallel (ring) block sparse attention forward.

"LongCat-Video Technical Report", section "Block Sparse Attention (BSA)",
ring block sparse attention: the latent sequence is split across the ranks of
a group along the latent frames; every rank pools its own keys, the pooled
keys of all ranks are gathered, each rank scores its query chunks against all
of them and keeps the top-k (or CDF) key chunks, and the attention is then
computed shard by shard while the K/V shards travel around the ring, the
partial results being combined by their log-sum-exps ("LongCat-Video
Technical Report #", section "开源实现": LSE and output correction). The
partial outputs stay in fp32 through the merges and are rounded to bf16 once.

The backward (``ring_backward``) runs the same ring again. At each step a rank
computes, with bsa_backward, the contributions of the K/V shard it holds to
its queries' dQ and to that shard's dK and dV, weighted with the merged
output and LSE of the forward (the softmax over all shards). dQ sums the
contributions of every shard on the rank (fp32, bsa_grad_accumulate); dK and
dV of a shard sum the contributions of every rank, which one NCCL
reduce-scatter of the ranks' fp32 contributions delivers to the shard's owner.

On one node of B200s the gather is an NCCL all-gather of the pooled keys
(Nc x d floats per head and rank) and the ring step an NCCL send/receive of
the next K/V shard, posted before the current shard's attention so that the
transfer overlaps it. Every computation runs in the library's kernels
(bsa_pool, bsa_select_pooled, bsa_csr_slice, bsa_forward_partial,
bsa_lse_merge_f32, bsa_grad_finalize);
torch.distributed only moves data.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (BSA_OK, BsaError, backward_workspace, bsa_backward, bsa_csr_slice,
               bsa_csr_slice_workspace_size, bsa_forward_partial, bsa_grad_accumulate,
               bsa_grad_finalize, bsa_lse_merge_f32, bsa_plan_sizes, bsa_pool, bsa_read_status,
               bsa_select_pooled, bsa_workspace_size, make_params, status_string)


class CudaOps:
    """The device steps of one rank, through the C ABI."""

    def __init__(self):
        self._status = []   # workspaces whose status words are read at the end

    def pool(self, p, x):
        B, heads, N, d = x.shape
        nc = ((p.T + 3) // 4) * ((p.H + 3) // 4) * ((p.W + 7) // 8)
        out = torch.empty((B, heads, nc, d), dtype=torch.float32, device=x.device)
        bsa_pool(p, x, out)
        return out

    def select_pooled(self, p, qpool, kpool_shards, kshard):
        rows, nnz = bsa_plan_sizes(p)
        dev = qpool.device
        ws = torch.zeros(bsa_workspace_size(p), dtype=torch.uint8, device=dev)
        row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
        col_idx = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
        bsa_select_pooled(p, qpool, kpool_shards, ws, row_ptr, col_idx, kshard=kshard)
        self._status.append(ws)
        return row_ptr, col_idx

    def slice(self, row_ptr, col_idx, lo, hi):
        dev = row_ptr.device
        ws = torch.zeros(bsa_csr_slice_workspace_size(row_ptr.numel() - 1), dtype=torch.uint8,
                         device=dev)
        out_rp = torch.empty_like(row_ptr)
        out_ci = torch.empty_like(col_idx)
        bsa_csr_slice(row_ptr, col_idx, lo, hi, ws, out_rp, out_ci)
        self._status.append(ws)
        return out_rp, out_ci

    def forward(self, p, q, k, v, row_ptr, col_idx):
        """Partial attention over one K/V shard: fp32 output and LSE."""
        ws = torch.zeros(256, dtype=torch.uint8, device=q.device)
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        B, heads, N, _ = q.shape
        lse = torch.empty((B, heads, N), dtype=torch.float32, device=q.device)
        bsa_forward_partial(p, q, k, v, row_ptr, col_idx, ws, out, lse)
        self._status.append(ws)
        return out, lse

    def merge(self, p, out, lse, out_part, lse_part):
        """fp32 accumulator <- LSE merge with an fp32 partial result."""
        bsa_lse_merge_f32(p, out, lse, out_part, lse_part)

    def backward(self, p, q, k, v, out, lse, dout, row_ptr, col_idx):
        ws = backward_workspace(p, q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bsa_backward(p, q, k, v, out, lse, dout, row_ptr, col_idx, ws, dq, dk, dv)
        self._status.append(ws)
        return dq, dk, dv

    def accumulate(self, p, part, acc, overwrite):
        bsa_grad_accumulate(p, part, acc, overwrite)

    def finalize(self, p, acc):
        out = torch.empty(acc.shape, dtype=torch.bfloat16, device=acc.device)
        bsa_grad_finalize(p, acc, out)
        return out

    def check(self):
        for ws in self._status:
            rc = bsa_read_status(ws)
            if rc != BSA_OK:
                raise BsaError(rc, "device status: " + status_string(rc))
        self._status.clear()


class TorchComm:
    """Group communication through torch.distributed (NCCL on GPUs)."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, x):
        """[world, *x.shape]: every rank's x in rank order (the views of one buffer
        are filled in place, so no reshuffle follows)."""
        out = torch.empty((self.world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        dist.all_gather(list(out.unbind(0)), x.contiguous(), group=self.group)
        return out

    def start_shift(self, tensors):
        """Send `tensors` to the next rank and receive the previous rank's into
        new buffers; returns a handle for finish_shift."""
        nxt = (self.rank + 1) % self.world
        prv = (self.rank - 1) % self.world
        recv = [torch.empty_like(t) for t in tensors]
        ops = [dist.P2POp(dist.isend, t, dist.get_global_rank(self.group, nxt)
                          if self.group is not None else nxt, self.group) for t in tensors]
        ops += [dist.P2POp(dist.irecv, r, dist.get_global_rank(self.group, prv)
                           if self.group is not None else prv, self.group) for r in recv]
        return recv, dist.batch_isend_irecv(ops)

    @staticmethod
    def finish_shift(handle):
        recv, reqs = handle
        for r in reqs:
            r.wait()
        return recv

    def reduce_scatter(self, x):
        """x: [world, *shape] on every rank; returns the sum over ranks of their
        x[rank] slice, on each rank."""
        out = torch.empty(tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        if dist.get_backend(self.group) == "gloo":
            # gloo has no reduce-scatter: reduce the whole buffer, keep this slice
            buf = x.contiguous().clone()
            dist.all_reduce(buf, group=self.group)
            out.copy_(buf[self.rank])
        else:
            dist.reduce_scatter_tensor(out, x.contiguous(), group=self.group)
        return out


def ring_forward(q, k, v, grid, topk=None, mode="topk", cdf_p=0.9, cdf_cap_frac=0.25, t_cond=0,
                 scale=0.0, comm=None, ops=None, return_csr=False):
    """Block sparse attention of this rank's queries over the whole group's sequence.

    q, k, v: this rank's shard, [B, heads, T_l*H*W, d] bf16, holding latent frames
    [rank*T_l, (rank+1)*T_l) of the group's grid (T_l * world, H, W); grid = (T_l, H, W),
    T_l a multiple of 4. topk defaults to 1/16 of the group's key chunks. t_cond counts
    frames of the whole sequence. Returns (out, lse) for the local queries, as
    bsa_forward would give for these rows of the unsplit sequence; with
    return_csr also the rank's selection (row_ptr, col_idx over the key chunks of
    the whole sequence, shard layout), which ring_backward takes.
    """
    comm = comm or TorchComm()
    ops = ops or CudaOps()
    world, rank = comm.world, comm.rank
    T_l, H, W = grid
    if T_l % 4:
        raise ValueError("each rank must hold whole chunks: T_l must be a multiple of 4")
    B, heads, N, d = q.shape
    T = T_l * world
    nc_l = (T_l // 4) * ((H + 3) // 4) * ((W + 7) // 8)
    if topk is None:
        topk = max(1, (nc_l * world) // 16)
    # the shard's own grid (pooling, attention, merge) and this rank's rows of the whole
    p_local = make_params(B, heads, T_l, H, W, d, mode, topk, cdf_p, cdf_cap_frac, 0, scale)
    p_rank = make_params(B, heads, T, H, W, d, mode, topk, cdf_p, cdf_cap_frac, t_cond, scale,
                         q_begin=rank * T_l, q_end=(rank + 1) * T_l)
    qp = ops.pool(p_local, q)
    kp = ops.pool(p_local, k)
    kp_all = comm.all_gather(kp)                 # [world][B, heads, nc_l, d]: shard layout
    row_ptr, col_idx = ops.select_pooled(p_rank, qp, kp_all, nc_l)

    out = lse = None
    k_cur, v_cur = k, v
    for s in range(world):
        j = (rank - s) % world                   # the shard held at this step
        handle = comm.start_shift([k_cur, v_cur]) if s + 1 < world else None
        srp, sci = ops.slice(row_ptr, col_idx, j * nc_l, (j + 1) * nc_l)
        o_part, l_part = ops.forward(p_local, q, k_cur, v_cur, srp, sci)
        if out is None:
            out, lse = o_part, l_part
        else:
            ops.merge(p_local, out, lse, o_part, l_part)
        if handle is not None:
            k_cur, v_cur = comm.finish_shift(handle)
    # the partial results were merged in fp32; round once, as the unsplit call does
    out = ops.finalize(p_local, out)
    ops.check()
    if return_csr:
        return out, lse, row_ptr, col_idx
    return out, lse


def _local_params(q, grid, scale):
    B, heads, N, d = q.shape
    T_l, H, W = grid
    if T_l % 4:
        raise ValueError("each rank must hold whole chunks: T_l must be a multiple of 4")
    if N != T_l * H * W:
        raise ValueError("q does not hold T_l*H*W tokens")
    nc_l = (T_l // 4) * ((H + 3) // 4) * ((W + 7) // 8)
    return make_params(B, heads, T_l, H, W, d, "topk", 1, 0.9, 0.25, 0, scale), nc_l


def ring_backward_partials(q, k, v, out, lse, dout, row_ptr, col_idx, grid, scale=0.0,
                           comm=None, ops=None):
    """The per-rank part of ring_backward, before the dK/dV reduction.

    Returns (dq_acc, dkv_parts): dq_acc fp32 [B, heads, N_l, d], the complete dQ of
    the local queries; dkv_parts fp32 [2, world, B, heads, N_l, d], this rank's
    contributions to dK (index 0) and dV (index 1) of every shard.
    """
    comm = comm or TorchComm()
    ops = ops or CudaOps()
    world, rank = comm.world, comm.rank
    p, nc_l = _local_params(q, grid, scale)
    dq_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dkv_parts = torch.empty((2, world) + tuple(k.shape), dtype=torch.float32, device=k.device)
    k_cur, v_cur = k, v
    for s in range(world):
        j = (rank - s) % world                   # the shard held at this step
        handle = comm.start_shift([k_cur, v_cur]) if s + 1 < world else None
        srp, sci = ops.slice(row_ptr, col_idx, j * nc_l, (j + 1) * nc_l)
        dq_p, dk_p, dv_p = ops.backward(p, q, k_cur, v_cur, out, lse, dout, srp, sci)
        ops.accumulate(p, dq_p, dq_acc, s == 0)
        ops.accumulate(p, dk_p, dkv_parts[0, j], True)
        ops.accumulate(p, dv_p, dkv_parts[1, j], True)
        if handle is not None:
            k_cur, v_cur = comm.finish_shift(handle)
    return dq_acc, dkv_parts


def ring_backward(q, k, v, out, lse, dout, row_ptr, col_idx, grid, scale=0.0, comm=None,
                  ops=None):
    """Gradients of ring_forward for this rank's upstream gradient dout.

    q, k, v, dout: this rank's shard [B, heads, T_l*H*W, d] bf16; out, lse: what
    ring_forward returned (the merged output and LSE over all shards); row_ptr,
    col_idx: the selection ring_forward returned with return_csr. Returns
    (dq, dk, dv) bf16 for the local queries and the local K/V shard: the rows of
    the unsplit sequence's gradients. Each shard's contribution comes out of
    bsa_backward in bf16; the contributions are summed in fp32 and the sums
    rounded once more.
    """
    comm = comm or TorchComm()
    ops = ops or CudaOps()
    p, _ = _local_params(q, grid, scale)
    dq_acc, dkv_parts = ring_backward_partials(q, k, v, out, lse, dout, row_ptr, col_idx, grid,
                                               scale, comm, ops)
    dk_acc = comm.reduce_scatter(dkv_parts[0])
    dv_acc = comm.reduce_scatter(dkv_parts[1])
    dq, dk, dv = ops.finalize(p, dq_acc), ops.finalize(p, dk_acc), ops.finalize(p, dv_acc)
    ops.check()
    return dq, dk, dv
