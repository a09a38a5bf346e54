"""Block sparse attention as a differentiable PyTorch op (training).

The forward runs bsa_plan (block selection) and bsa_forward with the
log-sum-exp; the backward runs bsa_backward on the same selection, the saved
output and log-sum-exp. The selection itself has no gradient ("LongCat-Video
Technical Report", section "Block Sparse Attention (BSA)": the block mask is
computed from pooled scores and applied as -inf logits). Every step runs in the
library's kernels through the C ABI; this module only holds the tensors between
the two passes.
"""
from __future__ import annotations

import torch

from . import (BSA_OK, BsaError, allocate, backward_workspace, bsa_backward, bsa_forward, bsa_plan,
               bsa_read_status, make_params, status_string)


def _check(ws):
    rc = bsa_read_status(ws)
    if rc != BSA_OK:
        raise BsaError(rc, "device status: " + status_string(rc))


class _BlockSparseAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, p):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        pl = allocate(p, q.device)
        bsa_plan(p, q, k, pl.workspace, pl.row_ptr, pl.col_idx)
        out = torch.empty_like(q)
        B, heads, N, _ = q.shape
        lse = torch.empty((B, heads, N), dtype=torch.float32, device=q.device)
        bsa_forward(p, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out, lse)
        _check(pl.workspace)
        ctx.p = p
        # only the selection is kept for the backward, not the plan's workspace
        # (tens to hundreds of MB per call on video grids)
        ctx.csr = (pl.row_ptr, pl.col_idx)
        ctx.save_for_backward(q, k, v, out, lse)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        row_ptr, col_idx = ctx.csr
        ws = backward_workspace(ctx.p, q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bsa_backward(ctx.p, q, k, v, out, lse, dout.contiguous(), row_ptr, col_idx, ws, dq, dk, dv)
        _check(ws)
        return dq, dk, dv, None


def block_sparse_attention_train(q, k, v, grid, topk=None, mode="topk", cdf_p=0.9,
                                 cdf_cap_frac=0.25, t_cond=0, scale=0.0, chunk=(4, 4, 8),
                                 kchunk=(0, 0, 0)):
    """Differentiable block sparse attention of q, k, v [B, heads, T*H*W, d] bf16
    (CUDA tensors, tokens in [T,H,W] order). grid = (T, H, W); chunk = the query
    chunk shape, (4, 4, 8) or (4, 4, 4); kchunk = the key chunk shape (0 = the query
    chunk's); topk defaults to 1/16 of the key chunks. Returns out; out.backward(...)
    fills q.grad, k.grad and v.grad through bsa_backward."""
    B, heads, N, d = q.shape
    T, H, W = grid
    if T * H * W != N:
        raise ValueError("grid does not match the token count")
    if topk is None:
        kc = tuple(c if c else q_ for c, q_ in zip(kchunk, chunk))
        topk = max(1, (-(-T // kc[0]) * -(-H // kc[1]) * -(-W // kc[2])) // 16)
    p = make_params(B, heads, T, H, W, d, mode, topk, cdf_p, cdf_cap_frac, t_cond, scale,
                    kchunk=kchunk, chunk=chunk)
    return _BlockSparseAttention.apply(q, k, v, p)
