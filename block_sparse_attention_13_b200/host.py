"""Block sparse attention on host (pinned) buffers with the copies overlapped.

Every (batch, head) pair is an independent problem for pooling, selection and
attention, so a call on host buffers is split into groups of pairs that run
on several CUDA streams: while one group computes, the next group's Q, K, V
are copied in and the previous group's output is copied out (the two copy
directions use separate copy engines). Each group runs bsa_plan and
bsa_forward through the C ABI on its own slice; the results are the ones the
device-resident path gives.
"""
from __future__ import annotations

import torch

from . import (BSA_OK, BsaError, allocate, bsa_forward, bsa_plan, bsa_read_status, bsa_params,
               status_string)


def _params_for_group(p: bsa_params, heads: int) -> bsa_params:
    q = bsa_params.from_buffer_copy(p)
    q.B = 1
    q.heads = heads
    return q


class HostForward:
    """plan + forward for q, k, v in pinned host memory, [B, heads, T*H*W, d] bf16.

    group: (batch, head) pairs per group; streams: groups in flight. Whole
    slices are copied back, so with q_begin > 0 the host output of the skipped
    frames is overwritten with unspecified values (the C entry bsa_forward_host
    copies only the computed frames).
    """

    def __init__(self, p: bsa_params, group: int = 2, streams: int = 3, device="cuda"):
        self.p = p
        self.BH = p.B * p.heads
        self.group = max(1, min(group, self.BH))
        self.device = torch.device(device)
        N = p.T * p.H * p.W
        self.N, self.d = N, p.d
        self.groups = [(g0, min(self.group, self.BH - g0)) for g0 in range(0, self.BH, self.group)]
        self.params = {n: _params_for_group(p, n) for _, n in self.groups}
        self.slots = []
        for _ in range(max(1, min(streams, len(self.groups)))):
            shape = (self.group, N, p.d)
            self.slots.append(dict(
                stream=torch.cuda.Stream(device=self.device),
                q=torch.empty(shape, dtype=torch.bfloat16, device=self.device),
                k=torch.empty(shape, dtype=torch.bfloat16, device=self.device),
                v=torch.empty(shape, dtype=torch.bfloat16, device=self.device),
                out=torch.empty(shape, dtype=torch.bfloat16, device=self.device),
                plan=allocate(self.params[self.groups[0][1]], self.device)))

    def __call__(self, q_host, k_host, v_host, out_host):
        """Enqueue the whole call; the caller's current stream waits for it."""
        qh, kh, vh = (x.view(self.BH, self.N, self.d) for x in (q_host, k_host, v_host))
        oh = out_host.view(self.BH, self.N, self.d)
        cur = torch.cuda.current_stream(self.device)
        for s in self.slots:
            s["stream"].wait_stream(cur)
        for i, (g0, n) in enumerate(self.groups):
            s = self.slots[i % len(self.slots)]
            p = self.params[n]
            pl = s["plan"]
            st = s["stream"]
            with torch.cuda.stream(st):
                q, k, v, out = s["q"][:n], s["k"][:n], s["v"][:n], s["out"][:n]
                q.copy_(qh[g0:g0 + n], non_blocking=True)
                k.copy_(kh[g0:g0 + n], non_blocking=True)
                v.copy_(vh[g0:g0 + n], non_blocking=True)
                q4, k4, v4, o4 = (x.view(1, n, self.N, self.d) for x in (q, k, v, out))
                bsa_plan(p, q4, k4, pl.workspace, pl.row_ptr, pl.col_idx, stream=st)
                bsa_forward(p, q4, k4, v4, pl.row_ptr, pl.col_idx, pl.workspace, o4, stream=st)
                oh[g0:g0 + n].copy_(out, non_blocking=True)
        for s in self.slots:
            cur.wait_stream(s["stream"])
        return out_host

    def check(self):
        """Device status of every group's plan and forward (synchronises)."""
        for s in self.slots:
            rc = bsa_read_status(s["plan"].workspace, stream=s["stream"])
            if rc != BSA_OK:
                raise BsaError(rc, "device status: " + status_string(rc))
