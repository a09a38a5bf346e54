"""Block sparse attention on host (pinned) buffers with the copies overlapped.

Every (batch, head) pair is an independent problem for pooling, selection and
attention ("LongCat-Video Technical Report", section "Block Sparse Attention
(BSA)": blocks, pooled scores and the kept set are per head), so a call on
host buffers is split into groups of pairs that run on several CUDA streams:
while one group computes, the next group's Q, K, V are copied in and the
previous group's output is copied out (the two copy directions use separate
copy engines). The whole pipeline -- copies, plan and forward kernels, stream
ordering -- runs inside the C ABI's ``bsa_forward_host``; this class only owns
the device staging workspace and the streams and passes them on.
"""
from __future__ import annotations

import torch

from . import (BSA_OK, BsaError, bsa_forward_host, bsa_forward_host_workspace_size,
               bsa_params, bsa_read_status, status_string)

MAX_SLOTS = 16


class HostForward:
    """plan + forward for q, k, v, out in pinned host memory, [B, heads, T*H*W, d] bf16.

    group: (batch, head) pairs per group; streams: groups in flight (1..16).
    Only the computed frames of the output are written: with q_begin > 0 the
    host output of the skipped frames keeps whatever the caller put there.
    """

    def __init__(self, p: bsa_params, group: int = 2, streams: int = 3, device="cuda"):
        self.p = p
        BH = p.B * p.heads
        self.group = max(1, min(int(group), BH))
        n_groups = -(-BH // self.group)
        self.n_slots = max(1, min(int(streams), n_groups, MAX_SLOTS))
        self.device = torch.device(device)
        size = bsa_forward_host_workspace_size(p, self.group, self.n_slots)
        if size == 0:
            raise BsaError(-1, "bsa_forward_host_workspace_size: parameters rejected")
        self.workspace = torch.empty(size, dtype=torch.uint8, device=self.device)
        self.workspace[:256].zero_()            # status block
        self.streams = [torch.cuda.Stream(device=self.device) for _ in range(self.n_slots)]

    def __call__(self, q_host, k_host, v_host, out_host):
        """Enqueue the whole call; the caller's current stream waits for it."""
        bsa_forward_host(self.p, q_host, k_host, v_host, out_host, self.group, self.streams,
                         self.workspace, stream=torch.cuda.current_stream(self.device))
        return out_host

    def check(self):
        """Device status of every group's plan and forward (synchronises)."""
        rc = bsa_read_status(self.workspace, stream=torch.cuda.current_stream(self.device))
        if rc != BSA_OK:
            raise BsaError(rc, "device status: " + status_string(rc))
