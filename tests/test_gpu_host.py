"""The host-buffer entry point bsa_forward_host (groups of (batch, head) pairs on
several streams, copies overlapping the kernels, all inside the C ABI) gives
exactly the device-resident path's output, leaves the skipped frames of a
KV-cached step untouched, and handles groups that do not divide B*heads.
HostForward, the Python class over it, is checked the same way."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import ATT_MAX_ABS, ATT_MEAN_ABS, compare_attention

pytestmark = pytest.mark.gpu

import block_sparse_attention_13_b200 as bsa  # noqa: E402
from block_sparse_attention_13_b200.host import HostForward  # noqa: E402

T_ = synth.WORKLOADS["tiny"]

CASES = [
    # B*heads = 6 in groups of 4 (a ragged last group), 3 slots
    (T_.with_(B=2, heads=3, T=8, H=16, W=32, d=128, topk=5), 4, 3),
    # block-causal CDF, 5 pairs in groups of 2
    (T_.with_(B=1, heads=5, T=16, H=16, W=32, d=64, mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25,
              t_cond=8), 2, 2),
    # partial edge chunks, one pair per group
    (T_.with_(B=1, heads=2, T=6, H=10, W=20, d=64, topk=4), 1, 3),
    # KV-cached step: only frames >= 8 are computed, 3 pairs in groups of 2
    (T_.with_(B=1, heads=3, T=16, H=16, W=32, d=128, mode="cdf", t_cond=8, q_begin=8), 2, 2),
    # key chunks of 512 tokens, one slot
    (T_.with_(B=1, heads=3, T=8, H=16, W=32, d=128, topk=2, kchunk=(8, 8, 8)), 2, 1),
    # 64-token query and key chunks
    (T_.with_(B=1, heads=3, T=8, H=16, W=20, d=64, topk=5, qchunk=(4, 4, 4), kchunk=(4, 4, 4)),
     2, 2),
]


def _pinned(x):
    return torch.from_numpy(x).view(torch.bfloat16).pin_memory()


def _device_reference(wl, host):
    """bsa_plan + bsa_forward on device copies; O of skipped frames = 3.0."""
    qd, kd, vd = (h.cuda() for h in host)
    p = bsa.params_for(wl)
    pl = bsa.plan(p, qd, kd)
    ref = torch.full_like(qd, 3.0)
    bsa.forward(pl, qd, kd, vd, out=ref)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    return p, ref.cpu()


@pytest.mark.parametrize("wl,group,slots", CASES)
def test_forward_host_equals_device_path(wl, group, slots):
    q, k, v = synth.make_qkv(wl)
    host = [_pinned(x) for x in (q, k, v)]
    p, ref = _device_reference(wl, host)
    ws = torch.zeros(bsa.bsa_forward_host_workspace_size(p, group, slots), dtype=torch.uint8,
                     device="cuda")
    streams = [torch.cuda.Stream() for _ in range(slots)]
    out_host = torch.full(ref.shape, 3.0, dtype=torch.bfloat16).pin_memory()
    for _ in range(2):                       # the slots' staging is reused across calls
        bsa.bsa_forward_host(p, host[0], host[1], host[2], out_host, group, streams, ws)
        torch.cuda.current_stream().synchronize()
        assert bsa.bsa_read_status(ws) == bsa.BSA_OK
        # bit-identical: the same kernels on the same inputs
        assert torch.equal(out_host.view(torch.int16), ref.view(torch.int16))
    if wl.q_begin:
        HW = wl.H * wl.W
        assert torch.all(out_host[:, :, : wl.q_begin * HW] == 3.0)   # never written


def test_forward_host_against_the_oracle():
    """Independent of the device path: the host-buffer output of a block-causal
    CDF grid against the fp64 oracle on the rows it computed."""
    wl, group, slots = CASES[1]
    q, k, v = synth.make_qkv(wl)
    host = [_pinned(x) for x in (q, k, v)]
    p = bsa.params_for(wl)
    hf = HostForward(p, group=group, streams=slots)
    out_host = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    hf(host[0], host[1], host[2], out_host)
    torch.cuda.synchronize()
    hf.check()
    scale = 1.0 / math.sqrt(wl.d)
    rp, ci, _ = oracle.plan(q, k, wl.T, wl.H, wl.W, scale, wl.mode, wl.topk, wl.cdf_p,
                            wl.cdf_cap_frac, wl.t_cond, fp32=True)
    rows = np.arange(wl.rows)
    o_out, _ = oracle.attend(q, k, v, wl.T, wl.H, wl.W, scale, rp, ci, rows)
    flat = out_host.float().numpy().reshape(wl.B * wl.heads, wl.N, wl.d)
    g = np.stack([flat[r // wl.Nc][oracle.chunk_tokens(wl.T, wl.H, wl.W, r % wl.Nc)]
                  for r in rows])
    mx, mean = compare_attention(g, o_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("wl,group,slots", CASES[:3])
def test_host_forward_class_equals_device_path(wl, group, slots):
    q, k, v = synth.make_qkv(wl)
    host = [_pinned(x) for x in (q, k, v)]
    p, ref = _device_reference(wl, host)
    out_host = torch.full(ref.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    hf = HostForward(p, group=group, streams=slots)
    for _ in range(2):
        hf(host[0], host[1], host[2], out_host)
        torch.cuda.synchronize()
        hf.check()
        assert torch.equal(out_host.view(torch.int16), ref.view(torch.int16))


def test_forward_host_orders_the_callers_stream():
    """Work queued on the caller's stream before the call is seen by the slot
    streams (the inputs are written there just before), and work queued after it
    sees the finished output."""
    wl, group, slots = CASES[0]
    q, k, v = synth.make_qkv(wl)
    host = [_pinned(x) for x in (q, k, v)]
    p, ref = _device_reference(wl, host)
    ws = torch.zeros(bsa.bsa_forward_host_workspace_size(p, group, slots), dtype=torch.uint8,
                     device="cuda")
    streams = [torch.cuda.Stream() for _ in range(slots)]
    main = torch.cuda.Stream()
    out_host = torch.zeros(ref.shape, dtype=torch.bfloat16).pin_memory()
    q_late = torch.zeros_like(host[0]).pin_memory()
    q_dev = host[0].cuda()
    with torch.cuda.stream(main):
        torch.cuda._sleep(20_000_000)                       # keep `main` busy for a while
        q_late.copy_(q_dev, non_blocking=True)              # the input lands late on `main`
        bsa.bsa_forward_host(p, q_late, host[1], host[2], out_host, group, streams, ws,
                             stream=main)
        dev_copy = out_host.cuda(non_blocking=True)         # queued after the call
    main.synchronize()
    assert torch.equal(out_host.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(dev_copy.cpu().view(torch.int16), ref.view(torch.int16))
