"""The host-buffer API (groups of (batch, head) pairs on several streams, copies
overlapping the kernels) gives exactly the device-resident path's output."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

import block_sparse_attention_13_b200 as bsa  # noqa: E402
from block_sparse_attention_13_b200.host import HostForward  # noqa: E402


@pytest.mark.parametrize("wl,group,streams", [
    (synth.WORKLOADS["tiny"].with_(B=2, heads=3, T=8, H=16, W=32, d=128, topk=5), 4, 3),
    (synth.WORKLOADS["tiny"].with_(B=1, heads=5, T=16, H=16, W=32, d=64, mode="cdf",
                                   cdf_p=0.9, cdf_cap_frac=0.25, t_cond=8), 2, 2),
    (synth.WORKLOADS["tiny"].with_(B=1, heads=2, T=6, H=10, W=20, d=64, topk=4), 1, 3),
])
def test_host_pipeline_equals_device_path(wl, group, streams):
    q, k, v = synth.make_qkv(wl)
    host = [torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in (q, k, v)]
    qd, kd, vd = (h.cuda() for h in host)
    p = bsa.params_for(wl)
    pl = bsa.plan(p, qd, kd)
    ref = bsa.forward(pl, qd, kd, vd)
    assert bsa.bsa_read_status(pl.workspace) == bsa.BSA_OK
    out_host = torch.full(ref.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    hf = HostForward(p, group=group, streams=streams)
    for _ in range(2):                       # reuse of the slots' buffers across calls
        hf(host[0], host[1], host[2], out_host)
        torch.cuda.synchronize()
        hf.check()
        assert torch.equal(out_host.view(torch.int16), ref.cpu().view(torch.int16))
