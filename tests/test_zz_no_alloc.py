"""bsa_plan_noalloc: the plan entry point for callers that cannot allocate
device memory (a plug-in whose host engine owns all device memory and passes
only input and output tensors, or code that must not call cudaMalloc because
it can synchronise the device). Its scratch is a fixed array inside the
library, so its results must equal bsa_plan's with a caller workspace.

This file is collected last on purpose: the other GPU tests have run by the
time it does, and it must also pass alone in a fresh process.
"""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")

import block_sparse_attention_13_b200 as bsa  # noqa: E402

W = synth.WORKLOADS


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()


def _plans(wl):
    """CSR from bsa_plan (caller workspace) and from bsa_plan_noalloc."""
    q, k, _ = synth.make_qkv(wl)
    qd, kd = _dev(q), _dev(k)
    p = bsa.params_for(wl)
    ref = bsa.allocate(p)
    bsa.bsa_plan(p, qd, kd, ref.workspace, ref.row_ptr, ref.col_idx)
    assert bsa.bsa_read_status(ref.workspace) == bsa.BSA_OK
    rows, nnz = bsa.bsa_plan_sizes(p)
    # poison the outputs so stale values cannot pass for results
    row_ptr = torch.full((rows + 1,), -7, dtype=torch.int32, device="cuda")
    col_idx = torch.full((max(nnz, 1),), -7, dtype=torch.int32, device="cuda")
    bsa.bsa_plan_noalloc(p, qd, kd, row_ptr, col_idx)
    torch.cuda.synchronize()
    return ref, row_ptr, col_idx


@pytest.mark.gpu
def test_plan_noalloc_matches_plan_on_two_calls_in_a_row():
    # two consecutive calls with different workloads and modes share the one
    # scratch array: the second must not see the first's contents
    for wl in (W["tiny"].with_(B=2, heads=2, T=16, H=16, W=32, d=128, mode="cdf",
                               cdf_p=0.9, cdf_cap_frac=0.25, t_cond=8),
               W["480p"]):
        ref, rp, ci = _plans(wl)
        rp_ref = ref.row_ptr.cpu().numpy()
        nnz = int(rp_ref[-1])
        # selection is integer output: it must be bit-identical
        np.testing.assert_array_equal(rp.cpu().numpy(), rp_ref)
        np.testing.assert_array_equal(ci[:nnz].cpu().numpy(), ref.col_idx[:nnz].cpu().numpy())


@pytest.mark.gpu
def test_plan_noalloc_allocates_no_device_memory():
    """A warm call changes neither the device's free memory nor torch's
    allocator: the scratch is the library's fixed array, nothing else."""
    wl = W["tiny"].with_(heads=2, T=16, H=16, W=32, d=128, topk=5)
    q, k, _ = synth.make_qkv(wl)
    qd, kd = _dev(q), _dev(k)
    p = bsa.params_for(wl)
    rows, nnz = bsa.bsa_plan_sizes(p)
    row_ptr = torch.empty((rows + 1,), dtype=torch.int32, device="cuda")
    col_idx = torch.empty((max(nnz, 1),), dtype=torch.int32, device="cuda")
    bsa.bsa_plan_noalloc(p, qd, kd, row_ptr, col_idx)   # first call in this context
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(3):
        bsa.bsa_plan_noalloc(p, qd, kd, row_ptr, col_idx)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0


@pytest.mark.gpu
def test_plan_noalloc_rejects_plans_beyond_its_scratch():
    p = bsa.params_for(W["720p"])  # needs ~90 MB of scratch > 32 MiB
    assert bsa.bsa_workspace_size(p) > (32 << 20)
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    ri = torch.empty(16, dtype=torch.int32, device="cuda")
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_plan_noalloc(p, x, x, ri, ri)
    assert e.value.code == bsa.BSA_ERR_WORKSPACE_TOO_SMALL
