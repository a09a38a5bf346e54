"""Host-side checks of the Python entry points that wrap the C ABI: argument
validation happens before any device call, so these run without a GPU."""
import pytest
import torch

from block_sparse_attention_13_b200 import context_parallel as cp
from block_sparse_attention_13_b200.autograd import block_sparse_attention_train


def test_autograd_op_rejects_a_grid_that_does_not_match_the_tokens():
    q = torch.zeros(1, 2, 4 * 8 * 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        block_sparse_attention_train(q, q, q, (4, 8, 8))


def test_autograd_op_keeps_only_the_selection_for_the_backward(monkeypatch):
    """The op's host plumbing, with the library calls replaced by recorders: the
    backward gets the forward's own CSR tensors, the gradients it writes come
    back to q, k, v, and the plan's workspace is released once the forward
    has returned (only row_ptr and col_idx stay with the graph)."""
    import weakref
    from block_sparse_attention_13_b200 import Plan, autograd
    seen, held = {}, []

    def allocate(p, device="cuda"):
        pl = Plan(p, torch.zeros(4096, dtype=torch.uint8), torch.zeros(9, dtype=torch.int32),
                  torch.zeros(16, dtype=torch.int32))
        held.append(weakref.ref(pl.workspace))
        seen["csr"] = (pl.row_ptr, pl.col_idx)
        return pl

    def forward(p, q, k, v, row_ptr, col_idx, ws, out, lse, stream=None):
        out.copy_(v)
        lse.zero_()

    def backward(p, q, k, v, out, lse, dout, row_ptr, col_idx, ws, dq, dk, dv, stream=None):
        seen["bwd_csr"] = (row_ptr, col_idx)
        dq.fill_(1.0)
        dk.fill_(2.0)
        dv.copy_(dout)

    monkeypatch.setattr(autograd, "allocate", allocate)
    monkeypatch.setattr(autograd, "bsa_plan", lambda *a, **kw: None)
    monkeypatch.setattr(autograd, "bsa_forward", forward)
    monkeypatch.setattr(autograd, "bsa_backward", backward)
    monkeypatch.setattr(autograd, "bsa_read_status", lambda ws, stream=None: autograd.BSA_OK)
    monkeypatch.setattr(autograd, "backward_workspace",
                        lambda p, device="cuda": torch.zeros(256, dtype=torch.uint8))
    q, k, v = (torch.randn(1, 2, 4 * 8 * 16, 64).to(torch.bfloat16).requires_grad_(True)
               for _ in range(3))
    out = block_sparse_attention_train(q, k, v, (4, 8, 16), topk=2)
    assert held and held[0]() is None                  # the plan's workspace is gone
    g = torch.randn_like(out)
    out.backward(g)
    assert seen["bwd_csr"][0] is seen["csr"][0] and seen["bwd_csr"][1] is seen["csr"][1]
    assert torch.all(q.grad == 1) and torch.all(k.grad == 2) and torch.equal(v.grad, g)


def test_ring_shards_must_hold_whole_chunks():
    q = torch.zeros(1, 2, 6 * 8 * 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        cp._local_params(q, (6, 8, 16), 0.0)      # 6 frames: not a multiple of 4
    with pytest.raises(ValueError):
        cp._local_params(q, (4, 8, 16), 0.0)      # token count does not match the grid


def test_ring_local_params_and_chunk_count():
    q = torch.zeros(2, 3, 8 * 13 * 37, 128, dtype=torch.bfloat16)
    p, nc_l = cp._local_params(q, (8, 13, 37), 0.0)
    assert (p.B, p.heads, p.T, p.H, p.W, p.d) == (2, 3, 8, 13, 37, 128)
    assert nc_l == 2 * 4 * 5                       # ceil(13/4) x ceil(37/8) partial edge chunks


class _FakeComm:
    """Records the ring's shifts for one rank of a `world`-rank group."""

    def __init__(self, rank, world, shape):
        self.rank, self.world, self.shape, self.shifts = rank, world, shape, []

    def start_shift(self, tensors):
        self.shifts.append(len(self.shifts) + 1)
        return self.shifts[-1]

    def finish_shift(self, handle):
        # the shard received at shift `handle`, tagged with that number
        return [torch.full(self.shape, float(handle)), torch.full(self.shape, float(handle))]


class _RecordingOps:
    """Stands in for the device steps; records which shard each step used."""

    def __init__(self):
        self.calls = []

    def slice(self, rp, ci, lo, hi):
        self.calls.append(("slice", lo, hi))
        return rp, ci

    def backward(self, p, q, k, v, out, lse, dout, rp, ci):
        self.calls.append(("backward", int(k.flatten()[0])))
        z = torch.zeros(q.shape, dtype=torch.float32)
        return z, z, z

    def accumulate(self, p, part, acc, overwrite):
        self.calls.append(("acc", overwrite))


def test_ring_backward_visits_every_shard_once_in_ring_order():
    world, rank = 4, 1
    q = torch.zeros(1, 1, 4 * 8 * 16, 64, dtype=torch.bfloat16)
    comm, ops = _FakeComm(rank, world, q.shape), _RecordingOps()
    own = torch.full(q.shape, -1.0)
    dq, parts = cp.ring_backward_partials(q, own, own, None, None, None, None, None, (4, 8, 16),
                                          comm=comm, ops=ops)
    nc_l = 1 * 2 * 2
    slices = [c for c in ops.calls if c[0] == "slice"]
    # step s holds shard (rank - s) mod world
    assert [s[1] // nc_l for s in slices] == [(rank - s) % world for s in range(world)]
    keys = [c[1] for c in ops.calls if c[0] == "backward"]
    assert keys == [-1, 1, 2, 3]                   # own shard first, then what the ring delivers
    assert len(comm.shifts) == world - 1           # no shift after the last step
    acc = [c[1] for c in ops.calls if c[0] == "acc"]
    # dQ: overwrite on the first step only; dK and dV: each shard's slot written once
    assert acc == [True, True, True] + [False, True, True] * (world - 1)
    assert parts.shape == (2, world) + tuple(q.shape)


def test_product_modules_never_import_the_oracle():
    """The library's Python modules (binding, host pipeline, autograd op, ring driver)
    must not load the CPU oracle: it is test infrastructure, and a product path that
    reached it would be a CPU fallback."""
    import subprocess
    import sys
    code = ("import sys\n"
            "import block_sparse_attention_13_b200, block_sparse_attention_13_b200.host\n"
            "import block_sparse_attention_13_b200.autograd\n"
            "import block_sparse_attention_13_b200.context_parallel\n"
            "assert 'oracle' not in sys.modules, sorted(m for m in sys.modules if 'oracle' in m)\n")
    root = __file__.rsplit("/tests/", 1)[0]
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


# ------------------------------------------------------------------ tensor shapes and checks

import ctypes  # noqa: E402

import block_sparse_attention_13_b200 as bsa  # noqa: E402


@pytest.mark.parametrize("kw,want", [
    # 8x8x16 grid: 2x2x2 chunks of 128 tokens
    (dict(B=1, heads=2, T=8, H=8, W=16, d=64), dict(BH=2, N=1024, Nc=8, Nq=8, Nk=8, rows=16)),
    # partial edge chunks: ceil(10/4) x ceil(13/4) x ceil(37/8) = 3 x 4 x 5
    (dict(B=2, heads=3, T=10, H=13, W=37, d=128), dict(BH=6, N=4810, Nc=60, Nq=60, Nk=60,
                                                         rows=360)),
    # frames [4, 8) of 16: query chunks 4..7 of 16
    (dict(B=1, heads=2, T=16, H=8, W=16, d=64, q_begin=4, q_end=8),
     dict(BH=2, N=2048, Nc=16, Nq=4, Nk=16, rows=8)),
    # key chunks of (8,8,8): 2 x 1 x 2 of them over 4 x 2 x 2 query chunks
    (dict(B=1, heads=1, T=16, H=8, W=16, d=128, kchunk=(8, 8, 8)),
     dict(BH=1, N=2048, Nc=16, Nq=16, Nk=4, rows=16)),
])
def test_shape_info(kw, want):
    kw = dict(kw)
    p = bsa.make_params(kw.pop("B"), kw.pop("heads"), kw.pop("T"), kw.pop("H"), kw.pop("W"),
                        kw.pop("d"), **kw)
    s = bsa.bsa_shape_info(p)
    assert {k: getattr(s, k) for k in want} == want
    assert s.rows == bsa.bsa_plan_sizes(p)[0]


def test_shape_info_rejects_invalid_params():
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_shape_info(bsa.make_params(1, 1, 0, 8, 8, 64))
    assert e.value.code == bsa.BSA_ERR_SHAPE
    p = bsa.make_params(1, 1, 8, 8, 8, 64)
    assert bsa.lib().bsa_shape_info(ctypes.byref(p), None) == bsa.BSA_ERR_INVALID_ARG


def _raises(fn):
    with pytest.raises(bsa.BsaError) as e:
        fn()
    return e.value.code, str(e.value)


def test_binding_checks_tensors_before_the_library_sees_them():
    """Every mirror checks dtype, contiguity, size and device before it hands a
    pointer to the library (a CPU or undersized tensor would otherwise reach the
    kernels as a bad address). Here, without a GPU, a tensor of the right kind
    and size fails on the device check."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    p = bsa.make_params(1, 2, 8, 8, 16, 64)
    x = 2 * 1024 * 64
    q = torch.zeros(x, dtype=bf)
    rp, ci = torch.zeros(17, dtype=i32), torch.zeros(64, dtype=i32)
    ws = torch.zeros(bsa.bsa_workspace_size(p), dtype=torch.uint8)
    lse = torch.zeros(2 * 1024, dtype=f32)
    INV, SHAPE = bsa.BSA_ERR_INVALID_ARG, bsa.BSA_ERR_SHAPE

    assert _raises(lambda: bsa.bsa_plan(p, q.float(), q, ws, rp, ci))[0] == INV
    strided = torch.zeros(2 * x, dtype=bf)[::2]
    c, m = _raises(lambda: bsa.bsa_plan(p, strided, q, ws, rp, ci))
    assert c == INV and "contiguous" in m
    c, m = _raises(lambda: bsa.bsa_plan(p, q, q[:-1], ws, rp, ci))
    assert c == SHAPE and "k holds" in m
    c, m = _raises(lambda: bsa.bsa_plan(p, q, q, ws, rp[:-1], ci))
    assert c == SHAPE and "row_ptr" in m
    c, m = _raises(lambda: bsa.bsa_plan(p, q, q, ws, rp, ci))
    assert c == INV and "not a CUDA tensor" in m
    assert _raises(lambda: bsa.bsa_plan(p, q, q, "ws", rp, ci))[0] == INV

    c, m = _raises(lambda: bsa.bsa_forward(p, q, q, q, rp, ci, ws, q, lse[:-1]))
    assert c == SHAPE and "lse" in m
    assert _raises(lambda: bsa.bsa_forward(p, q, q, q, rp, ci.long(), ws, q))[0] == INV
    assert _raises(lambda: bsa.bsa_forward_ex(p, q, q, q, rp, ci, ws, q[:-8]))[0] == SHAPE
    c, m = _raises(lambda: bsa.bsa_forward(p, q, q, q, rp, ci, ws, q, lse))
    assert c == INV and "not a CUDA tensor" in m

    c, m = _raises(lambda: bsa.bsa_backward(p, q, q, q, q, lse, q, rp, ci, ws, q, q, q.float()))
    assert c == INV and "dv" in m
    c, m = _raises(lambda: bsa.bsa_backward(p, q, q, q, q, lse, q[:-1], rp, ci, ws, q, q, q))
    assert c == SHAPE and "dout" in m
    c, m = _raises(lambda: bsa.bsa_backward_ex(p, q, q, q, q, lse, q, rp, ci, ws, q[:-1], q, q,
                                               timeout_ns=1000, debug_flags=1))
    assert c == SHAPE and "bsa_backward_ex" in m and "dq" in m
    c, m = _raises(lambda: bsa.bsa_backward_ex(p, q, q, q, q, lse, q, rp, ci, ws, q, q, q))
    assert c == INV and "not a CUDA tensor" in m

    # the chunk-major side of the rearrangement holds Nc x 128 slots (partial chunks padded)
    pr = bsa.make_params(1, 1, 10, 13, 37, 64)
    tok, blk = 10 * 13 * 37 * 64, 60 * 128 * 64
    t_tok, t_blk = torch.zeros(tok, dtype=bf), torch.zeros(blk, dtype=bf)
    c, m = _raises(lambda: bsa.bsa_rearrange(pr, t_tok, t_tok))
    assert c == SHAPE and "out" in m
    c, m = _raises(lambda: bsa.bsa_rearrange(pr, t_tok, t_blk, inverse=True))
    assert c == SHAPE and "x holds" in m
    assert _raises(lambda: bsa.bsa_rearrange(pr, t_tok, t_blk))[0] == INV       # not CUDA

    c, m = _raises(lambda: bsa.bsa_pool(p, q, torch.zeros(2 * 8 * 64 - 1, dtype=f32)))
    assert c == SHAPE and "pooled" in m
    pooled = torch.zeros(2 * 8 * 64, dtype=f32)
    c, m = _raises(lambda: bsa.bsa_scores(p, pooled, pooled, torch.zeros(2 * 8 * 8 - 1, dtype=f32)))
    assert c == SHAPE and "S holds" in m
    c, m = _raises(lambda: bsa.bsa_select_pooled(p, pooled, pooled[:-1], ws, rp, ci))
    assert c == SHAPE and "kpool" in m
    c, m = _raises(lambda: bsa.bsa_csr_slice(rp, ci, 0, 4, ws, rp[:-1], ci))
    assert c == SHAPE and "out_row_ptr" in m
    c, m = _raises(lambda: bsa.bsa_lse_merge(p, q, lse, q, lse[:-1]))
    assert c == SHAPE and "lse_part" in m
    assert _raises(lambda: bsa.bsa_grad_accumulate(p, q, q))[0] == INV        # acc must be fp32
    acc = torch.zeros(x, dtype=f32)
    assert _raises(lambda: bsa.bsa_grad_finalize(p, acc[:-1], q))[0] == SHAPE
    assert _raises(lambda: bsa.bsa_read_status(torch.zeros(255, dtype=torch.uint8)))[0] == SHAPE
    assert _raises(lambda: bsa.bsa_selftest_timeout(torch.zeros(255, dtype=torch.uint8),
                                                    1000))[0] == SHAPE
    y = torch.zeros(8, dtype=f32)
    assert _raises(lambda: bsa.bsa_selftest_exp2(y, y[:-2], y))[0] == SHAPE


def test_noalloc_binding_relies_on_the_library_rejecting_large_plans():
    """bsa_plan_noalloc's wrapper checks tensor sizes only for plans that fit the
    library's scratch: larger ones must be rejected by the library itself, before
    any pointer is used. Pins that the library's limit is not above the binding's."""
    p = None
    for heads in range(1, 256):
        cand = bsa.make_params(1, heads, 16, 48, 80, 128)
        if bsa.bsa_workspace_size(cand) > bsa.NOALLOC_SCRATCH_BYTES:
            p = cand
            break
    assert p is not None
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: the call fails on the host
    rc = bsa.lib().bsa_plan_noalloc(ctypes.byref(p), fake, fake, fake, fake, 1 << 30, None)
    assert rc == bsa.BSA_ERR_WORKSPACE_TOO_SMALL
