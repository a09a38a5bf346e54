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
