"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/bsa.h declares, and its host-side argument checks return the
documented status codes before any CUDA call."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_13_b200 as bsa
from block_sparse_attention_13_b200 import build as bsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    bsa_build.build()
    return bsa.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "bsa.h")).read()
    return re.findall(r"^BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", text, flags=re.M)


def test_header_declares_binding_names():
    names = declared_symbols()
    assert len(names) == len(set(names)) >= 12
    assert set(names) == set(bsa.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {bsa.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(declared_symbols())


def test_version_and_strings(L):
    assert bsa.bsa_version() == 302
    for code in range(0, 10):
        s = bsa.status_string(code)
        assert s and s != "unknown status"
    assert bsa.status_string(99) == "unknown status"


def P(**kw):
    base = dict(B=1, heads=2, T=4, H=8, W=16, d=64, mode="topk", topk=2)
    base.update(kw)
    return bsa.make_params(**base)


def rc_sizes(p):
    rows, nnz = ctypes.c_int64(), ctypes.c_int64()
    return bsa.lib().bsa_plan_sizes(ctypes.byref(p), ctypes.byref(rows), ctypes.byref(nnz)), \
        rows.value, nnz.value


def test_plan_sizes_topk_and_cdf(L):
    rc, rows, nnz = rc_sizes(P())
    assert (rc, rows, nnz) == (0, 8, 16)
    # 720p-like: 32 heads x 720 chunks, keep 45
    rc, rows, nnz = rc_sizes(P(heads=32, T=24, H=48, W=80, d=128, topk=45))
    assert (rc, rows, nnz) == (0, 23040, 23040 * 45)
    # block-causal CDF: 240 condition rows capped at 60, 480 noisy rows capped at 180
    rc, rows, nnz = rc_sizes(P(B=2, heads=32, T=24, H=48, W=80, d=128, mode="cdf", t_cond=8))
    assert (rc, rows, nnz) == (0, 46080, 64 * (240 * 60 + 480 * 180))
    # block-causal top-k clamps condition rows to the 240 condition chunks
    rc, rows, nnz = rc_sizes(P(heads=1, T=24, H=48, W=80, d=128, topk=300, t_cond=8))
    assert (rc, nnz) == (0, 240 * 240 + 480 * 300)


def test_plan_sizes_topk_cdf_combination(L):
    # per row at most min(k, cap): 720 noisy chunks, cap 180, k = 45
    rc, rows, nnz = rc_sizes(P(heads=32, T=24, H=48, W=80, d=128, mode="topk_cdf", topk=45,
                               cdf_p=0.1))
    assert (rc, rows, nnz) == (0, 23040, 23040 * 45)
    # k above the cap: the cap bounds
    rc, rows, nnz = rc_sizes(P(heads=1, T=24, H=48, W=80, d=128, mode="topk_cdf", topk=300,
                               cdf_p=0.9, t_cond=8))
    assert (rc, nnz) == (0, 240 * 60 + 480 * 180)
    ws_c = bsa.bsa_workspace_size(P(heads=1, T=24, H=48, W=80, d=128, mode="cdf"))
    ws_tc = bsa.bsa_workspace_size(P(heads=1, T=24, H=48, W=80, d=128, mode="topk_cdf", topk=45))
    assert ws_tc < ws_c   # padded rows hold min(k, cap) = 45 instead of 180 entries


def test_plan_sizes_partial_edge_chunks(L):
    # the actual 720p token grid 24 x 45 x 80: ceil(45/4) = 12 chunk rows, 720 chunks
    rc, rows, nnz = rc_sizes(P(heads=32, T=24, H=45, W=80, d=128, topk=45))
    assert (rc, rows, nnz) == (0, 32 * 720, 32 * 720 * 45)
    # 5 x 7 x 9 tokens: 2 x 2 x 2 chunks, all partial
    rc, rows, nnz = rc_sizes(P(heads=1, T=5, H=7, W=9, topk=3))
    assert (rc, rows, nnz) == (0, 8, 24)
    # a single token
    assert rc_sizes(P(heads=1, T=1, H=1, W=1, topk=1))[:2] == (0, 1)


def test_plan_sizes_key_chunks(L):
    # 720p-like grid with (8,8,8) key chunks (2 x 2 x 1 boxes): 180 key chunks, keep 11 -> 44 boxes
    rc, rows, nnz = rc_sizes(P(heads=32, T=24, H=48, W=80, d=128, topk=11, kchunk=(8, 8, 8)))
    assert (rc, rows, nnz) == (0, 23040, 23040 * 11 * 4)
    # (4,8,8) (2 boxes) on the block-causal grid: 360 key chunks, 120 of them condition
    # chunks; condition rows keep min(k, 120)
    rc, rows, nnz = rc_sizes(P(heads=1, T=24, H=48, W=80, d=128, topk=150, t_cond=8,
                               kchunk=(4, 8, 8)))
    assert (rc, nnz) == (0, (240 * 120 + 480 * 150) * 2)
    ws = bsa.bsa_workspace_size(P(heads=32, T=24, H=48, W=80, d=128, topk=11, kchunk=(8, 8, 8)))
    kpool, scores = 32 * 180 * 128 * 4, 32 * 720 * 180 * 4
    assert ws >= 256 + 32 * 720 * 128 * 4 + kpool + scores


@pytest.mark.parametrize("kchunk,code", [((4, 4, 12), bsa.BSA_ERR_UNSUPPORTED),
                                         ((6, 4, 8), bsa.BSA_ERR_UNSUPPORTED),
                                         ((8, 8, 16), 0), ((16, 8, 16), bsa.BSA_ERR_UNSUPPORTED),
                                         ((-4, 4, 8), bsa.BSA_ERR_UNSUPPORTED)])
def test_key_chunk_shape_validation(L, kchunk, code):
    assert rc_sizes(P(T=16, H=16, W=32, kchunk=kchunk))[0] == code


def test_plan_sizes_64_token_chunks(L):
    # 720p-like grid in 64-token chunks: 6 x 12 x 20 = 1,440 query chunks per head
    q64 = dict(heads=32, T=24, H=48, W=80, d=128, chunk=(4, 4, 4))
    rc, rows, nnz = rc_sizes(P(topk=90, **q64))
    assert (rc, rows, nnz) == (0, 32 * 1440, 32 * 1440 * 90)
    # with 128-token key chunks: 720 key chunks
    rc, rows, nnz = rc_sizes(P(topk=45, kchunk=(4, 4, 8), **q64))
    assert (rc, rows, nnz) == (0, 32 * 1440, 32 * 1440 * 45)
    # block-causal CDF: 480 condition chunks capped at 120, 960 noisy capped at 360
    rc, rows, nnz = rc_sizes(P(mode="cdf", t_cond=8, **q64))
    assert (rc, rows, nnz) == (0, 32 * 1440, 32 * (480 * 120 + 960 * 360))
    # the plan's workspace also holds the forward's CSR over (4,4,8) boxes: a row per
    # query box (720 per head) and at most the chunk CSR's entries
    p = P(topk=90, **q64)
    base = 256 + 2 * 32 * 1440 * 128 * 4 + 32 * 1440 * 1440 * 4
    assert bsa.bsa_workspace_size(p) >= base + 32 * 720 * 8 + 32 * 1440 * 90 * 5
    si = bsa.bsa_shape_info(p)
    assert (si.Nc, si.Nq, si.Nk, si.rows) == (1440, 1440, 1440, 32 * 1440)
    # W = 20: 5 chunk columns of 4 (boxes: 3, the last holding one chunk)
    assert rc_sizes(P(heads=1, T=4, H=4, W=20, topk=2, chunk=(4, 4, 4)))[:2] == (0, 5)
    # partial chunks: W = 10 -> 3 chunk columns, the last of 2 tokens
    assert rc_sizes(P(heads=1, T=4, H=4, W=10, topk=2, chunk=(4, 4, 4)))[:2] == (0, 3)


@pytest.mark.parametrize("kw,code", [
    (dict(chunk=(4, 4, 4)), 0),
    (dict(chunk=(4, 4, 4), kchunk=(4, 4, 8)), 0),
    (dict(chunk=(4, 4, 4), kchunk=(4, 8, 8)), bsa.BSA_ERR_UNSUPPORTED),   # not (4,4,4)/(4,4,8)
    (dict(chunk=(4, 4, 4), kchunk=(8, 4, 4)), bsa.BSA_ERR_UNSUPPORTED),
    (dict(chunk=(4, 4, 4), q_begin=4), bsa.BSA_ERR_UNSUPPORTED),          # every row computed
    (dict(chunk=(4, 4, 4), q_end=8), bsa.BSA_ERR_UNSUPPORTED),
    (dict(chunk=(4, 4, 2)), bsa.BSA_ERR_UNSUPPORTED),
    (dict(chunk=(4, 4, 16)), bsa.BSA_ERR_UNSUPPORTED),
    (dict(chunk=(8, 4, 4)), bsa.BSA_ERR_UNSUPPORTED),
])
def test_query_chunk_shape_validation(L, kw, code):
    assert rc_sizes(P(T=16, H=16, W=32, **kw))[0] == code


def test_64_token_chunks_limits_and_entries_that_take_128_token_chunks(L):
    # chunks per (batch, head) are limited to 2,048: the long grid in 64-token chunks
    # (14 x 12 x 20 = 3,360) is not supported
    assert rc_sizes(P(T=56, H=48, W=80, d=128, topk=5, chunk=(4, 4, 4)))[0] == \
        bsa.BSA_ERR_UNSUPPORTED
    p = P(T=16, H=16, W=32, chunk=(4, 4, 4))
    x = vp(FAKE)
    # the backward works on (4,4,8) boxes: its workspace holds the box CSR and the
    # backward layout over boxes, and it is checked before any CUDA call
    p128 = P(T=16, H=16, W=32)
    ws = L.bsa_backward_workspace_size(ctypes.byref(p))
    assert ws > L.bsa_backward_workspace_size(ctypes.byref(p128)) > 0
    assert L.bsa_backward(ctypes.byref(p), x, x, x, x, x, x, x, x, 64, x, ws - 1, x, x, x,
                          None) == bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    assert L.bsa_rearrange(ctypes.byref(p), x, x, 0, None) == bsa.BSA_ERR_UNSUPPORTED
    assert L.bsa_select_pooled(ctypes.byref(p), x, x, 0, x, 1 << 30, x, x, 1 << 20, None) == \
        bsa.BSA_ERR_UNSUPPORTED
    # the forward needs the plan's workspace (it builds the box CSR there)
    ws = bsa.bsa_workspace_size(p)
    assert L.bsa_forward(ctypes.byref(p), x, x, x, x, x, 64, x, ws - 1, x, None, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL


def test_key_chunk_needs_t_cond_multiple(L):
    assert rc_sizes(P(T=16, H=16, W=32, t_cond=4, kchunk=(8, 4, 8)))[0] == bsa.BSA_ERR_SHAPE
    assert rc_sizes(P(T=16, H=16, W=32, t_cond=8, kchunk=(8, 4, 8)))[0] == 0


def test_plan_sizes_kv_cached_step(L):
    # causal_cdf with only the noisy queries (frames >= 8): 480 of 720 rows per head
    rc, rows, nnz = rc_sizes(P(B=2, heads=32, T=24, H=48, W=80, d=128, mode="cdf", t_cond=8,
                               q_begin=8))
    assert (rc, rows, nnz) == (0, 64 * 480, 64 * 480 * 180)
    # q_begin inside the condition frames: 120 condition rows (k clamped to 240) + 480 noisy
    rc, rows, nnz = rc_sizes(P(heads=1, T=24, H=48, W=80, d=128, topk=300, t_cond=8, q_begin=4))
    assert (rc, rows, nnz) == (0, 600, 120 * 240 + 480 * 300)
    p = P(heads=32, T=24, H=48, W=80, d=128, topk=45, q_begin=8)
    assert bsa.bsa_workspace_size(p) == 256 + 32 * 480 * 128 * 4 + 32 * 720 * 128 * 4 + \
        32 * 480 * 720 * 4


@pytest.mark.parametrize("kw,code", [
    (dict(q_begin=2), bsa.BSA_ERR_SHAPE),
    (dict(q_begin=4), bsa.BSA_ERR_SHAPE),     # q_begin must leave at least one frame (T = 4)
    (dict(q_begin=-4), bsa.BSA_ERR_SHAPE),
    (dict(T=0), bsa.BSA_ERR_SHAPE),
    (dict(H=-4), bsa.BSA_ERR_SHAPE),
    (dict(W=0), bsa.BSA_ERR_SHAPE),
    (dict(B=0), bsa.BSA_ERR_SHAPE),
    (dict(d=96), bsa.BSA_ERR_UNSUPPORTED),
    (dict(t_cond=2), bsa.BSA_ERR_SHAPE),
    (dict(t_cond=8), bsa.BSA_ERR_SHAPE),
    (dict(topk=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(mode="topk_cdf", topk=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(mode="topk_cdf", cdf_p=0.0), bsa.BSA_ERR_INVALID_ARG),
    (dict(mode="cdf", cdf_p=0.0), bsa.BSA_ERR_INVALID_ARG),
    (dict(mode="cdf", cdf_p=1.5), bsa.BSA_ERR_INVALID_ARG),
    (dict(mode="cdf", cdf_cap_frac=0.0), bsa.BSA_ERR_INVALID_ARG),
    (dict(scale=-1.0), bsa.BSA_ERR_INVALID_ARG),
    (dict(T=4 * 64, H=4 * 8, W=8 * 8), bsa.BSA_ERR_UNSUPPORTED),  # Nc = 4096 > 2048
])
def test_invalid_params(L, kw, code):
    p = P(**kw)
    assert rc_sizes(p)[0] == code
    assert bsa.lib().bsa_workspace_size(ctypes.byref(p)) == 0


def test_size_limits_at_their_boundaries(L):
    # 2,048 chunks per (batch, head) is the largest grid; one more chunk axis step is rejected
    assert rc_sizes(P(T=4 * 32, H=4 * 8, W=8 * 8))[0] == 0                  # Nc = 2048
    assert rc_sizes(P(T=4 * 32, H=4 * 8, W=8 * 8 + 1))[0] == bsa.BSA_ERR_UNSUPPORTED
    # B * heads <= 65535
    assert rc_sizes(P(B=5, heads=13107, T=4, H=4, W=8))[0] == 0             # 65535
    assert rc_sizes(P(B=2, heads=32768, T=4, H=4, W=8))[0] == bsa.BSA_ERR_UNSUPPORTED
    # CSR offsets are int32: rows * Nc <= 2^31 - 1 (rows = heads * 2048 here)
    assert rc_sizes(P(B=1, heads=511, T=4 * 32, H=4 * 8, W=8 * 8))[0] == 0
    assert rc_sizes(P(B=1, heads=512, T=4 * 32, H=4 * 8, W=8 * 8))[0] == \
        bsa.BSA_ERR_UNSUPPORTED                                               # exactly 2^31


def test_chunk_shapes_other_than_448_and_444_unsupported(L):
    for shape in ((4, 4, 6), (4, 8, 8), (2, 4, 8), (4, 4, 12)):
        p = P()
        p.chunk_t, p.chunk_h, p.chunk_w = shape
        assert rc_sizes(p)[0] == bsa.BSA_ERR_UNSUPPORTED, shape


def test_workspace_size_layout(L):
    p = P(heads=32, T=24, H=48, W=80, d=128, topk=45)
    n = bsa.bsa_workspace_size(p)
    pool = 32 * 720 * 128 * 4
    assert n == 256 + 2 * pool + 32 * 720 * 720 * 4
    pc = P(B=2, heads=32, T=24, H=48, W=80, d=128, mode="cdf", t_cond=8)
    assert bsa.bsa_workspace_size(pc) > n


FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced


def vp(x):
    return ctypes.c_void_p(x)


def test_plan_host_checks_before_any_cuda_call(L):
    p = P()
    ws = bsa.bsa_workspace_size(p)
    f = L.bsa_plan
    pp = ctypes.byref(p)
    assert f(None, vp(FAKE), vp(FAKE), vp(FAKE), ws, vp(FAKE), vp(FAKE), 16, None) == \
        bsa.BSA_ERR_INVALID_ARG
    assert f(pp, None, vp(FAKE), vp(FAKE), ws, vp(FAKE), vp(FAKE), 16, None) == \
        bsa.BSA_ERR_INVALID_ARG
    assert f(pp, vp(FAKE + 8), vp(FAKE), vp(FAKE), ws, vp(FAKE), vp(FAKE), 16, None) == \
        bsa.BSA_ERR_ALIGNMENT
    assert f(pp, vp(FAKE), vp(FAKE), vp(FAKE), ws - 1, vp(FAKE), vp(FAKE), 16, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    assert f(pp, vp(FAKE), vp(FAKE), vp(FAKE), ws, vp(FAKE), vp(FAKE), 15, None) == \
        bsa.BSA_ERR_CAPACITY


def test_forward_host_checks_before_any_cuda_call(L):
    p = P()
    f = L.bsa_forward
    pp = ctypes.byref(p)
    a = [vp(FAKE)] * 5
    assert f(pp, *a, 16, vp(FAKE), 256, None, None, None) == bsa.BSA_ERR_INVALID_ARG
    assert f(pp, vp(FAKE), vp(FAKE), vp(FAKE + 4), vp(FAKE), vp(FAKE), 16, vp(FAKE), 256,
             vp(FAKE), None, None) == bsa.BSA_ERR_ALIGNMENT
    assert f(pp, *a, 16, vp(FAKE), 255, vp(FAKE), None, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    assert f(pp, *a, -1, vp(FAKE), 256, vp(FAKE), None, None) == bsa.BSA_ERR_INVALID_ARG
    # int32 CSR arrays and the fp32 lse are read element by element: 4-byte alignment
    x, odd = vp(FAKE), vp(FAKE + 2)
    assert f(pp, x, x, x, odd, x, 16, x, 256, x, None, None) == bsa.BSA_ERR_ALIGNMENT
    assert f(pp, x, x, x, x, odd, 16, x, 256, x, None, None) == bsa.BSA_ERR_ALIGNMENT
    assert f(pp, x, x, x, x, x, 16, x, 256, x, odd, None) == bsa.BSA_ERR_ALIGNMENT


def test_backward_workspace_size_layout(L):
    p = P(heads=32, T=24, H=48, W=80, d=128, topk=45)
    rows, cols, words = 32 * 720, 32 * 720, 23
    r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    expect = 256 + r256(rows * 256 * 4) + r256(cols * words * 4) + 2 * r256(cols * 4) + \
        r256((cols + 1) * 4) + r256(rows * 720 * 4)
    assert bsa.bsa_backward_workspace_size(p) == expect
    assert bsa.lib().bsa_backward_workspace_size(ctypes.byref(P(T=0))) == 0


@pytest.mark.parametrize("entry", ["bsa_backward", "bsa_backward_ex"])
def test_backward_host_checks_before_any_cuda_call(L, entry):
    p = P()
    ws = bsa.bsa_backward_workspace_size(p)
    if entry == "bsa_backward":
        f = L.bsa_backward
    else:  # the same checks, with a wait limit and debug flags before the stream
        f = lambda *a: L.bsa_backward_ex(*a[:-1], 0, 1, a[-1])
    pp = ctypes.byref(p)
    x = vp(FAKE)
    # q, k, v, out, lse, dout, row_ptr, col_idx, cap, ws, ws_bytes, dq, dk, dv, stream
    assert f(pp, x, x, x, x, None, x, x, x, 16, x, ws, x, x, x, None) == bsa.BSA_ERR_INVALID_ARG
    assert f(pp, x, x, x, x, x, x, x, x, -1, x, ws, x, x, x, None) == bsa.BSA_ERR_INVALID_ARG
    assert f(pp, x, x, x, x, x, x, x, x, 16, x, ws, x, vp(FAKE + 8), x, None) == \
        bsa.BSA_ERR_ALIGNMENT
    assert f(pp, x, x, x, x, vp(FAKE + 2), x, x, x, 16, x, ws, x, x, x, None) == \
        bsa.BSA_ERR_ALIGNMENT
    assert f(pp, x, x, x, x, x, x, x, x, 16, x, ws - 1, x, x, x, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    odd = vp(FAKE + 2)
    assert f(pp, x, x, x, x, x, x, odd, x, 16, x, ws, x, x, x, None) == bsa.BSA_ERR_ALIGNMENT
    assert f(pp, x, x, x, x, x, x, x, odd, 16, x, ws, x, x, x, None) == bsa.BSA_ERR_ALIGNMENT
    assert f(ctypes.byref(P(T=0)), x, x, x, x, x, x, x, x, 16, x, ws, x, x, x, None) == \
        bsa.BSA_ERR_SHAPE


def test_no_cpu_fallback_without_a_gpu(L):
    """With valid arguments and no usable GPU the call fails loudly."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = P()
    ws = bsa.bsa_workspace_size(p)
    rc = L.bsa_plan(ctypes.byref(p), vp(FAKE), vp(FAKE), vp(FAKE), ws, vp(FAKE), vp(FAKE), 16,
                    None)
    assert rc == bsa.BSA_ERR_CUDA
    x = vp(FAKE)
    bws = bsa.bsa_backward_workspace_size(p)
    assert L.bsa_backward_ex(ctypes.byref(p), x, x, x, x, x, x, x, x, 16, x, bws, x, x, x,
                             20_000_000, 3, None) == bsa.BSA_ERR_CUDA
    with pytest.raises(bsa.BsaError):
        bsa.bsa_plan_sizes(P(T=0))


def test_unknown_selection_mode_rejected(L):
    p = P()
    p.mode = 3
    assert rc_sizes(p)[0] == bsa.BSA_ERR_INVALID_ARG


def test_context_parallel_entries_host_checks(L):
    x = vp(FAKE)
    # csr slice: workspace size, argument checks
    assert bsa.bsa_csr_slice_workspace_size(100) == 256 + 512
    assert L.bsa_csr_slice_workspace_size(-1) == 0
    ws = bsa.bsa_csr_slice_workspace_size(10)
    f = L.bsa_csr_slice
    assert f(10, x, x, 16, 5, 2, x, ws, x, x, 16, None) == bsa.BSA_ERR_INVALID_ARG   # hi < lo
    assert f(10, x, x, 16, -1, 2, x, ws, x, x, 16, None) == bsa.BSA_ERR_INVALID_ARG
    assert f(10, x, x, 16, 0, 2, vp(FAKE + 8), ws, x, x, 16, None) == bsa.BSA_ERR_ALIGNMENT
    assert f(10, x, x, 16, 0, 2, x, ws - 1, x, x, 16, None) == bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    odd = vp(FAKE + 2)
    for i in range(4):   # row_ptr, col_idx, out_row_ptr, out_col_idx
        arrs = [x, x, x, x]
        arrs[i] = odd
        assert f(10, arrs[0], arrs[1], 16, 0, 2, x, ws, arrs[2], arrs[3], 16, None) == \
            bsa.BSA_ERR_ALIGNMENT
    # lse merge
    p = P()
    assert L.bsa_lse_merge(ctypes.byref(p), x, None, x, x, None) == bsa.BSA_ERR_INVALID_ARG
    assert L.bsa_lse_merge(ctypes.byref(p), x, vp(FAKE + 2), x, x, None) == \
        bsa.BSA_ERR_ALIGNMENT
    # the fp32 merge and the fp32-output forward of the ring's partial results
    m32 = L.bsa_lse_merge_f32
    assert m32(ctypes.byref(p), x, x, None, x, None) == bsa.BSA_ERR_INVALID_ARG
    assert m32(ctypes.byref(p), vp(FAKE + 8), x, x, x, None) == bsa.BSA_ERR_ALIGNMENT
    assert m32(ctypes.byref(p), x, x, x, vp(FAKE + 2), None) == bsa.BSA_ERR_ALIGNMENT
    assert m32(ctypes.byref(P(W=0)), x, x, x, x, None) == bsa.BSA_ERR_SHAPE
    fp = L.bsa_forward_partial
    assert fp(ctypes.byref(p), x, x, x, x, x, 16, x, 256, None, x, None) == \
        bsa.BSA_ERR_INVALID_ARG                                   # out_f32 required
    assert fp(ctypes.byref(p), x, x, x, x, x, 16, x, 256, x, None, None) == \
        bsa.BSA_ERR_INVALID_ARG                                   # lse required
    assert fp(ctypes.byref(p), x, x, x, x, x, 16, x, 256, vp(FAKE + 4), x, None) == \
        bsa.BSA_ERR_ALIGNMENT
    assert fp(ctypes.byref(p), x, x, x, x, x, 16, x, 255, x, x, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    # select from pooled inputs: kshard must divide the key chunks
    pr = P(T=16, H=8, W=16, q_begin=4, q_end=8)
    wsz = bsa.bsa_workspace_size(pr)
    g = L.bsa_select_pooled
    assert g(ctypes.byref(pr), x, x, 3, x, wsz, x, x, 64, None) == bsa.BSA_ERR_INVALID_ARG
    assert g(ctypes.byref(pr), x, x, 2, x, wsz - 1, x, x, 64, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    # gradient accumulation of the ring backward: arguments, overwrite flag, alignment
    a = L.bsa_grad_accumulate
    assert a(ctypes.byref(p), None, x, 1, None) == bsa.BSA_ERR_INVALID_ARG
    assert a(ctypes.byref(p), x, None, 0, None) == bsa.BSA_ERR_INVALID_ARG
    assert a(ctypes.byref(p), x, x, 2, None) == bsa.BSA_ERR_INVALID_ARG
    assert a(ctypes.byref(p), vp(FAKE + 4), x, 1, None) == bsa.BSA_ERR_ALIGNMENT
    assert a(ctypes.byref(P(T=0)), x, x, 1, None) == bsa.BSA_ERR_SHAPE
    fz = L.bsa_grad_finalize
    assert fz(ctypes.byref(p), None, x, None) == bsa.BSA_ERR_INVALID_ARG
    assert fz(ctypes.byref(p), x, vp(FAKE + 8), None) == bsa.BSA_ERR_ALIGNMENT


def test_exp2_selftest_host_checks(L):
    x = vp(FAKE)
    e = L.bsa_selftest_exp2
    assert e(x, x, x, 3, None) == bsa.BSA_ERR_INVALID_ARG          # n must be even
    assert e(x, x, x, -2, None) == bsa.BSA_ERR_INVALID_ARG
    assert e(None, x, x, 2, None) == bsa.BSA_ERR_INVALID_ARG
    assert e(vp(FAKE + 2), x, x, 2, None) == bsa.BSA_ERR_ALIGNMENT
    assert e(x, x, vp(FAKE + 1), 2, None) == bsa.BSA_ERR_ALIGNMENT


@pytest.mark.parametrize("kw,code", [(dict(q_begin=4, q_end=4), bsa.BSA_ERR_SHAPE),
                                     (dict(q_end=6), bsa.BSA_ERR_SHAPE),
                                     (dict(q_end=20), bsa.BSA_ERR_SHAPE),
                                     (dict(q_end=8), 0), (dict(T=10, q_end=10), 0)])
def test_query_frame_range(L, kw, code):
    base = dict(T=16, H=8, W=16)
    base.update(kw)
    rc, rows, _ = rc_sizes(P(**base))
    assert rc == code
    if code == 0 and base.get("q_end", 0) == 8:
        assert rows == 2 * 2 * 2 * 2     # heads 2 x chunk frames [0, 2) x (2 x 2) chunks


def test_plain_c_program_uses_the_header_and_library(L, tmp_path):
    """The header compiles as strict C99 and a C program linked against libbsa.so
    gets the same host-side answers as the Python binding."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(bsa.LIB_PATH)
    exe = str(tmp_path / "c_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_consumer.c"),
                    "-L", libdir, "-lbsa", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {ln.split()[0]: ln.split()[1:] for ln in out if ln.strip()}
    p = bsa.make_params(1, 32, 24, 48, 80, 128, "topk", 45)
    rows, nnz = bsa.bsa_plan_sizes(p)
    s = bsa.bsa_shape_info(p)
    assert got["plan_sizes"] == ["0", str(rows), str(nnz)]
    assert got["shape"] == ["0"] + [str(getattr(s, f)) for f in ("BH", "N", "rows", "d", "Nc",
                                                                    "Nq", "Nk")]
    assert got["workspace"] == [str(bsa.bsa_workspace_size(p)),
                                str(bsa.bsa_backward_workspace_size(p))]
    assert got["null_q"] == [str(bsa.BSA_ERR_INVALID_ARG)]
    assert got["null_bwd_ex"] == [str(bsa.BSA_ERR_INVALID_ARG)]
    assert got["null_status"] == [str(bsa.BSA_ERR_INVALID_ARG)]
    assert got["bad_d"][0] == str(bsa.BSA_ERR_UNSUPPORTED)
    assert got["version"] == [str(bsa.bsa_version())]


def _r256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("kw,group,slots", [
    (dict(B=1, heads=32, T=24, H=48, W=80, d=128, topk=45), 2, 3),
    (dict(B=2, heads=3, T=10, H=13, W=37, d=64, mode="cdf"), 4, 2),
    (dict(B=1, heads=5, T=16, H=8, W=16, d=128, topk=3, kchunk=(8, 8, 8)), 5, 1),
])
def test_forward_host_workspace_layout(L, kw, group, slots):
    """256-byte status block, then per slot: Q, K, V, O of one group, the plan's
    workspace and CSR of one group, each rounded up to 256 bytes."""
    p = P(**kw)
    N = p.T * p.H * p.W
    pg = P(**dict(kw, B=1, heads=group))
    rows, nnz = bsa.bsa_plan_sizes(pg)
    slot = (4 * _r256(group * N * p.d * 2) + _r256(bsa.bsa_workspace_size(pg)) +
            _r256((rows + 1) * 4) + _r256(max(nnz, 1) * 4))
    assert bsa.bsa_forward_host_workspace_size(p, group, slots) == 256 + slots * slot


def test_forward_host_host_checks(L):
    p = P(B=1, heads=4, T=8, H=8, W=16, d=64)
    f = L.bsa_forward_host_workspace_size
    assert f(ctypes.byref(p), 0, 1) == 0                    # group < 1
    assert f(ctypes.byref(p), 5, 1) == 0                    # group > B*heads
    assert f(ctypes.byref(p), 2, 0) == 0 and f(ctypes.byref(p), 2, 17) == 0
    assert f(ctypes.byref(P(T=0)), 1, 1) == 0
    ws = f(ctypes.byref(p), 2, 2)
    x = vp(FAKE)
    streams = (ctypes.c_void_p * 2)(None, None)
    g = L.bsa_forward_host
    pp = ctypes.byref(p)
    # q, k, v, out, group, slots, streams, workspace, ws_bytes, stream
    assert g(pp, None, x, x, x, 2, 2, streams, x, ws, None) == bsa.BSA_ERR_INVALID_ARG
    assert g(pp, x, x, x, x, 2, 2, None, x, ws, None) == bsa.BSA_ERR_INVALID_ARG
    assert g(pp, x, x, x, x, 0, 2, streams, x, ws, None) == bsa.BSA_ERR_INVALID_ARG
    assert g(pp, x, x, x, x, 2, 17, streams, x, ws, None) == bsa.BSA_ERR_INVALID_ARG
    assert g(pp, x, x, x, x, 2, 2, streams, vp(FAKE + 16), ws, None) == bsa.BSA_ERR_ALIGNMENT
    assert g(pp, x, x, x, x, 2, 2, streams, x, ws - 1, None) == \
        bsa.BSA_ERR_WORKSPACE_TOO_SMALL
    assert g(ctypes.byref(P(T=0)), x, x, x, x, 2, 2, streams, x, ws, None) == bsa.BSA_ERR_SHAPE


def test_forward_host_binding_checks():
    import torch
    p = bsa.make_params(1, 2, 8, 8, 16, 64)
    x = 2 * 1024 * 64
    h = torch.zeros(x, dtype=torch.bfloat16)
    ws = torch.zeros(bsa.bsa_forward_host_workspace_size(p, 1, 2), dtype=torch.uint8)
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_forward_host(p, h, h, h, h[:-1], 1, [None, None], ws)
    assert e.value.code == bsa.BSA_ERR_SHAPE and "out" in str(e.value)
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_forward_host(p, h, h, h.float(), h, 1, [None, None], ws)
    assert e.value.code == bsa.BSA_ERR_INVALID_ARG
    with pytest.raises(bsa.BsaError) as e:      # the staging workspace must be on the device
        bsa.bsa_forward_host(p, h, h, h, h, 1, [None, None], ws)
    assert e.value.code == bsa.BSA_ERR_INVALID_ARG and "CUDA" in str(e.value)
