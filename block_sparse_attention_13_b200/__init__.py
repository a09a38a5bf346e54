"""B200 (sm_100a) 3D Block Sparse Attention -- Python binding of libbsa.so.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels (include/bsa.h documents the C ABI). PyTorch supplies device memory
and streams. There is no CPU fallback: if libbsa.so is missing or cannot be
loaded, every call raises.

Method: "LongCat-Video Technical Report" (paper summary page), section
"Block Sparse Attention (BSA)"; "LongCat-Video Technical Report #" (detail
page), section "3D Block Sparse Attention".
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_OK = 0
BSA_ERR_INVALID_ARG = 1
BSA_ERR_SHAPE = 2
BSA_ERR_UNSUPPORTED = 3
BSA_ERR_ALIGNMENT = 4
BSA_ERR_WORKSPACE_TOO_SMALL = 5
BSA_ERR_CUDA = 6
BSA_ERR_DEVICE_BAD_INDEX = 7
BSA_ERR_DEVICE_TIMEOUT = 8
BSA_ERR_CAPACITY = 9

BSA_SEL_TOPK = 0
BSA_SEL_CDF = 1
BSA_SEL_TOPK_CDF = 2
MODES = {"topk": BSA_SEL_TOPK, "cdf": BSA_SEL_CDF, "topk_cdf": BSA_SEL_TOPK_CDF}

EXPORTED = ("bsa_version", "bsa_status_string", "bsa_workspace_size", "bsa_plan_sizes",
            "bsa_plan", "bsa_plan_noalloc", "bsa_forward", "bsa_forward_ex", "bsa_read_status",
            "bsa_rearrange", "bsa_pool", "bsa_scores", "bsa_selftest_exp2",
            "bsa_selftest_timeout", "bsa_backward_workspace_size", "bsa_backward", "bsa_backward_ex",
            "bsa_select_pooled", "bsa_csr_slice_workspace_size", "bsa_csr_slice",
            "bsa_lse_merge", "bsa_grad_accumulate", "bsa_grad_finalize", "bsa_shape_info",
            "bsa_forward_host_workspace_size", "bsa_forward_host", "bsa_forward_partial",
            "bsa_lse_merge_f32")

# Scratch array of bsa_plan_noalloc inside the library (include/bsa.h: 32 MiB);
# a plan whose workspace exceeds it is rejected by the library before any CUDA call.
NOALLOC_SCRATCH_BYTES = 32 << 20


class BsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class bsa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("d", ctypes.c_int32),
                ("chunk_t", ctypes.c_int32), ("chunk_h", ctypes.c_int32),
                ("chunk_w", ctypes.c_int32), ("scale", ctypes.c_float), ("mode", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("cdf_p", ctypes.c_float),
                ("cdf_cap_frac", ctypes.c_float), ("t_cond", ctypes.c_int32),
                ("q_begin", ctypes.c_int32), ("kchunk_t", ctypes.c_int32),
                ("kchunk_h", ctypes.c_int32), ("kchunk_w", ctypes.c_int32),
                ("q_end", ctypes.c_int32)]


class bsa_shape(ctypes.Structure):
    """Element counts of the tensors of a call (include/bsa.h, bsa_shape_info)."""
    _fields_ = [("BH", ctypes.c_int64), ("N", ctypes.c_int64), ("rows", ctypes.c_int64),
                ("d", ctypes.c_int32), ("Nc", ctypes.c_int32), ("Nq", ctypes.c_int32),
                ("Nk", ctypes.c_int32)]


def make_params(B, heads, T, H, W, d, mode="topk", topk=1, cdf_p=0.9, cdf_cap_frac=0.25,
                t_cond=0, scale=0.0, q_begin=0, kchunk=(0, 0, 0), q_end=0,
                chunk=(4, 4, 8)) -> bsa_params:
    """chunk: query chunk shape, (4, 4, 8) or (4, 4, 4) (64-token chunks). kchunk: key
    chunk shape (t, h, w); 0 on an axis = the query chunk's. [q_begin, q_end): latent
    frames whose queries are computed (q_end 0 = T)."""
    return bsa_params(B, heads, T, H, W, d, *map(int, chunk), float(scale),
                      MODES[mode], int(topk), float(cdf_p),
                      float(cdf_cap_frac), int(t_cond), int(q_begin), *map(int, kchunk),
                      int(q_end))


def params_for(wl) -> bsa_params:
    """Parameters of a workload description (anything with the Workload fields)."""
    return make_params(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, wl.mode, wl.topk, wl.cdf_p,
                       wl.cdf_cap_frac, wl.t_cond, scale=getattr(wl, "scale", 0.0),
                       q_begin=getattr(wl, "q_begin", 0), kchunk=getattr(wl, "kchunk", (0, 0, 0)),
                       chunk=getattr(wl, "qchunk", (4, 4, 8)))


_lib = None


def lib():
    """The loaded libbsa.so (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libbsa.so not built ({LIB_PATH}); run "
                               "block_sparse_attention_13_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(bsa_params)
        vp, i32, i64, sz, u64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                                 ctypes.c_uint64)
        sigs = {
            "bsa_version": (i32, []),
            "bsa_status_string": (ctypes.c_char_p, [i32]),
            "bsa_workspace_size": (sz, [P]),
            "bsa_plan_sizes": (i32, [P, ctypes.POINTER(i64), ctypes.POINTER(i64)]),
            "bsa_shape_info": (i32, [P, ctypes.POINTER(bsa_shape)]),
            "bsa_forward_host_workspace_size": (sz, [P, ctypes.c_int32, ctypes.c_int32]),
            "bsa_forward_host": (i32, [P, vp, vp, vp, vp, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.POINTER(vp), vp, sz, vp]),
            "bsa_plan": (i32, [P, vp, vp, vp, sz, vp, vp, i64, vp]),
            "bsa_plan_noalloc": (i32, [P, vp, vp, vp, vp, i64, vp]),
            "bsa_forward": (i32, [P, vp, vp, vp, vp, vp, i64, vp, sz, vp, vp, vp]),
            "bsa_forward_ex": (i32, [P, vp, vp, vp, vp, vp, i64, vp, sz, vp, vp, u64, i32, vp]),
            "bsa_read_status": (i32, [vp, vp]),
            "bsa_rearrange": (i32, [P, vp, vp, i32, vp]),
            "bsa_pool": (i32, [P, vp, vp, vp]),
            "bsa_scores": (i32, [P, vp, vp, vp, vp]),
            "bsa_selftest_exp2": (i32, [vp, vp, vp, i64, vp]),
            "bsa_selftest_timeout": (i32, [vp, u64, vp]),
            "bsa_backward_workspace_size": (sz, [P]),
            "bsa_select_pooled": (i32, [P, vp, vp, i32, vp, sz, vp, vp, i64, vp]),
            "bsa_csr_slice_workspace_size": (sz, [i64]),
            "bsa_csr_slice": (i32, [i64, vp, vp, i64, i32, i32, vp, sz, vp, vp, i64, vp]),
            "bsa_lse_merge": (i32, [P, vp, vp, vp, vp, vp]),
            "bsa_lse_merge_f32": (i32, [P, vp, vp, vp, vp, vp]),
            "bsa_forward_partial": (i32, [P, vp, vp, vp, vp, vp, i64, vp, sz, vp, vp, vp]),
            "bsa_grad_accumulate": (i32, [P, vp, vp, i32, vp]),
            "bsa_grad_finalize": (i32, [P, vp, vp, vp]),
            "bsa_backward": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, sz, vp, vp, vp,
                                   vp]),
            "bsa_backward_ex": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, sz, vp, vp, vp,
                                      u64, i32, vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().bsa_status_string(int(code)).decode()


def _check(rc: int, what: str):
    if rc != BSA_OK:
        raise BsaError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _tensors(what, *specs, where="cuda"):
    """Checks the tensors of one call before their pointers are passed on.

    Each spec is (name, tensor or None, dtype or None, minimum size). A tensor
    the library reads or writes must have that dtype, be contiguous, hold at
    least that many elements (bytes when dtype is None: a workspace) and live on
    the current CUDA device (where="cpu": in host memory): anything else would
    reach the kernels or the copies as a bad address. Raises BsaError:
    INVALID_ARG for the kind of tensor, SHAPE for its size; the device is
    checked after every tensor's kind and size. None entries (optional outputs)
    are skipped.
    """
    import torch
    given = [(name, t, dtype, need) for name, t, dtype, need in specs if t is not None]
    for name, t, dtype, need in given:
        if not isinstance(t, torch.Tensor):
            raise BsaError(BSA_ERR_INVALID_ARG, f"{what}: {name} is not a torch.Tensor")
        if dtype is not None and t.dtype != dtype:
            raise BsaError(BSA_ERR_INVALID_ARG, f"{what}: {name} is {t.dtype}, expected {dtype}")
        if not t.is_contiguous():
            raise BsaError(BSA_ERR_INVALID_ARG, f"{what}: {name} is not contiguous")
        have = t.numel() if dtype is not None else t.numel() * t.element_size()
        if have < need:
            unit = "elements" if dtype is not None else "bytes"
            raise BsaError(BSA_ERR_SHAPE, f"{what}: {name} holds {have} {unit}, needs {need}")
    if where == "cpu":
        for name, t, _, _ in given:
            if t.device.type != "cpu":
                raise BsaError(BSA_ERR_INVALID_ARG, f"{what}: {name} is not in host memory")
        return
    cur = None
    for name, t, _, _ in given:
        if not t.is_cuda:
            raise BsaError(BSA_ERR_INVALID_ARG, f"{what}: {name} is not a CUDA tensor")
        if cur is None:
            cur = torch.cuda.current_device()
        if t.device.index != cur:
            raise BsaError(BSA_ERR_INVALID_ARG,
                           f"{what}: {name} is on {t.device}, the current device is cuda:{cur}")


def _dtypes():
    import torch
    return torch.bfloat16, torch.float32, torch.int32


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------ C-ABI mirrors

def bsa_version() -> int:
    return lib().bsa_version()


def bsa_workspace_size(p: bsa_params) -> int:
    n = lib().bsa_workspace_size(ctypes.byref(p))
    if n == 0:
        raise BsaError(BSA_ERR_INVALID_ARG, "bsa_workspace_size")
    return n


def bsa_plan_sizes(p: bsa_params):
    rows, nnz = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().bsa_plan_sizes(ctypes.byref(p), ctypes.byref(rows), ctypes.byref(nnz)),
           "bsa_plan_sizes")
    return rows.value, nnz.value


def bsa_shape_info(p: bsa_params) -> bsa_shape:
    s = bsa_shape()
    _check(lib().bsa_shape_info(ctypes.byref(p), ctypes.byref(s)), "bsa_shape_info")
    return s


def bsa_plan(p, q, k, workspace, row_ptr, col_idx, stream=None):
    bf, _, i32 = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_plan", ("q", q, bf, x), ("k", k, bf, x), ("workspace", workspace, None, 0),
             ("row_ptr", row_ptr, i32, s.rows + 1), ("col_idx", col_idx, i32, 0))
    _check(lib().bsa_plan(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _ptr(row_ptr),
                          _ptr(col_idx), col_idx.numel(), _stream(stream)), "bsa_plan")


def bsa_plan_noalloc(p, q, k, row_ptr, col_idx, stream=None):
    """bsa_plan with the library's fixed scratch array instead of a workspace,
    for callers that cannot allocate device memory (see include/bsa.h)."""
    bf, _, i32 = _dtypes()
    if lib().bsa_workspace_size(ctypes.byref(p)) <= NOALLOC_SCRATCH_BYTES:
        s = bsa_shape_info(p)
        x, rows = s.BH * s.N * s.d, s.rows + 1
    else:
        x = rows = 0          # the library rejects this plan before touching any pointer
    _tensors("bsa_plan_noalloc", ("q", q, bf, x), ("k", k, bf, x), ("row_ptr", row_ptr, i32, rows),
             ("col_idx", col_idx, i32, 0))
    _check(lib().bsa_plan_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(row_ptr),
                                  _ptr(col_idx), col_idx.numel(), _stream(stream)),
           "bsa_plan_noalloc")


def _forward_tensors(what, p, q, k, v, row_ptr, col_idx, workspace, out, lse):
    bf, f32, i32 = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors(what, ("q", q, bf, x), ("k", k, bf, x), ("v", v, bf, x), ("out", out, bf, x),
             ("lse", lse, f32, s.BH * s.N), ("row_ptr", row_ptr, i32, s.rows + 1),
             ("col_idx", col_idx, i32, 0), ("workspace", workspace, None, 0))


def bsa_forward(p, q, k, v, row_ptr, col_idx, workspace, out, lse=None, stream=None):
    _forward_tensors("bsa_forward", p, q, k, v, row_ptr, col_idx, workspace, out, lse)
    _check(lib().bsa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                             _ptr(col_idx), col_idx.numel(), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse),
                             _stream(stream)), "bsa_forward")


def bsa_forward_ex(p, q, k, v, row_ptr, col_idx, workspace, out, lse=None, timeout_ns=0,
                   debug_flags=0, stream=None):
    _forward_tensors("bsa_forward_ex", p, q, k, v, row_ptr, col_idx, workspace, out, lse)
    _check(lib().bsa_forward_ex(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                                _ptr(col_idx), col_idx.numel(), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _ptr(out),
                                _ptr(lse), int(timeout_ns), int(debug_flags), _stream(stream)),
           "bsa_forward_ex")


def bsa_forward_partial(p, q, k, v, row_ptr, col_idx, workspace, out_f32, lse, stream=None):
    """bsa_forward with an fp32 output (a partial result to merge by LSE)."""
    bf, f32, i32 = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_forward_partial", ("q", q, bf, x), ("k", k, bf, x), ("v", v, bf, x),
             ("out_f32", out_f32, f32, x), ("lse", lse, f32, s.BH * s.N),
             ("row_ptr", row_ptr, i32, s.rows + 1), ("col_idx", col_idx, i32, 0),
             ("workspace", workspace, None, 0))
    if out_f32 is None or lse is None:
        raise BsaError(BSA_ERR_INVALID_ARG, "bsa_forward_partial: out_f32 and lse are required")
    _check(lib().bsa_forward_partial(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                                     _ptr(col_idx), col_idx.numel(), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _ptr(out_f32),
                                     _ptr(lse), _stream(stream)), "bsa_forward_partial")


def bsa_backward_workspace_size(p: bsa_params) -> int:
    n = lib().bsa_backward_workspace_size(ctypes.byref(p))
    if n == 0:
        raise BsaError(BSA_ERR_INVALID_ARG, "bsa_backward_workspace_size")
    return n


def bsa_backward(p, q, k, v, out, lse, dout, row_ptr, col_idx, workspace, dq, dk, dv,
                 stream=None):
    _backward("bsa_backward", p, q, k, v, out, lse, dout, row_ptr, col_idx, workspace, dq, dk,
              dv, stream)


def bsa_backward_ex(p, q, k, v, out, lse, dout, row_ptr, col_idx, workspace, dq, dk, dv,
                    timeout_ns=0, debug_flags=0, stream=None):
    """bsa_backward with an explicit device wait limit and debug flags."""
    _backward("bsa_backward_ex", p, q, k, v, out, lse, dout, row_ptr, col_idx, workspace, dq, dk,
              dv, stream, (int(timeout_ns), int(debug_flags)))


def _backward(name, p, q, k, v, out, lse, dout, row_ptr, col_idx, workspace, dq, dk, dv, stream,
              extra=()):
    bf, f32, i32 = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors(name, ("q", q, bf, x), ("k", k, bf, x), ("v", v, bf, x), ("out", out, bf, x),
             ("lse", lse, f32, s.BH * s.N), ("dout", dout, bf, x),
             ("row_ptr", row_ptr, i32, s.rows + 1), ("col_idx", col_idx, i32, 0),
             ("workspace", workspace, None, 0), ("dq", dq, bf, x), ("dk", dk, bf, x),
             ("dv", dv, bf, x))
    _check(getattr(lib(), name)(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                _ptr(dout), _ptr(row_ptr), _ptr(col_idx), col_idx.numel(),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(dq), _ptr(dk), _ptr(dv), *extra, _stream(stream)), name)


def bsa_forward_host_workspace_size(p: bsa_params, group: int, slots: int) -> int:
    n = lib().bsa_forward_host_workspace_size(ctypes.byref(p), int(group), int(slots))
    if n == 0:
        raise BsaError(BSA_ERR_INVALID_ARG, "bsa_forward_host_workspace_size")
    return n


def bsa_forward_host(p, q, k, v, out, group, streams, workspace, stream=None):
    """plan + forward for q, k, v, out in host memory (CPU tensors, pinned for
    overlap): groups of `group` (batch, head) pairs run on `streams` (torch
    streams or raw handles), staged in `workspace` (device, status block
    zeroed before the first call). The caller's stream waits for all of it."""
    bf, _, _ = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_forward_host", ("q", q, bf, x), ("k", k, bf, x), ("v", v, bf, x),
             ("out", out, bf, x), where="cpu")
    _tensors("bsa_forward_host", ("workspace", workspace, None, 0))
    handles = (ctypes.c_void_p * len(streams))(*[_stream(st).value for st in streams])
    _check(lib().bsa_forward_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                  int(group), len(streams), handles, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "bsa_forward_host")


def bsa_select_pooled(p, qpool, kpool, workspace, row_ptr, col_idx, kshard=0, stream=None):
    _, f32, i32 = _dtypes()
    s = bsa_shape_info(p)
    _tensors("bsa_select_pooled", ("qpool", qpool, f32, s.BH * s.Nq * s.d),
             ("kpool", kpool, f32, s.BH * s.Nk * s.d), ("workspace", workspace, None, 0),
             ("row_ptr", row_ptr, i32, s.rows + 1), ("col_idx", col_idx, i32, 0))
    _check(lib().bsa_select_pooled(ctypes.byref(p), _ptr(qpool), _ptr(kpool), int(kshard),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _ptr(row_ptr), _ptr(col_idx), col_idx.numel(),
                                   _stream(stream)), "bsa_select_pooled")


def bsa_csr_slice_workspace_size(n_rows: int) -> int:
    return lib().bsa_csr_slice_workspace_size(int(n_rows))


def bsa_csr_slice(row_ptr, col_idx, lo, hi, workspace, out_row_ptr, out_col_idx, stream=None):
    _, _, i32 = _dtypes()
    _tensors("bsa_csr_slice", ("row_ptr", row_ptr, i32, 1), ("col_idx", col_idx, i32, 0),
             ("workspace", workspace, None, 0),
             ("out_row_ptr", out_row_ptr, i32, row_ptr.numel()), ("out_col_idx", out_col_idx, i32, 0))
    _check(lib().bsa_csr_slice(row_ptr.numel() - 1, _ptr(row_ptr), _ptr(col_idx), col_idx.numel(),
                               int(lo), int(hi), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _ptr(out_row_ptr),
                               _ptr(out_col_idx), out_col_idx.numel(), _stream(stream)),
           "bsa_csr_slice")


def bsa_lse_merge(p, out, lse, out_part, lse_part, stream=None):
    bf, f32, _ = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_lse_merge", ("out", out, bf, x), ("lse", lse, f32, s.BH * s.N),
             ("out_part", out_part, bf, x), ("lse_part", lse_part, f32, s.BH * s.N))
    _check(lib().bsa_lse_merge(ctypes.byref(p), _ptr(out), _ptr(lse), _ptr(out_part),
                               _ptr(lse_part), _stream(stream)), "bsa_lse_merge")


def bsa_lse_merge_f32(p, out, lse, out_part, lse_part, stream=None):
    _, f32, _ = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_lse_merge_f32", ("out", out, f32, x), ("lse", lse, f32, s.BH * s.N),
             ("out_part", out_part, f32, x), ("lse_part", lse_part, f32, s.BH * s.N))
    _check(lib().bsa_lse_merge_f32(ctypes.byref(p), _ptr(out), _ptr(lse), _ptr(out_part),
                                   _ptr(lse_part), _stream(stream)), "bsa_lse_merge_f32")


def bsa_grad_accumulate(p, part, acc, overwrite=False, stream=None):
    bf, f32, _ = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_grad_accumulate", ("part", part, bf, x), ("acc", acc, f32, x))
    _check(lib().bsa_grad_accumulate(ctypes.byref(p), _ptr(part), _ptr(acc), 1 if overwrite else 0,
                                     _stream(stream)), "bsa_grad_accumulate")


def bsa_grad_finalize(p, acc, out, stream=None):
    bf, f32, _ = _dtypes()
    s = bsa_shape_info(p)
    x = s.BH * s.N * s.d
    _tensors("bsa_grad_finalize", ("acc", acc, f32, x), ("out", out, bf, x))
    _check(lib().bsa_grad_finalize(ctypes.byref(p), _ptr(acc), _ptr(out), _stream(stream)),
           "bsa_grad_finalize")


def bsa_read_status(workspace, stream=None) -> int:
    _tensors("bsa_read_status", ("workspace", workspace, None, 256))  # the status block
    return lib().bsa_read_status(_ptr(workspace), _stream(stream))


def bsa_rearrange(p, x, out, inverse=False, stream=None):
    bf, _, _ = _dtypes()
    s = bsa_shape_info(p)
    thw, blk = s.BH * s.N * s.d, s.BH * s.Nc * 128 * s.d
    _tensors("bsa_rearrange", ("x", x, bf, blk if inverse else thw),
             ("out", out, bf, thw if inverse else blk))
    _check(lib().bsa_rearrange(ctypes.byref(p), _ptr(x), _ptr(out), 1 if inverse else 0,
                               _stream(stream)), "bsa_rearrange")


def bsa_pool(p, x, pooled, stream=None):
    bf, f32, _ = _dtypes()
    s = bsa_shape_info(p)
    _tensors("bsa_pool", ("x", x, bf, s.BH * s.N * s.d), ("pooled", pooled, f32, s.BH * s.Nc * s.d))
    _check(lib().bsa_pool(ctypes.byref(p), _ptr(x), _ptr(pooled), _stream(stream)), "bsa_pool")


def bsa_scores(p, qp, kp, S, stream=None):
    _, f32, _ = _dtypes()
    s = bsa_shape_info(p)
    _tensors("bsa_scores", ("qp", qp, f32, s.BH * s.Nq * s.d), ("kp", kp, f32, s.BH * s.Nk * s.d),
             ("S", S, f32, s.BH * s.Nq * s.Nk))
    _check(lib().bsa_scores(ctypes.byref(p), _ptr(qp), _ptr(kp), _ptr(S), _stream(stream)),
           "bsa_scores")


def bsa_selftest_exp2(x, y_poly, y_mufu, stream=None):
    _, f32, _ = _dtypes()
    _tensors("bsa_selftest_exp2", ("x", x, f32, 0), ("y_poly", y_poly, f32, x.numel()),
             ("y_mufu", y_mufu, f32, x.numel()))
    _check(lib().bsa_selftest_exp2(_ptr(x), _ptr(y_poly), _ptr(y_mufu), x.numel(),
                                   _stream(stream)), "bsa_selftest_exp2")


def bsa_selftest_timeout(workspace, timeout_ns, stream=None):
    _tensors("bsa_selftest_timeout", ("workspace", workspace, None, 256))
    _check(lib().bsa_selftest_timeout(_ptr(workspace), int(timeout_ns), _stream(stream)),
           "bsa_selftest_timeout")


# ------------------------------------------------------------------ convenience

@dataclass
class Plan:
    params: bsa_params
    workspace: "object"
    row_ptr: "object"
    col_idx: "object"


def allocate(p: bsa_params, device="cuda"):
    """Workspace and CSR buffers for `p` (torch device tensors)."""
    import torch
    rows, nnz = bsa_plan_sizes(p)
    ws = torch.empty(bsa_workspace_size(p), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return Plan(p, ws, torch.empty(rows + 1, dtype=torch.int32, device=device),
                torch.empty(max(nnz, 1), dtype=torch.int32, device=device))


def plan(p: bsa_params, q, k, buffers: Plan | None = None, stream=None) -> Plan:
    buffers = buffers or allocate(p, q.device)
    bsa_plan(p, q, k, buffers.workspace, buffers.row_ptr, buffers.col_idx, stream)
    return buffers


def forward(pl: Plan, q, k, v, out=None, lse=None, stream=None):
    import torch
    out = torch.empty_like(q) if out is None else out
    bsa_forward(pl.params, q, k, v, pl.row_ptr, pl.col_idx, pl.workspace, out, lse, stream)
    return out


def backward_workspace(p: bsa_params, device="cuda"):
    """Device workspace for bsa_backward (status block zeroed)."""
    import torch
    ws = torch.empty(bsa_backward_workspace_size(p), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def backward(pl: Plan, q, k, v, out, lse, dout, workspace=None, dq=None, dk=None, dv=None,
             stream=None):
    """dq, dk, dv of forward(pl, q, k, v) for upstream gradient dout."""
    import torch
    workspace = backward_workspace(pl.params, q.device) if workspace is None else workspace
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    bsa_backward(pl.params, q, k, v, out, lse, dout, pl.row_ptr, pl.col_idx, workspace, dq, dk,
                 dv, stream)
    return dq, dk, dv, workspace


def block_sparse_attention(q, k, v, topk=None, mode="topk", cdf_p=0.9, cdf_cap_frac=0.25,
                           t_cond=0, grid=None, want_lse=False, chunk=(4, 4, 8), kchunk=(0, 0, 0),
                           scale=0.0):
    """One call: plan + forward for q, k, v [B, heads, T*H*W, d] bf16 on the GPU.

    grid = (T, H, W) of the latent video; chunk = the query chunk shape, (4, 4, 8) or
    (4, 4, 4); kchunk = the key chunk shape (0 = the query chunk's). Returns out (and
    lse if asked).
    """
    import torch
    B, heads, N, d = q.shape
    T, H, W = grid
    assert T * H * W == N
    if topk is None:  # 1/16 of the key chunks (ceil counts: edge chunks may be partial)
        kc = tuple(c if c else q_ for c, q_ in zip(kchunk, chunk))
        topk = max(1, (-(-T // kc[0]) * -(-H // kc[1]) * -(-W // kc[2])) // 16)
    p = make_params(B, heads, T, H, W, d, mode, topk, cdf_p, cdf_cap_frac, t_cond, scale=scale,
                    kchunk=kchunk, chunk=chunk)
    pl = plan(p, q, k)
    lse = torch.empty((B, heads, N), dtype=torch.float32, device=q.device) if want_lse else None
    out = forward(pl, q, k, v, lse=lse)
    rc = bsa_read_status(pl.workspace)
    _check(rc, "device status")
    return (out, lse) if want_lse else out


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
