"""Seeded synthetic inputs for 3D block sparse attention (inputs only).

The C generator in ``synth.c`` is the single implementation used by the CPU
oracle, the GPU tests and the benchmark. This module builds it on demand,
exposes it through ctypes and names the standard workloads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .workloads import WORKLOADS, Workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile libsynth.so with gcc/OpenMP (in-tree)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-D_GNU_SOURCE", "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            lib.synth_field_bf16.restype = ctypes.c_int
            lib.synth_field_bf16.argtypes = [
                ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int,
                ctypes.c_double, ctypes.c_int, ctypes.c_uint64]
            lib.synth_field_bf16_slice.restype = ctypes.c_int
            lib.synth_field_bf16_slice.argtypes = [
                ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                ctypes.c_uint32, ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_uint64]
            lib.synth_ctr_u64.restype = ctypes.c_uint64
            lib.synth_ctr_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            lib.synth_ctr_normal.restype = ctypes.c_double
            lib.synth_ctr_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            lib.synth_mix64.restype = ctypes.c_uint64
            lib.synth_mix64.argtypes = [ctypes.c_uint64]
            _lib = lib
    return _lib


TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_DO = 0, 1, 2, 3


def field_bf16(B, heads, T, H, W, d, seed, tensor, rms_norm, tfreq_mult=1.0,
               cond_frames=0, cond_seed=1, b_offset=0, out=None, h_offset=0):
    """One tensor as bf16 bit patterns, shape [B, heads, T*H*W, d], dtype uint16:
    batch elements [b_offset, b_offset + B) and heads [h_offset, h_offset + heads)
    of the virtual problem the seed defines."""
    lib = _load()
    shape = (B, heads, T * H * W, d)
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.shape == shape and out.dtype == np.uint16 and out.flags.c_contiguous
    rc = lib.synth_field_bf16_slice(out.ctypes.data, B, b_offset, heads, h_offset, T, H, W, d,
                                    seed, tensor, 1 if rms_norm else 0, float(tfreq_mult),
                                    int(cond_frames), int(cond_seed))
    if rc != 0:
        raise ValueError("synth_field_bf16: bad arguments")
    return out


def make_qkv(wl: "Workload", seed: int | None = None, batch_offset: int = 0,
             head_offset: int = 0):
    """Q, K, V (uint16 bf16 bits, [B, heads, N, d]) for a workload.

    ``batch_offset`` shifts the batch index of the streams, so that independent
    replicas (e.g. one per rank) draw different but reproducible inputs;
    ``head_offset`` shifts the head index, so that a rank holding heads
    [h0, h0 + heads) of one problem draws exactly those heads.
    """
    s = wl.seed if seed is None else seed
    return tuple(
        field_bf16(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, s, tensor,
                   rms_norm=(tensor != TENSOR_V), tfreq_mult=wl.tfreq_mult,
                   cond_frames=wl.t_cond, cond_seed=wl.cond_seed, b_offset=batch_offset,
                   h_offset=head_offset)
        for tensor in (TENSOR_Q, TENSOR_K, TENSOR_V))


def make_dout(wl: "Workload", seed: int | None = None, batch_offset: int = 0,
              head_offset: int = 0):
    """Upstream gradient dO for the backward (uint16 bf16 bits, [B, heads, N, d]):
    a smooth field of its own stream, not normalised (like V)."""
    s = wl.seed if seed is None else seed
    return field_bf16(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.d, s, TENSOR_DO, rms_norm=False,
                      tfreq_mult=wl.tfreq_mult, cond_frames=wl.t_cond, cond_seed=wl.cond_seed,
                      b_offset=batch_offset, h_offset=head_offset)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32)
