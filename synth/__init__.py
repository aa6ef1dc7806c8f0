"""Seeded synthetic inputs shared by the oracle and the CUDA path.

Only input generation lives here (see synth.c for the recipe); nothing in
this package computes any step of the attention method.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .workloads import A_LAT, A_NOISE, SINK_K_SCALE, Workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("bh", ctypes.c_int32),
        ("frames", ctypes.c_int32),
        ("tokens", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_sink", ctypes.c_int32),
        ("n_points", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("p_assign", ctypes.c_double),
        ("a_lat", ctypes.c_double),
        ("a_noise", ctypes.c_double),
        ("sink_k_scale", ctypes.c_double),
        ("seed", ctypes.c_uint64),
        ("out_bf16", ctypes.c_int32),
        ("n_threads", ctypes.c_int32),
        ("head0", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (plain gcc, no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.synth_generate.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_generate.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def generate(w: Workload, seed: int | None = None, heads: int | None = None,
             threads: int | None = None, dtype: str | None = None, head0: int = 0):
    """Return dict(q, k, v, point) as numpy arrays.

    q, k, v have shape [heads][S*N][d]; bf16 workloads come back as uint16
    bit patterns, f32 workloads as float32.  `point` is the int32 point id of
    every token (-1 = untied).  `heads` overrides the head count (heads are
    independent draws, so the first h heads of a larger draw are identical); `head0`
    draws heads head0 .. head0 + heads - 1 of that larger draw instead (a head shard).
    """
    lib = _load()
    dt = dtype or w.dtype
    bh = heads if heads is not None else w.heads
    cfg = _Cfg(bh, w.frames, w.tokens, w.head_dim, w.n_sink, w.n_points, w.window,
               float(w.p_assign), A_LAT, A_NOISE, SINK_K_SCALE,
               int(w.seed if seed is None else seed), 1 if dt == "bf16" else 0,
               int(threads or default_threads()), int(head0))
    shape = (bh, w.L, w.head_dim)
    npdt = np.uint16 if dt == "bf16" else np.float32
    q = np.empty(shape, npdt)
    k = np.empty(shape, npdt)
    v = np.empty(shape, npdt)
    point = np.empty((w.L,), np.int32)
    rc = lib.synth_generate(ctypes.byref(cfg), q.ctypes.data, k.ctypes.data, v.ctypes.data,
                            point.ctypes.data)
    if rc != 0:
        raise RuntimeError("synth_generate failed with code %d" % rc)
    return {"q": q, "k": k, "v": v, "point": point}


def generate_into(w: Workload, q, k, v, seed: int | None = None, threads: int | None = None, head0: int = 0):
    """Fill caller-owned host buffers (anything exposing a data pointer of the right size).

    q, k, v must be contiguous [heads][S*N][d] arrays of the workload's dtype
    (2 bytes per element for bf16, 4 for f32); `q.data_ptr()` (torch) or
    `q.ctypes.data` (numpy) is used.
    """
    lib = _load()
    ptr = lambda a: a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data  # noqa: E731
    bh = q.shape[0]
    cfg = _Cfg(bh, w.frames, w.tokens, w.head_dim, w.n_sink, w.n_points, w.window,
               float(w.p_assign), A_LAT, A_NOISE, SINK_K_SCALE,
               int(w.seed if seed is None else seed), 1 if w.dtype == "bf16" else 0,
               int(threads or default_threads()), int(head0))
    rc = lib.synth_generate(ctypes.byref(cfg), ptr(q), ptr(k), ptr(v), None)
    if rc != 0:
        raise RuntimeError("synth_generate failed with code %d" % rc)
