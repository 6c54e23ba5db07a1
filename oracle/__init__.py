"""fp64 CPU oracle for GDPA -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs import this package.  It shares no code with the CUDA library
and never imports it; both sides are fed from ``workloads.py``.

``forward`` / ``backward`` marshal numpy fp64 arrays into the plain C oracle
(``gdpa_oracle.c``, built on demand with gcc and OpenMP).  ``schedule`` holds
the pure-Python statement of the jagged tile schedule.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

from .schedule import tile_schedule  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdpa_oracle.c")
_LIB = os.path.join(_HERE, "libgdpa_oracle.so")
_lib = None


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
                ("total_q", ctypes.c_int64), ("total_kv", ctypes.c_int64),
                ("phi", ctypes.c_int), ("scale", ctypes.c_double),
                ("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("bias_kind", ctypes.c_int)]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libgdpa_oracle.so`` (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.gdpa_oracle_forward.argtypes = [ctypes.POINTER(_Params), dp, dp, dp, ip, ip, dp, dp, dp]
        lib.gdpa_oracle_forward.restype = ctypes.c_int
        lib.gdpa_oracle_backward.argtypes = [ctypes.POINTER(_Params), dp, dp, dp, dp, ip, ip, dp,
                                             dp, dp, dp, dp]
        lib.gdpa_oracle_backward.restype = ctypes.c_int
        lib.gdpa_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().gdpa_oracle_num_threads())


def _f64(a) -> np.ndarray:
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (bf16 values widen exactly)
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, ct=ctypes.c_double):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ct))


def _params(B, H, D, total_q, total_kv, phi, scale, window, bias_kind):
    wl, wr = window
    return _Params(B, H, D, total_q, total_kv, phi, float(scale), int(wl), int(wr), int(bias_kind))


def forward(q, k, v, q_offsets, kv_offsets, *, phi: int, scale: float,
            window=(-1, -1), bias=None, bias_kind: int = 0):
    """O [total_q,H,D] and LSE [H,total_q] in fp64 (LSE is 0 unless softmax)."""
    q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
    qo = np.ascontiguousarray(q_offsets, dtype=np.int32)
    ko = np.ascontiguousarray(kv_offsets, dtype=np.int32)
    tq, H, D = q.shape
    tk = k.shape[0]
    B = len(qo) - 1
    p = _params(B, H, D, tq, tk, phi, scale, window, bias_kind)
    o = np.zeros((tq, H, D), np.float64)
    lse = np.zeros((H, tq), np.float64)
    rc = _load().gdpa_oracle_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(qo, ctypes.c_int32), _ptr(ko, ctypes.c_int32),
                                     _ptr(bias), _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle forward rejected its arguments")
    return o, lse


def backward(q, k, v, dout, q_offsets, kv_offsets, *, phi: int, scale: float,
             window=(-1, -1), bias=None, bias_kind: int = 0):
    """dQ, dK, dV (shapes of Q, K, V) and dbias [H,total_kv] in fp64."""
    q, k, v, dout, bias = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(bias)
    qo = np.ascontiguousarray(q_offsets, dtype=np.int32)
    ko = np.ascontiguousarray(kv_offsets, dtype=np.int32)
    tq, H, D = q.shape
    tk = k.shape[0]
    B = len(qo) - 1
    p = _params(B, H, D, tq, tk, phi, scale, window, bias_kind)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dbias = np.zeros((H, tk), np.float64)
    rc = _load().gdpa_oracle_backward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                      _ptr(qo, ctypes.c_int32), _ptr(ko, ctypes.c_int32),
                                      _ptr(bias), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbias))
    if rc:
        raise ValueError("oracle backward rejected its arguments")
    return dq, dk, dv, dbias


def forward_workload(w, bias=None):
    """Oracle forward on a ``workloads.Workload``."""
    return forward(w.q, w.k, w.v, w.q_offsets, w.kv_offsets, phi=w.phi, scale=w.scale,
                   window=(w.window_left, w.window_right),
                   bias=w.bias if bias is None else bias, bias_kind=w.bias_kind)


def backward_workload(w, dout=None):
    """Oracle backward on a ``workloads.Workload`` (uses ``w.dout`` by default)."""
    return backward(w.q, w.k, w.v, w.dout if dout is None else dout, w.q_offsets,
                    w.kv_offsets, phi=w.phi, scale=w.scale,
                    window=(w.window_left, w.window_right), bias=w.bias,
                    bias_kind=w.bias_kind)
