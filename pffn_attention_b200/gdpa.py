"""ctypes binding of libgdpa (include/gdpa.h).

The ``gdpa_*`` functions keep the C names and take raw integers (device
pointers, sizes, a stream handle); they only marshal arguments.  ``forward``
and ``backward`` are the torch-facing conveniences: they allocate outputs and
the workspace with torch, pass pointers, and raise on a non-OK status.  Every
step of the computation runs in the CUDA library; if ``libgdpa.so`` is
missing, ``load`` raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdpa.so")

GDPA_OK = 0
STATUS_NAMES = {0: "GDPA_OK", 1: "GDPA_ERR_INVALID_ARG", 2: "GDPA_ERR_UNSUPPORTED",
                3: "GDPA_ERR_WORKSPACE", 4: "GDPA_ERR_CUDA", 5: "GDPA_ERR_TIMEOUT",
                6: "GDPA_ERR_DEVICE_CHECK"}
PHI = {"silu": 0, "softmax": 1, "identity": 2, "gelu": 3}
BIAS = {"none": 0, "add": 1, "gate": 2}

EXPORTED = ("gdpa_workspace_size", "gdpa_forward", "gdpa_backward", "gdpa_tile_schedule",
            "gdpa_forward_tile_shape", "gdpa_get_device_status", "gdpa_status_string",
            "gdpa_version", "gdpa_forward_no_alloc", "gdpa_forward_grouped_workspace_size",
            "gdpa_forward_grouped", "gdpa_rotary_table_bytes", "gdpa_rotary_table",
            "gdpa_rotary_apply", "gdpa_sumkron_workspace_size", "gdpa_sumkron_forward",
            "gdpa_sumkron_backward_workspace_size", "gdpa_sumkron_backward",
            "gdpa_backward_grouped_workspace_size", "gdpa_backward_grouped",
            "gdpa_forward_no_alloc_status")


class gdpa_params_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
                ("total_q", ctypes.c_int64), ("total_kv", ctypes.c_int64),
                ("max_seqlen_q", ctypes.c_int), ("max_seqlen_kv", ctypes.c_int),
                ("phi", ctypes.c_int), ("scale", ctypes.c_float),
                ("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("bias_kind", ctypes.c_int), ("debug_flags", ctypes.c_int),
                ("wait_timeout_us", ctypes.c_int),
                ("head_phi", ctypes.POINTER(ctypes.c_int32)),
                ("rope_q", ctypes.c_void_p), ("rope_kv", ctypes.c_void_p)]


class gdpa_sumkron_params_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("S", ctypes.c_int), ("T", ctypes.c_int), ("D", ctypes.c_int),
                ("k", ctypes.c_int), ("wait_timeout_us", ctypes.c_int),
                ("debug_flags", ctypes.c_int)]


class gdpa_rotary_params_t(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("time_scale", ctypes.c_float),
                ("theta", ctypes.POINTER(ctypes.c_float)), ("phi", ctypes.POINTER(ctypes.c_float))]


class gdpa_forward_problem_t(ctypes.Structure):
    _fields_ = [("params", gdpa_params_t), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("q_offsets", ctypes.c_void_p),
                ("kv_offsets", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


class gdpa_backward_problem_t(ctypes.Structure):
    _fields_ = [("params", gdpa_params_t)] + [
        (n, ctypes.c_void_p) for n in ("q", "k", "v", "o", "dout", "lse", "q_offsets",
                                       "kv_offsets", "bias", "dq", "dk", "dv", "dbias")]


class GdpaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load(path: str = LIB_PATH):
    """Load libgdpa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libgdpa.so not built at {path}; run python -m pffn_attention_b200.build")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(gdpa_params_t)
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
    lib.gdpa_workspace_size.argtypes = [P, ctypes.c_int]
    lib.gdpa_workspace_size.restype = sz
    lib.gdpa_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, st]
    lib.gdpa_forward.restype = ctypes.c_int
    lib.gdpa_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                  st]
    lib.gdpa_backward.restype = ctypes.c_int
    lib.gdpa_tile_schedule.argtypes = [P, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, st]
    lib.gdpa_tile_schedule.restype = ctypes.c_int
    lib.gdpa_forward_tile_shape.argtypes = [P, ctypes.POINTER(ctypes.c_int),
                                            ctypes.POINTER(ctypes.c_int)]
    lib.gdpa_forward_tile_shape.restype = ctypes.c_int
    lib.gdpa_get_device_status.argtypes = [vp, st]
    lib.gdpa_get_device_status.restype = ctypes.c_int
    lib.gdpa_status_string.argtypes = [ctypes.c_int]
    lib.gdpa_status_string.restype = ctypes.c_char_p
    lib.gdpa_forward_no_alloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, st]
    lib.gdpa_forward_no_alloc.restype = ctypes.c_int
    lib.gdpa_forward_no_alloc_status.argtypes = [st]
    lib.gdpa_forward_no_alloc_status.restype = ctypes.c_int
    lib.gdpa_version.argtypes = []
    lib.gdpa_version.restype = ctypes.c_int
    FP = ctypes.POINTER(gdpa_forward_problem_t)
    lib.gdpa_forward_grouped_workspace_size.argtypes = [FP, ctypes.c_int]
    lib.gdpa_forward_grouped_workspace_size.restype = sz
    lib.gdpa_forward_grouped.argtypes = [FP, ctypes.c_int, vp, sz, st]
    lib.gdpa_forward_grouped.restype = ctypes.c_int
    BP = ctypes.POINTER(gdpa_backward_problem_t)
    lib.gdpa_backward_grouped_workspace_size.argtypes = [BP, ctypes.c_int]
    lib.gdpa_backward_grouped_workspace_size.restype = sz
    lib.gdpa_backward_grouped.argtypes = [BP, ctypes.c_int, vp, sz, st]
    lib.gdpa_backward_grouped.restype = ctypes.c_int
    lib.gdpa_rotary_table_bytes.argtypes = [ctypes.c_int, ctypes.c_int64]
    lib.gdpa_rotary_table_bytes.restype = sz
    lib.gdpa_rotary_table.argtypes = [ctypes.POINTER(gdpa_rotary_params_t), ctypes.c_int,
                                      ctypes.c_int64, vp, vp, vp, st]
    lib.gdpa_rotary_table.restype = ctypes.c_int
    lib.gdpa_rotary_apply.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                      ctypes.c_int, st]
    lib.gdpa_rotary_apply.restype = ctypes.c_int
    SP = ctypes.POINTER(gdpa_sumkron_params_t)
    lib.gdpa_sumkron_workspace_size.argtypes = [SP]
    lib.gdpa_sumkron_workspace_size.restype = sz
    lib.gdpa_sumkron_forward.argtypes = [SP, vp, vp, vp, vp, vp, sz, st]
    lib.gdpa_sumkron_forward.restype = ctypes.c_int
    lib.gdpa_sumkron_backward_workspace_size.argtypes = [SP]
    lib.gdpa_sumkron_backward_workspace_size.restype = sz
    lib.gdpa_sumkron_backward.argtypes = [SP, vp, vp, vp, vp, vp, vp, vp, vp, sz, st]
    lib.gdpa_sumkron_backward.restype = ctypes.c_int
    _lib = lib
    return lib


# ----------------------------------------------------------------- raw C names
def gdpa_workspace_size(p: gdpa_params_t, backward: int) -> int:
    return int(load().gdpa_workspace_size(ctypes.byref(p), int(backward)))


def gdpa_forward(p, q, k, v, q_offsets, kv_offsets, bias, o, lse, workspace, workspace_bytes,
                 stream) -> int:
    return int(load().gdpa_forward(ctypes.byref(p), q, k, v, q_offsets, kv_offsets, bias, o, lse,
                                   workspace, workspace_bytes, stream))


def gdpa_rotary_table_bytes(D: int, total: int) -> int:
    return int(load().gdpa_rotary_table_bytes(int(D), int(total)))


def gdpa_rotary_table(r: gdpa_rotary_params_t, B, total, offsets, time, table, stream) -> int:
    return load().gdpa_rotary_table(ctypes.byref(r), int(B), int(total), offsets, time, table,
                                    stream)


def gdpa_rotary_apply(total, H, D, x, table, y, inverse, stream) -> int:
    return int(load().gdpa_rotary_apply(int(total), int(H), int(D), x, table, y, int(inverse),
                                        stream))


def gdpa_sumkron_workspace_size(p: gdpa_sumkron_params_t) -> int:
    return int(load().gdpa_sumkron_workspace_size(ctypes.byref(p)))


def gdpa_sumkron_forward(p, x, a, w, y, workspace, workspace_bytes, stream) -> int:
    return int(load().gdpa_sumkron_forward(ctypes.byref(p), x, a, w, y, workspace,
                                           workspace_bytes, stream))


def gdpa_sumkron_backward_workspace_size(p: gdpa_sumkron_params_t) -> int:
    return int(load().gdpa_sumkron_backward_workspace_size(ctypes.byref(p)))


def gdpa_sumkron_backward(p, x, a, w, dy, dx, da, dw, workspace, workspace_bytes, stream) -> int:
    return int(load().gdpa_sumkron_backward(ctypes.byref(p), x, a, w, dy, dx, da, dw, workspace,
                                            workspace_bytes, stream))


def gdpa_forward_grouped_workspace_size(problems) -> int:
    """problems: a ctypes array of gdpa_forward_problem_t (or None)."""
    n = 0 if problems is None else len(problems)
    return int(load().gdpa_forward_grouped_workspace_size(problems, n))


def gdpa_forward_grouped(problems, workspace, workspace_bytes, stream) -> int:
    n = 0 if problems is None else len(problems)
    return int(load().gdpa_forward_grouped(problems, n, workspace, workspace_bytes, stream))


def gdpa_forward_no_alloc(p, q, k, v, q_offsets, kv_offsets, bias, o, lse, stream) -> int:
    """Forward with the library's built-in scratch (no caller workspace)."""
    return int(load().gdpa_forward_no_alloc(ctypes.byref(p), q, k, v, q_offsets, kv_offsets,
                                            bias, o, lse, stream))


def gdpa_forward_no_alloc_status(stream) -> int:
    """Device status of the last no-alloc forward on the current device
    (synchronises the stream)."""
    return int(load().gdpa_forward_no_alloc_status(stream))


def gdpa_backward(p, q, k, v, o, dout, lse, q_offsets, kv_offsets, bias, dq, dk, dv, dbias,
                  workspace, workspace_bytes, stream) -> int:
    return int(load().gdpa_backward(ctypes.byref(p), q, k, v, o, dout, lse, q_offsets, kv_offsets,
                                    bias, dq, dk, dv, dbias, workspace, workspace_bytes, stream))


def gdpa_tile_schedule(p, block_m, block_n, q_offsets, kv_offsets, tile_start, order,
                       stream) -> int:
    return int(load().gdpa_tile_schedule(ctypes.byref(p), block_m, block_n, q_offsets, kv_offsets,
                                         tile_start, order, stream))


def gdpa_forward_tile_shape(p):
    bm, bn = ctypes.c_int(0), ctypes.c_int(0)
    rc = int(load().gdpa_forward_tile_shape(ctypes.byref(p), ctypes.byref(bm), ctypes.byref(bn)))
    return rc, bm.value, bn.value


def gdpa_get_device_status(workspace, stream) -> int:
    return int(load().gdpa_get_device_status(workspace, stream))


def gdpa_status_string(s: int) -> str:
    return load().gdpa_status_string(int(s)).decode()


def gdpa_version() -> int:
    return int(load().gdpa_version())


# ----------------------------------------------------------------- torch helpers
def make_params(B, H, D, total_q, total_kv, *, phi=0, scale=1.0, window=(-1, -1),
                bias_kind=0, max_seqlen_q=0, max_seqlen_kv=0, debug_flags=0,
                wait_timeout_us=0, head_phi=None, rope=None) -> gdpa_params_t:
    """head_phi: optional sequence of H activations (names or GDPA_PHI values),
    one per head; the params object keeps the array alive.  rope: optional
    (q table, kv table) pair of device tensors from rotary_table."""
    if isinstance(phi, str):
        phi = PHI[phi]
    if isinstance(bias_kind, str):
        bias_kind = BIAS[bias_kind]
    arr = None
    if head_phi is not None:
        vals = [PHI[x] if isinstance(x, str) else int(x) for x in head_phi]
        arr = (ctypes.c_int32 * len(vals))(*vals)
    p = gdpa_params_t(int(B), int(H), int(D), int(total_q), int(total_kv), int(max_seqlen_q),
                      int(max_seqlen_kv), int(phi), float(scale), int(window[0]),
                      int(window[1]), int(bias_kind), int(debug_flags), int(wait_timeout_us),
                      ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)) if arr is not None
                      else None)
    p._head_phi = arr  # owns the array the struct points to
    if rope is not None:
        p.rope_q, p.rope_kv = _ptr(rope[0]), _ptr(rope[1])
        p._rope = rope  # keeps the tables alive with the params
    return p


def _any_softmax(p) -> bool:
    if p.head_phi:
        return any(p.head_phi[h] == PHI["softmax"] for h in range(p.H))
    return p.phi == PHI["softmax"]


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def workspace_for(p: gdpa_params_t, backward: bool, device):
    import torch
    n = gdpa_workspace_size(p, int(backward))
    if n == 0:
        raise GdpaError(1, "gdpa_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _check(rc: int, where: str):
    if rc != GDPA_OK:
        raise GdpaError(rc, where)


def rotary_table(offsets, time, D, time_scale, *, theta=None, phi=None, out=None,
                 stream=None):
    """Rotation table [total, D/2] (int32 view of the fp16 (cos, sin) pairs) of
    the rotary temporal embedding for the jagged sequence of offsets (int32
    [B+1]) and time (int64 [total]) on the device.  theta / phi: optional
    sequences of D/2 position / time frequencies."""
    import torch
    total = time.numel()
    B = offsets.numel() - 1
    if out is None:
        out = torch.empty((total, D // 2), dtype=torch.int32, device=time.device)
    def arr(x):
        return None if x is None else (ctypes.c_float * len(x))(*[float(v) for v in x])
    th, ph = arr(theta), arr(phi)
    r = gdpa_rotary_params_t(int(D), float(time_scale),
                             ctypes.cast(th, ctypes.POINTER(ctypes.c_float)) if th else None,
                             ctypes.cast(ph, ctypes.POINTER(ctypes.c_float)) if ph else None)
    rc = gdpa_rotary_table(r, B, total, _ptr(offsets), _ptr(time), _ptr(out), _stream(stream))
    _check(rc, "gdpa_rotary_table")
    return out


def sumkron_forward(x, a, w, *, out=None, workspace=None, stream=None, wait_timeout_us=0,
                    debug_flags=0):
    """SumKronLinear: y [B,T,D] = sum_r a[r] @ x[b] @ w[r] for x [B,S,D],
    a [k,T,S], w [k,D,D] (bf16 CUDA tensors).  Returns (y, workspace)."""
    import torch
    B, S, D = x.shape
    k, T, _ = a.shape
    p = gdpa_sumkron_params_t(int(B), int(S), int(T), int(D), int(k), int(wait_timeout_us),
                              int(debug_flags))
    if out is None:
        out = torch.empty((B, T, D), dtype=x.dtype, device=x.device)
    if workspace is None:
        n = gdpa_sumkron_workspace_size(p)
        if n == 0:
            raise GdpaError(2, "gdpa_sumkron_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check(gdpa_sumkron_forward(p, _ptr(x), _ptr(a), _ptr(w), _ptr(out), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "gdpa_sumkron_forward")
    return out, workspace


def sumkron_backward(x, a, w, dy, *, workspace=None, stream=None, wait_timeout_us=0):
    """Gradients of SumKronLinear for dy [B,T,D]: returns (dx [B,S,D], da [k,T,S],
    dw [k,D,D], workspace) (bf16 CUDA tensors)."""
    import torch
    B, S, D = x.shape
    k, T, _ = a.shape
    p = gdpa_sumkron_params_t(int(B), int(S), int(T), int(D), int(k), int(wait_timeout_us), 0)
    dx = torch.empty_like(x)
    da = torch.empty_like(a)
    dw = torch.empty_like(w)
    if workspace is None:
        n = gdpa_sumkron_backward_workspace_size(p)
        if n == 0:
            raise GdpaError(2, "gdpa_sumkron_backward_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check(gdpa_sumkron_backward(p, _ptr(x), _ptr(a), _ptr(w), _ptr(dy), _ptr(dx), _ptr(da),
                                 _ptr(dw), _ptr(workspace), workspace.numel(), _stream(stream)),
           "gdpa_sumkron_backward")
    return dx, da, dw, workspace


def rotary_apply(x, table, *, inverse=False, out=None, stream=None):
    """x [total,H,D] bf16 turned by the table (or back); out may be x."""
    import torch
    total, H, D = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(gdpa_rotary_apply(total, H, D, _ptr(x), _ptr(table), _ptr(out), int(inverse),
                             _stream(stream)), "gdpa_rotary_apply")
    return out


def forward(q, k, v, q_offsets, kv_offsets, *, phi="silu", scale=1.0, window=(-1, -1),
            bias=None, bias_kind="none", max_seqlen_q=0, max_seqlen_kv=0, out=None, lse=None,
            workspace=None, stream=None, params=None, head_phi=None, rope=None):
    """O (and LSE for softmax) on the device.  Inputs are CUDA tensors:
    q [total_q,H,D] bf16, k/v [total_kv,H,D] bf16, offsets int32 [B+1];
    rope: optional (q table, kv table) from rotary_table."""
    import torch
    total_q, H, D = q.shape
    total_kv = k.shape[0]
    B = q_offsets.numel() - 1
    p = params or make_params(B, H, D, total_q, total_kv, phi=phi, scale=scale, window=window,
                              bias_kind=bias_kind, max_seqlen_q=max_seqlen_q,
                              max_seqlen_kv=max_seqlen_kv, head_phi=head_phi, rope=rope)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and _any_softmax(p):
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(p, False, q.device)
    rc = gdpa_forward(p, _ptr(q), _ptr(k), _ptr(v), _ptr(q_offsets), _ptr(kv_offsets), _ptr(bias),
                      _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "gdpa_forward")
    return out, lse, workspace


def forward_grouped(problems, *, workspace=None, stream=None):
    """Several GDPA problems in one call.  problems: a list of dicts with the
    tensors q, k, v, q_offsets, kv_offsets (and optional bias, out, lse) and the
    keyword arguments of forward() (phi, scale, window, bias_kind,
    max_seqlen_q, max_seqlen_kv, head_phi, rope).  Returns ([(o, lse), ...], workspace)."""
    import torch
    arr = (gdpa_forward_problem_t * len(problems))()
    outs, keep = [], []
    for i, d in enumerate(problems):
        q, k, v = d["q"], d["k"], d["v"]
        total_q, H, D = q.shape
        p = make_params(d["q_offsets"].numel() - 1, H, D, total_q, k.shape[0],
                        phi=d.get("phi", "silu"), scale=d.get("scale", 1.0),
                        window=d.get("window", (-1, -1)), bias_kind=d.get("bias_kind", "none"),
                        max_seqlen_q=d.get("max_seqlen_q", 0),
                        max_seqlen_kv=d.get("max_seqlen_kv", 0), head_phi=d.get("head_phi"),
                        rope=d.get("rope"))
        o = d.get("out") if d.get("out") is not None else torch.empty_like(q)
        lse = d.get("lse")
        if lse is None and _any_softmax(p):
            lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
        keep.append(p)
        arr[i].params = p
        for name, t in (("q", q), ("k", k), ("v", v), ("q_offsets", d["q_offsets"]),
                        ("kv_offsets", d["kv_offsets"]), ("bias", d.get("bias")), ("o", o),
                        ("lse", lse)):
            setattr(arr[i], name, _ptr(t))
        outs.append((o, lse))
    if workspace is None:
        n = gdpa_forward_grouped_workspace_size(arr)
        if n == 0:
            raise GdpaError(1, "gdpa_forward_grouped_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=problems[0]["q"].device)
    rc = gdpa_forward_grouped(arr, _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "gdpa_forward_grouped")
    return outs, workspace


def gdpa_backward_grouped_workspace_size(problems) -> int:
    """problems: a ctypes array of gdpa_backward_problem_t (or None)."""
    n = 0 if problems is None else len(problems)
    return int(load().gdpa_backward_grouped_workspace_size(problems, n))


def gdpa_backward_grouped(problems, workspace, workspace_bytes, stream) -> int:
    n = 0 if problems is None else len(problems)
    return int(load().gdpa_backward_grouped(problems, n, workspace, workspace_bytes, stream))


def backward_grouped(problems, *, workspace=None, stream=None):
    """Gradients of several GDPA problems in one call.  problems: a list of
    dicts with q, k, v, o, dout, lse, q_offsets, kv_offsets (optional bias,
    dbias) and the keyword arguments of backward().  Returns
    ([(dq, dk, dv), ...], workspace)."""
    import torch
    arr = (gdpa_backward_problem_t * len(problems))()
    outs, keep = [], []
    for i, d in enumerate(problems):
        q, k, v = d["q"], d["k"], d["v"]
        total_q, H, D = q.shape
        p = make_params(d["q_offsets"].numel() - 1, H, D, total_q, k.shape[0],
                        phi=d.get("phi", "silu"), scale=d.get("scale", 1.0),
                        window=d.get("window", (-1, -1)), bias_kind=d.get("bias_kind", "none"),
                        max_seqlen_q=d.get("max_seqlen_q", 0),
                        max_seqlen_kv=d.get("max_seqlen_kv", 0), head_phi=d.get("head_phi"),
                        rope=d.get("rope"))
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        keep.append(p)
        arr[i].params = p
        for name, t in (("q", q), ("k", k), ("v", v), ("o", d.get("o")), ("dout", d["dout"]),
                        ("lse", d.get("lse")), ("q_offsets", d["q_offsets"]),
                        ("kv_offsets", d["kv_offsets"]), ("bias", d.get("bias")), ("dq", dq),
                        ("dk", dk), ("dv", dv), ("dbias", d.get("dbias"))):
            setattr(arr[i], name, _ptr(t))
        outs.append((dq, dk, dv))
    if workspace is None:
        n = gdpa_backward_grouped_workspace_size(arr)
        if n == 0:
            raise GdpaError(1, "gdpa_backward_grouped_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=problems[0]["q"].device)
    rc = gdpa_backward_grouped(arr, _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "gdpa_backward_grouped")
    return outs, workspace


def backward(q, k, v, o, dout, lse, q_offsets, kv_offsets, *, phi="silu", scale=1.0,
             window=(-1, -1), bias=None, bias_kind="none", max_seqlen_q=0, max_seqlen_kv=0,
             dq=None, dk=None, dv=None, dbias=None, workspace=None, stream=None, params=None,
             head_phi=None, rope=None):
    """dQ, dK, dV on the device (bf16, shapes of q, k, v).  With a bias or gate,
    pass dbias (fp32 [H, total_kv]) to also receive the bias gradient.  rope:
    the forward's (q table, kv table); q and k stay the unturned inputs."""
    import torch
    total_q, H, D = q.shape
    total_kv = k.shape[0]
    B = q_offsets.numel() - 1
    p = params or make_params(B, H, D, total_q, total_kv, phi=phi, scale=scale, window=window,
                              bias_kind=bias_kind, max_seqlen_q=max_seqlen_q,
                              max_seqlen_kv=max_seqlen_kv, head_phi=head_phi, rope=rope)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = workspace_for(p, True, q.device)
    rc = gdpa_backward(p, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                       _ptr(q_offsets), _ptr(kv_offsets), _ptr(bias), _ptr(dq), _ptr(dk),
                       _ptr(dv), _ptr(dbias), _ptr(workspace), workspace.numel(),
                       _stream(stream))
    _check(rc, "gdpa_backward")
    return dq, dk, dv, workspace


def device_status(workspace, stream=None) -> int:
    return gdpa_get_device_status(_ptr(workspace), _stream(stream))
