"""Rotary temporal embedding, fp64 -- TEST INFRASTRUCTURE ONLY (see ``oracle``).

Kunlun paper review §2.2 (feature preprocessing and time encoding): RoPE extended from
positions to time gaps.  The gap between adjacent events is log-scaled with a
time scale tau_scale, and each rotation angle combines a position frequency
theta_i and a time frequency phi_i.  The display formulas were lost in the
page; the reading implemented here:

* within a sample, token t (0-based) has gap dt_t = time_t - time_{t-1}
  (dt_0 = 0; a negative gap counts as 0) and scaled gap
  tau_t = ln(1 + dt_t / tau_scale);
* pair i = (2i, 2i+1) of a head vector turns by alpha_{t,i} = t theta_i +
  tau_t phi_i;
* theta_i = 10000^(-2i/D) unless given; phi_i = theta_i unless given;
* queries and keys are rotated (each with its own positions and times),
  values are not; every head uses the same angles.

The backward of a rotation is the rotation by the opposite angle.
"""
from __future__ import annotations

import numpy as np

from . import backward as _backward
from . import forward as _forward


def default_theta(D: int) -> np.ndarray:
    """Position frequencies 10000^(-2i/D), i = 0..D/2-1."""
    return 10000.0 ** (-2.0 * np.arange(D // 2, dtype=np.float64) / D)


def scaled_gaps(offsets, times, time_scale: float) -> np.ndarray:
    """tau_t = ln(1 + max(dt_t, 0) / tau_scale) per token, dt_0 = 0 in each sample."""
    offsets = np.asarray(offsets, np.int64)
    times = np.asarray(times, np.int64)
    dt = np.zeros(len(times), np.float64)
    dt[1:] = np.maximum(times[1:] - times[:-1], 0).astype(np.float64)
    dt[offsets[:-1][offsets[:-1] < len(times)]] = 0.0  # first token of each sample
    return np.log1p(dt / time_scale)


def positions(offsets) -> np.ndarray:
    """Index of each token within its sample."""
    offsets = np.asarray(offsets, np.int64)
    lens = np.diff(offsets)
    starts = np.repeat(offsets[:-1], lens)
    return (np.arange(int(offsets[-1]), dtype=np.int64) - starts).astype(np.float64)


def angles(offsets, times, D: int, time_scale: float, theta=None, phi=None) -> np.ndarray:
    """alpha [total, D/2] = t theta_i + tau_t phi_i."""
    th = default_theta(D) if theta is None else np.asarray(theta, np.float64)
    ph = th if phi is None else np.asarray(phi, np.float64)
    t = positions(offsets)
    tau = scaled_gaps(offsets, times, time_scale)
    return t[:, None] * th[None, :] + tau[:, None] * ph[None, :]


def rotate(x, alpha) -> np.ndarray:
    """Turn each pair (x_2i, x_2i+1) of x [total, H, D] by alpha [total, D/2]."""
    x = np.asarray(x, np.float64)
    c = np.cos(alpha)[:, None, :]
    s = np.sin(alpha)[:, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def _f64(a):
    if hasattr(a, "detach"):
        import torch
        return a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, np.float64)


def forward(q, k, v, q_offsets, kv_offsets, alpha_q, alpha_k, **kw):
    """GDPA forward on rotated queries and keys: O, LSE (fp64)."""
    return _forward(rotate(_f64(q), alpha_q), rotate(_f64(k), alpha_k), v, q_offsets,
                    kv_offsets, **kw)


def backward(q, k, v, dout, q_offsets, kv_offsets, alpha_q, alpha_k, **kw):
    """dQ, dK, dV, dbias with respect to the unrotated Q and K (fp64)."""
    dqr, dkr, dv, dbias = _backward(rotate(_f64(q), alpha_q), rotate(_f64(k), alpha_k), v, dout,
                                    q_offsets, kv_offsets, **kw)
    return rotate(dqr, -alpha_q), rotate(dkr, -alpha_k), dv, dbias
