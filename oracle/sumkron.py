"""SumKronLinear, fp64 -- TEST INFRASTRUCTURE ONLY (see ``oracle``).

Kunlun paper review §2.4 (HSP and SumKronLinear): the second stage of
Hierarchical Seed Pooling compresses the seed summaries X [B, S, D] to
Y [B, T, D] with a rank-k sum of Kronecker products, using O(k (S T + D^2))
parameters instead of the O(S D T D) of a full linear map.  The page's display
formula was lost; the reading implemented here is the map whose parameters
are exactly that count:

    vec(Y_b) = sum_r (A_r kron W_r^T) vec(X_b)   (row-major vec)
    i.e.  Y_b = sum_r A_r X_b W_r,   A_r in R^{T x S}, W_r in R^{D x D},

with no bias.  The page's "about 14x fewer parameters" for S=256, T=32,
D=384, k=8 does not follow from its own two counts (they give about 970x);
the counts are taken as the definition.

Evaluated in fp64 as one sum over r, s and d per output element (an einsum;
the grouping of the products is numpy's).
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    if hasattr(a, "detach"):
        import torch
        return a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, np.float64)


def forward(x, a, w) -> np.ndarray:
    """Y [B, T, D] = sum_r A_r X_b W_r for X [B, S, D], A [k, T, S], W [k, D, D]."""
    x, a, w = _f64(x), _f64(a), _f64(w)
    return np.einsum("rts,bsd,rde->bte", a, x, w, optimize=True)


def backward(x, a, w, dy):
    """dX [B,S,D], dA [k,T,S], dW [k,D,D] of sum(Y * dY)."""
    x, a, w, dy = _f64(x), _f64(a), _f64(w), _f64(dy)
    dx = np.einsum("rts,bte,rde->bsd", a, dy, w, optimize=True)
    da = np.einsum("bte,bsd,rde->rts", dy, x, w, optimize=True)
    dw = np.einsum("rts,bsd,bte->rde", a, x, dy, optimize=True)
    return dx, da, dw


def parameter_count(S: int, T: int, D: int, k: int) -> int:
    """Parameters of the rank-k map: k (S T + D^2)."""
    return k * (S * T + D * D)
