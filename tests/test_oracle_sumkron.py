"""Pins for the SumKronLinear oracle (``oracle/sumkron.py``).

The page (Kunlun paper review §2.4) gives SumKronLinear by its shapes and
parameter counts only.  What pins the oracle:

* the explicit Kronecker-sum matrix, built with ``numpy.kron`` and applied to
  the row-major flattened sample (a library routine, the definition itself);
* brute-force Python sums on tiny shapes;
* a selection special case (k = 1, A = [I | 0], W = I gives the first T rows);
* the sum structure: each term alone, summed, gives the whole; permuting the
  (A_r, W_r) pairs together changes nothing;
* the parameter counts the page states;
* central finite differences for the backward.

Planted mistakes at the end must each fail at least one pin.
"""
import types

import numpy as np
import pytest

from oracle import sumkron


def _impl(**over):
    ns = types.SimpleNamespace(forward=sumkron.forward, backward=sumkron.backward)
    for k, v in over.items():
        setattr(ns, k, v)
    return ns


def _rand(rng, B=2, S=5, T=3, D=4, k=3):
    return (rng.standard_normal((B, S, D)), rng.standard_normal((k, T, S)),
            rng.standard_normal((k, D, D)))


def pin_kron(impl):
    rng = np.random.default_rng(1)
    x, a, w = _rand(rng)
    B, S, D = x.shape
    T = a.shape[1]
    full = sum(np.kron(a[r], w[r].T) for r in range(a.shape[0]))  # [T D, S D]
    ref = (full @ x.reshape(B, S * D).T).T.reshape(B, T, D)
    np.testing.assert_allclose(impl.forward(x, a, w), ref, rtol=1e-12, atol=1e-12)


def pin_brute(impl):
    rng = np.random.default_rng(2)
    x, a, w = _rand(rng, B=1, S=3, T=2, D=2, k=2)
    y = impl.forward(x, a, w)
    for t in range(2):
        for e in range(2):
            acc = 0.0
            for r in range(2):
                for s in range(3):
                    for d in range(2):
                        acc += a[r, t, s] * x[0, s, d] * w[r, d, e]
            assert abs(y[0, t, e] - acc) < 1e-12


def pin_selection(impl):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 6, 4))
    a = np.zeros((1, 2, 6))
    a[0, 0, 0] = a[0, 1, 1] = 1.0
    w = np.eye(4)[None]
    np.testing.assert_allclose(impl.forward(x, a, w), x[:, :2], rtol=0, atol=0)
    # a single term with a non-symmetric W: Y = X[:, :T] W (W on the right, untransposed)
    w2 = rng.standard_normal((1, 4, 4))
    np.testing.assert_allclose(impl.forward(x, a, w2), x[:, :2] @ w2[0], rtol=1e-12, atol=1e-12)


def pin_sum_structure(impl):
    rng = np.random.default_rng(4)
    x, a, w = _rand(rng, k=4)
    y = impl.forward(x, a, w)
    parts = sum(impl.forward(x, a[r:r + 1], w[r:r + 1]) for r in range(4))
    np.testing.assert_allclose(y, parts, rtol=1e-12, atol=1e-12)
    perm = [2, 0, 3, 1]
    np.testing.assert_allclose(impl.forward(x, a[perm], w[perm]), y, rtol=1e-12, atol=1e-12)


def pin_counts(impl):
    # the page's typical configuration: S = 256 seeds, T = 32 tokens, D = 384, k = 8
    assert sumkron.parameter_count(256, 32, 384, 8) == 8 * (256 * 32 + 384 * 384)
    rng = np.random.default_rng(5)
    x, a, w = _rand(rng)
    assert a.size + w.size == sumkron.parameter_count(5, 3, 4, 3)
    assert impl.forward(x, a, w).shape == (2, 3, 4)


def pin_backward_fd(impl):
    rng = np.random.default_rng(6)
    x, a, w = _rand(rng, B=2, S=3, T=2, D=2, k=2)
    dy = rng.standard_normal((2, 2, 2))
    dx, da, dw = impl.backward(x, a, w, dy)
    h = 1e-6

    def loss(x_, a_, w_):
        return float((impl.forward(x_, a_, w_) * dy).sum())

    for which, g in ((0, dx), (1, da), (2, dw)):
        args = [x, a, w]
        fd = np.zeros_like(args[which])
        for idx in np.ndindex(fd.shape):
            p = [t.copy() for t in args]
            m = [t.copy() for t in args]
            p[which][idx] += h
            m[which][idx] -= h
            fd[idx] = (loss(*p) - loss(*m)) / (2 * h)
        np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-8)


PINS = [pin_kron, pin_brute, pin_selection, pin_sum_structure, pin_counts, pin_backward_fd]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(_impl())


# ---------------------------------------------------------------- planted mistakes
def _fwd_transposed_w(x, a, w):
    return np.einsum("rts,bsd,red->bte", a, x, w)


def _fwd_shifted_pairs(x, a, w):
    return np.einsum("rts,bsd,rde->bte", a, x, np.roll(w, 1, axis=0))


def _fwd_first_term_only(x, a, w):
    return np.einsum("ts,bsd,de->bte", a[0], x, w[0])


def _fwd_transposed_a(x, a, w):  # A applied as its transpose would need T = S
    return np.einsum("rst,bsd,rde->bte", a.reshape(a.shape[0], a.shape[2], a.shape[1]), x, w)


def _bwd_dx_untransposed_w(x, a, w, dy):
    dx, da, dw = sumkron.backward(x, a, w, dy)
    return np.einsum("rts,bte,red->bsd", a, dy, w), da, dw


def _bwd_da_missing_w(x, a, w, dy):
    dx, da, dw = sumkron.backward(x, a, w, dy)
    return dx, np.einsum("bte,bsd->ts", dy, x)[None].repeat(a.shape[0], 0), dw


MUTANTS = {
    "transposed_w": dict(forward=_fwd_transposed_w),
    "shifted_pairs": dict(forward=_fwd_shifted_pairs),
    "first_term_only": dict(forward=_fwd_first_term_only),
    "reshaped_a": dict(forward=_fwd_transposed_a),
    "dx_untransposed_w": dict(backward=_bwd_dx_untransposed_w),
    "da_missing_w": dict(backward=_bwd_da_missing_w),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    impl = _impl(**MUTANTS[name])
    failed = []
    for pin in PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
