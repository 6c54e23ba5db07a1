"""Pins for the rotary temporal embedding oracle (``oracle/rotary.py``).

The Kunlun pages give the rotary temporal embedding in words only (Kunlun
paper review §2.2): RoPE whose angles also carry log-scaled time gaps.  What
pins the oracle here:

* with equal times the angles are RoPE's, and the rotation equals GPT-J's
  interleaved rotary routine from ``transformers`` (a library routine);
* the time part composes with the position part as a second rotation;
* the scaled gap has closed forms (ln(1 + (e - 1)) = 1, ln 4, 0);
* rotations keep norms, and with evenly spaced times the scores of constant
  queries and keys depend only on i - j (RoPE's relative property);
* zero frequencies give back the plain oracle; the backward matches central
  finite differences of the forward.

Each pin takes the implementation as an argument, and the planted mistakes at
the end must each fail at least one pin.
"""
import math
import types

import numpy as np
import pytest

import oracle
from oracle import rotary

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _impl(**over):
    """The oracle's rotary functions, with some replaced (planted mistakes)."""
    ns = types.SimpleNamespace(angles=rotary.angles, rotate=rotary.rotate,
                               scaled_gaps=rotary.scaled_gaps, backward=rotary.backward,
                               forward=rotary.forward)
    for k, v in over.items():
        setattr(ns, k, v)
    return ns


def _sample(rng, lens, H=2, D=8):
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = rng.standard_normal((int(off[-1]), H, D))
    return off, x


# ---------------------------------------------------------------- pins
def pin_gptj(impl):
    """Equal times: the rotation is RoPE, as GPT-J's routine computes it."""
    import torch
    from transformers.models.gptj.modeling_gptj import (apply_rotary_pos_emb,
                                                        create_sinusoidal_positions)
    rng = np.random.default_rng(1)
    D = 16
    off, x = _sample(rng, [5, 1, 9], H=3, D=D)
    times = np.full(int(off[-1]), 7, np.int64)
    got = impl.rotate(x, impl.angles(off, times, D, 3.0))
    table = create_sinusoidal_positions(32, D).to(torch.float64)  # [pos, D]: sin | cos
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        sincos = table[: e - s]
        sin, cos = sincos[:, : D // 2], sincos[:, D // 2:]
        ref = apply_rotary_pos_emb(torch.from_numpy(x[s:e])[None], sin[None], cos[None])[0]
        # transformers builds its sin/cos table in fp32: agreement to fp32 precision
        np.testing.assert_allclose(got[s:e], ref.numpy(), rtol=1e-6, atol=1e-6)


def pin_compose(impl):
    """Position and time angles add: one rotation equals the two in sequence."""
    rng = np.random.default_rng(2)
    D = 8
    off, x = _sample(rng, [6, 4], D=D)
    times = np.cumsum(rng.integers(0, 500, int(off[-1]))).astype(np.int64)
    th = rng.uniform(0.01, 1.0, D // 2)
    ph = rng.uniform(0.01, 1.0, D // 2)
    z = np.zeros(D // 2)
    both = impl.rotate(x, impl.angles(off, times, D, 40.0, th, ph))
    seq = impl.rotate(impl.rotate(x, impl.angles(off, times, D, 40.0, th, z)),
                      impl.angles(off, times, D, 40.0, z, ph))
    np.testing.assert_allclose(both, seq, rtol=1e-12, atol=1e-12)
    # the time part alone turns pair i of token t by tau_t * phi_i: with unit
    # phi and the scaled gaps of the closed-form pin, angles are known numbers
    a = impl.angles(np.array([0, 3]), np.array([0, 1000, 4000]), 2, 1000.0 / (math.e - 1),
                    np.zeros(1), np.ones(1))
    np.testing.assert_allclose(a[:, 0], [0.0, 1.0, math.log1p(3 * (math.e - 1))], rtol=1e-12)


def pin_gaps(impl):
    """Closed forms of tau = ln(1 + dt / tau_scale)."""
    sc = 1000.0 / (math.e - 1)
    off = np.array([0, 4, 6])
    times = np.array([5, 1005, 1005, 905, 0, 3 * 1000], np.int64)
    tau = impl.scaled_gaps(off, times, sc)
    ref = [0.0, 1.0, 0.0, 0.0, 0.0, math.log1p(3 * (math.e - 1))]
    np.testing.assert_allclose(tau, ref, rtol=1e-12, atol=1e-15)
    tau2 = impl.scaled_gaps(np.array([0, 2]), np.array([0, 300], np.int64), 100.0)
    np.testing.assert_allclose(tau2, [0.0, math.log(4.0)], rtol=1e-12)


def pin_relative(impl):
    """Norms are kept; with evenly spaced times, constant q and k give
    Toeplitz scores."""
    rng = np.random.default_rng(3)
    D, L = 8, 12
    off = np.array([0, L])
    times = np.arange(L, dtype=np.int64) * 60
    a = impl.angles(off, times, D, 30.0, rng.uniform(0.05, 1, D // 2), rng.uniform(0.05, 1, D // 2))
    q = np.repeat(rng.standard_normal((1, 1, D)), L, axis=0)
    k = np.repeat(rng.standard_normal((1, 1, D)), L, axis=0)
    qr, kr = impl.rotate(q, a), impl.rotate(k, a)
    np.testing.assert_allclose(np.linalg.norm(qr.reshape(L, -1, 2), axis=-1),
                               np.linalg.norm(q.reshape(L, -1, 2), axis=-1), rtol=1e-12)
    # token 0 has no gap (tau = 0); every later token has the same one, so
    # among tokens 1.. the score depends on i - j alone
    s = (qr[:, 0] @ kr[:, 0].T)[1:, 1:]
    for d in range(-(L - 2), L - 1):
        diag = np.diagonal(s, d)
        np.testing.assert_allclose(diag, diag[0], rtol=1e-10, atol=1e-10)
    assert np.ptp(np.diagonal(s, 0)) < 1e-10 and np.ptp(s) > 1e-3  # not constant overall


def pin_zero_frequencies(impl):
    """theta = phi = 0: the rotary forward is the plain oracle forward."""
    rng = np.random.default_rng(4)
    D = 8
    off, q = _sample(rng, [3, 5], D=D)
    k, v = rng.standard_normal(q.shape), rng.standard_normal(q.shape)
    times = np.arange(len(q), dtype=np.int64) * 9
    z = np.zeros(D // 2)
    a = impl.angles(off, times, D, 5.0, z, z)
    o, _ = impl.forward(q, k, v, off, off, a, a, phi=1, scale=0.3)
    ref, _ = oracle.forward(q, k, v, off, off, phi=1, scale=0.3)
    np.testing.assert_allclose(o, ref, rtol=1e-13, atol=1e-13)


def pin_backward_fd(impl):
    """dQ, dK of the rotary backward against central differences of the forward."""
    rng = np.random.default_rng(5)
    D = 4
    off, q = _sample(rng, [3, 2], H=1, D=D)
    k, v = rng.standard_normal(q.shape), rng.standard_normal(q.shape)
    dout = rng.standard_normal(q.shape)
    times = np.array([0, 40, 100, 7, 8], np.int64)
    a = impl.angles(off, times, D, 20.0)
    kw = dict(phi=1, scale=0.7, window=(1, 0))
    dq, dk, _, _ = impl.backward(q, k, v, dout, off, off, a, a, **kw)

    def loss(qq, kk):
        o, _ = impl.forward(qq, kk, v, off, off, a, a, **kw)
        return float((o * dout).sum())

    h = 1e-6
    for which, x, g in (("q", q, dq), ("k", k, dk)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            lp = loss(xp, k) if which == "q" else loss(q, xp)
            lm = loss(xm, k) if which == "q" else loss(q, xm)
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-8)


PINS = [pin_gptj, pin_compose, pin_gaps, pin_relative, pin_zero_frequencies, pin_backward_fd]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(_impl())


# ---------------------------------------------------------------- planted mistakes
def _rotate_wrong_sign(x, alpha):
    x = np.asarray(x, np.float64)
    c, s = np.cos(alpha)[:, None, :], np.sin(alpha)[:, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c + b * s
    out[..., 1::2] = a * s + b * c
    return out


def _rotate_half_split(x, alpha):
    x = np.asarray(x, np.float64)
    n = x.shape[-1] // 2
    c, s = np.cos(alpha)[:, None, :], np.sin(alpha)[:, None, :]
    a, b = x[..., :n], x[..., n:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _gaps_cumulative(offsets, times, time_scale):
    tau = rotary.scaled_gaps(offsets, times, time_scale)
    out = tau.copy()
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        out[s:e] = np.cumsum(tau[s:e])
    return out


def _angles_with(gaps):
    def angles(offsets, times, D, time_scale, theta=None, phi=None):
        th = rotary.default_theta(D) if theta is None else np.asarray(theta, np.float64)
        ph = th if phi is None else np.asarray(phi, np.float64)
        return (rotary.positions(offsets)[:, None] * th[None, :] +
                gaps(offsets, times, time_scale)[:, None] * ph[None, :])
    return angles


def _angles_one_based(offsets, times, D, time_scale, theta=None, phi=None):
    th = rotary.default_theta(D) if theta is None else np.asarray(theta, np.float64)
    ph = th if phi is None else np.asarray(phi, np.float64)
    return ((rotary.positions(offsets) + 1)[:, None] * th[None, :] +
            rotary.scaled_gaps(offsets, times, time_scale)[:, None] * ph[None, :])


def _backward_plus(q, k, v, dout, q_offsets, kv_offsets, alpha_q, alpha_k, **kw):
    dqr, dkr, dv, db = oracle.backward(rotary.rotate(q, alpha_q), rotary.rotate(k, alpha_k), v,
                                       dout, q_offsets, kv_offsets, **kw)
    return rotary.rotate(dqr, alpha_q), rotary.rotate(dkr, alpha_k), dv, db


def _with_rotate(rot):
    def fwd(q, k, v, qo, ko, aq, ak, **kw):
        return oracle.forward(rot(q, aq), rot(k, ak), v, qo, ko, **kw)

    def bwd(q, k, v, dout, qo, ko, aq, ak, **kw):
        dqr, dkr, dv, db = oracle.backward(rot(q, aq), rot(k, ak), v, dout, qo, ko, **kw)
        return rot(dqr, -aq), rot(dkr, -ak), dv, db
    return dict(rotate=rot, forward=fwd, backward=bwd)


MUTANTS = {
    "wrong_sign": _with_rotate(_rotate_wrong_sign),
    "half_split_pairs": _with_rotate(_rotate_half_split),
    "cumulative_time": dict(angles=_angles_with(_gaps_cumulative)),
    "one_based_positions": dict(angles=_angles_one_based),
    "backward_same_direction": dict(backward=_backward_plus),
}


def _gaps_plain_log(offsets, times, time_scale):
    offsets = np.asarray(offsets, np.int64)
    times = np.asarray(times, np.int64)
    dt = np.zeros(len(times))
    dt[1:] = np.maximum(times[1:] - times[:-1], 0)
    dt[offsets[:-1][offsets[:-1] < len(times)]] = 0.0
    return np.log(np.maximum(dt / time_scale, 1e-300))


MUTANTS["log_not_log1p"] = dict(scaled_gaps=_gaps_plain_log, angles=_angles_with(_gaps_plain_log))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    impl = _impl(**MUTANTS[name])
    failed = []
    for pin in PINS:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
