"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a library routine (numpy matmul, torch SDPA, torch autograd), a
closed form, an invariant of the definition, finite differences, or brute
force with hand-expanded sums.  No GPU is used here.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import (BIAS_ADD, BIAS_GATE, BIAS_NONE, PHI_GELU, PHI_IDENTITY, PHI_SILU,
                       PHI_SOFTMAX, offsets_from_lengths)


def rand_problem(rng, q_lens, kv_lens, H, D, std=1.0):
    qo = offsets_from_lengths(np.asarray(q_lens))
    ko = offsets_from_lengths(np.asarray(kv_lens))
    q = rng.standard_normal((qo[-1], H, D)) * std
    k = rng.standard_normal((ko[-1], H, D)) * std
    v = rng.standard_normal((ko[-1], H, D)) * std
    return q, k, v, qo, ko


def band_mask(Lq, Lk, wl, wr):
    i = np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    m = np.ones((Lq, Lk), bool)
    if wl >= 0:
        m &= j >= i - wl
    if wr >= 0:
        m &= j <= i + wr
    return m


def silu_np(x):
    return x * (1.0 / (1.0 + np.exp(-x)))


# ---------------------------------------------------------------- forward pins

def test_pffn_two_matmul_form():
    """SiLU GDPA equals the personalised FFN act(S W1) W2 with W1 = K^T, W2 = V
    (Kunlun paper review §2.3 / Fig. 2: the PFFN rewritten as attention)."""
    rng = np.random.default_rng(11)
    q, k, v, qo, ko = rand_problem(rng, [5, 17, 1], [8, 3, 6], H=2, D=7)
    scale = 0.37
    o, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_SILU, scale=scale)
    for b in range(3):
        for h in range(2):
            S = q[qo[b]:qo[b + 1], h, :]
            W1 = k[ko[b]:ko[b + 1], h, :].T          # D x Lk
            W2 = v[ko[b]:ko[b + 1], h, :]            # Lk x D
            ref = silu_np(scale * (S @ W1)) @ W2
            np.testing.assert_allclose(o[qo[b]:qo[b + 1], h, :], ref, rtol=1e-12, atol=1e-13)


def test_gelu_two_matmul_form_matches_torch():
    """GELU GDPA (the pages' example of an element-wise activation in place of
    softmax, Kunlun paper review §2.3) equals gelu(scale S W1) W2 with torch's
    exact (erf) GELU in fp64 and numpy matmuls, with a gate and a band."""
    rng = np.random.default_rng(16)
    q, k, v, qo, ko = rand_problem(rng, [6, 13, 1], [9, 4, 7], H=2, D=5)
    g = rng.standard_normal((2, ko[-1]))
    scale, (wl, wr) = 0.61, (3, 1)
    o, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_GELU, scale=scale, window=(wl, wr),
                          bias=g, bias_kind=BIAS_GATE)
    for b in range(3):
        Lq, Lk = qo[b + 1] - qo[b], ko[b + 1] - ko[b]
        vis = band_mask(Lq, Lk, wl, wr)
        for h in range(2):
            S = q[qo[b]:qo[b + 1], h, :]
            W1 = k[ko[b]:ko[b + 1], h, :].T
            W2 = v[ko[b]:ko[b + 1], h, :]
            gate = torch.nn.functional.logsigmoid(torch.tensor(g[h, ko[b]:ko[b + 1]])).numpy()
            x = torch.tensor(scale * (S @ W1) + gate[None, :])
            ref = (torch.nn.functional.gelu(x, approximate="none").numpy() * vis) @ W2
            np.testing.assert_allclose(o[qo[b]:qo[b + 1], h, :], ref, rtol=1e-12, atol=1e-13)


def test_identity_associativity():
    """phi = identity: (Q K^T) V = Q (K^T V), the right side by numpy."""
    rng = np.random.default_rng(12)
    q, k, v, qo, ko = rand_problem(rng, [9, 4], [5, 11], H=3, D=6)
    o, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_IDENTITY, scale=0.5)
    for b in range(2):
        for h in range(3):
            Q = q[qo[b]:qo[b + 1], h]
            K = k[ko[b]:ko[b + 1], h]
            V = v[ko[b]:ko[b + 1], h]
            np.testing.assert_allclose(o[qo[b]:qo[b + 1], h], 0.5 * (Q @ (K.T @ V)),
                                       rtol=1e-12, atol=1e-12)


def test_softmax_rows_sum_to_one():
    """With V = 1 every softmax output is exactly a probability sum: O = 1."""
    rng = np.random.default_rng(13)
    q, k, v, qo, ko = rand_problem(rng, [7, 30], [13, 2], H=2, D=4, std=3.0)
    o, _ = oracle.forward(q, k, np.ones_like(v), qo, ko, phi=PHI_SOFTMAX, scale=1.0)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


@pytest.mark.parametrize("window", [(-1, -1), (3, 0), (2, 5), (0, 0)])
@pytest.mark.parametrize("bias_kind", [BIAS_NONE, BIAS_ADD, BIAS_GATE])
def test_softmax_matches_torch_sdpa(window, bias_kind):
    """Softmax GDPA equals torch's scaled_dot_product_attention (fp64, CPU)
    with an explicit band mask and the bias (or torch's logsigmoid of the gate)
    as an additive float mask; LSE equals scipy's logsumexp of the scores."""
    from scipy.special import logsumexp
    rng = np.random.default_rng(14)
    H, D = 2, 8
    q, k, v, qo, ko = rand_problem(rng, [6, 19, 12], [6, 19, 25], H=H, D=D)
    g = rng.standard_normal((H, ko[-1])) * 2.0
    scale = 1.0 / math.sqrt(D)
    wl, wr = window
    o, lse = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=scale, window=window,
                            bias=g if bias_kind else None, bias_kind=bias_kind)
    for b in range(3):
        Lq, Lk = qo[b + 1] - qo[b], ko[b + 1] - ko[b]
        vis = band_mask(Lq, Lk, wl, wr)
        for h in range(H):
            Q = torch.tensor(q[qo[b]:qo[b + 1], h])
            K = torch.tensor(k[ko[b]:ko[b + 1], h])
            V = torch.tensor(v[ko[b]:ko[b + 1], h])
            gb = torch.tensor(g[h, ko[b]:ko[b + 1]])
            if bias_kind == BIAS_ADD:
                beta = gb
            elif bias_kind == BIAS_GATE:
                beta = torch.nn.functional.logsigmoid(gb)
            else:
                beta = torch.zeros(Lk, dtype=torch.float64)
            mask = torch.where(torch.tensor(vis), beta[None, :].expand(Lq, Lk),
                               torch.tensor(-math.inf, dtype=torch.float64))
            rows = vis.any(1)
            ref = torch.nn.functional.scaled_dot_product_attention(
                Q[None, None], K[None, None], V[None, None], attn_mask=mask[None, None],
                scale=scale)[0, 0].numpy()
            got = o[qo[b]:qo[b + 1], h]
            np.testing.assert_allclose(got[rows], ref[rows], rtol=1e-11, atol=1e-12)
            assert np.all(got[~rows] == 0.0)
            scores = scale * (q[qo[b]:qo[b + 1], h] @ k[ko[b]:ko[b + 1], h].T) + beta.numpy()
            scores = np.where(vis, scores, -np.inf)
            ref_lse = logsumexp(scores, axis=1)
            np.testing.assert_allclose(lse[h, qo[b]:qo[b + 1]][rows], ref_lse[rows],
                                       rtol=1e-12, atol=1e-12)
            assert np.all(np.isneginf(lse[h, qo[b]:qo[b + 1]][~rows]))


def test_single_key_closed_forms():
    """Lk = 1: softmax gives O_i = V_0 for any Q; SiLU gives silu(scale q.k) V_0."""
    rng = np.random.default_rng(15)
    q, k, v, qo, ko = rand_problem(rng, [4, 9], [1, 1], H=2, D=5)
    o, lse = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=0.7)
    for b in range(2):
        for h in range(2):
            np.testing.assert_array_equal(o[qo[b]:qo[b + 1], h],
                                          np.broadcast_to(v[ko[b], h], (qo[b + 1] - qo[b], 5)))
            s = 0.7 * q[qo[b]:qo[b + 1], h] @ k[ko[b], h]
            np.testing.assert_allclose(lse[h, qo[b]:qo[b + 1]], s, rtol=1e-14, atol=1e-14)
    o, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_SILU, scale=0.7)
    for b in range(2):
        for h in range(2):
            s = 0.7 * q[qo[b]:qo[b + 1], h] @ k[ko[b], h]
            ref = (s / (1.0 + np.exp(-s)))[:, None] * v[ko[b], h][None, :]
            np.testing.assert_allclose(o[qo[b]:qo[b + 1], h], ref, rtol=1e-13, atol=1e-14)


def test_two_key_worked_example():
    """Hand-worked case: Q = K = I (D = 2), V = [[1,2],[3,4]], scale 1.
    Scores are the identity, so softmax row 0 weighs the keys e:1 and row 1
    weighs them 1:e; SiLU gives weights silu(1) and silu(0) = 0."""
    e = math.e
    q = np.eye(2).reshape(2, 1, 2)
    k = np.eye(2).reshape(2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(2, 1, 2)
    off = np.array([0, 2], np.int32)
    o, lse = oracle.forward(q, k, v, off, off, phi=PHI_SOFTMAX, scale=1.0)
    r0 = np.array([(e * 1 + 3) / (e + 1), (e * 2 + 4) / (e + 1)])
    r1 = np.array([(1 + 3 * e) / (e + 1), (2 + 4 * e) / (e + 1)])
    np.testing.assert_allclose(o[:, 0], np.stack([r0, r1]), rtol=1e-15)
    np.testing.assert_allclose(lse[0], [math.log(e + 1)] * 2, rtol=1e-15)
    o, _ = oracle.forward(q, k, v, off, off, phi=PHI_SILU, scale=1.0)
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(o[:, 0], [[s1 * 1, s1 * 2], [s1 * 3, s1 * 4]], rtol=1e-15)


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX, PHI_IDENTITY])
def test_window_wider_than_sequence_is_dense(phi):
    rng = np.random.default_rng(16)
    q, k, v, qo, ko = rand_problem(rng, [7, 12], [7, 12], H=1, D=4)
    dense, dl = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.4)
    wide, wl = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.4, window=(12, 12))
    np.testing.assert_array_equal(dense, wide)
    np.testing.assert_array_equal(dl, wl)


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_IDENTITY])
def test_elementwise_window_equals_numpy_masked(phi):
    """Element-wise phi under a band: masked pairs contribute nothing."""
    rng = np.random.default_rng(17)
    q, k, v, qo, ko = rand_problem(rng, [10, 20], [10, 20], H=2, D=3)
    o, _ = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.9, window=(4, 1))
    for b in range(2):
        L = qo[b + 1] - qo[b]
        m = band_mask(L, L, 4, 1)
        for h in range(2):
            s = 0.9 * q[qo[b]:qo[b + 1], h] @ k[ko[b]:ko[b + 1], h].T
            p = silu_np(s) if phi == PHI_SILU else s
            ref = np.where(m, p, 0.0) @ v[ko[b]:ko[b + 1], h]
            np.testing.assert_allclose(o[qo[b]:qo[b + 1], h], ref, rtol=1e-12, atol=1e-13)


def test_gate_limits_and_add_equivalence():
    """A gate of G = +40 is log sigma = -4e-18: indistinguishable from no bias.
    A gate equals an additive bias of torch's logsigmoid(G)."""
    rng = np.random.default_rng(18)
    q, k, v, qo, ko = rand_problem(rng, [8, 3], [9, 16], H=2, D=4)
    none, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=0.5)
    g40 = np.full((2, ko[-1]), 40.0)
    gated, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=0.5, bias=g40,
                              bias_kind=BIAS_GATE)
    np.testing.assert_allclose(gated, none, rtol=1e-15, atol=1e-15)
    g = rng.standard_normal((2, ko[-1])) * 4
    ls = torch.nn.functional.logsigmoid(torch.tensor(g)).numpy()
    for phi in (PHI_SOFTMAX, PHI_SILU):
        a, la = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.5, bias=g, bias_kind=BIAS_GATE)
        b_, lb = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.5, bias=ls, bias_kind=BIAS_ADD)
        np.testing.assert_allclose(a, b_, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(la, lb, rtol=1e-13, atol=1e-14)


def test_softmax_shift_invariance_of_bias():
    """Adding one constant to every key's bias leaves softmax O unchanged."""
    rng = np.random.default_rng(19)
    q, k, v, qo, ko = rand_problem(rng, [6], [10], H=1, D=4)
    g = rng.standard_normal((1, 10))
    a, la = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=1.0, bias=g, bias_kind=BIAS_ADD)
    b_, lb = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=1.0, bias=g + 3.25,
                            bias_kind=BIAS_ADD)
    np.testing.assert_allclose(a, b_, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lb - la, 3.25, rtol=1e-13)


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX])
def test_jagged_batch_is_concatenation(phi):
    rng = np.random.default_rng(20)
    ql, kl = [5, 0, 13, 1], [3, 4, 9, 1]
    q, k, v, qo, ko = rand_problem(rng, ql, kl, H=2, D=3)
    g = rng.standard_normal((2, ko[-1]))
    o, lse = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.3, bias=g, bias_kind=BIAS_GATE)
    for b in range(4):
        sq, sk = slice(qo[b], qo[b + 1]), slice(ko[b], ko[b + 1])
        o1, l1 = oracle.forward(q[sq], k[sk], v[sk], [0, ql[b]], [0, kl[b]], phi=phi, scale=0.3,
                                bias=np.ascontiguousarray(g[:, sk]), bias_kind=BIAS_GATE)
        np.testing.assert_array_equal(o[sq], o1)
        np.testing.assert_array_equal(lse[:, sq], l1)


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX])
def test_key_permutation_equivariance(phi):
    """Permuting (K_j, V_j, G_j) jointly leaves O unchanged (no window)."""
    rng = np.random.default_rng(21)
    q, k, v, qo, ko = rand_problem(rng, [11], [17], H=2, D=5)
    g = rng.standard_normal((2, 17))
    perm = rng.permutation(17)
    a, la = oracle.forward(q, k, v, qo, ko, phi=phi, scale=0.6, bias=g, bias_kind=BIAS_GATE)
    b_, lb = oracle.forward(q, k[perm], v[perm], qo, ko, phi=phi, scale=0.6,
                            bias=np.ascontiguousarray(g[:, perm]), bias_kind=BIAS_GATE)
    np.testing.assert_allclose(a, b_, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=1e-13, atol=1e-13)


def test_empty_rows_and_samples():
    """No visible key: O = 0 and LSE = -inf.  Empty samples produce nothing."""
    rng = np.random.default_rng(22)
    q, k, v, qo, ko = rand_problem(rng, [0, 4, 3, 5], [2, 0, 3, 4], H=1, D=3)
    o, lse = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=1.0)
    np.testing.assert_array_equal(o[qo[1]:qo[2]], 0.0)            # Lk = 0
    assert np.all(np.isneginf(lse[0, qo[1]:qo[2]]))
    # band that lies entirely to the right of the keys for late rows
    o, lse = oracle.forward(q, k, v, qo, ko, phi=PHI_SOFTMAX, scale=1.0, window=(0, 0))
    # sample 3 has Lq = 5 > Lk = 4: row 4 sees key 4, which does not exist
    assert np.all(o[qo[3] + 4] == 0.0) and np.isneginf(lse[0, qo[3] + 4])
    o, _ = oracle.forward(q, k, v, qo, ko, phi=PHI_SILU, scale=1.0)
    np.testing.assert_array_equal(o[qo[1]:qo[2]], 0.0)


def brute_force_forward(q, k, v, Lq, Lk, phi, scale, window, beta):
    """Hand-expanded sums with Python floats and the math module."""
    wl, wr = window
    D = len(q[0])
    out = []
    lse = []
    for i in range(Lq):
        s = {}
        for j in range(Lk):
            if (wl >= 0 and j < i - wl) or (wr >= 0 and j > i + wr):
                continue
            dot = 0.0
            for d in range(D):
                dot += q[i][d] * k[j][d]
            s[j] = scale * dot + beta[j]
        if phi == PHI_SOFTMAX:
            if not s:
                out.append([0.0] * D)
                lse.append(-math.inf)
                continue
            m = max(s.values())
            z = sum(math.exp(x - m) for x in s.values())
            w = {j: math.exp(x - m) / z for j, x in s.items()}
            lse.append(m + math.log(z))
        elif phi == PHI_SILU:
            w = {j: x / (1.0 + math.exp(-x)) for j, x in s.items()}
        else:
            w = dict(s)
        out.append([sum(w[j] * v[j][d] for j in w) for d in range(D)])
    return out, lse


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX, PHI_IDENTITY])
@pytest.mark.parametrize("window", [(-1, -1), (1, 0), (0, 1)])
def test_brute_force_tiny(phi, window):
    rng = np.random.default_rng(23)
    for Lq in (1, 2, 3):
        for Lk in (1, 2, 3):
            D = 1 + (Lq + Lk) % 4
            q = rng.standard_normal((Lq, 1, D))
            k = rng.standard_normal((Lk, 1, D))
            v = rng.standard_normal((Lk, 1, D))
            g = rng.standard_normal((1, Lk))
            o, lse = oracle.forward(q, k, v, [0, Lq], [0, Lk], phi=phi, scale=0.8,
                                    window=window, bias=g, bias_kind=BIAS_ADD)
            ref, rlse = brute_force_forward(q[:, 0].tolist(), k[:, 0].tolist(), v[:, 0].tolist(),
                                            Lq, Lk, phi, 0.8, window, g[0].tolist())
            np.testing.assert_allclose(o[:, 0], np.array(ref).reshape(Lq, D), rtol=1e-13,
                                       atol=1e-14)
            if phi == PHI_SOFTMAX:
                np.testing.assert_allclose(lse[0], rlse, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------- backward pins

def _loss(q, k, v, dout, qo, ko, phi, scale, window, g, bias_kind):
    o, _ = oracle.forward(q, k, v, qo, ko, phi=phi, scale=scale, window=window, bias=g,
                          bias_kind=bias_kind)
    return float(np.sum(o * dout))


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX, PHI_IDENTITY, PHI_GELU])
@pytest.mark.parametrize("bias_kind,window", [(BIAS_NONE, (-1, -1)), (BIAS_ADD, (1, 0)),
                                              (BIAS_GATE, (-1, -1)), (BIAS_GATE, (0, 2))])
def test_finite_difference_gradients(phi, bias_kind, window):
    """Central differences of L = sum(O * dO) in fp64, h = 1e-6, every input."""
    rng = np.random.default_rng(24)
    H, D = 2, 3
    q, k, v, qo, ko = rand_problem(rng, [3, 2], [3, 4], H=H, D=D)
    dout = rng.standard_normal(q.shape)
    g = rng.standard_normal((H, ko[-1])) if bias_kind else None
    args = dict(phi=phi, scale=0.7, window=window)
    dq, dk, dv, db = oracle.backward(q, k, v, dout, qo, ko, bias=g, bias_kind=bias_kind, **args)
    eps = 1e-6
    for x, grad in ((q, dq), (k, dk), (v, dv)) + (((g, db),) if bias_kind else ()):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + eps
            lp = _loss(q, k, v, dout, qo, ko, args["phi"], 0.7, window, g, bias_kind)
            x[idx] = old - eps
            lm = _loss(q, k, v, dout, qo, ko, args["phi"], 0.7, window, g, bias_kind)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX, PHI_GELU])
def test_backward_matches_torch_autograd(phi):
    """Gradients equal torch autograd (fp64, CPU) of the formula built from
    torch's own softmax / silu / logsigmoid / matmul, with a band and gate."""
    rng = np.random.default_rng(25)
    H, D = 2, 6
    ql, kl = [9, 14], [9, 14]
    q, k, v, qo, ko = rand_problem(rng, ql, kl, H=H, D=D)
    dout = rng.standard_normal(q.shape)
    g = rng.standard_normal((H, ko[-1]))
    wl, wr = 3, 1
    dq, dk, dv, db = oracle.backward(q, k, v, dout, qo, ko, phi=phi, scale=0.45, window=(wl, wr),
                                     bias=g, bias_kind=BIAS_GATE)
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    tg = torch.tensor(g, requires_grad=True)
    outs = []
    for b in range(2):
        Lq, Lk = ql[b], kl[b]
        vis = torch.tensor(band_mask(Lq, Lk, wl, wr))
        rows = []
        for h in range(H):
            Q = tq[qo[b]:qo[b + 1], h]
            K = tk[ko[b]:ko[b + 1], h]
            V = tv[ko[b]:ko[b + 1], h]
            s = 0.45 * Q @ K.T + torch.nn.functional.logsigmoid(tg[h, ko[b]:ko[b + 1]])[None]
            if phi == PHI_SOFTMAX:
                p = torch.softmax(s.masked_fill(~vis, -math.inf), dim=1)
            elif phi == PHI_GELU:
                p = torch.nn.functional.gelu(s, approximate="none") * vis
            else:
                p = torch.nn.functional.silu(s) * vis
            rows.append(p @ V)
        outs.append(torch.stack(rows, 1))
    O = torch.cat(outs, 0)
    (O * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db, tg.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_softmax_score_gradients_sum_to_zero():
    """For softmax, sum_j dS_ij = 0 for every row; with an additive bias the
    bias gradient is sum_i dS_ij, so it sums to zero over each sample's keys."""
    rng = np.random.default_rng(26)
    q, k, v, qo, ko = rand_problem(rng, [7, 5], [12, 3], H=3, D=4)
    dout = rng.standard_normal(q.shape)
    g = rng.standard_normal((3, ko[-1]))
    _, _, _, db = oracle.backward(q, k, v, dout, qo, ko, phi=PHI_SOFTMAX, scale=1.0, bias=g,
                                  bias_kind=BIAS_ADD)
    for b in range(2):
        np.testing.assert_allclose(db[:, ko[b]:ko[b + 1]].sum(1), 0.0, atol=1e-12)


def test_backward_empty_samples_give_zero():
    rng = np.random.default_rng(27)
    q, k, v, qo, ko = rand_problem(rng, [0, 4], [5, 0], H=1, D=2)
    dout = rng.standard_normal(q.shape)
    dq, dk, dv, _ = oracle.backward(q, k, v, dout, qo, ko, phi=PHI_SOFTMAX, scale=1.0)
    assert np.all(dq == 0) and np.all(dk == 0) and np.all(dv == 0)


def test_bf16_inputs_widen_exactly():
    """Workload tensors are bf16; the oracle sees their exact values."""
    from workloads import make_workload
    w = make_workload(1)
    qd = w.q.to(torch.float64)
    assert torch.equal(qd.to(torch.bfloat16), w.q)
    o, _ = oracle.forward_workload(w)
    assert o.shape == tuple(w.q.shape) and np.isfinite(o).all()
