"""Rotary temporal embedding on the GPU vs the fp64 oracle (``oracle.rotary``):
the rotation table, and the forward with Q and K turned in shared memory."""
import numpy as np
import pytest
import torch

import oracle
from oracle import rotary
from parity import LSE_ABS, compare
from workloads import (BIAS_GATE, BIAS_NONE, EVENT_TIME_SCALE, PHI_GELU, PHI_SILU, PHI_SOFTMAX,
                       event_times, make_workload)

pytestmark = pytest.mark.gpu


def _dev(x, dtype=None):
    return torch.as_tensor(x, dtype=dtype).cuda()


def gpu_table(gdpa, offsets, times, D, **kw):
    t = gdpa.rotary_table(_dev(offsets, torch.int32), _dev(times, torch.int64), D,
                          EVENT_TIME_SCALE, **kw)
    torch.cuda.synchronize()
    return t


def table_cos_sin(t):
    h = t.view(torch.float16).float().cpu().numpy()  # [total, D] as (cos, sin) pairs
    return h[:, 0::2], h[:, 1::2]


@pytest.mark.parametrize("D", [32, 64, 128])
def test_table_matches_oracle_angles(cuda_lib, D):
    lens = [1, 5, 0, 300, 2048]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    times = event_times(lens, seed=D)
    c, s = table_cos_sin(gpu_table(cuda_lib, off, times, D))
    a = rotary.angles(off, times, D, EVENT_TIME_SCALE)
    # fp16 rounding of values in [-1, 1] (half an ulp <= 2^-12) plus the fp32
    # cosine and sine of the reduced angle
    np.testing.assert_allclose(c, np.cos(a), rtol=0, atol=5e-4)
    np.testing.assert_allclose(s, np.sin(a), rtol=0, atol=5e-4)


def test_table_custom_frequencies(cuda_lib):
    D = 64
    lens = [7, 130]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    times = event_times(lens, seed=3)
    rng = np.random.default_rng(9)
    th = rng.uniform(0, 1, D // 2).astype(np.float32)
    ph = rng.uniform(0, 2, D // 2).astype(np.float32)
    c, s = table_cos_sin(gpu_table(cuda_lib, off, times, D, theta=th, phi=ph))
    a = rotary.angles(off, times, D, EVENT_TIME_SCALE, th.astype(np.float64), ph.astype(np.float64))
    np.testing.assert_allclose(c, np.cos(a), atol=5e-4)
    np.testing.assert_allclose(s, np.sin(a), atol=5e-4)


def check_lse(lse, rlse, w, aq, ak):
    """LSE against the oracle with a bound derived from the rotated operands.

    The MMA takes the turned Q and K as bf16, so each turned element carries a
    relative error of up to 2^-8 (bf16 rounding) plus about 2^-10 (the fp16
    cosine and sine).  A score then moves by at most
    scale * 2 * (2^-8 + 2^-10) * sum_d |q'_d k'_d| (used here with 2^-6), and
    an LSE by at most the largest move of its row's scores; fp32 accumulation
    keeps the plain bound of 2e-3 on top.
    """
    got = lse.detach().cpu().double().numpy()
    ref = np.asarray(rlse)
    neg = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), neg), "LSE -inf pattern differs"
    qr = np.abs(rotary.rotate(w.q.double().numpy(), aq))
    kr = np.abs(rotary.rotate(w.k.double().numpy(), ak))
    bound = np.full(ref.shape, LSE_ABS)
    for b in range(w.B):
        qs = slice(int(w.q_offsets[b]), int(w.q_offsets[b + 1]))
        ks = slice(int(w.kv_offsets[b]), int(w.kv_offsets[b + 1]))
        if qs.stop == qs.start or ks.stop == ks.start:
            continue
        for h in range(w.H):
            m = (qr[qs, h] @ kr[ks, h].T).max(axis=1)
            bound[h, qs] += abs(w.scale) * 2.0 ** -6 * m
    err = np.where(neg, 0.0, np.abs(np.where(neg, 0.0, got) - np.where(neg, 0.0, ref)))
    assert (err <= bound).all(), f"LSE err {err.max():.3e} beyond bound (worst excess " \
        f"{(err - bound).max():.3e})"


FUSED = 4  # debug_flags bit 2: turn Q and K inside the attention kernel


def params(gdpa, w, tq, tk, debug_flags=0):
    return gdpa.make_params(w.B, w.H, w.D, int(w.q_offsets[-1]), int(w.kv_offsets[-1]),
                            phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right),
                            bias_kind=w.bias_kind, max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv,
                            debug_flags=debug_flags, rope=(tq, tk))


def run(gdpa, w, tq, tk, mode="streamed"):
    qo, ko = _dev(w.q_offsets, torch.int32), _dev(w.kv_offsets, torch.int32)
    bias = w.bias.cuda() if w.bias is not None else None
    p = params(gdpa, w, tq, tk, FUSED if mode == "fused" else 0)
    o, lse, ws = gdpa.forward(w.q.cuda(), w.k.cuda(), w.v.cuda(), qo, ko, bias=bias, params=p)
    assert gdpa.device_status(ws) == 0
    torch.cuda.synchronize()
    return o, lse


def tables(gdpa, w, seed, same_sequence):
    """Self-attention (same_sequence) shares one table; otherwise queries and
    keys have their own times.  Returns the device tables and oracle angles."""
    tq_np = event_times(w.q_lens, seed)
    tk_np = tq_np if same_sequence else event_times(w.kv_lens, seed + 1)
    tq = gpu_table(gdpa, w.q_offsets, tq_np, w.D)
    tk = tq if same_sequence else gpu_table(gdpa, w.kv_offsets, tk_np, w.D)
    aq = rotary.angles(w.q_offsets, tq_np, w.D, EVENT_TIME_SCALE)
    ak = rotary.angles(w.kv_offsets, tk_np, w.D, EVENT_TIME_SCALE)
    return tq, tk, aq, ak


def check(gdpa, w, seed, same_sequence, mode="streamed"):
    tq, tk, aq, ak = tables(gdpa, w, seed, same_sequence)
    o, lse = run(gdpa, w, tq, tk, mode)
    ro, rlse = rotary.forward(w.q, w.k, w.v, w.q_offsets, w.kv_offsets, aq, ak, phi=w.phi,
                              scale=w.scale, window=(w.window_left, w.window_right),
                              bias=w.bias, bias_kind=w.bias_kind)
    compare("O", o, ro)
    if w.phi == PHI_SOFTMAX:
        check_lse(lse, rlse, w, aq, ak)
    return o


# sliding-window self-attention is where the pages use temporal rotary; the
# band keeps every key block streamed through the ring
MODES = ["streamed", "fused"]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("window", [(127, 0), (40, 40), (-1, -1)])
def test_self_attention(cuda_lib, D, window, mode):
    ql = [1, 60, 200, 333, 520, 129]
    w = make_workload(4, seed=70 + D, q_lens=ql, kv_lens=ql, D=D, window=window,
                      scale=1.0 / np.sqrt(D))
    check(cuda_lib, w, seed=D, same_sequence=True, mode=mode)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("phi", [PHI_SILU, PHI_GELU, PHI_SOFTMAX])
@pytest.mark.parametrize("bias", [BIAS_NONE, BIAS_GATE])
def test_activations_and_gate(cuda_lib, phi, bias, mode):
    ql = [300, 17, 256, 129]
    kl = [200, 64, 256, 1]
    extra = {} if phi == PHI_SOFTMAX else dict(scale=1.0, kv_std=1.0 / np.sqrt(128))
    w = make_workload(5, seed=80 + phi + bias, q_lens=ql, kv_lens=kl, phi=phi, bias=bias,
                      with_dout=False, **extra)
    check(cuda_lib, w, seed=5, same_sequence=False, mode=mode)


@pytest.mark.parametrize("kv_len", [64, 256, 700])  # 64-key blocks; resident ring; streamed
def test_resident_and_streamed_keys(cuda_lib, kv_len):
    """In the kernel, a unit whose key blocks stay in the ring for all its query
    tiles turns them once; streamed blocks are turned at every load."""
    ql = [600, 130, 5]
    kl = [kv_len, kv_len, kv_len]
    w = make_workload(3, seed=90, q_lens=ql, kv_lens=kl, H=2, D=128)
    check(cuda_lib, w, seed=11, same_sequence=False, mode="fused")


def test_streamed_and_fused_agree(cuda_lib):
    """Both turn the same bf16 inputs with the same table and round the turned
    values to bf16 the same way, so the attention sees identical operands."""
    ql = [200, 513, 64]
    w = make_workload(4, seed=14, q_lens=ql, kv_lens=ql)
    tq, tk, _, _ = tables(cuda_lib, w, 14, True)
    o1, l1 = run(cuda_lib, w, tq, tk, "streamed")
    o2, l2 = run(cuda_lib, w, tq, tk, "fused")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("D", [32, 64, 128])
def test_apply_and_inverse(cuda_lib, D):
    lens = [3, 400, 129]
    w = make_workload(4, seed=15 + D, q_lens=lens, kv_lens=lens, H=3, D=D)
    tq, _, aq, _ = tables(cuda_lib, w, 15, True)
    x = w.q.cuda()
    y = cuda_lib.rotary_apply(x, tq)
    compare("turned", y, rotary.rotate(w.q.double().numpy(), aq))
    back = cuda_lib.rotary_apply(y, tq, inverse=True)
    compare("turned back", back, w.q.double().numpy())
    z = x.clone()
    cuda_lib.rotary_apply(z, tq, out=z)  # in place
    torch.cuda.synchronize()
    assert torch.equal(z, y)


# -------------------------------------------------- backward
def gpu_backward(gdpa, w, tq, tk):
    dev = torch.device("cuda")
    qo, ko = _dev(w.q_offsets, torch.int32), _dev(w.kv_offsets, torch.int32)
    bias = w.bias.cuda() if w.bias is not None else None
    p = params(gdpa, w, tq, tk)
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    o, lse, _ = gdpa.forward(q, k, v, qo, ko, bias=bias, params=p)
    dbias = (torch.empty((w.H, int(w.kv_offsets[-1])), dtype=torch.float32, device=dev)
             if bias is not None else None)
    dq, dk, dv, ws = gdpa.backward(q, k, v, o, w.dout.cuda(), lse, qo, ko, bias=bias,
                                   dbias=dbias, params=p)
    assert gdpa.device_status(ws) == 0
    torch.cuda.synchronize()
    return dq, dk, dv, dbias


@pytest.mark.parametrize("phi", [PHI_SOFTMAX, PHI_SILU])
@pytest.mark.parametrize("window", [(127, 0), (-1, -1)])
def test_backward_self_attention(cuda_lib, phi, window):
    ql = [1, 60, 200, 333, 129]
    extra = dict(dout_std=0.125) if phi == PHI_SOFTMAX else dict(
        scale=1.0, kv_std=1.0 / np.sqrt(128), dout_std=0.125)
    w = make_workload(4, seed=16, q_lens=ql, kv_lens=ql, phi=phi, window=window, with_dout=True,
                      **extra)
    tq, tk, aq, ak = tables(cuda_lib, w, 16, True)
    dq, dk, dv, _ = gpu_backward(cuda_lib, w, tq, tk)
    rdq, rdk, rdv, _ = rotary.backward(w.q, w.k, w.v, w.dout, w.q_offsets, w.kv_offsets, aq, ak,
                                       phi=w.phi, scale=w.scale,
                                       window=(w.window_left, w.window_right))
    compare("dQ", dq, rdq)
    compare("dK", dk, rdk)
    compare("dV", dv, rdv)


def test_backward_gate_cross_sequences(cuda_lib):
    ql = [300, 17, 256]
    kl = [200, 64, 256]
    w = make_workload(5, seed=17, q_lens=ql, kv_lens=kl, bias=BIAS_GATE, with_dout=True,
                      dout_std=0.125)
    tq, tk, aq, ak = tables(cuda_lib, w, 17, False)
    dq, dk, dv, dg = gpu_backward(cuda_lib, w, tq, tk)
    rdq, rdk, rdv, rdg = rotary.backward(w.q, w.k, w.v, w.dout, w.q_offsets, w.kv_offsets, aq,
                                         ak, phi=w.phi, scale=w.scale, bias=w.bias,
                                         bias_kind=w.bias_kind)
    compare("dQ", dq, rdq)
    compare("dK", dk, rdk)
    compare("dV", dv, rdv)
    compare("dG", dg, rdg, max_abs=3e-2 * max(1.0, float(np.abs(rdg).max())), bf16_out=False)


def test_zero_frequencies_give_the_plain_forward(cuda_lib):
    """theta = phi = 0: every angle is 0, the turn is exact, and the result is
    bit-identical to the forward without rotation."""
    ql = [50, 300]
    w = make_workload(4, seed=12, q_lens=ql, kv_lens=ql, window=(127, 0))
    z = np.zeros(64, np.float32)
    tq = gpu_table(cuda_lib, w.q_offsets, event_times(ql, 4), 128, theta=z, phi=z)
    o, lse = run(cuda_lib, w, tq, tq)
    qo, ko = _dev(w.q_offsets, torch.int32), _dev(w.kv_offsets, torch.int32)
    o2, lse2, _ = cuda_lib.forward(w.q.cuda(), w.k.cuda(), w.v.cuda(), qo, ko, phi=w.phi,
                                   scale=w.scale, window=(127, 0), max_seqlen_q=w.max_q,
                                   max_seqlen_kv=w.max_kv)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_empty_samples(cuda_lib):
    ql = [0, 3, 0, 140]
    kl = [5, 0, 0, 140]
    w = make_workload(4, seed=13, q_lens=ql, kv_lens=kl, window=(-1, -1))
    check(cuda_lib, w, seed=13, same_sequence=False)


# -------------------------------------------------- full size, per-head activations
@pytest.mark.slow
def test_full_size_sliding_window_sampled(cuda_lib):
    """The sliding-window workload at full size (B=512) with the rotary
    embedding, forward and backward; samples spread over the batch (the
    shortest, the longest, the last, random ones) against the oracle one by
    one."""
    from workloads import subset
    w = make_workload(4, device="cuda", with_dout=True)
    times = event_times(w.q_lens, 4)
    tab = gpu_table(cuda_lib, w.q_offsets, times, w.D)
    qo = _dev(w.q_offsets, torch.int32)
    p = params(cuda_lib, w, tab, tab)
    o, lse, _ = cuda_lib.forward(w.q, w.k, w.v, qo, qo, params=p)
    dq, dk, dv, wsb = cuda_lib.backward(w.q, w.k, w.v, o, w.dout, lse, qo, qo, params=p)
    assert cuda_lib.device_status(wsb) == 0
    torch.cuda.synchronize()
    order = np.argsort(w.q_lens)
    picks = sorted({int(order[0]), int(order[-1]), w.B - 1, 0,
                    *np.random.default_rng(44).choice(w.B, 4, replace=False).tolist()})
    sub = subset(w, picks)
    for name in ("q", "k", "v", "dout"):
        setattr(sub, name, getattr(sub, name).cpu())
    stimes = np.concatenate([times[w.q_offsets[b]:w.q_offsets[b + 1]] for b in picks])
    ang = rotary.angles(sub.q_offsets, stimes, w.D, EVENT_TIME_SCALE)
    kw = dict(phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right))
    ro, rlse = rotary.forward(sub.q, sub.k, sub.v, sub.q_offsets, sub.kv_offsets, ang, ang, **kw)
    rdq, rdk, rdv, _ = rotary.backward(sub.q, sub.k, sub.v, sub.dout, sub.q_offsets,
                                       sub.kv_offsets, ang, ang, **kw)
    rows = torch.tensor(np.concatenate([np.arange(w.q_offsets[b], w.q_offsets[b + 1])
                                        for b in picks]), device="cuda")
    compare("O", o[rows], ro)
    compare("dQ", dq[rows], rdq)
    compare("dK", dk[rows], rdk)
    compare("dV", dv[rows], rdv)


def test_head_phi_with_rotary(cuda_lib):
    """A per-head activation vector with the rotary embedding: each head
    matches the oracle with its own activation, forward and backward."""
    import copy
    from workloads import PHI_IDENTITY
    ql = [200, 17, 129]
    heads = [PHI_SOFTMAX, PHI_SILU, PHI_GELU, PHI_IDENTITY]
    names = {PHI_SOFTMAX: "softmax", PHI_SILU: "silu", PHI_GELU: "gelu", PHI_IDENTITY: "identity"}
    w = make_workload(2, seed=18, q_lens=ql, kv_lens=ql, H=4, D=64, scale=1.0,
                      kv_std=1.0 / np.sqrt(64), window=(63, 0), with_dout=True, dout_std=0.125)
    tq, tk, aq, ak = tables(cuda_lib, w, 18, True)
    qo = _dev(w.q_offsets, torch.int32)
    p = cuda_lib.make_params(w.B, w.H, w.D, int(w.q_offsets[-1]), int(w.kv_offsets[-1]),
                             phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right),
                             max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv,
                             head_phi=[names[h] for h in heads], rope=(tq, tk))
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    o, lse, _ = cuda_lib.forward(q, k, v, qo, qo, params=p)
    dq, dk, dv, wsb = cuda_lib.backward(q, k, v, o, w.dout.cuda(), lse, qo, qo, params=p)
    assert cuda_lib.device_status(wsb) == 0
    torch.cuda.synchronize()
    for h, phi in enumerate(heads):
        wp = copy.copy(w)
        wp.phi = phi
        kw = dict(phi=phi, scale=w.scale, window=(w.window_left, w.window_right))
        ro, _ = rotary.forward(w.q, w.k, w.v, w.q_offsets, w.kv_offsets, aq, ak, **kw)
        rdq, rdk, rdv, _ = rotary.backward(w.q, w.k, w.v, w.dout, w.q_offsets, w.kv_offsets, aq,
                                           ak, **kw)
        compare(f"O[h{h}]", o[:, h], ro[:, h])
        compare(f"dQ[h{h}]", dq[:, h], rdq[:, h])
        compare(f"dK[h{h}]", dk[:, h], rdk[:, h])
        compare(f"dV[h{h}]", dv[:, h], rdv[:, h])
