"""Grouped forward: several problems with their own shapes, activations,
bands and biases in one call, as event-level personalisation runs them.

Each problem's output must equal gdpa_forward on that problem alone (the same
per-unit arithmetic, so bit for bit) and match the oracle.
"""
import copy

import numpy as np
import pytest
import torch

import oracle
from parity import compare, compare_lse
from workloads import (BIAS_ADD, BIAS_GATE, BIAS_NONE, PHI_GELU, PHI_IDENTITY, PHI_SILU,
                       PHI_SOFTMAX, make_workload)

pytestmark = pytest.mark.gpu

NAMES = {PHI_SILU: "silu", PHI_SOFTMAX: "softmax", PHI_IDENTITY: "identity", PHI_GELU: "gelu"}


def _problems():
    """(workload, head_phi or None) per problem."""
    out = []
    # D = 128, softmax, gate, causal band (the sliding-window shape)
    out.append((make_workload(4, seed=400, q_lens=[300, 1, 129], kv_lens=[300, 1, 129], H=3,
                              window=(127, 0), bias=BIAS_GATE), None))
    # D = 128, SiLU, at most 64 keys (64-key blocks)
    out.append((make_workload(2, seed=401, q_lens=[200, 64, 7, 130], kv_lens=[64, 1, 33, 64],
                              H=2, D=128, phi=PHI_SILU, scale=1.0,
                              kv_std=1.0 / np.sqrt(128)), None))
    # D = 64, one activation per head, additive bias
    out.append((make_workload(2, seed=402, q_lens=[150, 90, 1], kv_lens=[200, 64, 300], H=4,
                              D=64, scale=1.0, kv_std=1.0 / np.sqrt(64), bias=BIAS_ADD),
                [PHI_SOFTMAX, PHI_SILU, PHI_GELU, PHI_IDENTITY]))
    # D = 128, softmax, no bias: shares a launch with the first problem
    out.append((make_workload(3, seed=403, q_lens=[32, 32, 32, 5, 250], kv_lens=[700, 128, 9, 1,
                                                                                   256], H=5),
                None))
    # a problem whose samples have no queries
    out.append((make_workload(2, seed=404, q_lens=[0, 0], kv_lens=[10, 3], H=2, D=64, scale=1.0,
                              kv_std=1.0 / np.sqrt(64)), None))
    return out


def _to_dev(w, head_phi):
    dev = torch.device("cuda")
    d = dict(q=w.q.to(dev), k=w.k.to(dev), v=w.v.to(dev),
             q_offsets=torch.tensor(w.q_offsets, dtype=torch.int32, device=dev),
             kv_offsets=torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev),
             bias=None if w.bias is None else w.bias.to(dev), phi=NAMES[w.phi], scale=w.scale,
             window=(w.window_left, w.window_right), bias_kind=w.bias_kind,
             max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv)
    if head_phi is not None:
        d["head_phi"] = [NAMES[x] for x in head_phi]
    return d


def test_grouped_equals_separate_calls_and_oracle(cuda_lib):
    probs = _problems()
    dev_probs = [_to_dev(w, hp) for w, hp in probs]
    outs, ws = cuda_lib.forward_grouped(dev_probs)
    assert cuda_lib.device_status(ws) == 0
    torch.cuda.synchronize()
    for (w, hp), d, (o, lse) in zip(probs, dev_probs, outs):
        # the same problem alone
        kw = {k: d[k] for k in ("phi", "scale", "window", "bias", "bias_kind", "max_seqlen_q",
                                "max_seqlen_kv")}
        if hp is not None:
            kw["head_phi"] = d["head_phi"]
        o1, lse1, ws1 = cuda_lib.forward(d["q"], d["k"], d["v"], d["q_offsets"],
                                         d["kv_offsets"], **kw)
        assert cuda_lib.device_status(ws1) == 0
        assert torch.equal(o, o1)
        heads = hp if hp is not None else [w.phi] * w.H
        for h, phi in enumerate(heads):
            if phi == PHI_SOFTMAX:
                assert torch.equal(lse[h], lse1[h])
        # and the oracle, head by head with that head's activation
        for phi in sorted(set(heads)):
            wp = copy.copy(w)
            wp.phi = phi
            ro, rlse = oracle.forward_workload(wp)
            for h in [i for i, x in enumerate(heads) if x == phi]:
                compare(f"O[h{h}]", o[:, h], ro[:, h])
                if phi == PHI_SOFTMAX:
                    compare_lse(lse[h], rlse[h])


def test_grouped_many_small_problems(cuda_lib):
    """Forty event-type problems of mixed shapes in one call."""
    rng = np.random.default_rng(405)
    probs = []
    for i in range(40):
        H = int(rng.integers(1, 5))
        D = int(rng.choice([32, 64, 128]))
        B = int(rng.integers(1, 4))
        ql = rng.integers(1, 200, B).tolist()
        kl = rng.integers(1, 150, B).tolist()
        phi = int(rng.choice([PHI_SOFTMAX, PHI_SILU]))
        if phi == PHI_SOFTMAX:
            w = make_workload(3, seed=500 + i, q_lens=ql, kv_lens=kl, H=H, D=D,
                              scale=1.0 / np.sqrt(D))
        else:
            w = make_workload(2, seed=500 + i, q_lens=ql, kv_lens=kl, H=H, D=D, phi=phi,
                              scale=1.0, kv_std=1.0 / np.sqrt(D))
        probs.append((w, None))
    dev_probs = [_to_dev(w, None) for w, _ in probs]
    outs, ws = cuda_lib.forward_grouped(dev_probs)
    assert cuda_lib.device_status(ws) == 0
    torch.cuda.synchronize()
    for (w, _), (o, lse) in zip(probs, outs):
        ro, rlse = oracle.forward_workload(w)
        compare("O", o, ro)
        if w.phi == PHI_SOFTMAX:
            compare_lse(lse, rlse)


def test_grouped_with_rotary_problems(cuda_lib):
    """Problems with the rotary temporal embedding in a grouped call: each one
    equals its own single call (turned Q and K, bit for bit) and the oracle."""
    from oracle import rotary
    from workloads import EVENT_TIME_SCALE, event_times
    specs = [
        (make_workload(4, seed=410, q_lens=[300, 1, 129], kv_lens=[300, 1, 129], H=3,
                       window=(127, 0)), 1),
        (make_workload(4, seed=411, q_lens=[64, 500], kv_lens=[64, 500], H=2, D=64,
                       window=(31, 0), scale=1.0 / 8), 2),
        (make_workload(3, seed=412, q_lens=[32, 32], kv_lens=[200, 17], H=2), None),  # none
    ]
    dev_probs, angs = [], []
    for w, seed in specs:
        d = _to_dev(w, None)
        if seed is not None:
            times = event_times(w.q_lens, seed)
            table = cuda_lib.rotary_table(d["q_offsets"], torch.tensor(times, device="cuda"),
                                          w.D, EVENT_TIME_SCALE)
            d["rope"] = (table, table)
            angs.append(rotary.angles(w.q_offsets, times, w.D, EVENT_TIME_SCALE))
        else:
            angs.append(None)
        dev_probs.append(d)
    outs, ws = cuda_lib.forward_grouped(dev_probs)
    assert cuda_lib.device_status(ws) == 0
    torch.cuda.synchronize()
    for (w, _), d, a, (o, lse) in zip(specs, dev_probs, angs, outs):
        kw = {k: d[k] for k in ("phi", "scale", "window", "bias", "bias_kind", "max_seqlen_q",
                                "max_seqlen_kv")}
        o1, lse1, ws1 = cuda_lib.forward(d["q"], d["k"], d["v"], d["q_offsets"],
                                         d["kv_offsets"], rope=d.get("rope"), **kw)
        assert cuda_lib.device_status(ws1) == 0
        assert torch.equal(o, o1) and torch.equal(lse, lse1)
        if a is None:
            ro, _ = oracle.forward_workload(w)
        else:
            ro, _ = rotary.forward(w.q, w.k, w.v, w.q_offsets, w.kv_offsets, a, a, phi=w.phi,
                                   scale=w.scale, window=(w.window_left, w.window_right))
        compare("O", o, ro)


def test_grouped_at_the_entry_limit(cuda_lib):
    """One launch group holding 16384 entries (its limit): two problems of the
    same class, 12000 + 4384 tiny samples."""
    rng = np.random.default_rng(420)
    probs = []
    for i, B in enumerate((12000, 4384)):
        ql = rng.integers(0, 9, B).tolist()
        kl = rng.integers(1, 17, B).tolist()
        w = make_workload(2, seed=420 + i, q_lens=ql, kv_lens=kl, H=2, D=32, phi=PHI_SILU,
                          scale=1.0, kv_std=1.0 / np.sqrt(32))
        probs.append((w, None))
    dev_probs = [_to_dev(w, None) for w, _ in probs]
    outs, ws = cuda_lib.forward_grouped(dev_probs)
    assert cuda_lib.device_status(ws) == 0
    torch.cuda.synchronize()
    for (w, _), (o, _) in zip(probs, outs):
        ro, _ = oracle.forward_workload(w)
        compare("O", o, ro)


def _kw(d):
    return {k: d[k] for k in ("phi", "scale", "window", "bias", "bias_kind", "max_seqlen_q",
                              "max_seqlen_kv")}


def test_backward_grouped_equals_separate_calls_and_oracle(cuda_lib):
    """The grouped backward gives each problem exactly gdpa_backward's
    gradients (bit for bit) and matches the oracle."""
    items = []
    for i, (w, hp) in enumerate(_problems()):
        if hp is not None:
            continue
        d = _to_dev(w, None)
        o, lse, ws0 = cuda_lib.forward(d["q"], d["k"], d["v"], d["q_offsets"], d["kv_offsets"],
                                       **_kw(d))
        assert cuda_lib.device_status(ws0) == 0
        g = torch.Generator().manual_seed(600 + i)
        dout = (torch.randn(w.q.shape, generator=g) * 0.25).to(torch.bfloat16)
        d.update(o=o, lse=lse, dout=dout.cuda())
        items.append((w, d, dout))
    outs, ws = cuda_lib.backward_grouped([d for _, d, _ in items])
    assert cuda_lib.device_status(ws) == 0
    torch.cuda.synchronize()
    for (w, d, dout), (dq, dk, dv) in zip(items, outs):
        dq1, dk1, dv1, ws1 = cuda_lib.backward(d["q"], d["k"], d["v"], d["o"], d["dout"],
                                               d["lse"], d["q_offsets"], d["kv_offsets"],
                                               **_kw(d))
        assert cuda_lib.device_status(ws1) == 0
        assert torch.equal(dq, dq1) and torch.equal(dk, dk1) and torch.equal(dv, dv1)
        rdq, rdk, rdv, _ = oracle.backward_workload(w, dout=dout)
        compare("dQ", dq, rdq)
        compare("dK", dk, rdk)
        compare("dV", dv, rdv)
