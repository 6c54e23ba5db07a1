"""The oracles reproduce their stored records (tests/golden/, written by
tests/golden/make_golden.py from the oracles only)."""
import json
import os

import numpy as np

import oracle
from workloads import make_workload

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_silu_fwd.json")


def test_tiny_silu_golden_record():
    with open(GOLDEN) as f:
        g = json.load(f)
    w = make_workload(1)
    assert [int(x) for x in w.q_lens] == g["q_lens"]
    assert [int(x) for x in w.kv_lens] == g["kv_lens"]
    o, _ = oracle.forward_workload(w)
    for r, h, d, val in g["samples"]:
        assert abs(o[r, h, d] - val) <= 1e-12 * max(1.0, abs(val))
    for b in range(w.B):
        for h in range(w.H):
            n = np.linalg.norm(o[w.q_offsets[b]:w.q_offsets[b + 1], h])
            assert abs(n - g["norms"][b][h]) <= 1e-12 * n


HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_rotary_golden_record():
    from oracle import rotary
    from workloads import EVENT_TIME_SCALE, event_times
    with open(os.path.join(HERE, "rotary_small.json")) as f:
        g = json.load(f)
    lens = g["lens"]
    times = event_times(lens, 31)
    assert [int(t) for t in times] == g["times"]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ang = rotary.angles(off, times, 8, g["time_scale"])
    np.testing.assert_allclose(ang, np.array(g["angles"]), rtol=1e-13, atol=1e-13)
    w = make_workload(4, seed=31, q_lens=lens, kv_lens=lens, H=2, D=8, window=(3, 0),
                      scale=1.0 / np.sqrt(8))
    o, lse = rotary.forward(w.q, w.k, w.v, w.q_offsets, w.kv_offsets, ang, ang, phi=w.phi,
                            scale=w.scale, window=(w.window_left, w.window_right))
    for r, h, d, val in g["forward"]["samples"]:
        assert abs(o[r, h, d] - val) <= 1e-12 * max(1.0, abs(val))
    np.testing.assert_allclose(lse, np.array(g["forward"]["lse"]), rtol=1e-12, atol=1e-12)


def test_sumkron_golden_record():
    from oracle import sumkron
    from workloads import make_sumkron
    with open(os.path.join(HERE, "sumkron_small.json")) as f:
        g = json.load(f)
    x, a, wk = make_sumkron(3, 64, 32, 128, 4, seed=77)
    y = sumkron.forward(x, a, wk)
    for b, t, e, val in g["samples"]:
        assert abs(y[b, t, e] - val) <= 1e-12 * max(1.0, abs(val))
    assert abs(np.linalg.norm(y) - g["norm"]) <= 1e-12 * g["norm"]
