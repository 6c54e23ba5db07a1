"""Writes the oracle regression records in tests/golden/ from the fp64 oracle only.

The Kunlun pages print no worked example with numbers, so these fixtures are
oracle regression records (the oracles are pinned against the mathematics in
tests/test_oracle*.py; these files catch later changes to their arithmetic):

* tiny_silu_fwd.json -- the tiny SiLU workload (B=4, H=2, D=32, query lengths
  uniform in [1, 64], K/V length 16, scale 1/sqrt(32); Kunlun paper review
  §2.3 "GDPA": the personalised FFN as attention with an element-wise
  activation): the seeded lengths, 64 sampled output elements and the
  per-(sample, head) Frobenius norms of O.
* rotary_small.json -- the rotary temporal embedding (Kunlun paper review
  §2.2): angles of a small jagged sequence with seeded event times, and a
  rotary self-attention forward on it (sampled outputs).
* sumkron_small.json -- SumKronLinear (Kunlun paper review §2.4) on a small
  seeded case: sampled outputs.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import make_workload  # noqa: E402


HERE = os.path.dirname(os.path.abspath(__file__))


def rotary_record():
    from oracle import rotary
    from workloads import EVENT_TIME_SCALE, event_times
    lens = [5, 1, 12]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    times = event_times(lens, 31)
    ang = rotary.angles(off, times, 8, EVENT_TIME_SCALE)
    w = make_workload(4, seed=31, q_lens=lens, kv_lens=lens, H=2, D=8, window=(3, 0),
                      scale=1.0 / np.sqrt(8))
    a = rotary.angles(w.q_offsets, times, 8, EVENT_TIME_SCALE)
    o, lse = rotary.forward(w.q, w.k, w.v, w.q_offsets, w.kv_offsets, a, a, phi=w.phi,
                            scale=w.scale, window=(w.window_left, w.window_right))
    rng = np.random.default_rng(4321)
    idx = [(int(rng.integers(o.shape[0])), int(rng.integers(2)), int(rng.integers(8)))
           for _ in range(24)]
    return {
        "source": "fp64 oracle (oracle/rotary.py); reading of the Kunlun paper review §2.2",
        "lens": lens, "times": [int(t) for t in times], "time_scale": EVENT_TIME_SCALE,
        "angles": ang.tolist(),
        "forward": {"workload": "sliding_window_softmax_fwd shapes, seed 31, H=2, D=8, band (3, 0)",
                    "samples": [[r, h, d, float(o[r, h, d])] for r, h, d in idx],
                    "lse": lse.tolist()},
    }


def sumkron_record():
    from oracle import sumkron
    from workloads import make_sumkron
    x, a, wk = make_sumkron(3, 64, 32, 128, 4, seed=77)
    y = sumkron.forward(x, a, wk)
    rng = np.random.default_rng(99)
    idx = [(int(rng.integers(3)), int(rng.integers(32)), int(rng.integers(128)))
           for _ in range(32)]
    return {
        "source": "fp64 oracle (oracle/sumkron.py); reading of the Kunlun paper review §2.4",
        "case": "make_sumkron(B=3, S=64, T=32, D=128, k=4, seed=77)",
        "samples": [[b, t, e, float(y[b, t, e])] for b, t, e in idx],
        "norm": float(np.linalg.norm(y)),
    }


def main():
    for name, rec in (("rotary_small.json", rotary_record()),
                      ("sumkron_small.json", sumkron_record())):
        path = os.path.join(HERE, name)
        with open(path, "w") as f:
            json.dump(rec, f, indent=1)
        print("wrote", path)
    w = make_workload(1)
    o, _ = oracle.forward_workload(w)
    rng = np.random.default_rng(1234)
    idx = [(int(rng.integers(w.total_q)), int(rng.integers(w.H)), int(rng.integers(w.D)))
           for _ in range(64)]
    norms = [[float(np.linalg.norm(o[w.q_offsets[b]:w.q_offsets[b + 1], h]))
              for h in range(w.H)] for b in range(w.B)]
    out = {
        "workload": "tiny_silu_fwd (seed 1)",
        "source": "fp64 oracle (oracle/gdpa_oracle.c); definition from the Kunlun paper "
                  "review §2.3 GDPA / Fig. 2",
        "q_lens": [int(x) for x in w.q_lens],
        "kv_lens": [int(x) for x in w.kv_lens],
        "samples": [[r, h, d, float(o[r, h, d])] for r, h, d in idx],
        "norms": norms,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_silu_fwd.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
