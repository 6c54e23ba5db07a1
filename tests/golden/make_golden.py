"""Writes tests/golden/tiny_silu_fwd.json from the fp64 oracle only.

The Kunlun pages print no worked example with numbers, so this fixture is an
oracle regression record for the tiny SiLU workload (B=4, H=2, D=32, query
lengths uniform in [1, 64], K/V length 16, scale 1/sqrt(32); Kunlun paper
review §2.3 "GDPA": the personalised FFN as attention with an element-wise
activation).  It stores the seeded lengths, 64 sampled output elements and the
per-(sample, head) Frobenius norms of O.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import make_workload  # noqa: E402


def main():
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
