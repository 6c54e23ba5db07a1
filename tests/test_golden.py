"""The oracle reproduces its stored record for the tiny SiLU workload."""
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
