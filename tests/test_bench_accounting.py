"""The bench's useful-FLOP and algorithmic-byte counts, pinned by brute force
on small workloads (host logic only: no GDPA arithmetic, no GPU)."""
import json
import os

import numpy as np
import pytest

import bench
from workloads import make_workload


def brute_pairs(w) -> int:
    """Visible (query, key) pairs per head, one pair at a time: query i of a
    sample sees key j iff j is inside the sample and, where a side of the band
    is set, i - wl <= j <= i + wr."""
    n = 0
    for Lq, Lk in zip(w.q_lens, w.kv_lens):
        for i in range(int(Lq)):
            for j in range(int(Lk)):
                if w.window_left >= 0 and j < i - w.window_left:
                    continue
                if w.window_right >= 0 and j > i + w.window_right:
                    continue
                n += 1
    return n


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(q_lens=[1, 130, 0, 257], kv_lens=[64, 64, 64, 64])),
    (3, dict(q_lens=[32, 32, 32], kv_lens=[128, 300, 0])),
    (4, dict(q_lens=[200, 1, 0, 333], kv_lens=[200, 1, 0, 333])),
    (4, dict(q_lens=[50, 260], kv_lens=[50, 260], window=(3, 5))),
    (5, dict(q_lens=[256, 7], kv_lens=[256, 256])),
])
def test_visible_pairs_and_flops_match_brute_force(cfg, kw):
    w = make_workload(cfg, seed=11, **kw)
    pairs = brute_pairs(w)
    assert int(bench.visible_pairs_per_sample(w).sum()) == pairs
    fwd, bwd = bench.useful_flops(w, backward=True)
    # QK^T and PV: two multiply-adds per pair, head and feature
    assert fwd == 4.0 * w.D * w.H * pairs
    # dV, dP, dQ, dK: four more products of the same size
    assert bwd == 2 * fwd
    assert bench.useful_flops(w, backward=False)[1] == 0.0


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_algorithmic_bytes_are_the_tensors_read_and_written(cfg):
    w = make_workload(cfg, B=5, seed=12, with_dout=True)
    bf16 = 2
    q, k, v = w.q.numel() * bf16, w.k.numel() * bf16, w.v.numel() * bf16
    o = q                                     # O has Q's shape
    gate = w.bias.numel() * 4 if w.bias is not None else 0
    lse = 4 * w.H * w.total_q if w.phi == 1 else 0
    fwd, bwd = bench.algorithmic_bytes(w, backward=True)
    assert fwd == q + k + v + o + gate + lse
    # read Q, K, V, O, dO (and the gate, the LSE); write dQ, dK, dV (and the gate's gradient)
    assert bwd == (q + k + v + o + o) + (q + k + v) + 2 * gate + lse


def test_traffic_records_are_complete_and_hash_gated():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        d = json.load(f)
    for kernel, rec in d.items():
        if kernel.startswith("_"):
            continue
        assert kernel in bench.KERNEL_SOURCES
        assert rec["samples"] > 0
        assert rec["dram_bytes"] == pytest.approx(sum(rec["kernels"].values()))
        got = bench.measured_traffic(kernel, 2 * rec["samples"])
        if rec["source_hash"] == bench.kernel_source_hash(kernel):
            assert got == pytest.approx(2 * rec["dram_bytes"])  # scaled by samples
        else:
            assert got is None  # a stale capture is never reported
