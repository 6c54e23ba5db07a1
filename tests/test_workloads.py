"""The seeded input recipes do what the documentation says (no GDPA arithmetic
here): event times for the rotary embedding, SumKronLinear tensors."""
import math

import numpy as np
import torch

from workloads import event_times, make_sumkron


def test_event_times_recipe():
    lens = np.array([1, 0, 500, 2000, 37])
    t = event_times(lens, 5)
    assert t.dtype == np.int64 and len(t) == lens.sum()
    off = np.concatenate([[0], np.cumsum(lens)])
    gaps = []
    for b in range(len(lens)):
        s, e = off[b], off[b + 1]
        if e == s:
            continue
        seg = t[s:e]
        assert 1_704_067_200 <= seg[0] < 1_735_689_600  # starts in 2024
        d = np.diff(seg)
        assert (d >= 0).all()  # non-decreasing within a sample
        gaps.append(d)
    g = np.concatenate(gaps)
    zero = (g == 0).mean()
    assert 0.07 < zero < 0.13  # zero with probability 0.1
    nz = g[g > 0]
    assert nz.min() >= 1 and nz.max() <= 1e7
    # log-uniform between 1 s and 1e7 s: the mean of ln(gap) is ln(1e7) / 2
    assert abs(np.log(nz).mean() - math.log(1e7) / 2) < 0.3
    # seeded: the same seed gives the same times, another seed others
    assert (event_times(lens, 5) == t).all() and not (event_times(lens, 6) == t).all()


def test_sumkron_recipe_unit_variance():
    x, a, w = make_sumkron(8, 256, 32, 128, 4, seed=3)
    assert x.dtype == a.dtype == w.dtype == torch.bfloat16
    assert x.shape == (8, 256, 128) and a.shape == (4, 32, 256) and w.shape == (4, 128, 128)
    xf, af, wf = x.double(), a.double(), w.double()
    assert abs(xf.std().item() - 1.0) < 0.02
    assert abs(af.std().item() - 1.0 / math.sqrt(256)) < 0.002
    assert abs(wf.std().item() - 1.0 / math.sqrt(4 * 128)) < 0.002
    y = torch.einsum("rts,bsd,rde->bte", af, xf, wf)
    assert abs(y.std().item() - 1.0) < 0.1  # Y has unit variance by construction
