"""SumKronLinear on the GPU vs the fp64 oracle (``oracle.sumkron``)."""
import numpy as np
import pytest
import torch

from oracle import sumkron
from parity import compare
from workloads import SUMKRON_CONFIG, make_sumkron

pytestmark = pytest.mark.gpu


def run(gdpa, x, a, w):
    y, ws = gdpa.sumkron_forward(x.cuda(), a.cuda(), w.cuda())
    assert gdpa.device_status(ws) == 0
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("D", [128, 256, 384])
@pytest.mark.parametrize("T,k", [(32, 4), (32, 8), (64, 2), (64, 4)])
def test_shapes(cuda_lib, D, T, k):
    # B = 7: a partial last group; S = 128: two 64-seed chunks
    x, a, w = make_sumkron(7, 128, T, D, k, seed=D + T + k)
    compare("Y", run(cuda_lib, x, a, w), sumkron.forward(x, a, w))


@pytest.mark.parametrize("S", [64, 192, 256])
@pytest.mark.parametrize("B", [1, 4, 150, 333])
def test_seeds_and_batch(cuda_lib, S, B):
    """Batches below, at and above one group per SM (148); seeds from one
    chunk to four."""
    x, a, w = make_sumkron(B, S, 32, 128, 4, seed=S + B)
    compare("Y", run(cuda_lib, x, a, w), sumkron.forward(x, a, w))


def test_empty_batch(cuda_lib):
    x, a, w = make_sumkron(0, 64, 32, 128, 4)
    y = run(cuda_lib, x, a, w)
    assert y.shape == (0, 32, 128)


def test_full_size_sampled(cuda_lib):
    """The page's typical configuration at full batch: samples spread over
    the batch (first, last, every CTA's first and later groups) against the
    oracle one by one."""
    c = SUMKRON_CONFIG
    x, a, w = make_sumkron(c["B"], c["S"], c["T"], c["D"], c["k"], seed=1)
    y = run(cuda_lib, x, a, w).cpu()
    idx = np.unique(np.concatenate([[0, 1, 2, 3, c["B"] - 1], np.arange(5, c["B"], 97)]))
    ref = sumkron.forward(x[idx], a, w)
    compare("Y", y[idx], ref)


def test_rows_are_independent(cuda_lib):
    """Each sample's output depends on its own X only: changing one sample
    leaves the others bit-identical."""
    x, a, w = make_sumkron(9, 64, 32, 256, 4, seed=3)
    y1 = run(cuda_lib, x, a, w)
    x2 = x.clone()
    x2[4] = -x2[4]
    y2 = run(cuda_lib, x2, a, w)
    keep = [i for i in range(9) if i != 4]
    assert torch.equal(y1[keep], y2[keep])
    assert torch.equal(y2[4], -y1[4])  # linear in X, and negation is exact


@pytest.mark.parametrize("D", [128, 384])
def test_t64_larger_batch(cuda_lib, D):
    """T = 64 (two samples per 128-row tile) over a batch of 301 samples (151
    groups: one CTA takes two), k = 4, S = 256."""
    x, a, w = make_sumkron(301, 256, 64, D, 4, seed=D + 64)
    y = run(cuda_lib, x, a, w).cpu()
    idx = np.arange(0, 301, 7)
    compare("Y", y[idx], sumkron.forward(x[idx], a, w))


# -------------------------------------------------------------------- backward
def run_bwd(gdpa, x, a, w, dy):
    dx, da, dw, ws = gdpa.sumkron_backward(x.cuda(), a.cuda(), w.cuda(), dy.cuda())
    assert gdpa.device_status(ws) == 0
    torch.cuda.synchronize()
    return dx, da, dw


def make_dy(B, T, D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((B, T, D), generator=g).to(torch.bfloat16)


def compare_scaled(name, got, ref):
    """The GPU rounds the intermediates dY W^T and A X to bf16 (as the forward
    rounds A X), so each gradient's error scales with its own magnitude: the
    bounds (relative L2 1e-2, max abs 3e-2) apply after dividing both sides by
    the reference's RMS."""
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 1.0
    rms = rms if rms > 0 else 1.0
    got = got.float().cpu().numpy().astype(np.float64)
    compare(name, got / rms, ref / rms, bf16_out=False)


def check_bwd(gdpa, B, S, T, D, k, seed):
    x, a, w = make_sumkron(B, S, T, D, k, seed=seed)
    dy = make_dy(B, T, D, seed + 1)
    dx, da, dw = run_bwd(gdpa, x, a, w, dy)
    rdx, rda, rdw = sumkron.backward(x, a, w, dy)
    compare_scaled("dX", dx, rdx)
    compare_scaled("dA", da, rda)
    compare_scaled("dW", dw, rdw)
    return x, a, w, dy, (dx, da, dw)


@pytest.mark.parametrize("D", [128, 384])
@pytest.mark.parametrize("S,T,k", [(64, 32, 4), (128, 64, 2), (256, 32, 8), (192, 64, 4)])
def test_backward_shapes(cuda_lib, D, S, T, k):
    # B = 7: partial row tiles of the (sample, t) products; S = 64, 192: a
    # partial 128-wide tile of dX rows and of dA columns
    check_bwd(cuda_lib, 7, S, T, D, k, seed=D + S + T + k)


@pytest.mark.parametrize("B", [1, 70, 333])
def test_backward_batch(cuda_lib, B):
    """One sample (one split), fewer samples than dA splits, and more (uneven
    split ranges)."""
    check_bwd(cuda_lib, B, 128, 32, 256, 4, seed=B)


def test_backward_empty_batch(cuda_lib):
    x, a, w = make_sumkron(0, 64, 32, 128, 4)
    dx, da, dw = run_bwd(cuda_lib, x, a, w, make_dy(0, 32, 128, 0))
    assert dx.shape == (0, 64, 128)
    assert torch.all(da == 0) and torch.all(dw == 0)


def test_backward_linear_in_dy(cuda_lib):
    """The gradients are linear in dY and scaling by 2 is exact in bf16 and
    fp32: backward(2 dY) = 2 backward(dY) bit for bit."""
    x, a, w = make_sumkron(9, 128, 32, 128, 4, seed=5)
    dy = make_dy(9, 32, 128, 6)
    g1 = run_bwd(cuda_lib, x, a, w, dy)
    g2 = run_bwd(cuda_lib, x, a, w, dy * 2)
    for u, v in zip(g1, g2):
        assert torch.equal(v, u * 2)
