"""GPU backward (dQ, dK, dV) vs the fp64 oracle on the same seeded inputs.

The GPU backward consumes the GPU forward's O and LSE, as a training step
does; the oracle recomputes everything from Q, K, V and dO in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import compare
from workloads import (BIAS_ADD, BIAS_GATE, BIAS_NONE, PHI_GELU, PHI_IDENTITY, PHI_SILU,
                       PHI_SOFTMAX,
                       make_workload, subset)

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(gdpa, w):
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    bias = w.bias.to(dev) if w.bias is not None else None
    q, k, v, do = w.q.to(dev), w.k.to(dev), w.v.to(dev), w.dout.to(dev)
    kw = dict(phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right), bias=bias,
              bias_kind=w.bias_kind, max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv)
    o, lse, ws = gdpa.forward(q, k, v, qo, ko, **kw)
    assert gdpa.device_status(ws) == 0
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    # with a bias or gate, its gradient too (NaN-filled: every element is written)
    dbias = (torch.full((w.H, w.total_kv), float("nan"), dtype=torch.float32, device=dev)
             if w.bias is not None else None)
    dq, dk, dv, wsb = gdpa.backward(q, k, v, o, do, lse, qo, ko, dq=dq, dk=dk, dv=dv,
                                    dbias=dbias, **kw)
    assert gdpa.device_status(wsb) == 0
    torch.cuda.synchronize()
    return o, dq, dk, dv, dbias


def check_backward(gdpa, w):
    _, dq, dk, dv, dbias = gpu_fwd_bwd(gdpa, w)
    rdq, rdk, rdv, rdb = oracle.backward_workload(w)
    compare("dQ", dq, rdq)
    compare("dK", dk, rdk)
    compare("dV", dv, rdv)
    if dbias is not None:
        compare_dbias(dbias, rdb)
    return dq, dk, dv


def compare_dbias(got, ref):
    """The bias gradient is fp32: no output rounding, but each key sums dS over
    up to a sample's queries, and dS uses delta = dO . O with the forward's bf16
    O (relative error up to 2^-9 of |delta|), so the max abs bound scales with
    the tensor's magnitude; relative L2 stays <= 1e-2."""
    ref = np.asarray(ref, np.float64)
    scale = max(1.0, float(np.abs(ref).max())) if ref.size else 1.0
    compare("dbias", got, ref, max_abs=3e-2 * scale, bf16_out=False)


def test_gated_training_step_parity(cuda_lib):
    """The gated softmax training workload (oracle-sized batch)."""
    check_backward(cuda_lib, make_workload(5, B=4))


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("phi", [PHI_SOFTMAX, PHI_SILU, PHI_IDENTITY, PHI_GELU])
def test_head_dims_and_activations(cuda_lib, D, phi):
    ql = [1, 127, 128, 129, 250]
    kl = [40, 1, 127, 200, 129]
    if phi == PHI_SOFTMAX:
        w = make_workload(5, seed=200 + D, q_lens=ql, kv_lens=kl, H=2, D=D,
                          scale=1.0 / np.sqrt(D))
    else:  # PFFN distributions; dO scaled so gradient sums stay O(1)
        w = make_workload(2, seed=210 + D + phi, q_lens=ql, kv_lens=kl, H=2, D=D, phi=phi,
                          scale=1.0, kv_std=1.0 / np.sqrt(D), with_dout=True,
                          dout_std=1.0 / np.sqrt(16.0))
    check_backward(cuda_lib, w)


@pytest.mark.parametrize("bias_kind", [BIAS_NONE, BIAS_ADD, BIAS_GATE])
def test_bias_kinds_softmax(cuda_lib, bias_kind):
    check_backward(cuda_lib, make_workload(5, B=3, seed=220 + bias_kind, bias=bias_kind))


@pytest.mark.parametrize("window", [(127, 0), (5, 3), (0, 0), (-1, 0), (300, 300)])
def test_windows_softmax(cuda_lib, window):
    ql = [1, 60, 200, 333, 520]
    w = make_workload(4, seed=230, q_lens=ql, kv_lens=ql, window=window, with_dout=True)
    check_backward(cuda_lib, w)


def test_window_silu(cuda_lib):
    ql = [70, 200, 333]
    w = make_workload(4, seed=231, q_lens=ql, kv_lens=ql, window=(127, 0), phi=PHI_SILU,
                      scale=1.0, kv_std=1.0 / np.sqrt(128), with_dout=True, dout_std=0.25)
    check_backward(cuda_lib, w)


def test_empty_and_degenerate_samples(cuda_lib):
    # Lq = 0 with keys (dK = dV = 0), Lk = 0 with queries (dQ = 0), single pairs
    w = make_workload(5, seed=240, q_lens=[0, 5, 130, 1, 0, 1], kv_lens=[7, 0, 256, 1, 0, 300])
    dq, dk, dv = check_backward(cuda_lib, w)
    assert torch.all(dk[0:7].float() == 0) and torch.all(dv[0:7].float() == 0)
    assert torch.all(dq[0:5].float() == 0)


def test_rows_without_keys_get_zero_gradient(cuda_lib):
    w = make_workload(4, seed=241, q_lens=[300, 17], kv_lens=[100, 3], window=(0, 0),
                      with_dout=True)
    dq, dk, dv = check_backward(cuda_lib, w)
    assert torch.all(dq[100:300].float() == 0)


def test_repeat_calls_bit_identical(cuda_lib):
    w = make_workload(5, B=4)
    a = gpu_fwd_bwd(cuda_lib, w)
    b = gpu_fwd_bwd(cuda_lib, w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)  # dbias too: its two adds per key commute exactly


@pytest.mark.slow
def test_full_size_gated_training_sampled(cuda_lib):
    """Full gated training workload on the GPU; a sample of it checked against
    the oracle (samples are independent, so a subset is an exact sub-problem)."""
    w = make_workload(5, device="cuda")
    _, dq, dk, dv, dbias = gpu_fwd_bwd(cuda_lib, w)
    rng = np.random.default_rng(5)
    picks = sorted({0, w.B - 1, int(np.argmax(w.q_lens)), int(np.argmin(w.q_lens)),
                    *rng.choice(w.B, 4, replace=False).tolist()})
    sub = subset(w, picks)
    for name in ("q", "k", "v", "dout", "bias"):
        setattr(sub, name, getattr(sub, name).cpu())
    rdq, rdk, rdv, rdb = oracle.backward_workload(sub)
    qrows = torch.tensor(np.concatenate([np.arange(w.q_offsets[b], w.q_offsets[b + 1])
                                         for b in picks]), device="cuda")
    krows = torch.tensor(np.concatenate([np.arange(w.kv_offsets[b], w.kv_offsets[b + 1])
                                         for b in picks]), device="cuda")
    compare("dQ", dq[qrows], rdq)
    compare("dK", dk[krows], rdk)
    compare("dV", dv[krows], rdv)
    compare_dbias(dbias[:, krows], rdb)


# -------------------------------------------------- bias / gate gradient
@pytest.mark.parametrize("phi", [PHI_SOFTMAX, PHI_SILU, PHI_GELU])
@pytest.mark.parametrize("bias_kind", [BIAS_ADD, BIAS_GATE])
@pytest.mark.parametrize("window", [(-1, -1), (127, 0)])
def test_bias_gradient(cuda_lib, phi, bias_kind, window):
    """d bias_j = sum_i dS_ij (add) and dG_j = (1 - sigma(G_j)) sum_i dS_ij (gate),
    over samples with one and several key blocks, ragged tails, a key block
    beyond every query's band (its keys get exactly 0) and an empty sample."""
    ql = [1, 130, 300, 0, 64]
    kl = [1, 129, 300, 50, 500]
    if phi == PHI_SOFTMAX:
        w = make_workload(5, seed=250 + bias_kind, q_lens=ql, kv_lens=kl, H=3, bias=bias_kind,
                          window=window)
    else:
        # SiLU's P is unnormalised and an N(0, 1) bias widens the scores; dO is
        # scaled so bf16 rounding of P before the dV MMA stays inside the bound
        ql = [1, 130, 200, 0, 64]
        w = make_workload(2, seed=260 + bias_kind, q_lens=ql, kv_lens=kl, H=3, D=128,
                          phi=phi, scale=1.0, kv_std=1.0 / np.sqrt(128), bias=bias_kind,
                          window=window, with_dout=True, dout_std=0.125)
    check_backward(cuda_lib, w)
    if window == (127, 0):
        # sample 4 (64 queries, 500 keys): query i sees keys [i - 127, i], so
        # keys 64.. are outside every band (partly inside a processed key block)
        _, _, _, _, dbias = gpu_fwd_bwd(cuda_lib, w)
        k0 = int(w.kv_offsets[4])
        assert torch.all(dbias[:, k0 + 64:k0 + 500] == 0)
        assert torch.all(dbias[:, int(w.kv_offsets[3]):int(w.kv_offsets[4])] == 0)


def test_max_batch_backward(cuda_lib):
    """16384 samples (the batch limit), softmax with a gate: dQ, dK, dV and dG
    against the oracle."""
    rng = np.random.default_rng(16385)
    ql = rng.integers(0, 9, 16384)
    kl = rng.integers(0, 17, 16384)
    w = make_workload(5, seed=17, q_lens=ql, kv_lens=kl, H=2, D=32, with_dout=True,
                      dout_std=0.125)
    check_backward(cuda_lib, w)
