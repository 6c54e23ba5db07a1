"""GPU forward vs the fp64 oracle, element by element, on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from parity import compare, compare_lse
from workloads import (BIAS_ADD, BIAS_GATE, BIAS_NONE, PHI_GELU, PHI_IDENTITY, PHI_SILU,
                       PHI_SOFTMAX,
                       make_workload, subset)

pytestmark = pytest.mark.gpu


def run_gpu_forward(gdpa, w, max_q=None, max_kv=None):
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    bias = w.bias.to(dev) if w.bias is not None else None
    o, lse, ws = gdpa.forward(w.q.to(dev), w.k.to(dev), w.v.to(dev), qo, ko, phi=w.phi,
                              scale=w.scale, window=(w.window_left, w.window_right), bias=bias,
                              bias_kind=w.bias_kind,
                              max_seqlen_q=w.max_q if max_q is None else max_q,
                              max_seqlen_kv=w.max_kv if max_kv is None else max_kv)
    assert gdpa.device_status(ws) == 0
    torch.cuda.synchronize()
    return o, lse


def check_against_oracle(gdpa, w, **kw):
    o, lse = run_gpu_forward(gdpa, w, **kw)
    ro, rlse = oracle.forward_workload(w)
    compare("O", o, ro)
    if w.phi == PHI_SOFTMAX:
        compare_lse(lse, rlse)
    return o, lse


# -------------------------------------------------- the five workloads, oracle-sized
@pytest.mark.parametrize("cfg,B", [(1, None), (2, 12), (3, 24), (4, 6), (5, 6)])
def test_workload_parity(cuda_lib, cfg, B):
    w = make_workload(cfg, B=B, with_dout=False)
    check_against_oracle(cuda_lib, w)


# -------------------------------------------------- shapes, activations, biases
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX, PHI_IDENTITY, PHI_GELU])
@pytest.mark.parametrize("kv_len", [40, 200])  # one and two 128-key blocks
def test_head_dims_and_activations(cuda_lib, D, phi, kv_len):
    ql = [1, 127, 128, 129, 300]
    kl = [kv_len, 1, kv_len - 1, kv_len, 63]
    if phi == PHI_SOFTMAX:  # seed-pooling distributions, scale 1/sqrt(D)
        w = make_workload(3, seed=100 + D + phi, q_lens=ql, kv_lens=kl, H=2, D=D, phi=phi,
                          scale=1.0 / np.sqrt(D))
    else:  # PFFN distributions: K, V ~ N(0, 1/D), scale 1
        w = make_workload(2, seed=100 + D + phi, q_lens=ql, kv_lens=kl, H=2, D=D, phi=phi,
                          scale=1.0, kv_std=1.0 / np.sqrt(D))
    check_against_oracle(cuda_lib, w)


@pytest.mark.parametrize("bias_kind", [BIAS_ADD, BIAS_GATE])
@pytest.mark.parametrize("phi", [PHI_SILU, PHI_SOFTMAX])
def test_bias_and_gate(cuda_lib, bias_kind, phi):
    extra = {} if phi == PHI_SOFTMAX else dict(scale=1.0, kv_std=1.0 / np.sqrt(128))
    w = make_workload(5, B=5, seed=31 + bias_kind, phi=phi, bias=bias_kind, with_dout=False,
                      **extra)
    check_against_oracle(cuda_lib, w)


@pytest.mark.parametrize("window", [(127, 0), (0, 0), (5, 3), (300, 300), (-1, 0), (0, -1)])
@pytest.mark.parametrize("phi", [PHI_SOFTMAX, PHI_SILU])
def test_windows(cuda_lib, window, phi):
    ql = [1, 60, 200, 333, 520]
    extra = {} if phi == PHI_SOFTMAX else dict(scale=1.0, kv_std=1.0 / np.sqrt(128))
    w = make_workload(4, seed=40, q_lens=ql, kv_lens=ql, window=window, phi=phi, **extra)
    check_against_oracle(cuda_lib, w)


def test_window_rows_without_keys(cuda_lib):
    # right-bounded band with more queries than keys: late rows see nothing
    w = make_workload(4, seed=41, q_lens=[300, 17], kv_lens=[100, 3], window=(0, 0))
    o, lse = check_against_oracle(cuda_lib, w)
    assert torch.all(o[100:300].float() == 0)
    assert torch.all(torch.isneginf(lse[:, 100:300]))


def test_empty_samples_and_keys(cuda_lib):
    for phi in (PHI_SILU, PHI_SOFTMAX):
        extra = {} if phi == PHI_SOFTMAX else dict(scale=1.0, kv_std=1.0 / np.sqrt(128))
        w = make_workload(5, seed=42, q_lens=[0, 5, 130, 0, 1], kv_lens=[7, 0, 0, 0, 256],
                          phi=phi, with_dout=False, **extra)
        o, lse = check_against_oracle(cuda_lib, w)
        assert torch.all(o[0:135].float() == 0)


def test_single_sample_single_key(cuda_lib):
    w = make_workload(3, seed=43, q_lens=[1], kv_lens=[1])
    o, _ = check_against_oracle(cuda_lib, w)
    assert torch.equal(o.cpu(), w.v)  # softmax over one key returns V_0 exactly


@pytest.mark.parametrize("slope", [0.15, 2.0, -2.0])
def test_softmax_running_max_moves(cuda_lib, slope):
    # An additive bias rising along the keys moves each row's maximum up
    # within and across 128-key blocks: with slope 2.0 every 32-key chunk moves
    # it far past the rescale threshold (earlier P chunks, the partial sums, l
    # and O are all rescaled); with 0.15 only every second chunk or so; a
    # falling bias never moves it after the first chunk.
    kl = [300, 513, 64, 1000]
    w = make_workload(5, seed=44, q_lens=[130, 7, 64, 200], kv_lens=kl, bias=BIAS_ADD,
                      with_dout=False)
    for b in range(w.B):
        k0, k1 = int(w.kv_offsets[b]), int(w.kv_offsets[b + 1])
        w.bias[:, k0:k1] = slope * torch.arange(k1 - k0, dtype=torch.float32)
    check_against_oracle(cuda_lib, w)


def test_repeat_calls_bit_identical(cuda_lib):
    w = make_workload(2, B=8)
    o1, _ = run_gpu_forward(cuda_lib, w)
    o2, _ = run_gpu_forward(cuda_lib, w)
    assert torch.equal(o1, o2)


def test_declared_max_length_violation_is_reported(cuda_lib):
    w = make_workload(2, B=4)
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    _, _, ws = cuda_lib.forward(w.q.to(dev), w.k.to(dev), w.v.to(dev), qo, ko, phi=w.phi,
                                scale=w.scale, max_seqlen_q=int(w.q_lens.max()) - 1,
                                max_seqlen_kv=64)
    assert cuda_lib.device_status(ws) == 6


# -------------------------------------------------- full sizes, sampled checks
def _sampled_full(gdpa, cfg, n_samples=6):
    w = make_workload(cfg, device="cuda", with_dout=False)
    o, lse = run_gpu_forward(gdpa, w)
    order = np.argsort(w.q_lens * np.maximum(w.kv_lens, 1))
    picks = sorted({int(order[0]), int(order[-1]), w.B - 1, 0,
                    *np.random.default_rng(cfg).choice(w.B, n_samples, replace=False).tolist()})
    sub = subset(w, picks)
    sub.q, sub.k, sub.v = sub.q.cpu(), sub.k.cpu(), sub.v.cpu()
    if sub.bias is not None:
        sub.bias = sub.bias.cpu()
    ro, rlse = oracle.forward_workload(sub)
    rows = np.concatenate([np.arange(w.q_offsets[b], w.q_offsets[b + 1]) for b in picks])
    rows_t = torch.tensor(rows, device="cuda")
    compare("O", o[rows_t], ro)
    if w.phi == PHI_SOFTMAX:
        compare_lse(lse[:, rows_t], rlse)


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_sampled(cuda_lib, cfg):
    _sampled_full(cuda_lib, cfg)


# -------------------------------------------------- K/V ring: resident and streamed units
# A unit without a band keeps its key blocks in the shared K/V ring when they
# fit (D = 128: up to 2 blocks of 128 keys) and streams them per tile otherwise;
# tiles alternate between the two slots, so odd tile counts end a unit on
# either slot and the next unit's loads wait for the ring stages it reuses.
@pytest.mark.parametrize("phi", [PHI_SOFTMAX, PHI_SILU])
@pytest.mark.parametrize("kv_lens", [[256, 256, 256, 256], [257, 600, 1, 320],
                                     [64, 256, 257, 192]])
def test_kv_ring_resident_and_streamed(cuda_lib, phi, kv_lens):
    ql = [385, 128, 700, 1]
    if phi == PHI_SOFTMAX:
        w = make_workload(3, seed=7 + sum(kv_lens), q_lens=ql, kv_lens=kv_lens, H=3, D=128,
                          phi=phi, scale=1.0 / np.sqrt(128))
    else:
        w = make_workload(2, seed=7 + sum(kv_lens), q_lens=ql, kv_lens=kv_lens, H=3, D=128,
                          phi=phi, scale=1.0, kv_std=1.0 / np.sqrt(128))
    check_against_oracle(cuda_lib, w)


# -------------------------------------------------- the batch limit
def test_max_batch(cuda_lib):
    """16384 samples, the library's batch limit (the schedule's single-CTA
    sort), with jagged tiny lengths including empty samples: every output row
    against the oracle.  SiLU with the PFFN value distributions (K, V ~
    N(0, 1/D), scale 1), as every element-wise test uses."""
    rng = np.random.default_rng(16384)
    ql = rng.integers(0, 9, 16384)
    kl = rng.integers(0, 17, 16384)
    w = make_workload(2, seed=16, q_lens=ql, kv_lens=kl, H=2, D=32, phi=PHI_SILU, scale=1.0,
                      kv_std=1.0 / np.sqrt(32))
    check_against_oracle(cuda_lib, w)
