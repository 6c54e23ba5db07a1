"""Device-side failure detection, without faulting the GPU.

Every wait inside the kernels is bounded.  A debug flag drops one Q-tile load
(forward) or one Q/dO-tile load (backward) in CTA 0, so the MMA issuer's wait
for it runs out after 20 ms; the kernel must record GDPA_ERR_TIMEOUT, leave
cleanly, and leave the context usable.  Malformed offsets are caught by the
schedule and reported instead of being read or written past the tensors.
"""
import pytest
import torch

import oracle
from parity import compare
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _args(w):
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    return w.q.to(dev), w.k.to(dev), w.v.to(dev), qo, ko


@pytest.mark.parametrize("cfg", [2, 5])
def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib, cfg):
    w = make_workload(cfg, B=6, with_dout=False)
    q, k, v, qo, ko = _args(w)
    bias = w.bias.cuda() if w.bias is not None else None
    p = cuda_lib.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, phi=w.phi, scale=w.scale,
                             bias_kind=w.bias_kind, max_seqlen_q=w.max_q,
                             max_seqlen_kv=w.max_kv, debug_flags=1, wait_timeout_us=20000)
    _, _, ws = cuda_lib.forward(q, k, v, qo, ko, bias=bias, params=p)
    assert cuda_lib.device_status(ws) == 5  # GDPA_ERR_TIMEOUT
    # the same context, a normal call afterwards
    o, _, ws2 = cuda_lib.forward(q, k, v, qo, ko, phi=w.phi, scale=w.scale, bias=bias,
                                 bias_kind=w.bias_kind, max_seqlen_q=w.max_q,
                                 max_seqlen_kv=w.max_kv)
    assert cuda_lib.device_status(ws2) == 0
    ro, _ = oracle.forward_workload(w)
    compare("O", o, ro)


def test_launch_errors_are_reported_at_the_call(cuda_lib):
    w = make_workload(2, B=2)
    q, k, v, qo, ko = _args(w)
    p = cuda_lib.make_params(w.B, w.H, w.D, w.total_q, w.total_kv)
    o = torch.empty_like(q)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = cuda_lib.gdpa_forward(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), qo.data_ptr(),
                               ko.data_ptr(), None, o.data_ptr(), None, small.data_ptr(), 16,
                               torch.cuda.current_stream().cuda_stream)
    assert rc == 3  # GDPA_ERR_WORKSPACE


def test_sumkron_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    """The SumKronLinear kernel's waits are bounded too: one dropped X load in
    CTA 0 ends in GDPA_ERR_TIMEOUT, and the next call on the context is exact."""
    from oracle import sumkron
    from workloads import make_sumkron
    x, a, w = make_sumkron(9, 128, 32, 128, 4, seed=7)
    xd, ad, wd = x.cuda(), a.cuda(), w.cuda()
    _, ws = cuda_lib.sumkron_forward(xd, ad, wd, wait_timeout_us=20000, debug_flags=1)
    assert cuda_lib.device_status(ws) == 5  # GDPA_ERR_TIMEOUT
    y, ws2 = cuda_lib.sumkron_forward(xd, ad, wd)
    assert cuda_lib.device_status(ws2) == 0
    compare("Y", y, sumkron.forward(x, a, w))


@pytest.mark.parametrize("cfg", [2, 5])
def test_backward_bounded_wait_reports_timeout_and_context_survives(cuda_lib, cfg):
    # element-wise phi takes the PFFN value scales, dO included (as the other
    # SiLU backward tests do)
    extra = {"dout_std": 0.125} if cfg == 2 else {}
    w = make_workload(cfg, B=6, with_dout=True, **extra)
    q, k, v, qo, ko = _args(w)
    bias = w.bias.cuda() if w.bias is not None else None
    dout = w.dout.cuda()
    kw = dict(phi=w.phi, scale=w.scale, bias=bias, bias_kind=w.bias_kind,
              max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv)
    o, lse, ws = cuda_lib.forward(q, k, v, qo, ko, **kw)
    assert cuda_lib.device_status(ws) == 0
    p = cuda_lib.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, phi=w.phi, scale=w.scale,
                             bias_kind=w.bias_kind, max_seqlen_q=w.max_q,
                             max_seqlen_kv=w.max_kv, debug_flags=1, wait_timeout_us=20000)
    _, _, _, wsb = cuda_lib.backward(q, k, v, o, dout, lse, qo, ko, bias=bias, params=p)
    assert cuda_lib.device_status(wsb) == 5  # GDPA_ERR_TIMEOUT
    # the same context, a normal call afterwards
    dq, dk, dv, wsb2 = cuda_lib.backward(q, k, v, o, dout, lse, qo, ko, **kw)
    assert cuda_lib.device_status(wsb2) == 0
    rdq, rdk, rdv, _ = oracle.backward_workload(w)
    compare("dQ", dq, rdq)
    compare("dK", dk, rdk)
    compare("dV", dv, rdv)


@pytest.mark.parametrize("which", ["decreasing", "past_total", "negative_start"])
def test_malformed_offsets_are_reported_and_skipped(cuda_lib, which):
    """Offsets that decrease, or that reach past total_q, must neither be read
    nor written past the tensors: the schedule reports GDPA_ERR_DEVICE_CHECK and
    skips the sample, and the other samples' rows are still exact."""
    w = make_workload(2, B=4)
    q, k, v, qo, ko = _args(w)
    good = list(w.q_offsets)
    bad = list(good)
    if which == "decreasing":
        bad[2] = bad[1] - 5          # sample 1 gets a negative length
    elif which == "past_total":
        bad[3] = int(w.total_q) + 7  # sample 2 ends past the tensor, sample 3 starts there
    else:
        bad[1] = -3                  # sample 0 has a negative length, sample 1 starts outside
    qo_bad = torch.tensor(bad, dtype=torch.int32, device="cuda")
    sentinel = float("nan")
    o = torch.full_like(q, sentinel)
    _, _, ws = cuda_lib.forward(q, k, v, qo_bad, ko, phi=w.phi, scale=w.scale,
                                max_seqlen_q=0, max_seqlen_kv=0, out=o)
    assert cuda_lib.device_status(ws) == 6  # GDPA_ERR_DEVICE_CHECK
    ro, _ = oracle.forward_workload(w)
    # samples whose offsets are intact still match the oracle
    for b in range(w.B):
        lo, hi = bad[b], bad[b + 1]
        if lo == good[b] and hi == good[b + 1] and hi >= lo:
            compare(f"O sample {b}", o[lo:hi], ro[lo:hi])
