"""Device-side failure detection, without faulting the GPU.

Every wait inside the kernels is bounded.  A debug flag drops one Q-tile load
in CTA 0, so the MMA issuer's wait for it runs out after 20 ms; the kernel
must record GDPA_ERR_TIMEOUT, leave cleanly, and leave the context usable.
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
