"""gdpa_forward_no_alloc, the forward for callers that cannot allocate device
memory (for example a plugin inside a framework that owns all device memory,
or a serving process that must not allocate on its request path).  It must
give what gdpa_forward gives, on consecutive calls that share its built-in
scratch.  This file is collected last so that a failure here never hides
another test's result."""
import numpy as np
import pytest
import torch

from parity import compare
from workloads import PHI_SILU, make_workload

pytestmark = pytest.mark.gpu


def _run_both(gdpa, w):
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    bias = w.bias.to(dev) if w.bias is not None else None
    kw = dict(phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right),
              bias_kind=w.bias_kind, max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv)
    ref_o, ref_lse, ws = gdpa.forward(q, k, v, qo, ko, bias=bias, **kw)
    assert gdpa.device_status(ws) == 0
    p = gdpa.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, **kw)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.H, w.total_q), float("nan"), device=dev)
    stream = torch.cuda.current_stream()
    rc = gdpa.gdpa_forward_no_alloc(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), qo.data_ptr(),
                                    ko.data_ptr(), None if bias is None else bias.data_ptr(),
                                    o.data_ptr(), lse.data_ptr(), stream.cuda_stream)
    assert rc == 0, gdpa.gdpa_status_string(rc)
    assert gdpa.gdpa_forward_no_alloc_status(stream.cuda_stream) == 0
    torch.cuda.synchronize()
    return ref_o, ref_lse, o, lse


def test_no_alloc_forward_matches_forward_on_consecutive_calls(cuda_lib):
    """Both calls run the same kernels on the same inputs as gdpa_forward, so
    the results must agree bit for bit.  The second call has a smaller batch
    than the first, so entries the first call left in the shared array past the
    second call's batch must not be read."""
    import oracle
    cases = [make_workload(5, B=23, seed=501, with_dout=False),   # gated softmax
             make_workload(2, B=7, seed=502, phi=PHI_SILU)]       # SiLU, other D, fewer samples
    for w in cases:
        ref_o, ref_lse, o, lse = _run_both(cuda_lib, w)
        assert torch.equal(o, ref_o), f"O differs from gdpa_forward ({w.name})"
        if w.phi == 1:
            assert torch.equal(lse, ref_lse), f"LSE differs from gdpa_forward ({w.name})"
        # and directly against the fp64 oracle
        ro, rlse = oracle.forward_workload(w)
        compare("O", o, ro)
        if w.phi == 1:
            np.testing.assert_allclose(lse.cpu().numpy(), rlse, atol=2e-3, rtol=0)


def test_no_alloc_status_reports_malformed_offsets(cuda_lib):
    """A sample whose offsets decrease is skipped and reported: the call
    returns GDPA_OK, the built-in status block holds GDPA_ERR_DEVICE_CHECK, and
    the next (well-formed) call clears it."""
    w = make_workload(2, B=4, seed=503)
    dev = torch.device("cuda")
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    good = list(w.q_offsets)
    bad = list(good)
    bad[2] = bad[1] - 5  # sample 1 gets a negative length
    stream = torch.cuda.current_stream().cuda_stream
    p = cuda_lib.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, phi=w.phi, scale=w.scale)
    o = torch.full_like(q, float("nan"))
    for offsets, expect in ((bad, 6), (good, 0)):  # 6: GDPA_ERR_DEVICE_CHECK
        qo = torch.tensor(offsets, dtype=torch.int32, device=dev)
        rc = cuda_lib.gdpa_forward_no_alloc(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            qo.data_ptr(), ko.data_ptr(), None, o.data_ptr(),
                                            None, stream)
        assert rc == 0, cuda_lib.gdpa_status_string(rc)
        assert cuda_lib.gdpa_forward_no_alloc_status(stream) == expect


def test_no_alloc_rejects_batches_beyond_its_scratch(cuda_lib):
    p = cuda_lib.make_params(16385, 1, 64, 16385, 16385)
    assert cuda_lib.gdpa_forward_no_alloc(p, 16, 16, 16, 16, 16, None, 16, None, None) == 3


def test_no_alloc_with_rotary_matches_forward(cuda_lib):
    """With rotary tables the no-alloc call turns Q and K inside the attention
    kernel (no copies to hold) and gives gdpa_forward's streamed result bit for
    bit."""
    from workloads import EVENT_TIME_SCALE, event_times
    ql = [300, 5, 129]
    w = make_workload(4, seed=21, q_lens=ql, kv_lens=ql)
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    table = cuda_lib.rotary_table(qo, torch.tensor(event_times(ql, 21), device=dev), w.D,
                                  EVENT_TIME_SCALE)
    kw = dict(phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right),
              max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv)
    ref_o, ref_lse, ws = cuda_lib.forward(q, k, v, qo, qo, rope=(table, table), **kw)
    assert cuda_lib.device_status(ws) == 0
    p = cuda_lib.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, rope=(table, table), **kw)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.H, w.total_q), float("nan"), device=dev)
    rc = cuda_lib.gdpa_forward_no_alloc(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        qo.data_ptr(), qo.data_ptr(), None, o.data_ptr(),
                                        lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, cuda_lib.gdpa_status_string(rc)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse)
