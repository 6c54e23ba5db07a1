"""Per-head activation vector: each head of one call uses its own phi.

The GPU result for head h is compared with the oracle run with head h's
activation on the same inputs (heads are independent, so the oracle needs no
per-head form of its own).
"""
import copy

import numpy as np
import pytest
import torch

import oracle
from parity import compare, compare_lse
from workloads import BIAS_GATE, PHI_GELU, PHI_IDENTITY, PHI_SILU, PHI_SOFTMAX, make_workload

pytestmark = pytest.mark.gpu

HEAD_PHI = [PHI_SOFTMAX, PHI_SILU, PHI_GELU, PHI_IDENTITY, PHI_SOFTMAX]


def _workload(D, bias):
    ql = [1, 130, 257, 64, 0]
    kl = [40, 129, 300, 1, 7]
    # PFFN distributions (K, V ~ N(0, 1/D), scale 1) keep the unnormalised
    # activations in range; dO is scaled so bf16 rounding of unnormalised P
    # (identity, SiLU, GELU heads) before the dV MMA stays inside the bound
    return make_workload(2, seed=300 + D, q_lens=ql, kv_lens=kl, H=len(HEAD_PHI), D=D,
                         scale=1.0, kv_std=1.0 / np.sqrt(D), bias=bias, with_dout=True,
                         dout_std=0.125)


def _with_phi(w, phi):
    c = copy.copy(w)
    c.phi = phi
    return c


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bias", [0, BIAS_GATE])
def test_head_phi_forward_and_backward(cuda_lib, D, bias):
    w = _workload(D, bias)
    dev = torch.device("cuda")
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    q, k, v, do = w.q.to(dev), w.k.to(dev), w.v.to(dev), w.dout.to(dev)
    b = w.bias.to(dev) if w.bias is not None else None
    kw = dict(scale=w.scale, bias=b, bias_kind=w.bias_kind, max_seqlen_q=w.max_q,
              max_seqlen_kv=w.max_kv, head_phi=HEAD_PHI)
    o, lse, ws = cuda_lib.forward(q, k, v, qo, ko, **kw)
    assert cuda_lib.device_status(ws) == 0
    dbias = (torch.full((w.H, w.total_kv), float("nan"), device=dev) if b is not None else None)
    dq, dk, dv, wsb = cuda_lib.backward(q, k, v, o, do, lse, qo, ko, dbias=dbias, **kw)
    assert cuda_lib.device_status(wsb) == 0
    torch.cuda.synchronize()
    for phi in sorted(set(HEAD_PHI)):
        heads = [h for h, x in enumerate(HEAD_PHI) if x == phi]
        wp = _with_phi(w, phi)
        ro, rlse = oracle.forward_workload(wp)
        rdq, rdk, rdv, rdb = oracle.backward_workload(wp)
        for h in heads:
            compare(f"O[h{h}]", o[:, h], ro[:, h])
            if phi == PHI_SOFTMAX:
                compare_lse(lse[h], rlse[h])
            compare(f"dQ[h{h}]", dq[:, h], rdq[:, h])
            compare(f"dK[h{h}]", dk[:, h], rdk[:, h])
            compare(f"dV[h{h}]", dv[:, h], rdv[:, h])
            if dbias is not None:
                scale = max(1.0, float(np.abs(rdb[h]).max()))
                compare(f"dbias[h{h}]", dbias[h], rdb[h], max_abs=3e-2 * scale, bf16_out=False)
