"""Seeded synthetic GDPA workloads (inputs only; no GDPA arithmetic lives here).

Both the fp64 oracle (``oracle/``) and the CUDA path (``pffn_attention_b200``)
are fed from this module, so that a parity test hands the two sides the very
same bf16 bits.  It holds nothing of the method: lengths and values are drawn,
rounded to bf16, and laid out in the jagged ``[total, H, D]`` convention.

Shapes follow the workloads the Kunlun pages describe: jagged behaviour
sequences of hundreds to thousands of events, short context-generated K/V,
small head dims (Kunlun paper review, §1 and §3.1; Kunlun Breakdown, "The Core
Architecture and Mechanics").  The pages' data (Meta Ads, private) is absent;
these synthetic inputs stand in for it.

Recipe: sequence lengths come from ``numpy.random.default_rng(seed)``; values
from a ``torch.Generator`` seeded with the same seed on the target device,
drawn as fp32 normals, scaled, and cast to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

PHI_SILU, PHI_SOFTMAX, PHI_IDENTITY, PHI_GELU = 0, 1, 2, 3
BIAS_NONE, BIAS_ADD, BIAS_GATE = 0, 1, 2


@dataclass
class Workload:
    """One GDPA problem: shapes, options and the seeded tensors."""

    name: str
    B: int
    H: int
    D: int
    phi: int
    scale: float
    window_left: int = -1
    window_right: int = -1
    bias_kind: int = BIAS_NONE
    q_lens: np.ndarray = field(default=None, repr=False)
    kv_lens: np.ndarray = field(default=None, repr=False)
    q_offsets: np.ndarray = field(default=None, repr=False)   # int32 [B+1]
    kv_offsets: np.ndarray = field(default=None, repr=False)  # int32 [B+1]
    q: torch.Tensor = field(default=None, repr=False)         # bf16 [total_q, H, D]
    k: torch.Tensor = field(default=None, repr=False)         # bf16 [total_kv, H, D]
    v: torch.Tensor = field(default=None, repr=False)         # bf16 [total_kv, H, D]
    bias: Optional[torch.Tensor] = field(default=None, repr=False)  # fp32 [H, total_kv]
    dout: Optional[torch.Tensor] = field(default=None, repr=False)  # bf16 [total_q, H, D]

    @property
    def total_q(self) -> int:
        return int(self.q_offsets[-1])

    @property
    def total_kv(self) -> int:
        return int(self.kv_offsets[-1])

    @property
    def max_q(self) -> int:
        return int(self.q_lens.max()) if self.B else 0

    @property
    def max_kv(self) -> int:
        return int(self.kv_lens.max()) if self.B else 0


# The five workloads, with the distributions stated for each.  ``B`` is the
# full batch; tests pass a smaller ``B`` to get oracle-sized problems with the
# same per-sample distributions.
CONFIGS = {
    1: dict(name="tiny_silu_fwd", B=4, H=2, D=32, phi=PHI_SILU,
            scale=1.0 / math.sqrt(32.0), q_len=("uniform", 1, 64),
            kv_len=("fixed", 16), q_std=1.0, kv_std=1.0),
    2: dict(name="pffn_silu_fwd", B=1024, H=4, D=64, phi=PHI_SILU, scale=1.0,
            q_len=("uniform", 100, 1000), kv_len=("fixed", 64),
            q_std=1.0, kv_std=1.0 / math.sqrt(64.0)),
    3: dict(name="seed_pooling_softmax_fwd", B=2048, H=8, D=128, phi=PHI_SOFTMAX,
            scale=1.0 / math.sqrt(128.0), q_len=("fixed", 32),
            kv_len=("loguniform", 128, 2048), q_std=1.0, kv_std=1.0),
    4: dict(name="sliding_window_softmax_fwd", B=512, H=4, D=128, phi=PHI_SOFTMAX,
            scale=1.0 / math.sqrt(128.0), q_len=("uniform", 200, 2000),
            kv_len=("same",), q_std=1.0, kv_std=1.0, window=(127, 0)),
    5: dict(name="gated_softmax_train", B=4096, H=8, D=128, phi=PHI_SOFTMAX,
            scale=1.0 / math.sqrt(128.0), q_len=("uniform", 256, 1024),
            kv_len=("fixed", 256), q_std=1.0, kv_std=1.0, bias=BIAS_GATE,
            dout=True),
}


def _draw_lengths(spec, n: int, rng: np.random.Generator, other=None) -> np.ndarray:
    kind = spec[0]
    if kind == "fixed":
        return np.full(n, spec[1], dtype=np.int64)
    if kind == "uniform":
        return rng.integers(spec[1], spec[2] + 1, size=n, dtype=np.int64)
    if kind == "loguniform":
        lo, hi = spec[1], spec[2]
        u = rng.uniform(math.log(lo), math.log(hi), size=n)
        return np.clip(np.rint(np.exp(u)), lo, hi).astype(np.int64)
    if kind == "same":
        return other.copy()
    raise ValueError(f"unknown length spec {spec}")


def offsets_from_lengths(lens: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lens) + 1, dtype=np.int64)
    np.cumsum(lens, out=off[1:])
    if off[-1] >= 2**31:
        raise ValueError("total length does not fit int32 offsets")
    return off.astype(np.int32)


def _normal_bf16(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)  # round-to-nearest-even


def make_workload(cfg: int, B: Optional[int] = None, seed: Optional[int] = None,
                  device="cpu", with_dout: Optional[bool] = None,
                  q_lens=None, kv_lens=None, **overrides) -> Workload:
    """Build workload ``cfg`` (1..5), optionally with a smaller batch ``B``.

    ``seed`` defaults to the workload number.  ``q_lens`` / ``kv_lens``
    override the drawn lengths (edge-case tests).  ``overrides`` may replace
    H, D, phi, scale, window, bias kind, q_std, kv_std or dout_std for
    edge-case tests.
    """
    spec = dict(CONFIGS[cfg])
    seed = cfg if seed is None else seed
    Bn = spec["B"] if B is None else B
    H = overrides.get("H", spec["H"])
    D = overrides.get("D", spec["D"])
    phi = overrides.get("phi", spec["phi"])
    scale = overrides.get("scale", spec["scale"])
    wl, wr = overrides.get("window", spec.get("window", (-1, -1)))
    bias_kind = overrides.get("bias", spec.get("bias", BIAS_NONE))
    if with_dout is None:
        with_dout = bool(spec.get("dout", False))

    rng = np.random.default_rng(seed)
    ql = _draw_lengths(spec["q_len"], Bn, rng) if q_lens is None else np.asarray(q_lens, np.int64)
    if kv_lens is not None:
        kl = np.asarray(kv_lens, np.int64)
    else:
        kl = _draw_lengths(spec["kv_len"], Bn, rng, other=ql)
    Bn = len(ql)
    assert len(kl) == Bn
    qo = offsets_from_lengths(ql)
    ko = offsets_from_lengths(kl)
    tq, tk = int(qo[-1]), int(ko[-1])

    q_std = overrides.get("q_std", spec["q_std"])
    kv_std = overrides.get("kv_std", spec["kv_std"])
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _normal_bf16((tq, H, D), q_std, gen, device)
    k = _normal_bf16((tk, H, D), kv_std, gen, device)
    v = _normal_bf16((tk, H, D), kv_std, gen, device)
    bias = None
    if bias_kind != BIAS_NONE:
        bias = torch.randn((H, tk), generator=gen, device=device, dtype=torch.float32)
    dout_std = overrides.get("dout_std", 1.0)
    dout = _normal_bf16((tq, H, D), dout_std, gen, device) if with_dout else None
    return Workload(name=spec["name"], B=Bn, H=H, D=D, phi=phi, scale=float(scale),
                    window_left=int(wl), window_right=int(wr), bias_kind=bias_kind,
                    q_lens=ql, kv_lens=kl, q_offsets=qo, kv_offsets=ko,
                    q=q, k=k, v=v, bias=bias, dout=dout)


def subset(w: Workload, samples) -> Workload:
    """The same problem restricted to the listed samples (for sampled checks).

    Slices the jagged rows of each chosen sample out of the full tensors and
    re-packs them, so a per-sample check can run on a handful of samples of a
    full-size workload.  ``samples`` are indices into ``w``'s batch.
    """
    samples = [int(s) for s in samples]
    qsl = [slice(int(w.q_offsets[b]), int(w.q_offsets[b + 1])) for b in samples]
    ksl = [slice(int(w.kv_offsets[b]), int(w.kv_offsets[b + 1])) for b in samples]
    cat = lambda t, sl: torch.cat([t[s] for s in sl], 0) if sl else t[:0]
    ql = w.q_lens[samples]
    kl = w.kv_lens[samples]
    out = Workload(name=w.name + "_subset", B=len(samples), H=w.H, D=w.D, phi=w.phi,
                   scale=w.scale, window_left=w.window_left, window_right=w.window_right,
                   bias_kind=w.bias_kind, q_lens=ql, kv_lens=kl,
                   q_offsets=offsets_from_lengths(ql), kv_offsets=offsets_from_lengths(kl),
                   q=cat(w.q, qsl), k=cat(w.k, ksl), v=cat(w.v, ksl))
    if w.bias is not None:
        out.bias = torch.cat([w.bias[:, s] for s in ksl], 1) if ksl else w.bias[:, :0]
    if w.dout is not None:
        out.dout = cat(w.dout, qsl)
    return out


# Event times for the rotary temporal embedding: behaviour logs hold events
# from seconds to months apart, often several in the same second.  Per sample:
# a start time in 2024 (Unix seconds), then gaps that are 0 with probability
# 0.1 and otherwise log-uniform between 1 s and 10^7 s (about four months),
# rounded to whole seconds.  int64 [total], non-decreasing within a sample.
EVENT_TIME_SCALE = 3600.0  # tau_scale of the rotary workloads: one hour


def event_times(lens, seed: int) -> np.ndarray:
    lens = np.asarray(lens, np.int64)
    rng = np.random.default_rng(seed)
    total = int(lens.sum())
    gaps = np.rint(np.exp(rng.uniform(0.0, math.log(1e7), total))).astype(np.int64)
    gaps[rng.uniform(size=total) < 0.1] = 0
    starts = rng.integers(1_704_067_200, 1_735_689_600, len(lens))
    out = np.empty(total, np.int64)
    pos = 0
    for b, L in enumerate(lens):
        L = int(L)
        if L:
            g = gaps[pos:pos + L].copy()
            g[0] = 0
            out[pos:pos + L] = starts[b] + np.cumsum(g)
        pos += L
    return out


# SumKronLinear (second stage of Hierarchical Seed Pooling): the page's typical
# configuration is S = 256 seeds, T = 32 tokens, D = 384, rank k = 8; the batch
# is the seed-pooling workload's (2048 samples).  X ~ N(0, 1); A ~ N(0, 1/S)
# and W ~ N(0, 1/(k D)), so Y = sum_r A_r X W_r has unit variance.  All bf16.
SUMKRON_CONFIG = dict(B=2048, S=256, T=32, D=384, k=8)


def make_sumkron(B, S, T, D, k, seed=0, device="cpu"):
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = _normal_bf16((B, S, D), 1.0, gen, device)
    a = _normal_bf16((k, T, S), 1.0 / math.sqrt(S), gen, device)
    w = _normal_bf16((k, D, D), 1.0 / math.sqrt(k * D), gen, device)
    return x, a, w
