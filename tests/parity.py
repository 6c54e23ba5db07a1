"""Helpers for GPU-vs-oracle comparisons (no GDPA arithmetic here)."""
import numpy as np
import torch

# Tolerances on O, dQ, dK, dV: relative L2 error <= 1e-2 and max abs error <= 3e-2
# per tensor (bf16 inputs, fp32 accumulation, bf16 outputs).  The outputs are
# bf16, and rounding the exact result to bf16 alone errs by half an ulp of the
# value (0.0304 on the tiny SiLU workload, whose |O| reaches 14.3), so the max
# abs bound is applied to the error beyond that half ulp.
REL_L2 = 1e-2
MAX_ABS = 3e-2


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers (8-bit significand) at |x|."""
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 0.5 * np.exp2(e - 7)
# LSE is fp32 on the device; its error comes from fp32 accumulation and the
# approximate exp2/log2 units (relative error ~1e-6), far below this bound.
LSE_ABS = 2e-3


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def compare(name, got, ref, rel_l2=REL_L2, max_abs=MAX_ABS, bf16_out=True):
    """bf16_out=False for fp32 outputs (the bias gradient): no half-ulp allowance."""
    got = to_np(got) if torch.is_tensor(got) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    mx = float(np.abs(err).max()) if err.size else 0.0
    allow = bf16_half_ulp(ref) if bf16_out else 0.0
    excess = float((np.abs(err) - allow).max()) if err.size else 0.0
    assert rel <= rel_l2 and excess <= max_abs, (
        f"{name}: rel_l2={rel:.3e} max_abs={mx:.3e} beyond_half_ulp={excess:.3e}")
    return rel, mx


def compare_lse(got, ref, q_lens=None):
    got = to_np(got)
    ref = np.asarray(ref)
    neg = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), neg), "LSE -inf pattern differs"
    if (~neg).any():
        mx = np.abs(got[~neg] - ref[~neg]).max()
        assert mx <= LSE_ABS, f"LSE max abs err {mx:.3e}"
