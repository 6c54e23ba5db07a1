"""The oracle's pins must catch plausible mistakes.

Each case compiles a copy of the C oracle with one planted mistake (a flipped
sign, a dropped term, an off-by-one index, a transposed operand), swaps it in
on the CPU, and checks that at least one pin of ``test_oracle`` fails.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle as pins
from workloads import (BIAS_ADD, BIAS_GATE, BIAS_NONE, PHI_GELU, PHI_IDENTITY, PHI_SILU,
                       PHI_SOFTMAX)

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdpa_oracle.c")

MUTATIONS = {
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    "bias_dropped": ("s[j] = p->scale * dot + score_bias(p, bias, h, kv_base + j);",
                     "s[j] = p->scale * dot;"),
    "window_left_off_by_one": ("if (wl >= 0 && j < i - wl) return 0;",
                               "if (wl >= 0 && j <= i - wl) return 0;"),
    "window_right_off_by_one": ("if (wr >= 0 && j > i + wr) return 0;",
                                "if (wr >= 0 && j >= i + wr) return 0;"),
    "key_head_index": ("const double* kj = k + ((kv_base + j) * H + h) * D;\n    double dot",
                       "const double* kj = k + ((kv_base + j) * H + 0) * D;\n    double dot"),
    "pv_uses_keys": ("acc += pr[j] * v[((k0 + j) * H + h) * D + d];",
                     "acc += pr[j] * k[((k0 + j) * H + h) * D + d];"),
    "lse_drops_max": ("return m + log(l);", "return log(l);"),
    "gate_negative_branch": ("return g - log1p(exp(g));", "return -log1p(exp(g));"),
    "softmax_delta_dropped": ("ds[j] = pr[j] * (dp[j] - delta);", "ds[j] = pr[j] * dp[j];"),
    "silu_grad_term_dropped": ("ds[j] = dp[j] * (sg + s[j] * sg * (1.0 - sg));",
                               "ds[j] = dp[j] * sg;"),
    "dk_scale_dropped": ("dkj[d] += p->scale * ds[j] * qi[d];", "dkj[d] += ds[j] * qi[d];"),
    "dq_uses_queries": ("dqi[d] += p->scale * ds[j] * kj[d];", "dqi[d] += p->scale * ds[j] * qi[d];"),
    "gate_grad_sign": ("1.0 - sigmoid(g);", "sigmoid(g);"),
    "dv_uses_dp": ("dvj[d] += pr[j] * doi[d];", "dvj[d] += dp[j] * doi[d];"),
    # GELU: the tanh approximation instead of erf, and a dropped derivative term
    "gelu_tanh_approximation": ("return 0.5 * (1.0 + erf(x / sqrt(2.0)));",
                                "return 0.5 * (1.0 + tanh(0.7978845608 * (x + 0.044715 * x * x * x)));"),
    "gelu_grad_term_dropped": ("ds[j] = dp[j] * (normal_cdf(s[j]) + s[j] * normal_pdf(s[j]));",
                               "ds[j] = dp[j] * normal_cdf(s[j]);"),
}

PIN_CALLS = [
    lambda: pins.test_pffn_two_matmul_form(),
    lambda: pins.test_identity_associativity(),
    lambda: pins.test_softmax_rows_sum_to_one(),
    lambda: pins.test_softmax_matches_torch_sdpa((2, 5), BIAS_GATE),
    lambda: pins.test_softmax_matches_torch_sdpa((3, 0), BIAS_ADD),
    lambda: pins.test_single_key_closed_forms(),
    lambda: pins.test_two_key_worked_example(),
    lambda: pins.test_gate_limits_and_add_equivalence(),
    lambda: pins.test_brute_force_tiny(PHI_SILU, (1, 0)),
    lambda: pins.test_brute_force_tiny(PHI_SOFTMAX, (0, 1)),
    lambda: pins.test_backward_matches_torch_autograd(PHI_SILU),
    lambda: pins.test_backward_matches_torch_autograd(PHI_SOFTMAX),
    lambda: pins.test_finite_difference_gradients(PHI_IDENTITY, BIAS_NONE, (-1, -1)),
    lambda: pins.test_gelu_two_matmul_form_matches_torch(),
    lambda: pins.test_backward_matches_torch_autograd(PHI_GELU),
]


@pytest.fixture(scope="module")
def src_text():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, src_text, tmp_path):
    old, new = MUTATIONS[name]
    assert src_text.count(old) == 1, f"mutation anchor for {name} not unique"
    c = tmp_path / "mut.c"
    c.write_text(src_text.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(so), str(c), "-lm"])
    good = oracle._load()
    lib = ctypes.CDLL(str(so))
    for fn in ("gdpa_oracle_forward", "gdpa_oracle_backward", "gdpa_oracle_num_threads"):
        getattr(lib, fn).argtypes = getattr(good, fn).argtypes
        getattr(lib, fn).restype = getattr(good, fn).restype
    caught = 0
    try:
        oracle._lib = lib
        for call in PIN_CALLS:
            try:
                call()
            except AssertionError:
                caught += 1
    finally:
        oracle._lib = good
    assert caught > 0, f"no pin caught the planted mistake {name}"
