"""The polynomial 2^x that the attention kernel evaluates on the FMA pipe for
one pair of softmax exponentials in four (host-side checks of its constants
and of its fp32 steps, emulated in numpy)."""
import importlib.util
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_context_prefill_dhsa_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coeffs():
    src = open(os.path.join(CSRC, "attn_fwd.cu")).read()
    m = re.search(r"kExpC1 = ([0-9.eE+-]+)f, kExpC2 = ([0-9.eE+-]+)f, kExpC3 = ([0-9.eE+-]+)f;", src)
    assert m, "coefficients not found in attn_fwd.cu"
    return np.array([float(v) for v in m.groups()], np.float32)


def test_kernel_constants_are_the_fit():
    c, err = _gen().fit()
    assert err < 1.02e-4
    np.testing.assert_allclose(_kernel_coeffs(), c, rtol=0, atol=2e-7)


def test_fp32_steps_within_the_bound():
    g = _gen()
    c = _kernel_coeffs()
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-126, 8, 400_000), np.linspace(-1.5, 1.5, 30_001),
                        np.arange(-126, 9) + 0.5, np.arange(-125, 9) - 0.49999997]).astype(np.float32)
    assert x.min() >= -126.0   # below that the results are only bounded (checked separately)
    rel = np.abs(g.exp2_fp32(x, c).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.05e-4


def test_integers_are_exact_powers_of_two():
    # f = 0 there, the polynomial is exactly 1 and only the exponent add acts
    j = np.arange(-126, 9)
    v = _gen().exp2_fp32(j.astype(np.float32), _kernel_coeffs())
    assert [float(a) for a in v] == [math.ldexp(1.0, int(e)) for e in j]


def test_masked_and_halfway_inputs():
    g = _gen()
    c = _kernel_coeffs()
    # masked scores are -inf: P must be exactly 0, as the MUFU's 2^-inf is
    lo = g.exp2_fp32(np.array([-np.inf, -1e30, -200.0, -127.0], np.float32), c)
    assert [float(v) for v in lo] == [0.0, 0.0, 0.0, 0.0]
    # between -127 and -126 only a bound holds: non-negative, below 2^-126
    mid = g.exp2_fp32(np.linspace(-127, -126, 100_001).astype(np.float32), c)
    assert np.all(mid >= 0) and np.all(mid <= 2.0 ** -126) and np.all(np.isfinite(mid))
    # x = -0.5 and +0.5 sit at the ends of the fitted interval
    v = g.exp2_fp32(np.array([-0.5, 0.5], np.float32), c).astype(np.float64)
    assert np.all(np.abs(v / np.exp2([-0.5, 0.5]) - 1) < 1.05e-4)
