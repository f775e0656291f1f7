"""The forward kernel's polynomial 2^x (exp2_poly.py), checked on the CPU.

The kernel computes a share of the softmax probabilities as 2^n * p(f) with
n = rint(x), f = x - n, p the degree-3 minimax polynomial that exp2_poly.py
fits.  Here the same steps run in numpy fp32 (each fused multiply-add rounded
once) and are compared with exp2 in fp64: the relative error stays below
the fit's bound, far under the bf16 rounding of P (2^-9).  The coefficients
written in sm100_ptx.cuh are the ones the fit produces.
"""
import os
import re
import runpy

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "block_sparse_attention_38_b200", "csrc")


def _fit():
    mod = runpy.run_path(os.path.join(CSRC, "exp2_poly.py"))
    return mod["remez"]()


def _kernel_coeffs():
    src = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"([0-9]\.[0-9]+)f", body) if float(v) < 1.0]
    return list(dict.fromkeys(vals))   # c3 initialises both lanes


def _emulate(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-126.5))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, np.float32(c[3]))
    for k in (2, 1, 0):   # one rounding per step, as a fused multiply-add
        p = (p.astype(np.float64) * f + np.float64(np.float32(c[k]))).astype(np.float32)
    return p.astype(np.float64) * 2.0 ** n.astype(np.float64)


def test_fit_error_bound():
    c, err = _fit()
    assert err < 8e-5
    x = np.linspace(-0.5, 0.5, 20001)
    rel = np.abs(np.polyval(c[::-1], x) / 2.0 ** x - 1.0)
    assert rel.max() <= err * 1.0001


def test_kernel_coefficients_are_the_fit():
    c, _ = _fit()
    kc = _kernel_coeffs()          # c3, c2, c1, c0 in the order the kernel uses them
    assert len(kc) == 4
    np.testing.assert_allclose(kc[::-1], np.float32(c), rtol=2e-7)


def test_range_reduction_matches_exp2():
    c, err = _fit()
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001), np.array([0.0, -0.5, 0.5, 8.0, -1.25])])
    got = _emulate(x, c)
    rel = np.abs(got / 2.0 ** x - 1.0)
    assert rel.max() < 1.5e-4


def test_masked_inputs_give_zero_or_tiny():
    c, _ = _fit()
    got = _emulate(np.array([-np.inf, -1e30, -200.0, -126.5]), c)
    assert np.all(got >= 0.0) and np.all(got < 2.0 ** -125)
