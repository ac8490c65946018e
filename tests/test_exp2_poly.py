"""The FMA-pipe 2^x the forward kernel uses for a quarter of its exponentials.

The device function (csrc/sm100.cuh, ex2_poly) is restated here in float32 numpy,
operation by operation, and checked against exact 2^x: relative error below 1e-4
over the range the kernels feed it (x in [-125, 8], plus the lazy-rescale headroom
up to 127), exact 0 below -125 and for -inf.  The coefficients are re-derived with
the committed Remez script and must match the ones in the kernel source.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc", "sm100.cuh")


def kernel_coeffs():
    text = open(SRC).read()
    body = text[text.index("float ex2_poly("):]
    body = body[:body.index("return x < -125.0f")]
    return [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body) if abs(float(v)) < 2.0]


def ex2_poly_f32(x, c3, c2, c1, c0):
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    t = (xc + np.float32(12582912.0)).astype(np.float32)
    f = (xc - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = (np.float32(c3) * f + np.float32(c2)).astype(np.float32)
    p = (p * f + np.float32(c1)).astype(np.float32)
    p = (p * f + np.float32(c0)).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    r = bits.astype(np.int32).view(np.float32)
    return np.where(x < np.float32(-125.0), np.float32(0.0), r)


def test_coefficients_match_remez_script():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc",
                                                        "gen_exp2_poly.py"), "3"],
                         capture_output=True, text=True, check=True).stdout
    fitted = [float(v) for v in re.findall(r"c\d = (-?[\d.e-]+)f", out)]
    c = kernel_coeffs()
    # kernel order: c3, c2, c1, c0
    assert len(c) >= 4
    c3, c2, c1, c0 = c[0], c[1], c[2], c[3]
    np.testing.assert_allclose([c0, c1, c2, c3], fitted, rtol=1e-6)


def test_relative_error_over_kernel_range():
    c = kernel_coeffs()
    x = np.concatenate([np.linspace(-125.0, 127.0, 2_000_001), np.linspace(-2, 2, 400_001)]).astype(np.float32)
    got = ex2_poly_f32(x, *c[:4]).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_masked_and_tiny_inputs_give_zero():
    c = kernel_coeffs()
    x = np.array([-np.inf, -1e30, -200.0, -125.5, -126.0], dtype=np.float32)
    assert (ex2_poly_f32(x, *c[:4]) == 0).all()
