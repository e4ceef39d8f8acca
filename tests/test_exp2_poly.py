"""The FMA-pipe 2^x used for part of the softmax (ex2_poly2 in
csrc/attn_tc.cuh), replayed step by step in float32 on the CPU, against
numpy's exp2: relative error within the fitted bound over the whole range
the kernel feeds it (x <= 8), and the coefficients in the kernel equal a
fresh run of the fitting script."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_diffusion_lm_attn_b200", "csrc")


def kernel_coeffs():
    src = open(os.path.join(CSRC, "attn_tc.cuh")).read()
    m = re.search(r"c0 = ([-0-9.e+]+)f, c1 = ([-0-9.e+]+)f,\s*"
                  r"c2 = ([-0-9.e+]+)f, c3 = ([-0-9.e+]+)f", src)
    assert m, "coefficients not found in attn_tc.cuh"
    return [np.float32(float(v)) for v in m.groups()]


def f32(x):
    return np.float32(x)


def fma32(a, b, c):
    # single rounding: the product of two float32 is exact in float64
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def ex2_poly(x, c):
    x = np.maximum(x.astype(np.float32), f32(-126.0))
    magic = f32(12582912.0)
    j = (x + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    fr = fma32(n, f32(-1.0), x)
    p = fma32(c[3], fr, c[2])
    p = fma32(p, fr, c[1])
    p = fma32(p, fr, c[0])
    bits = p.view(np.int32) + (j.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    c = kernel_coeffs()
    x = np.concatenate([np.linspace(-126, 8, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 1_000_000))])
    y = ex2_poly(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    normal = x >= -125  # below, the result is a float32 subnormal
    assert rel[normal].max() < 1.0e-4, rel[normal].max()
    assert rel[~normal].max() < 1e-3
    # bf16 P needs 2^-9; the row sums use the float32 values
    assert y.min() > 0


def test_coefficients_match_fit_script():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2.py")],
                         check=True, capture_output=True, text=True).stdout
    fit = [np.float32(float(v)) for v in re.findall(r"c\d = ([-0-9.e+]+)", out)]
    assert fit == kernel_coeffs()
