"""Pins the constants of the kernel's FMA-pipe 2^x polynomial (exp2_poly2 in
csrc/sm100_ptx.cuh): they must be the ones the committed minimax fit
produces, and that fit must stay within its stated relative-error bound."""
import os
import re

import numpy as np

from sliding_window_gqa_cu_b200 import fit_exp2_poly

PTX = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sliding_window_gqa_cu_b200", "csrc", "sm100_ptx.cuh")


def test_fit_error_bound():
    coeffs, err = fit_exp2_poly.coefficients_f32()
    assert err < 1e-4           # far below the bf16 step of P (2^-8 relative)


def test_kernel_constants_match_the_fit():
    src = open(PTX).read()
    found = dict(re.findall(r"kC(\d) = ([0-9.]+)f", src))
    coeffs, _ = fit_exp2_poly.coefficients_f32()
    for i, c in enumerate(coeffs):
        assert np.float32(float(found[str(i)])) == np.float32(c)


def test_range_reduction_reproduces_exp2():
    # the kernel's arithmetic, in float32 numpy: n = round(x), f = x - n, p(f) * 2^n
    coeffs, _ = fit_exp2_poly.coefficients_f32()
    x = np.linspace(-125.0, 8.0, 100001, dtype=np.float32)
    magic = np.float32(12582912.0)
    t = x + magic
    n = t - magic
    f = x - n
    p = np.float32(coeffs[3])
    for c in coeffs[2::-1]:
        p = p * f + np.float32(c)
    bits = (t.view(np.int32).astype(np.int64) * (1 << 23) + p.view(np.int32).astype(np.int64))
    y = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
