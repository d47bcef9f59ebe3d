"""The FMA-pipe 2^x the prefill softmax uses for part of P (no GPU: the same float32 steps in
numpy, checked against exp2 and against the error bound of the fit)."""
import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "exact_attention_158_b200", "csrc",
                   "sm100_ptx.cuh")


def kernel_coefficients():
    text = open(SRC).read()
    body = text[text.index("exp2_poly_x2"):]
    body = body[:body.index("return f2_pack(__uint_as_float(r0)")]
    lits = re.findall(r"f2_pack\((0x[0-9a-fA-Fp.+-]+)f,", body)
    return [float.fromhex(h) for h in lits]  # c3, c2, c1, c0 in Horner order


def exp2_poly(x):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c3, c2, c1, c0 = (np.float32(c) for c in kernel_coefficients())
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(np.float32)
    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = (t.view(np.uint32).astype(np.uint64) * (1 << 23) + p.view(np.uint32)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_parsed():
    c = kernel_coefficients()
    assert len(c) == 4 and abs(c[3] - 1.0) < 1e-3 and abs(c[2] - np.log(2)) < 1e-3


def test_relative_error_bound_over_softmax_range():
    # above -125 (below it the result is a denormal, 2^-125 times the row maximum at most)
    x = np.linspace(-125.0, 8.0, 4_000_001).astype(np.float32)
    y = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 8e-5, rel.max()


def test_clamps_masked_and_tiny_inputs():
    x = np.array([-np.inf, -1e30, -500.0, -127.0, -126.0], dtype=np.float32)
    y = exp2_poly(x)
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -125)


def test_integers_nearly_exact():
    n = np.arange(-120, 9, dtype=np.float32)
    y = exp2_poly(n).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(n) - 1) < 8e-5)
