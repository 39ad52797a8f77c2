"""Bounds of the hand-written arithmetic inside the CUDA kernels that does not
come from a library call, checked on the CPU by re-evaluating it in float32
with the constants read out of the kernel source.

The forward kernel takes part of its softmax exponentials on the FMA pipe:
2^x = 2^n * 2^f with n = rint(x) (the 1.5 * 2^23 rounding trick), f in
[-1/2, 1/2], 2^f a degree-3 polynomial, and n added to the exponent field.
The kernel comment claims a relative error below 7.5e-5 over the range the
softmax uses (x <= the lazy-rescale threshold of 8) and 2^-125 for -inf;
these tests hold it to that.
"""
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "causal_sliding_window_rope_b200", "csrc")


def _poly_constants():
    src = open(os.path.join(CSRC, "fwd_sm100.cuh")).read()
    body = src[src.index("void exp2_fma_x2"):]
    body = body[:body.index("\n}\n")]
    clamp = float(re.search(r"fmaxf\(x0, (-?[0-9.]+)f\)", body).group(1))
    magic = float(re.search(r"f2_pack\(([0-9.]+)f, \1f\)", body).group(1))
    coeffs = [float(c) for c in re.findall(r"f2_pack\((0\.[0-9]+)f, \1f\)", body)]
    # q = ((c3 f + c2) f + c1) f + c0, in the order the source lists them
    assert len(coeffs) == 4, coeffs
    return clamp, magic, coeffs


def _fma32(a, b, c):
    # a*b of two float32 values is exact in float64; one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_model(x, clamp, magic, coeffs):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(clamp))
    t = (x + f32(magic)).astype(f32)
    n = (t - f32(magic)).astype(f32)
    fr = _fma32(n, np.full_like(n, -1.0), x)
    c3, c2, c1, c0 = (np.full_like(x, f32(c)) for c in coeffs)
    q = _fma32(c3, fr, c2)
    q = _fma32(q, fr, c1)
    q = _fma32(q, fr, c0)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_polynomial_relative_error():
    clamp, magic, coeffs = _poly_constants()
    assert magic == 1.5 * 2 ** 23
    x = np.concatenate([np.linspace(-124.0, 8.0, 2_000_001), np.arange(-124, 9, dtype=np.float64),
                        np.arange(-124, 9) + 0.5, np.arange(-124, 9) - 0.5]).astype(np.float32)
    got = exp2_fma_model(x, clamp, magic, coeffs).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 7.6e-5, rel.max()
    # bf16 keeps 8 significant bits: the error is below half its ulp (2^-9)
    assert rel.max() < 2.0 ** -9 / 2


def test_exp2_polynomial_masked_inputs():
    clamp, magic, coeffs = _poly_constants()
    x = np.array([-np.inf, -1e30, -200.0, -125.0, -126.5], dtype=np.float32)
    got = exp2_fma_model(x, clamp, magic, coeffs)
    assert np.all(np.isfinite(got)) and np.all(got >= 0)
    # a masked key's weight is negligible next to the row maximum's 1
    assert got.max() < 2.0 ** -120
