"""Host-side checks of arithmetic the tensor-core kernel does outside library
calls: the polynomial exp2 that takes part of the exponentials off the MUFU.
The coefficients are read from the kernel source and the kernel's float32
steps are replayed in numpy (round-to-nearest float32 at every step)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "vision_transformer_shifted_window_b200", "csrc", "k_attn_tc.cu")


def _poly_coeffs():
    src = open(SRC).read()
    body = src[src.index("float2 exp2_poly2(float2 e)"):]
    body = body[:body.index("\n}\n")]
    c = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    assert len(c) == 4, c  # c3, c2 (first FMA), then c1, c0
    return np.float32(c[0]), np.float32(c[1]), np.float32(c[2]), np.float32(c[3])


def _exp2_poly(e):
    """The kernel's exp2_poly2 on one float32 lane."""
    c3, c2, c1, c0 = _poly_coeffs()
    f32 = np.float32
    e = np.maximum(e.astype(np.float32), f32(-125.0))
    t = (e + f32(12582912.0)).astype(np.float32)
    r = (t + f32(-12582912.0)).astype(np.float32)
    f = (r * f32(-1.0) + e).astype(np.float32)  # exact
    q = (f * c3 + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error_below_half_fp16_ulp():
    # the softmax exponent lies in (-inf, 8]: the running maximum is kept
    # until a block exceeds it by more than 8
    e = np.linspace(-24.0, 8.0, 2_000_001, dtype=np.float32)
    got = _exp2_poly(e).astype(np.float64)
    want = np.exp2(e.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.0e-4, rel.max()  # fp16 keeps 2^-11 = 4.9e-4 relative


def test_exp2_poly_exact_at_integers_within_bound_and_tiny_below_range():
    e = np.arange(-24, 9, dtype=np.float32)
    rel = np.abs(_exp2_poly(e).astype(np.float64) - np.exp2(e.astype(np.float64))) / np.exp2(e.astype(np.float64))
    assert rel.max() < 1.0e-4
    # masked keys (-inf) and very negative arguments give at most 2^-125
    for v in (-np.inf, -1.0e30, -200.0, -126.0):
        out = _exp2_poly(np.array([v], dtype=np.float32))[0]
        assert 0.0 <= out <= 2.0 ** -124, (v, out)
