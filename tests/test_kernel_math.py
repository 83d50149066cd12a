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


def _kernel_consts():
    src = open(SRC).read()
    env = {}
    for name in ["kStages", "kTileBytes", "kBlk", "kQOff", "kKVOff", "kOnesOff", "kScaleOff", "kRopeOff",
                 "kKofsOff", "kRposOff", "kKcolOff", "kSlotFloats", "kBiasOff", "kBarOff", "kNumBars",
                 "kSmemBytes", "kCopy1"]:
        expr = re.search(r"constexpr int %s = ([^;]+);" % name, src).group(1)
        env[name] = eval(expr.split("//")[0], {}, env)
    return env


def _seg_len(k, L, M, s):
    a = k * M if s == 0 else (0 if k == 0 else s + (k - 1) * M)
    b = (k + 1) * M if s == 0 else s + k * M
    return min(b, L) - a


def _nseg(L, M, s):
    if s == 0:
        return (L + M - 1) // M
    return 1 if L <= s else 1 + (L - s + M - 1) // M


def test_bias_slot_reads_stay_inside_shared_memory():
    """The bias loads of the tensor-core softmax are unconditional (rows past
    the tile use row M-1; keys past the block read whatever sits there and are
    masked afterwards).  Replay their slot indices for every rectangle width,
    tile, block, query lane and key of the workloads and test shapes, for every
    row stride the host may choose, in both warpgroups' slots: each read must
    fall inside the kernel's shared memory, and each paired load must be 8-byte
    aligned."""
    c = _kernel_consts()
    lo_lim = -c["kBiasOff"] // 4
    hi_lim = (c["kSmemBytes"] - c["kBiasOff"]) // 4
    shapes = [(56, 56, 7, 3), (64, 64, 16, 8), (112, 112, 32, 16), (384, 384, 24, 12), (16, 16, 8, 4),
              (20, 13, 7, 3), (40, 36, 16, 8), (33, 70, 24, 12), (64, 64, 32, 16), (50, 45, 32, 5),
              (5, 130, 3, 1), (6, 7, 1, 0), (24, 24, 12, 6), (17, 23, 11, 10), (32, 32, 8, 4), (35, 30, 7, 3),
              (48, 40, 24, 12), (9, 200, 8, 4), (3, 3, 2, 1), (70, 64, 32, 0)]
    t = np.arange(128)[:, None, None]
    col = np.arange(96)[None, None, :]
    for H, W, M, s in shapes:
        lxs = {_seg_len(k, W, M, s) for k in range(_nseg(W, M, s))}
        lys = {_seg_len(k, H, M, s) for k in range(_nseg(H, M, s))}
        for R2e in range(2 * M, 2 * M + 15, 2):
            if (2 * M - 1) * R2e > c["kSlotFloats"] - c["kCopy1"]:
                break  # the host never picks it
            for lx in lxs:
                R, Rk = 128 // lx, 96 // lx
                kofs = (col // lx) * R2e + col % lx
                for ly in lys:
                    nb = (ly + Rk - 1) // Rk
                    j = np.arange(nb)[None, :, None]
                    for tile in range((ly + R - 1) // R):
                        qy, qx = tile * R + t // lx, t % lx
                        bbase = (np.minimum(qy, M - 1) + M - 1) * R2e + qx + M - 1
                        if lx % 2 == 0:
                            e = bbase - 1 - j * Rk * R2e - kofs[:, :, 0::2]
                            idx = np.where((bbase - 1) % 2 == 0, e, c["kCopy1"] + e - 1)
                            assert np.all(idx % 2 == 0)
                            idx = np.concatenate([idx, idx + 1], axis=2)
                        else:
                            idx = bbase - j * Rk * R2e - kofs
                        for g in (0, 1):
                            a = g * c["kSlotFloats"] + idx
                            assert a.min() >= lo_lim and a.max() < hi_lim, (H, W, M, s, R2e, lx, ly, tile)
