"""Seeded synthetic workloads for shifted-window attention.

This module only draws random numbers and names shapes; it holds none of the
attention arithmetic.  Tests, the smoke check and the benchmark all take their
inputs from here, so the CUDA path and the CPU oracle see identical values.

Recipe (one ``numpy.random.SeedSequence(1000 + index)`` per workload, spawned
into eight PCG64 streams used in this fixed order): q, k, v, then the bias
table or W1, b1, W2, b2, tau.  Q/K/V entries are N(0, 1) in float32; bf16
workloads round them to bf16 (round-to-nearest-even) before either side reads
them.  Bias tables and CPB-MLP weights are N(0, 0.02); tau is U(0.05, 0.2)
where the workload says so; RoPE frequencies are 100^(-t/(d/4)) per axis.

The shapes follow the workloads the pages describe: Swin-T stage 1 (56x56, C=96,
M=7), SwinV2-T at 256 px (64x64, M=16), FlashSwin-T with dense p=2 tokens
(112x112, M=32), a SwinV2-G-like stage 1 at 1536 px (384x384, C=512, M=24),
and Iwin-T's stage 1 (Swin-T's shape with interleaved windows and no position
bias); no dataset is read.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np

MODE_DOT_BIAS = 0
MODE_COSINE_CPB = 1
MODE_ROPE = 2


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    H: int
    W: int
    heads: int
    d: int
    M: int
    shifts: Tuple[int, ...]
    mode: int
    tau: Optional[Tuple[float, float]] = None  # fixed value (a, a) or U(a, b)
    cpb_hidden: int = 0  # 0: a bias table is drawn instead (modes 0 and 1)
    rope_base: float = 0.0
    partition: int = 0  # 0 shifted windows, 1 interleaved windows (shift 0)
    bias: bool = True  # False: no bias table (position-free attention)

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.W


WORKLOADS: Dict[int, Workload] = {
    0: Workload(0, "tiny-swinv2-fp32-16x16-M8", "f32", 1, 16, 16, 2, 32, 8, (0, 4),
                MODE_COSINE_CPB, tau=(0.1, 0.1), cpb_hidden=512),
    1: Workload(1, "swin-t-stage1-56x56-M7", "bf16", 32, 56, 56, 3, 32, 7, (3,), MODE_DOT_BIAS),
    2: Workload(2, "swinv2-t-stage1-64x64-M16", "bf16", 64, 64, 64, 3, 32, 16, (8,),
                MODE_COSINE_CPB, tau=(0.05, 0.2), cpb_hidden=512),
    3: Workload(3, "flashswin-t-dense-112x112-M32", "bf16", 16, 112, 112, 3, 32, 32, (16,),
                MODE_ROPE, rope_base=100.0),
    4: Workload(4, "swinv2-g-stage1-384x384-M24", "bf16", 2, 384, 384, 16, 32, 24, (12,),
                MODE_COSINE_CPB, tau=(0.05, 0.2), cpb_hidden=512),
    # Iwin-T stage 1 at 224 px: Swin-T's shape, interleaved windows, no
    # position bias (the depthwise convolution beside it is not attention)
    5: Workload(5, "iwin-t-stage1-56x56-M7-interleaved", "bf16", 32, 56, 56, 3, 32, 7, (0,), MODE_DOT_BIAS,
                partition=1, bias=False),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return rounded.astype(np.uint32).view(np.float32)


def make_inputs(w: Workload, B: Optional[int] = None, H: Optional[int] = None,
                W: Optional[int] = None, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw one workload's tensors (float32 numpy; bf16 workloads pre-rounded).

    ``B``, ``H``, ``W`` and ``seed`` override the workload's values for reduced
    test cases; the distributions stay the same.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    W = w.W if W is None else W
    ss = np.random.SeedSequence(1000 + w.index if seed is None else seed)
    gens = [np.random.Generator(np.random.PCG64(c)) for c in ss.spawn(8)]
    shape = (B, H, W, w.heads, w.d)
    out: Dict[str, np.ndarray] = {}
    for name, g in zip(("q", "k", "v"), gens[:3]):
        x = g.standard_normal(shape, dtype=np.float32)
        out[name] = round_to_bf16(x) if w.dtype == "bf16" else x
    R = 2 * w.M - 1
    if w.mode in (MODE_DOT_BIAS, MODE_COSINE_CPB) and w.bias:
        if w.cpb_hidden:
            hid = w.cpb_hidden
            out["w1"] = (0.02 * gens[3].standard_normal((hid, 2))).astype(np.float32)
            out["b1"] = (0.02 * gens[4].standard_normal((hid,))).astype(np.float32)
            out["w2"] = (0.02 * gens[5].standard_normal((w.heads, hid))).astype(np.float32)
            out["b2"] = (0.02 * gens[6].standard_normal((w.heads,))).astype(np.float32)
        else:
            out["table"] = (0.02 * gens[3].standard_normal((R * R, w.heads))).astype(np.float32)
    if w.mode == MODE_COSINE_CPB:
        lo, hi = w.tau
        out["tau"] = gens[7].uniform(lo, hi, size=(w.heads,)).astype(np.float32)
    if w.mode == MODE_ROPE:
        q4 = w.d // 4
        t = np.arange(q4, dtype=np.float64)
        f = (w.rope_base ** (-t / q4)).astype(np.float32)
        out["rope_freqs"] = np.stack([f, f]).astype(np.float32)  # [2][d/4]: row axis, col axis
    return out


def make_dout(w: Workload, B: Optional[int] = None, H: Optional[int] = None, W: Optional[int] = None,
              seed: Optional[int] = None) -> np.ndarray:
    """An output gradient for the backward pass: N(0, 1) of q's shape (its own
    stream, SeedSequence(5000 + index) unless ``seed`` is given), rounded to
    bf16 for bf16 workloads."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    W = w.W if W is None else W
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(5000 + w.index if seed is None else seed)))
    x = g.standard_normal((B, H, W, w.heads, w.d), dtype=np.float32)
    return round_to_bf16(x) if w.dtype == "bf16" else x


def make_block_inputs(w: Workload, B: Optional[int] = None, H: Optional[int] = None, W: Optional[int] = None,
                      seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Block input x [B, H, W, C] ~ N(0, 1) and the parameters around the
    attention (SeedSequence(9000 + index) unless ``seed``, spawned into eight
    streams in this order): w_qkv [3C, C] and w_o [C, C] ~ N(0, 1/C) (so q, k,
    v and the projection keep unit scale), b_qkv [3C] and b_o [C] ~ N(0, 0.02),
    gamma ~ 1 + N(0, 0.1) and beta ~ N(0, 0.1) over C; x and the weights are
    rounded to bf16 for bf16 workloads, biases and norm parameters stay fp32.
    The attention's own parameters come from ``make_inputs``."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    W = w.W if W is None else W
    C = w.heads * w.d
    ss = np.random.SeedSequence(9000 + w.index if seed is None else seed)
    g = [np.random.Generator(np.random.PCG64(c)) for c in ss.spawn(8)]
    rb = (lambda a: round_to_bf16(a)) if w.dtype == "bf16" else (lambda a: a)
    f32 = lambda a: a.astype(np.float32)
    return {
        "x": rb(g[0].standard_normal((B, H, W, C), dtype=np.float32)),
        "w_qkv": rb(f32(g[1].standard_normal((3 * C, C)) / np.sqrt(C))),
        "b_qkv": f32(0.02 * g[2].standard_normal(3 * C)),
        "w_o": rb(f32(g[3].standard_normal((C, C)) / np.sqrt(C))),
        "b_o": f32(0.02 * g[4].standard_normal(C)),
        "gamma": f32(1.0 + 0.1 * g[5].standard_normal(C)),
        "beta": f32(0.1 * g[6].standard_normal(C)),
    }
