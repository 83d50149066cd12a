"""Double-precision oracle of the steps either side of the window attention in
a Swin V2 block — TEST INFRASTRUCTURE (only ``tests/``, ``smoke()`` and the
benchmark's CPU leg may import it).

"Swin Transformer V2" wiki card, Method item 1 "Residual post-norm" (§3.2,
fig. 1) and the ``swin_v2_block`` pseudocode: the attention branch's output is
layer-normalised before it is added to the main path,
    features = features + norm_1(attention(features)).
The attention branch is the usual linear projection of the block input to
queries, keys and values, the window attention per head, and a linear output
projection.  Plain numpy in float64; nothing is blocked, fused or reordered.
"""
from __future__ import annotations

import numpy as np

from . import PARTITION_SHIFTED, window_attn


def linear(x, w, b=None):
    """x W^T + b over the last axis (w [out, in], the linear-layer layout)."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    return y if b is None else y + np.asarray(b, dtype=np.float64)


def qkv_proj(x, w_qkv, b_qkv=None):
    """Queries, keys and values of the block input: one linear map to 3C
    channels, split in that order."""
    C = x.shape[-1]
    y = linear(x, w_qkv, b_qkv)
    return y[..., :C], y[..., C:2 * C], y[..., 2 * C:]


def layer_norm(y, gamma=None, beta=None, eps=1e-5):
    """(y - mean) / sqrt(var + eps) * gamma + beta over the last axis, with the
    biased variance."""
    y = np.asarray(y, dtype=np.float64)
    mean = y.mean(axis=-1, keepdims=True)
    var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)
    z = (y - mean) / np.sqrt(var + eps)
    if gamma is not None:
        z = z * np.asarray(gamma, dtype=np.float64)
    if beta is not None:
        z = z + np.asarray(beta, dtype=np.float64)
    return z


def proj_postnorm_residual(a, w_o, b_o, x, gamma=None, beta=None, eps=1e-5):
    """x + LN(a W_o^T + b_o): the residual post-norm of §3.2."""
    return np.asarray(x, dtype=np.float64) + layer_norm(linear(a, w_o, b_o), gamma, beta, eps)


def attn_block(x, heads, w_qkv, b_qkv, w_o, b_o, gamma, beta, M, shift, mode, eps=1e-5, tau=None, table=None,
               rope_freqs=None, partition=PARTITION_SHIFTED, round_to=None):
    """The attention half of swin_v2_block for x [B, H, W, C].  ``round_to``
    (a function) is applied to q, k, v and to the attention output, the
    tensors a bf16 implementation stores between its steps; None keeps float64
    throughout."""
    B, H, W, C = x.shape
    d = C // heads
    rnd = round_to or (lambda t: t)
    q, k, v = (rnd(t).reshape(B, H, W, heads, d) for t in qkv_proj(x, w_qkv, b_qkv))
    a = window_attn(q, k, v, M, shift, mode, tau=tau, table=table, rope_freqs=rope_freqs, partition=partition)
    return proj_postnorm_residual(rnd(a.reshape(B, H, W, C)), w_o, b_o, x, gamma, beta, eps)
