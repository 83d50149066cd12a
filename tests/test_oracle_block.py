"""Pins of the block oracle (oracle.block): the projections and the residual
post-norm around the window attention ("Swin Transformer V2", Method item 1,
§3.2, fig. 1, swin_v2_block pseudocode), against float64 library routines,
closed forms and special cases."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from oracle import block


def rnd(*shape, seed=0, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


def test_linear_and_layer_norm_match_library_routines():
    x, w, b = rnd(5, 7, 24, seed=1), rnd(40, 24, seed=2), rnd(40, seed=3)
    np.testing.assert_allclose(block.linear(x, w, b), F.linear(*(torch.tensor(t) for t in (x, w, b))).numpy(),
                               rtol=1e-13, atol=1e-13)
    y, g, be = rnd(6, 96, seed=4, scale=3.0), rnd(96, seed=5), rnd(96, seed=6)
    ref = F.layer_norm(torch.tensor(y), (96,), torch.tensor(g), torch.tensor(be), eps=1e-5).numpy()
    np.testing.assert_allclose(block.layer_norm(y, g, be, 1e-5), ref, rtol=1e-12, atol=1e-12)


def test_layer_norm_closed_form():
    """gamma = 1, beta = 0: every row has mean 0 and variance var / (var + eps)."""
    y = rnd(9, 32, seed=7, scale=0.01)
    z = block.layer_norm(y, eps=1e-5)
    var = y.var(axis=-1)
    np.testing.assert_allclose(z.mean(axis=-1), 0.0, atol=1e-14)
    np.testing.assert_allclose(z.var(axis=-1), var / (var + 1e-5), rtol=1e-12)


def test_qkv_split_order():
    """W_qkv = [I; 2I; 3I] gives q = x, k = 2x, v = 3x (+ their bias slices)."""
    C = 16
    x = rnd(3, 4, C, seed=8)
    w = np.concatenate([np.eye(C), 2 * np.eye(C), 3 * np.eye(C)])
    b = np.arange(3 * C, dtype=np.float64)
    q, k, v = block.qkv_proj(x, w, b)
    np.testing.assert_allclose(q, x + b[:C], atol=1e-15)
    np.testing.assert_allclose(k, 2 * x + b[C:2 * C], atol=1e-15)
    np.testing.assert_allclose(v, 3 * x + b[2 * C:], atol=1e-15)


def test_zero_projection_leaves_the_residual_plus_beta():
    """With W_o = 0 and b_o = 0 the normalised branch is 0, so out = x + beta."""
    x, a, be = rnd(2, 5, 32, seed=9), rnd(2, 5, 32, seed=10), rnd(32, seed=11)
    out = block.proj_postnorm_residual(a, np.zeros((32, 32)), None, x, rnd(32, seed=12), be)
    np.testing.assert_allclose(out, x + be, rtol=0, atol=1e-15)


def test_post_norm_is_on_the_branch_not_the_input():
    """Scaling the branch (W_o, b_o by c > 0) leaves the output unchanged up to
    eps: the norm sits after the branch (post-norm), not before it."""
    x, a = rnd(4, 3, 48, seed=13), rnd(4, 3, 48, seed=14)
    w, b = rnd(48, 48, seed=15), rnd(48, seed=16)
    o1 = block.proj_postnorm_residual(a, w, b, x, eps=1e-12)
    o2 = block.proj_postnorm_residual(a, 7.0 * w, 7.0 * b, x, eps=1e-12)
    np.testing.assert_allclose(o1, o2, rtol=1e-9, atol=1e-9)


def test_block_with_identity_projections_is_attention_plus_norm():
    """W_qkv = [I; I; I], W_o = I, no biases: the block is x + LN(attn(x, x, x))."""
    B, H, W, heads, d, M, s = 1, 8, 8, 2, 8, 4, 2
    C = heads * d
    x = rnd(B, H, W, C, seed=17)
    table = rnd((2 * M - 1) ** 2, heads, seed=18, scale=0.1)
    w = np.concatenate([np.eye(C)] * 3)
    out = block.attn_block(x, heads, w, None, np.eye(C), None, None, None, M, s, 0, table=table)
    xh = x.reshape(B, H, W, heads, d)
    a = oracle.window_attn(xh, xh, xh, M, s, 0, table=table).reshape(B, H, W, C)
    np.testing.assert_allclose(out, x + block.layer_norm(a), rtol=1e-13, atol=1e-13)
