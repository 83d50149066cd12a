"""Pins of the oracle's interleaved-window partition ("Iwin Transformer",
abstract: interleaved window attention; the index map is a reading).

With G = ceil(L / M) windows per axis, window a holds the tokens a + G i
(i < M) inside the axis, and i is the window-local coordinate that offsets and
RoPE positions use.  Each pin ties the interleaved path to the shifted one,
which has its own pins:
  * gathering one interleaved window's tokens into a small grid (in i order)
    and running the shifted oracle with shift 0 on it (one window then covers
    the whole small grid) gives that window's outputs and gradients, also when
    M does not divide the grid;
  * on a grid that M divides, interleaved attention equals shifted attention
    (shift 0) on the grid permuted so that every interleaved window becomes
    one contiguous M x M block;
  * with M covering the grid (G = 1) both partitions are global attention.
"""
import numpy as np
import pytest

import oracle

IL = oracle.PARTITION_INTERLEAVED


def inputs(B, H, W, nh, d, M, seed):
    rng = np.random.default_rng(seed)
    q, k, v, g = (rng.standard_normal((B, H, W, nh, d)) for _ in range(4))
    table = 0.3 * rng.standard_normal(((2 * M - 1) ** 2, nh))
    tau = rng.uniform(0.05, 0.3, nh)
    freqs = rng.uniform(0.1, 1.2, (2, d // 4))
    return q, k, v, g, table, tau, freqs


def kw(mode, table, tau, freqs):
    return dict(tau=tau if mode == 1 else None, table=table if mode != 2 else None,
                rope_freqs=freqs if mode == 2 else None)


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,H,W,nh,d,M", [(1, 12, 8, 2, 8, 4), (2, 13, 10, 1, 8, 4), (1, 9, 14, 2, 4, 3),
                                          (1, 7, 7, 1, 8, 5), (1, 15, 11, 2, 8, 7)])
def test_each_window_is_a_single_window_problem(mode, B, H, W, nh, d, M):
    q, k, v, g, table, tau, freqs = inputs(B, H, W, nh, d, M, 3 * H + W + mode)
    a = kw(mode, table, tau, freqs)
    out = oracle.window_attn(q, k, v, M, 0, mode, partition=IL, **a)
    grads = oracle.window_attn_bwd(q, k, v, g, M, 0, mode, partition=IL, **a)
    Gy, Gx = -(-H // M), -(-W // M)
    summed = {n: np.zeros_like(grads[n]) for n in ("dtable", "dtau", "drope") if n in grads}
    seen = np.zeros((H, W), dtype=int)
    for ay in range(Gy):
        ys = np.arange(ay, H, Gy)
        for ax in range(Gx):
            xs = np.arange(ax, W, Gx)
            sub = np.ix_(range(B), ys, xs)
            seen[np.ix_(ys, xs)] += 1
            o1 = oracle.window_attn(q[sub], k[sub], v[sub], M, 0, mode, **a)
            np.testing.assert_allclose(out[sub], o1, rtol=0, atol=1e-13)
            g1 = oracle.window_attn_bwd(q[sub], k[sub], v[sub], g[sub], M, 0, mode, **a)
            for n in ("dq", "dk", "dv"):
                np.testing.assert_allclose(grads[n][sub], g1[n], rtol=0, atol=1e-12)
            for n in summed:
                summed[n] += g1[n]
    assert np.all(seen == 1)  # the windows partition the grid
    for n in summed:
        np.testing.assert_allclose(grads[n], summed[n], rtol=1e-12, atol=1e-12)


def permute_axis(L, M):
    """Index array p with permuted[j] = original[p[j]]: block a holds a + G i."""
    G = L // M
    return np.array([a + G * i for a in range(G) for i in range(M)])


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,H,W,nh,d,M", [(1, 12, 8, 2, 8, 4), (2, 9, 6, 1, 8, 3), (1, 10, 10, 1, 4, 5)])
def test_equals_regular_windows_on_the_permuted_grid(mode, B, H, W, nh, d, M):
    q, k, v, g, table, tau, freqs = inputs(B, H, W, nh, d, M, 5 * H + W + mode)
    a = kw(mode, table, tau, freqs)
    py, px = permute_axis(H, M), permute_axis(W, M)
    perm = lambda t: t[:, py][:, :, px]
    inv_y, inv_x = np.argsort(py), np.argsort(px)
    unperm = lambda t: t[:, inv_y][:, :, inv_x]
    out = oracle.window_attn(q, k, v, M, 0, mode, partition=IL, **a)
    ref = unperm(oracle.window_attn(perm(q), perm(k), perm(v), M, 0, mode, **a))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)
    gi = oracle.window_attn_bwd(q, k, v, g, M, 0, mode, partition=IL, **a)
    gs = oracle.window_attn_bwd(perm(q), perm(k), perm(v), perm(g), M, 0, mode, **a)
    for n in ("dq", "dk", "dv"):
        np.testing.assert_allclose(gi[n], unperm(gs[n]), rtol=0, atol=1e-12)
    for n in ("dtable", "dtau", "drope"):
        if n in gi:
            np.testing.assert_allclose(gi[n], gs[n], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", [0, 2])
def test_one_window_covering_the_grid(mode):
    q, k, v, g, table, tau, freqs = inputs(1, 6, 5, 2, 8, 8, 17)
    a = kw(mode, table, tau, freqs)
    np.testing.assert_array_equal(oracle.window_attn(q, k, v, 8, 0, mode, partition=IL, **a),
                                  oracle.window_attn(q, k, v, 8, 0, mode, **a))


def test_interleaved_rejects_a_shift():
    q = np.zeros((1, 8, 8, 1, 8))
    with pytest.raises(ValueError):
        oracle.window_attn(q, q, q, 4, 2, 0, partition=IL)
    with pytest.raises(ValueError):
        oracle.window_attn_bwd(q, q, q, q, 4, 2, 0, partition=IL)
