"""Pins for the CPU oracle: checks against facts fixed outside the oracle itself.

Each test compares the oracle with something it does not share code with:
values printed in the pages (tests/golden), closed forms, invariances of the
definition, library routines (torch float64 scaled_dot_product_attention and
Linear layers), and an independent route to the same attention (Swin's literal
cyclic roll + window partition + band mask, written here with torch ops).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from conftest import read_golden

torch.set_default_dtype(torch.float64)


# ---------------------------------------------------------------------------
# eq. 4 worked example ("Swin Transformer V2", Method item 3 / §3.3)
# ---------------------------------------------------------------------------
def test_log_coords_worked_example():
    g = read_golden("log_cpb_worked_example.txt")
    tol = 0.5 * 10 ** (-g["printed_decimals"])
    small = oracle.log_coords(int(g["M_small"]))
    large = oracle.log_coords(int(g["M_large"]))
    assert abs(np.abs(small).max() - g["log_max_small"]) <= tol
    assert abs(np.abs(large).max() - g["log_max_large"]) <= tol
    # symmetric range: the minimum is the negated maximum
    assert small.min() == -small.max() and large.min() == -large.max()
    ratio = (np.abs(large).max() - np.abs(small).max()) / np.abs(small).max()
    assert abs(ratio - g["log_extrapolation_ratio"]) <= 0.005
    raw = (g["M_large"] - 1) / (g["M_small"] - 1) - 1.0
    assert abs(raw + 1.0 - (1.0 + 8.0 / 7.0)) < 1e-12 and abs(raw - g["raw_extrapolation_ratio"]) < 0.005


def test_log_coords_closed_form_and_layout():
    M = 5
    t = oracle.log_coords(M)
    R = 2 * M - 1
    for dy in range(-(M - 1), M):
        for dx in range(-(M - 1), M):
            row = (dy + M - 1) * R + (dx + M - 1)
            assert t[row, 0] == pytest.approx(math.copysign(math.log1p(abs(dx)), dx) if dx else 0.0, abs=1e-15)
            assert t[row, 1] == pytest.approx(math.copysign(math.log1p(abs(dy)), dy) if dy else 0.0, abs=1e-15)
    assert oracle.log_map(0.0) == 0.0
    assert oracle.log_map(-3.0) == -oracle.log_map(3.0)


# ---------------------------------------------------------------------------
# eq. 3: G = Linear -> ReLU -> Linear
# ---------------------------------------------------------------------------
def test_cpb_zero_w2_gives_b2():
    rng = np.random.default_rng(1)
    w1 = rng.standard_normal((16, 2))
    b1 = rng.standard_normal(16)
    w2 = np.zeros((3, 16))
    b2 = rng.standard_normal(3)
    t = oracle.cpb_table(6, 3, w1, b1, w2, b2)
    assert np.array_equal(t, np.broadcast_to(b2, t.shape))


def test_cpb_single_unit_closed_form():
    # hidden = 1, w1 picks dx_hat (then dy_hat): table = relu(+-ln(1+|d|))
    M = 4
    R = 2 * M - 1
    for pick in (0, 1):
        w1 = np.zeros((1, 2))
        w1[0, pick] = 1.0
        t = oracle.cpb_table(M, 1, w1, None, np.ones((1, 1)), None)
        for dy in range(-(M - 1), M):
            for dx in range(-(M - 1), M):
                dd = dx if pick == 0 else dy
                want = math.log(1 + dd) if dd > 0 else 0.0
                assert t[(dy + M - 1) * R + (dx + M - 1), 0] == pytest.approx(want, abs=1e-15)


def test_cpb_matches_torch_linear_stack():
    rng = np.random.default_rng(2)
    M, heads, hid = 7, 4, 512
    w1 = 0.5 * rng.standard_normal((hid, 2))
    b1 = 0.5 * rng.standard_normal(hid)
    w2 = 0.1 * rng.standard_normal((heads, hid))
    b2 = rng.standard_normal(heads)
    d = torch.arange(-(M - 1), M, dtype=torch.float64)
    dy, dx = torch.meshgrid(d, d, indexing="ij")
    coords = torch.stack([dx, dy], -1).reshape(-1, 2)
    coords = torch.sign(coords) * torch.log1p(coords.abs())
    ref = F.linear(F.relu(F.linear(coords, torch.tensor(w1), torch.tensor(b1))), torch.tensor(w2), torch.tensor(b2))
    got = oracle.cpb_table(M, heads, w1, b1, w2, b2)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Swin bookkeeping tables: literal roll (oracle) vs closed form (here)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("H,W,M,s", [(8, 8, 4, 0), (8, 8, 4, 2), (12, 10, 4, 3), (14, 14, 7, 3),
                                     (9, 11, 5, 1), (5, 7, 8, 3), (56, 56, 7, 3), (112, 112, 32, 16),
                                     (64, 64, 16, 8)])
def test_index_tables_closed_form(H, W, M, s):
    tw, tr, tl, ri = oracle.index_tables(H, W, M, s)
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    y = np.arange(H)[:, None]
    x = np.arange(W)[None, :]
    u = (y - s) % Hp
    v = (x - s) % Wp
    assert np.array_equal(tw, (u // M) * (Wp // M) + v // M)
    assert np.array_equal(tl, (u % M) * M + v % M)
    band = lambda a, L: np.where(a < L - M, 0, np.where(a < L - s, 1, 2)) if s else np.zeros_like(a)
    assert np.array_equal(tr, band(u, Hp) * 3 + band(v, Wp))
    i = np.arange(M * M)
    yi, xi = i // M, i % M
    assert np.array_equal(ri, (yi[:, None] - yi[None, :] + M - 1) * (2 * M - 1) + (xi[:, None] - xi[None, :] + M - 1))


@pytest.mark.parametrize("H,M,s", [(16, 8, 4), (56, 7, 3), (112, 32, 16), (10, 4, 3), (5, 8, 7)])
def test_segments_equal_window_and_band(H, M, s):
    """Same segment  <=>  same rolled window and same band (1-D cut of the tables)."""
    tw, tr, _, _ = oracle.index_tables(H, 1, M, s)
    seg = np.array([oracle.segment_of(M, s, y) for y in range(H)])
    same_seg = seg[:, None] == seg[None, :]
    same_win = (tw[:, 0][:, None] == tw[:, 0][None, :]) & (tr[:, 0][:, None] == tr[:, 0][None, :])
    assert np.array_equal(same_seg, same_win)
    # boundaries sit at s + kM
    starts = [y for y in range(1, H) if seg[y] != seg[y - 1]]
    assert all((y - s) % M == 0 for y in starts)


# ---------------------------------------------------------------------------
# Independent route: Swin's cyclic roll + window partition + band mask (torch)
# ---------------------------------------------------------------------------
def rope_complex(x, py, px, freqs):
    """RoPE written with complex exponentials: pairs (2t, 2t+1) as a + ib."""
    d = x.shape[-1]
    h = d // 2
    out = x.clone()
    for half, p, f in ((0, py, freqs[0]), (1, px, freqs[1])):
        seg = x[..., half * h:(half + 1) * h]
        z = torch.complex(seg[..., 0::2], seg[..., 1::2])
        rot = torch.exp(1j * p[..., None].to(torch.float64) * torch.tensor(f)[None, :])
        z = z * rot
        out[..., half * h:(half + 1) * h][..., 0::2] = z.real
        out[..., half * h:(half + 1) * h][..., 1::2] = z.imag
    return out


def roll_route(q, k, v, M, s, mode, tau=None, table=None, freqs=None):
    """Swin-style computation on padded, rolled windows; padding keys masked out."""
    q, k, v = (torch.tensor(a) for a in (q, k, v))
    B, H, W, nh, d = q.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    pad = lambda t: F.pad(t, (0, 0, 0, 0, 0, Wp - W, 0, Hp - H))
    real = torch.zeros(Hp, Wp, dtype=torch.bool)
    real[:H, :W] = True
    q, k, v = pad(q), pad(k), pad(v)
    roll = lambda t, dims: torch.roll(t, shifts=(-s, -s), dims=dims)
    q, k, v = roll(q, (1, 2)), roll(k, (1, 2)), roll(v, (1, 2))
    real = roll(real, (0, 1))
    band = torch.zeros(Hp, Wp, dtype=torch.long)
    if s:
        cnt = 0
        for hs in (slice(0, Hp - M), slice(Hp - M, Hp - s), slice(Hp - s, None)):
            for ws in (slice(0, Wp - M), slice(Wp - M, Wp - s), slice(Wp - s, None)):
                band[hs, ws] = cnt
                cnt += 1
    nWy, nWx, N = Hp // M, Wp // M, M * M

    def part(t):  # [B, Hp, Wp, ...] -> [B, nW, N, ...]
        b0 = t.shape[0]
        t = t.reshape(b0, nWy, M, nWx, M, *t.shape[3:]).transpose(2, 3)
        return t.reshape(b0, nWy * nWx, N, *t.shape[5:])

    qw, kw, vw = part(q), part(k), part(v)  # [B, nW, N, nh, d]
    bw = part(band[None, ..., None])[0, ..., 0]  # [nW, N]
    rw = part(real[None, ..., None])[0, ..., 0]
    mask = (bw[:, :, None] == bw[:, None, :]) & rw[:, None, :]  # [nW, N, N]
    i = torch.arange(N)
    yi, xi = i // M, i % M
    rel = (yi[:, None] - yi[None, :] + M - 1) * (2 * M - 1) + (xi[:, None] - xi[None, :] + M - 1)
    qh, kh, vh = (t.permute(0, 1, 3, 2, 4) for t in (qw, kw, vw))  # [B, nW, nh, N, d]
    add = torch.zeros(nh, N, N)
    if table is not None and mode != 2:
        add = torch.tensor(table)[rel].permute(2, 0, 1)
    amask = torch.where(mask[None, :, None], add[None, None], torch.tensor(-math.inf))
    if mode == 0:
        o = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=amask, scale=1 / math.sqrt(d))
    elif mode == 1:
        t = torch.clamp(torch.tensor(tau), min=0.01)
        qn, kn = F.normalize(qh, dim=-1), F.normalize(kh, dim=-1)
        qn = qn / t[None, None, :, None, None]
        o = F.scaled_dot_product_attention(qn, kn, vh, attn_mask=amask, scale=1.0)
    else:
        py, px = yi % M, xi % M  # window-local coordinates in the rolled frame
        qr = rope_complex(qh, py, px, freqs)
        kr = rope_complex(kh, py, px, freqs)
        o = F.scaled_dot_product_attention(qr, kr, vh, attn_mask=amask, scale=1 / math.sqrt(d))
    o = o.permute(0, 1, 3, 2, 4).reshape(B, nWy, nWx, M, M, nh, d).transpose(2, 3).reshape(B, Hp, Wp, nh, d)
    o = torch.roll(o, shifts=(s, s), dims=(1, 2))
    return o[:, :H, :W].numpy()


def rand_case(B, H, W, nh, d, M, seed, mode):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, W, nh, d)) for _ in range(3))
    R = 2 * M - 1
    table = 0.5 * rng.standard_normal((R * R, nh))
    tau = rng.uniform(0.05, 0.5, nh)
    f = rng.uniform(0.0, 1.5, (2, d // 4))
    return q, k, v, table, tau, f


CASES = [(8, 8, 4, 2), (12, 10, 4, 3), (14, 14, 7, 3), (9, 11, 5, 1), (5, 7, 8, 3), (16, 12, 8, 4),
         (24, 24, 8, 4), (7, 7, 7, 3), (8, 8, 4, 0), (13, 9, 3, 2)]


@pytest.mark.parametrize("H,W,M,s", CASES)
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_window_attn_equals_roll_route(H, W, M, s, mode):
    q, k, v, table, tau, f = rand_case(2, H, W, 2, 8, M, 10 * H + W + M + s, mode)
    got = oracle.window_attn(q, k, v, M, s, mode, tau=tau, table=table, rope_freqs=f)
    ref = roll_route(q, k, v, M, s, mode, tau=tau, table=table, freqs=f)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("s", range(5))
def test_all_shifts_small_window(s):
    q, k, v, table, tau, f = rand_case(1, 10, 9, 2, 8, 5, 77 + s, 0)
    for mode in (0, 1, 2):
        got = oracle.window_attn(q, k, v, 5, s, mode, tau=tau, table=table, rope_freqs=f)
        ref = roll_route(q, k, v, 5, s, mode, tau=tau, table=table, freqs=f)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_one_window_is_global_attention():
    """M >= H, W and shift 0: one window, i.e. plain attention over the grid."""
    rng = np.random.default_rng(5)
    B, H, W, nh, d = 2, 6, 5, 3, 8
    q, k, v = (rng.standard_normal((B, H, W, nh, d)) for _ in range(3))
    tq, tk, tv = (torch.tensor(a).reshape(B, H * W, nh, d).transpose(1, 2) for a in (q, k, v))
    ref0 = F.scaled_dot_product_attention(tq, tk, tv, scale=1 / math.sqrt(d))
    got0 = oracle.window_attn(q, k, v, 8, 0, 0).reshape(B, H * W, nh, d).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(got0, ref0.numpy(), rtol=0, atol=1e-12)
    tau = np.array([0.07, 0.2, 1.3])
    ref1 = F.scaled_dot_product_attention(F.normalize(tq, dim=-1) / torch.tensor(tau)[None, :, None, None],
                                          F.normalize(tk, dim=-1), tv, scale=1.0)
    got1 = oracle.window_attn(q, k, v, 8, 0, 1, tau=tau).reshape(B, H * W, nh, d).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(got1, ref1.numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Invariances fixed by eq. 2 and by softmax
# ---------------------------------------------------------------------------
def test_cosine_scale_invariance_and_tau_clamp():
    q, k, v, table, tau, _ = rand_case(1, 9, 9, 2, 8, 4, 11, 1)
    rng = np.random.default_rng(12)
    a = rng.uniform(0.1, 10.0, q.shape[:-1] + (1,))
    b = rng.uniform(0.1, 10.0, k.shape[:-1] + (1,))
    base = oracle.window_attn(q, k, v, 4, 2, 1, tau=tau, table=table)
    scaled = oracle.window_attn(q * a, k * b, v, 4, 2, 1, tau=tau, table=table)
    np.testing.assert_allclose(scaled, base, rtol=0, atol=1e-12)
    lo = oracle.window_attn(q, k, v, 4, 2, 1, tau=np.array([0.001, 1e-9]), table=table)
    at = oracle.window_attn(q, k, v, 4, 2, 1, tau=np.array([0.01, 0.01]), table=table)
    np.testing.assert_array_equal(lo, at)
    # a changed tau must change the output (the clamp is not applied everywhere)
    assert np.abs(oracle.window_attn(q, k, v, 4, 2, 1, tau=np.array([0.02, 0.02]), table=table) - at).max() > 1e-3


def test_constant_values_and_constant_bias():
    q, k, v, table, tau, f = rand_case(1, 10, 10, 2, 8, 4, 13, 0)
    vc = np.broadcast_to(np.arange(8.0), v.shape).copy()
    for mode in (0, 1, 2):
        o = oracle.window_attn(q, k, vc, 4, 3, mode, tau=tau, table=table, rope_freqs=f)
        np.testing.assert_allclose(o, vc, rtol=0, atol=1e-12)
    for mode in (0, 1):
        zero = oracle.window_attn(q, k, v, 4, 3, mode, tau=tau, table=np.zeros_like(table))
        const = oracle.window_attn(q, k, v, 4, 3, mode, tau=tau, table=np.full_like(table, 3.25))
        np.testing.assert_allclose(const, zero, rtol=0, atol=1e-12)
        nob = oracle.window_attn(q, k, v, 4, 3, mode, tau=tau, table=None)
        np.testing.assert_allclose(nob, zero, rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,W,M,s", [(6, 6, 4, 2), (7, 5, 3, 1), (6, 6, 7, 3)])
def test_one_hot_values_recover_weights(H, W, M, s):
    """v = one-hot(token) makes the output the attention row: masked weights are
    exactly zero, rows sum to one, and the support is the query's rectangle."""
    n = H * W
    rng = np.random.default_rng(H * W + M)
    q, k = rng.standard_normal((2, 1, H, W, 1, 4))
    v = np.eye(n).reshape(1, H, W, 1, n)
    qd = np.concatenate([q, np.zeros((1, H, W, 1, n - 4))], -1)
    kd = np.concatenate([k, np.zeros((1, H, W, 1, n - 4))], -1)
    R = 2 * M - 1
    table = rng.standard_normal((R * R, 1))
    P = oracle.window_attn(qd, kd, v, M, s, 0, table=table).reshape(n, n)
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=0, atol=1e-12)
    # support from Swin's band/window labels, computed independently
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    yy, xx = np.divmod(np.arange(n), W)
    u, vv = (yy - s) % Hp, (xx - s) % Wp
    win = (u // M) * (Wp // M) + vv // M
    band = lambda a, L: np.where(a < L - M, 0, np.where(a < L - s, 1, 2)) if s else np.zeros_like(a)
    lab = win * 9 + band(u, Hp) * 3 + band(vv, Wp)
    allowed = lab[:, None] == lab[None, :]
    assert np.all(P[~allowed] == 0.0)
    assert np.all(P[allowed] > 0.0)


# ---------------------------------------------------------------------------
# RoPE (FlashSwin abstract: window-local 2D RoPE, no bias)
# ---------------------------------------------------------------------------
def test_rope_zero_frequency_is_plain_dot_product():
    q, k, v, _, _, _ = rand_case(2, 12, 12, 2, 8, 4, 21, 2)
    a = oracle.window_attn(q, k, v, 4, 2, 2, rope_freqs=np.zeros((2, 2)))
    b = oracle.window_attn(q, k, v, 4, 2, 0, table=None)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_rope_scores_depend_on_offsets_only():
    """Within a rectangle the RoPE logit is Re(sum z_q conj(z_k) e^{i (p_q - p_k) w}):
    only the offset between the two tokens enters, whatever the window frame."""
    rng = np.random.default_rng(31)
    H = W = 9
    M, s, d = 6, 3, 8
    q, k, v = (rng.standard_normal((1, H, W, 1, d)) for _ in range(3))
    f = rng.uniform(0.1, 1.0, (2, d // 4))
    for (yq, xq) in [(0, 0), (4, 7), (8, 2), (2, 5)]:
        seg = lambda a: (a + (M - s) % M) // M
        keys = [(y, x) for y in range(H) for x in range(W) if seg(y) == seg(yq) and seg(x) == seg(xq)]
        lg = []
        for (y, x) in keys:
            acc = 0.0
            for half, dd in ((0, yq - y), (1, xq - x)):
                zq = q[0, yq, xq, 0, half * 4:(half + 1) * 4]
                zk = k[0, y, x, 0, half * 4:(half + 1) * 4]
                zq = zq[0::2] + 1j * zq[1::2]
                zk = zk[0::2] + 1j * zk[1::2]
                acc += np.real(np.sum(zq * np.conj(zk) * np.exp(1j * dd * f[half])))
            lg.append(acc / math.sqrt(d))
        lg = np.array(lg)
        w = np.exp(lg - lg.max())
        w /= w.sum()
        want = sum(wi * v[0, y, x, 0] for wi, (y, x) in zip(w, keys))
        got = oracle.window_attn(q, k, v, M, s, 2, rope_freqs=f, queries=[yq * W + xq])[0, 0]
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_query_subset_matches_full_output():
    q, k, v, table, tau, f = rand_case(2, 11, 9, 2, 8, 4, 41, 1)
    full = oracle.window_attn(q, k, v, 4, 1, 1, tau=tau, table=table)
    ids = np.array([0, 5, 98, 99, 150, 197])
    sub = oracle.window_attn(q, k, v, 4, 1, 1, tau=tau, table=table, queries=ids)
    np.testing.assert_array_equal(sub, full.reshape(-1, 2, 8)[ids])


def test_rejects_bad_arguments():
    q = np.zeros((1, 4, 4, 1, 8))
    with pytest.raises(ValueError):
        oracle.window_attn(q, q, q, 4, 4, 0)  # shift must be < M
    with pytest.raises(ValueError):
        oracle.window_attn(q, q, q, 4, 0, 1)  # cosine needs tau


# ---- the released code's form of G ("Swin Transformer V2", "Paper vs code")

def test_code_coordinates_endpoints_do_not_depend_on_the_window():
    """Offsets are normalised by (window - 1) and scaled by 8 before the
    log2 map, so the extreme offsets +-(M-1) land on +-log2(9)/log2(8) for
    every window size (normalising by M, or a natural log, would not)."""
    end = math.log2(9.0) / 3.0
    for M in (2, 3, 7, 8, 12, 16, 24, 32):
        assert oracle.log2_map(M - 1, M) == pytest.approx(end, abs=1e-15)
        assert oracle.log2_map(-(M - 1), M) == pytest.approx(-end, abs=1e-15)
        assert oracle.log2_map(0, M) == 0.0


def test_code_coordinates_odd_and_increasing():
    for M in (5, 16):
        vals = [oracle.log2_map(d, M) for d in range(-(M - 1), M)]
        assert all(b > a for a, b in zip(vals, vals[1:]))
        for d in range(M):
            assert oracle.log2_map(-d, M) == -oracle.log2_map(d, M)


def test_code_window_of_one_has_coordinate_zero():
    assert oracle.log2_map(0, 1) == 0.0
    rng = np.random.default_rng(5)
    w1, b1, w2, b2 = rng.normal(size=(6, 2)), rng.normal(size=6), rng.normal(size=(2, 6)), rng.normal(size=2)
    t = oracle.cpb_table_code(1, 2, w1, b1, w2, b2)
    z = w2 @ np.maximum(b1, 0.0) + b2
    np.testing.assert_allclose(t[0], 16.0 / (1.0 + np.exp(-z)), rtol=1e-14)


def test_code_table_bounded_and_half_scale_for_zero_output_layer():
    rng = np.random.default_rng(6)
    w1, b1 = rng.normal(size=(16, 2)), rng.normal(size=16)
    t = oracle.cpb_table_code(8, 3, w1, b1, np.zeros((3, 16)), np.zeros(3))
    assert np.all(t == 8.0)  # 16 sigmoid(0)
    # outputs near +-8: strictly inside (0, 16) (far larger |G| rounds to the ends in double)
    t = oracle.cpb_table_code(8, 2, w1, b1, 0.01 * rng.normal(size=(2, 16)), np.array([8.0, -8.0]))
    assert np.all((t > 0.0) & (t < 16.0))
    assert np.all(t[:, 0] > 15.9) and np.all(t[:, 1] < 0.1)


def test_code_table_is_sigmoid_of_g_on_code_coordinates():
    """One hidden unit reading dx only, identity output layer: the table is
    16 sigmoid(relu(dx_hat)) row by row, with dx_hat the code coordinate."""
    M = 6
    t = oracle.cpb_table_code(M, 1, np.array([[1.0, 0.0]]), None, np.array([[1.0]]), None)
    R = 2 * M - 1
    for dy in range(-(M - 1), M):
        for dx in range(-(M - 1), M):
            x = max(oracle.log2_map(dx, M), 0.0)
            assert t[(dy + M - 1) * R + dx + M - 1, 0] == pytest.approx(16.0 / (1.0 + math.exp(-x)), rel=1e-14)


def test_code_table_transfer_to_a_larger_window_extends_the_pretrained_table():
    """With the pretrained window Mp as normaliser, a table for a larger
    test-time window agrees with the Mp table on every offset both have, and
    pretrained_M = M is the same as giving none."""
    rng = np.random.default_rng(7)
    w1, b1, w2, b2 = rng.normal(size=(32, 2)), rng.normal(size=32), rng.normal(size=(2, 32)), rng.normal(size=2)
    Mp, M = 8, 12
    small = oracle.cpb_table_code(Mp, 2, w1, b1, w2, b2)
    big = oracle.cpb_table_code(M, 2, w1, b1, w2, b2, pretrained_M=Mp)
    Rs, Rb = 2 * Mp - 1, 2 * M - 1
    for dy in range(-(Mp - 1), Mp):
        for dx in range(-(Mp - 1), Mp):
            np.testing.assert_array_equal(big[(dy + M - 1) * Rb + dx + M - 1], small[(dy + Mp - 1) * Rs + dx + Mp - 1])
    np.testing.assert_array_equal(oracle.cpb_table_code(M, 2, w1, b1, w2, b2, pretrained_M=M),
                                  oracle.cpb_table_code(M, 2, w1, b1, w2, b2))
