"""Pins of the oracle's backward pass (gradients of L = sum(dout * out)).

The backward is the chain rule through the forward definition ("Swin
Transformer V2" eq. 1 / eq. 2, FlashSwin's window-local RoPE), with the softmax
recomputed.  It is pinned to things other than itself:
  * central finite differences of the (separately pinned) forward oracle;
  * float64 autograd through an independent torch route (cyclic roll, window
    partition, region mask, scaled_dot_product_attention) written here;
  * exact identities: per window sum_j dv_j = sum_i dout_i (softmax rows sum to
    one); the logit gradients of each query sum to zero, so the table gradient
    sums to zero over its entries.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

SHAPES = [(1, 6, 5, 2, 8, 4, 2), (2, 7, 7, 1, 8, 3, 1), (1, 5, 9, 2, 4, 4, 0), (1, 8, 6, 1, 8, 8, 5)]


def rand_inputs(B, H, W, nh, d, M, seed):
    rng = np.random.default_rng(seed)
    q, k, v, do = (rng.standard_normal((B, H, W, nh, d)) for _ in range(4))
    R = 2 * M - 1
    table = 0.5 * rng.standard_normal((R * R, nh))
    tau = rng.uniform(0.05, 0.5, nh)
    freqs = rng.uniform(0.1, 1.5, (2, d // 4))
    return q, k, v, do, table, tau, freqs


def loss(q, k, v, do, M, s, mode, tau, table, freqs):
    out = oracle.window_attn(q, k, v, M, s, mode, tau=tau, table=table if mode != 2 else None, rope_freqs=freqs)
    return float(np.sum(out * do))


def grads(q, k, v, do, M, s, mode, tau, table, freqs):
    return oracle.window_attn_bwd(q, k, v, do, M, s, mode, tau=tau if mode == 1 else None,
                                  table=table if mode != 2 else None, rope_freqs=freqs if mode == 2 else None)


@pytest.mark.parametrize("B,H,W,nh,d,M,s", SHAPES)
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_backward_matches_finite_differences(B, H, W, nh, d, M, s, mode):
    q, k, v, do, table, tau, freqs = rand_inputs(B, H, W, nh, d, M, 31 * H + W + mode)
    if mode == 1:
        tau[0] = 0.004  # clamped to 0.01: no gradient reaches it
    g = grads(q, k, v, do, M, s, mode, tau, table, freqs)
    args = {"q": q, "k": k, "v": v, "table": table, "tau": tau, "freqs": freqs}
    names = ["q", "k", "v"] + {0: ["table"], 1: ["table", "tau"], 2: ["freqs"]}[mode]
    gkey = {"q": "dq", "k": "dk", "v": "dv", "table": "dtable", "tau": "dtau", "freqs": "drope"}
    rng = np.random.default_rng(7)
    h = 1e-6
    for name in names:
        x = args[name]
        flat = x.reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 24), replace=False)
        for i in idx:
            old = flat[i]
            flat[i] = old + h
            lp = loss(args["q"], args["k"], args["v"], do, M, s, mode, args["tau"], args["table"], args["freqs"])
            flat[i] = old - h
            lm = loss(args["q"], args["k"], args["v"], do, M, s, mode, args["tau"], args["table"], args["freqs"])
            flat[i] = old
            fd = (lp - lm) / (2 * h)
            an = g[gkey[name]].reshape(-1)[i]
            assert abs(fd - an) <= 2e-7 * max(1.0, abs(an)), (name, int(i), fd, an)
    if mode == 1:
        assert g["dtau"][0] == 0.0


def roll_route_t(q, k, v, M, s, mode, tau=None, table=None, freqs=None):
    """The forward as Swin computes it, on padded rolled windows, in torch
    float64 so that autograd gives every gradient."""
    B, H, W, nh, d = q.shape
    Hp, Wp = -(-H // M) * M, -(-W // M) * M
    pad = lambda t: F.pad(t, (0, 0, 0, 0, 0, Wp - W, 0, Hp - H))
    real = torch.zeros(Hp, Wp, dtype=torch.bool)
    real[:H, :W] = True
    roll = lambda t, dims: torch.roll(t, shifts=(-s, -s), dims=dims)
    q, k, v = (roll(pad(t), (1, 2)) for t in (q, k, v))
    real = roll(real, (0, 1))
    band = torch.zeros(Hp, Wp, dtype=torch.long)
    if s:
        cnt = 0
        for hs in (slice(0, Hp - M), slice(Hp - M, Hp - s), slice(Hp - s, None)):
            for ws in (slice(0, Wp - M), slice(Wp - M, Wp - s), slice(Wp - s, None)):
                band[hs, ws] = cnt
                cnt += 1
    nWy, nWx, N = Hp // M, Wp // M, M * M

    def part(t):
        b0 = t.shape[0]
        t = t.reshape(b0, nWy, M, nWx, M, *t.shape[3:]).transpose(2, 3)
        return t.reshape(b0, nWy * nWx, N, *t.shape[5:])

    qh, kh, vh = (part(t).permute(0, 1, 3, 2, 4) for t in (q, k, v))  # [B, nW, nh, N, d]
    bw = part(band[None, ..., None])[0, ..., 0]
    rw = part(real[None, ..., None])[0, ..., 0]
    mask = (bw[:, :, None] == bw[:, None, :]) & rw[:, None, :]
    i = torch.arange(N)
    yi, xi = i // M, i % M
    rel = (yi[:, None] - yi[None, :] + M - 1) * (2 * M - 1) + (xi[:, None] - xi[None, :] + M - 1)
    add = torch.zeros(nh, N, N, dtype=torch.float64)
    if table is not None:
        add = table[rel].permute(2, 0, 1)
    neg = torch.full((), -math.inf, dtype=torch.float64)
    amask = torch.where(mask[None, :, None], add[None, None], neg)
    if mode == 0:
        o = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=amask, scale=1 / math.sqrt(d))
    elif mode == 1:
        t = torch.clamp(tau, min=0.01)
        qn = F.normalize(qh, dim=-1) / t[None, None, :, None, None]
        o = F.scaled_dot_product_attention(qn, F.normalize(kh, dim=-1), vh, attn_mask=amask, scale=1.0)
    else:
        def rot(x, py, px):
            hd = d // 2
            parts = []
            for half, p in ((0, py), (1, px)):
                seg = x[..., half * hd:(half + 1) * hd]
                z = torch.complex(seg[..., 0::2], seg[..., 1::2])
                ang = p[:, None].to(torch.float64) * freqs[half][None, :]
                z = z * torch.polar(torch.ones_like(ang), ang)
                parts.append(torch.stack([z.real, z.imag], dim=-1).reshape(*seg.shape))
            return torch.cat(parts, dim=-1)
        py, px = yi % M, xi % M
        o = F.scaled_dot_product_attention(rot(qh, py, px), rot(kh, py, px), vh, attn_mask=amask,
                                           scale=1 / math.sqrt(d))
    o = o.permute(0, 1, 3, 2, 4).reshape(B, nWy, nWx, M, M, nh, d).transpose(2, 3).reshape(B, Hp, Wp, nh, d)
    o = torch.roll(o, shifts=(s, s), dims=(1, 2))
    return o[:, :H, :W]


@pytest.mark.parametrize("B,H,W,nh,d,M,s", SHAPES + [(1, 12, 10, 2, 8, 4, 3), (2, 9, 9, 3, 4, 3, 2)])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_backward_matches_autograd_of_the_roll_route(B, H, W, nh, d, M, s, mode):
    q, k, v, do, table, tau, freqs = rand_inputs(B, H, W, nh, d, M, 17 * H + 3 * W + mode)
    g = grads(q, k, v, do, M, s, mode, tau, table, freqs)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    tt = torch.tensor(table, requires_grad=True)
    ttau = torch.tensor(tau, requires_grad=True)
    tf = torch.tensor(freqs, requires_grad=True)
    out = roll_route_t(tq, tk, tv, M, s, mode, tau=ttau if mode == 1 else None, table=tt if mode != 2 else None,
                       freqs=tf if mode == 2 else None)
    (out * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(g["dq"], tq.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(g["dk"], tk.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(g["dv"], tv.grad.numpy(), rtol=0, atol=1e-10)
    if mode != 2:
        np.testing.assert_allclose(g["dtable"], tt.grad.numpy(), rtol=0, atol=1e-10)
    if mode == 1:
        np.testing.assert_allclose(g["dtau"], ttau.grad.numpy(), rtol=1e-10, atol=1e-10)
    if mode == 2:
        np.testing.assert_allclose(g["drope"], tf.grad.numpy(), rtol=1e-10, atol=1e-9)


def _segments(L, M, s):
    starts = list(range(0, L, M)) if s == 0 else [0] + list(range(s, L, M))
    return list(zip(starts, starts[1:] + [L]))


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_backward_identities(mode):
    B, H, W, nh, d, M, s = 2, 11, 9, 2, 8, 4, 2
    q, k, v, do, table, tau, freqs = rand_inputs(B, H, W, nh, d, M, 5 + mode)
    g = grads(q, k, v, do, M, s, mode, tau, table, freqs)
    # softmax rows sum to one: per window the value gradients add up to the output gradients
    for y0, y1 in _segments(H, M, s):
        for x0, x1 in _segments(W, M, s):
            np.testing.assert_allclose(g["dv"][:, y0:y1, x0:x1].sum(axis=(1, 2)),
                                       do[:, y0:y1, x0:x1].sum(axis=(1, 2)), rtol=0, atol=1e-11)
    if mode != 2:
        # adding one constant to every logit changes nothing: the bias gradient sums to zero per head
        np.testing.assert_allclose(g["dtable"].sum(axis=0), 0.0, atol=1e-11)
    # a zero output gradient gives zero gradients everywhere
    z = grads(q, k, v, np.zeros_like(do), M, s, mode, tau, table, freqs)
    for key, val in z.items():
        assert np.all(val == 0.0), key
