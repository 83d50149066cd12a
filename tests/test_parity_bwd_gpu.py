"""GPU parity of the backward pass (swin_window_attn_bwd through the C ABI)
against the oracle's gradients, on the same seeded inputs: dq, dk, dv and the
parameter gradients (bias table, tau, RoPE frequencies) within
max|gpu - oracle| / rms(oracle) <= 1e-5 (fp32 tensors) and 2e-2 (bf16
tensors, checked on fp32 gradients; the bf16 gradients must then be their
round-to-nearest-even rounding bit for bit).  The parameter gradients are
summed by double atomic additions and rounded once: between calls they may
differ in the last fp32 bit, never more."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from swin_testutil import TOL_BF16, TOL_F32, rel_err
from vision_transformer_shifted_window_b200 import swin_attn as sa
from vision_transformer_shifted_window_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sa.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def tables(inp, w):
    """(GPU table from the library's own CPB kernel, oracle table) or the drawn table."""
    if "table" in inp:
        return dev(inp["table"]), inp["table"]
    if "w1" in inp:
        gpu = sa.swin_cpb_eval(w.M, w.heads, *(dev(inp[n]) for n in ("w1", "b1", "w2", "b2")))
        return gpu, oracle.cpb_table(w.M, w.heads, inp["w1"], inp["b1"], inp["w2"], inp["b2"])
    return None, None


def run_gpu(inp, dout, w, shift, table, grad_dtype=None):
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q, k, v, g = (dev(a).to(dt) for a in (inp["q"], inp["k"], inp["v"], dout))
    out = sa.swin_window_attn_bwd(q, k, v, g, w.M, shift, w.mode, tau=dev(inp["tau"]) if "tau" in inp else None,
                                  bias_table=table,
                                  rope_freqs=dev(inp["rope_freqs"]) if "rope_freqs" in inp else None,
                                  grad_dtype=grad_dtype)
    assert sa.swin_stream_status() == 0
    return out


def run_oracle(inp, dout, w, shift, table):
    return oracle.window_attn_bwd(inp["q"], inp["k"], inp["v"], dout, w.M, shift, w.mode, tau=inp.get("tau"),
                                  table=table, rope_freqs=inp.get("rope_freqs"))


def compare(got, want, tol, names=None):
    names = names or sorted(want)
    errs = {}
    for n in names:
        assert n in got, n
        g = got[n].float().cpu().numpy()
        if not np.any(want[n]):  # e.g. d(tau) of heads all clamped: exactly zero
            assert not np.any(g), n
            errs[n] = 0.0
            continue
        errs[n] = rel_err(g, want[n])
    assert all(e <= tol for e in errs.values()), errs
    return errs


def check_case(w, shift, B=None, H=None, W=None, seed=None, mutate=None):
    inp = syn.make_inputs(w, B=B, H=H, W=W, seed=seed)
    dout = syn.make_dout(w, B=B, H=H, W=W, seed=None if seed is None else seed + 1)
    if mutate:
        mutate(inp)
    tg, to = tables(inp, w)
    want = run_oracle(inp, dout, w, shift, to)
    if w.dtype == "f32":
        got = run_gpu(inp, dout, w, shift, tg)
        return compare(got, want, TOL_F32), got, want
    g32 = run_gpu(inp, dout, w, shift, tg, grad_dtype=torch.float32)
    g16 = run_gpu(inp, dout, w, shift, tg)
    for n in ("dq", "dk", "dv"):
        assert g16[n].dtype == torch.bfloat16
        assert torch.equal(g32[n].to(torch.bfloat16).view(torch.int16), g16[n].view(torch.int16)), n
    for n in ("dtable", "dtau", "drope"):
        if n in g32:
            # double atomic sums rounded once to fp32: the order of the
            # additions varies between calls, so the last fp32 bit may too
            a, b = g32[n].cpu().numpy(), g16[n].cpu().numpy()
            ulp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float32))
            assert np.all(np.abs(a - b) <= ulp + 1e-9 * np.abs(a).max()), n
    return compare(g32, want, TOL_BF16), g32, want


W0 = syn.WORKLOADS[0]


def case(dtype, heads, d, M, mode, tau=None, rope=0.0, index=0):
    """A workload-shaped case (the drawing recipe of the synthetic module)."""
    return syn.Workload(index, "case", dtype, 1, 8, 8, heads, d, M, (0,), mode, tau=tau,
                        cpb_hidden=0, rope_base=rope)


# ---------------------------------------------------------------------------
# fp32 (double arithmetic inside): 1e-5
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shift", [0, 4])
def test_tiny_fp32_workload_all_gradients(shift):
    """The tiny SwinV2 fp32 workload (16x16, M=8, cosine + CPB table, tau 0.1)."""
    errs, got, _ = check_case(W0, shift)
    assert set(got) == {"dq", "dk", "dv", "dtable", "dtau"}


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,H,W,heads,d,M,s", [
    (1, 16, 16, 2, 32, 8, 4), (2, 13, 10, 2, 16, 5, 2), (1, 20, 20, 1, 8, 7, 3), (1, 9, 11, 2, 64, 4, 1),
    (1, 40, 36, 1, 32, 16, 8),
])
def test_fp32_shapes_and_modes(mode, B, H, W, heads, d, M, s):
    w = case("f32", heads, d, M, mode, tau=(0.05, 0.2) if mode == 1 else None, rope=100.0 if mode == 2 else 0.0)
    check_case(w, s, B=B, H=H, W=W, seed=7 * H + W + mode)


def test_fp32_large_window_m64():
    """M = 64: 4096-token windows (32 CTAs of queries per rectangle) and a
    127 x 127 bias-table gradient held in shared memory."""
    w = case("f32", 1, 8, 64, 0)
    check_case(w, 32, B=1, H=70, W=66, seed=64)


def test_fp32_window_of_one_token():
    """M = 1: every token attends to itself only, so P = 1, dl = 0: dq = dk = 0
    and dv = dout exactly."""
    w = case("f32", 2, 16, 1, 0)
    inp = syn.make_inputs(w, H=5, W=6, seed=3)
    dout = syn.make_dout(w, H=5, W=6, seed=4)
    got = run_gpu(inp, dout, w, 0, dev(inp["table"]))
    assert torch.count_nonzero(got["dq"]) == 0 and torch.count_nonzero(got["dk"]) == 0
    assert torch.equal(got["dv"].cpu(), torch.from_numpy(dout))
    assert torch.count_nonzero(got["dtable"]) == 0


def test_fp32_tau_clamp_and_zero_rows():
    """Cosine mode: a head with tau below 0.01 gets d(tau) = 0 exactly; zero q
    and k rows (norms held at 1e-12) still match the oracle."""
    w = case("f32", 3, 32, 8, 1, tau=(0.05, 0.2))

    def mutate(inp):
        inp["tau"][1] = 0.004
        inp["tau"][2] = 0.0125
        inp["q"][0, 3, 5, 0, :] = 0.0
        inp["k"][0, 6, 2, 2, :] = 0.0

    errs, got, want = check_case(w, 4, H=16, W=16, seed=11, mutate=mutate)
    assert float(got["dtau"][1]) == 0.0 and want["dtau"][1] == 0.0
    assert float(got["dtau"][2]) != 0.0


def test_fp32_sharp_softmax():
    """tau at its 0.01 floor: logits up to 100, the sharpest softmax the mode
    allows.  The fp32 tau nearest 0.01 lies below 0.01, so it is clamped and
    its gradient is exactly zero."""
    w = case("f32", 2, 32, 8, 1, tau=(0.01, 0.01))
    errs, got, want = check_case(w, 4, H=16, W=16, seed=12)
    assert not np.any(want["dtau"]) and torch.count_nonzero(got["dtau"]) == 0


# ---------------------------------------------------------------------------
# bf16 (fp32 arithmetic inside): 2e-2, reduced and full-size workloads
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("idx,B,H,W", [(1, 2, 56, 56), (2, 2, 64, 64), (3, 1, 112, 112), (4, 1, 96, 96)])
def test_bf16_workloads_reduced(idx, B, H, W):
    check_case(syn.WORKLOADS[idx], syn.WORKLOADS[idx].shifts[0], B=B, H=H, W=W)


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("d", [8, 16, 64])
def test_bf16_other_head_widths(mode, d):
    w = case("bf16", 2, d, 6, mode, tau=(0.05, 0.2) if mode == 1 else None, rope=100.0 if mode == 2 else 0.0)
    check_case(w, 3, B=1, H=15, W=17, seed=d + mode)


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_bf16_workload_full_size_every_window(idx):
    """Every gradient element of the full-size workload against the oracle."""
    w = syn.WORKLOADS[idx]
    errs, _, _ = check_case(w, w.shifts[0])
    print(w.name, errs)


# ---------------------------------------------------------------------------
# the tensor-core backward (bf16, d = 32, M <= 32): tiling shapes
# ---------------------------------------------------------------------------
TC_SHAPES = [  # B, H, W, heads, M, s
    (1, 16, 16, 1, 8, 4), (2, 20, 13, 2, 7, 3), (1, 40, 36, 3, 16, 8), (1, 33, 70, 2, 24, 12),
    (1, 64, 64, 1, 32, 16), (1, 50, 45, 2, 32, 5), (1, 5, 130, 1, 3, 1), (3, 6, 7, 2, 1, 0),
    (1, 24, 24, 4, 12, 6), (2, 17, 23, 1, 11, 10),
]


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,H,W,heads,M,s", TC_SHAPES)
def test_bf16_tensor_core_backward_shapes(B, H, W, heads, M, s, mode):
    """Every rectangle width class, partial query tiles (128 tokens) and key
    blocks (64), odd and large windows, H != W, M = 1; tables with large
    entries so the bias gradient matters."""
    w = syn.Workload(90, "bwd-tc", "bf16", B, H, W, heads, 32, M, (s,), mode,
                     tau=(0.05, 0.2) if mode == 1 else None, rope_base=100.0 if mode == 2 else 0.0)

    def mutate(inp):
        if "table" in inp:
            inp["table"] = (0.5 * np.random.default_rng(M).standard_normal(inp["table"].shape)).astype(np.float32)

    check_case(w, s, seed=7 * H + W + 100 * mode + M, mutate=mutate)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_bf16_tensor_core_backward_interleaved(mode):
    w = syn.Workload(91, "bwd-tc-il", "bf16", 2, 30, 27, 2, 32, 8, (0,), mode,
                     tau=(0.05, 0.2) if mode == 1 else None, rope_base=100.0 if mode == 2 else 0.0, partition=1)
    inp = syn.make_inputs(w, seed=5 + mode)
    dout = syn.make_dout(w, seed=6 + mode)
    kw = dict(tau=dev(inp["tau"]) if "tau" in inp else None,
              bias_table=dev(inp["table"]) if "table" in inp else None,
              rope_freqs=dev(inp["rope_freqs"]) if "rope_freqs" in inp else None)
    q, k, v, g = (dev(a).to(torch.bfloat16) for a in (inp["q"], inp["k"], inp["v"], dout))
    got = sa.swin_window_attn_bwd(q, k, v, g, w.M, 0, mode, grad_dtype=torch.float32, partition=1, **kw)
    assert sa.swin_stream_status() == 0
    want = oracle.window_attn_bwd(inp["q"], inp["k"], inp["v"], dout, w.M, 0, mode, tau=inp.get("tau"),
                                  table=inp.get("table"), rope_freqs=inp.get("rope_freqs"), partition=1)
    compare(got, want, TOL_BF16)
