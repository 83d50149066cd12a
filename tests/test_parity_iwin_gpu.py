"""GPU parity of attention in interleaved windows ("Iwin Transformer",
abstract: interleaved window attention; the strided index map is the reading
that the oracle states and pins): the forward through swin_window_attn_fwd_ex
and the gradients through swin_window_attn_bwd, both with
SWIN_PARTITION_INTERLEAVED, against the oracle with the same partition, within
max|gpu - oracle| / rms(oracle) <= 1e-5 (fp32) and 2e-2 (bf16, fp32 output;
the bf16 output is its round-to-nearest-even rounding bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
from swin_testutil import TOL_BF16, TOL_F32, rel_err
from vision_transformer_shifted_window_b200 import swin_attn as sa
from vision_transformer_shifted_window_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
IL = sa.SWIN_PARTITION_INTERLEAVED


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sa.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def params(inp):
    kw = {}
    if "tau" in inp:
        kw["tau"] = dev(inp["tau"])
    if "table" in inp:
        kw["bias_table"] = dev(inp["table"])
    if "rope_freqs" in inp:
        kw["rope_freqs"] = dev(inp["rope_freqs"])
    return kw


def oracle_kw(inp):
    return dict(tau=inp.get("tau"), table=inp.get("table"), rope_freqs=inp.get("rope_freqs"), partition=IL)


def case(dtype, heads, d, M, mode, bias=True):
    return syn.Workload(5, "iwin-case", dtype, 1, 8, 8, heads, d, M, (0,), mode,
                        tau=(0.05, 0.2) if mode == 1 else None, rope_base=100.0 if mode == 2 else 0.0,
                        partition=IL, bias=bias)


def run_case(w, B=None, H=None, W=None, seed=None, backward=True):
    inp = syn.make_inputs(w, B=B, H=H, W=W, seed=seed)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    tol = TOL_F32 if w.dtype == "f32" else TOL_BF16
    q, k, v = (dev(inp[n]).to(dt) for n in ("q", "k", "v"))
    kw = params(inp)
    o32 = sa.swin_window_attn_fwd(q, k, v, w.M, 0, w.mode, out_dtype=torch.float32, partition=IL, **kw)
    if dt == torch.bfloat16:
        o16 = sa.swin_window_attn_fwd(q, k, v, w.M, 0, w.mode, partition=IL, **kw)
        assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o16.view(torch.int16))
    assert sa.swin_stream_status() == 0
    want = oracle.window_attn(inp["q"], inp["k"], inp["v"], w.M, 0, w.mode, **oracle_kw(inp))
    err = rel_err(o32.cpu().numpy(), want)
    assert err <= tol, err
    if not backward:
        return err
    dout = syn.make_dout(w, B=B, H=H, W=W, seed=None if seed is None else seed + 1)
    g = sa.swin_window_attn_bwd(q, k, v, dev(dout).to(dt), w.M, 0, w.mode, grad_dtype=torch.float32,
                                partition=IL, **kw)
    assert sa.swin_stream_status() == 0
    gw = oracle.window_attn_bwd(inp["q"], inp["k"], inp["v"], dout, w.M, 0, w.mode, **oracle_kw(inp))
    errs = {n: rel_err(g[n].cpu().numpy(), gw[n]) for n in gw if np.any(gw[n])}
    assert all(e <= tol for e in errs.values()), errs
    return err, errs


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,W,heads,d,M", [(1, 16, 16, 2, 32, 8), (2, 13, 10, 2, 16, 4), (1, 21, 17, 1, 8, 7),
                                             (1, 40, 36, 2, 32, 16)])
def test_interleaved_forward_and_backward(mode, dtype, B, H, W, heads, d, M):
    run_case(case(dtype, heads, d, M, mode), B=B, H=H, W=W, seed=11 * H + W + mode)


def test_interleaved_position_free():
    """Iwin's attention has no position embedding: mode 0 with no bias table."""
    run_case(case("bf16", 3, 32, 7, 0, bias=False), B=2, H=56, W=56, seed=5)


def test_interleaved_differs_from_shifted():
    """The partition argument reaches the kernel: on a grid of several windows
    the two partitions give different outputs."""
    w = case("f32", 1, 16, 4, 0)
    inp = syn.make_inputs(w, H=8, W=8, seed=9)
    q, k, v = (dev(inp[n]) for n in ("q", "k", "v"))
    a = sa.swin_window_attn_fwd(q, k, v, 4, 0, 0, bias_table=dev(inp["table"]), partition=IL)
    b = sa.swin_window_attn_fwd(q, k, v, 4, 0, 0, bias_table=dev(inp["table"]))
    assert not torch.allclose(a, b)


def test_iwin_workload_full_size():
    """The Iwin-T stage-1 workload (B=32, 56x56, M=7, no bias), every window,
    forward and backward."""
    w = syn.WORKLOADS[5]
    run_case(w)
