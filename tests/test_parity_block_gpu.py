"""GPU parity of the steps either side of the attention in a Swin V2 block
("Swin Transformer V2", Method item 1 "Residual post-norm", §3.2, fig. 1,
swin_v2_block pseudocode): swin_qkv_proj, swin_proj_postnorm_residual and the
composed swin_attn_block_fwd against oracle.block in float64, within
max|gpu - oracle| / rms(oracle) <= 1e-5 (fp32) and 2e-2 (bf16).  As for the
attention, a bf16 call's bound is checked on its fp32 output and the bf16
output must be that result rounded to nearest even, bit for bit (half a bf16
ulp of the largest outputs alone is ~1.5 % of their RMS).  The bf16 block
stores q, k, v and the attention output in bf16 between its steps; its oracle
takes the same roundings (float64 -> fp32 -> bf16, round to nearest even), so
the bound covers the arithmetic.  The storage itself costs up to ~2.5 % of
the RMS in the cosine mode, where 1/tau (up to 20) scales the rounding of q
and k: the comparison with the exact float64 block is bounded at 5e-2."""
import numpy as np
import pytest
import torch

import oracle
from oracle import block
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


def bf16_storage(t):
    """A float64 array as the bf16 tensor a bf16 step stores (via fp32, RNE)."""
    return torch.from_numpy(np.asarray(t, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def case(dtype, heads, d, M=8, mode=0, partition=0):
    return syn.Workload(0, "block-case", dtype, 1, 8, 8, heads, d, M, (0,), mode,
                        tau=(0.05, 0.2) if mode == 1 else None, rope_base=100.0 if mode == 2 else 0.0,
                        partition=partition)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("heads,d,B,H,W", [(3, 32, 2, 7, 9), (4, 32, 1, 16, 16), (16, 32, 1, 5, 13), (2, 8, 3, 3, 3)])
def test_qkv_proj(dtype, heads, d, B, H, W):
    w = case(dtype, heads, d)
    p = syn.make_block_inputs(w, B=B, H=H, W=W, seed=heads * 100 + H)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    x, wq = dev(p["x"]).to(tdt), dev(p["w_qkv"]).to(tdt)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    for bias in (dev(p["b_qkv"]), None):
        got = sa.swin_qkv_proj(x, wq, bias, out_dtype=torch.float32)
        want = block.qkv_proj(p["x"], p["w_qkv"], None if bias is None else p["b_qkv"])
        for g, ref in zip(got, want):
            assert g.shape == x.shape
            assert rel_err(g.cpu().numpy(), ref) <= tol
        if dtype == "bf16":
            for g16, g32 in zip(sa.swin_qkv_proj(x, wq, bias), got):
                assert g16.dtype == torch.bfloat16
                assert torch.equal(g32.to(torch.bfloat16).view(torch.int16), g16.view(torch.int16))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("C,tokens", [(96, 1000), (128, 37), (512, 300), (1024, 17), (8, 5)])
def test_proj_postnorm_residual(dtype, C, tokens):
    w = case(dtype, C // 8 if C >= 8 else 1, 8)
    p = syn.make_block_inputs(w, B=1, H=1, W=tokens, seed=C + tokens)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    a = syn.make_block_inputs(w, B=1, H=1, W=tokens, seed=C + tokens + 1)["x"]
    args = (dev(a).to(tdt), dev(p["w_o"]).to(tdt), dev(p["b_o"]), dev(p["x"]).to(tdt), dev(p["gamma"]),
            dev(p["beta"]))
    got = sa.swin_proj_postnorm_residual(*args, eps=1e-5, out_dtype=torch.float32)
    want = block.proj_postnorm_residual(a, p["w_o"], p["b_o"], p["x"], p["gamma"], p["beta"], 1e-5)
    err = rel_err(got.cpu().numpy(), want)
    assert err <= (TOL_F32 if dtype == "f32" else TOL_BF16), err
    if dtype == "bf16":
        g16 = sa.swin_proj_postnorm_residual(*args, eps=1e-5)
        assert torch.equal(got.to(torch.bfloat16).view(torch.int16), g16.view(torch.int16))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode,partition,M,s", [(0, 0, 7, 3), (1, 0, 8, 4), (2, 0, 8, 4), (0, 1, 7, 0)])
def test_attn_block(dtype, mode, partition, M, s):
    w = case(dtype, 3, 32, M=M, mode=mode, partition=partition)
    B, H, W = 2, 21, 19
    p = syn.make_block_inputs(w, B=B, H=H, W=W, seed=31 + mode)
    att = syn.make_inputs(w, B=1, H=1, W=1, seed=41 + mode)  # only the attention parameters are used
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    kw = {}
    if "tau" in att:
        kw["tau"] = dev(att["tau"])
    if "table" in att:
        kw["bias_table"] = dev(att["table"])
    if "rope_freqs" in att:
        kw["rope_freqs"] = dev(att["rope_freqs"])
    args = (dev(p["x"]).to(tdt), 3, dev(p["w_qkv"]).to(tdt), dev(p["b_qkv"]), dev(p["w_o"]).to(tdt), dev(p["b_o"]),
            dev(p["gamma"]), dev(p["beta"]), M, s, mode)
    got = sa.swin_attn_block_fwd(*args, partition=partition, out_dtype=torch.float32, **kw)
    assert sa.swin_stream_status() == 0
    if dtype == "bf16":
        g16 = sa.swin_attn_block_fwd(*args, partition=partition, **kw)
        assert torch.equal(got.to(torch.bfloat16).view(torch.int16), g16.view(torch.int16))
    ref = lambda rnd: block.attn_block(p["x"], 3, p["w_qkv"], p["b_qkv"], p["w_o"], p["b_o"], p["gamma"], p["beta"],
                                       M, s, mode, tau=att.get("tau"), table=att.get("table"),
                                       rope_freqs=att.get("rope_freqs"), partition=partition, round_to=rnd)
    exact = ref(None)
    if dtype == "f32":
        err = rel_err(got.cpu().numpy(), exact)
        print(dtype, mode, partition, err)
        assert err <= TOL_F32, err
    else:
        stored = ref(bf16_storage)
        err = rel_err(got.cpu().numpy(), stored)
        err_exact = rel_err(got.cpu().numpy(), exact)
        print(dtype, mode, partition, err, err_exact)
        assert err <= TOL_BF16, err
        assert err_exact <= 5e-2, err_exact


def test_block_rejects_before_launch():
    x = torch.zeros(1, 8, 8, 96, device="cuda", dtype=torch.bfloat16)
    w3 = torch.zeros(288, 96, device="cuda", dtype=torch.bfloat16)
    w1 = torch.zeros(96, 96, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(sa.SwinError, match="shift"):
        sa.swin_attn_block_fwd(x, 3, w3, None, w1, None, None, None, 4, 4, 0)
    with pytest.raises(sa.SwinError, match="no shift"):
        sa.swin_attn_block_fwd(x, 3, w3, None, w1, None, None, None, 4, 2, 0, partition=1)


@pytest.mark.parametrize("C", [32, 64, 96, 128])
@pytest.mark.parametrize("tokens", [1, 127, 128, 129, 300, 2000])
def test_fused_block_kernels_tiles_and_optional_parameters(C, tokens):
    """The fused tensor-core block kernels (bf16, C a multiple of 32): partial
    and single tiles, several tiles per CTA, every supported C, with and
    without bias, gamma and beta; fp32 output against the oracle and the bf16
    output its RNE, bit for bit."""
    w = case("bf16", C // 32, 32)
    p = syn.make_block_inputs(w, B=1, H=1, W=tokens, seed=7 * C + tokens)
    a = syn.make_block_inputs(w, B=1, H=1, W=tokens, seed=7 * C + tokens + 1)["x"]
    x = dev(p["x"]).to(torch.bfloat16)
    wq, wo = dev(p["w_qkv"]).to(torch.bfloat16), dev(p["w_o"]).to(torch.bfloat16)
    for with_params in (True, False):
        bq = dev(p["b_qkv"]) if with_params else None
        got = sa.swin_qkv_proj(x, wq, bq, out_dtype=torch.float32)
        want = block.qkv_proj(p["x"], p["w_qkv"], p["b_qkv"] if with_params else None)
        for g, ref in zip(got, want):
            assert rel_err(g.cpu().numpy(), ref) <= TOL_BF16
        for g16, g32 in zip(sa.swin_qkv_proj(x, wq, bq), got):
            assert torch.equal(g32.to(torch.bfloat16).view(torch.int16), g16.view(torch.int16))
        bo, gam, bet = ((dev(p["b_o"]), dev(p["gamma"]), dev(p["beta"])) if with_params else (None, None, None))
        args = (dev(a).to(torch.bfloat16), wo, bo, x, gam, bet)
        got = sa.swin_proj_postnorm_residual(*args, eps=1e-5, out_dtype=torch.float32)
        want = block.proj_postnorm_residual(a, p["w_o"], p["b_o"] if with_params else None, p["x"],
                                            p["gamma"] if with_params else None, p["beta"] if with_params else None,
                                            1e-5)
        assert rel_err(got.cpu().numpy(), want) <= TOL_BF16
        g16 = sa.swin_proj_postnorm_residual(*args, eps=1e-5)
        assert torch.equal(got.to(torch.bfloat16).view(torch.int16), g16.view(torch.int16))
    assert sa.swin_stream_status() == sa.SWIN_OK
