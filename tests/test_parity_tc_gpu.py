"""Tensor-core path (bf16, d = 32) against the oracle on shapes that exercise
its tiling: every rectangle width class (first / middle / last segment), query
tiles of floor(128 / width) rows, partial tiles and partial K/V blocks, odd and
large windows, H != W, grids smaller than a window, and the failure path."""
import numpy as np
import pytest
import torch

from swin_testutil import TOL_BF16, gpu_run_bf16_checked, oracle_run, rel_err
from vision_transformer_shifted_window_b200 import swin_attn as sa
from vision_transformer_shifted_window_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sa.lib()


SHAPES = [  # B, H, W, heads, M, s
    (1, 16, 16, 1, 8, 4), (2, 20, 13, 2, 7, 3), (1, 40, 36, 3, 16, 8), (1, 33, 70, 2, 24, 12),
    (1, 64, 64, 1, 32, 16), (1, 50, 45, 2, 32, 5), (1, 9, 9, 1, 64, 0), (1, 70, 66, 1, 64, 33),
    (1, 5, 130, 1, 3, 1), (3, 6, 7, 2, 1, 0), (1, 24, 24, 4, 12, 6), (2, 17, 23, 1, 11, 10),
]


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,H,W,heads,M,s", SHAPES)
def test_tc_shapes(B, H, W, heads, M, s, mode):
    w = syn.Workload(80, "tc", "bf16", B, H, W, heads, 32, M, (s,), mode, tau=(0.05, 0.2),
                     cpb_hidden=64 if mode == 1 else 0, rope_base=100.0)
    inp = syn.make_inputs(w, seed=7 * H + W + 100 * mode + M)
    if mode == 0:
        inp["table"] = (0.5 * np.random.default_rng(3).standard_normal(((2 * M - 1) ** 2, heads))).astype(np.float32)
    got = gpu_run_bf16_checked(inp, w, s).cpu().numpy()
    want = oracle_run(inp, w, s)
    err = rel_err(got, want)
    assert err <= TOL_BF16, err


def test_tc_large_logits_rescale():
    """Scores that grow along the key order force the online rescale."""
    w = syn.Workload(81, "tc", "bf16", 1, 32, 32, 1, 32, 32, (0,), 0)
    inp = syn.make_inputs(w, seed=5)
    ramp = np.linspace(0.0, 3.0, 32 * 32, dtype=np.float32).reshape(1, 32, 32, 1, 1)
    inp["k"] = syn.round_to_bf16(inp["k"] * (1.0 + ramp))
    inp["q"] = syn.round_to_bf16(inp["q"] * 3.0)
    inp["table"] = np.zeros((63 * 63, 1), dtype=np.float32)
    got = gpu_run_bf16_checked(inp, w, 0).cpu().numpy()
    want = oracle_run(inp, w, 0)
    assert rel_err(got, want) <= TOL_BF16


def test_tc_forced_timeout_reports_status_and_recovers():
    w = syn.Workload(82, "tc", "bf16", 1, 32, 32, 2, 32, 16, (8,), 2, rope_base=100.0)
    inp = syn.make_inputs(w, seed=9)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q, k, v = (dev(inp[n]).to(torch.bfloat16) for n in ("q", "k", "v"))
    rope = dev(inp["rope_freqs"])
    sa.swin_debug_set(1, 2_000_000)  # ~1 ms waits
    try:
        sa.swin_window_attn_fwd(q, k, v, 16, 8, 2, rope_freqs=rope)
        assert sa.swin_stream_status() == sa.SWIN_ERR_TIMEOUT
    finally:
        sa.swin_debug_set(0, 0)
    out = sa.swin_window_attn_fwd(q, k, v, 16, 8, 2, rope_freqs=rope, out_dtype=torch.float32)
    assert sa.swin_stream_status() == sa.SWIN_OK
    want = oracle_run(inp, w, 8)
    assert rel_err(out.cpu().numpy(), want) <= TOL_BF16


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("B,H,W,heads,M,s", [(3, 32, 32, 12, 8, 4), (2, 35, 30, 9, 7, 3), (1, 48, 40, 6, 24, 12)])
def test_tc_bias_head_changes(B, H, W, heads, M, s, mode):
    """More work items than SMs and many heads: every CTA walks several items
    and reloads its warpgroups' bias-table slots when the head changes; even
    rectangle widths take the paired-load path, odd ones the general path."""
    w = syn.Workload(83, "tc", "bf16", B, H, W, heads, 32, M, (s,), mode, tau=(0.05, 0.2),
                     cpb_hidden=64 if mode == 1 else 0)
    inp = syn.make_inputs(w, seed=11 * heads + M + mode)
    if mode == 0:
        inp["table"] = (0.5 * np.random.default_rng(4).standard_normal(((2 * M - 1) ** 2, heads))).astype(np.float32)
    got = gpu_run_bf16_checked(inp, w, s).cpu().numpy()
    want = oracle_run(inp, w, s)
    assert rel_err(got, want) <= TOL_BF16


def test_tc_v_out_of_fp16_range_reports_unsupported():
    """V is carried in fp16 on the tensor-core path: an entry at or beyond
    65504 saturates and the call reports SWIN_ERR_UNSUPPORTED (no fault); the
    next call with in-range inputs is clean."""
    w = syn.Workload(84, "tc", "bf16", 1, 16, 16, 1, 32, 8, (4,), 0)
    inp = syn.make_inputs(w, seed=3)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q, k, v = (dev(inp[n]).to(torch.bfloat16) for n in ("q", "k", "v"))
    v_big = v.clone()
    v_big[0, 5, 7, 0, 3] = 70000.0
    sa.swin_window_attn_fwd(q, k, v_big, 8, 4, 0)
    assert sa.swin_stream_status() == sa.SWIN_ERR_UNSUPPORTED
    sa.swin_window_attn_fwd(q, k, v, 8, 4, 0)
    assert sa.swin_stream_status() == sa.SWIN_OK


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("B,H,W,heads,M,s", [(2, 40, 36, 3, 16, 8), (1, 50, 45, 2, 32, 5), (3, 24, 24, 4, 12, 6)])
def test_tc_no_bias_table_position_major(B, H, W, heads, M, s, mode):
    """Without a bias table the kernel walks its work items position-major
    (all heads and images of one item position, then the next): dot-product
    and cosine scores with no relative bias, ragged and multi-head shapes."""
    w = syn.Workload(86, "tc", "bf16", B, H, W, heads, 32, M, (s,), mode, tau=(0.05, 0.2))
    inp = syn.make_inputs(w, seed=13 * H + W + mode)
    inp.pop("table", None)
    for key in ("w1", "b1", "w2", "b2"):
        inp.pop(key, None)
    got = gpu_run_bf16_checked(inp, w, s).cpu().numpy()
    want = oracle_run(inp, w, s)
    assert rel_err(got, want) <= TOL_BF16
