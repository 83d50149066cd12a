"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, on the
same seeded inputs.  Integer tables must match bit for bit; outputs must agree
within max|gpu - oracle| / rms(oracle) <= 1e-5 (fp32) and 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import oracle
from swin_testutil import (TOL_BF16, TOL_F32, boundary_queries, gpu_run, gpu_run_bf16_checked, oracle_run,
                           oracle_table, rel_err)
from vision_transformer_shifted_window_b200 import swin_attn as sa
from vision_transformer_shifted_window_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sa.lib()


# ---------------------------------------------------------------------------
# integer tables, bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("H,W,M,s", [(16, 16, 8, 0), (16, 16, 8, 4), (56, 56, 7, 3), (64, 64, 16, 8),
                                     (112, 112, 32, 16), (384, 384, 24, 12), (10, 13, 4, 3), (5, 7, 8, 7),
                                     (1, 1, 1, 0), (9, 20, 64, 63)])
def test_index_tables_bit_exact(H, W, M, s):
    got = [t.cpu().numpy() for t in sa.swin_index_tables(H, W, M, s)]
    want = oracle.index_tables(H, W, M, s)
    for g, w in zip(got, want):
        assert g.dtype == np.int32 and np.array_equal(g, w)


# ---------------------------------------------------------------------------
# CPB meta network
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,heads,hidden", [(8, 2, 512), (16, 3, 512), (24, 16, 512), (7, 5, 33), (1, 1, 1)])
def test_cpb_eval(M, heads, hidden):
    rng = np.random.default_rng(M * 100 + heads)
    w1 = rng.standard_normal((hidden, 2)).astype(np.float32)
    b1 = rng.standard_normal(hidden).astype(np.float32)
    w2 = (0.05 * rng.standard_normal((heads, hidden))).astype(np.float32)
    b2 = rng.standard_normal(heads).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    got = sa.swin_cpb_eval(M, heads, dev(w1), dev(b1), dev(w2), dev(b2)).cpu().numpy()
    want = oracle.cpb_table(M, heads, w1, b1, w2, b2)
    assert rel_err(got, want) <= TOL_F32


@pytest.mark.parametrize("M,pretrained_M,heads,hidden", [(8, 0, 2, 512), (16, 0, 3, 512), (24, 16, 16, 512),
                                                       (12, 8, 4, 64), (1, 0, 1, 1), (5, 1, 2, 7)])
def test_cpb_eval_code_form(M, pretrained_M, heads, hidden):
    """The released code's form of G (normalised log2 coordinates, 16 sigmoid
    output), also at a test-time window larger than the pretrained one."""
    rng = np.random.default_rng(M * 100 + heads + 7)
    w1 = rng.standard_normal((hidden, 2)).astype(np.float32)
    b1 = rng.standard_normal(hidden).astype(np.float32)
    w2 = (0.05 * rng.standard_normal((heads, hidden))).astype(np.float32)
    b2 = rng.standard_normal(heads).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    got = sa.swin_cpb_eval_form(M, heads, dev(w1), dev(b1), dev(w2), dev(b2), sa.SWIN_CPB_CODE,
                                pretrained_M).cpu().numpy()
    want = oracle.cpb_table_code(M, heads, w1, b1, w2, b2, pretrained_M=pretrained_M)
    assert rel_err(got, want) <= TOL_F32
    assert np.all((got > 0.0) & (got < 16.0))


def test_cpb_eval_form_paper_equals_cpb_eval():
    rng = np.random.default_rng(3)
    w1, b1 = rng.standard_normal((64, 2)).astype(np.float32), rng.standard_normal(64).astype(np.float32)
    w2, b2 = rng.standard_normal((3, 64)).astype(np.float32), rng.standard_normal(3).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    a = sa.swin_cpb_eval(9, 3, dev(w1), dev(b1), dev(w2), dev(b2))
    b = sa.swin_cpb_eval_form(9, 3, dev(w1), dev(b1), dev(w2), dev(b2), sa.SWIN_CPB_PAPER)
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# fp32 workload (16x16, M=8, cosine + CPB), both shifts, full output
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shift", [0, 4])
def test_tiny_fp32_workload(shift):
    w = syn.WORKLOADS[0]
    inp = syn.make_inputs(w)
    got = gpu_run(inp, w, shift).cpu().numpy()
    want = oracle_run(inp, w, shift)
    assert rel_err(got, want) <= TOL_F32


# ---------------------------------------------------------------------------
# fp32, random shapes: odd M, ragged grids, H != W, every shift of one M
# ---------------------------------------------------------------------------
SHAPES = [(2, 13, 9, 2, 16, 5, 2), (1, 23, 17, 3, 8, 7, 3), (2, 10, 12, 1, 32, 4, 1), (1, 9, 9, 2, 64, 9, 4),
          (1, 33, 20, 2, 32, 16, 8), (1, 40, 35, 1, 32, 32, 16), (3, 6, 6, 2, 8, 8, 3), (1, 1, 1, 1, 8, 1, 0),
          (1, 4, 70, 1, 16, 3, 2)]


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,H,W,heads,d,M,s", SHAPES)
def test_fp32_random_shapes(B, H, W, heads, d, M, s, mode):
    w = syn.Workload(90, "t", "f32", B, H, W, heads, d, M, (s,), mode, tau=(0.05, 0.5),
                     cpb_hidden=32 if mode == 1 else 0, rope_base=100.0)
    inp = syn.make_inputs(w, seed=B * 1000 + H * 10 + W + mode)
    if mode == 0:
        inp["table"] = (0.5 * np.random.default_rng(1).standard_normal(((2 * M - 1) ** 2, heads))).astype(np.float32)
    got = gpu_run(inp, w, s).cpu().numpy()
    want = oracle_run(inp, w, s)
    assert rel_err(got, want) <= TOL_F32


@pytest.mark.parametrize("s", range(6))
def test_fp32_every_shift(s):
    w = syn.Workload(91, "t", "f32", 1, 15, 14, 2, 16, 6, (s,), 1, tau=(0.05, 0.2), cpb_hidden=64)
    inp = syn.make_inputs(w, seed=500 + s)
    got = gpu_run(inp, w, s).cpu().numpy()
    want = oracle_run(inp, w, s)
    assert rel_err(got, want) <= TOL_F32


def test_window_of_one_token_returns_v():
    w = syn.Workload(92, "t", "f32", 2, 5, 6, 2, 8, 1, (0,), 0)
    inp = syn.make_inputs(w, seed=3)
    got = gpu_run(inp, w, 0).cpu().numpy()
    assert np.array_equal(got, inp["v"])


# ---------------------------------------------------------------------------
# bf16 workloads: reduced batch (full output), then full size (sampled queries)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_bf16_workload_reduced_batch(idx):
    w = syn.WORKLOADS[idx]
    H = W = min(w.H, 96) if idx == 4 else w.H
    inp = syn.make_inputs(w, B=1, H=H, W=W)
    got = gpu_run_bf16_checked(inp, w, w.shifts[0]).cpu().numpy()
    want = oracle_run(inp, w, w.shifts[0])
    assert rel_err(got, want) <= TOL_BF16


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_bf16_workload_full_size_sampled(idx):
    w = syn.WORKLOADS[idx]
    s = w.shifts[0]
    inp = syn.make_inputs(w)
    got = gpu_run_bf16_checked(inp, w, s).cpu().numpy()
    for b in sorted({0, w.B - 1}):
        ids = boundary_queries(w.H, w.W, w.M, s, 64, seed=idx * 10 + b)
        want = oracle_run(inp, w, s, queries=ids, b_slice=slice(b, b + 1))
        g = got[b].reshape(w.H * w.W, w.heads, w.d)[ids]
        assert rel_err(g, want) <= TOL_BF16, (b, rel_err(g, want))
