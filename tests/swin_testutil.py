"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them with the stated tolerances."""
import numpy as np
import torch

import oracle
from vision_transformer_shifted_window_b200 import swin_attn as sa
from vision_transformer_shifted_window_b200 import synthetic as syn

# Tolerances: max |gpu - oracle| / rms(oracle).  For bf16 inputs the bound is
# checked on the kernel's fp32 result (fp32 output); the bf16 output is then
# required to be exactly that result rounded to nearest even, so its distance
# to the oracle is at most the bound plus half a bf16 ulp per element.
TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def gpu_run_bf16_checked(inp, w: syn.Workload, shift: int) -> torch.Tensor:
    """Run a bf16 workload twice (fp32 and bf16 output) and check that the bf16
    output is the RNE rounding of the fp32 one, bit for bit.  Returns fp32."""
    o32 = gpu_run(inp, w, shift, out_dtype=torch.float32)
    o16 = gpu_run(inp, w, shift)
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o16.view(torch.int16))
    return o32


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.sqrt(np.mean(ref * ref)))


def torch_dtype(w: syn.Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def gpu_run(inp, w: syn.Workload, shift: int, dtype=None, out=None, out_dtype=None) -> torch.Tensor:
    dtype = dtype or torch_dtype(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q, k, v = (dev(inp[n]).to(dtype) for n in ("q", "k", "v"))
    kw = {}
    if "tau" in inp:
        kw["tau"] = dev(inp["tau"])
    if "table" in inp:
        kw["bias_table"] = dev(inp["table"])
    if "w1" in inp:
        kw["cpb"] = tuple(dev(inp[n]) for n in ("w1", "b1", "w2", "b2"))
    if "rope_freqs" in inp:
        kw["rope_freqs"] = dev(inp["rope_freqs"])
    o = sa.swin_window_attn_fwd(q, k, v, w.M, shift, w.mode, out=out, out_dtype=out_dtype, **kw)
    assert sa.swin_stream_status() == 0
    return o


def oracle_table(inp, w: syn.Workload):
    if "table" in inp:
        return inp["table"]
    if "w1" in inp:
        return oracle.cpb_table(w.M, w.heads, inp["w1"], inp["b1"], inp["w2"], inp["b2"])
    return None


def oracle_run(inp, w: syn.Workload, shift: int, queries=None, b_slice=None):
    q, k, v = inp["q"], inp["k"], inp["v"]
    if b_slice is not None:
        q, k, v = q[b_slice], k[b_slice], v[b_slice]
    return oracle.window_attn(q, k, v, w.M, shift, w.mode, tau=inp.get("tau"),
                              table=oracle_table(inp, w), rope_freqs=inp.get("rope_freqs"),
                              queries=queries)


def boundary_queries(H: int, W: int, M: int, s: int, n_random: int, seed: int):
    """Token ids of one image covering first/last segments, segment edges and
    corners on both axes, plus random ones."""
    def coords(L):
        c = {0, L - 1, L // 2}
        for base in ([s] if s else []) + list(range(s, L, M)):
            for dlt in (-1, 0, 1, M - 1):
                if 0 <= base + dlt < L:
                    c.add(base + dlt)
        return sorted(c)
    ys, xs = coords(H), coords(W)
    rng = np.random.default_rng(seed)
    pick_y = rng.choice(ys, size=min(len(ys), 24), replace=False)
    pick_x = rng.choice(xs, size=min(len(xs), 24), replace=False)
    ids = {int(y) * W + int(x) for y in pick_y for x in pick_x}
    ids |= set(int(t) for t in rng.integers(0, H * W, n_random))
    return np.array(sorted(ids), dtype=np.int64)
