"""The entry point for callers that cannot allocate device memory.

swin_window_attn_fwd_noalloc keeps the cosine mode's CPB bias table in a fixed
device array of the library instead of a caller workspace.  Called through the
C ABI (ctypes, no Python wrapper), it must give the regular entry point's
output, within the bf16/fp32 tolerances used everywhere else, on two calls in
a row (the second call reuses the array the first one filled).  This file
sorts last so that a run stopping at its first failure has run everything
else already; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from swin_testutil import TOL_BF16, TOL_F32, rel_err
from vision_transformer_shifted_window_b200 import swin_attn as sa
from vision_transformer_shifted_window_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)])
def test_noalloc_matches_workspace_entry_point(dtype, tol):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = sa.lib()
    outs = []
    for call, seed in enumerate((11, 12)):
        w = syn.Workload(95, "noalloc", "bf16" if dtype == torch.bfloat16 else "f32", 2, 40, 36, 3, 32, 16,
                         (8,), sa.SWIN_MODE_COSINE_CPB, tau=(0.05, 0.2), cpb_hidden=512)
        inp = syn.make_inputs(w, seed=seed)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        q, k, v = (dev(inp[n]).to(dtype) for n in ("q", "k", "v"))
        tau = dev(inp["tau"])
        cpb = tuple(dev(inp[n]) for n in ("w1", "b1", "w2", "b2"))
        ref = sa.swin_window_attn_fwd(q, k, v, 16, 8, sa.SWIN_MODE_COSINE_CPB, tau=tau, cpb=cpb,
                                      out_dtype=torch.float32)
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        g = sa.swin_cpb_weights(512, cpb[0].data_ptr(), cpb[1].data_ptr(), cpb[2].data_ptr(), cpb[3].data_ptr())
        dt = sa.SWIN_BF16 if dtype == torch.bfloat16 else sa.SWIN_F32
        rc = L.swin_window_attn_fwd_noalloc(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dt, sa.SWIN_F32, 2, 40, 36, 3, 32, 16, 8,
            sa.SWIN_MODE_COSINE_CPB, tau.data_ptr(), None, ctypes.byref(g), None,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == sa.SWIN_OK, L.swin_last_error().decode()
        assert sa.swin_stream_status() == sa.SWIN_OK
        err = rel_err(out.cpu().numpy(), ref.cpu().numpy())
        assert err <= tol, (call, err)
        outs.append(out)
    assert not torch.equal(outs[0], outs[1])  # the second call really recomputed


def test_noalloc_rejects_oversized_table():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = sa.lib()
    x = torch.zeros(1, 8, 8, 64, 32, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    w = torch.zeros(16, 2, device="cuda")
    w2 = torch.zeros(64, 16, device="cuda")
    t = torch.ones(64, device="cuda")
    g = sa.swin_cpb_weights(16, w.data_ptr(), None, w2.data_ptr(), None)
    rc = L.swin_window_attn_fwd_noalloc(x.data_ptr(), x.data_ptr(), x.data_ptr(), o.data_ptr(), sa.SWIN_BF16,
                                        sa.SWIN_BF16, 1, 8, 8, 64, 32, 64, 0, sa.SWIN_MODE_COSINE_CPB,
                                        t.data_ptr(), None, ctypes.byref(g), None, None)
    assert rc == sa.SWIN_ERR_UNSUPPORTED
    assert "exceeds" in L.swin_last_error().decode()
