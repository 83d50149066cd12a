"""Full-size parity: every query of every window of every image.

Each bf16 workload runs at its full size, with the inputs and the call that
bench.py times, through the C ABI.  The kernel's fp32 result (fp32 output) is
compared element by element with the double-precision oracle over the whole
output, image by image: max |gpu - oracle| / rms(oracle) <= 2e-2, with the max
and the rms taken over all images.  The bf16 output is then checked to be that
fp32 result rounded to nearest even, bit for bit.  The oracle runs on the
host's cores (OpenMP); the largest workload (2 x 384 x 384 tokens, 16 heads,
576 keys per query) takes tens of seconds there.
"""
import numpy as np
import pytest
import torch

from swin_testutil import TOL_BF16, gpu_run_bf16_checked, oracle_run
from vision_transformer_shifted_window_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_bf16_workload_full_size_every_window(idx):
    w = syn.WORKLOADS[idx]
    s = w.shifts[0]
    inp = syn.make_inputs(w)
    got = gpu_run_bf16_checked(inp, w, s).cpu().numpy()
    torch.cuda.empty_cache()
    max_err, sum_sq, n, worst = 0.0, 0.0, 0, None
    for b in range(w.B):
        want = oracle_run(inp, w, s, b_slice=slice(b, b + 1))[0]
        diff = np.abs(got[b].astype(np.float64) - want)
        e = float(diff.max())
        if e > max_err:
            max_err = e
            worst = (b,) + tuple(int(i) for i in np.unravel_index(int(diff.argmax()), diff.shape))
        sum_sq += float(np.sum(want * want))
        n += want.size
        del want, diff
    rel = max_err / np.sqrt(sum_sq / n)
    assert rel <= TOL_BF16, (w.name, rel, "worst (b, y, x, head, channel)", worst)
