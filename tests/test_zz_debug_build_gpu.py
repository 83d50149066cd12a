"""The range-checking build (SWIN_DEBUG; build.py --debug): its kernels check
TMA coordinates, bias-slot reads of unmasked keys, output stores and global
row offsets, and record a failed check in the device status word instead of
faulting.  Here the tensor-core, CUDA-core, backward and interleaved parity
tests run again with that library loaded (SWIN_ATTN_DEBUG=1) in a child
process; every one of them asserts swin_stream_status() == 0 after its calls,
so a single failed check fails the run."""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from vision_transformer_shifted_window_b200 import build as swin_build
    swin_build.build(debug=True)


def _child(args, timeout=1500):
    env = dict(os.environ, SWIN_ATTN_DEBUG="1")
    return subprocess.run([sys.executable] + args, env=env, cwd=ROOT, capture_output=True, text=True,
                          timeout=timeout)


def test_child_loads_the_debug_library():
    r = _child(["-c", "from vision_transformer_shifted_window_b200 import swin_attn as sa; "
                      "sa.lib(); print(sa.LIB_PATH)"])
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().endswith("libswinattn_debug.so")


def test_parity_suites_pass_with_range_checks():
    r = _child(["-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
                "tests/test_parity_tc_gpu.py", "tests/test_parity_gpu.py",
                "tests/test_parity_bwd_gpu.py::test_fp32_shapes_and_modes",
                "tests/test_parity_bwd_gpu.py::test_bf16_workloads_reduced",
                "tests/test_parity_iwin_gpu.py::test_interleaved_forward_and_backward"])
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
