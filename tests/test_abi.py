"""Host-side checks of the C ABI (no GPU needed): the library builds, loads,
exports every function include/swin_attn.h declares, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest
import torch

from vision_transformer_shifted_window_b200 import build as swin_build
from vision_transformer_shifted_window_b200 import swin_attn as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    swin_build.build()
    return sa.lib()


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            src = open(os.path.join(inc, fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(swin_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert names, "no declarations found"
    assert names == set(sa.EXPORTED)
    for n in names:
        assert hasattr(L, n), n
    assert L.swin_version() >= 100


def test_workspace_size_rules(L):
    assert sa.swin_window_attn_workspace_size(16, 3, sa.SWIN_MODE_COSINE_CPB, False) == 31 * 31 * 3 * 4 + 244
    assert sa.swin_window_attn_workspace_size(16, 3, sa.SWIN_MODE_COSINE_CPB, True) == 0
    assert sa.swin_window_attn_workspace_size(16, 3, sa.SWIN_MODE_ROPE, False) == 0
    assert sa.swin_window_attn_workspace_size(16, 3, sa.SWIN_MODE_DOT_BIAS, False) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def call_fwd(L, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, out=FAKE * 64, dt=sa.SWIN_BF16, B=1, H=8, W=8, heads=1,
             d=32, M=4, shift=2, mode=sa.SWIN_MODE_DOT_BIAS, tau=None, table=None, cpb=None,
             rope=None, ws=None, wsb=0)
    a.update(kw)
    return L.swin_window_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["dt"], a.get("odt", a["dt"]), a["B"], a["H"], a["W"],
                                  a["heads"], a["d"], a["M"], a["shift"], a["mode"], a["tau"],
                                  a["table"], a["cpb"], a["rope"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,why", [
    (dict(q=None), "NULL"), (dict(shift=4), "shift"), (dict(shift=-1), "shift"), (dict(M=0), "M"),
    (dict(M=65, shift=0), "M"), (dict(B=0), ">= 1"), (dict(H=0), ">= 1"), (dict(W=0), ">= 1"),
    (dict(heads=0), ">= 1"), (dict(d=0), ">= 1"), (dict(q=FAKE + 8), "aligned"),
    (dict(out=FAKE * 2), "overlaps"), (dict(mode=1), "tau"), (dict(mode=2), "rope"),
    (dict(mode=2, rope=FAKE * 5, d=30), "d % 4"), (dict(mode=2, rope=FAKE * 5, table=FAKE * 6), "no bias"),
    (dict(mode=7), "mode"), (dict(dt=5), "dtype"), (dict(dt=0, odt=1), "output dtype"),
])
def test_rejects_bad_arguments(L, kw, why):
    rc = call_fwd(L, **kw)
    assert rc == sa.SWIN_ERR_INVALID_ARG
    assert why in L.swin_last_error().decode()


def test_cpb_form_arguments_rejected_before_launch(L):
    w = sa.swin_cpb_weights(8, FAKE, None, FAKE, None)
    assert L.swin_cpb_eval_form(8, 3, ctypes.byref(w), 2, 0, FAKE, None) == sa.SWIN_ERR_INVALID_ARG
    assert "form" in L.swin_last_error().decode()
    assert L.swin_cpb_eval_form(8, 3, ctypes.byref(w), sa.SWIN_CPB_PAPER, 8, FAKE, None) == sa.SWIN_ERR_INVALID_ARG
    assert "SWIN_CPB_CODE only" in L.swin_last_error().decode()
    assert L.swin_cpb_eval_form(8, 3, ctypes.byref(w), sa.SWIN_CPB_CODE, 65, FAKE, None) == sa.SWIN_ERR_INVALID_ARG
    assert "pretrained_M" in L.swin_last_error().decode()


def test_cpu_entry_points_reject_before_launch(L):
    assert L.swin_index_tables(8, 8, 4, 4, None, None, None, None, None) == sa.SWIN_ERR_INVALID_ARG
    assert L.swin_cpb_eval(0, 3, None, FAKE, None) == sa.SWIN_ERR_INVALID_ARG
    w = sa.swin_cpb_weights(0, FAKE, None, FAKE, None)
    assert L.swin_cpb_eval(8, 3, ctypes.byref(w), FAKE, None) == sa.SWIN_ERR_INVALID_ARG
    assert "hidden" in L.swin_last_error().decode()


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 4, 1, 32)
    with pytest.raises(ValueError):
        sa.swin_window_attn_fwd(x, x, x, 4, 0, 0)


def _z(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


@pytest.mark.parametrize("kw,why", [
    (dict(mode=1, tau=_z(3)), "tau"),
    (dict(bias_table=_z(48, 2)), "bias_table"),
    (dict(mode=2, rope_freqs=_z(2, 4)), "rope_freqs"),
    (dict(mode=1, tau=_z(2), cpb=(_z(16, 2), None, _z(3, 16), None)), "cpb w2"),
    (dict(mode=1, tau=_z(2), cpb=(_z(16, 2), _z(8), _z(2, 16), None)), "cpb b1"),
])
def test_binding_checks_parameter_shapes_before_the_call(kw, why):
    """The C ABI sees bare pointers; the binding checks every parameter
    tensor's shape against the sizes the call implies ((2M-1)^2 x heads
    table, [heads] tau, [2, d/4] RoPE frequencies, G's weights)."""
    q = _z(1, 8, 8, 2, 32)
    args = dict(q=q, k=q, v=q, M=4, shift=2, mode=0)
    args.update(kw)
    with pytest.raises(ValueError, match=why):
        sa.swin_window_attn_fwd(**args)


def test_binding_checks_cpb_weight_shapes():
    w1, w2 = _z(16, 2), _z(4, 16)
    with pytest.raises(ValueError, match="cpb w2"):
        sa.swin_cpb_eval(8, 3, w1, None, w2, None)
    with pytest.raises(ValueError, match="cpb b2"):
        sa.swin_cpb_eval_form(8, 4, w1, None, w2, _z(3), sa.SWIN_CPB_CODE)


def test_bwd_workspace_size(L):
    acc = ((31 * 31 * 3 + 3 + 2 * 8) * 8 + 255) // 256 * 256
    stats = (8 * 2 * 2 * 64 * 64 * 3 + 255) // 256 * 256  # (lse, D) doubles per row and head, B = 2
    assert sa.swin_window_attn_bwd_workspace_size(2, 64, 64, 3, 32, 16) == acc + stats
    assert sa.swin_window_attn_bwd_workspace_size(0, 64, 64, 3, 32, 16) == 0
    assert sa.swin_window_attn_bwd_workspace_size(1, 8, 8, 1, 32, 65) == 0


def call_bwd(L, **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, dout=FAKE * 4, dq=FAKE * 64, dk=FAKE * 65, dv=FAKE * 66,
             dt=sa.SWIN_F32, gdt=None, B=1, H=8, W=8, heads=1, d=32, M=4, shift=2, part=0,
             mode=sa.SWIN_MODE_DOT_BIAS,
             tau=None, table=None, rope=None, dtable=None, dtau=None, drope=None, ws=FAKE * 128, wsb=1 << 20)
    a.update(kw)
    return L.swin_window_attn_bwd(a["q"], a["k"], a["v"], a["dout"], a["dq"], a["dk"], a["dv"], a["dt"],
                                  a["dt"] if a["gdt"] is None else a["gdt"], a["B"], a["H"], a["W"], a["heads"],
                                  a["d"], a["M"], a["shift"], a["part"], a["mode"], a["tau"], a["table"], a["rope"],
                                  a["dtable"], a["dtau"], a["drope"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status,why", [
    (dict(q=None), 1, "NULL"), (dict(dout=None), 1, "NULL"), (dict(dv=None), 1, "NULL"),
    (dict(shift=4), 1, "shift"), (dict(M=65, shift=0), 1, "M"), (dict(heads=0), 1, ">= 1"),
    (dict(dout=FAKE * 4 + 8), 1, "aligned"), (dict(dk=FAKE * 3), 1, "overlap"),
    (dict(dk=FAKE * 64 + 16), 1, "overlap"), (dict(dq=FAKE), 1, "overlaps"),
    (dict(mode=1), 1, "tau"), (dict(mode=2), 1, "rope"), (dict(dtable=FAKE * 7), 1, "dtable needs"),
    (dict(dtau=FAKE * 7), 1, "dtau"), (dict(drope=FAKE * 7), 1, "drope"),
    (dict(dt=0, gdt=1), 1, "output dtype"), (dict(d=24), 2, "d in"), (dict(ws=None), 1, "workspace"),
    (dict(wsb=256), 1, "workspace"), (dict(ws=FAKE * 128 + 16), 1, "256-byte"),
    (dict(part=2), 1, "partition"), (dict(part=1), 1, "no shift"),
])
def test_bwd_rejects_bad_arguments(L, kw, status, why):
    assert call_bwd(L, **kw) == status
    assert why in L.swin_last_error().decode()


def test_fwd_ex_rejects_bad_partitions(L):
    def call(part, shift):
        return L.swin_window_attn_fwd_ex(FAKE, FAKE * 2, FAKE * 3, FAKE * 64, sa.SWIN_BF16, sa.SWIN_BF16, 1, 8, 8, 1,
                                         32, 4, shift, part, sa.SWIN_MODE_DOT_BIAS, None, None, None, None, None, 0,
                                         None)
    assert call(2, 0) == sa.SWIN_ERR_INVALID_ARG and "partition" in L.swin_last_error().decode()
    assert call(1, 2) == sa.SWIN_ERR_INVALID_ARG and "no shift" in L.swin_last_error().decode()
    assert call(-1, 0) == sa.SWIN_ERR_INVALID_ARG
