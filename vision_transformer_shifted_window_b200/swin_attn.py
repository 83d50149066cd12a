"""Python binding of libswinattn.so (include/swin_attn.h), argument marshalling only.

Every function keeps its C name.  Tensors are torch CUDA tensors used as plain
device buffers; the computation happens in the library's kernels on the
current torch stream (or the stream passed in).  There is no fallback: if the
shared library is missing or a call fails, a RuntimeError is raised.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
#: SWIN_ATTN_DEBUG=1 selects the range-checking build (build.py --debug)
DEBUG_BUILD = os.environ.get("SWIN_ATTN_DEBUG", "0") == "1"
LIB_PATH = os.path.join(_PKG, "libswinattn_debug.so" if DEBUG_BUILD else "libswinattn.so")

SWIN_OK = 0
SWIN_ERR_INVALID_ARG = 1
SWIN_ERR_UNSUPPORTED = 2
SWIN_ERR_CUDA = 3
SWIN_ERR_TIMEOUT = 4

SWIN_MODE_DOT_BIAS = 0
SWIN_MODE_COSINE_CPB = 1
SWIN_MODE_ROPE = 2

SWIN_F32 = 0
SWIN_BF16 = 1
SWIN_CPB_PAPER = 0
SWIN_CPB_CODE = 1

SWIN_PARTITION_SHIFTED = 0
SWIN_PARTITION_INTERLEAVED = 1

#: every symbol include/swin_attn.h declares
EXPORTED = ("swin_cpb_eval", "swin_cpb_eval_form", "swin_window_attn_fwd", "swin_window_attn_fwd_ex",
            "swin_window_attn_fwd_noalloc",
            "swin_window_attn_workspace_size", "swin_window_attn_bwd", "swin_window_attn_bwd_workspace_size",
            "swin_qkv_proj", "swin_proj_postnorm_residual", "swin_attn_block_fwd", "swin_attn_block_workspace_size",
            "swin_qkv_proj_workspace_size", "swin_proj_postnorm_workspace_size",
            "swin_index_tables", "swin_stream_status", "swin_last_error", "swin_version",
            "swin_debug_set")


class SwinError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("swin status %d: %s" % (status, msg))
        self.status = status


class swin_cpb_weights(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


_lib = None


def lib():
    """Load the shared library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("%s is not built; run `python -m vision_transformer_shifted_window_b200.build%s`"
                               % (os.path.basename(LIB_PATH), " --debug" if DEBUG_BUILD else ""))
        L = ctypes.CDLL(LIB_PATH)
        vp, i, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
        L.swin_cpb_eval.argtypes = [i, i, ctypes.POINTER(swin_cpb_weights), vp, st]
        L.swin_cpb_eval.restype = i
        L.swin_cpb_eval_form.argtypes = [i, i, ctypes.POINTER(swin_cpb_weights), i, i, vp, st]
        L.swin_cpb_eval_form.restype = i
        L.swin_window_attn_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp, vp,
                                           ctypes.POINTER(swin_cpb_weights), vp, vp,
                                           ctypes.c_size_t, st]
        L.swin_window_attn_fwd.restype = i
        L.swin_window_attn_fwd_ex.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, i, vp, vp,
                                              ctypes.POINTER(swin_cpb_weights), vp, vp, ctypes.c_size_t, st]
        L.swin_window_attn_fwd_ex.restype = i
        L.swin_window_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp,
                                                   vp, ctypes.POINTER(swin_cpb_weights), vp, st]
        L.swin_window_attn_fwd_noalloc.restype = i
        L.swin_window_attn_workspace_size.argtypes = [i, i, i, i]
        L.swin_window_attn_workspace_size.restype = ctypes.c_size_t
        L.swin_window_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, i, vp, vp,
                                           vp, vp, vp, vp, vp, ctypes.c_size_t, st]
        L.swin_window_attn_bwd.restype = i
        L.swin_window_attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
        L.swin_window_attn_bwd_workspace_size.restype = ctypes.c_size_t
        L.swin_qkv_proj.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, vp, ctypes.c_size_t, st]
        L.swin_qkv_proj.restype = i
        L.swin_qkv_proj_workspace_size.argtypes = [i, i]
        L.swin_qkv_proj_workspace_size.restype = ctypes.c_size_t
        L.swin_proj_postnorm_residual.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, i, i, i, i, vp,
                                                  ctypes.c_size_t, st]
        L.swin_proj_postnorm_residual.restype = i
        L.swin_proj_postnorm_workspace_size.argtypes = [i, i]
        L.swin_proj_postnorm_workspace_size.restype = ctypes.c_size_t
        L.swin_attn_block_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, i, i, i, i, i, i, i, i,
                                          i, i, i, vp, vp, ctypes.POINTER(swin_cpb_weights), vp, vp,
                                          ctypes.c_size_t, st]
        L.swin_attn_block_fwd.restype = i
        L.swin_attn_block_workspace_size.argtypes = [i, i, i, i, i, i, i, i, i]
        L.swin_attn_block_workspace_size.restype = ctypes.c_size_t
        L.swin_index_tables.argtypes = [i, i, i, i, vp, vp, vp, vp, st]
        L.swin_index_tables.restype = i
        L.swin_stream_status.argtypes = [st]
        L.swin_stream_status.restype = i
        L.swin_last_error.argtypes = []
        L.swin_last_error.restype = ctypes.c_char_p
        L.swin_debug_set.argtypes = [i, ctypes.c_longlong]
        L.swin_debug_set.restype = i
        L.swin_version.argtypes = []
        L.swin_version.restype = i
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != SWIN_OK:
        raise SwinError(rc, lib().swin_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _on(stream):
    """Allocate temporaries and copies on the stream the kernels run on, so the
    caching allocator never hands their memory to other work while those
    kernels may still read it."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _f32(t: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if t is None:
        return None
    if t.dtype != torch.float32:
        raise ValueError("parameter tensors must be float32")
    return t.contiguous()


def _shape(name: str, t: Optional[torch.Tensor], shape: Tuple[int, ...]) -> None:
    """The C ABI takes bare pointers; sizes it cannot see are checked here."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _cpb_struct(cpb: Optional[Tuple[torch.Tensor, ...]], heads: int):
    if cpb is None:
        return None, ()
    w1, b1, w2, b2 = (_f32(t) for t in cpb)
    if w1 is None or w2 is None or w1.dim() != 2:
        raise ValueError("cpb needs w1 [hidden, 2] and w2 [heads, hidden]")
    hidden = int(w1.shape[0])
    _shape("cpb w1", w1, (hidden, 2))
    _shape("cpb b1", b1, (hidden,))
    _shape("cpb w2", w2, (heads, hidden))
    _shape("cpb b2", b2, (heads,))
    s = swin_cpb_weights(hidden, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2))
    return s, (w1, b1, w2, b2)


def _param_shapes(M: int, heads: int, d: int, tau, bias_table, rope_freqs) -> None:
    _shape("tau", tau, (heads,))
    _shape("bias_table", bias_table, ((2 * M - 1) ** 2, heads))
    _shape("rope_freqs", rope_freqs, (2, d // 4))


def swin_debug_set(flags: int, wait_limit_cycles: int = 0) -> None:
    """Failure-path test hook (see include/swin_attn.h)."""
    _check(lib().swin_debug_set(int(flags), int(wait_limit_cycles)))


def swin_version() -> int:
    return int(lib().swin_version())


def swin_last_error() -> str:
    return lib().swin_last_error().decode()


def swin_window_attn_workspace_size(M: int, heads: int, mode: int, have_table: bool) -> int:
    return int(lib().swin_window_attn_workspace_size(M, heads, mode, int(bool(have_table))))


def swin_cpb_eval(M: int, heads: int, w1, b1, w2, b2, out: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """Evaluate the Log-CPB MLP for every offset -> fp32 [(2M-1)^2, heads]."""
    R = 2 * M - 1
    with _on(stream):
        if out is None:
            out = torch.empty((R * R, heads), dtype=torch.float32, device=w1.device)
        s, keep = _cpb_struct((w1, b1, w2, b2), heads)
        _check(lib().swin_cpb_eval(M, heads, ctypes.byref(s), _ptr(out), _stream(stream)))
        del keep
    return out


def swin_cpb_eval_form(M: int, heads: int, w1, b1, w2, b2, form: int, pretrained_M: int = 0,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """swin_cpb_eval with a choice of form (SWIN_CPB_PAPER or SWIN_CPB_CODE: the
    released code's normalised log2 coordinates and 16 sigmoid bound); pretrained_M
    is the window G was trained at (0: M)."""
    R = 2 * M - 1
    with _on(stream):
        if out is None:
            out = torch.empty((R * R, heads), dtype=torch.float32, device=w1.device)
        s, keep = _cpb_struct((w1, b1, w2, b2), heads)
        _check(lib().swin_cpb_eval_form(M, heads, ctypes.byref(s), int(form), int(pretrained_M), _ptr(out),
                                        _stream(stream)))
        del keep
    return out


def swin_window_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, M: int, shift: int,
                         mode: int, tau: Optional[torch.Tensor] = None,
                         bias_table: Optional[torch.Tensor] = None, cpb=None,
                         rope_freqs: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, stream=None,
                         out_dtype: Optional[torch.dtype] = None,
                         partition: int = SWIN_PARTITION_SHIFTED) -> torch.Tensor:
    """Shifted-window attention forward; q, k, v, out are [B, H, W, heads, d].

    ``out_dtype`` (or the dtype of ``out``) may be float32 for bfloat16 inputs;
    ``partition`` SWIN_PARTITION_INTERLEAVED (with shift 0) selects Iwin's
    interleaved windows (swin_window_attn_fwd_ex)."""
    if q.dtype == torch.float32:
        dt = SWIN_F32
    elif q.dtype == torch.bfloat16:
        dt = SWIN_BF16
    else:
        raise ValueError("q, k, v must be float32 or bfloat16")
    if k.dtype != q.dtype or v.dtype != q.dtype or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share dtype and shape")
    if q.dim() != 5:
        raise ValueError("q, k, v must be [B, H, W, heads, d]")
    B, H, W, heads, d = q.shape
    with _on(stream):
        return _fwd_on_stream(q, k, v, M, shift, mode, dt, B, H, W, heads, d, tau, bias_table, cpb, rope_freqs,
                              out, workspace, stream, out_dtype, partition)


def _fwd_on_stream(q, k, v, M, shift, mode, dt, B, H, W, heads, d, tau, bias_table, cpb, rope_freqs, out,
                   workspace, stream, out_dtype, partition=SWIN_PARTITION_SHIFTED):
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    odt = {torch.float32: SWIN_F32, torch.bfloat16: SWIN_BF16}.get(out.dtype)
    if odt is None:
        raise ValueError("out must be float32 or bfloat16")
    tau, bias_table, rope_freqs = _f32(tau), _f32(bias_table), _f32(rope_freqs)
    _param_shapes(M, heads, d, tau, bias_table, rope_freqs)
    cs, keep = _cpb_struct(cpb, heads)
    need = swin_window_attn_workspace_size(M, heads, mode, bias_table is not None) if cs else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().swin_window_attn_fwd_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), dt, odt, B, H, W, heads, d, M, shift, int(partition), mode,
        _ptr(tau), _ptr(bias_table), ctypes.byref(cs) if cs is not None else None,
        _ptr(rope_freqs), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc)
    del keep
    return out


def swin_window_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, M: int, shift: int,
                                 mode: int, tau: Optional[torch.Tensor] = None,
                                 bias_table: Optional[torch.Tensor] = None, cpb=None,
                                 rope_freqs: Optional[torch.Tensor] = None,
                                 out: Optional[torch.Tensor] = None, stream=None,
                                 out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """Forward pass for callers that cannot allocate device memory: the CPB
    table lives in a fixed device array of the library, not in a workspace.
    ``out`` must be given by such callers (this wrapper allocates it only when
    it is None, as a convenience for Python users)."""
    dt = {torch.float32: SWIN_F32, torch.bfloat16: SWIN_BF16}.get(q.dtype)
    if dt is None or k.dtype != q.dtype or v.dtype != q.dtype or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share a float32/bfloat16 dtype and shape")
    B, H, W, heads, d = q.shape
    with _on(stream):
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
        odt = {torch.float32: SWIN_F32, torch.bfloat16: SWIN_BF16}.get(out.dtype)
        if odt is None or out.shape != q.shape:
            raise ValueError("out must be float32 or bfloat16 with q's shape")
        tau, bias_table, rope_freqs = _f32(tau), _f32(bias_table), _f32(rope_freqs)
        _param_shapes(M, heads, d, tau, bias_table, rope_freqs)
        cs, keep = _cpb_struct(cpb, heads)
        rc = lib().swin_window_attn_fwd_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), dt, odt, B, H, W, heads, d, M, shift, mode,
            _ptr(tau), _ptr(bias_table), ctypes.byref(cs) if cs is not None else None,
            _ptr(rope_freqs), _stream(stream))
        _check(rc)
        del keep
    return out


def swin_window_attn_bwd_workspace_size(B: int, H: int, W: int, heads: int, d: int, M: int) -> int:
    return int(lib().swin_window_attn_bwd_workspace_size(B, H, W, heads, d, M))


def swin_window_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dout: torch.Tensor, M: int,
                         shift: int, mode: int, tau: Optional[torch.Tensor] = None,
                         bias_table: Optional[torch.Tensor] = None,
                         rope_freqs: Optional[torch.Tensor] = None, param_grads: bool = True,
                         grad_dtype: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                         stream=None, partition: int = SWIN_PARTITION_SHIFTED) -> dict:
    """Gradients of sum(dout * swin_window_attn_fwd(...)): a dict with dq, dk, dv
    ([B, H, W, heads, d], dtype ``grad_dtype`` or q's) and, when ``param_grads``,
    dtable (with a bias table), dtau (mode 1) and drope (mode 2), fp32."""
    dt = {torch.float32: SWIN_F32, torch.bfloat16: SWIN_BF16}.get(q.dtype)
    if dt is None or any(t.dtype != q.dtype or t.shape != q.shape for t in (k, v, dout)):
        raise ValueError("q, k, v, dout must share a float32/bfloat16 dtype and shape")
    if q.dim() != 5:
        raise ValueError("q, k, v, dout must be [B, H, W, heads, d]")
    B, H, W, heads, d = q.shape
    gdt = grad_dtype or q.dtype
    gcode = {torch.float32: SWIN_F32, torch.bfloat16: SWIN_BF16}.get(gdt)
    if gcode is None:
        raise ValueError("grad_dtype must be float32 or bfloat16")
    with _on(stream):
        tau, bias_table, rope_freqs = _f32(tau), _f32(bias_table), _f32(rope_freqs)
        _param_shapes(M, heads, d, tau, bias_table, rope_freqs)
        mk = lambda: torch.empty(q.shape, dtype=gdt, device=q.device)
        g = {"dq": mk(), "dk": mk(), "dv": mk()}
        f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=q.device)
        if param_grads and bias_table is not None and mode != SWIN_MODE_ROPE:
            g["dtable"] = f32((2 * M - 1) ** 2, heads)
        if param_grads and mode == SWIN_MODE_COSINE_CPB:
            g["dtau"] = f32(heads)
        if param_grads and mode == SWIN_MODE_ROPE:
            g["drope"] = f32(2, d // 4)
        need = swin_window_attn_bwd_workspace_size(B, H, W, heads, d, M)
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        rc = lib().swin_window_attn_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), dt, gcode,
            B, H, W, heads, d, M, shift, int(partition), mode, _ptr(tau), _ptr(bias_table), _ptr(rope_freqs),
            _ptr(g.get("dtable")), _ptr(g.get("dtau")), _ptr(g.get("drope")), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
        _check(rc)
    return g


def _dtcode(t: torch.Tensor) -> int:
    dt = {torch.float32: SWIN_F32, torch.bfloat16: SWIN_BF16}.get(t.dtype)
    if dt is None:
        raise ValueError("tensors must be float32 or bfloat16")
    return dt


def _scratch(workspace, need, device):
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def swin_qkv_proj(x: torch.Tensor, w_qkv: torch.Tensor, b_qkv: Optional[torch.Tensor] = None,
                  out_dtype: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """q, k, v = x W^T + b split three ways: x [..., C], w_qkv [3C, C] (x's
    dtype), b_qkv fp32 [3C] or None.  Returns three tensors of x's shape
    (dtype ``out_dtype``: x's, or float32 for bfloat16 x)."""
    dt = _dtcode(x)
    C = int(x.shape[-1])
    tokens = x.numel() // C
    _shape("w_qkv", w_qkv, (3 * C, C))
    if w_qkv.dtype != x.dtype:
        raise ValueError("w_qkv must have x's dtype")
    odt = out_dtype or x.dtype
    with _on(stream):
        b_qkv = _f32(b_qkv)
        _shape("b_qkv", b_qkv, (3 * C,))
        q, k, v = (torch.empty(x.shape, dtype=odt, device=x.device) for _ in range(3))
        ws, wsb = _scratch(workspace, int(lib().swin_qkv_proj_workspace_size(tokens, C)), x.device)
        _check(lib().swin_qkv_proj(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(q), _ptr(k), _ptr(v), dt, _dtcode(q),
                                   tokens, C, _ptr(ws), wsb, _stream(stream)))
    return q, k, v


def swin_proj_postnorm_residual(a: torch.Tensor, w_o: torch.Tensor, b_o: Optional[torch.Tensor], x: torch.Tensor,
                                gamma: Optional[torch.Tensor] = None, beta: Optional[torch.Tensor] = None,
                                eps: float = 1e-5, out: Optional[torch.Tensor] = None,
                                out_dtype: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """out = x + LayerNorm(a W_o^T + b_o) (gamma, beta fp32 [C]); a, x [..., C];
    out of dtype ``out_dtype`` (x's, or float32 for bfloat16 x)."""
    dt = _dtcode(x)
    C = int(x.shape[-1])
    tokens = x.numel() // C
    if a.shape != x.shape or a.dtype != x.dtype or w_o.dtype != x.dtype:
        raise ValueError("a must match x; w_o must have x's dtype")
    _shape("w_o", w_o, (C, C))
    with _on(stream):
        b_o, gamma, beta = _f32(b_o), _f32(gamma), _f32(beta)
        for n, t in (("b_o", b_o), ("gamma", gamma), ("beta", beta)):
            _shape(n, t, (C,))
        if out is None:
            out = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
        ws, wsb = _scratch(workspace, int(lib().swin_proj_postnorm_workspace_size(tokens, C)), x.device)
        _check(lib().swin_proj_postnorm_residual(_ptr(a), _ptr(w_o), _ptr(b_o), _ptr(x), _ptr(gamma), _ptr(beta),
                                                 float(eps), _ptr(out), dt, _dtcode(out), tokens, C, _ptr(ws), wsb,
                                                 _stream(stream)))
    return out


def swin_attn_block_workspace_size(B, H, W, heads, d, M, mode, have_table, dtype) -> int:
    return int(lib().swin_attn_block_workspace_size(B, H, W, heads, d, M, mode, int(bool(have_table)),
                                                    SWIN_F32 if dtype == torch.float32 else SWIN_BF16))


def swin_attn_block_fwd(x: torch.Tensor, heads: int, w_qkv: torch.Tensor, b_qkv: Optional[torch.Tensor],
                        w_o: torch.Tensor, b_o: Optional[torch.Tensor], gamma: Optional[torch.Tensor],
                        beta: Optional[torch.Tensor], M: int, shift: int, mode: int, eps: float = 1e-5,
                        tau=None, bias_table=None, cpb=None, rope_freqs=None, partition: int = SWIN_PARTITION_SHIFTED,
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream=None, out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """x + LN(proj(window_attention(qkv(x)))) for x [B, H, W, C], C = heads * d;
    out of dtype ``out_dtype`` (x's, or float32 for bfloat16 x)."""
    dt = _dtcode(x)
    if x.dim() != 4:
        raise ValueError("x must be [B, H, W, C]")
    B, H, W, C = x.shape
    if C % heads:
        raise ValueError("C must be a multiple of heads")
    d = C // heads
    _shape("w_qkv", w_qkv, (3 * C, C))
    _shape("w_o", w_o, (C, C))
    if w_qkv.dtype != x.dtype or w_o.dtype != x.dtype:
        raise ValueError("weights must have x's dtype")
    with _on(stream):
        b_qkv, b_o, gamma, beta = _f32(b_qkv), _f32(b_o), _f32(gamma), _f32(beta)
        _shape("b_qkv", b_qkv, (3 * C,))
        for n, t in (("b_o", b_o), ("gamma", gamma), ("beta", beta)):
            _shape(n, t, (C,))
        tau, bias_table, rope_freqs = _f32(tau), _f32(bias_table), _f32(rope_freqs)
        _param_shapes(M, heads, d, tau, bias_table, rope_freqs)
        cs, keep = _cpb_struct(cpb, heads)
        need = swin_attn_block_workspace_size(B, H, W, heads, d, M, mode, bias_table is not None, x.dtype)
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        if out is None:
            out = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
        _check(lib().swin_attn_block_fwd(
            _ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(w_o), _ptr(b_o), _ptr(gamma), _ptr(beta), float(eps), _ptr(out),
            dt, _dtcode(out), B, H, W, heads, d, M, shift, int(partition), mode, _ptr(tau), _ptr(bias_table),
            ctypes.byref(cs) if cs is not None else None, _ptr(rope_freqs), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream)))
        del keep
    return out


def swin_index_tables(H: int, W: int, M: int, shift: int, device="cuda", stream=None):
    """(tok_window, tok_region, tok_local) int32 [H, W] and rel_index int32 [M*M, M*M]."""
    mk = lambda *s: torch.empty(s, dtype=torch.int32, device=device)
    tw, tr, tl, ri = mk(H, W), mk(H, W), mk(H, W), mk(M * M, M * M)
    _check(lib().swin_index_tables(H, W, M, shift, _ptr(tw), _ptr(tr), _ptr(tl), _ptr(ri),
                                   _stream(stream)))
    return tw, tr, tl, ri


def swin_stream_status(stream=None) -> int:
    """Synchronise and return/clear the device status word (0 = OK)."""
    return int(lib().swin_stream_status(_stream(stream)))
