"""Double-precision CPU oracle for shifted-window attention — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
Python binding) never calls it, and it shares no code with the CUDA sources.

The arithmetic lives in ``swin_oracle.c`` (plain C, double, OpenMP); this file
only compiles it with gcc when needed and marshals numpy arrays through ctypes.
Every function states the passage it follows:

* ``window_attn`` — "Swin Transformer V2" wiki card, Method, eq. 1 (mode 0) and
  eq. 2 with the ``window_attention`` pseudocode (mode 1); "FLASHSWIN" abstract
  (mode 2, window-local 2D RoPE, exact softmax).
* ``cpb_table`` / ``log_coords`` — "Swin Transformer V2", Method §3.3, eq. 3 and
  eq. 4, ``continuous_bias`` pseudocode; hidden width 512 from the
  hyperparameter table's note on the code.
* ``window_attn_bwd`` — the gradients of ``window_attn`` (chain rule through
  the same definition; see the C source for the formulas).
* ``index_tables`` — the Swin bookkeeping (window, band, local index, relative
  index) built by literally rolling a padded grid.
* ``block`` (a submodule, plain numpy) — the projections and the residual
  post-norm around the attention: "Swin Transformer V2", Method item 1, §3.2,
  fig. 1, ``swin_v2_block`` pseudocode.
* ``window_attn`` / ``window_attn_bwd`` with ``partition`` =
  PARTITION_INTERLEAVED — the interleaved windows of the "Iwin Transformer"
  abstract (the strided index map is a reading; see the C source).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swin_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_swin.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``swin_oracle.c`` into ``liboracle_swin.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lp = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_segment_of.argtypes = [ctypes.c_int] * 3
        lib.oracle_segment_of.restype = ctypes.c_int
        lib.oracle_log_map.argtypes = [ctypes.c_double]
        lib.oracle_log_map.restype = ctypes.c_double
        lib.oracle_log_coords.argtypes = [ctypes.c_int, dp]
        lib.oracle_log_coords.restype = None
        lib.oracle_cpb_table.argtypes = [ctypes.c_int] * 3 + [dp] * 5
        lib.oracle_cpb_table.restype = None
        lib.oracle_log2_map.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.oracle_log2_map.restype = ctypes.c_double
        lib.oracle_cpb_table_code.argtypes = [ctypes.c_int] * 4 + [dp] * 5
        lib.oracle_cpb_table_code.restype = None
        lib.oracle_index_tables.argtypes = [ctypes.c_int] * 4 + [ip] * 4
        lib.oracle_index_tables.restype = None
        lib.oracle_window_attn.argtypes = (
            [dp] * 4 + [ctypes.c_int] * 9 + [dp] * 3 + [lp, ctypes.c_int64, ctypes.c_int]
        )
        lib.oracle_window_attn.restype = ctypes.c_int
        lib.oracle_window_attn_bwd.argtypes = ([dp] * 10 + [ctypes.c_int] * 9 + [dp] * 3 + [ctypes.c_int])
        lib.oracle_window_attn_bwd.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dp(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def segment_of(M: int, shift: int, y: int) -> int:
    """Segment id of coordinate ``y`` (boundaries at shift + kM)."""
    return int(_load().oracle_segment_of(M, shift, y))


def log_map(delta: float) -> float:
    """eq. 4 for one offset component: sign(delta) * ln(1 + |delta|)."""
    return float(_load().oracle_log_map(float(delta)))


def log_coords(M: int) -> np.ndarray:
    """[(2M-1)^2, 2] table of (dx_hat, dy_hat), rows (dy+M-1)*(2M-1)+(dx+M-1)."""
    R = 2 * M - 1
    out = np.zeros((R * R, 2), dtype=np.float64)
    _load().oracle_log_coords(M, _dp(out))
    return out


def cpb_table(M: int, heads: int, w1, b1, w2, b2) -> np.ndarray:
    """eq. 3: G over every window offset -> [(2M-1)^2, heads] float64."""
    w1 = _f64(w1)
    w2 = _f64(w2)
    hidden = w1.shape[0]
    assert w1.shape == (hidden, 2) and w2.shape == (heads, hidden)
    b1 = _f64(b1)
    b2 = _f64(b2)
    R = 2 * M - 1
    out = np.zeros((R * R, heads), dtype=np.float64)
    _load().oracle_cpb_table(M, heads, hidden, _dp(w1), _dp(b1), _dp(w2), _dp(b2), _dp(out))
    return out


def log2_map(delta: float, Mp: int) -> float:
    """The released code's coordinate: sign(x) log2(1 + |x|) / log2(8) of
    x = delta * 8 / (Mp - 1)."""
    return float(_load().oracle_log2_map(float(delta), int(Mp)))


def cpb_table_code(M: int, heads: int, w1, b1, w2, b2, pretrained_M: int = 0) -> np.ndarray:
    """G in the released code's form (normalised log2 coordinates, output
    16 sigmoid(G)) over every offset of an MxM window; pretrained_M = 0 means
    M.  [(2M-1)^2, heads] float64."""
    w1 = _f64(w1)
    w2 = _f64(w2)
    hidden = w1.shape[0]
    assert w1.shape == (hidden, 2) and w2.shape == (heads, hidden)
    b1 = _f64(b1)
    b2 = _f64(b2)
    R = 2 * M - 1
    out = np.zeros((R * R, heads), dtype=np.float64)
    _load().oracle_cpb_table_code(M, pretrained_M if pretrained_M > 0 else M, heads, hidden, _dp(w1), _dp(b1),
                                  _dp(w2), _dp(b2), _dp(out))
    return out


def index_tables(H: int, W: int, M: int, shift: int):
    """(tok_window, tok_region, tok_local) int32 [H, W] and rel_index int32 [N, N]."""
    tw = np.zeros((H, W), dtype=np.int32)
    tr = np.zeros((H, W), dtype=np.int32)
    tl = np.zeros((H, W), dtype=np.int32)
    ri = np.zeros((M * M, M * M), dtype=np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)
    _load().oracle_index_tables(
        H, W, M, shift, tw.ctypes.data_as(ip), tr.ctypes.data_as(ip), tl.ctypes.data_as(ip),
        ri.ctypes.data_as(ip),
    )
    return tw, tr, tl, ri


MODE_DOT_BIAS = 0
MODE_COSINE_CPB = 1
MODE_ROPE = 2

PARTITION_SHIFTED = 0
PARTITION_INTERLEAVED = 1


def window_attn(q, k, v, M: int, shift: int, mode: int, tau=None, table=None,
                rope_freqs=None, queries=None, nthreads: int = 0, partition: int = PARTITION_SHIFTED) -> np.ndarray:
    """Shifted-window attention in float64 (or, with ``partition`` =
    PARTITION_INTERLEAVED and shift 0, attention in Iwin's interleaved windows).

    q, k, v: [B, H, W, heads, d] (any float dtype; read as float64).
    Returns [B, H, W, heads, d] float64, or [len(queries), heads, d] when
    ``queries`` (flat token ids b*H*W + y*W + x) is given.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, H, W, heads, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    tau = _f64(tau)
    table = _f64(table)
    rope_freqs = _f64(rope_freqs)
    if queries is None:
        out = np.zeros((B, H, W, heads, d), dtype=np.float64)
        qp = ctypes.POINTER(ctypes.c_int64)()
        nq = B * H * W
    else:
        qarr = np.ascontiguousarray(np.asarray(queries, dtype=np.int64))
        nq = int(qarr.shape[0])
        out = np.zeros((nq, heads, d), dtype=np.float64)
        qp = qarr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    rc = _load().oracle_window_attn(
        _dp(q), _dp(k), _dp(v), _dp(out), B, H, W, heads, d, M, shift, int(partition), mode,
        _dp(tau), _dp(table), _dp(rope_freqs), qp, nq, int(nthreads),
    )
    if rc != 0:
        raise ValueError("oracle_window_attn rejected its arguments")
    return out


def window_attn_bwd(q, k, v, dout, M: int, shift: int, mode: int, tau=None, table=None, rope_freqs=None,
                    nthreads: int = 0, partition: int = PARTITION_SHIFTED) -> dict:
    """Gradients of L = sum(dout * window_attn(...)) in float64: dq, dk, dv
    ([B, H, W, heads, d]), dtable ([(2M-1)^2, heads], modes 0 and 1 with a table), dtau
    ([heads], mode 1), drope ([2, d/4], mode 2)."""
    q, k, v, dout = (_f64(a) for a in (q, k, v, dout))
    B, H, W, heads, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape and dout.shape == q.shape
    tau, table, rope_freqs = _f64(tau), _f64(table), _f64(rope_freqs)
    R = 2 * M - 1
    dq, dk, dv = (np.zeros_like(q) for _ in range(3))
    dtable = np.zeros((R * R, heads)) if mode != 2 and table is not None else None
    dtau = np.zeros(heads) if mode == 1 else None
    drope = np.zeros((2, d // 4)) if mode == 2 else None
    rc = _load().oracle_window_attn_bwd(
        _dp(q), _dp(k), _dp(v), _dp(dout), _dp(dq), _dp(dk), _dp(dv), _dp(dtable), _dp(dtau), _dp(drope),
        B, H, W, heads, d, M, shift, int(partition), mode, _dp(tau), _dp(table), _dp(rope_freqs), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_window_attn_bwd rejected its arguments")
    out = {"dq": dq, "dk": dk, "dv": dv}
    if dtable is not None:
        out["dtable"] = dtable
    if dtau is not None:
        out["dtau"] = dtau
    if drope is not None:
        out["drope"] = drope
    return out
