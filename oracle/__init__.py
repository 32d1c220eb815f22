"""Python face of the CPU oracle (test infrastructure only).

Thin ctypes wrappers around ``h3_oracle.cpp``; every arithmetic step lives in the
C++ file. Only the test suite, the smoke check and the benchmark's CPU-baseline
leg may import this package. It imports nothing from the CUDA library package.

Arrays are numpy: bf16 values travel as ``uint16`` bit patterns, fp64 results as
``float64``.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        _LIB = C.CDLL(path)
        _declare(_LIB)
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _declare(L):
    vp, i64, i32, dbl = C.c_void_p, C.c_int64, C.c_int, C.c_double
    L.orc_f64_to_bf16.restype = C.c_uint16
    L.orc_f64_to_bf16.argtypes = [dbl]
    L.orc_bf16_to_f64.restype = dbl
    L.orc_bf16_to_f64.argtypes = [C.c_uint16]
    L.orc_bf16_round.argtypes = [vp, i64, vp]
    L.orc_bf16_decode.argtypes = [vp, i64, vp]
    L.orc_quantize_rows.argtypes = [vp, i64, i64, vp, vp]
    L.orc_gemm_i8.restype = i64
    L.orc_gemm_i8.argtypes = [vp, vp, i64, i64, i64, vp]
    L.orc_gemm_f64.argtypes = [vp, vp, i64, i64, i64, vp]
    L.orc_dequant.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    L.orc_adaln_linear.argtypes = [vp, vp, vp, i64, vp]
    L.orc_layernorm.argtypes = [vp, i64, i64, dbl, vp]
    L.orc_modulate_bf16.argtypes = [vp, i64, i64, vp, vp, vp]
    L.orc_grid_positions.argtypes = [i64, i64, i64, vp, vp, vp]
    L.orc_rope_3d.argtypes = [vp, i64, vp, vp, vp, i32, i32, i32, i32, i32, dbl]
    L.orc_attention.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp]
    L.orc_gelu_tanh.argtypes = [vp, i64, vp]
    L.orc_gated_residual.argtypes = [vp, vp, vp, i64, i64, vp]
    L.orc_token_pair.argtypes = [vp, i64, i64, i64, i64, i64, vp]
    L.orc_token_unpair.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, vp]
    L.orc_range_delta.argtypes = [vp, vp, i64, vp]
    L.orc_range_apply.argtypes = [vp, vp, i64, vp]
    L.orc_threads.restype = i32
    L.orc_threads.argtypes = []
    L.orc_block_forward.restype = i32
    L.orc_block_forward.argtypes = [vp, vp, vp, vp, vp, i64, vp, vp]


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- steps

def threads() -> int:
    return lib().orc_threads()


def bf16_round(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().orc_bf16_round(_p(v), v.size, _p(out))
    return out


def bf16_decode(b) -> np.ndarray:
    b = _c(b, np.uint16)
    out = np.empty(b.shape, np.float64)
    lib().orc_bf16_decode(_p(b), b.size, _p(out))
    return out


def quantize_rows(v):
    """Per-row symmetric int8 with an F32 scale. v: float32 [rows, cols]."""
    v = _c(v, np.float32)
    rows, cols = v.shape
    q = np.empty((rows, cols), np.int8)
    s = np.empty(rows, np.float32)
    lib().orc_quantize_rows(_p(v), rows, cols, _p(q), _p(s))
    return q, s


def gemm_i8(A, W):
    A = _c(A, np.int8)
    W = _c(W, np.int8)
    M, K = A.shape
    N, K2 = W.shape
    assert K == K2
    out = np.empty((M, N), np.int32)
    over = lib().orc_gemm_i8(_p(A), _p(W), M, N, K, _p(out))
    if over:
        raise OverflowError(f"{over} accumulators exceed int32")
    return out


def gemm_f64(A, W):
    A = _c(A, np.float64)
    W = _c(W, np.float64)
    M, K = A.shape
    N, _ = W.shape
    out = np.empty((M, N), np.float64)
    lib().orc_gemm_f64(_p(A), _p(W), M, N, K, _p(out))
    return out


def dequant(acc, s_tok, s_ch, bias=None):
    acc = _c(acc, np.int32)
    rows, cols = acc.shape
    out = np.empty((rows, cols), np.float64)
    lib().orc_dequant(_p(acc), rows, cols, _p(_c(s_tok, np.float32)), _p(_c(s_ch, np.float32)),
                      _p(None if bias is None else _c(bias, np.float32)), _p(out))
    return out


def adaln_linear(w_ada_bf16, b_ada, c):
    w = _c(w_ada_bf16, np.uint16)
    c = _c(c, np.float32)
    d = c.shape[-1]
    assert w.shape == (6 * d, d)
    out = np.empty(6 * d, np.float64)
    lib().orc_adaln_linear(_p(w), _p(None if b_ada is None else _c(b_ada, np.float32)), _p(c), d, _p(out))
    return out


def layernorm(x, eps):
    x = _c(x, np.float64)
    rows, d = x.shape
    out = np.empty_like(x)
    lib().orc_layernorm(_p(x), rows, d, eps, _p(out))
    return out


def modulate_bf16(y, shift, scale):
    y = _c(y, np.float64)
    rows, d = y.shape
    out = np.empty((rows, d), np.uint16)
    lib().orc_modulate_bf16(_p(y), rows, d, _p(_c(shift, np.float64)), _p(_c(scale, np.float64)), _p(out))
    return out


def grid_positions(T, H, W):
    n = T * H * W
    t, h, w = (np.empty(n, np.int32) for _ in range(3))
    lib().orc_grid_positions(T, H, W, _p(t), _p(h), _p(w))
    return t, h, w


def rope_3d(x, tpos, hpos, wpos, n_heads, head_dim, split, theta=10000.0):
    """Returns a rotated copy of x [rows, n_heads*head_dim]."""
    x = np.array(x, dtype=np.float64, order="C", copy=True)
    rows = x.shape[0]
    rt, rh, rw = split
    lib().orc_rope_3d(_p(x), rows, _p(_c(tpos, np.int32)), _p(_c(hpos, np.int32)), _p(_c(wpos, np.int32)),
                      n_heads, head_dim, rt, rh, rw, theta)
    return x


def attention(Q, K, V, n_heads, head_dim):
    Q, K, V = (_c(a, np.float64) for a in (Q, K, V))
    nq, L = Q.shape[0], K.shape[0]
    out = np.empty_like(Q)
    lib().orc_attention(_p(Q), _p(K), _p(V), nq, L, n_heads, head_dim, _p(out))
    return out


def gelu_tanh(x):
    x = _c(x, np.float64)
    out = np.empty_like(x)
    lib().orc_gelu_tanh(_p(x), x.size, _p(out))
    return out


def gated_residual(x, y, gate):
    x = _c(x, np.float64)
    y = _c(y, np.float64)
    rows, d = x.shape
    out = np.empty_like(x)
    lib().orc_gated_residual(_p(x), _p(y), _p(_c(gate, np.float64)), rows, d, _p(out))
    return out


def token_pair(x_bf16, B, T, H, W, d):
    x = _c(x_bf16, np.uint16)
    assert W % 2 == 0
    out = np.empty((B, T, H, W // 2, d), np.uint16)
    lib().orc_token_pair(_p(x), B, T, H, W, d, _p(out))
    return out


def token_unpair(x_bf16, xm_bf16, ym, B, T, H, W, d):
    out = np.empty((B, T, H, W, d), np.float64)
    lib().orc_token_unpair(_p(_c(x_bf16, np.uint16)), _p(_c(xm_bf16, np.uint16)), _p(_c(ym, np.float64)),
                           B, T, H, W, d, _p(out))
    return out


def range_delta(before_bf16, after_bf16):
    """delta = after - before (fp64 of bf16 values)."""
    a, b = _c(before_bf16, np.uint16), _c(after_bf16, np.uint16)
    out = np.empty(a.shape, np.float64)
    lib().orc_range_delta(_p(a), _p(b), a.size, _p(out))
    return out


def range_apply(x_bf16, delta):
    """bf16(x + delta)."""
    x, d = _c(x_bf16, np.uint16), _c(delta, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_range_apply(_p(x), _p(d), x.size, _p(out))
    return out


# --------------------------------------------------------------------------- block

@dataclass
class Dims:
    B: int
    T: int
    H: int
    W: int
    d: int
    n_heads: int
    head_dim: int
    d_ff: int
    rope: tuple
    rope_theta: float = 10000.0
    ln_eps: float = 1e-6
    qkv_int8: bool = True
    wo_bf16: bool = False

    @property
    def L(self):
        return self.T * self.H * self.W


class _CDims(C.Structure):
    _fields_ = [("B", C.c_int64), ("T", C.c_int64), ("H", C.c_int64), ("W", C.c_int64),
                ("d", C.c_int64), ("n_heads", C.c_int64), ("head_dim", C.c_int64), ("d_ff", C.c_int64),
                ("rope_t", C.c_int), ("rope_h", C.c_int), ("rope_w", C.c_int),
                ("rope_theta", C.c_double), ("ln_eps", C.c_double), ("qkv_int8", C.c_int),
                ("wo_bf16", C.c_int)]


class _CWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("w_ada", "b_ada", "wqkv", "sqkv", "wqkv_bf16", "bqkv", "wo", "so", "bo",
                 "w1", "s1", "b1", "w2", "s2", "b2", "wo_bf16")]


class _CTrace(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("mod", "h1", "qkv", "attn", "x1", "h2", "gelu")]


_WEIGHT_DTYPES = {"w_ada": np.uint16, "b_ada": np.float32, "wqkv": np.int8, "sqkv": np.float32,
                  "wqkv_bf16": np.uint16, "bqkv": np.float32, "wo": np.int8, "so": np.float32,
                  "bo": np.float32, "w1": np.int8, "s1": np.float32, "b1": np.float32,
                  "w2": np.int8, "s2": np.float32, "b2": np.float32, "wo_bf16": np.uint16}


def block_forward(dims: Dims, weights: dict, c, x_bf16, rows: Optional[np.ndarray] = None,
                  trace: bool = False):
    """One block forward. Returns fp64 [n_rows, d] (and a dict of intermediates
    when ``trace``). ``weights`` holds int8 codes and F32 scales (see
    ``_WEIGHT_DTYPES``); missing entries are NULL."""
    R = dims.B * dims.L
    d, F = dims.d, dims.d_ff
    keep = {}
    cw = _CWeights()
    for name, dt in _WEIGHT_DTYPES.items():
        a = weights.get(name)
        if a is not None:
            a = _c(a, dt)
            keep[name] = a
            setattr(cw, name, a.ctypes.data)
    cd = _CDims(dims.B, dims.T, dims.H, dims.W, d, dims.n_heads, dims.head_dim, F,
                dims.rope[0], dims.rope[1], dims.rope[2], dims.rope_theta, dims.ln_eps,
                1 if dims.qkv_int8 else 0, 1 if dims.wo_bf16 else 0)
    x = _c(x_bf16, np.uint16).reshape(R, d)
    c = _c(c, np.float32).reshape(dims.B, d)
    if rows is None:
        sel = None
        n_rows = R
    else:
        sel = _c(rows, np.int64)
        n_rows = sel.size
    out = np.empty((n_rows, d), np.float64)
    tr = None
    bufs = {}
    if trace:
        bufs = {"mod": np.empty((dims.B, 6 * d)), "h1": np.empty((R, d), np.uint16),
                "qkv": np.empty((R, 3 * d)), "attn": np.empty((n_rows, d)), "x1": np.empty((n_rows, d)),
                "h2": np.empty((n_rows, d), np.uint16), "gelu": np.empty((n_rows, F))}
        tr = _CTrace(**{k: v.ctypes.data for k, v in bufs.items()})
    rc = lib().orc_block_forward(C.byref(cd), C.byref(cw), _p(c), _p(x), _p(sel), n_rows, _p(out),
                                 C.byref(tr) if tr is not None else None)
    if rc != 0:
        raise OverflowError("int8 accumulator overflow in the oracle block")
    return (out, bufs) if trace else out
