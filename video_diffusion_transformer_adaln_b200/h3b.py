"""ctypes binding of the h3b C ABI (include/h3b.h): argument marshalling only.

Every function has the C entry point's name and takes torch CUDA tensors (or
None for optional pointers); all computation happens in the CUDA library. If the
library has not been built this module raises on first use: there is no
fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# H3B_CHECKED=1 selects the checked build (indices tested against buffer extents in every kernel)
LIB_PATH = os.path.join(_HERE, "_lib", "libh3b_checked.so" if os.environ.get("H3B_CHECKED") == "1" else "libh3b.so")

H3B_OK = 0
STATUS = {0: "H3B_OK", -1: "H3B_ERR_ARG", -2: "H3B_ERR_SHAPE", -3: "H3B_ERR_ALIGN",
          -4: "H3B_ERR_WORKSPACE", -5: "H3B_ERR_ARCH", -6: "H3B_ERR_CUDA", -7: "H3B_ERR_DEVICE_CHECK"}


class H3BError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")


class Dims(C.Structure):
    _fields_ = [("B", C.c_int), ("T", C.c_int), ("H", C.c_int), ("W", C.c_int),
                ("d", C.c_int), ("n_heads", C.c_int), ("head_dim", C.c_int), ("d_ff", C.c_int),
                ("rope_t", C.c_int), ("rope_h", C.c_int), ("rope_w", C.c_int),
                ("rope_theta", C.c_float), ("ln_eps", C.c_float), ("qkv_int8", C.c_int),
                ("wo_bf16", C.c_int)]

    @property
    def L(self) -> int:
        return self.T * self.H * self.W


WEIGHT_FIELDS = ("w_ada", "b_ada", "wqkv", "sqkv", "wqkv_bf16", "bqkv", "wo", "so", "bo",
                 "w1", "s1", "b1", "w2", "s2", "b2", "wo_bf16")


class BlockWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_FIELDS]


class KernelTime(C.Structure):
    _fields_ = [("name", C.c_char_p), ("launches", C.c_int), ("total_ms", C.c_double)]


_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"h3b CUDA library not built ({LIB_PATH}); run "
                               "video_diffusion_transformer_adaln_b200/build.py"
                               + (" --checked" if LIB_PATH.endswith("_checked.so") else ""))
        L = C.CDLL(LIB_PATH)
        _declare(L)
        _LIB = L
    return _LIB


def _declare(L):
    vp, i32, f32, sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t
    L.h3b_status_string.restype = C.c_char_p
    L.h3b_status_string.argtypes = [i32]
    L.h3b_last_error_detail.restype = C.c_char_p
    L.h3b_last_error_detail.argtypes = []
    sigs = {
        "h3b_workspace_size": [vp, C.POINTER(sz)],
        "h3b_block_forward": [vp, vp, vp, vp, vp, sz, vp],
        "h3b_block_forward_noalloc": [vp, vp, vp, vp, vp],
        "h3b_blocks_forward": [vp, vp, i32, vp, vp, vp, sz, vp],
        "h3b_blocks_forward_reduced": [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp],
        "h3b_token_pair": [vp, vp, vp, vp, vp],
        "h3b_token_unpair": [vp, vp, vp, vp, vp, vp],
        "h3b_quantize_weights": [vp, i32, i32, vp, vp, vp],
        "h3b_device_error": [C.POINTER(C.c_uint), i32],
        "h3b_test_bounded_wait": [C.c_ulonglong, C.POINTER(C.c_int)],
        "h3b_adaln_modulation": [vp, vp, vp, vp, vp, vp],
        "h3b_ln_modulate_quantize": [vp, i32, i32, f32, vp, vp, i32, i32, vp, vp, vp, vp, i32, vp],
        "h3b_quantize_rows": [vp, i32, i32, vp, vp, vp, vp],
        "h3b_gemm_i8_s32": [vp, vp, vp, i32, i32, i32, vp],
        "h3b_gemm_i8_dequant": [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp],
        "h3b_qkv_projection": [vp, vp, vp, vp, vp, vp, vp],
        "h3b_attention": [vp, vp, vp, vp, vp],
        "h3b_gemm_i8_gated_residual": [vp, vp, vp, vp, vp, vp, i32, i32, vp, i32, i32, i32, vp],
        "h3b_gemm_bf16_gated_residual": [vp, vp, vp, vp, i32, i32, vp, i32, i32, i32, vp],
        "h3b_graph_capture_blocks": [vp, vp, i32, vp, vp, vp, sz, vp],
        "h3b_graph_launch": [vp, vp],
        "h3b_blocks_forward_cached": [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp],
        "h3b_range_delta": [vp, vp, vp, C.c_longlong, vp],
        "h3b_range_apply": [vp, vp, C.c_longlong, vp],
        "h3b_gemm_i8_gelu": [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp],
    }
    for name, args in sigs.items():
        f = getattr(L, name)
        f.restype = i32
        f.argtypes = args
    L.h3b_rope_table_bytes.restype = sz
    L.h3b_rope_table_bytes.argtypes = [vp]
    L.h3b_profile_enable.restype = i32
    L.h3b_profile_enable.argtypes = [i32]
    L.h3b_profile_read.restype = i32
    L.h3b_profile_read.argtypes = [C.POINTER(KernelTime), i32]
    L.h3b_graph_kernel_count.restype = i32
    L.h3b_graph_kernel_count.argtypes = [vp]
    L.h3b_graph_destroy.restype = None
    L.h3b_graph_destroy.argtypes = [vp]
    L.h3b_checked_build.restype = i32
    L.h3b_checked_build.argtypes = []


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return int(t)
    return t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != H3B_OK:
        detail = lib().h3b_last_error_detail().decode(errors="replace")
        raise H3BError(status, where, detail)


def status_string(status: int) -> str:
    return lib().h3b_status_string(status).decode()


# --------------------------------------------------------------------------- block level

def make_dims(B, T, H, W, d, n_heads, head_dim, d_ff, rope, rope_theta=10000.0, ln_eps=1e-6,
              qkv_int8=True, wo_bf16=False) -> Dims:
    return Dims(B, T, H, W, d, n_heads, head_dim, d_ff, rope[0], rope[1], rope[2], rope_theta, ln_eps,
                1 if qkv_int8 else 0, 1 if wo_bf16 else 0)


def make_weights(tensors: Dict[str, Optional[torch.Tensor]]) -> BlockWeights:
    """Weight struct from a dict of device tensors (missing names are NULL)."""
    w = BlockWeights()
    for n in WEIGHT_FIELDS:
        t = tensors.get(n)
        setattr(w, n, _p(t) if t is not None else None)
    return w


def h3b_workspace_size(dims: Dims) -> int:
    n = C.c_size_t(0)
    _check(lib().h3b_workspace_size(C.byref(dims), C.byref(n)), "h3b_workspace_size")
    return n.value


def h3b_block_forward(dims: Dims, w: BlockWeights, c, x, ws, stream=None):
    _check(lib().h3b_block_forward(C.byref(dims), C.byref(w), _p(c), _p(x), _p(ws), ws.numel() * ws.element_size(),
                                   _s(stream)), "h3b_block_forward")


def h3b_block_forward_noalloc(dims: Dims, w: BlockWeights, c, x, stream=None):
    """Block forward with the library's fixed 32 MiB device scratch (no workspace,
    no allocation); see include/h3b.h for its limits and sharing rules."""
    _check(lib().h3b_block_forward_noalloc(C.byref(dims), C.byref(w), _p(c), _p(x), _s(stream)),
           "h3b_block_forward_noalloc")


def h3b_blocks_forward(dims: Dims, ws_list: Sequence[BlockWeights], c, x, ws, stream=None):
    arr = (BlockWeights * len(ws_list))(*ws_list)
    _check(lib().h3b_blocks_forward(C.byref(dims), arr, len(ws_list), _p(c), _p(x), _p(ws),
                                    ws.numel() * ws.element_size(), _s(stream)), "h3b_blocks_forward")


def h3b_blocks_forward_cached(dims: Dims, ws_list: Sequence[BlockWeights], first: int, last: int, fresh: bool,
                              c, x, x_save, delta, ws, stream=None):
    arr = (BlockWeights * len(ws_list))(*ws_list)
    _check(lib().h3b_blocks_forward_cached(C.byref(dims), arr, len(ws_list), first, last, 1 if fresh else 0, _p(c),
                                           _p(x), _p(x_save), _p(delta), _p(ws), ws.numel() * ws.element_size(),
                                           _s(stream)), "h3b_blocks_forward_cached")


def h3b_range_delta(before, after, delta, stream=None):
    _check(lib().h3b_range_delta(_p(before), _p(after), _p(delta), before.numel(), _s(stream)), "h3b_range_delta")


def h3b_range_apply(x, delta, stream=None):
    _check(lib().h3b_range_apply(_p(x), _p(delta), x.numel(), _s(stream)), "h3b_range_apply")


class Graph:
    """A captured multi-block pass (h3b_graph_capture_blocks); replay with launch()."""

    def __init__(self, handle: int, keep):
        self.handle = handle
        self._keep = keep  # the argument structs the capture referenced

    def launch(self, stream=None):
        _check(lib().h3b_graph_launch(self.handle, _s(stream)), "h3b_graph_launch")

    @property
    def kernel_count(self) -> int:
        return lib().h3b_graph_kernel_count(self.handle)

    def destroy(self):
        if self.handle:
            lib().h3b_graph_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def h3b_graph_launch(g: Graph, stream=None):
    g.launch(stream)


def h3b_graph_kernel_count(g: Graph) -> int:
    return g.kernel_count


def h3b_graph_destroy(g: Graph):
    g.destroy()


def h3b_graph_capture_blocks(dims: Dims, blocks, c, x, ws) -> Graph:
    arr = (BlockWeights * len(blocks))(*blocks)
    h = C.c_void_p()
    _check(lib().h3b_graph_capture_blocks(C.byref(dims), arr, len(blocks), _p(c), _p(x), _p(ws),
                                          ws.numel() * ws.element_size(), C.byref(h)), "h3b_graph_capture_blocks")
    return Graph(h.value, (dims, arr))


def h3b_blocks_forward_reduced(full: Dims, ws_list: Sequence[BlockWeights], first: int, last: int, c, x, xm, ym,
                               ws, stream=None):
    arr = (BlockWeights * len(ws_list))(*ws_list)
    _check(lib().h3b_blocks_forward_reduced(C.byref(full), arr, len(ws_list), first, last, _p(c), _p(x), _p(xm),
                                            _p(ym), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "h3b_blocks_forward_reduced")


def h3b_token_pair(full: Dims, x, xm, xm_copy=None, stream=None):
    _check(lib().h3b_token_pair(C.byref(full), _p(x), _p(xm), _p(xm_copy), _s(stream)), "h3b_token_pair")


def h3b_token_unpair(full: Dims, x, xm, ym, out, stream=None):
    _check(lib().h3b_token_unpair(C.byref(full), _p(x), _p(xm), _p(ym), _p(out), _s(stream)), "h3b_token_unpair")


def h3b_quantize_weights(w, q, s, stream=None):
    rows, cols = w.shape
    _check(lib().h3b_quantize_weights(_p(w), rows, cols, _p(q), _p(s), _s(stream)), "h3b_quantize_weights")


def h3b_checked_build() -> bool:
    return bool(lib().h3b_checked_build())


def h3b_device_error(clear: bool = True) -> int:
    code = C.c_uint(0)
    st = lib().h3b_device_error(C.byref(code), 1 if clear else 0)
    if st not in (H3B_OK, -7):
        _check(st, "h3b_device_error")
    return code.value


def h3b_test_bounded_wait(limit_ns: int) -> int:
    """Run the library's bounded-wait test hook (see include/h3b.h); 1 when the wait ran out."""
    out = C.c_int(-1)
    _check(lib().h3b_test_bounded_wait(limit_ns, C.byref(out)), "h3b_test_bounded_wait")
    return out.value


# --------------------------------------------------------------------------- steps

def h3b_adaln_modulation(dims: Dims, w_ada, b_ada, c, mod, stream=None):
    _check(lib().h3b_adaln_modulation(C.byref(dims), _p(w_ada), _p(b_ada), _p(c), _p(mod), _s(stream)),
           "h3b_adaln_modulation")


def h3b_ln_modulate_quantize(x, rows, d, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out=None,
                             absmax_zero=None, write_codes=True, stream=None):
    _check(lib().h3b_ln_modulate_quantize(_p(x), rows, d, eps, _p(shift), _p(scale), rows_per_item, mod_stride,
                                          _p(q), _p(s), _p(h_out), _p(absmax_zero), 1 if write_codes else 0,
                                          _s(stream)), "h3b_ln_modulate_quantize")


def h3b_quantize_rows(h, q, s, absmax=None, stream=None):
    rows, cols = h.shape
    _check(lib().h3b_quantize_rows(_p(h), rows, cols, _p(absmax), _p(q), _p(s), _s(stream)), "h3b_quantize_rows")


def h3b_gemm_i8_s32(A, W, C_out, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _check(lib().h3b_gemm_i8_s32(_p(A), _p(W), _p(C_out), M, N, K, _s(stream)), "h3b_gemm_i8_s32")


def h3b_gemm_i8_dequant(A, sA, W, sW, bias, out, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _check(lib().h3b_gemm_i8_dequant(_p(A), _p(sA), _p(W), _p(sW), _p(bias), _p(out), M, N, K, _s(stream)),
           "h3b_gemm_i8_dequant")


def h3b_rope_table_bytes(dims: Dims) -> int:
    return lib().h3b_rope_table_bytes(C.byref(dims))


def h3b_qkv_projection(dims: Dims, A, sA, w: BlockWeights, qkv, rope_ws, stream=None):
    _check(lib().h3b_qkv_projection(C.byref(dims), _p(A), _p(sA), C.byref(w), _p(qkv), _p(rope_ws), _s(stream)),
           "h3b_qkv_projection")


def h3b_attention(dims: Dims, qkv, o, absmax, stream=None):
    _check(lib().h3b_attention(C.byref(dims), _p(qkv), _p(o), _p(absmax), _s(stream)), "h3b_attention")


def h3b_gemm_i8_gated_residual(A, sA, W, sW, bias, gate, rows_per_item, gate_stride, x, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _check(lib().h3b_gemm_i8_gated_residual(_p(A), _p(sA), _p(W), _p(sW), _p(bias), _p(gate), rows_per_item,
                                            gate_stride, _p(x), M, N, K, _s(stream)), "h3b_gemm_i8_gated_residual")


def h3b_gemm_bf16_gated_residual(A, W, bias, gate, rows_per_item, gate_stride, x, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _check(lib().h3b_gemm_bf16_gated_residual(_p(A), _p(W), _p(bias), _p(gate), rows_per_item, gate_stride,
                                              _p(x), M, N, K, _s(stream)), "h3b_gemm_bf16_gated_residual")


def h3b_gemm_i8_gelu(A, sA, W, sW, bias, g, absmax, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _check(lib().h3b_gemm_i8_gelu(_p(A), _p(sA), _p(W), _p(sW), _p(bias), _p(g), _p(absmax), M, N, K, _s(stream)),
           "h3b_gemm_i8_gelu")


# --------------------------------------------------------------------------- profiling

def h3b_profile_enable(on: bool = True):
    _check(lib().h3b_profile_enable(1 if on else 0), "h3b_profile_enable")


def h3b_profile_read(max_entries: int = 64) -> Dict[str, tuple]:
    """{kernel name: (launches, total device ms)} since the last read."""
    arr = (KernelTime * max_entries)()
    n = lib().h3b_profile_read(arr, max_entries)
    if n < 0:
        _check(n, "h3b_profile_read")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n)}
