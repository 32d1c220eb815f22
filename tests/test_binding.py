"""The ctypes binding's marshalling, on the CPU: each same-name wrapper passes its
tensors' addresses, the sizes it derives from their shapes and the stream to the C
entry point in the order include/h3b.h declares. A recording stand-in replaces the
library for these tests (no GPU, nothing executes)."""
import ctypes as C

import pytest
import torch

from video_diffusion_transformer_adaln_b200 import h3b


class Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(h3b, "_LIB", r)
    return r


def t(*shape, dtype=torch.float32):
    return torch.empty(shape, dtype=dtype)


def ptr(x):
    return x.data_ptr()


def last(rec, name):
    assert rec.calls and rec.calls[-1][0] == name
    return rec.calls[-1][1]


def test_gemm_wrappers_pass_operands_then_m_n_k(rec):
    A, W = t(48, 32, dtype=torch.int8), t(64, 32, dtype=torch.int8)
    sA, sW, bias, Cout = t(48), t(64), t(64), t(48, 64, dtype=torch.int32)
    h3b.h3b_gemm_i8_s32(A, W, Cout, stream=7)
    assert last(rec, "h3b_gemm_i8_s32") == (ptr(A), ptr(W), ptr(Cout), 48, 64, 32, 7)
    out = t(48, 64, dtype=torch.bfloat16)
    h3b.h3b_gemm_i8_dequant(A, sA, W, sW, bias, out, stream=7)
    assert last(rec, "h3b_gemm_i8_dequant") == (ptr(A), ptr(sA), ptr(W), ptr(sW), ptr(bias), ptr(out), 48, 64, 32, 7)
    am = t(48)
    h3b.h3b_gemm_i8_gelu(A, sA, W, sW, None, out, am, stream=7)
    assert last(rec, "h3b_gemm_i8_gelu") == (ptr(A), ptr(sA), ptr(W), ptr(sW), None, ptr(out), ptr(am), 48, 64, 32, 7)
    gate = t(2, 6 * 64)
    h3b.h3b_gemm_i8_gated_residual(A, sA, W, sW, bias, gate, 24, 6 * 64, out, stream=7)
    assert last(rec, "h3b_gemm_i8_gated_residual") == (ptr(A), ptr(sA), ptr(W), ptr(sW), ptr(bias), ptr(gate), 24,
                                                       384, ptr(out), 48, 64, 32, 7)
    Ab, Wb = t(48, 32, dtype=torch.bfloat16), t(64, 32, dtype=torch.bfloat16)
    h3b.h3b_gemm_bf16_gated_residual(Ab, Wb, None, gate, 24, 384, out, stream=7)
    assert last(rec, "h3b_gemm_bf16_gated_residual") == (ptr(Ab), ptr(Wb), None, ptr(gate), 24, 384, ptr(out), 48, 64,
                                                         32, 7)


def test_row_wrappers_derive_rows_and_columns(rec):
    h, q, s, am = t(5, 256, dtype=torch.bfloat16), t(5, 256, dtype=torch.int8), t(5), t(5)
    h3b.h3b_quantize_rows(h, q, s, absmax=am, stream=3)
    assert last(rec, "h3b_quantize_rows") == (ptr(h), 5, 256, ptr(am), ptr(q), ptr(s), 3)
    w = t(7, 32)
    qw, sw = t(7, 32, dtype=torch.int8), t(7)
    h3b.h3b_quantize_weights(w, qw, sw, stream=3)
    assert last(rec, "h3b_quantize_weights") == (ptr(w), 7, 32, ptr(qw), ptr(sw), 3)
    x, sh, sc, hout, az = t(5, 256, dtype=torch.bfloat16), t(256), t(256), t(5, 256, dtype=torch.bfloat16), t(5)
    h3b.h3b_ln_modulate_quantize(x, 5, 256, 1e-6, sh, sc, 5, 0, q, s, h_out=hout, absmax_zero=az, stream=3)
    args = last(rec, "h3b_ln_modulate_quantize")
    assert args[:3] == (ptr(x), 5, 256) and args[3] == pytest.approx(1e-6)
    assert args[4:] == (ptr(sh), ptr(sc), 5, 0, ptr(q), ptr(s), ptr(hout), ptr(az), 1, 3)
    before, after, delta = t(64, dtype=torch.bfloat16), t(64, dtype=torch.bfloat16), t(64)
    h3b.h3b_range_delta(before, after, delta, stream=3)
    assert last(rec, "h3b_range_delta") == (ptr(before), ptr(after), ptr(delta), 64, 3)
    h3b.h3b_range_apply(after, delta, stream=3)
    assert last(rec, "h3b_range_apply") == (ptr(after), ptr(delta), 64, 3)


def test_block_wrappers_pass_dims_weights_and_workspace_size(rec):
    dims = h3b.make_dims(1, 2, 16, 16, 256, 4, 64, 1024, (16, 24, 24))
    blk = {n: t(16) for n in h3b.WEIGHT_FIELDS}
    w = h3b.make_weights(blk)
    assert [getattr(w, n) for n in h3b.WEIGHT_FIELDS] == [ptr(blk[n]) for n in h3b.WEIGHT_FIELDS]
    c, x, ws = t(1, 256), t(512, 256, dtype=torch.bfloat16), t(1000, dtype=torch.uint8)
    h3b.h3b_block_forward(dims, w, c, x, ws, stream=5)
    args = last(rec, "h3b_block_forward")
    assert args[0]._obj is dims and args[1]._obj is w
    assert args[2:] == (ptr(c), ptr(x), ptr(ws), 1000, 5)
    h3b.h3b_blocks_forward(dims, [w, w, w], c, x, ws, stream=5)
    args = last(rec, "h3b_blocks_forward")
    assert len(args[1]) == 3 and args[2] == 3 and args[3:] == (ptr(c), ptr(x), ptr(ws), 1000, 5)
    assert [a.w1 for a in args[1]] == [ptr(blk["w1"])] * 3
    xs, delta = t(512, 256, dtype=torch.bfloat16), t(512 * 256)
    h3b.h3b_blocks_forward_cached(dims, [w, w], 0, 1, True, c, x, xs, delta, ws, stream=5)
    args = last(rec, "h3b_blocks_forward_cached")
    assert args[2:] == (2, 0, 1, 1, ptr(c), ptr(x), ptr(xs), ptr(delta), ptr(ws), 1000, 5)
    xm, ym = t(256, 256, dtype=torch.bfloat16), t(256, 256, dtype=torch.bfloat16)
    h3b.h3b_blocks_forward_reduced(dims, [w, w], 1, 2, c, x, xm, ym, ws, stream=5)
    args = last(rec, "h3b_blocks_forward_reduced")
    assert args[2:] == (2, 1, 2, ptr(c), ptr(x), ptr(xm), ptr(ym), ptr(ws), 1000, 5)
    h3b.h3b_token_pair(dims, x, xm, ym, stream=5)
    assert last(rec, "h3b_token_pair")[1:] == (ptr(x), ptr(xm), ptr(ym), 5)
    out = t(512, 256, dtype=torch.bfloat16)
    h3b.h3b_token_unpair(dims, x, xm, ym, out, stream=5)
    assert last(rec, "h3b_token_unpair")[1:] == (ptr(x), ptr(xm), ptr(ym), ptr(out), 5)
    qkv, o, am = t(3 * 512 * 256, dtype=torch.bfloat16), t(512, 256, dtype=torch.bfloat16), t(512)
    h3b.h3b_attention(dims, qkv, o, am, stream=5)
    assert last(rec, "h3b_attention")[1:] == (ptr(qkv), ptr(o), ptr(am), 5)
    A, sA, rope = t(512, 256, dtype=torch.int8), t(512), t(64, dtype=torch.uint8)
    h3b.h3b_qkv_projection(dims, A, sA, w, qkv, rope, stream=5)
    args = last(rec, "h3b_qkv_projection")
    assert (args[1], args[2], args[4], args[5], args[6]) == (ptr(A), ptr(sA), ptr(qkv), ptr(rope), 5)
    assert args[3]._obj is w


def test_stream_argument_forms(rec):
    A, W, Cout = t(16, 16, dtype=torch.int8), t(16, 16, dtype=torch.int8), t(16, 16, dtype=torch.int32)
    h3b.h3b_gemm_i8_s32(A, W, Cout, stream=0)
    assert last(rec, "h3b_gemm_i8_s32")[-1] == 0
    h3b.h3b_gemm_i8_s32(A, W, Cout, stream=0x1234)
    assert last(rec, "h3b_gemm_i8_s32")[-1] == 0x1234


def test_a_failing_status_raises_with_the_library_detail(monkeypatch):
    class Failing(Recorder):
        def __getattr__(self, name):
            if name == "h3b_last_error_detail":
                return lambda: b"N must be a multiple of 16"
            return lambda *a: -2
    monkeypatch.setattr(h3b, "_LIB", Failing())
    with pytest.raises(h3b.H3BError) as e:
        h3b.h3b_gemm_i8_s32(t(16, 16, dtype=torch.int8), t(24, 16, dtype=torch.int8), t(16, 24, dtype=torch.int32),
                            stream=0)
    assert e.value.status == -2 and "multiple of 16" in str(e.value) and "H3B_ERR_SHAPE" in str(e.value)


def test_remaining_wrappers(rec):
    dims = h3b.make_dims(2, 2, 16, 16, 256, 4, 64, 1024, (16, 24, 24))
    w_ada, b_ada, c, mod = t(1536, 256, dtype=torch.bfloat16), t(1536), t(2, 256), t(2, 1536)
    h3b.h3b_adaln_modulation(dims, w_ada, b_ada, c, mod, stream=9)
    args = last(rec, "h3b_adaln_modulation")
    assert args[0]._obj is dims and args[1:] == (ptr(w_ada), ptr(b_ada), ptr(c), ptr(mod), 9)
    w = h3b.make_weights({"w1": t(4)})
    assert w.w_ada is None and w.w1 is not None  # missing names are NULL
    x = t(1024, 256, dtype=torch.bfloat16)
    h3b.h3b_block_forward_noalloc(dims, w, c, x, stream=9)
    args = last(rec, "h3b_block_forward_noalloc")
    assert args[1]._obj is w and args[2:] == (ptr(c), ptr(x), 9)
    ws = t(4096, dtype=torch.uint8)
    g = h3b.h3b_graph_capture_blocks(dims, [w, w], c, x, ws)
    args = last(rec, "h3b_graph_capture_blocks")
    assert args[2:6] == (2, ptr(c), ptr(x), ptr(ws)) and args[6] == 4096
    g.handle = None  # the stand-in returned no graph; nothing to destroy
    assert h3b.h3b_device_error(clear=False) == 0
    assert last(rec, "h3b_device_error")[1] == 0
