"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes as C
import os
import re

import pytest
import torch

from video_diffusion_transformer_adaln_b200 import build, h3b, synth
from video_diffusion_transformer_adaln_b200.runtime import dims_of

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "h3b.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return h3b.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(h3b_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 19
    for n in names:
        assert hasattr(L, n), n
    # and the binding wraps each of them under the same name
    for n in names:
        assert hasattr(h3b, n) or n in ("h3b_status_string", "h3b_last_error_detail"), n


def test_status_strings(L):
    for code in h3b.STATUS:
        assert h3b.status_string(code)


def _dims(**kw):
    wl = synth.WORKLOADS["d256_L512"]
    d = dims_of(wl)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_size_host_only(L):
    n = h3b.h3b_workspace_size(_dims())
    wl = synth.WORKLOADS["d256_L512"]
    R, D, F = wl.L, wl.d, wl.d_ff
    # at least the int8 activations (R x F) and the bf16 Q/K/V + attention output (8 R D bytes)
    assert n >= R * F + 8 * R * D
    big = h3b.h3b_workspace_size(dims_of(synth.WORKLOADS["d5120_L18432"]))
    assert 1.0e9 < big < 1.3e9


@pytest.mark.parametrize("field,value", [("head_dim", 96), ("d", 300), ("d_ff", 1000), ("rope_t", 15),
                                         ("B", 0), ("W", 0), ("n_heads", 3), ("B", 9)])
def test_bad_dims_are_rejected(L, field, value):
    with pytest.raises(h3b.H3BError) as e:
        h3b.h3b_workspace_size(_dims(**{field: value}))
    assert e.value.status in (-1, -2)


def test_block_forward_validation_order(L):
    d = _dims()
    w = h3b.BlockWeights()
    for n in h3b.WEIGHT_FIELDS:
        setattr(w, n, 0x10000)
    x = 0x20000
    c = 0x30000
    ws = 0x40000
    need = h3b.h3b_workspace_size(d)
    # NULL x
    assert L.h3b_block_forward(C.byref(d), C.byref(w), c, None, ws, need, None) == -1
    # misaligned x / workspace
    assert L.h3b_block_forward(C.byref(d), C.byref(w), c, x + 2, ws, need, None) == -3
    assert L.h3b_block_forward(C.byref(d), C.byref(w), c, x, ws + 16, need, None) == -3
    # workspace too small
    assert L.h3b_block_forward(C.byref(d), C.byref(w), c, x, ws, need - 1, None) == -4
    # bad shape
    bad = _dims(d_ff=100)
    assert L.h3b_block_forward(C.byref(bad), C.byref(w), c, x, ws, need, None) == -2
    # missing or misaligned weight (placeholder pointers are never dereferenced:
    # every host check runs before the device query and any launch)
    w.w1 = None
    assert L.h3b_block_forward(C.byref(d), C.byref(w), c, x, ws, need, None) == -1
    w.w1 = 0x10008
    assert L.h3b_block_forward(C.byref(d), C.byref(w), c, x, ws, need, None) == -3


def test_multi_block_entry_points_check_every_block_on_the_host(L):
    d = _dims()
    blocks = (h3b.BlockWeights * 3)()
    for b in blocks:
        for n in h3b.WEIGHT_FIELDS:
            setattr(b, n, 0x10000)
    blocks[2].s2 = None  # the last block's W2 scales are missing
    x, c, ws, xm, ym = 0x20000, 0x30000, 0x40000, 0x50000, 0x60000
    need = h3b.h3b_workspace_size(d)
    assert L.h3b_blocks_forward(C.byref(d), blocks, 3, c, x, ws, need, None) == -1
    assert L.h3b_blocks_forward(C.byref(d), blocks, -1, c, x, ws, need, None) == -1
    assert L.h3b_blocks_forward(C.byref(d), None, 3, c, x, ws, need, None) == -1
    # reduced pass: range, pairing shape and buffers
    assert L.h3b_blocks_forward_reduced(C.byref(d), blocks, 3, 1, 2, c, x, xm, ym, ws, need, None) == -1
    assert L.h3b_blocks_forward_reduced(C.byref(d), blocks, 3, 2, 1, c, x, xm, ym, ws, need, None) == -1
    assert L.h3b_blocks_forward_reduced(C.byref(d), blocks, 3, 1, 2, c, x, xm, None, ws, need, None) == -1
    assert L.h3b_blocks_forward_reduced(C.byref(d), blocks, 3, 1, 2, c, x, xm, ym + 8, ws, need, None) == -3
    # xm is not used (the unpairing recomputes the merged input): NULL or unaligned is accepted,
    # and the call goes on to the per-block weight check
    assert L.h3b_blocks_forward_reduced(C.byref(d), blocks, 3, 1, 2, c, x, None, ym, ws, need, None) == -1
    assert L.h3b_blocks_forward_reduced(C.byref(d), blocks, 3, 1, 2, c, x, xm + 8, ym, ws, need, None) == -1
    odd = _dims(W=15)
    need_odd = h3b.h3b_workspace_size(odd)
    assert L.h3b_blocks_forward_reduced(C.byref(odd), blocks, 3, 1, 2, c, x, xm, ym, ws, need_odd, None) == -2
    # cached pass: range, buffers, and the same per-block weight check
    assert L.h3b_blocks_forward_cached(C.byref(d), blocks, 3, 0, 4, 1, c, x, 0x70000, 0x80000, ws, need,
                                       None) == -1
    assert L.h3b_blocks_forward_cached(C.byref(d), blocks, 3, 0, 2, 1, c, x, None, 0x80000, ws, need,
                                       None) == -1
    assert L.h3b_blocks_forward_cached(C.byref(d), blocks, 3, 0, 2, 1, c, x, 0x70000, 0x80000, ws, need,
                                       None) == -1


@pytest.mark.parametrize("T,H,W", [(2 ** 31 - 1, 2 ** 31 - 1, 2 ** 31 - 1), (65536, 65536, 2),
                                   (2 ** 20, 2 ** 11, 1), (1, 2, 2 ** 30), (2 ** 16, 2 ** 16, 2 ** 16)])
def test_grids_of_2_31_tokens_or_more_are_rejected_without_overflow(L, T, H, W):
    # Extents whose product wraps a 64-bit integer, or lands exactly on 2^31, must
    # not pass the size checks of any entry point that takes the grid.
    d = _dims(T=T, H=H, W=W)
    with pytest.raises(h3b.H3BError) as e:
        h3b.h3b_workspace_size(d)
    assert e.value.status == -2
    full = _dims(T=T, H=H, W=W + (W & 1))
    assert L.h3b_token_pair(C.byref(full), 0x1000, 0x2000, None, None) == -2
    assert L.h3b_token_unpair(C.byref(full), 0x1000, 0x2000, 0x3000, 0x4000, None) == -2
    assert L.h3b_attention(C.byref(d), 0x1000, 0x2000, 0x3000, None) == -2


def test_batch_times_grid_limit(L):
    # B * L must stay below 2^31 even when L alone is below it.
    big = _dims(B=2, T=2 ** 15, H=2 ** 10, W=2 ** 5)  # L = 2^30, B*L = 2^31
    with pytest.raises(h3b.H3BError):
        h3b.h3b_workspace_size(big)
    assert L.h3b_attention(C.byref(big), 0x1000, 0x2000, 0x3000, None) == -2
    assert L.h3b_token_pair(C.byref(big), 0x1000, 0x2000, None, None) == -2


def test_token_pair_validation(L):
    full = _dims(W=15)
    assert L.h3b_token_pair(C.byref(full), 0x1000, 0x2000, None, None) == -2
    full = _dims()
    assert L.h3b_token_pair(C.byref(full), None, 0x2000, None, None) == -1
    assert L.h3b_token_pair(C.byref(full), 0x1008, 0x2000, None, None) == -3


def test_gemm_validation(L):
    assert L.h3b_gemm_i8_s32(0x1000, 0x2000, 0x3000, 128, 24, 128, None) == -2   # N % 16
    assert L.h3b_gemm_i8_s32(0x1000, 0x2000, 0x3000, 128, 256, 100, None) == -2  # K % 16
    assert L.h3b_gemm_i8_s32(0x1001, 0x2000, 0x3000, 128, 256, 128, None) == -3
    assert L.h3b_gemm_i8_s32(None, 0x2000, 0x3000, 128, 256, 128, None) == -1


def test_empty_problems_return_ok_after_their_size_checks(L):
    # An empty problem returns OK once its sizes are checked: NULL pointers are
    # accepted, the device is not queried (so this holds on a host without a GPU
    # too) and nothing is launched.
    assert L.h3b_gemm_i8_s32(None, None, None, 0, 256, 128, None) == 0
    assert L.h3b_gemm_i8_dequant(None, None, None, None, None, None, 0, 256, 128, None) == 0
    assert L.h3b_gemm_i8_gelu(None, None, None, None, None, None, None, 0, 256, 128, None) == 0
    assert L.h3b_gemm_i8_gated_residual(None, None, None, None, None, None, 1, 0, None, 0, 256, 128, None) == 0
    assert L.h3b_gemm_bf16_gated_residual(None, None, None, None, 1, 0, None, 0, 256, 128, None) == 0
    assert L.h3b_quantize_rows(None, 0, 256, None, None, None, None) == 0
    assert L.h3b_quantize_weights(None, 0, 256, None, None, None) == 0
    assert L.h3b_ln_modulate_quantize(None, 0, 256, 1e-6, None, None, 1, 0, None, None, None, None, 1, None) == 0
    assert L.h3b_range_delta(None, None, None, 0, None) == 0
    assert L.h3b_range_apply(None, None, 0, None) == 0
    # the sizes themselves are still checked
    assert L.h3b_gemm_i8_s32(None, None, None, 0, 24, 128, None) == -2
    assert L.h3b_gemm_i8_s32(None, None, None, -1, 256, 128, None) == -2
    assert L.h3b_quantize_rows(None, 0, 17, None, None, None, None) == -2
    assert L.h3b_ln_modulate_quantize(None, 0, 300, 1e-6, None, None, 1, 0, None, None, None, None, 1, None) == -2
    assert L.h3b_ln_modulate_quantize(None, 0, 256, 1e-6, None, None, 0, 0, None, None, None, None, 1, None) == -1
    assert L.h3b_range_apply(None, None, 4, None) == -2


def test_step_arguments_are_checked_before_the_device_query(L):
    # Every host check of a step entry point runs before the device is queried, so
    # these are reported as argument errors even on a host without a GPU.
    A, W, out = 0x10000, 0x20000, 0x30000
    assert L.h3b_gemm_i8_dequant(A, None, W, 0x40000, None, out, 128, 256, 128, None) == -1      # sA NULL
    assert L.h3b_gemm_i8_dequant(A, 0x40000, W, 0x40008, None, out, 128, 256, 128, None) == -3  # sW misaligned
    assert L.h3b_gemm_i8_gelu(A, 0x40000, W, 0x40000, None, out, None, 128, 256, 128, None) == -1  # absmax NULL
    assert L.h3b_gemm_i8_gated_residual(A, 0x40000, W, 0x40000, None, 0x50008, 1, 0, out,
                                        128, 256, 128, None) == -3                                 # gate misaligned
    assert L.h3b_gemm_i8_gated_residual(A, 0x40000, W, 0x40000, None, 0x50000, 0, 0, out,
                                        128, 256, 128, None) == -1                                 # rows_per_item
    assert L.h3b_gemm_bf16_gated_residual(A, W, None, None, 1, 0, out, 128, 256, 128, None) == -1  # gate NULL
    assert L.h3b_gemm_bf16_gated_residual(A, W, None, 0x50000, 1, 6, out, 128, 256, 128, None) == -1  # stride % 4
    assert L.h3b_ln_modulate_quantize(0x1000, 8, 256, 1e-6, None, 0x2000, 8, 0, 0x3000, 0x4000, None, None, 1,
                                      None) == -1                                                  # shift NULL
    assert L.h3b_ln_modulate_quantize(0x1000, 8, 256, 1e-6, 0x2000, 0x2000, 8, 0, 0x3000, 0x4000, 0x5008, None, 1,
                                      None) == -3                                                  # h_out misaligned
    assert L.h3b_quantize_rows(0x1000, 8, 256, None, None, 0x2000, None) == -1                     # q NULL
    assert L.h3b_range_delta(0x1000, 0x2008, 0x3000, 64, None) == -3                                # after misaligned


@pytest.mark.skipif(torch.cuda.is_available(), reason="would launch on the placeholder pointers")
def test_valid_call_without_a_b200_launches_nothing(L):
    # On a host without a compute-capability-10.0 device the call stops at the
    # device query with ARCH or CUDA status; it never reports success.
    assert L.h3b_quantize_weights(0x1000, 4, 16, 0x2000, 0x3000, None) in (-5, -6)


def test_reuse_and_graph_validation(L):
    d = _dims()
    w = h3b.BlockWeights()
    for n in h3b.WEIGHT_FIELDS:
        setattr(w, n, 0x10000)
    arr = (h3b.BlockWeights * 4)(w, w, w, w)
    x, c, ws, xs, dl = 0x20000, 0x30000, 0x40000, 0x50000, 0x60000
    need = h3b.h3b_workspace_size(d)
    f = L.h3b_blocks_forward_cached
    # range outside [0, n_blocks] or reversed; a missing delta or x_save where the range needs it
    assert f(C.byref(d), arr, 4, 3, 2, 1, c, x, xs, dl, ws, need, None) == -1
    assert f(C.byref(d), arr, 4, 1, 5, 1, c, x, xs, dl, ws, need, None) == -1
    assert f(C.byref(d), arr, 4, 1, 3, 0, c, x, None, None, ws, need, None) == -1
    assert f(C.byref(d), arr, 4, 1, 3, 1, c, x, None, dl, ws, need, None) == -1
    assert f(C.byref(d), arr, 4, 1, 3, 1, c, x, xs + 4, dl, ws, need, None) == -3
    # the elementwise steps alone
    assert L.h3b_range_delta(0x1000, 0x2000, 0x3000, 12, None) == -2
    assert L.h3b_range_delta(None, 0x2000, 0x3000, 16, None) == -1
    assert L.h3b_range_apply(0x1008, 0x3000, 16, None) == -3
    # bf16 gated residual GEMM: gate and its stride are checked first
    assert L.h3b_gemm_bf16_gated_residual(0x1000, 0x2000, None, None, 1, 256, 0x3000, 128, 256, 128, None) == -1
    assert L.h3b_gemm_bf16_gated_residual(0x1000, 0x2000, None, 0x4000, 0, 256, 0x3000, 128, 256, 128, None) == -1
    # graph handles
    assert L.h3b_graph_capture_blocks(C.byref(d), arr, 4, c, x, ws, need, None) == -1
    assert L.h3b_graph_launch(None, None) == -1
    assert L.h3b_graph_kernel_count(None) == 0
    L.h3b_graph_destroy(None)  # a no-op


def test_bounded_wait_hook_validation(L):
    out = C.c_int(-1)
    assert L.h3b_test_bounded_wait(10, C.byref(out)) == -1  # below 1 us
    assert L.h3b_test_bounded_wait(2_000_000_000, C.byref(out)) == -1  # above 1 s
    assert L.h3b_test_bounded_wait(1_000_000, None) == -1
    assert out.value == -1


_I32 = (-2 ** 31, 2 ** 31 - 1)


def _int_field(lo, hi):
    from hypothesis import strategies as st
    # mostly valid-looking values, plus edges and arbitrary int32
    return st.one_of(st.integers(lo, hi), st.sampled_from([0, -1, 1, 2 ** 31 - 1, -2 ** 31, 2 ** 16, 2 ** 30]),
                     st.integers(*_I32))


def test_dims_checks_accept_exactly_the_documented_shapes(L):
    """Property test of the host dims check (h3b_workspace_size): any int values either give
    an error status, or satisfy every documented limit; nothing crashes or overflows."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    @settings(max_examples=400, deadline=None, suppress_health_check=list(HealthCheck))
    @given(B=_int_field(1, 9), T=_int_field(1, 64), H=_int_field(1, 64), W=_int_field(1, 64),
           heads=_int_field(1, 64), hd=st.sampled_from([64, 128, 96, 0, -64]), dff=_int_field(256, 40000),
           split=st.sampled_from([(16, 24, 24), (32, 48, 48), (15, 25, 24), (0, 0, 64), (64, 64, 0)]))
    def check(B, T, H, W, heads, hd, dff, split):
        d = _dims(B=B, T=T, H=H, W=W, n_heads=heads, head_dim=hd, d=heads * hd if abs(heads * hd) < 2 ** 31 else 0,
                  d_ff=dff, rope_t=split[0], rope_h=split[1], rope_w=split[2])
        n = C.c_size_t(0)
        st_ = L.h3b_workspace_size(C.byref(d), C.byref(n))
        if st_ == 0:
            Lt = d.T * d.H * d.W
            assert 1 <= d.B <= 8 and min(d.T, d.H, d.W) >= 1 and d.B * Lt < 2 ** 31
            assert d.head_dim in (64, 128) and d.d == d.n_heads * d.head_dim and d.d % 256 == 0 and d.d <= 8192
            assert d.d_ff % 256 == 0 and 256 <= d.d_ff <= 32768 and d.B * Lt * d.d_ff <= 2 ** 40
            assert d.rope_t + d.rope_h + d.rope_w == d.head_dim
            assert n.value >= d.B * Lt * max(d.d, d.d_ff)
        else:
            assert st_ in (-1, -2)
    check()


def test_head_count_overflow_is_rejected(L):
    # n_heads * head_dim wraps a 32-bit int to 0 here; d = 0 must not pass as "a multiple of 256"
    d = _dims(n_heads=2 ** 30, head_dim=64, d=0)
    with pytest.raises(h3b.H3BError):
        h3b.h3b_workspace_size(d)
    with pytest.raises(h3b.H3BError):
        h3b.h3b_workspace_size(_dims(d=0, n_heads=0))


def test_gemm_sizes_property(L):
    """Any int M, N, K: either an error before any device query, or sizes within the
    documented rules (here checked with NULL operands, so a passing size reports the
    NULL pointer, or OK for M == 0)."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st
    ints = st.one_of(st.integers(-64, 4096), st.integers(*_I32),
                     st.sampled_from([0, 16, 2 ** 31 - 16, 2 ** 20 * 16, 2 ** 24]))

    @settings(max_examples=400, deadline=None, suppress_health_check=list(HealthCheck))
    @given(M=ints, N=ints, K=ints)
    def check(M, N, K):
        st_ = L.h3b_gemm_i8_s32(None, None, None, M, N, K, None)
        ok_sizes = M >= 0 and N >= 16 and N % 16 == 0 and K >= 16 and K % 16 == 0 and \
            max(M * N, M * K, N * K) <= 2 ** 40
        if not ok_sizes:
            assert st_ == -2
        else:
            assert st_ == (0 if M == 0 else -1)
    check()


def test_step_size_checks_property(L):
    """Arbitrary int32 sizes for the row, pairing and attention entry points, with NULL
    pointers: a size outside the documented rules gives SHAPE (or ARG for the item
    layout); a legal size gives OK when the problem is empty, else the NULL-pointer ARG."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st
    ints = st.one_of(st.integers(-4, 9000), st.integers(*_I32), st.sampled_from([0, 8, 16, 256, 2 ** 30, 2 ** 31 - 1]))
    cfg = settings(max_examples=300, deadline=None, suppress_health_check=list(HealthCheck))

    @cfg
    @given(rows=ints, cols=ints)
    def quant(rows, cols):
        st_ = L.h3b_quantize_rows(None, rows, cols, None, None, None, None)
        if rows < 0 or cols < 16 or cols % 16:
            assert st_ == -2
        else:
            assert st_ == (0 if rows == 0 else -1)
    quant()

    @cfg
    @given(rows=ints, d=ints, rpi=ints, ms=ints)
    def ln(rows, d, rpi, ms):
        st_ = L.h3b_ln_modulate_quantize(None, rows, d, 1e-6, None, None, rpi, ms, None, None, None, None, 1, None)
        if rows < 0 or d < 256 or d % 256 or d > 8192:
            assert st_ == -2
        elif rpi < 1 or ms < 0 or ms % 4:
            assert st_ == -1
        else:
            assert st_ == (0 if rows == 0 else -1)
    ln()

    @cfg
    @given(B=ints, T=ints, H=ints, W=ints, d=ints)
    def pair(B, T, H, W, d):
        full = _dims(B=B, T=T, H=H, W=W, d=d)
        st_ = L.h3b_token_pair(C.byref(full), None, None, None, None)
        legal = B >= 1 and T >= 1 and H >= 1 and W >= 2 and W % 2 == 0 and 8 <= d <= 65536 and d % 8 == 0 and \
            B * T * H * W < 2 ** 31
        assert st_ == (-1 if legal else -2)
    pair()

    @cfg
    @given(B=ints, T=ints, H=ints, W=ints, nh=ints, hd=st.sampled_from([64, 128, 32, 0]))
    def attn(B, T, H, W, nh, hd):
        dims = _dims(B=B, T=T, H=H, W=W, n_heads=nh, head_dim=hd)
        st_ = L.h3b_attention(C.byref(dims), None, None, None, None)
        legal = min(B, T, H, W, nh) >= 1 and hd in (64, 128) and B * nh <= 65535 and B * T * H * W < 2 ** 31
        assert st_ == (-1 if legal else -2)
    attn()
