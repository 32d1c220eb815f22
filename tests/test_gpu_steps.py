"""Step-by-step parity of the CUDA kernels against the CPU oracle, on the same
seeded inputs (every input is generated on the host; no oracle input comes
from the GPU except where a test re-quantizes the GPU's own bf16 quantizer
input to check the bit-exact decision).

Bars: integer/byte work bit-exact; bf16 outputs within the rounding the kernel
performs (stated per test)."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import (bf16_f64, bf16_dev, bf16_host, bf16_ulp_diff, no_device_error, oracle_weights, rel_l2,
                         require_gpu, to_dev)
from video_diffusion_transformer_adaln_b200 import h3b, synth
from video_diffusion_transformer_adaln_b200.runtime import DeviceBlock, dims_of, quantize_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    h3b.h3b_device_error(clear=True)
    yield


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- quantizers

@pytest.mark.parametrize("rows,cols", [(1, 16), (768, 256), (256, 1024), (37, 8192), (1000, 48)])
def test_weight_quantizer_bit_exact(rows, cols):
    r = _rng(rows * 7 + cols)
    w = (r.standard_normal((rows, cols)) * r.uniform(0.001, 10, (rows, 1))).astype(np.float32)
    w[0, :3] = [127.0, 2.5, -3.5] if cols >= 3 else w[0, :3]
    if rows > 3:
        w[3] = 0.0
    q, s = quantize_weight(to_dev(w))
    qo, so = O.quantize_rows(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)
    no_device_error()


@pytest.mark.parametrize("rows,cols,with_absmax", [(33, 1024, False), (33, 1024, True), (512, 256, False),
                                                   (129, 20480, True), (5, 16, False), (37, 5120, True)])
def test_row_quantizer_bit_exact(rows, cols, with_absmax):
    r = _rng(rows + cols)
    hf0 = (r.standard_normal((rows, cols)) * r.uniform(0.01, 30, (rows, 1))).astype(np.float32)
    if rows > 3:  # tiny rows: scale below 2^-100 (the division for every element), then subnormal
        hf0[2] *= np.float32(1e-33)
        hf0[3] *= np.float32(1e-37)
    h = synth.f32_to_bf16_bits(hf0)
    h[1] = 0  # an all-zero row
    hf = synth.bf16_bits_to_f32(h)
    q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    am = to_dev(np.abs(hf).max(axis=1).astype(np.float32)) if with_absmax else None
    h3b.h3b_quantize_rows(bf16_dev(h), q, s, absmax=am)
    qo, so = O.quantize_rows(hf)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)
    no_device_error()


@pytest.mark.parametrize("with_absmax", [False, True])
def test_row_quantizer_every_bf16_value(with_absmax):
    """Every finite bf16 value up to a row's absmax, for 64 random scales and for
    scale 1 (absmax 127: exact half-integer ties): the int8 decision matches the
    oracle's binary32 division bit for bit, with the absmax found by the kernel
    and with it given (the pass that requantizes O and G)."""
    allb = np.arange(0, 0x7F80, dtype=np.uint16)  # non-negative finite bf16 bit patterns
    pos = synth.bf16_bits_to_f32(allb)
    r = _rng(77)
    amaxes = np.concatenate([[127.0], r.uniform(0.5, 3000.0, 63)]).astype(np.float32)
    amaxes = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(amaxes))
    rows = []
    for a in amaxes:
        vals = pos[pos <= a]
        row = np.concatenate([[a], vals, -vals])
        rows.append(row)
    cols = max(len(x) for x in rows)
    cols += (-cols) % 16
    h = np.zeros((len(rows), cols), np.float32)
    for i, row in enumerate(rows):
        h[i, :len(row)] = row
    hb = synth.f32_to_bf16_bits(h)
    q = torch.empty((len(rows), cols), dtype=torch.int8, device="cuda")
    s = torch.empty(len(rows), dtype=torch.float32, device="cuda")
    hf = synth.bf16_bits_to_f32(hb)
    am = to_dev(np.abs(hf).max(axis=1).astype(np.float32)) if with_absmax else None
    h3b.h3b_quantize_rows(bf16_dev(hb), q, s, absmax=am)
    qo, so = O.quantize_rows(hf)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)
    no_device_error()


@pytest.mark.parametrize("rows,d,items", [(512, 256, 1), (37, 2048, 1), (64, 5120, 1), (96, 256, 3), (8, 8192, 2),
                                           (40, 768, 2), (19, 3072, 1), (16, 5376, 1), (23, 7936, 1)])
def test_ln_modulate_quantize(rows, d, items):
    r = _rng(rows * d)
    wl = synth.WORKLOADS["d256_L512"].with_(d=d, n_heads=d // 64)
    xf = (r.standard_normal((rows, d)).astype(np.float32) *
          np.where(np.isin(np.arange(d), synth.outlier_channels(wl)), 16, 1).astype(np.float32))
    if rows > 2:  # rows with zero variance: a constant row and an all-zero row (h = shift)
        xf[rows // 2] = 3.0
        xf[rows - 1] = 0.0
    x = synth.f32_to_bf16_bits(xf)
    mod = r.standard_normal((items, 6 * d)).astype(np.float32)
    rpi = (rows + items - 1) // items
    q = torch.empty((rows, d), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    h = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    az = torch.full((rows,), 7.0, dtype=torch.float32, device="cuda")
    md = to_dev(mod)
    h3b.h3b_ln_modulate_quantize(bf16_dev(x), rows, d, 1e-6, md[:, 3 * d:], md[:, 4 * d:], rpi, 6 * d, q, s,
                                 h_out=h, absmax_zero=az)
    hg = bf16_host(h)
    qg, sg = q.cpu().numpy(), s.cpu().numpy()
    assert np.all(az.cpu().numpy() == 0)
    # (1) the bf16 quantizer input matches the oracle's fp64 LN + modulation to one
    #     bf16 ulp of the value (at most 2^-7 |h|), plus the fp32 error of y*(1+scale)+shift when
    #     the two terms nearly cancel (bounded relative to the row's magnitude)
    y = O.layernorm(bf16_f64(x), 1e-6)
    ho = np.empty_like(hg)
    for i in range(rows):
        it = i // rpi
        ho[i] = O.modulate_bf16(y[i:i + 1], mod[it, 3 * d:4 * d].astype(np.float64),
                                mod[it, 4 * d:5 * d].astype(np.float64))[0]
    hgd, hod = bf16_f64(hg), bf16_f64(ho)
    bound = 2.0 ** -7 * np.abs(hod) + 2.0 ** -16 * np.abs(hod).max(axis=1, keepdims=True)
    assert np.all(np.abs(hgd - hod) <= bound)
    assert (hg != ho).mean() < 0.02
    # (2) codes and scales against the oracle's quantization of its own h. Rows whose h equals
    #     the oracle's match bit for bit. Elsewhere each h element, and so the row absmax A,
    #     differs by at most 2^-7 relative plus 2^-16 A (1); the scale then moves by at most
    #     2^-7 + 2^-15 relative, v/s by at most 127 * (2^-6 + 2^-15 + 2^-16) / (1 - 2^-7) < 2.01,
    #     and a rounded code by at most 3.
    qo, so = O.quantize_rows(hod.astype(np.float32))
    same = np.all(hg == ho, axis=1)
    assert np.array_equal(qg[same], qo[same]) and np.array_equal(sg[same], so[same])
    assert np.all(np.abs(qg.astype(np.int32) - qo.astype(np.int32)) <= 3)
    assert np.all(np.abs(sg.astype(np.float64) - so) <= (2.0 ** -7 + 2.0 ** -15) * so)
    # (3) the kernel's int8 decision on its own h is the binary32 rule, bit for bit: s = absmax/127
    #     and q = rint(h/s) in float32, restated here in numpy (the oracle only sees seeded inputs)
    hf = synth.bf16_bits_to_f32(hg)
    amax = np.abs(hf).max(axis=1)
    sc = amax / np.float32(127)
    with np.errstate(divide="ignore", invalid="ignore"):
        qn = np.where(amax[:, None] > 0, np.clip(np.rint(hf / sc[:, None]), -127, 127), 0).astype(np.int8)
    assert np.array_equal(sg, sc) and np.array_equal(qg, qn)
    no_device_error()


def test_adaln_modulation():
    wl = synth.WORKLOADS["d2048_L4096"].with_(B=2)
    raw = synth.block_weights(wl)
    c = synth.cond(wl)
    mod = torch.empty((2, 6 * wl.d), dtype=torch.float32, device="cuda")
    h3b.h3b_adaln_modulation(dims_of(wl), bf16_dev(raw["w_ada"]), to_dev(raw["b_ada"]), to_dev(c), mod)
    for b in range(2):
        ref = O.adaln_linear(raw["w_ada"], raw["b_ada"], c[b])
        assert np.max(np.abs(mod[b].cpu().numpy() - ref)) <= 1e-5 * np.max(np.abs(ref)) + 1e-6
    no_device_error()


# ----------------------------------------------------------------------------- int8 GEMM

@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (512, 768, 256), (300, 272, 144), (1, 16, 16),
                                   (1024, 1536, 2048), (256, 512, 20480), (129, 6144, 2048)])
def test_gemm_i8_s32_bit_exact(M, N, K):
    r = _rng(M + N + K)
    A = r.integers(-128, 128, (M, K), dtype=np.int8)
    W = r.integers(-128, 128, (N, K), dtype=np.int8)
    C_ = torch.empty((M, N), dtype=torch.int32, device="cuda")
    h3b.h3b_gemm_i8_s32(to_dev(A), to_dev(W), C_)
    assert np.array_equal(C_.cpu().numpy(), O.gemm_i8(A, W))
    no_device_error()


def _quant_operands(M, N, K, seed):
    r = _rng(seed)
    a = (r.standard_normal((M, K)) * r.uniform(0.1, 5, (M, 1))).astype(np.float32)
    w = (r.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32)
    qa, sa = O.quantize_rows(a)
    qw, sw = O.quantize_rows(w)
    bias = r.standard_normal(N).astype(np.float32) * 0.1
    return qa, sa, qw, sw, bias


@pytest.mark.parametrize("M,N,K", [(512, 768, 256), (200, 1040, 512)])
def test_gemm_i8_dequant(M, N, K):
    qa, sa, qw, sw, bias = _quant_operands(M, N, K, 11)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h3b.h3b_gemm_i8_dequant(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), to_dev(bias), out)
    ref = O.dequant(O.gemm_i8(qa, qw), sa, sw, bias)
    ulp = bf16_ulp_diff(bf16_host(out), O.bf16_round(ref))
    assert ulp.max() <= 1
    no_device_error()


@pytest.mark.parametrize("M,N,K", [(512, 1024, 256), (77, 8192, 2048), (77, 1040, 256)])
def test_gemm_i8_gelu(M, N, K):
    qa, sa, qw, sw, bias = _quant_operands(M, N, K, 12)
    g = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(M, dtype=torch.float32, device="cuda")
    h3b.h3b_gemm_i8_gelu(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), to_dev(bias), g, am)
    gg = bf16_host(g)
    ref = O.gelu_tanh(O.dequant(O.gemm_i8(qa, qw), sa, sw, bias))
    assert rel_l2(bf16_f64(gg), ref) < 4e-3
    assert np.max(np.abs(bf16_f64(gg) - ref)) <= 2 ** -7 * np.max(np.abs(ref)) + 1e-3
    # the reported absmax is exactly the max |g| of the written bf16 row
    assert np.array_equal(am.cpu().numpy(), np.abs(bf16_f64(gg)).max(axis=1).astype(np.float32))
    no_device_error()


@pytest.mark.parametrize("M,N,K,items", [(512, 256, 256, 1), (256, 2048, 8192, 2), (100, 512, 1024, 1),
                                         (100, 512, 1024, 3), (100, 272, 160, 3)])
def test_gemm_i8_gated_residual(M, N, K, items):
    """items=3 over 100 rows gives 34 rows per item, so some warps' 32 rows straddle two
    items and read their gates row by row instead of from the staged per-item copy.
    N=272 ends in a half-filled 32-column chunk: its x loads and its TMA-stored box are
    cut at N."""
    qa, sa, qw, sw, bias = _quant_operands(M, N, K, 13)
    r = _rng(14)
    x = synth.f32_to_bf16_bits(r.standard_normal((M, N)).astype(np.float32))
    gate = r.standard_normal((items, 3 * N)).astype(np.float32)
    rpi = (M + items - 1) // items
    xd = bf16_dev(x)
    gd = to_dev(gate)
    h3b.h3b_gemm_i8_gated_residual(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), to_dev(bias), gd[:, N:], rpi,
                                   3 * N, xd)
    y = O.dequant(O.gemm_i8(qa, qw), sa, sw, bias)
    ref = np.empty((M, N))
    for i in range(M):
        ref[i] = O.gated_residual(bf16_f64(x[i:i + 1]), y[i:i + 1], gate[i // rpi, N:2 * N])[0]
    # one bf16 rounding of the result, plus the fp32 error of x + gate*y when the
    # two terms nearly cancel (relative to the terms' magnitude)
    got = bf16_f64(bf16_host(xd))
    terms = np.abs(bf16_f64(x)) + np.abs(np.stack([gate[i // rpi, N:2 * N] for i in range(M)]) * y)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * terms + 1e-30)
    # a zero gate leaves x bit-identical
    xd2 = bf16_dev(x)
    h3b.h3b_gemm_i8_gated_residual(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), to_dev(bias),
                                   torch.zeros((items, N), device="cuda"), rpi, N, xd2)
    assert np.array_equal(bf16_host(xd2), x)
    no_device_error()


@pytest.mark.parametrize("M,N,K,items", [(512, 256, 256, 1), (256, 2048, 2048, 2), (100, 512, 1040, 1),
                                         (100, 512, 1040, 3)])
def test_gemm_bf16_gated_residual(M, N, K, items):
    """bf16 output projection (the block's Wo when wo_bf16 is set) with the gated residual."""
    r = _rng(M + N + K)
    a = synth.f32_to_bf16_bits((r.standard_normal((M, K)) * r.uniform(0.1, 3, (M, 1))).astype(np.float32))
    w = synth.f32_to_bf16_bits((r.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    bias = r.standard_normal(N).astype(np.float32) * 0.1
    x = synth.f32_to_bf16_bits(r.standard_normal((M, N)).astype(np.float32))
    gate = r.standard_normal((items, 2 * N)).astype(np.float32)
    rpi = (M + items - 1) // items
    xd = bf16_dev(x)
    gd = to_dev(gate)
    h3b.h3b_gemm_bf16_gated_residual(bf16_dev(a), bf16_dev(w), to_dev(bias), gd[:, N:], rpi, 2 * N, xd)
    ad, wd = bf16_f64(a), bf16_f64(w)
    y = O.gemm_f64(ad, wd) + bias
    g = np.stack([gate[i // rpi, N:] for i in range(M)])
    ref = bf16_f64(x) + g * y
    got = bf16_f64(bf16_host(xd))
    # one bf16 rounding of the result; fp32 accumulation over K (|error| <= K 2^-24 sum|a w|)
    # and the fp32 error of x + gate*y relative to the terms' magnitude
    absum = np.abs(ad) @ np.abs(wd).T + np.abs(bias)
    terms = np.abs(bf16_f64(x)) + np.abs(g * y)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * terms + K * 2.0 ** -24 * np.abs(g) * absum + 1e-30
    assert np.all(np.abs(got - ref) <= bound)
    # a zero gate leaves x bit-identical
    xd2 = bf16_dev(x)
    h3b.h3b_gemm_bf16_gated_residual(bf16_dev(a), bf16_dev(w), to_dev(bias), torch.zeros((items, N), device="cuda"),
                                     rpi, N, xd2)
    assert np.array_equal(bf16_host(xd2), x)
    no_device_error()


# ----------------------------------------------------------------------------- QKV + RoPE

def _qkv_reference(wl, A_f32, sA, raw_w):
    """Oracle Q,K,V (token-major [R][3d]) after dequant and RoPE."""
    d = wl.d
    if wl.qkv_int8:
        qa, _ = O.quantize_rows(A_f32) if sA is None else (A_f32, None)
        w, s = O.quantize_rows(raw_w["wqkv"])
        acc = O.gemm_i8(qa, w)
        qkv = O.dequant(acc, sA, s)
    else:
        qkv = O.gemm_f64(bf16_f64(A_f32), bf16_f64(raw_w["wqkv_bf16"]))
    t, h, w_ = O.grid_positions(wl.T, wl.H, wl.W)
    t, h, w_ = (np.tile(a, wl.B) for a in (t, h, w_))
    Q = O.rope_3d(qkv[:, :d], t, h, w_, wl.n_heads, wl.head_dim, wl.rope)
    K = O.rope_3d(qkv[:, d:2 * d], t, h, w_, wl.n_heads, wl.head_dim, wl.rope)
    return np.concatenate([Q, K, qkv[:, 2 * d:]], axis=1)


def _head_major_to_token_major(qkv_dev, wl):
    B, H, L, dh = wl.B, wl.n_heads, wl.L, wl.head_dim
    a = bf16_f64(bf16_host(qkv_dev)).reshape(3, B, H, L, dh)
    return a.transpose(1, 3, 0, 2, 4).reshape(B * L, 3 * H * dh)


@pytest.mark.parametrize("name,B,qkv_int8", [("d256_L512", 1, True), ("d256_L512", 2, True),
                                              ("d2048_L4096", 1, True), ("d256_L512", 1, False)])
def test_qkv_projection_rope_head_major(name, B, qkv_int8):
    wl = synth.WORKLOADS[name].with_(B=B, qkv_int8=qkv_int8)
    if name == "d2048_L4096":
        wl = wl.with_(T=2, H=16, W=16)  # 512 tokens keep the oracle GEMM quick
    raw = synth.block_weights(wl)
    r = _rng(21)
    R, d = wl.B * wl.L, wl.d
    dims = dims_of(wl)
    qkv = torch.empty(3 * R * d, dtype=torch.bfloat16, device="cuda")
    rope_ws = torch.empty(h3b.h3b_rope_table_bytes(dims), dtype=torch.uint8, device="cuda")
    blk = DeviceBlock.from_host(raw, qkv_int8=qkv_int8)
    if qkv_int8:
        a = (r.standard_normal((R, d)) * 2).astype(np.float32)
        qa, sa = O.quantize_rows(a)
        h3b.h3b_qkv_projection(dims, to_dev(qa), to_dev(sa), blk.struct, qkv, rope_ws)
        ref = _qkv_reference(wl, qa, sa, raw)
    else:
        a = synth.f32_to_bf16_bits((r.standard_normal((R, d)) * 2).astype(np.float32))
        h3b.h3b_qkv_projection(dims, bf16_dev(a), None, blk.struct, qkv, rope_ws)
        ref = _qkv_reference(wl, a, None, raw)
    got = _head_major_to_token_major(qkv, wl)
    assert np.max(np.abs(got - ref)) <= 2 ** -8 * np.max(np.abs(ref)) * 2
    assert rel_l2(got, ref) < 4e-3
    no_device_error()


@pytest.mark.parametrize("T,HW,qkv_int8", [(8, 48, True), (16, 48, True), (8, 48, False), (2, 64, True)])
def test_qkv_projection_rope_full_video_grids(T, HW, qkv_int8):
    """QKV + 3D RoPE on the full T x 48 x 48 grids of the d=5120 workloads (18432 and 36864
    tokens), head_dim 128 with the (32, 48, 48) split, so every position up to (T-1, 47, 47)
    is rotated and written head-major. The width is 512 (4 heads) to keep the oracle's GEMM
    short: positions and the split, not the width, decide the rotation. All rows compared.
    The 2 x 64 x 64 grid's RoPE table (3104 cos/sin entries) is larger than the shared memory
    the GEMM has left for it, so the epilogue reads it from global memory instead."""
    wl = synth.WORKLOADS["d5120_L18432"].with_(T=T, H=HW, W=HW, d=512, n_heads=4, d_ff=2048, qkv_int8=qkv_int8)
    raw = synth.block_weights(wl)
    r = _rng(31 + T)
    R, d = wl.B * wl.L, wl.d
    dims = dims_of(wl)
    qkv = torch.empty(3 * R * d, dtype=torch.bfloat16, device="cuda")
    rope_ws = torch.empty(h3b.h3b_rope_table_bytes(dims), dtype=torch.uint8, device="cuda")
    blk = DeviceBlock.from_host(raw, qkv_int8=qkv_int8)
    if qkv_int8:
        qa, sa = O.quantize_rows((r.standard_normal((R, d)) * 2).astype(np.float32))
        h3b.h3b_qkv_projection(dims, to_dev(qa), to_dev(sa), blk.struct, qkv, rope_ws)
        ref = _qkv_reference(wl, qa, sa, raw)
    else:
        a = synth.f32_to_bf16_bits((r.standard_normal((R, d)) * 2).astype(np.float32))
        h3b.h3b_qkv_projection(dims, bf16_dev(a), None, blk.struct, qkv, rope_ws)
        ref = _qkv_reference(wl, a, None, raw)
    got = _head_major_to_token_major(qkv, wl)
    assert np.max(np.abs(got - ref)) <= 2 ** -8 * np.max(np.abs(ref)) * 2
    assert rel_l2(got, ref) < 4e-3
    # per token: the last token (position (T-1, H-1, W-1)) and the first agree as closely
    for row in (0, R - 1):
        assert rel_l2(got[row], ref[row]) < 8e-3
    no_device_error()


# ----------------------------------------------------------------------------- attention

@pytest.mark.parametrize("B,H,L,dh,n_q", [(1, 4, 512, 64, 512), (1, 2, 200, 128, 200), (2, 2, 777, 128, 128),
                                          (1, 16, 4096, 128, 96), (1, 1, 128, 64, 128), (1, 1, 1, 128, 1),
                                          (1, 40, 36864, 128, 48)])
def test_attention(B, H, L, dh, n_q):
    """The last case is the frame sweep's longest grid at its launch shape: 40 heads of 128
    over 36864 tokens (144 key tiles per query tile)."""
    r = _rng(B * H * L * dh)
    # head-major bf16 Q, K, V with a spread of score magnitudes
    qkv_bits = synth.f32_to_bf16_bits((r.standard_normal((3, B, H, L, dh), dtype=np.float32) *
                                       r.uniform(0.3, 2.0, (3, B, H, 1, 1))).astype(np.float32))
    wl = synth.Workload("attn", 1, 1, L, H * dh, H, dh, 256, (0, 0, dh), 0, B=B)
    dims = dims_of(wl)
    o = torch.empty((B, L, H * dh), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(B * L, dtype=torch.float32, device="cuda")
    h3b.h3b_attention(dims, bf16_dev(qkv_bits), o, am)
    og = bf16_f64(bf16_host(o))
    q = bf16_f64(qkv_bits)
    rows = synth.sample_rows(L, n_q)
    for b in range(B):
        tm = lambda part: q[part, b].transpose(1, 0, 2).reshape(L, H * dh)
        ref = O.attention(tm(0)[rows], tm(1), tm(2), H, dh)
        got = og[b, rows]
        assert rel_l2(got, ref) < 1e-2
        assert np.max(np.abs(got - ref)) < 2e-2 * np.max(np.abs(ref)) + 1e-3
    assert np.array_equal(am.cpu().numpy(), np.abs(og).max(axis=2).reshape(-1).astype(np.float32))
    no_device_error()


def test_attention_running_max_jumps():
    """Key tiles whose scores grow from one 128-key tile to the next by far more than 2^8 (head
    0: keys scaled 1, 4, 7, 10, 13 by tile), so that the kernel's lazily kept running max moves
    and O and the row sum are rescaled at every tile, and shrink the same way (head 1: the
    first tile holds the max throughout)."""
    B, H, L, dh = 1, 2, 640, 128
    r = _rng(4242)
    q = r.standard_normal((B, H, L, dh)).astype(np.float32)
    k = r.standard_normal((B, H, L, dh)).astype(np.float32)
    v = r.standard_normal((B, H, L, dh)).astype(np.float32)
    tile = np.arange(L) // 128
    k[:, 0] *= (1.0 + 3.0 * tile).astype(np.float32)[None, :, None]
    k[:, 1] *= (1.0 + 3.0 * (tile.max() - tile)).astype(np.float32)[None, :, None]
    qkv_bits = synth.f32_to_bf16_bits(np.stack([q, k, v]))
    wl = synth.Workload("attn", 1, 1, L, H * dh, H, dh, 256, (0, 0, dh), 0, B=B)
    dims = dims_of(wl)
    o = torch.empty((B, L, H * dh), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(B * L, dtype=torch.float32, device="cuda")
    h3b.h3b_attention(dims, bf16_dev(qkv_bits), o, am)
    og = bf16_f64(bf16_host(o))
    qb = bf16_f64(qkv_bits)
    rows = synth.sample_rows(L, 128)
    tm = lambda part: qb[part, 0].transpose(1, 0, 2).reshape(L, H * dh)  # noqa: E731
    ref = O.attention(tm(0)[rows], tm(1), tm(2), H, dh)
    got = og[0, rows]
    assert rel_l2(got, ref) < 1e-2
    assert np.max(np.abs(got - ref)) < 2e-2 * np.max(np.abs(ref)) + 1e-3
    no_device_error()


# ----------------------------------------------------------------------------- token pairing

@pytest.mark.parametrize("B,T,H,W,d", [(1, 2, 16, 16, 256), (2, 1, 3, 6, 8), (1, 8, 48, 48, 5120)])
def test_token_pair_unpair(B, T, H, W, d):
    r = _rng(B * T * H * W)
    x = synth.f32_to_bf16_bits(r.standard_normal((B, T, H, W, d)).astype(np.float32))
    full = h3b.make_dims(B, T, H, W, d, 1, 64, 256, (0, 0, 64))
    xm = torch.empty((B, T, H, W // 2, d), dtype=torch.bfloat16, device="cuda")
    xm2 = torch.empty_like(xm)
    xd = bf16_dev(x)
    h3b.h3b_token_pair(full, xd, xm, xm2)
    xo = O.token_pair(x, B, T, H, W, d)
    assert np.array_equal(bf16_host(xm), xo) and np.array_equal(bf16_host(xm2), xo)
    ym_bits = synth.f32_to_bf16_bits(r.standard_normal((B, T, H, W // 2, d)).astype(np.float32))
    out = torch.empty_like(xd)
    h3b.h3b_token_unpair(full, xd, xm, bf16_dev(ym_bits), out)
    ref = O.token_unpair(x, xo, bf16_f64(ym_bits), B, T, H, W, d)
    # one bf16 rounding of the result plus the fp32 error of x + (ym - xm) when
    # the terms nearly cancel (relative to the terms' magnitude)
    got = bf16_f64(bf16_host(out))
    terms = np.abs(bf16_f64(x)) + np.repeat(np.abs(bf16_f64(ym_bits)) + np.abs(bf16_f64(xo)), 2,
                                                 axis=3)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * terms)
    # without xm the merged input is recomputed from x: the same bits
    out2 = torch.empty_like(xd)
    h3b.h3b_token_unpair(full, xd, None, bf16_dev(ym_bits), out2)
    assert torch.equal(out2, out)
    # in place on x, as the token-reduction pass runs it
    xd2 = bf16_dev(x)
    h3b.h3b_token_unpair(full, xd2, None, bf16_dev(ym_bits), xd2)
    assert torch.equal(xd2, out)
    # identity block: unpair(x, xm, xm) == x exactly
    h3b.h3b_token_unpair(full, xd, xm, xm, out)
    assert np.array_equal(bf16_host(out), x)
    no_device_error()
