"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test checks one oracle step against a hand-worked golden value, a closed
form, an invariant the definition implies, a brute-force evaluation, or a
library routine that the step reduces to. Together they are chosen so that a
dropped term, a wrong sign or index, or a transposed operand in any step fails
at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from video_diffusion_transformer_adaln_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [p.strip() for p in line.split(";")]


# ----------------------------------------------------------------------------- bf16

def test_bf16_rounding_golden():
    for expr, bits in _golden_lines("bf16_rounding.txt"):
        v = float(eval(expr))  # fixture expressions are plain arithmetic
        assert O.lib().orc_f64_to_bf16(v) == int(bits, 16), expr


def test_bf16_rounding_matches_torch_on_float32_inputs():
    # For binary32 inputs a single rounding to bf16 is what torch's RNE cast does.
    rng = np.random.default_rng(1)
    f = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    ours = O.bf16_round(f.astype(np.float64))
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_decode_roundtrip():
    b = np.arange(0, 65536, dtype=np.uint16)
    b = b[((b & 0x7F80) != 0x7F80)]  # finite values only
    assert np.array_equal(O.bf16_round(O.bf16_decode(b)), np.where(b == 0x8000, 0x8000, b))


# ----------------------------------------------------------------------------- quantizer

def test_quantize_rows_golden():
    for vals, scale, codes in _golden_lines("quantize_rows.txt"):
        v = np.array([float(t) for t in vals.split()], np.float32)[None, :]
        q, s = O.quantize_rows(v)
        assert s[0] == np.float32(float(scale))
        assert q[0].tolist() == [int(t) for t in codes.split()]


def test_quantize_rows_invariants():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal((300, 517)) * rng.uniform(0.01, 50, (300, 1))).astype(np.float32)
    v[7] = 0.0
    q, s = O.quantize_rows(v)
    assert q.min() >= -127 and q.max() <= 127
    nz = np.abs(v).max(axis=1) > 0
    # the row's absmax element maps to +-127
    am = np.abs(v).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(300), am])[nz] == 127)
    # reconstruction error at most half a step, plus the binary32 rounding of the
    # quotient v/s (which can land exactly on a tie): |v| * 2^-24 per element
    err = np.abs(q.astype(np.float64) * s[:, None] - v)
    assert np.all(err <= 0.5 * s[:, None] + np.abs(v) * 2.0 ** -23)
    # odd symmetry and exact power-of-two scaling
    qn, sn = O.quantize_rows(-v)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    q4, s4 = O.quantize_rows(v * np.float32(4.0))
    assert np.array_equal(q4, q) and np.array_equal(s4, s * np.float32(4.0))
    assert np.all(q[7] == 0) and s[7] == 0


# ----------------------------------------------------------------------------- GEMM

def test_gemm_i8_brute_force_small():
    rng = np.random.default_rng(3)
    A = rng.integers(-128, 128, (5, 33), dtype=np.int8)
    W = rng.integers(-128, 128, (7, 33), dtype=np.int8)
    C = O.gemm_i8(A, W)
    for m in range(5):
        for n in range(7):
            assert C[m, n] == sum(int(A[m, k]) * int(W[n, k]) for k in range(33))


def test_gemm_i8_matches_float64_matmul():
    rng = np.random.default_rng(4)
    A = rng.integers(-127, 128, (64, 1000), dtype=np.int8)
    W = rng.integers(-127, 128, (96, 1000), dtype=np.int8)
    ref = A.astype(np.float64) @ W.astype(np.float64).T  # exact: |sum| << 2^53
    assert np.array_equal(O.gemm_i8(A, W), ref.astype(np.int32))


def test_gemm_i8_extremes_and_long_k():
    K = 20480
    A = np.full((2, K), -128, np.int8)
    W = np.full((3, K), -128, np.int8)
    W[1] = 127
    C = O.gemm_i8(A, W)
    assert C[0, 0] == 16384 * K and C[1, 1] == -128 * 127 * K
    Kbig = 140000  # beyond the int32-exact bound: the int64 path reports overflow
    A = np.full((1, Kbig), 127, np.int8)
    with pytest.raises(OverflowError):
        O.gemm_i8(A, A)


def test_dequant_closed_form():
    acc = np.array([[3, -4], [0, 100]], np.int32)
    out = O.dequant(acc, np.array([0.5, 2.0], np.float32), np.array([0.25, 4.0], np.float32),
                    np.array([1.0, -1.0], np.float32))
    assert out.tolist() == [[3 * 0.5 * 0.25 + 1, -4 * 0.5 * 4 - 1], [1.0, 100 * 2 * 4 - 1]]


# ----------------------------------------------------------------------------- LayerNorm / modulation

def test_layernorm_matches_torch_and_invariants():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((40, 256)) * 3 + 1.5
    y = O.layernorm(x, 1e-6)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (256,), eps=1e-6).numpy()
    assert np.max(np.abs(y - ref)) < 1e-12
    # constant row -> zeros; affine invariance
    assert np.all(O.layernorm(np.full((1, 64), 7.25), 1e-6) == 0.0)
    y2 = O.layernorm(x * 5.0 - 2.0, 0.0)
    assert np.max(np.abs(y2 - O.layernorm(x, 0.0))) < 1e-12
    assert np.max(np.abs(y2.mean(axis=1))) < 1e-12
    assert np.max(np.abs((y2 ** 2).mean(axis=1) - 1.0)) < 1e-12


def test_modulate_special_cases():
    rng = np.random.default_rng(6)
    y = rng.standard_normal((8, 64))
    z = np.zeros(64)
    # no modulation: the bf16 rounding of y itself
    assert np.array_equal(O.modulate_bf16(y, z, z), O.bf16_round(y))
    # scale = -1 kills y: every row becomes bf16(shift)
    shift = rng.standard_normal(64)
    h = O.modulate_bf16(y, shift, -np.ones(64))
    assert np.all(h == O.bf16_round(shift)[None, :])
    # scale = 1 doubles, shift adds
    h = O.modulate_bf16(y, np.full(64, 0.5), np.ones(64))
    assert np.array_equal(h, O.bf16_round(2 * y + 0.5))


def test_adaln_linear_matches_matmul():
    rng = np.random.default_rng(7)
    d = 48
    w = rng.standard_normal((6 * d, d)).astype(np.float32)
    wb = torch.from_numpy(w).to(torch.bfloat16)
    wbits = wb.view(torch.int16).numpy().view(np.uint16)
    c = rng.standard_normal(d).astype(np.float32)
    b = rng.standard_normal(6 * d).astype(np.float32)
    ref = wb.double().numpy() @ c.astype(np.float64) + b
    assert np.max(np.abs(O.adaln_linear(wbits, b, c) - ref)) < 1e-12
    assert np.max(np.abs(O.adaln_linear(wbits, None, c) - (ref - b))) < 1e-12


# ----------------------------------------------------------------------------- RoPE

def test_grid_positions_golden():
    t, h, w = O.grid_positions(2, 3, 4)
    # token i = (t*3 + h)*4 + w
    assert (t[0], h[0], w[0]) == (0, 0, 0)
    assert (t[5], h[5], w[5]) == (0, 1, 1)
    assert (t[11], h[11], w[11]) == (0, 2, 3)
    assert (t[12], h[12], w[12]) == (1, 0, 0)
    assert (t[23], h[23], w[23]) == (1, 2, 3)


def test_rope_golden_angles():
    for dims, pos, lane, angle in _golden_lines("rope_3d.txt"):
        dh, rt, rh, rw = (int(v) for v in dims.split())
        tp, hp, wp = (np.array([int(v)], np.int32) for v in pos.split())
        lane = int(lane)
        a = float(eval(angle))
        x = np.zeros((1, dh))
        x[0, lane] = 1.0
        y = O.rope_3d(x, tp, hp, wp, 1, dh, (rt, rh, rw))
        assert abs(y[0, lane] - math.cos(a)) < 1e-12 and abs(y[0, lane + 1] - math.sin(a)) < 1e-12
        others = np.delete(y[0], [lane, lane + 1])
        assert np.all(others == 0.0)
        # the second lane of the pair rotates as (-sin, cos)
        x = np.zeros((1, dh))
        x[0, lane + 1] = 1.0
        y = O.rope_3d(x, tp, hp, wp, 1, dh, (rt, rh, rw))
        assert abs(y[0, lane] + math.sin(a)) < 1e-12 and abs(y[0, lane + 1] - math.cos(a)) < 1e-12


def test_rope_invariants():
    rng = np.random.default_rng(8)
    nh, dh, split = 3, 64, (16, 24, 24)
    n = 50
    tp, hp, wp = (rng.integers(0, 40, n).astype(np.int32) for _ in range(3))
    x = rng.standard_normal((n, nh * dh))
    y = O.rope_3d(x, tp, hp, wp, nh, dh, split)
    # per-pair norms preserved
    assert np.max(np.abs(np.hypot(y[:, 0::2], y[:, 1::2]) - np.hypot(x[:, 0::2], x[:, 1::2]))) < 1e-12
    # position 0 is the identity
    z = np.zeros(n, np.int32)
    assert np.array_equal(O.rope_3d(x, z, z, z, nh, dh, split), x)
    # <R(m)q, R(n)k> depends only on m - n, along each axis
    q = rng.standard_normal((1, dh))
    k = rng.standard_normal((1, dh))

    def dot(m, nn, axis):
        p = [np.zeros(1, np.int32) for _ in range(3)]
        pm, pn = [a.copy() for a in p], [a.copy() for a in p]
        pm[axis][0], pn[axis][0] = m, nn
        return float((O.rope_3d(q, *pm, 1, dh, split) @ O.rope_3d(k, *pn, 1, dh, split).T).item())

    for axis in range(3):
        assert abs(dot(9, 4, axis) - dot(25, 20, axis)) < 1e-10
        assert abs(dot(9, 4, axis) - dot(4, 9, axis)) > 1e-6  # not symmetric in general


# ----------------------------------------------------------------------------- attention

def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(9)
    nh, dh, L, nq = 3, 16, 37, 11
    Q = rng.standard_normal((nq, nh * dh))
    K = rng.standard_normal((L, nh * dh))
    V = rng.standard_normal((L, nh * dh))
    out = O.attention(Q, K, V, nh, dh)

    def heads(a):
        return torch.from_numpy(a).view(a.shape[0], nh, dh).transpose(0, 1)

    ref = torch.nn.functional.scaled_dot_product_attention(heads(Q), heads(K), heads(V))
    ref = ref.transpose(0, 1).reshape(nq, nh * dh).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12


def test_attention_matches_a_naive_loop_on_tiny_inputs():
    """Scores, a max-free softmax and the weighted sum, written as plain Python loops."""
    rng = np.random.default_rng(12)
    nh, dh, L, nq = 2, 4, 5, 3
    Q, K, V = (rng.standard_normal((n, nh * dh)) for n in (nq, L, L))
    out = O.attention(Q, K, V, nh, dh)
    for i in range(nq):
        for h in range(nh):
            cols = range(h * dh, (h + 1) * dh)
            w = [math.exp(sum(Q[i, c] * K[j, c] for c in cols) / math.sqrt(dh)) for j in range(L)]
            tot = sum(w)
            for c in cols:
                assert abs(out[i, c] - sum(w[j] / tot * V[j, c] for j in range(L))) < 1e-12


def test_attention_special_cases():
    rng = np.random.default_rng(10)
    nh, dh, L = 2, 8, 9
    Q = rng.standard_normal((4, nh * dh))
    V = rng.standard_normal((L, nh * dh))
    # identical keys -> uniform weights -> the mean of V
    K = np.tile(rng.standard_normal((1, nh * dh)), (L, 1))
    assert np.max(np.abs(O.attention(Q, K, V, nh, dh) - V.mean(axis=0))) < 1e-12
    # a single key -> V itself
    assert np.max(np.abs(O.attention(Q, K[:1], V[:1], nh, dh) - V[:1])) < 1e-15
    # V constant -> that constant (softmax rows sum to one)
    K = rng.standard_normal((L, nh * dh)) * 4
    assert np.max(np.abs(O.attention(Q, K, np.full((L, nh * dh), 2.5), nh, dh) - 2.5)) < 1e-13
    # key order does not matter
    perm = rng.permutation(L)
    assert np.max(np.abs(O.attention(Q, K, V, nh, dh) - O.attention(Q, K[perm], V[perm], nh, dh))) < 1e-13
    # a dominating key selects its value row
    K2 = np.zeros((L, nh * dh))
    K2[3] = Q[0] * 1e3
    out = O.attention(Q[:1], K2, V, nh, dh)
    assert np.max(np.abs(out - V[3])) < 1e-9


# ----------------------------------------------------------------------------- GELU / residual

def test_gelu_tanh_matches_torch_and_identities():
    x = np.linspace(-12, 12, 20001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    g = O.gelu_tanh(x)
    assert np.max(np.abs(g - ref)) < 1e-14
    assert O.gelu_tanh(np.zeros(1))[0] == 0.0
    assert np.max(np.abs(g - O.gelu_tanh(-x) - x)) < 1e-12  # gelu(x) - gelu(-x) = x
    assert abs(O.gelu_tanh(np.array([30.0]))[0] - 30.0) < 1e-12


def test_gated_residual_closed_form():
    rng = np.random.default_rng(11)
    x, y = rng.standard_normal((5, 16)), rng.standard_normal((5, 16))
    assert np.array_equal(O.gated_residual(x, y, np.zeros(16)), x)
    assert np.array_equal(O.gated_residual(x, y, np.ones(16)), x + y)
    g = rng.standard_normal(16)
    assert np.max(np.abs(O.gated_residual(x, y, g) - (x + g[None] * y))) < 1e-15


# ----------------------------------------------------------------------------- token pairing

def test_token_pair_closed_form():
    B, T, H, W, d = 1, 2, 3, 4, 8
    rng = np.random.default_rng(12)
    x = O.bf16_round(rng.standard_normal((B, T, H, W, d)))
    xm = O.token_pair(x, B, T, H, W, d)
    xd = O.bf16_decode(x)
    # mean of each horizontal pair (k = w // 2); the mean of two bf16 is exact in fp64
    assert np.array_equal(xm, O.bf16_round((xd[..., 0::2, :] + xd[..., 1::2, :]) / 2))
    # golden: 1.0 and 2.0 -> 1.5 ; 1.0 and 1.0 + 2^-7 -> tie -> even (1.0)
    g = O.bf16_round(np.array([1.0, 2.0, 1.0, 1.0 + 2 ** -7])).reshape(1, 1, 1, 4, 1)
    gm = O.token_pair(g, 1, 1, 1, 4, 1)
    assert O.bf16_decode(gm).ravel().tolist() == [1.5, 1.0]


def test_token_pair_unpair_identities():
    B, T, H, W, d = 2, 2, 3, 6, 5
    rng = np.random.default_rng(13)
    half = O.bf16_round(rng.standard_normal((B, T, H, W // 2, d)))
    x = np.repeat(half, 2, axis=3)  # constant along each horizontal pair
    xm = O.token_pair(x, B, T, H, W, d)
    assert np.array_equal(xm, half)
    # an identity block (ym == xm) gives back x, bit for bit
    out = O.token_unpair(x, xm, O.bf16_decode(xm), B, T, H, W, d)
    assert np.array_equal(out, O.bf16_decode(x))
    # arbitrary x with an identity block is also returned exactly
    x2 = O.bf16_round(rng.standard_normal((B, T, H, W, d)))
    xm2 = O.token_pair(x2, B, T, H, W, d)
    assert np.array_equal(O.token_unpair(x2, xm2, O.bf16_decode(xm2), B, T, H, W, d), O.bf16_decode(x2))
    # zero residual: the merged output is copied to both positions
    ym = rng.standard_normal((B, T, H, W // 2, d))
    z = np.zeros((B, T, H, W, d), np.uint16)
    out = O.token_unpair(z, np.zeros_like(xm), ym, B, T, H, W, d)
    assert np.array_equal(out[..., 0::2, :], ym) and np.array_equal(out[..., 1::2, :], ym)


def test_range_delta_and_apply_closed_form():
    """Residual reuse: delta = after - before exactly; re-applying it to the same stream
    gives `after` back; applied to another stream it is the plain sum, rounded once."""
    r = np.random.default_rng(31)
    before = synth.f32_to_bf16_bits(r.standard_normal(4096).astype(np.float32))
    after = synth.f32_to_bf16_bits((synth.bf16_bits_to_f32(before) + r.standard_normal(4096) * 0.3).astype(np.float32))
    delta = O.range_delta(before, after)
    assert np.array_equal(delta, synth.bf16_bits_to_f32(after).astype(np.float64)
                          - synth.bf16_bits_to_f32(before).astype(np.float64))
    assert np.array_equal(O.range_apply(before, delta), after)
    other = synth.f32_to_bf16_bits(r.standard_normal(4096).astype(np.float32))
    got = synth.bf16_bits_to_f32(O.range_apply(other, delta)).astype(np.float64)
    exact = synth.bf16_bits_to_f32(other).astype(np.float64) + delta
    # one rounding to bf16: within half a bf16 ulp of the exact sum
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    assert np.all(np.abs(got - exact) <= 0.5 * ulp)
    # a zero delta is the identity
    assert np.array_equal(O.range_apply(other, np.zeros(4096)), other)


def test_bf16_rounding_is_one_rounding_of_the_double():
    """Random doubles across the normal bf16 range, plus exact ties and values one float64
    ulp either side of a tie (where rounding first to float32 would go wrong): the oracle's
    rounding equals round-half-even applied once to the float64 bit pattern."""
    rng = np.random.default_rng(14)
    mant = rng.integers(0, 2 ** 52, 20000, dtype=np.uint64)
    expo = rng.integers(1023 - 120, 1023 + 120, 20000, dtype=np.uint64)
    sign = rng.integers(0, 2, 20000, dtype=np.uint64)
    bits = (sign << np.uint64(63)) | (expo << np.uint64(52)) | mant
    # ties: 7 kept fraction bits, then exactly half an ulp; and the neighbours of each tie
    tie = (bits & ~np.uint64((1 << 45) - 1)) | np.uint64(1 << 44)
    v = np.concatenate([bits.view(np.float64), tie.view(np.float64), (tie + np.uint64(1)).view(np.float64),
                        (tie - np.uint64(1)).view(np.float64)])
    u = v.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    r = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    want = (r.view(np.float64).astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    assert np.array_equal(O.bf16_round(v), want)
