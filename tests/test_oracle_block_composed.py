"""The oracle's block, pinned against the same block composed from library primitives.

test_oracle_pins.py pins the oracle's steps one at a time. The tests here pin how
orc_block_forward wires those steps together: which modulation chunk feeds which
step, which tensor serves as the attention's query, key and value, where the bf16
roundings and the int8 re-quantizations sit, and which scales and biases each
dequantization takes. A mistake in that wiring can pass every step pin.

The block is recomposed below in float64 from PyTorch and numpy primitives that
share nothing with the oracle's C++:
  * LayerNorm: torch.nn.functional.layer_norm (no affine);
  * attention: torch.nn.functional.scaled_dot_product_attention;
  * GELU: torch.nn.functional.gelu(approximate="tanh");
  * RoPE: a complex rotation per lane pair, with grid positions from np.unravel_index;
  * int8 products: exact int64 matrix products;
  * bf16 rounding: round-half-even applied to the float64 bit pattern.
The steps follow the gated-AdaLN block described on the MiniMax-H3 h3-metal README,
sections "Int8 양자화" (int8 weights with per-output-channel scales and dynamic
per-token activation scales, gated AdaLN fused ahead of the projections) and
"Metal 4 및 TensorOps" (a BF16 attention-output projection), and the h3.c/MLX
comparison page, section "性能上限" (AdaLN gating and RoPE folded in before the
projections). The dimensions, chunk order, RoPE split and GELU form are the same
readings the oracle states for the points the pages leave open.
"""
import numpy as np
import torch
import torch.nn.functional as F

import oracle as O
from video_diffusion_transformer_adaln_b200 import synth

# 2 frames x 4 rows x 8 columns: every RoPE axis has more than one position, and
# H != W, so a swapped row/column index shows.
WL = synth.WORKLOADS["d256_L512"].with_(T=2, H=4, W=8)


# --------------------------------------------------------------- independent primitives

def bf16_bits(x):
    """Round float64 to bf16 (ties to even) in one step, on the float64 bit pattern.
    Covers zero and the normal bf16 range, which is all the block produces."""
    x = np.ascontiguousarray(x, np.float64)
    a = np.abs(x)
    assert np.all((a == 0) | ((a >= 2.0 ** -126) & (a < 2.0 ** 127)))
    u = x.view(np.uint64)
    drop = 45  # float64 keeps 52 fraction bits, bf16 keeps 7
    lsb = (u >> np.uint64(drop)) & np.uint64(1)
    u = (u + np.uint64((1 << (drop - 1)) - 1) + lsb) & ~np.uint64((1 << drop) - 1)
    f32 = u.view(np.float64).astype(np.float32)  # exact: at most 8 significant bits remain
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_value(b):
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def quant(v):
    """Per-row symmetric int8 with an F32 scale: s = absmax/127, code = rint(v/s) (both in F32)."""
    v = np.ascontiguousarray(v, np.float32)
    amax = np.abs(v).max(axis=1)
    s = amax / np.float32(127)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(v / s[:, None])
    q = np.where(amax[:, None] == 0, np.float32(0), np.clip(q, -127, 127))
    return q.astype(np.int8), s


def int_product(a, w):
    acc = a.astype(np.int64) @ w.astype(np.int64).T
    assert np.abs(acc).max() < 2 ** 31
    return acc


def dequant(acc, s_tok, s_ch, bias):
    return acc.astype(np.float64) * s_tok.astype(np.float64)[:, None] * s_ch.astype(np.float64)[None, :] + bias


def layer_norm(x, eps):
    t = torch.from_numpy(np.ascontiguousarray(x, np.float64))
    return F.layer_norm(t, (t.shape[-1],), eps=eps).numpy()


def rope(x, wl):
    """Rotate lane pairs (2j, 2j+1) of every head by position x frequency theta^(-2j/r),
    the frame index driving the first rope_t lanes, the row index the next rope_h, the
    column index the rest."""
    L, nh, dh = wl.L, wl.n_heads, wl.head_dim
    pos = np.unravel_index(np.arange(L), (wl.T, wl.H, wl.W))
    angles = []
    for p, r in zip(pos, wl.rope):
        j = np.arange(r // 2)
        angles.append(p[:, None] * wl.rope_theta ** (-2.0 * j / r)[None, :])
    ang = np.concatenate(angles, axis=1)  # [L, dh/2]
    pairs = x.reshape(L, nh, dh // 2, 2)
    z = (pairs[..., 0] + 1j * pairs[..., 1]) * np.exp(1j * ang)[:, None, :]
    return np.stack([z.real, z.imag], axis=-1).reshape(L, nh * dh)


def attention(Q, K, V, wl):
    heads = lambda a: torch.from_numpy(a.reshape(wl.L, wl.n_heads, wl.head_dim).transpose(1, 0, 2).copy())
    o = F.scaled_dot_product_attention(heads(Q)[None], heads(K)[None], heads(V)[None])[0]
    return o.permute(1, 0, 2).reshape(wl.L, wl.d).numpy()


def gelu(x):
    return F.gelu(torch.from_numpy(x), approximate="tanh").numpy()


# ------------------------------------------------------------------------ composition

def composed_block(wl, w, c, x_bits):
    """Block output and intermediates, batch item by batch item."""
    d = wl.d
    xd = bf16_value(x_bits).reshape(wl.B, wl.L, d)
    bias = lambda name, n: w[name].astype(np.float64) if w.get(name) is not None else np.zeros(n)
    tr = {k: [] for k in ("mod", "h1", "qkv", "attn", "x1", "h2", "gelu")}
    outs = []
    for b in range(wl.B):
        mod = bf16_value(w["w_ada"]).reshape(6 * d, d) @ c[b].astype(np.float64) + bias("b_ada", 6 * d)
        shift_a, scale_a, gate_a, shift_m, scale_m, gate_m = np.split(mod, 6)
        h1 = bf16_bits(layer_norm(xd[b], wl.ln_eps) * (1 + scale_a) + shift_a)
        if wl.qkv_int8:
            q1, s1 = quant(bf16_value(h1))
            qkv = dequant(int_product(q1, w["wqkv"]), s1, w["sqkv"], bias("bqkv", 3 * d))
        else:
            qkv = bf16_value(h1) @ bf16_value(w["wqkv_bf16"]).reshape(3 * d, d).T + bias("bqkv", 3 * d)
        Q, K, V = np.split(qkv, 3, axis=1)
        Q, K = rope(Q, wl), rope(K, wl)
        # the attention's inputs are bf16
        Q, K, V = (bf16_value(bf16_bits(a)) for a in (Q, K, V))
        o = attention(Q, K, V, wl)
        ob = bf16_value(bf16_bits(o))
        if wl.wo_bf16:
            yo = ob @ bf16_value(w["wo_bf16"]).reshape(d, d).T + bias("bo", d)
        else:
            q2, s2 = quant(ob)
            yo = dequant(int_product(q2, w["wo"]), s2, w["so"], bias("bo", d))
        x1 = xd[b] + gate_a * yo
        h2 = bf16_bits(layer_norm(x1, wl.ln_eps) * (1 + scale_m) + shift_m)
        q3, s3 = quant(bf16_value(h2))
        g = gelu(dequant(int_product(q3, w["w1"]), s3, w["s1"], bias("b1", wl.d_ff)))
        q4, s4 = quant(bf16_value(bf16_bits(g)))
        y4 = dequant(int_product(q4, w["w2"]), s4, w["s2"], bias("b2", d))
        outs.append(x1 + gate_m * y4)
        for k, v in (("mod", mod), ("h1", h1), ("qkv", np.concatenate([Q, K, V], axis=1)), ("attn", o),
                     ("x1", x1), ("h2", h2), ("gelu", g)):
            tr[k].append(v)
    return np.concatenate(outs), {k: (np.stack(v) if k == "mod" else np.concatenate(v)) for k, v in tr.items()}


def _inputs(wl, biases=True):
    """Seeded weights of the workload, quantized here; optional nonzero biases on every
    projection so that each dequantization's bias term is exercised."""
    raw = synth.block_weights(wl)
    w = {"w_ada": raw["w_ada"], "b_ada": raw["b_ada"]}
    for name, sname in (("wqkv", "sqkv"), ("wo", "so"), ("w1", "s1"), ("w2", "s2")):
        w[name], w[sname] = quant(raw[name])
    for name in ("wqkv_bf16", "wo_bf16"):
        if name in raw:
            w[name] = raw[name]
    if biases:
        rng = np.random.default_rng(7)
        for name, n in (("bqkv", 3 * wl.d), ("bo", wl.d), ("b1", wl.d_ff), ("b2", wl.d)):
            w[name] = (0.1 * rng.standard_normal(n)).astype(np.float32)
    return w, synth.cond(wl), synth.x_input(wl)


def _dims(wl):
    return O.Dims(wl.B, wl.T, wl.H, wl.W, wl.d, wl.n_heads, wl.head_dim, wl.d_ff, wl.rope,
                  wl.rope_theta, wl.ln_eps, wl.qkv_int8, wl.wo_bf16)


def _check(wl, biases=True):
    w, c, x = _inputs(wl, biases)
    out, tr = O.block_forward(_dims(wl), w, c, x, trace=True)
    ref, rtr = composed_block(wl, w, c.reshape(wl.B, wl.d), x)

    def close(a, b, tol=1e-11):
        return np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b)))

    # Integer-valued steps (bf16 codes) match exactly; float64 steps up to summation order.
    assert close(tr["mod"], rtr["mod"])
    assert np.array_equal(tr["h1"], rtr["h1"])
    assert close(tr["qkv"], rtr["qkv"])
    assert close(tr["attn"], rtr["attn"])
    assert close(tr["x1"], rtr["x1"])
    assert np.array_equal(tr["h2"], rtr["h2"])
    assert close(tr["gelu"], rtr["gelu"])
    assert close(out, ref)


def test_int8_block_equals_composition_two_batch_items():
    _check(WL.with_(B=2))


def test_int8_block_equals_composition_without_biases():
    _check(WL, biases=False)


def test_bf16_projection_variants_equal_composition():
    _check(WL.with_(qkv_int8=False, wo_bf16=True))


def test_composition_helpers_against_known_values():
    """The test's own primitives, pinned on values fixed by the definitions."""
    # bf16: 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); 1 + 3*2^-8 -> 1 + 2^-6 (even)
    v = np.array([1.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -2.5, 0.0, 3.0e38 / 2 ** 10])
    got = bf16_value(bf16_bits(v))
    assert list(got[:5]) == [1.0, 1.0, 1 + 2.0 ** -6, -2.5, 0.0]
    assert abs(got[5] - v[5]) <= 2.0 ** -9 * abs(v[5])
    # quantizer with absmax 127 -> scale 1, ties to even
    q, s = quant(np.array([[127.0, 2.5, 3.5, -2.5, 0.4]], np.float32))
    assert s[0] == 1.0 and list(q[0]) == [127, 2, 4, -2, 0]
    q, s = quant(np.zeros((1, 4), np.float32))
    assert s[0] == 0 and not q.any()
    # RoPE: token 0 is unrotated; a rotation keeps the norm of every pair
    x = np.random.default_rng(1).standard_normal((WL.L, WL.d))
    r = rope(x, WL)
    assert np.array_equal(r[0], x[0])
    assert np.allclose(np.hypot(r[:, 0::2], r[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-12)


def test_composition_holds_on_random_small_grids():
    """The same comparison over random small grids, head shapes, RoPE splits and batch
    sizes, including one-frame, one-row and one-column grids."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    @settings(max_examples=12, deadline=None, suppress_health_check=list(HealthCheck))
    @given(T=st.integers(1, 3), H=st.integers(1, 4), W=st.integers(1, 5), B=st.integers(1, 2),
           head=st.sampled_from([(4, 64, (16, 24, 24)), (2, 128, (32, 48, 48)), (4, 64, (0, 32, 32)),
                                 (2, 128, (64, 0, 64))]),
           qkv_int8=st.booleans(), wo_bf16=st.booleans())
    def check(T, H, W, B, head, qkv_int8, wo_bf16):
        nh, dh, rope = head
        wl = synth.WORKLOADS["d256_L512"].with_(T=T, H=H, W=W, B=B, n_heads=nh, head_dim=dh, rope=rope,
                                                 qkv_int8=qkv_int8, wo_bf16=wo_bf16)
        _check(wl)
    check()
