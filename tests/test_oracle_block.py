"""Block-level pins of the CPU oracle (no GPU needed).

The steps are pinned one by one in test_oracle_pins.py; these check how the
block composes them: the gate chunks really gate (a zero gate gives an exact
identity), a sampled-row evaluation equals the full evaluation on those rows,
batch items are independent, and the quantities fed between steps have the
sizes the method implies.
"""
import numpy as np
import pytest

import oracle as O
from video_diffusion_transformer_adaln_b200 import synth

WL = synth.WORKLOADS["d256_L512"].with_(T=1, H=8, W=8)  # 64 tokens, d=256: seconds on one core


def _weights(wl, block=0, zero_gates=False):
    raw = synth.block_weights(wl, block)
    w = {"w_ada": raw["w_ada"], "b_ada": raw["b_ada"].copy()}
    if zero_gates:
        d = wl.d
        w["b_ada"][2 * d:3 * d] = 0
        w["b_ada"][5 * d:6 * d] = 0
    for name, sname in (("wqkv", "sqkv"), ("wo", "so"), ("w1", "s1"), ("w2", "s2")):
        w[name], w[sname] = O.quantize_rows(raw[name])
    if "wqkv_bf16" in raw:
        w["wqkv_bf16"] = raw["wqkv_bf16"]
    if "wo_bf16" in raw:
        w["wo_bf16"] = raw["wo_bf16"]
    return w


def _dims(wl):
    return O.Dims(wl.B, wl.T, wl.H, wl.W, wl.d, wl.n_heads, wl.head_dim, wl.d_ff, wl.rope,
                  wl.rope_theta, wl.ln_eps, wl.qkv_int8, wl.wo_bf16)


def test_zero_gates_give_exact_identity():
    wl = WL
    x = synth.x_input(wl)
    out = O.block_forward(_dims(wl), _weights(wl, zero_gates=True), synth.cond(wl), x)
    assert np.array_equal(out, O.bf16_decode(x).reshape(-1, wl.d))


def test_zero_mlp_gate_leaves_attention_residual():
    wl = WL
    w = _weights(wl)
    w["b_ada"][5 * wl.d:] = 0
    x = synth.x_input(wl)
    out, tr = O.block_forward(_dims(wl), w, synth.cond(wl), x, trace=True)
    assert np.array_equal(out, tr["x1"])
    assert not np.array_equal(out, O.bf16_decode(x).reshape(-1, wl.d))


def test_sampled_rows_equal_full_rows():
    wl = WL
    w = _weights(wl)
    x, c = synth.x_input(wl), synth.cond(wl)
    full = O.block_forward(_dims(wl), w, c, x)
    rows = synth.sample_rows(wl.L, 9)
    part = O.block_forward(_dims(wl), w, c, x, rows=rows)
    assert np.array_equal(part, full[rows])


def test_batch_items_are_independent():
    wl = WL
    w = _weights(wl)
    wl2 = wl.with_(B=2)
    x2, c2 = synth.x_input(wl2), synth.cond(wl2)
    out2 = O.block_forward(_dims(wl2), w, c2, x2)
    for b in range(2):
        ob = O.block_forward(_dims(wl), w, c2[b:b + 1], x2[b:b + 1])
        assert np.array_equal(out2[b * wl.L:(b + 1) * wl.L], ob)


def test_trace_quantities_are_consistent():
    wl = WL
    w = _weights(wl)
    x, c = synth.x_input(wl), synth.cond(wl)
    out, tr = O.block_forward(_dims(wl), w, c, x, trace=True)
    d = wl.d
    # mod = AdaLN Linear(c), gates = the seeded gate biases (gate rows are zero)
    assert np.max(np.abs(tr["mod"][0] - O.adaln_linear(w["w_ada"], w["b_ada"], c[0]))) == 0
    assert np.max(np.abs(tr["mod"][0, 2 * d:3 * d] - w["b_ada"][2 * d:3 * d])) < 1e-12
    # h1 = bf16(LN(x) (1 + scale) + shift)
    y = O.layernorm(O.bf16_decode(x).reshape(-1, d), wl.ln_eps)
    assert np.array_equal(tr["h1"], O.modulate_bf16(y, tr["mod"][0, :d], tr["mod"][0, d:2 * d]))
    # Q and K are rotated (norm per pair preserved vs unrotated projections, up to the bf16
    # rounding of the attention's inputs), V is not rotated; all three are bf16 values
    q1, s1 = O.quantize_rows(O.bf16_decode(tr["h1"]).astype(np.float32))
    raw = O.dequant(O.gemm_i8(q1, w["wqkv"]), s1, w["sqkv"])
    assert np.array_equal(tr["qkv"][:, 2 * d:], O.bf16_decode(O.bf16_round(raw[:, 2 * d:])))
    assert np.array_equal(tr["qkv"], O.bf16_decode(O.bf16_round(tr["qkv"])))
    qk = tr["qkv"][:, :2 * d]
    n_rot = np.hypot(qk[:, 0::2], qk[:, 1::2])
    n_raw = np.hypot(raw[:, :2 * d:2], raw[:, 1:2 * d:2])
    assert np.all(np.abs(n_rot - n_raw) <= 2.0 ** -8 * n_raw + 1e-300)
    assert not np.allclose(qk, raw[:, :2 * d])
    # GELU output feeds a per-row quantizer of width d_ff
    assert tr["gelu"].shape == (wl.L, wl.d_ff)
    assert np.isfinite(out).all()


def test_bf16_qkv_variant_runs_and_differs_slightly():
    wl = WL.with_(qkv_int8=False)
    w = _weights(wl)
    x, c = synth.x_input(wl), synth.cond(wl)
    a = O.block_forward(_dims(wl), w, c, x)
    b = O.block_forward(_dims(WL), _weights(WL), c, x)
    xd = O.bf16_decode(x).reshape(-1, wl.d)
    rel = np.linalg.norm((a - xd) - (b - xd)) / np.linalg.norm(a - xd)
    assert 0 < rel < 0.1  # int8 vs bf16 QKV: close but not identical deltas


def test_bf16_wo_projection_is_the_plain_product():
    """bf16 output projection ([README] "Metal 4 및 TensorOps": BF16 for the attention-output
    projection): x1 = x + gate_a * (bf16(O) @ bf16(Wo)^T), checked against a numpy product."""
    wl = WL.with_(wo_bf16=True)
    raw = synth.block_weights(wl)
    w = _weights(wl)
    x, c = synth.x_input(wl), synth.cond(wl)
    out, tr = O.block_forward(_dims(wl), w, c, x, trace=True)
    d = wl.d
    ob = O.bf16_decode(O.bf16_round(tr["attn"]))
    wo = O.bf16_decode(raw["wo_bf16"]).reshape(d, d)
    expect = O.bf16_decode(x).reshape(-1, d) + tr["mod"][0, 2 * d:3 * d] * np.dot(ob, wo.T)
    assert np.max(np.abs(tr["x1"] - expect)) <= 1e-12 * np.max(np.abs(expect))
    # the int8 projection of the same draws is close but not the same
    out8 = O.block_forward(_dims(WL), _weights(WL), c, x)
    xd = O.bf16_decode(x).reshape(-1, d)
    rel = np.linalg.norm((out - xd) - (out8 - xd)) / np.linalg.norm(out8 - xd)
    assert 0 < rel < 0.1


def test_single_thread_run_gives_identical_results(tmp_path):
    """No reduction crosses OpenMP threads, so one thread and all threads give the same
    bytes (the block is run in a child process with OMP_NUM_THREADS=1)."""
    import os
    import subprocess
    import sys
    wl = WL.with_(B=2)
    w = _weights(wl)
    x, c = synth.x_input(wl), synth.cond(wl)
    many = O.block_forward(_dims(wl), w, c, x)
    out = tmp_path / "one.npy"
    code = (
        "import sys, numpy as np\n"
        f"sys.path.insert(0, {os.path.dirname(os.path.dirname(os.path.abspath(__file__)))!r})\n"
        f"sys.path.insert(0, {os.path.dirname(os.path.abspath(__file__))!r})\n"
        "import oracle as O, test_oracle_block as T\n"
        "assert O.threads() == 1\n"
        "wl = T.WL.with_(B=2)\n"
        "y = O.block_forward(T._dims(wl), T._weights(wl), T.synth.cond(wl), T.synth.x_input(wl))\n"
        f"np.save({str(out)!r}, y)\n")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    subprocess.run([sys.executable, "-c", code], check=True, env=env, timeout=300)
    assert np.array_equal(np.load(out), many)
