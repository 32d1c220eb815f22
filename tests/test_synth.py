"""The seeded input generator: deterministic, keyed per tensor, right distributions."""
import numpy as np

from video_diffusion_transformer_adaln_b200 import synth


def test_deterministic_and_keyed():
    wl = synth.WORKLOADS["d256_L512"]
    assert np.array_equal(synth.x_input(wl), synth.x_input(wl))
    assert not np.array_equal(synth.cond(wl, 0), synth.cond(wl, 1))
    w0, w1 = synth.block_weights(wl, 0), synth.block_weights(wl, 1)
    assert not np.array_equal(w0["w1"], w1["w1"])
    # variants of one workload share draws
    wb = synth.block_weights(wl.with_(qkv_int8=False), 0)
    assert np.array_equal(wb["wqkv"], w0["wqkv"])
    assert np.array_equal(wb["wqkv_bf16"], synth.f32_to_bf16_bits(w0["wqkv"]))


def test_distributions():
    wl = synth.WORKLOADS["d256_L512"]
    x = synth.bf16_bits_to_f32(synth.x_input(wl))[0]
    out = synth.outlier_channels(wl)
    assert out.size == 4
    std = x.std(axis=0)
    assert np.all(std[out] > 10) and np.all(np.delete(std, out) < 1.3)
    w = synth.block_weights(wl)
    d = wl.d
    assert abs(w["w1"].std() * np.sqrt(d) - 1) < 0.02
    assert abs(w["w2"].std() * np.sqrt(wl.d_ff) - 1) < 0.02
    wa = synth.bf16_bits_to_f32(w["w_ada"])
    assert np.all(wa[2 * d:3 * d] == 0) and np.all(wa[5 * d:] == 0)
    assert abs(wa[:d].std() * np.sqrt(d) - 1) < 0.02
    g = w["b_ada"][2 * d:3 * d]
    assert abs(g.var() - 0.5) < 0.1 and np.all(w["b_ada"][:2 * d] == 0)


def test_workload_sizes():
    W = synth.WORKLOADS
    assert W["d256_L512"].L == 512 and W["d2048_L4096"].L == 4096 and W["d5120_L18432"].L == 18432
    assert W["d5120_L18432_pair"].merged().L == 9216
    assert [W[f"d5120_depth50_T{t}"].L for t in (2, 4, 8, 12, 16)] == [4608, 9216, 18432, 27648, 36864]
    assert synth.outlier_channels(W["d2048_L4096"]).size == 20
    assert synth.outlier_channels(W["d5120_L18432"]).size == 51


def test_bf16_encoding_of_draws():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], np.float32)
    assert synth.f32_to_bf16_bits(f).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020]
    assert np.array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(f))[[0, 3]], f[[0, 3]])


def test_sample_rows():
    r = synth.sample_rows(1000, 20)
    assert r[0] == 0 and r[-1] == 999 and len(set(r.tolist())) == 20 and np.all(np.diff(r) > 0)


def test_variant_workloads():
    W = synth.WORKLOADS
    base = W["d5120_L18432"]
    # the variants share the base block's draws (same sizes), differing only in flags
    for name, flag in (("d5120_L18432_bf16wo", "wo_bf16"), ("d5120_L18432_bf16qkv", "qkv_int8")):
        v = W[name]
        assert (v.T, v.H, v.W, v.d, v.d_ff) == (base.T, base.H, base.W, base.d, base.d_ff)
        assert getattr(v, flag) != getattr(base, flag)
    small = synth.WORKLOADS["d256_L512"].with_(wo_bf16=True)
    w = synth.block_weights(small)
    assert np.array_equal(w["wo_bf16"], synth.f32_to_bf16_bits(w["wo"]))
    # ranges of the multi-block variants lie inside the pass; merging clears them
    for name, field in (("d5120_depth50_T8_pairmid", "pair_blocks"), ("d5120_depth50_T8_reuse", "reuse_blocks")):
        v = W[name]
        first, last = getattr(v, field)
        assert 0 <= first < last <= v.n_blocks == 50
        m = v.merged()
        assert m.pair_blocks == (0, 0) and m.reuse_blocks == (0, 0) and m.W == v.W // 2
