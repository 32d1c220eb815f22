"""The benchmark's work model, on the CPU: the algorithmic work bench.py divides
by each kernel's device time (the numerator of every roofline fraction it prints)
equals the closed forms of the block's arithmetic.

Per block over R = B*L tokens, model width d, MLP width F:
  QKV 2*R*3d*d, output projection 2*R*d*d, W1 and W2 2*R*d*F multiply-add ops
  (24*R*d^2 in all when F = 4d); attention 4*B*L^2*d flops (QK^T and PV);
  fused LN + modulation + quantizer: read 2d bytes, write d codes, a 4-byte
  scale and a 4-byte zeroed absmax per token; quantizer of a width-n row: read
  2n, write n, read the 4-byte absmax, write the 4-byte scale;
  token pairing: read 2d per original token, write d/2 tokens' worth (2 bytes
  each) to each of its two destinations; unpairing: read x (2d) and the merged
  xm and ym (d each) per original token, write 2d."""
import pytest

import bench
from video_diffusion_transformer_adaln_b200 import synth

GEMMS = ("gemm_qkv", "gemm_wo", "gemm_w1", "gemm_w2")


def work(name, wl):
    return bench.kernel_work(name, wl)[0]


@pytest.mark.parametrize("name", ["d256_L512", "d2048_L4096", "d5120_L18432"])
def test_tensor_work_closed_forms(name):
    wl = synth.WORKLOADS[name]
    R, d, F = wl.B * wl.L, wl.d, wl.d_ff
    assert F == 4 * d
    assert sum(work(k, wl) for k in GEMMS) == 24 * R * d * d
    assert work("gemm_qkv", wl) == 2 * R * 3 * d * d
    assert work("attention", wl) == 4 * wl.B * wl.L ** 2 * d


def test_largest_block_matches_the_quoted_totals():
    # 18432 tokens, d = 5120: 1.16e13 int8 ops and 6.96e12 attention flops per block
    wl = synth.WORKLOADS["d5120_L18432"]
    assert abs(sum(work(k, wl) for k in GEMMS) / 1.16e13 - 1) < 0.005
    assert abs(work("attention", wl) / 6.96e12 - 1) < 0.005


@pytest.mark.parametrize("name", ["d2048_L4096", "d5120_L18432"])
def test_memory_bound_bytes_per_token(name):
    wl = synth.WORKLOADS[name]
    R, d, F = wl.B * wl.L, wl.d, wl.d_ff
    assert work("ln_mod_quant", wl) == R * (3 * d + 8)
    assert work("ln_mod_quant_mlp", wl) == R * (3 * d + 8)
    assert work("quant_o", wl) == R * (3 * d + 8)
    assert work("quant_g", wl) == R * (3 * F + 8)
    assert work("adaln_gemv", wl) == 12 * d * d + wl.B * 28 * d
    for k in ("gemm_qkv", "attention"):
        assert bench.kernel_work(k, wl)[2].startswith("tensor")
    for k in ("ln_mod_quant", "quant_g", "adaln_gemv"):
        assert bench.kernel_work(k, wl)[2] == "hbm"


def test_token_reduction_work():
    wl = synth.WORKLOADS["d5120_L18432_pair"]
    R, d = wl.B * wl.L, wl.d
    assert work("token_pair", wl) == R * 4 * d
    assert work("token_unpair", wl) == R * 6 * d
    # the block between them runs on the merged grid of L/2 tokens
    assert work("gemm_qkv", wl) == 2 * (R // 2) * 3 * d * d
    assert work("attention", wl) == 4 * wl.B * (wl.L // 2) ** 2 * d


def test_partially_paired_pass_averages_over_its_blocks():
    wl = synth.WORKLOADS["d5120_depth50_T8_pairmid"]
    first, last = wl.pair_blocks
    n_m = last - first
    d, L = wl.d, wl.L
    per_launch = (n_m * 2 * (L // 2) * 3 * d * d + (wl.n_blocks - n_m) * 2 * L * 3 * d * d) / wl.n_blocks
    assert work("gemm_qkv", wl) == pytest.approx(per_launch, rel=1e-12)


def test_variant_precisions_pick_their_roofline():
    assert bench.kernel_work("gemm_qkv", synth.WORKLOADS["d5120_L18432_bf16qkv"])[2] == "tensor_bf16"
    assert bench.kernel_work("gemm_wo", synth.WORKLOADS["d5120_L18432_bf16wo"])[2] == "tensor_bf16"
    assert bench.kernel_work("gemm_wo", synth.WORKLOADS["d5120_L18432"])[2] == "tensor_i8"
