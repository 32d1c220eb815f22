"""The benchmark's work model, on the CPU: the algorithmic work bench.py divides
by each kernel's device time (the numerator of every roofline fraction it prints)
equals the closed forms of the block's arithmetic.

Per block over R = B*L tokens, model width d, MLP width F:
  QKV 2*R*3d*d, output projection 2*R*d*d, W1 and W2 2*R*d*F multiply-add ops
  (24*R*d^2 in all when F = 4d); attention 4*B*L^2*d flops (QK^T and PV);
  fused LN + modulation + quantizer: read 2d bytes, write d codes, a 4-byte
  scale and a 4-byte zeroed absmax per token; quantizer of a width-n row: read
  2n, write n, read the 4-byte absmax, write the 4-byte scale;
  token pairing: read 2d per original token, write the merged tokens once (d
  per original token); unpairing: read x (2d) and the block's merged output
  ym (d) per original token, write 2d (the merged input is recomputed from x).

The reference arm (the CPU oracle) is also run here end to end: it needs no GPU,
and its JSON line follows the same contract as the CUDA arm's."""
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
    assert work("token_pair", wl) == R * 3 * d
    assert work("token_unpair", wl) == R * 5 * d
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


def _run_bench(args, env_extra=None, timeout=600):
    import json
    import os
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, capture_output=True, text=True,
                       timeout=timeout, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_prints_one_contract_line():
    # The reference arm is the CPU oracle (no GPU needed): one JSON line with the same
    # metric and unit as the CUDA arm, its own cpu_baseline and an e2e with no copies.
    out = _run_bench(["--impl", "reference", "--workload", "d256_L512", "--steps", "3", "--warmup", "3"])
    assert len(out) == 1
    line = out[0]
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 3, 3)
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["config"]["workload"] == "d256_L512"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    # the smallest block runs whole each step: value is its tokens over the step time
    assert line["extrapolated"] is False
    assert line["value"] == pytest.approx(512 / (line["ms_per_step"] / 1e3), rel=1e-3)
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_0_only():
    assert _run_bench(["--impl", "reference", "--workload", "d256_L512", "--steps", "3", "--warmup", "3"],
                      {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_bench_rejects_fewer_than_three_warmup_steps():
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr


def test_clock_summary_of_nvidia_smi_rows():
    rows = "\n".join([
        "1965, 1965, 310.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1920, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1890, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "345, 1965, 120.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",  # idle
        "[N/A], 1965, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",
        "garbage line",
    ])
    c = bench.ClockSampler.summarize(rows)
    assert c["sm_mhz"] == 1920.0  # median of the busy samples 1965, 1920, 1890
    assert c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 5
    hot = bench.ClockSampler.summarize("1500, 1965, 700, 0x40, Not Active, Active, Not Active, Not Active")
    assert hot["reasons"] == ["hw_thermal_slowdown"]
    assert bench.ClockSampler.summarize("") is None
    assert bench.ClockSampler.summarize("[N/A], [N/A], 1, 2, 3, 4, 5, 6")["sm_mhz"] is None


def test_roofline_summary_of_a_profile():
    # 10 steps of the d=2048 block: attention 1.50 ms over 10 launches (dominant), QKV 0.60 ms,
    # the attention LN quantizer 0.20 ms
    wl = synth.WORKLOADS["d2048_L4096"]
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    prof = {"attention": (10, 1.5), "gemm_qkv": (10, 0.6), "ln_mod_quant": (10, 0.2)}
    roof, shares, all_roof = bench.roofline_summary(prof, wl, peaks, "measured")
    assert list(shares) == ["attention", "gemm_qkv", "ln_mod_quant"]
    assert shares["attention"] == pytest.approx(1.5 / 2.3, abs=1e-4)
    flops = 4.0 * wl.L ** 2 * wl.d
    assert roof["kernel"] == "attention" and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] == pytest.approx(flops / 150e-6 / 1e12, abs=0.01)
    # kernels timed inside the steps: the sustained figure, with the burst one beside it
    assert roof["peak"] == 1400.0 and roof["frac"] == pytest.approx(roof["achieved"] / 1400.0, abs=1e-4)
    assert roof["peak_burst"] == 1600.0 and roof["frac_burst"] == pytest.approx(roof["achieved"] / 1600.0, abs=1e-4)
    assert roof["launch_ms"] == 0.15 and roof["work_per_launch"] == flops
    # the int8 GEMM against twice the bf16 peak, the LN quantizer against HBM
    ops = 2.0 * wl.L * 3 * wl.d * wl.d
    assert all_roof["gemm_qkv"]["TOP/s"] == pytest.approx(ops / 60e-6 / 1e12, abs=0.05)
    assert all_roof["gemm_qkv"]["frac"] == pytest.approx(ops / 60e-6 / 1e12 / 2800.0, abs=1e-3)
    assert all_roof["gemm_qkv"]["frac_burst"] == pytest.approx(ops / 60e-6 / 1e12 / 3200.0, abs=1e-3)
    byts = wl.L * (3 * wl.d + 8)
    assert all_roof["ln_mod_quant"]["GB/s"] == pytest.approx(byts / 20e-6 / 1e9, abs=0.05)
    assert all_roof["ln_mod_quant"]["frac"] == pytest.approx(byts / 20e-6 / 1e9 / 6500.0, abs=1e-3)
    # an empty profile gives no roofline
    assert bench.roofline_summary({}, wl, peaks, "measured") == (None, {}, {})


def test_step_blocks_of_every_workload_kind():
    wl = synth.WORKLOADS["d5120_L18432"]
    assert bench.step_blocks(wl) == ([(18432, 1)], 18432)
    assert bench.step_blocks(synth.WORKLOADS["d5120_L18432_pair"]) == ([(9216, 1)], 18432)
    assert bench.step_blocks(synth.WORKLOADS["d5120_depth50_T16"]) == ([(36864, 50)], 36864)
    # blocks 13..37 on the merged grid, the other 25 on the full grid
    assert bench.step_blocks(synth.WORKLOADS["d5120_depth50_T8_pairmid"]) == ([(9216, 25), (18432, 25)], 18432)
    # a fresh pass over 50 blocks and a reuse pass that skips 25: two denoise steps
    assert bench.step_blocks(synth.WORKLOADS["d5120_depth50_T8_reuse"]) == ([(18432, 75)], 2 * 18432)
    assert bench.block_ops(wl, wl.L) == 24 * wl.L * wl.d ** 2 + 4 * wl.L ** 2 * wl.d


def test_cpu_baseline_times_the_small_block_whole():
    orc = bench.OracleRunner(synth.WORKLOADS["d256_L512"])
    assert orc.can_time_full_block()
    v, text, extrap = orc.baseline(budget_s=30.0)
    assert v > 0 and not extrap and "no extrapolation" in text
    assert not bench.OracleRunner(synth.WORKLOADS["d5120_L18432"]).can_time_full_block()


def test_cpu_baseline_sample_extrapolates_near_the_whole_block():
    # the bounded sample (a 1x4x16 slice run whole, plus attention of 16 queries against
    # all 512 keys) against the whole block's own time, on the smallest block
    orc = bench.OracleRunner(synth.WORKLOADS["d256_L512"])
    full = min(orc.full_block() for _ in range(3))
    est = min(orc.sample(64, 16)[0] for _ in range(3))
    assert 0.2 * full < est < 5 * full, (est, full)
    assert "1x4x16 slice" in orc.sample_text(64, 16)


def test_reference_arm_sampled_steps_report_their_wall_time():
    out = _run_bench(["--impl", "reference", "--workload", "d2048_L4096", "--steps", "3", "--warmup", "3",
                      "--ref-full-ops", "0", "--ref-sub-tokens", "64", "--ref-queries", "4"])
    line = out[0]
    assert line["extrapolated"] is True and line["cpu_baseline"]["extrapolated"] is True
    # value is the step's tokens over the extrapolated step time, which is longer than
    # the bounded sample each step actually ran
    assert line["value"] == pytest.approx(4096 / (line["step_ms_extrapolated"] / 1e3), rel=1e-3)
    assert line["step_ms_extrapolated"] > line["ms_per_step"] > 0
