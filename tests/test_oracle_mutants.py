"""Planted mistakes in a copy of the oracle: the pins must catch every one.

Each mutant below is one plausible slip written into a private copy of
oracle/h3_oracle.cpp: a wrong sign, index, constant, operand, rounding mode or
modulation chunk, or a dropped term. The copy is built into a temporary library
and swapped in for the real one while the oracle's pin tests run against it
(test_oracle_pins.py, test_oracle_block.py, test_oracle_block_composed.py). A
mutant that passes every pin is a mistake the pins would let through, and fails
this test.

Every mutant reads and writes only inside the buffers the original touches, so a
mutated library cannot corrupt the test process. An unmutated copy built the same
way must pass every pin (the control).
"""
import ctypes
import importlib.util
import inspect
import os
import subprocess

import pytest

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "h3_oracle.cpp")
PIN_MODULES = ("test_oracle_pins", "test_oracle_block", "test_oracle_block_composed")
# Same IEEE-preserving flags as the oracle's own build; -O1 builds faster and,
# without fast-math, rounds identically.
CXX = ["g++", "-O1", "-march=x86-64-v3", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
       "-fPIC", "-shared", "-std=c++17"]

# (name, where the home pins live, exact original text, mutated text)
MUTANTS = [
    # bf16 rounding
    ("bf16_ties_away", "step", "r = std::nearbyint(std::ldexp(a, -q));", "r = std::round(std::ldexp(a, -q));"),
    ("bf16_seven_bits", "step", "int q = e - 8;", "int q = e - 7;"),
    ("bf16_no_subnormals", "step", "if (q < -133) q = -133;", "if (q < -126) q = -126;"),
    ("bf16_rounds_via_float", "step", "double a = std::fabs(v);", "double a = std::fabs((double)(float)v);"),
    # quantizer
    ("quant_scale_128", "step", "const float scale = absmax / 127.0f;", "const float scale = absmax / 128.0f;"),
    ("quant_truncates", "step", "float t = std::nearbyint(row[c] / scale);", "float t = std::trunc(row[c] / scale);"),
    ("quant_absmax_signed", "step", "absmax = std::max(absmax, std::fabs(row[c]));",
     "absmax = std::max(absmax, row[c]);"),
    # GEMMs and dequantization
    ("gemm_i8_reversed_k", "step", "acc += (int32_t)a[k] * (int32_t)w[k];", "acc += (int32_t)a[k] * (int32_t)w[K - 1 - k];"),
    ("gemm_i8_no_overflow_check", "step", "if (acc > INT32_MAX || acc < INT32_MIN) ++overflow;", "(void)0;"),
    ("gemm_f64_reversed_k", "block", "acc += a[k] * w[k];", "acc += a[k] * w[K - 1 - k];"),
    ("dequant_channel_index", "step", "* (double)s_ch[c] +", "* (double)s_ch[r % cols] +"),
    ("dequant_no_bias", "step", "(bias ? (double)bias[c] : 0.0)", "0.0"),
    # AdaLN, LayerNorm, modulation
    ("adaln_no_bias", "step", "mod[j] = acc + (b_ada ? (double)b_ada[j] : 0.0);", "mod[j] = acc;"),
    ("adaln_transposed", "step", "orc_bf16_to_f64(w_ada[j * d + k])", "orc_bf16_to_f64(w_ada[k * 6 * d + j])"),
    ("ln_unbiased_var", "step", "var /= (double)d;", "var /= (double)(d - 1);"),
    ("ln_eps_outside_sqrt", "step", "const double inv = 1.0 / std::sqrt(var + eps);",
     "const double inv = 1.0 / (std::sqrt(var) + eps);"),
    ("modulate_scale_without_one", "step", "y[r * d + i] * (1.0 + scale[i]) + shift[i]", "y[r * d + i] * scale[i] + shift[i]"),
    ("modulate_shift_scale_swapped", "step", "y[r * d + i] * (1.0 + scale[i]) + shift[i]",
     "y[r * d + i] * (1.0 + shift[i]) + scale[i]"),
    # grid and RoPE
    ("grid_row_index", "step", "hp[i] = (int32_t)((i / W) % H);", "hp[i] = (int32_t)((i / H) % W);"),
    ("rope_sign", "step", "v[lane] = x0 * c - x1 * s;", "v[lane] = x0 * c + x1 * s;"),
    ("rope_frequency_exponent", "step", "std::pow(theta, -2.0 * j / (double)seg_len)", "std::pow(theta, -1.0 * j / (double)seg_len)"),
    ("rope_row_uses_column", "step", "seg_start = rt; seg_len = rh; pos = hp[r];", "seg_start = rt; seg_len = rh; pos = wp[r];"),
    ("rope_pair_index_global", "step", "const int j = (lane - seg_start) / 2;", "const int j = lane / 2;"),
    # attention, GELU, gated residual
    ("attn_no_scale", "step", "sc[(size_t)j] = dot * inv_sqrt;", "sc[(size_t)j] = dot;"),
    ("attn_unnormalised", "step", "const double p = sc[(size_t)j] / sum;", "const double p = sc[(size_t)j];"),
    ("gelu_square_not_cube", "step", "(v + 0.044715 * v * v * v)", "(v + 0.044715 * v * v)"),
    ("gelu_drops_x", "step", "y[i] = 0.5 * v * (1.0 +", "y[i] = 0.5 * (1.0 +"),
    ("residual_ungated", "step", "out[r * d + i] = x[r * d + i] + gate[i] * y[r * d + i];",
     "out[r * d + i] = x[r * d + i] + y[r * d + i];"),
    # token reduction and residual reuse
    ("pair_sum_not_mean", "step", "orc_f64_to_bf16((a + b) / 2.0)", "orc_f64_to_bf16(a + b)"),
    ("pair_wrong_partner", "step", "x[(row * W + 2 * k + 1) * d + i]", "x[(row * W + k) * d + i]"),
    ("unpair_delta_sign", "step", "(ym[m] - orc_bf16_to_f64(xm[m]))", "(orc_bf16_to_f64(xm[m]) - ym[m])"),
    ("unpair_merged_index", "step", "const int64_t m = (row * Wm + w / 2) * d + i;",
     "const int64_t m = (row * Wm + w % Wm) * d + i;"),
    ("range_delta_sign", "step", "delta[i] = orc_bf16_to_f64(after[i]) - orc_bf16_to_f64(before[i]);",
     "delta[i] = orc_bf16_to_f64(before[i]) - orc_bf16_to_f64(after[i]);"),
    # the block's wiring
    ("block_attn_chunks_swapped", "block", "L, d, chunk(b, 0), chunk(b, 1),", "L, d, chunk(b, 1), chunk(b, 0),"),
    ("block_mlp_chunks_swapped", "block", "chunk(b, 3), chunk(b, 4)", "chunk(b, 4), chunk(b, 3)"),
    ("block_attn_gate_is_mlp_gate", "block", "chunk(b, 2), 1, d, &x1", "chunk(b, 5), 1, d, &x1"),
    ("block_mlp_gate_is_attn_gate", "block", "chunk(b, 5), 1, d, &out", "chunk(b, 2), 1, d, &out"),
    ("block_k_v_swapped", "block", "&K[(size_t)(b * L * d)], &V[(size_t)(b * L * d)], 1, L,",
     "&V[(size_t)(b * L * d)], &K[(size_t)(b * L * d)], 1, L,"),
    ("block_k_from_v_columns", "block", "K[(size_t)(r * d + i)] = qkv[(size_t)(r * 3 * d + d + i)];",
     "K[(size_t)(r * d + i)] = qkv[(size_t)(r * 3 * d + 2 * d + i)];"),
    ("block_rope_on_v_not_k", "block", "orc_rope_3d(&K[(size_t)(b * L * d)], L,", "orc_rope_3d(&V[(size_t)(b * L * d)], L,"),
    ("block_o_not_rounded", "block", "Of[(size_t)i] = (float)orc_bf16_to_f64(orc_f64_to_bf16(O[(size_t)i]));",
     "Of[(size_t)i] = (float)O[(size_t)i];"),
    ("block_gelu_not_rounded", "block", "gf[(size_t)i] = (float)orc_bf16_to_f64(orc_f64_to_bf16(g[(size_t)i]));",
     "gf[(size_t)i] = (float)g[(size_t)i];"),
    ("block_mlp_ln_of_x", "block", "orc_layernorm(x1.data(), n_rows, d,", "orc_layernorm(xd.data(), n_rows, d,"),
    ("block_no_gelu", "block", "orc_gelu_tanh(pre.data(), n_rows * F, g.data());", "g = pre;"),
    ("block_w2_with_w1_scales", "block", "s4.data(), wt->s2, wt->b2", "s4.data(), wt->s1, wt->b2"),
    ("block_attn_keys_of_item0", "block", "const int64_t r = sel[(size_t)i], b = r / L;\n    orc_attention(",
     "const int64_t r = sel[(size_t)i], b = 0;\n    orc_attention("),
    ("block_final_residual_from_x", "block", "orc_gated_residual(&x1[(size_t)(i * d)], &y4",
     "orc_gated_residual(&xd[(size_t)(sel[(size_t)i] * d)], &y4"),
    ("block_rows_ignored", "block", "sel[(size_t)i] = rows ? rows[i] : i;", "sel[(size_t)i] = i;"),
    ("block_bf16_qkv_no_bias", "block", "qkv[(size_t)(r * 3 * d + o)] += wt->bqkv[o];", "(void)0;"),
    ("block_bf16_wo_no_bias", "block", "yo[(size_t)(r * d + o)] += wt->bo[o];", "(void)0;"),
    ("block_v_not_rounded", "block", "V[i] = orc_bf16_to_f64(orc_f64_to_bf16(V[i]));", "(void)0;"),
]


def _load_pins():
    mods = {}
    for name in PIN_MODULES:
        spec = importlib.util.spec_from_file_location("_mutant_pins_" + name, os.path.join(HERE, name + ".py"))
        m = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(m)
        mods[name] = [f for n, f in sorted(vars(m).items())
                      if n.startswith("test_") and callable(f) and not inspect.signature(f).parameters]
    return mods["test_oracle_pins"], mods["test_oracle_block"] + mods["test_oracle_block_composed"]


@pytest.fixture(scope="module")
def built(tmp_path_factory):
    """Build the control copy and every mutant, a few compilers at a time."""
    src = open(SRC).read()
    out_dir = tmp_path_factory.mktemp("oracle_mutants")
    jobs = [("control", src)]
    for name, _, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: the original text must occur exactly once"
        jobs.append((name, src.replace(old, new)))
    libs, running = {}, []
    width = max(1, min(8, os.cpu_count() or 1))
    for name, text in jobs:
        cpp = out_dir / f"{name}.cpp"
        cpp.write_text(text)
        so = str(out_dir / f"lib{name}.so")
        running.append((name, so, subprocess.Popen(CXX + [str(cpp), "-o", so])))
        if len(running) >= width:
            n, s, p = running.pop(0)
            assert p.wait() == 0, f"{n} did not build"
            libs[n] = s
    for n, s, p in running:
        assert p.wait() == 0, f"{n} did not build"
        libs[n] = s
    return libs, _load_pins()


def _first_failing_pin(lib_path, pins):
    """Run the pins against the library at lib_path; the name of the first one that
    fails, or None when all pass. The real oracle library is restored afterwards."""
    O.lib()  # make sure the real library is loaded, so that it is what gets restored
    saved = O._LIB
    mutant = ctypes.CDLL(lib_path)
    O._declare(mutant)
    O._LIB = mutant
    try:
        for fn in pins:
            try:
                fn()
            except (Exception, pytest.fail.Exception):
                return fn.__name__
        return None
    finally:
        O._LIB = saved


def test_control_copy_passes_every_pin(built):
    libs, (step_pins, block_pins) = built
    assert _first_failing_pin(libs["control"], step_pins + block_pins) is None


@pytest.mark.parametrize("name,home", [(m[0], m[1]) for m in MUTANTS], ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(built, name, home):
    libs, (step_pins, block_pins) = built
    order = step_pins + block_pins if home == "step" else block_pins + step_pins
    assert _first_failing_pin(libs[name], order) is not None, f"mutant {name} passes every pin"
