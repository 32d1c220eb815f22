"""The checked build of the library (libh3b_checked.so), and launches without
programmatic dependent launch, on the block and its steps.

In the checked build every kernel tests each global-memory index it computes
against the extent of its buffer before the access; an index outside records
bit 1 << 6 in the device error word and the access is skipped. It stands in for
a memory checker, which cannot run here. The test runs the block (two batch
items, and a ragged grid), attention at a ragged length, the fused LN
quantizer, the quantizer with a known absmax, token pairing and unpairing, the
raw int8 GEMM at ragged sizes and the QKV projection, first with the normal
library in this process and then with the checked library in a child process
(the binding picks the library when it is first loaded). The checked run must
leave the error word clear, and its outputs must equal the normal build's bit
for bit: the checks change no arithmetic.

The same cases (with the bf16-output GEMM epilogues at ragged sizes, whose TMA
stores the hardware clips at M and N, and a two-block pass) run once more in a
child process with H3B_PDL=0, which launches every kernel without the
programmatic-serialization attribute: the outputs must again be identical, so
the early launch of a grid ahead of its grid-dependency wait changes nothing."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from gpu_helpers import bf16_dev, bf16_host, require_gpu, to_dev

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def run_cases():
    """Every case's outputs as numpy arrays (bf16 as uint16 bit patterns)."""
    import oracle as O
    from video_diffusion_transformer_adaln_b200 import h3b, synth
    from video_diffusion_transformer_adaln_b200.runtime import (DeviceBlock, block_forward, blocks_forward, dims_of,
                                                                workspace)

    out = {}
    r = np.random.default_rng(5)
    for name, wl in (("block_b2", synth.WORKLOADS["d256_L512"].with_(B=2)),
                     ("block_ragged", synth.WORKLOADS["d256_L512"].with_(T=3, H=5, W=7))):
        raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
        dims = dims_of(wl)
        blk = DeviceBlock.from_host(raw)
        xd = bf16_dev(x)
        block_forward(dims, blk, to_dev(c), xd, workspace(dims))
        out[name] = bf16_host(xd)
    # a two-block pass (grids of consecutive blocks launched back to back)
    wl = synth.WORKLOADS["d256_L512"]
    dims = dims_of(wl)
    blocks = [DeviceBlock.from_host(synth.block_weights(wl, block=b)) for b in (0, 1)]
    xd = bf16_dev(synth.x_input(wl))
    blocks_forward(dims, blocks, to_dev(synth.cond(wl)), xd, workspace(dims))
    out["blocks2"] = bf16_host(xd)
    # attention at a ragged length
    B, H, L, dh = 2, 2, 777, 128
    qkv = synth.f32_to_bf16_bits(r.standard_normal((3, B, H, L, dh)).astype(np.float32))
    wl = synth.Workload("attn", 1, 1, L, H * dh, H, dh, 256, (0, 0, dh), 0, B=B)
    o = torch.empty((B, L, H * dh), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(B * L, dtype=torch.float32, device="cuda")
    h3b.h3b_attention(dims_of(wl), bf16_dev(qkv), o, am)
    out["attention"], out["attention_absmax"] = bf16_host(o), am.cpu().numpy()
    # fused LN quantizer, two batch items
    rows, d = 37, 2048
    x = synth.f32_to_bf16_bits(r.standard_normal((rows, d)).astype(np.float32))
    sh = to_dev((r.standard_normal((2, d)) * 0.1).astype(np.float32))
    sc = to_dev((r.standard_normal((2, d)) * 0.1).astype(np.float32))
    q = torch.empty((rows, d), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    h = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    h3b.h3b_ln_modulate_quantize(bf16_dev(x), rows, d, 1e-6, sh, sc, 20, d, q, s, h_out=h)
    out["ln_q"], out["ln_s"], out["ln_h"] = q.cpu().numpy(), s.cpu().numpy(), bf16_host(h)
    # quantizer with a known absmax
    rows, cols = 129, 20480
    hq = synth.f32_to_bf16_bits(r.standard_normal((rows, cols)).astype(np.float32))
    amx = to_dev(np.abs(synth.bf16_bits_to_f32(hq)).max(axis=1).astype(np.float32))
    q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    h3b.h3b_quantize_rows(bf16_dev(hq), q, s, absmax=amx)
    out["quant_q"], out["quant_s"] = q.cpu().numpy(), s.cpu().numpy()
    # token pairing and unpairing
    full = h3b.make_dims(2, 1, 3, 6, 8, 1, 64, 256, (0, 0, 64))
    xp = synth.f32_to_bf16_bits(r.standard_normal((2, 1, 3, 6, 8)).astype(np.float32))
    xm = torch.empty((2, 1, 3, 3, 8), dtype=torch.bfloat16, device="cuda")
    h3b.h3b_token_pair(full, bf16_dev(xp), xm)
    ym = synth.f32_to_bf16_bits(r.standard_normal((2, 1, 3, 3, 8)).astype(np.float32))
    un = torch.empty((2, 1, 3, 6, 8), dtype=torch.bfloat16, device="cuda")
    h3b.h3b_token_unpair(full, bf16_dev(xp), None, bf16_dev(ym), un)
    out["pair"], out["unpair"] = bf16_host(xm), bf16_host(un)
    # raw int8 GEMM at ragged sizes
    M, N, K = 300, 272, 144
    A = r.integers(-127, 128, (M, K), dtype=np.int8)
    W = r.integers(-127, 128, (N, K), dtype=np.int8)
    Cg = torch.empty((M, N), dtype=torch.int32, device="cuda")
    h3b.h3b_gemm_i8_s32(to_dev(A), to_dev(W), Cg)
    out["gemm_s32"] = Cg.cpu().numpy()
    # bf16-output epilogues at ragged sizes: 100 rows (a partial 32-row box) and 272 columns
    # (a partial 32-column chunk); the gated residual's 34 rows per item straddle warps
    M, N, K = 100, 272, 160
    A = to_dev(r.integers(-127, 128, (M, K), dtype=np.int8))
    W = to_dev(r.integers(-127, 128, (N, K), dtype=np.int8))
    sa = to_dev(r.uniform(1e-3, 1e-2, M).astype(np.float32))
    sw = to_dev(r.uniform(1e-3, 1e-2, N).astype(np.float32))
    bias = to_dev((r.standard_normal(N) * 0.1).astype(np.float32))
    o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h3b.h3b_gemm_i8_dequant(A, sa, W, sw, bias, o)
    out["gemm_dequant"] = bf16_host(o)
    g = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(M, dtype=torch.float32, device="cuda")
    h3b.h3b_gemm_i8_gelu(A, sa, W, sw, bias, g, am)
    out["gemm_gelu"], out["gemm_gelu_absmax"] = bf16_host(g), am.cpu().numpy()
    xr = bf16_dev(synth.f32_to_bf16_bits(r.standard_normal((M, N)).astype(np.float32)))
    gate = to_dev(r.standard_normal((3, N)).astype(np.float32))
    h3b.h3b_gemm_i8_gated_residual(A, sa, W, sw, bias, gate, 34, N, xr)
    out["gemm_resid"] = bf16_host(xr)
    # QKV projection with RoPE, head-major
    wl = synth.WORKLOADS["d256_L512"]
    raw = synth.block_weights(wl)
    dims = dims_of(wl)
    qa, sa = O.quantize_rows((r.standard_normal((wl.L, wl.d)) * 2).astype(np.float32))
    qkv_out = torch.empty(3 * wl.L * wl.d, dtype=torch.bfloat16, device="cuda")
    rope_ws = torch.empty(h3b.h3b_rope_table_bytes(dims), dtype=torch.uint8, device="cuda")
    h3b.h3b_qkv_projection(dims, to_dev(qa), to_dev(sa), DeviceBlock.from_host(raw).struct, qkv_out, rope_ws)
    out["qkv"] = bf16_host(qkv_out)
    torch.cuda.synchronize()
    out["error_word"] = np.array([h3b.h3b_device_error(clear=True)], np.uint32)
    out["checked"] = np.array([int(h3b.h3b_checked_build())], np.int32)
    return out


def child(path):
    np.savez(path, **run_cases())


def test_checked_build_matches_the_normal_build_and_records_nothing(tmp_path):
    require_gpu()
    from video_diffusion_transformer_adaln_b200 import build
    build.build(checked=True)
    ref = run_cases()
    assert ref["checked"][0] == 0 and ref["error_word"][0] == 0
    path = str(tmp_path / "checked.npz")
    env = dict(os.environ, H3B_CHECKED="1")
    code = f"import sys; sys.path[:0] = [{HERE!r}, {os.path.dirname(HERE)!r}]; import test_gpu_checked as t; t.child({path!r})"
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = dict(np.load(path))
    assert got["checked"][0] == 1
    assert got["error_word"][0] == 0, f"checked build recorded error word {got['error_word'][0]:#x}"
    for k, v in ref.items():
        if k in ("checked", "error_word"):
            continue
        assert np.array_equal(got[k], v), k


def test_launches_without_dependent_launch_match(tmp_path):
    require_gpu()
    ref = run_cases()
    assert ref["checked"][0] == 0 and ref["error_word"][0] == 0
    path = str(tmp_path / "no_pdl.npz")
    env = dict(os.environ, H3B_PDL="0")
    env.pop("H3B_CHECKED", None)
    code = f"import sys; sys.path[:0] = [{HERE!r}, {os.path.dirname(HERE)!r}]; import test_gpu_checked as t; t.child({path!r})"
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = dict(np.load(path))
    assert got["checked"][0] == 0 and got["error_word"][0] == 0
    for k, v in ref.items():
        assert np.array_equal(got[k], v), k
