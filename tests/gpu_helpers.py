"""Shared helpers for the GPU parity tests: moving bytes between numpy and
torch, tolerance metrics, and the oracle-side view of a block's weights."""
import numpy as np
import pytest
import torch

import oracle as O
from video_diffusion_transformer_adaln_b200 import build, h3b, synth
from video_diffusion_transformer_adaln_b200.runtime import bf16_from_bits, bits_from_bf16


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    h3b.lib()


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16_dev(bits):
    return bf16_from_bits(bits, "cuda")


def bf16_host(t):
    return bits_from_bf16(t)


def bf16_f64(bits):
    """bf16 bit patterns as float64 (exact), decoded in numpy: GPU results are
    compared without passing through the oracle."""
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def rel_l2(a, ref):
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm((a - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def bf16_ulp_diff(a_bits, b_bits):
    """Distance in bf16 units in the last place (same-sign finite values)."""
    a = np.asarray(a_bits, np.uint16).astype(np.int32)
    b = np.asarray(b_bits, np.uint16).astype(np.int32)
    # map sign-magnitude to a monotone integer line
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(a - b)


def no_device_error():
    code = h3b.h3b_device_error(clear=True)
    assert code == 0, f"device error word = {code:#x}"


def oracle_weights(raw, qkv_int8=True):
    """The oracle's own per-output-channel quantization of the fp32 draws."""
    w = {"w_ada": raw["w_ada"], "b_ada": raw["b_ada"]}
    for name, sname in (("wqkv", "sqkv"), ("wo", "so"), ("w1", "s1"), ("w2", "s2")):
        w[name], w[sname] = O.quantize_rows(raw[name])
    if not qkv_int8:
        w["wqkv_bf16"] = raw["wqkv_bf16"]
    if "wo_bf16" in raw:
        w["wo_bf16"] = raw["wo_bf16"]
    return w


def oracle_dims(wl):
    return O.Dims(wl.B, wl.T, wl.H, wl.W, wl.d, wl.n_heads, wl.head_dim, wl.d_ff, wl.rope, wl.rope_theta,
                  wl.ln_eps, wl.qkv_int8, wl.wo_bf16)
