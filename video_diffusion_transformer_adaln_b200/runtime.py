"""Device-side holders for the block's inputs, weights and workspace.

PyTorch is used only to allocate device memory and to move bytes; the weights'
per-output-channel quantization runs in the library (h3b_quantize_weights).
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np
import torch

from . import h3b
from .synth import Workload


def dims_of(wl: Workload) -> h3b.Dims:
    return h3b.make_dims(wl.B, wl.T, wl.H, wl.W, wl.d, wl.n_heads, wl.head_dim, wl.d_ff, wl.rope,
                         wl.rope_theta, wl.ln_eps, wl.qkv_int8, wl.wo_bf16)


def bf16_from_bits(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def bits_from_bf16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def quantize_weight(w: torch.Tensor):
    """fp32 [rows][cols] device tensor -> (int8 codes, fp32 scales) via the library."""
    rows, cols = w.shape
    q = torch.empty((rows, cols), dtype=torch.int8, device=w.device)
    s = torch.empty(rows, dtype=torch.float32, device=w.device)
    h3b.h3b_quantize_weights(w, q, s)
    return q, s


class DeviceBlock:
    """One block's weights in device memory, in the layout the C ABI takes."""

    def __init__(self, tensors: Dict[str, torch.Tensor]):
        self.tensors = tensors
        self.struct = h3b.make_weights(tensors)

    @classmethod
    def from_host(cls, raw: dict, qkv_int8: bool = True, device="cuda") -> "DeviceBlock":
        """raw: host arrays from synth.block_weights (fp32 projections, bf16 AdaLN)."""
        t = {"w_ada": bf16_from_bits(raw["w_ada"], device),
             "b_ada": torch.from_numpy(raw["b_ada"]).to(device)}
        for name, sname in (("wqkv", "sqkv"), ("wo", "so"), ("w1", "s1"), ("w2", "s2")):
            if name == "wqkv" and not qkv_int8:
                continue
            w32 = torch.from_numpy(raw[name]).to(device)
            t[name], t[sname] = quantize_weight(w32)
            del w32
        if not qkv_int8:
            t["wqkv_bf16"] = bf16_from_bits(raw["wqkv_bf16"], device)
        if "wo_bf16" in raw:
            t["wo_bf16"] = bf16_from_bits(raw["wo_bf16"], device)
        return cls(t)

    @classmethod
    def random_on_device(cls, wl: Workload, generator: torch.Generator, device="cuda") -> "DeviceBlock":
        """Same distributions as synth.block_weights, drawn by a seeded device RNG
        (for workloads too large to generate on the host)."""
        d, F = wl.d, wl.d_ff
        w_ada = torch.zeros((6 * d, d), dtype=torch.bfloat16, device=device)
        for k in (0, 1, 3, 4):
            w_ada[k * d:(k + 1) * d] = (torch.randn((d, d), generator=generator, device=device) / d ** 0.5).to(
                torch.bfloat16)
        b_ada = torch.zeros(6 * d, dtype=torch.float32, device=device)
        b_ada[2 * d:3 * d] = torch.randn(d, generator=generator, device=device) * 0.5 ** 0.5
        b_ada[5 * d:] = torch.randn(d, generator=generator, device=device) * 0.5 ** 0.5
        t = {"w_ada": w_ada, "b_ada": b_ada}
        for name, sname, n_out, n_in in (("wqkv", "sqkv", 3 * d, d), ("wo", "so", d, d),
                                         ("w1", "s1", F, d), ("w2", "s2", d, F)):
            w32 = torch.randn((n_out, n_in), generator=generator, device=device) / n_in ** 0.5
            if name == "wqkv" and not wl.qkv_int8:
                t["wqkv_bf16"] = w32.to(torch.bfloat16)
            elif name == "wo" and wl.wo_bf16:
                t["wo_bf16"] = w32.to(torch.bfloat16)
            else:
                t[name], t[sname] = quantize_weight(w32)
            del w32
        return cls(t)


def workspace(dims: h3b.Dims, device="cuda") -> torch.Tensor:
    n = h3b.h3b_workspace_size(dims)
    return torch.empty(n, dtype=torch.uint8, device=device)


def block_forward(dims: h3b.Dims, blk: DeviceBlock, c: torch.Tensor, x: torch.Tensor, ws: torch.Tensor):
    h3b.h3b_block_forward(dims, blk.struct, c, x, ws)


def blocks_forward(dims: h3b.Dims, blocks: List[DeviceBlock], c: torch.Tensor, x: torch.Tensor,
                   ws: torch.Tensor):
    h3b.h3b_blocks_forward(dims, [b.struct for b in blocks], c, x, ws)


def paired_block_forward(full: h3b.Dims, merged: h3b.Dims, blk: DeviceBlock, c: torch.Tensor, x: torch.Tensor,
                         ws: torch.Tensor, ym: Optional[torch.Tensor] = None):
    """Token reduction around one block: pair -> block on the merged grid -> unpair (in place
    on x). The pairing writes the merged tokens once, into ym, where the block then runs; the
    unpairing recomputes the merged input from x. Returns ym (the block's merged output)."""
    shape = (full.B, full.T, full.H, full.W // 2, full.d)
    ym = ym if ym is not None else torch.empty(shape, dtype=torch.bfloat16, device=x.device)
    h3b.h3b_token_pair(full, x, ym)
    h3b.h3b_block_forward(merged, blk.struct, c, ym, ws)
    h3b.h3b_token_unpair(full, x, None, ym, x)
    return ym
