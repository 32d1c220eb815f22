"""Seeded synthetic workloads for the DiT block (inputs only, no block arithmetic).

Both the CUDA path and the CPU oracle are fed from here; this module computes
nothing the block computes. Random draws use numpy's Philox counter-based
generator, keyed per (base seed, workload, block, tensor, row chunk), so any
tensor of any block can be regenerated on its own, and large tensors are drawn
by several host threads with the same values for any thread count.

Distributions (model dimensions are synthetic; the pages give none):
  x        ~ N(0, 1), with a fixed set of outlier channels scaled by 16, stored bf16
  c        ~ N(0, 1) fp32, one vector of length d per block and batch item
  W_ada    bf16 [6d][d]: shift/scale rows ~ N(0, 1/d); gate rows 0
  b_ada    fp32 [6d]: 0 for shift/scale; gate entries ~ N(0, 0.5), so the gates
           themselves are N(0, 0.5)
  Wqkv, Wo, W1, W2 ~ N(0, 1/d_in) fp32 ([out][in]); quantized per output channel
           by each side's own quantizer; biases are zero (passed as NULL)
  Wqkv_bf16 = the same Wqkv draws stored bf16 (for the bf16-QKV variant)
  Wo_bf16   = the same Wo draws stored bf16 (for the bf16 output-projection variant)
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np

BASE_SEED = 20261202


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    W: int
    d: int
    n_heads: int
    head_dim: int
    d_ff: int
    rope: Tuple[int, int, int]
    n_outliers: int
    B: int = 1
    n_blocks: int = 1
    token_pair: bool = False
    qkv_int8: bool = True
    wo_bf16: bool = False
    rope_theta: float = 10000.0
    ln_eps: float = 1e-6
    # multi-block pass: blocks [first, last) run on the paired grid (empty: none)
    pair_blocks: Tuple[int, int] = (0, 0)
    # residual reuse: a step is one fresh pass (blocks [first, last) run, their delta is
    # cached) and one reuse pass (the range is replaced by the cached delta)
    reuse_blocks: Tuple[int, int] = (0, 0)

    @property
    def L(self) -> int:
        return self.T * self.H * self.W

    def merged(self) -> "Workload":
        """The grid the block sees under token reduction (W halved)."""
        assert self.W % 2 == 0
        return self.with_(name=self.name + "/merged", W=self.W // 2, token_pair=False, pair_blocks=(0, 0),
                          reuse_blocks=(0, 0))

    def with_(self, **kw) -> "Workload":
        args = dict(self.__dict__)
        args.update(kw)
        return Workload(**args)


def _large(T, **kw):
    return Workload(name=kw.pop("name"), T=T, H=48, W=48, d=5120, n_heads=40, head_dim=128,
                    d_ff=20480, rope=(32, 48, 48), n_outliers=51, **kw)


WORKLOADS: Dict[str, Workload] = {
    # one block, d=256, 4 heads x 64, MLP 1024, grid 2x16x16 = 512 tokens
    "d256_L512": Workload("d256_L512", 2, 16, 16, 256, 4, 64, 1024, (16, 24, 24), 4),
    # one block, d=2048, 16 heads x 128, MLP 8192, grid 4x32x32 = 4096 tokens
    "d2048_L4096": Workload("d2048_L4096", 4, 32, 32, 2048, 16, 128, 8192, (32, 48, 48), 20),
    # one block, d=5120, 40 heads x 128, MLP 20480, grid 8x48x48 = 18432 tokens
    "d5120_L18432": _large(8, name="d5120_L18432"),
    # the same block with bf16 QKV (int8 MLP): the A/B of QKV quantization
    "d5120_L18432_bf16qkv": _large(8, name="d5120_L18432_bf16qkv", qkv_int8=False),
    # the same block with a bf16 output projection on the bf16 attention output
    "d5120_L18432_bf16wo": _large(8, name="d5120_L18432_bf16wo", wo_bf16=True),
    # token reduction around the d=5120 block: 8x48x48 -> 8x48x24 = 9216 merged tokens
    "d5120_L18432_pair": _large(8, name="d5120_L18432_pair", token_pair=True),
}
# 50 distinct blocks at d=5120 over one latent, frame sweep T in {2,4,8,12,16}
for _T in (2, 4, 8, 12, 16):
    WORKLOADS[f"d5120_depth50_T{_T}"] = _large(_T, name=f"d5120_depth50_T{_T}", n_blocks=50)
# the same pass with token reduction over the middle half of the blocks (13..37)
WORKLOADS["d5120_depth50_T8_pairmid"] = _large(8, name="d5120_depth50_T8_pairmid", n_blocks=50,
                                               pair_blocks=(13, 38))
# two denoise steps of the pass: fresh (blocks 13..37 run, their delta cached), then reuse
WORKLOADS["d5120_depth50_T8_reuse"] = _large(8, name="d5120_depth50_T8_reuse", n_blocks=50,
                                             reuse_blocks=(13, 38))

_TENSOR_IDS = {"x": 1, "outliers": 2, "c": 3, "w_ada": 4, "b_gate": 5, "wqkv": 6, "wo": 7,
               "w1": 8, "w2": 9}


def _key(wl: Workload, seed: int, block: int, tensor: str) -> list:
    # The stream depends on the grid and model sizes, not on the variant flags, so
    # variants of one workload (bf16 QKV, token pairing) see identical draws.
    key = f"{wl.B}x{wl.T}x{wl.H}x{wl.W}|{wl.d}|{wl.n_heads}x{wl.head_dim}|{wl.d_ff}"
    return [seed, zlib.crc32(key.encode()), block, _TENSOR_IDS[tensor]]


def _rng(wl: Workload, seed: int, block: int, tensor: str) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence(_key(wl, seed, block, tensor))))


_CHUNK_ELEMS = 1 << 21


def _normal(wl: Workload, seed: int, block: int, tensor: str, shape, part: int = 0) -> np.ndarray:
    """N(0, 1) float32 draws of `shape`, in row chunks of about 2M values. Chunk j comes
    from its own Philox stream keyed (tensor key, part, j), so the values do not depend
    on how many host threads fill them; chunks are filled in parallel."""
    shape = tuple(int(v) for v in shape)
    cols = shape[-1]
    rows = int(np.prod(shape[:-1], dtype=np.int64)) if len(shape) > 1 else 1
    out = np.empty((rows, cols), np.float32)
    step = max(1, _CHUNK_ELEMS // max(cols, 1))
    starts = list(range(0, rows, step))
    base = _key(wl, seed, block, tensor) + [part]

    def fill(j):
        r0 = starts[j]
        g = np.random.Generator(np.random.Philox(np.random.SeedSequence(base + [j])))
        g.standard_normal(out=out[r0:r0 + step], dtype=np.float32)

    if len(starts) == 1:
        fill(0)
    else:
        import os
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(len(starts))))
    return out.reshape(shape)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Encode float32 draws as bf16 bit patterns (nearest, ties to even)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_channels(wl: Workload, seed: int = BASE_SEED) -> np.ndarray:
    perm = _rng(wl, seed, 0, "outliers").permutation(wl.d)
    return np.sort(perm[: wl.n_outliers])


def x_input(wl: Workload, seed: int = BASE_SEED) -> np.ndarray:
    """bf16 bits [B, L, d]."""
    z = _normal(wl, seed, 0, "x", (wl.B, wl.L, wl.d))
    z[..., outlier_channels(wl, seed)] *= np.float32(16.0)
    return f32_to_bf16_bits(z)


def cond(wl: Workload, block: int = 0, seed: int = BASE_SEED) -> np.ndarray:
    """fp32 [B, d]."""
    return _rng(wl, seed, block, "c").standard_normal((wl.B, wl.d), dtype=np.float32)


def block_weights(wl: Workload, block: int = 0, seed: int = BASE_SEED) -> dict:
    """Unquantized weights of one block: fp32 projections and bf16 AdaLN weights."""
    d, F = wl.d, wl.d_ff
    w_ada = np.zeros((6 * d, d), np.float32)
    for k in (0, 1, 3, 4):  # shift/scale chunks; the gate chunks (2, 5) stay zero
        w_ada[k * d:(k + 1) * d] = _normal(wl, seed, block, "w_ada", (d, d), part=k) * np.float32(1.0 / np.sqrt(d))
    b_ada = np.zeros(6 * d, np.float32)
    g = _rng(wl, seed, block, "b_gate").standard_normal(2 * d, dtype=np.float32) * np.float32(np.sqrt(0.5))
    b_ada[2 * d:3 * d] = g[:d]
    b_ada[5 * d:6 * d] = g[d:]

    def lin(name, n_out, n_in):
        w = _normal(wl, seed, block, name, (n_out, n_in))
        w *= np.float32(1.0 / np.sqrt(n_in))
        return w

    out = {"w_ada": f32_to_bf16_bits(w_ada), "b_ada": b_ada,
           "wqkv": lin("wqkv", 3 * d, d), "wo": lin("wo", d, d),
           "w1": lin("w1", F, d), "w2": lin("w2", d, F)}
    if not wl.qkv_int8:
        out["wqkv_bf16"] = f32_to_bf16_bits(out["wqkv"])
    if wl.wo_bf16:
        out["wo_bf16"] = f32_to_bf16_bits(out["wo"])
    return out


def sample_rows(n_total: int, n: int, seed: int = BASE_SEED) -> np.ndarray:
    """Seeded sorted sample of row indices, always including the first and last row."""
    r = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, n_total, n, 99])))
    if n >= n_total:
        return np.arange(n_total, dtype=np.int64)
    pick = r.choice(n_total - 2, size=n - 2, replace=False) + 1
    return np.sort(np.concatenate([[0, n_total - 1], pick])).astype(np.int64)
