#!/usr/bin/env python
"""Benchmark of the gated-AdaLN DiT block forward on B200.

One step = one forward of the whole block (AdaLN GEMV, fused LN+modulation+
int8 quantizer, int8 QKV GEMM with 3D RoPE, bf16 attention, quantizer, int8
output projection with gated residual, fused LN+quantizer, int8 W1 + GELU,
quantizer, int8 W2 with gated residual) over one synthetic latent of the
chosen workload, through the library's C ABI. Token-reduction workloads add
the pair/unpair kernels around the block; depth-50 workloads run 50 distinct
blocks per step; residual-reuse workloads run a fresh and a reuse pass per
step (two denoise steps).

Timing: the pass is captured once as a CUDA graph (h3b_graph_capture_blocks)
and each timed step replays it (`launch.mode` = "graph"); workloads with
pairing or reuse launch on the stream ("stream"). K steps are timed with CUDA
events, the input restored and L2 flushed between steps outside the events.
The same K steps are then run with the library's per-launch profiler on; those
per-kernel device times give kernel_share, kernel_roofline and the dominant
kernel's roofline.

Prints one JSON line (rank 0). Under torchrun each rank runs its own
independent latent (replicas; no data-path collective): the value is the
total tokens/s of all ranks over the slowest rank's device time.

The default workload is the largest single block: d=5120, 40 heads x 128,
MLP 20480, an 8x48x48 latent grid (18432 tokens).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl h3b|reference]
  python bench.py --oracle-table   (host timings of the CPU oracle only)
  python bench.py --profile-kernel attention   (one kernel alone, for ncu captures)
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from video_diffusion_transformer_adaln_b200 import build as cuda_build  # noqa: E402
from video_diffusion_transformer_adaln_b200 import h3b, replicas, synth  # noqa: E402
from video_diffusion_transformer_adaln_b200.runtime import (DeviceBlock, bf16_from_bits, dims_of,  # noqa: E402
                                                            workspace)

METRIC = "DiT block tokens/s (int8 MLP+QKV, bf16 attn); % of B200 INT8/BF16/HBM roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "d5120_L18432"
L2_FLUSH_BYTES = 512 << 20
E2E_FLUSH_BYTES = 160 << 20  # larger than the 126 MB L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the recipe's nominal dense ratio of 8-bit to bf16 tensor throughput (4.5 / 2.25 PFLOP/s)
INT8_OVER_BF16 = 2.0


# ----------------------------------------------------------------------------- helpers

def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_work(name, wl):
    """Algorithmic work of one launch: (amount, unit, bound). Tensor-core
    kernels count useful multiply-adds x 2; memory-bound kernels count the
    bytes they must move (read once + write once). For passes that run some
    blocks on the paired grid, block kernels average over their launches."""
    full = wl.B * wl.L * wl.d
    if name == "token_pair":  # read x, write the merged tokens once
        return 2.0 * full + 2.0 * full / 2, "byte", "hbm"
    if name == "token_unpair":  # read x and the block's merged output, write x (merged input recomputed)
        return 2.0 * full + 2.0 * full / 2 + 2.0 * full, "byte", "hbm"
    if wl.token_pair:
        Ls = [wl.L // 2]
    elif wl.pair_blocks[0] < wl.pair_blocks[1]:
        n_m = wl.pair_blocks[1] - wl.pair_blocks[0]
        Ls = [wl.L // 2] * n_m + [wl.L] * (wl.n_blocks - n_m)
    else:
        Ls = [wl.L]
    works = [_block_kernel_work(name, wl, L) for L in Ls]
    return sum(w[0] for w in works) / len(works), works[0][1], works[0][2]


def _block_kernel_work(name, wl, L):
    B, d, F = wl.B, wl.d, wl.d_ff
    R = B * L
    if name == "gemm_qkv":
        return 2.0 * R * 3 * d * d, "op", "tensor_i8" if wl.qkv_int8 else "tensor_bf16"
    if name == "gemm_wo":
        return 2.0 * R * d * d, "op", "tensor_bf16" if wl.wo_bf16 else "tensor_i8"
    if name in ("gemm_w1", "gemm_w2"):
        return 2.0 * R * d * F, "op", "tensor_i8"
    if name == "attention":
        return 4.0 * B * L * L * d, "flop", "tensor_bf16"
    if name in ("ln_mod_quant", "ln_mod_quant_mlp"):
        return R * (2.0 * d + d + 4 + 4), "byte", "hbm"
    if name == "ln_mod":
        return R * (2.0 * d + 2 * d + 4), "byte", "hbm"
    if name == "quant_o":
        return R * (2.0 * d + d + 8), "byte", "hbm"
    if name == "quant_g":
        return R * (2.0 * F + F + 8), "byte", "hbm"
    if name in ("range_delta", "range_apply"):  # 2 + 2 + 4 or 2 + 4 + 2 bytes per element
        return 8.0 * R * d, "byte", "hbm"
    if name == "adaln_gemv":  # (its trailing blocks also fill the small RoPE table)
        return 12.0 * d * d + B * (4.0 * d + 24 * d), "byte", "hbm"
    return 0.0, "byte", "hbm"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, with host timestamps."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", sel], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.started = time.time()
        except Exception:
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        return self.summarize(out)

    @staticmethod
    def summarize(csv_text):
        """Median SM clock of the busy samples (above half the highest one), the max clock,
        and every throttle reason seen active, from nvidia-smi's csv,noheader,nounits rows
        of FIELDS; None when no row parses."""
        rows = [r.split(",") for r in csv_text.strip().splitlines() if r.strip()]
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 8]
        if not rows:
            return None
        mhz = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        busy = ([m for m in mhz if m > 0.5 * max(mhz)] or mhz) if mhz else []
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "window": "nvidia-smi every 50 ms from warm-up start to the end of the timed steps"}


# ----------------------------------------------------------------------------- workload

class Workload:
    """Device buffers and the step callable for one named workload on this rank."""

    def __init__(self, name, rank):
        self.wl = synth.WORKLOADS[name]
        wl = self.wl
        seed = replicas.latent_seed(rank)  # one independent latent per rank
        self.name = name
        x_bits = synth.x_input(wl, seed)
        self.x_ref = bf16_from_bits(x_bits, "cuda")
        self.x = self.x_ref.clone()
        if wl.n_blocks > 1:
            g = torch.Generator(device="cuda").manual_seed(synth.BASE_SEED)
            self.blocks = [DeviceBlock.random_on_device(wl, g) for _ in range(wl.n_blocks)]
            self.c = torch.randn((wl.n_blocks, wl.B, wl.d), generator=g, device="cuda")
        else:
            self.blocks = [DeviceBlock.from_host(synth.block_weights(wl), qkv_int8=wl.qkv_int8)]
            self.c = torch.from_numpy(synth.cond(wl, 0, seed)).cuda()
        self.full = dims_of(wl)
        self.dims = dims_of(wl.merged()) if wl.token_pair else self.full
        self.ws = workspace(self.dims)
        if wl.token_pair or wl.pair_blocks[0] < wl.pair_blocks[1]:
            shp = (wl.B, wl.T, wl.H, wl.W // 2, wl.d)
            self.ym = torch.empty(shp, dtype=torch.bfloat16, device="cuda")
        self.reuse = wl.reuse_blocks[0] < wl.reuse_blocks[1]
        if self.reuse:
            self.x_save = torch.empty_like(self.x)
            self.delta = torch.empty(self.x.numel(), dtype=torch.float32, device="cuda")
        # tokens per step: a reuse step is two denoise steps (one fresh pass, one reuse pass)
        self.tokens = wl.B * wl.L * (2 if self.reuse else 1)

    def step(self, x=None, c=None):
        x = self.x if x is None else x
        c = self.c if c is None else c
        wl = self.wl
        if wl.token_pair:
            h3b.h3b_token_pair(self.full, x, self.ym)
            h3b.h3b_block_forward(self.dims, self.blocks[0].struct, c, self.ym, self.ws)
            h3b.h3b_token_unpair(self.full, x, None, self.ym, x)
        elif self.reuse:
            structs = [b.struct for b in self.blocks]
            f, l = wl.reuse_blocks
            h3b.h3b_blocks_forward_cached(self.dims, structs, f, l, True, c, x, self.x_save, self.delta, self.ws)
            h3b.h3b_blocks_forward_cached(self.dims, structs, f, l, False, c, x, None, self.delta, self.ws)
        elif wl.n_blocks > 1 and wl.pair_blocks[0] < wl.pair_blocks[1]:
            h3b.h3b_blocks_forward_reduced(self.full, [b.struct for b in self.blocks], wl.pair_blocks[0],
                                           wl.pair_blocks[1], c, x, None, self.ym, self.ws)
        elif wl.n_blocks > 1:
            h3b.h3b_blocks_forward(self.dims, [b.struct for b in self.blocks], c, x, self.ws)
        else:
            h3b.h3b_block_forward(self.dims, self.blocks[0].struct, c, x, self.ws)


# ----------------------------------------------------------------------------- CPU oracle leg

FULL_BLOCK_OPS = 1.0e12  # blocks up to this many ops are timed whole on the host


def step_blocks(wl):
    """The blocks one bench step runs: ([(tokens per batch item, count)], tokens per step).
    Paired blocks run on the merged grid (L/2); a residual-reuse step is one fresh pass
    over every block and one pass that skips the cached range (two denoise steps)."""
    if wl.token_pair:
        return [(wl.L // 2, 1)], wl.B * wl.L
    f, l = wl.pair_blocks
    if f < l:
        return [(wl.L // 2, l - f), (wl.L, wl.n_blocks - (l - f))], wl.B * wl.L
    f, l = wl.reuse_blocks
    if f < l:
        return [(wl.L, 2 * wl.n_blocks - (l - f))], 2 * wl.B * wl.L
    return [(wl.L, wl.n_blocks)], wl.B * wl.L


def block_ops(wl, L):
    """Multiply-add ops x 2 of one block over L tokens per batch item: projections and attention."""
    return 24.0 * wl.B * L * wl.d * wl.d + 4.0 * wl.B * L * L * wl.d


class OracleRunner:
    """The CPU oracle, as it stands, timed on the host cores.

    full_block(): one whole block over every token of the workload's grid, timed
    directly. Used when the step is that one block and it is small enough
    (FULL_BLOCK_OPS).

    sample(sub_tokens, n_q): a bounded sample for workloads whose block takes
    minutes on the host. Three pieces of the oracle are timed:
      t_sub  the whole block over every token of a slice of the grid (the first
             frame, its first rows: about sub_tokens tokens), same dimensions and
             weight distributions;
      t_ada  the AdaLN Linear alone, a fixed cost per block and batch item;
      t_att  the attention step for n_q query rows against L keys (seeded Q, K, V).
    Attention costs c = t_att / (n_q L) per query-key pair; the slice's other work
    grows linearly with its tokens. One block over L tokens per batch item is then
        t(L) = B t_ada + (t_sub - B t_ada - c B L_sub^2) L / L_sub + c B L^2
    and a step is the sum of t over the blocks it runs (step_blocks)."""

    def __init__(self, wl):
        import oracle as O  # the CPU oracle: benchmark baseline leg only

        self.O = O
        self.wl = wl
        self.blocks, self.tokens = step_blocks(wl)
        self.block_wl = wl.merged() if wl.token_pair else wl.with_(n_blocks=1, pair_blocks=(0, 0),
                                                                   reuse_blocks=(0, 0))
        self._sub = None
        self._full = None
        self._att = None

    def _prepare(self, wl):
        O = self.O
        raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
        w = {"w_ada": raw["w_ada"], "b_ada": raw["b_ada"]}
        for name, sname in (("wqkv", "sqkv"), ("wo", "so"), ("w1", "s1"), ("w2", "s2")):
            w[name], w[sname] = O.quantize_rows(raw[name])
        if not wl.qkv_int8:
            w["wqkv_bf16"] = raw["wqkv_bf16"]
        if wl.wo_bf16:
            w["wo_bf16"] = raw["wo_bf16"]
        dm = O.Dims(wl.B, wl.T, wl.H, wl.W, wl.d, wl.n_heads, wl.head_dim, wl.d_ff, wl.rope,
                    wl.rope_theta, wl.ln_eps, wl.qkv_int8, wl.wo_bf16)
        return dm, w, c, x

    def can_time_full_block(self):
        return self.blocks == [(self.wl.L, 1)] and block_ops(self.wl, self.wl.L) <= FULL_BLOCK_OPS

    def full_block(self):
        """Seconds of one whole block over every token (all rows)."""
        if self._full is None:
            self._full = self._prepare(self.block_wl)
        dm, w, c, x = self._full
        t0 = time.perf_counter()
        self.O.block_forward(dm, w, c, x)
        return time.perf_counter() - t0

    def sample(self, sub_tokens, n_q):
        """Extrapolated seconds of one bench step and the sample's own wall seconds."""
        bw = self.block_wl
        if self._sub is None or self._sub[0] != sub_tokens:
            h = max(1, min(bw.H, sub_tokens // bw.W))
            self._sub = (sub_tokens, self._prepare(bw.with_(T=1, H=h)), bw.with_(T=1, H=h).L)
        if self._att is None or self._att[0] != n_q:
            r = np.random.default_rng(synth.BASE_SEED)
            kv = [r.standard_normal((bw.L, bw.d)) for _ in range(2)]
            self._att = (n_q, r.standard_normal((n_q, bw.d)), kv[0], kv[1])
        _, (dm, w, c, x), L_sub = self._sub
        _, q, k, v = self._att
        O, B = self.O, bw.B
        t0 = time.perf_counter()
        O.adaln_linear(w["w_ada"], w["b_ada"], c[0])
        t1 = time.perf_counter()
        O.block_forward(dm, w, c, x)
        t2 = time.perf_counter()
        O.attention(q, k, v, bw.n_heads, bw.head_dim)
        t3 = time.perf_counter()
        t_ada, t_sub, t_att = t1 - t0, t2 - t1, t3 - t2
        pair = t_att / (n_q * bw.L)
        per_token = max(t_sub - B * t_ada - pair * B * L_sub * L_sub, 0.0) / (B * L_sub)
        step = sum(n * (B * t_ada + per_token * B * L + pair * B * L * L) for L, n in self.blocks)
        return step, t3 - t0

    def sample_text(self, sub_tokens, n_q):
        bw = self.block_wl
        h = max(1, min(bw.H, sub_tokens // bw.W))
        blocks = " + ".join(f"{n} x {L}-token block" for L, n in self.blocks)
        return (f"oracle pieces timed: the whole block over a 1x{h}x{bw.W} slice ({h * bw.W} tokens, all rows), "
                f"the AdaLN Linear, and attention of {n_q} query rows against all {bw.L} keys; extrapolated "
                f"to the step ({blocks}) as linear-in-tokens work plus attention per query-key pair")

    def full_text(self):
        return f"the whole block over all {self.tokens} tokens, timed directly (no extrapolation)"

    def baseline(self, budget_s=30.0, sub_tokens=2304, n_q=32):
        """(tokens/s, description, extrapolated): the median of up to three timings within
        about budget_s of host work; the first of them also warms the oracle's buffers."""
        t0 = time.perf_counter()
        vals = []
        if self.can_time_full_block():
            while len(vals) < 3 and (not vals or time.perf_counter() - t0 + vals[-1] < budget_s):
                vals.append(self.full_block())
            return self.tokens / statistics.median(vals), self.full_text() + f" (median of {len(vals)})", False
        while len(vals) < 3 and (not vals or time.perf_counter() - t0 < budget_s):
            vals.append(self.sample(sub_tokens, n_q)[0])
        return (self.tokens / statistics.median(vals),
                self.sample_text(sub_tokens, n_q) + f" (median of {len(vals)})", True)

    def threads(self):
        return self.O.threads()


def roofline_summary(prof, wl, peaks, peak_src):
    """From the profiler's {kernel: (launches, total ms)}: each kernel's share of the device
    time, every kernel's achieved rate and fraction of its roofline (algorithmic work per
    launch / mean launch duration), and the dominant kernel's roofline object.

    The kernels are timed inside the benchmark's steps, back to back for the whole timed
    region, so tensor-core kernels are held to the sustained bf16 figure (a GEMM loop under
    the power cap), x 2 for int8; the fraction of the burst figure is reported beside it.
    Memory-bound kernels are held to the copy bandwidth."""
    ktot = sum(ms for _, ms in prof.values()) or 1.0
    shares = {k: round(ms / ktot, 4) for k, (n, ms) in sorted(prof.items(), key=lambda kv: -kv[1][1])}

    def peak_of(bound, key="bf16_tflops_sustained"):
        if bound == "hbm":
            return peaks["hbm_gbs"]
        return peaks[key] * (INT8_OVER_BF16 if bound == "tensor_i8" else 1.0)

    def rate(work, seconds, bound):  # GB/s for bytes, T(FL)OP/s for tensor work
        return work / seconds / (1e9 if bound == "hbm" else 1e12)

    dom = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
    roof = None
    if dom:
        n_launch, ms = prof[dom]
        per_launch_s = ms / n_launch / 1e3
        work, unit, bound = kernel_work(dom, wl)
        achieved, peak = rate(work, per_launch_s, bound), peak_of(bound)
        runit = "GB/s" if bound == "hbm" else ("TOP/s" if bound == "tensor_i8" else "TFLOP/s")
        source = {"tensor_i8": "bf16 sustained x 2 nominal int8/bf16 ratio", "tensor_bf16": "bf16 sustained"}.get(
            bound, "copy bandwidth")
        roof = {"bound": "hbm" if bound == "hbm" else "tensor", "kernel": dom, "achieved": round(achieved, 2),
                "peak": round(peak, 1), "unit": runit, "frac": round(achieved / peak, 4),
                "traffic": traffic_for(dom, wl, n_launch), "peak_source": f"{peak_src} ({source})",
                "work_per_launch": work, "work_unit": unit, "launch_ms": round(per_launch_s * 1e3, 4)}
        if bound != "hbm":
            burst = peak_of(bound, "bf16_tflops")
            roof["peak_burst"] = round(burst, 1)
            roof["frac_burst"] = round(achieved / burst, 4)
    all_roof = {}
    for k, (n, ms) in prof.items():
        work, unit, bound = kernel_work(k, wl)
        if work <= 0:
            continue
        r = rate(work, ms / n / 1e3, bound)
        if bound == "hbm":
            all_roof[k] = {"GB/s": round(r, 1), "frac": round(r / peak_of(bound), 3)}
        else:
            all_roof[k] = {("TOP/s" if bound == "tensor_i8" else "TFLOP/s"): round(r, 1),
                           "frac": round(r / peak_of(bound), 3),
                           "frac_burst": round(r / peak_of(bound, "bf16_tflops"), 3)}
    return roof, shares, all_roof


# ----------------------------------------------------------------------------- arms

# multi-GPU bookkeeping (replicas, no data-path collective): see replicas.py
dist_init = lambda: replicas.init("nccl")  # noqa: E731
barrier = replicas.barrier
max_over_ranks = replicas.max_over_ranks
sum_over_ranks = replicas.sum_over_ranks


def run_h3b(args, rank, world, local):
    cuda_build.build()
    h3b.lib()
    peaks, peak_src = load_peaks()
    W = Workload(args.workload, rank)
    wl = W.wl
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    h3b.h3b_device_error(clear=True)

    def prep():
        W.x.copy_(W.x_ref)
        flush.zero_()

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    for _ in range(args.warmup):
        prep()
        W.step()
    torch.cuda.synchronize()
    barrier(world)

    # The pass is captured once as a CUDA graph (h3b_graph_capture_blocks) where the workload
    # is a plain multi-block pass; paired and residual-reuse steps launch on the stream.
    graph = None
    if not wl.token_pair and not wl.pair_blocks[0] < wl.pair_blocks[1] and not W.reuse:
        graph = h3b.h3b_graph_capture_blocks(W.dims, [b.struct for b in W.blocks], W.c, W.x, W.ws)
        for _ in range(2):
            prep()
            graph.launch()
        torch.cuda.synchronize()
    run_step = graph.launch if graph is not None else W.step

    def timed(step_fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize()
        barrier(world)
        for i in range(args.steps):
            prep()  # restore the input and flush L2 outside the timed events
            ev[i][0].record()
            step_fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world)

    # (1) the headline: K steps of the pass, nothing else on the stream
    total_ms = timed(run_step)
    stream_ms = timed(W.step) if graph is not None else total_ms
    clocks = sampler.stop() if sampler else None
    # (2) per-kernel device times: the same K steps on the stream with the library's
    #     profiler bracketing every launch with CUDA events
    h3b.h3b_profile_read()  # drop anything recorded before
    h3b.h3b_profile_enable(True)
    prof_ms = timed(W.step)
    h3b.h3b_profile_enable(False)
    prof = h3b.h3b_profile_read()
    err = h3b.h3b_device_error(clear=True)
    if err:
        raise RuntimeError(f"device error word set during the benchmark: {err:#x}")

    tokens_all = sum_over_ranks(W.tokens * args.steps, world)
    value = tokens_all / (total_ms / 1e3)

    # ---- end to end through the same API: every step copies its input (x, c) from pinned host
    # memory, runs the pass and copies its result back into pinned host memory. Steps are
    # pipelined over two device buffers and three streams: step i+1's input copy and step
    # i-1's result copy overlap step i's pass. Before each pass the compute stream rewrites a
    # buffer larger than L2 (inside the timed region).
    x_host = torch.empty(W.x.shape, dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(W.x_ref.cpu())
    c_host = torch.empty(W.c.shape, dtype=W.c.dtype, pin_memory=True)
    c_host.copy_(W.c.cpu())
    out_host = [torch.empty_like(x_host, pin_memory=True) for _ in range(2)]
    xs = [W.x, torch.empty_like(W.x)]
    cs = [W.c, torch.empty_like(W.c)]
    graphs = None
    if graph is not None:
        graphs = [graph, h3b.h3b_graph_capture_blocks(W.dims, [b.struct for b in W.blocks], cs[1], xs[1], W.ws)]
    e2e_flush = flush[:E2E_FLUSH_BYTES]
    s_h2d, s_comp, s_d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        h2d_done = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        d2h_done = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(s_h2d)
        for i in range(n):
            k = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(d2h_done[i - 2])  # buffer k is free again
                xs[k].copy_(x_host, non_blocking=True)
                cs[k].copy_(c_host, non_blocking=True)
                h2d_done[i].record(s_h2d)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(h2d_done[i])
                e2e_flush.zero_()
                if graphs is not None:
                    graphs[k].launch(s_comp)
                else:
                    W.step(x=xs[k], c=cs[k])
                comp_done[i].record(s_comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(comp_done[i])
                out_host[k].copy_(xs[k], non_blocking=True)
                d2h_done[i].record(s_d2h)
        s_d2h.wait_event(d2h_done[n - 1])
        t1.record(s_d2h)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_run(2)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_run(e2e_steps), world)
    barrier(world)
    if graphs is not None:
        graphs[1].destroy()
    e2e_value = sum_over_ranks(W.tokens * e2e_steps, world) / (e2e_ms / 1e3)
    h2d = x_host.numel() * x_host.element_size() + c_host.numel() * c_host.element_size()
    d2h = out_host[0].numel() * out_host[0].element_size()
    launch = {"mode": "graph" if graph is not None else "stream",
              "stream_ms_per_step": round(stream_ms / args.steps, 4),
              "profiled_ms_per_step": round(prof_ms / args.steps, 4)}
    if graph is not None:
        launch["graph_ms_per_step"] = round(total_ms / args.steps, 4)
        launch["kernels_per_step"] = graph.kernel_count
        graph.destroy()

    roof, shares, all_roof = roofline_summary(prof, wl, peaks, peak_src)

    gpu_launches = int(sum(n for n, _ in prof.values()))
    kernel_ms = {k: round(ms / args.steps, 4) for k, (n, ms) in prof.items()}
    gap_ms = prof_ms / args.steps - sum(ms for _, ms in prof.values()) / args.steps
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        orc = OracleRunner(wl)
        v, text, extrap = orc.baseline(sub_tokens=args.cpu_sub_tokens, n_q=args.cpu_queries)
        cpu = {"value": round(v, 2), "unit": UNIT, "cores": orc.threads(), "kind": "oracle", "sample": text,
               "extrapolated": extrap}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8+bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl.B, "grid_THW": [wl.T, wl.H, wl.W], "tokens": wl.L,
                   "d": wl.d, "heads": wl.n_heads, "head_dim": wl.head_dim, "d_ff": wl.d_ff,
                   "blocks_per_step": wl.n_blocks, "token_pair": wl.token_pair,
                   "paired_blocks": list(wl.pair_blocks), "reuse_blocks": list(wl.reuse_blocks),
                   "qkv": "int8" if wl.qkv_int8 else "bf16", "wo": "bf16" if wl.wo_bf16 else "int8",
                   "attention": "bf16",
                   "l2": "flushed between steps (512 MiB write outside the timed events)",
                   "parallelism": "replicas: one independent latent per GPU, no collective"},
        "roofline": roof, "kernel_share": shares, "kernel_roofline": all_roof,
        "kernel_ms_per_step": kernel_ms, "launch_gap_ms_per_step": round(gap_ms, 4), "launch": launch,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipelined": True,
                "l2": f"a {E2E_FLUSH_BYTES >> 20} MiB write on the compute stream before each pass, inside the timed region"},
        "gpu_launches": gpu_launches, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, rank, world, local):
    """The CPU oracle as the reference arm (rank 0 only). Each step is one bounded
    timing of the oracle: the whole block when it is small (the step's tokens over
    its measured seconds), else one OracleRunner.sample whose extrapolated step time
    gives the value. ms_per_step is always the wall time the steps actually took."""
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    orc = OracleRunner(wl)
    full = orc.can_time_full_block() and block_ops(wl, wl.L) <= args.ref_full_ops
    walls, ests = [], []
    for i in range(args.warmup + args.steps):
        if full:
            wall = orc.full_block()
            est = wall
        else:
            est, wall = orc.sample(args.ref_sub_tokens, args.ref_queries)
        if i >= args.warmup:
            walls.append(wall)
            ests.append(est)
    threads = orc.threads()
    ms = 1e3 * sum(walls) / len(walls)
    est_ms = 1e3 * sum(ests) / len(ests)
    value = orc.tokens / (est_ms / 1e3)
    sample = orc.full_text() if full else orc.sample_text(args.ref_sub_tokens, args.ref_queries)
    line = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (int8 decisions in f32)", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "tokens": wl.L, "d": wl.d, "heads": wl.n_heads,
                       "head_dim": wl.head_dim, "d_ff": wl.d_ff, "blocks_per_step": wl.n_blocks},
            "extrapolated": not full,
            "step_ms_extrapolated": None if full else round(est_ms, 1),
            "step": ("one whole block per step" if full else
                     "one bounded sample per step (ms_per_step is its wall time); value = the step's tokens over "
                     "the step time extrapolated from the sample (step_ms_extrapolated)"),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample, "extrapolated": not full},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


PROFILE_KERNELS = ("attention", "ln_mod_quant", "quant_o", "adaln_gemv", "token_pair", "token_unpair",
                   "gemm_qkv", "gemm_wo", "gemm_w1", "gemm_w2")


def run_profile_kernel(name, workload):
    """One step kernel alone at the workload's shape, three launches (for ncu captures of a
    single kernel: `ncu -k regex:<kernel> -s 2 -c 1 python bench.py --profile-kernel NAME`)."""
    cuda_build.build()
    h3b.lib()
    wl = synth.WORKLOADS[workload]
    B, L, d, H, dh = wl.B, wl.L, wl.d, wl.n_heads, wl.head_dim
    g = torch.Generator(device="cuda").manual_seed(synth.BASE_SEED)
    dims = dims_of(wl)
    if name == "attention":
        qkv = (torch.randn(3 * B * H * L * dh, generator=g, device="cuda") * 0.8).to(torch.bfloat16)
        o = torch.empty((B, L, d), dtype=torch.bfloat16, device="cuda")
        am = torch.zeros(B * L, dtype=torch.float32, device="cuda")
        fn = lambda: h3b.h3b_attention(dims, qkv, o, am)  # noqa: E731
    elif name in ("ln_mod_quant", "quant_o"):
        x = torch.randn((B * L, d), generator=g, device="cuda").to(torch.bfloat16)
        q = torch.empty((B * L, d), dtype=torch.int8, device="cuda")
        s = torch.empty(B * L, dtype=torch.float32, device="cuda")
        if name == "ln_mod_quant":
            sh = torch.randn(d, generator=g, device="cuda") * 0.1
            sc = torch.randn(d, generator=g, device="cuda") * 0.1
            fn = lambda: h3b.h3b_ln_modulate_quantize(x, B * L, d, wl.ln_eps, sh, sc, L, d, q, s)  # noqa: E731
        else:
            am = x.float().abs().amax(dim=1).contiguous()
            fn = lambda: h3b.h3b_quantize_rows(x, q, s, absmax=am)  # noqa: E731
    elif name == "gemm_qkv":
        # QKV + 3D RoPE, written head-major, from int8 codes of a random activation
        blk = DeviceBlock.random_on_device(wl, g)
        A = torch.randint(-127, 128, (B * L, d), generator=g, device="cuda", dtype=torch.int8)
        sA = torch.rand(B * L, generator=g, device="cuda") * 0.01
        qkv = torch.empty(3 * B * L * d, dtype=torch.bfloat16, device="cuda")
        rope_ws = torch.empty(h3b.h3b_rope_table_bytes(dims), dtype=torch.uint8, device="cuda")
        fn = lambda: h3b.h3b_qkv_projection(dims, A, sA, blk.struct, qkv, rope_ws)  # noqa: E731
    elif name in ("gemm_wo", "gemm_w1", "gemm_w2"):
        # the output and MLP projections at the workload's shape: int8 codes of a random
        # activation and weight
        K, N = {"gemm_wo": (d, d), "gemm_w1": (d, wl.d_ff), "gemm_w2": (wl.d_ff, d)}[name]
        A = torch.randint(-127, 128, (B * L, K), generator=g, device="cuda", dtype=torch.int8)
        Wq = torch.randint(-127, 128, (N, K), generator=g, device="cuda", dtype=torch.int8)
        sA = torch.rand(B * L, generator=g, device="cuda") * 0.01
        sW = torch.rand(N, generator=g, device="cuda") * 0.01
        if name == "gemm_w1":
            out = torch.empty((B * L, N), dtype=torch.bfloat16, device="cuda")
            am = torch.zeros(B * L, dtype=torch.float32, device="cuda")
            fn = lambda: h3b.h3b_gemm_i8_gelu(A, sA, Wq, sW, None, out, am)  # noqa: E731
        else:
            x = torch.randn((B * L, N), generator=g, device="cuda").to(torch.bfloat16)
            gate = torch.randn((B, N), generator=g, device="cuda") * 0.5
            fn = lambda: h3b.h3b_gemm_i8_gated_residual(A, sA, Wq, sW, None, gate, L, N, x)  # noqa: E731
    elif name == "adaln_gemv":
        w = (torch.randn((6 * d, d), generator=g, device="cuda") * d ** -0.5).to(torch.bfloat16)
        c = torch.randn((B, d), generator=g, device="cuda")
        mod = torch.empty((B, 6 * d), device="cuda")
        fn = lambda: h3b.h3b_adaln_modulation(dims, w, None, c, mod)  # noqa: E731
    else:
        x = torch.randn((B, wl.T, wl.H, wl.W, d), generator=g, device="cuda").to(torch.bfloat16)
        ym = torch.empty((B, wl.T, wl.H, wl.W // 2, d), dtype=torch.bfloat16, device="cuda")
        h3b.h3b_token_pair(dims, x, ym)
        out = torch.empty_like(x)
        fn = ((lambda: h3b.h3b_token_pair(dims, x, ym)) if name == "token_pair" else
              (lambda: h3b.h3b_token_unpair(dims, x, None, ym, out)))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    err = h3b.h3b_device_error(clear=True)
    log(f"{name} at {workload}: 3 launches, device error word {err:#x}")
    if err:
        raise SystemExit(1)


ORACLE_TABLE = (("d256_L512", (1, None)), ("d2048_L4096", (1, None)), ("d5120_L18432", (None,)))


def run_oracle_table(args):
    """Host timings of the oracle for the baseline table: the whole block at 1 thread and
    at every core for the small workloads, the bounded sample at every core for the
    largest single block. Each entry runs in a child process (OMP_NUM_THREADS is read
    when the oracle library loads) and prints one JSON object."""
    rows = []
    for name, thread_opts in ORACLE_TABLE:
        for th in thread_opts:
            env = dict(os.environ)
            if th is not None:
                env["OMP_NUM_THREADS"] = str(th)
            else:
                env.pop("OMP_NUM_THREADS", None)
            r = subprocess.run([sys.executable, os.path.abspath(__file__), "--oracle-entry", name],
                               capture_output=True, text=True, env=env, cwd=ROOT)
            if r.returncode != 0:
                rows.append({"workload": name, "threads": th, "error": r.stderr[-500:]})
            else:
                rows.append(json.loads(r.stdout.strip().splitlines()[-1]))
            log(json.dumps(rows[-1]))
    print(json.dumps({"oracle_table": rows, "nproc": os.cpu_count()}), flush=True)


def run_oracle_entry(name):
    wl = synth.WORKLOADS[name]
    orc = OracleRunner(wl)
    out = {"workload": name, "threads": orc.threads()}
    if orc.can_time_full_block():
        orc.full_block()  # load the library and touch the buffers once
        t = orc.full_block()
        out.update(block_s=round(t, 3), tokens_per_s=round(orc.tokens / t, 2), how=orc.full_text())
    # the bounded sample the benchmark uses for large blocks, beside the whole block where both exist
    est, wall = orc.sample(2304, 32)
    out.update(sample_block_s=round(est, 3), sample_tokens_per_s=round(orc.tokens / est, 2),
               sample_wall_s=round(wall, 2), sample_how=orc.sample_text(2304, 32))
    print(json.dumps(out), flush=True)


_TRAFFIC = None


def traffic_for(kernel, wl, n_launch):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, scaled to
    this workload when it was captured on a smaller case of the same kernel; None
    when no capture exists or the kernel source changed since it was taken."""
    global _TRAFFIC
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if _TRAFFIC is None:
        try:
            with open(path) as f:
                _TRAFFIC = json.load(f)
        except Exception:
            _TRAFFIC = {}
    ent = _TRAFFIC.get(kernel)
    if not ent:
        return None
    src = os.path.join(ROOT, "video_diffusion_transformer_adaln_b200", "csrc", ent.get("source", ""))
    try:
        import hashlib
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != ent.get("source_sha256_16"):
                return None
    except Exception:
        return None
    if ent.get("workload") == wl.name:
        return ent.get("bytes_per_launch")
    scale = ent.get("scale_to", {}).get(wl.name)
    return None if scale is None else ent["bytes_per_launch"] * scale


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="h3b", choices=["h3b", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sub-tokens", type=int, default=2304,
                    help="tokens of the grid slice the oracle baseline runs whole (large workloads)")
    ap.add_argument("--cpu-queries", type=int, default=32, help="query rows of the baseline's attention piece")
    ap.add_argument("--ref-sub-tokens", type=int, default=384,
                    help="tokens of the grid slice each reference-arm step runs whole (large workloads)")
    ap.add_argument("--ref-queries", type=int, default=16, help="query rows of each reference step's attention")
    ap.add_argument("--ref-full-ops", type=float, default=1.0e11,
                    help="reference steps run the whole block when it is at most this many ops")
    ap.add_argument("--oracle-table", action="store_true",
                    help="print host timings of the oracle (1 thread and all cores) and exit")
    ap.add_argument("--oracle-entry", help=argparse.SUPPRESS)
    ap.add_argument("--profile-kernel", choices=PROFILE_KERNELS,
                    help="run one step kernel alone at the workload's shape (three launches) and exit")
    args = ap.parse_args()
    if args.profile_kernel:
        run_profile_kernel(args.profile_kernel, args.workload)
        return
    if args.oracle_entry:
        run_oracle_entry(args.oracle_entry)
        return
    if args.oracle_table:
        run_oracle_table(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world, 0)
        return
    rank, world, local = dist_init()
    if world != args.gpus and rank == 0:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")
    try:
        run_h3b(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
