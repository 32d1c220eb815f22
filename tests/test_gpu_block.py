"""End-to-end parity of the block forward (and its multi-block and
token-reduction forms) against the CPU oracle on the same seeded inputs.

Bar: relative L2 error of the block output <= 1e-2 against the fp64 oracle.
The relative L2 of the block's delta (output - input), which the input
dominates less, is held to 5e-2. Large workloads are compared on a seeded
sample of token rows that the oracle evaluates one by one (it still projects
K and V for every token)."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import (bf16_f64, bf16_dev, bf16_host, no_device_error, oracle_dims, oracle_weights, rel_l2, require_gpu,
                         to_dev, bf16_ulp_diff)
from video_diffusion_transformer_adaln_b200 import h3b, synth
from video_diffusion_transformer_adaln_b200.runtime import (DeviceBlock, blocks_forward, block_forward, dims_of,
                                                            paired_block_forward, workspace)

pytestmark = pytest.mark.gpu

TOL = 1e-2
TOL_DELTA = 5e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    h3b.h3b_device_error(clear=True)
    yield


def _run_gpu_block(wl, raw, c, x_bits):
    dims = dims_of(wl)
    blk = DeviceBlock.from_host(raw, qkv_int8=wl.qkv_int8)
    x = bf16_dev(x_bits)
    ws = workspace(dims)
    block_forward(dims, blk, to_dev(c), x, ws)
    torch.cuda.synchronize()
    return bf16_host(x), blk


def _compare(got_bits, ref, x_bits, rows=None, n_blocks=1):
    got = bf16_f64(got_bits).reshape(-1, ref.shape[-1])
    xin = bf16_f64(x_bits).reshape(-1, ref.shape[-1])
    if rows is not None:
        got, xin = got[rows], xin[rows]
    e = rel_l2(got, ref)
    ed = rel_l2(got - xin, ref - xin)
    print(f"rel-L2 out {e:.3e} delta {ed:.3e}")
    assert np.isfinite(got).all()
    # the 1e-2 bar is per block; through a chain of blocks the two sides'
    # roundings compound, so the chain is held to n_blocks x the per-block bar
    assert e <= TOL * n_blocks, (e, ed)
    assert ed <= TOL_DELTA * n_blocks, (e, ed)
    return e, ed


def _weights_agree(raw, blk, qkv_int8=True):
    """The library's weight quantization equals the oracle's, byte for byte."""
    ow = oracle_weights(raw, qkv_int8)
    for name, sname in (("wqkv", "sqkv"), ("wo", "so"), ("w1", "s1"), ("w2", "s2")):
        if name == "wqkv" and not qkv_int8:
            continue
        assert np.array_equal(blk.tensors[name].cpu().numpy(), ow[name]), name
        assert np.array_equal(blk.tensors[sname].cpu().numpy(), ow[sname]), sname
    return ow


@pytest.mark.parametrize("B,qkv_int8", [(1, True), (2, True), (1, False)])
def test_block_d256_full(B, qkv_int8):
    wl = synth.WORKLOADS["d256_L512"].with_(B=B, qkv_int8=qkv_int8)
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    got, blk = _run_gpu_block(wl, raw, c, x)
    ow = _weights_agree(raw, blk, qkv_int8)
    ref = O.block_forward(oracle_dims(wl), ow, c, x)
    _compare(got, ref, x)
    no_device_error()


def test_block_zero_gates_is_exact_identity():
    wl = synth.WORKLOADS["d256_L512"]
    raw = synth.block_weights(wl)
    raw["b_ada"][2 * wl.d:3 * wl.d] = 0
    raw["b_ada"][5 * wl.d:] = 0
    x = synth.x_input(wl)
    got, _ = _run_gpu_block(wl, raw, synth.cond(wl), x)
    assert np.array_equal(got, x)
    no_device_error()


def test_block_ragged_grid():
    # L = 3*5*7 = 105 tokens: one partial query/key tile and ragged GEMM rows
    wl = synth.WORKLOADS["d256_L512"].with_(T=3, H=5, W=7)
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    got, blk = _run_gpu_block(wl, raw, c, x)
    ref = O.block_forward(oracle_dims(wl), oracle_weights(raw), c, x)
    _compare(got, ref, x)
    no_device_error()


def test_block_d2048_sampled():
    wl = synth.WORKLOADS["d2048_L4096"]
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    got, blk = _run_gpu_block(wl, raw, c, x)
    ow = _weights_agree(raw, blk)
    rows = synth.sample_rows(wl.L, 192)
    ref = O.block_forward(oracle_dims(wl), ow, c, x, rows=rows)
    _compare(got, ref, x, rows)
    no_device_error()


def test_block_d256_full_bf16_wo():
    """The block with the bf16 output projection on the bf16 attention output."""
    wl = synth.WORKLOADS["d256_L512"].with_(wo_bf16=True)
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    got, blk = _run_gpu_block(wl, raw, c, x)
    ow = _weights_agree(raw, blk)
    ref = O.block_forward(oracle_dims(wl), ow, c, x)
    _compare(got, ref, x)
    no_device_error()


@pytest.mark.parametrize("name", ["d5120_L18432", "d5120_L18432_bf16qkv", "d5120_L18432_bf16wo"])
def test_block_d5120_sampled(name):
    wl = synth.WORKLOADS[name]
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    got, blk = _run_gpu_block(wl, raw, c, x)
    ow = _weights_agree(raw, blk, wl.qkv_int8)
    del blk
    torch.cuda.empty_cache()
    rows = synth.sample_rows(wl.L, 64)
    ref = O.block_forward(oracle_dims(wl), ow, c, x, rows=rows)
    _compare(got, ref, x, rows)
    no_device_error()


def _paired_reference(wl, ow, c, x):
    m = wl.merged()
    xm = O.token_pair(x, wl.B, wl.T, wl.H, wl.W, wl.d)
    ym = O.block_forward(oracle_dims(m), ow, c, xm)
    return O.token_unpair(x, xm, ym, wl.B, wl.T, wl.H, wl.W, wl.d).reshape(-1, wl.d)


def test_token_reduction_d256():
    wl = synth.WORKLOADS["d256_L512"]
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    blk = DeviceBlock.from_host(raw)
    full, merged = dims_of(wl), dims_of(wl.merged())
    xd = bf16_dev(x)
    paired_block_forward(full, merged, blk, to_dev(c), xd, workspace(merged))
    ref = _paired_reference(wl, oracle_weights(raw), c, x)
    _compare(bf16_host(xd), ref, x)
    no_device_error()


def test_token_reduction_d5120_sampled():
    wl = synth.WORKLOADS["d5120_L18432_pair"]
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    blk = DeviceBlock.from_host(raw)
    full, merged = dims_of(wl), dims_of(wl.merged())
    xd = bf16_dev(x)
    xm = torch.empty((wl.B, wl.T, wl.H, wl.W // 2, wl.d), dtype=torch.bfloat16, device="cuda")
    h3b.h3b_token_pair(full, xd, xm)
    paired_block_forward(full, merged, blk, to_dev(c), xd, workspace(merged))
    got = bf16_host(xd)
    ow = oracle_weights(raw)
    del blk
    torch.cuda.empty_cache()
    # sampled merged rows; each covers unmerged tokens w = 2k and 2k+1
    m = wl.merged()
    xm_o = O.token_pair(x, wl.B, wl.T, wl.H, wl.W, wl.d)
    assert np.array_equal(bf16_host(xm).reshape(xm_o.shape), xm_o)
    mrows = synth.sample_rows(m.L, 48)
    ym_o = O.block_forward(oracle_dims(m), ow, c, xm_o, rows=mrows)
    xm_flat = bf16_f64(xm_o).reshape(-1, wl.d)
    urows = np.concatenate([2 * mrows, 2 * mrows + 1])
    ref = np.concatenate([bf16_f64(x).reshape(-1, wl.d)[2 * mrows] + ym_o - xm_flat[mrows],
                          bf16_f64(x).reshape(-1, wl.d)[2 * mrows + 1] + ym_o - xm_flat[mrows]])
    _compare(got, ref, x, urows)
    no_device_error()


def test_blocks_forward_three_blocks_d256():
    wl = synth.WORKLOADS["d256_L512"].with_(n_blocks=3)
    x = synth.x_input(wl)
    raws = [synth.block_weights(wl, b) for b in range(3)]
    cs = np.stack([synth.cond(wl, b) for b in range(3)])
    dims = dims_of(wl)
    blocks = [DeviceBlock.from_host(r) for r in raws]
    xd = bf16_dev(x)
    blocks_forward(dims, blocks, to_dev(cs), xd, workspace(dims))
    got = bf16_host(xd)
    # the oracle chains the same blocks; the residual stream between blocks is bf16
    xr = x
    for b in range(3):
        out = O.block_forward(oracle_dims(wl), oracle_weights(raws[b]), cs[b], xr)
        xr = O.bf16_round(out).reshape(x.shape)
    _compare(got, out, x, n_blocks=3)
    # blocks_forward equals three block_forward calls, bit for bit
    xd2 = bf16_dev(x)
    ws = workspace(dims)
    for b in range(3):
        block_forward(dims, blocks[b], to_dev(cs[b]), xd2, ws)
    assert np.array_equal(bf16_host(xd2), got)
    no_device_error()


def test_graph_replay_equals_stream_launches_d256():
    """A captured three-block pass replays to the same bits as h3b_blocks_forward."""
    wl = synth.WORKLOADS["d256_L512"].with_(n_blocks=3)
    x = synth.x_input(wl)
    raws = [synth.block_weights(wl, b) for b in range(3)]
    cs = to_dev(np.stack([synth.cond(wl, b) for b in range(3)]))
    dims = dims_of(wl)
    blocks = [DeviceBlock.from_host(r) for r in raws]
    ws = workspace(dims)
    xd = bf16_dev(x)
    blocks_forward(dims, blocks, cs, xd, ws)  # also loads every kernel before the capture
    ref = bf16_host(xd)
    xg = bf16_dev(x)
    g = h3b.h3b_graph_capture_blocks(dims, [b.struct for b in blocks], cs, xg, ws)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_host(xg), x)  # capturing runs nothing
    assert g.kernel_count == 3 * 10
    g.launch()
    torch.cuda.synchronize()
    assert np.array_equal(bf16_host(xg), ref)
    xg.copy_(bf16_dev(x))  # a replay reads x as it is at launch time
    g.launch()
    torch.cuda.synchronize()
    assert np.array_equal(bf16_host(xg), ref)
    g.destroy()
    # capturing with the profiler on is refused, and nothing is left captured
    h3b.h3b_profile_enable(True)
    try:
        with pytest.raises(h3b.H3BError):
            h3b.h3b_graph_capture_blocks(dims, [b.struct for b in blocks], cs, xg, ws)
    finally:
        h3b.h3b_profile_enable(False)
        h3b.h3b_profile_read()
    no_device_error()


def test_blocks_forward_cached_range_d256():
    """Residual reuse: a fresh pass caches the delta of blocks 1..3 (the last three of four);
    a reuse pass skips them and re-applies the delta."""
    wl = synth.WORKLOADS["d256_L512"].with_(n_blocks=4)
    first, last = 1, 4
    x = synth.x_input(wl)
    raws = [synth.block_weights(wl, b) for b in range(4)]
    cs = to_dev(np.stack([synth.cond(wl, b) for b in range(4)]))
    dims = dims_of(wl)
    blocks = [DeviceBlock.from_host(r) for r in raws]
    structs = [b.struct for b in blocks]
    ws = workspace(dims)
    n = x.size
    # reference: the plain pass, and block 0 alone
    xr = bf16_dev(x)
    blocks_forward(dims, blocks, cs, xr, ws)
    ref = bf16_host(xr)
    x0 = bf16_dev(x)
    h3b.h3b_blocks_forward(dims, structs[:1], cs, x0, ws)
    after0 = bf16_host(x0)
    # fresh pass: the same result bit for bit; x_save is the range's input; delta = after - before
    xf = bf16_dev(x)
    x_save = torch.empty_like(xf)
    delta = torch.empty(n, dtype=torch.float32, device="cuda")
    h3b.h3b_blocks_forward_cached(dims, structs, first, last, True, cs, xf, x_save, delta, ws)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_host(xf), ref)
    assert np.array_equal(bf16_host(x_save), after0)
    # delta is the fp32 difference of the range's bf16 output and input (restated in numpy on
    # the pass's own values; the oracle is held to seeded inputs below)
    f32 = synth.bf16_bits_to_f32
    d_got = delta.cpu().numpy()
    assert np.array_equal(d_got, (f32(ref) - f32(after0)).reshape(-1))
    # reuse pass on another step's stream: block 0 runs, the range is replaced by the delta,
    # x = bf16(x + delta) with the sum in fp32
    x2_bits = synth.f32_to_bf16_bits((synth.bf16_bits_to_f32(x) * 0.9).astype(np.float32))
    x2 = bf16_dev(x2_bits)
    h3b.h3b_blocks_forward_cached(dims, structs, first, last, False, cs, x2, None, delta, ws)
    x2b = bf16_dev(x2_bits)
    h3b.h3b_blocks_forward(dims, structs[:1], cs, x2b, ws)
    want = synth.f32_to_bf16_bits(f32(bf16_host(x2b)).reshape(-1) + d_got).reshape(x.shape)
    assert np.array_equal(bf16_host(x2), want)
    # the step entry points alone agree with the pass
    d2 = torch.empty_like(delta)
    h3b.h3b_range_delta(x_save, xf, d2)
    assert torch.equal(d2, delta)
    x3 = bf16_dev(after0)
    h3b.h3b_range_apply(x3, delta)
    assert np.array_equal(bf16_host(x3).reshape(-1), synth.f32_to_bf16_bits(f32(after0).reshape(-1) + d_got))
    # the two elementwise steps against the oracle, on seeded inputs
    r = np.random.default_rng(11)
    before = synth.f32_to_bf16_bits(r.standard_normal(n).astype(np.float32))
    after = synth.f32_to_bf16_bits((f32(before) + 0.1 * r.standard_normal(n)).astype(np.float32))
    d3 = torch.empty(n, dtype=torch.float32, device="cuda")
    h3b.h3b_range_delta(bf16_dev(before), bf16_dev(after), d3)
    d_ref = O.range_delta(before, after)
    d_dev = d3.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(d_dev - d_ref) <= 2.0 ** -24 * np.abs(d_ref))
    x5 = bf16_dev(before)
    h3b.h3b_range_apply(x5, to_dev(d_ref.astype(np.float32)))
    # fp32 sum then bf16 vs one rounding of the exact sum
    assert bf16_ulp_diff(bf16_host(x5), O.range_apply(before, d_ref.astype(np.float32))).max() <= 1
    no_device_error()


def test_blocks_forward_reduced_middle_range_d256():
    """Five blocks; blocks 1..3 run on the merged grid (paired once, unpaired once)."""
    wl = synth.WORKLOADS["d256_L512"].with_(n_blocks=5)
    first, last = 1, 4
    x = synth.x_input(wl)
    raws = [synth.block_weights(wl, b) for b in range(5)]
    cs = np.stack([synth.cond(wl, b) for b in range(5)])
    full, merged = dims_of(wl), dims_of(wl.merged())
    blocks = [DeviceBlock.from_host(r) for r in raws]
    xd = bf16_dev(x)
    shape = (wl.B, wl.T, wl.H, wl.W // 2, wl.d)
    ym = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    h3b.h3b_blocks_forward_reduced(full, [b.struct for b in blocks], first, last, to_dev(cs), xd, None, ym,
                                   workspace(full))
    got = bf16_host(xd)
    # the oracle composes the same pass; between blocks the stream is bf16
    m = wl.merged()
    xr = x
    for b in range(first):
        xr = O.bf16_round(O.block_forward(oracle_dims(wl), oracle_weights(raws[b]), cs[b], xr)).reshape(x.shape)
    xmo = O.token_pair(xr, wl.B, wl.T, wl.H, wl.W, wl.d)
    yr = xmo
    for b in range(first, last):
        yr = O.bf16_round(O.block_forward(oracle_dims(m), oracle_weights(raws[b]), cs[b], yr)).reshape(xmo.shape)
    xr = O.bf16_round(O.token_unpair(xr, xmo, bf16_f64(yr), wl.B, wl.T, wl.H, wl.W, wl.d))
    for b in range(last, 5):
        out = O.block_forward(oracle_dims(wl), oracle_weights(raws[b]), cs[b], xr)
        xr = O.bf16_round(out).reshape(x.shape)
    _compare(got, out, x, n_blocks=5)
    # with an empty merged range it is the plain multi-block pass, bit for bit
    xa, xb = bf16_dev(x), bf16_dev(x)
    h3b.h3b_blocks_forward_reduced(full, [b.struct for b in blocks], 2, 2, to_dev(cs), xa, None, None,
                                   workspace(full))
    blocks_forward(full, blocks, to_dev(cs), xb, workspace(full))
    assert np.array_equal(bf16_host(xa), bf16_host(xb))
    no_device_error()


def test_depth50_pass_properties_d5120_T2():
    """The 50-block pass at d=5120, L=4608: finite, deterministic, and bit-identical
    to 50 single-block calls. Each of those calls is the d=5120 block that
    test_block_d5120_sampled checks against the oracle (with weights the oracle
    quantizes itself); this pass's weights are drawn on the device, so its blocks
    are not fed to the oracle."""
    wl = synth.WORKLOADS["d5120_depth50_T2"]
    dims = dims_of(wl)
    g = torch.Generator(device="cuda").manual_seed(synth.BASE_SEED)
    blocks = [DeviceBlock.random_on_device(wl, g) for _ in range(wl.n_blocks)]
    c = torch.randn((wl.n_blocks, wl.B, wl.d), generator=g, device="cuda")
    x0 = synth.x_input(wl)
    ws = workspace(dims)
    xa = bf16_dev(x0)
    blocks_forward(dims, blocks, c, xa, ws)
    xb = bf16_dev(x0)
    blocks_forward(dims, blocks, c, xb, ws)
    xc = bf16_dev(x0)
    for i in range(wl.n_blocks):
        block_forward(dims, blocks[i], c[i], xc, ws)
    a, b_, cc = bf16_host(xa), bf16_host(xb), bf16_host(xc)
    assert np.array_equal(a, b_) and np.array_equal(a, cc)
    assert np.isfinite(bf16_f64(a)).all()
    no_device_error()


# ----------------------------------------------------------------------------- the 50-block pass's grids

@pytest.mark.parametrize("T,block", [(4, 0), (12, 24), (16, 49)])
def test_depth_pass_block_at_long_grids_sampled(T, block):
    """One block of the 50-block pass (d=5120, 40x128 heads, MLP 20480, RoPE (32,48,48)) on
    the T x 48 x 48 grids of the frame sweep, up to 36864 tokens: attention runs over up to
    144 key tiles of 256 per query tile and RoPE reaches positions (T-1, 47, 47). The weights
    and c of the pass's block index and a seeded x are generated on the host, so the oracle
    sees seeded inputs only; 48 sampled rows (always the first and last token) are compared
    at the block bar. The oracle projects Q, K and V for every token."""
    wl = synth.WORKLOADS[f"d5120_depth50_T{T}"].with_(n_blocks=1)
    raw, c, x = synth.block_weights(wl, block), synth.cond(wl, block), synth.x_input(wl)
    got, blk = _run_gpu_block(wl, raw, c, x)
    ow = _weights_agree(raw, blk)
    del blk
    torch.cuda.empty_cache()
    rows = synth.sample_rows(wl.L, 48)
    ref = O.block_forward(oracle_dims(wl), ow, c, x, rows=rows)
    _compare(got, ref, x, rows)
    no_device_error()


def test_blocks_forward_three_blocks_d5120_T2():
    """The pass's chaining at its real width: blocks 0, 1, 2 of the d=5120 pass on the 2x48x48
    grid (4608 tokens) through h3b_blocks_forward, against the oracle chaining the same blocks
    (full rows for blocks 0 and 1, since the next block's keys need every token; 64 sampled
    rows of block 2). Between blocks the oracle's stream is bf16, as the library's is."""
    wl = synth.WORKLOADS["d5120_depth50_T2"].with_(n_blocks=3)
    x = synth.x_input(wl)
    raws = [synth.block_weights(wl, b) for b in range(3)]
    cs = np.stack([synth.cond(wl, b) for b in range(3)])
    dims = dims_of(wl)
    blocks = [DeviceBlock.from_host(r) for r in raws]
    ows = [_weights_agree(r, b) for r, b in zip(raws, blocks)]
    xd = bf16_dev(x)
    blocks_forward(dims, blocks, to_dev(cs), xd, workspace(dims))
    torch.cuda.synchronize()
    got = bf16_host(xd)
    del blocks
    torch.cuda.empty_cache()
    xr = x
    for b in range(2):
        xr = O.bf16_round(O.block_forward(oracle_dims(wl), ows[b], cs[b], xr)).reshape(x.shape)
    rows = synth.sample_rows(wl.L, 64)
    ref = O.block_forward(oracle_dims(wl), ows[2], cs[2], xr, rows=rows)
    _compare(got, ref, x, rows, n_blocks=3)
    no_device_error()
