"""The allocation-free block entry point (h3b_block_forward_noalloc).

It serves callers that cannot allocate device memory when they run the block
(for example, code whose device allocator belongs to a host framework that
forbids side allocations). The test calls it twice in a row through the C ABI
and checks each result against the workspace entry point's result, within the
block tolerance used elsewhere (relative L2 <= 1e-2). It also checks that
dimensions needing more than the fixed scratch are refused before any launch.
This file sorts last so a run that stops at the first failure has already run
every other test; it passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import bf16_dev, bf16_host, no_device_error, rel_l2, require_gpu, to_dev
from video_diffusion_transformer_adaln_b200 import h3b, synth
from video_diffusion_transformer_adaln_b200.runtime import DeviceBlock, block_forward, dims_of, workspace

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    require_gpu()
    h3b.h3b_device_error(clear=True)
    wl = synth.WORKLOADS["d256_L512"]
    raw, c, x = synth.block_weights(wl), synth.cond(wl), synth.x_input(wl)
    dims = dims_of(wl)
    blk = DeviceBlock.from_host(raw)
    c_dev = to_dev(c)
    ref = bf16_dev(x)
    block_forward(dims, blk, c_dev, ref, workspace(dims))
    torch.cuda.synchronize()
    want = O.bf16_decode(bf16_host(ref))
    for _ in range(2):
        xa = bf16_dev(x)
        h3b.h3b_block_forward_noalloc(dims, blk.struct, c_dev, xa)
        torch.cuda.synchronize()
        got = O.bf16_decode(bf16_host(xa))
        assert np.isfinite(got).all()
        assert rel_l2(got, want) <= 1e-2
    no_device_error()


def test_noalloc_refuses_dims_beyond_its_scratch():
    require_gpu()
    wl = synth.WORKLOADS["d2048_L4096"]  # needs about 100 MB of scratch
    dims = dims_of(wl)
    assert h3b.h3b_workspace_size(dims) > (32 << 20)
    x = torch.zeros((wl.L, wl.d), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((1, wl.d), dtype=torch.float32, device="cuda")
    w = h3b.BlockWeights()  # never dereferenced: the size check comes first
    with pytest.raises(h3b.H3BError) as e:
        h3b.h3b_block_forward_noalloc(dims, w, c, x)
    assert e.value.status == -4
