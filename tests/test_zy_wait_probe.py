"""Failure detection without a GPU fault: a bounded device-side wait that nothing
completes runs out, records its code in the device error word and returns; the host
reads the code and the context goes on running kernels. (Last in the GPU run.)"""
import time

import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import bf16_dev, require_gpu
from video_diffusion_transformer_adaln_b200 import h3b, synth

pytestmark = pytest.mark.gpu

ERR_WAIT_PROBE = 1 << 5


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    require_gpu()
    h3b.h3b_device_error(clear=True)
    t0 = time.perf_counter()
    assert h3b.h3b_test_bounded_wait(20_000_000) == 1  # 20 ms, nothing arrives
    assert time.perf_counter() - t0 < 10.0
    code = h3b.h3b_device_error(clear=True)
    assert code & ERR_WAIT_PROBE
    assert h3b.h3b_device_error(clear=True) == 0
    # the same context still runs the library's kernels correctly
    r = np.random.default_rng(5)
    hb = synth.f32_to_bf16_bits(r.standard_normal((64, 256)).astype(np.float32))
    q = torch.empty((64, 256), dtype=torch.int8, device="cuda")
    s = torch.empty(64, dtype=torch.float32, device="cuda")
    h3b.h3b_quantize_rows(bf16_dev(hb), q, s)
    qo, so = O.quantize_rows(synth.bf16_bits_to_f32(hb))
    assert np.array_equal(q.cpu().numpy(), qo) and np.array_equal(s.cpu().numpy(), so)
    assert h3b.h3b_device_error(clear=True) == 0
