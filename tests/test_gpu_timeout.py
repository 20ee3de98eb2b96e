"""Failure detection on the device: a bounded wait that runs out.

Every wait inside the kernels is bounded (q4_set_wait_limit); when one runs
out the kernel records Q4_ERR_TIMEOUT, winds down and exits, and the CUDA
context stays usable.  Here the quantizer's producer is told to load nothing
for each CTA's first tile (Q4_INJECT_STALL), so its consumers wait on a stage
that never fills: a flag that nothing sets.  With a short limit the launch ends
by itself, q4_get_device_error reports the time-out once, and the same call
without the injection is then bit-exact against the oracle on the same
stream.  The quantizer holds no tensor memory, so nothing can be left
allocated by the abandoned launch."""
import numpy as np
import pytest
import torch

import mxfp4_w4a4_block_b200 as q4
import oracle
import synth
from gpu_util import dev, gscale_dev, host

pytestmark = pytest.mark.gpu

TIMEOUT = 6          # Q4_ERR_TIMEOUT


def test_quantize_wait_runs_out_and_the_context_stays_usable():
    x32 = synth.small_like("heavy", 5, 4096, 1024)
    x_t = dev(synth.to_bf16(x32))
    x32 = synth.bf16_to_f32(synth.to_bf16(x32))
    s_t = oracle.tensor_scale(oracle.amax(x32), 2688.0)
    g = gscale_dev(s_t)
    assert q4.q4_get_device_error() == 0
    try:
        q4.q4_set_wait_limit(100_000)           # ~50 us at B200 clocks
        q4.q4_quantize(q4.NVFP4, x_t, gscale=g, flags=q4.LAYOUT_TC | q4.INJECT_STALL)
        assert q4.q4_get_device_error() == TIMEOUT
        assert q4.q4_get_device_error() == 0    # read once, then cleared
    finally:
        q4.q4_set_wait_limit(0)
    codes, scales = q4.q4_quantize(q4.NVFP4, x_t, gscale=g, flags=q4.LAYOUT_TC)
    oc, os_ = oracle.nvfp4_quantize(x32, s_t)
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(host(scales), oracle.scales_to_tc(os_))
    assert q4.q4_get_device_error() == 0
