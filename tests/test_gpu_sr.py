"""GPU parity of the stochastic-rounding requant: codes bit for bit against the
oracle (same Philox4x32-10 stream, same rounding rule), through the C-ABI."""
import numpy as np
import pytest

import oracle
import synth
import mxfp4_w4a4_block_b200 as q4
from gpu_util import dev, host
from test_gpu_sigma_delta import setup_scales

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("tc", [True, False])
@pytest.mark.parametrize("shape,seed,visit", [((200, 352), 42, 0), ((64, 512), 42, 31), ((33, 1024), 2**40 + 5, 7)])
def test_sr_requant_bit_exact(fmt, tc, shape, seed, visit):
    rows, cols = shape
    w = synth.small_like("weight", rows + cols + visit, rows, cols)
    s_t, g_t, g_sc, o_sc = setup_scales(fmt, w, tc)
    flags = q4.LAYOUT_TC if tc else 0
    gc = q4.q4_sr_requant(fmt, dev(w), g_sc, seed, visit, gscale=g_t, flags=flags)
    oc = oracle.sr_requant(fmt, w, o_sc, s_t, seed, visit)
    assert np.array_equal(host(gc), oc)


def test_sr_requant_looped_weight_visits():
    """A 4096 x 1024 looped-core weight over four visits (seed 42): bit exact on
    every visit, and consecutive visits draw different codes."""
    w = synth.looped()["w"][-1]
    s_t, g_t, g_sc, o_sc = setup_scales(q4.NVFP4, w)
    prev = None
    for visit in range(4):
        gc = host(q4.q4_sr_requant(q4.NVFP4, dev(w), g_sc, 42, visit, gscale=g_t))
        assert np.array_equal(gc, oracle.sr_requant(q4.NVFP4, w, o_sc, s_t, 42, visit))
        if prev is not None:
            assert not np.array_equal(gc, prev)
        prev = gc
