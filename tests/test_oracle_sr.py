"""Pins for the oracle's stochastic-rounding requant ("Looped Transformer
quantization", sec. 2.1: the SR baseline draws each code so that its
conditional expectation equals the weight) and its counter-based generator.

Philox4x32-10 is pinned to the known-answer vectors published with the
generator's reference implementation (Salmon et al., "Parallel Random Numbers:
As Easy as 1, 2, 3", SC 2011); the rounding rule to the grid facts (only the
two neighbours, grid points fixed, saturation) and to unbiasedness.
"""
import numpy as np
import pytest

import synth

KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]
MAGS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


@pytest.mark.parametrize("ctr,key,want", KAT)
def test_philox_known_answers(orc, ctr, key, want):
    assert tuple(int(v) for v in orc.philox4x32_10(ctr, key)) == want


def _values(orc, codes):
    c = orc.unpack_codes(codes)
    v = MAGS[c & 7]
    return np.where(c & 8, -v, v)


def _unit_scale_input(vals):
    """A 1 x 16k NVFP4 row whose every block has scale 1 (s_t = 1, E4M3 byte 0x38),
    so the normalised values are the inputs themselves."""
    x = np.asarray(vals, np.float32).reshape(1, -1)
    sc = np.full((1, x.shape[1] // 16), 0x38, np.uint8)
    return x, sc


def test_sr_only_neighbours_and_fixed_points(orc):
    rng = np.random.default_rng(0)
    x = rng.uniform(-7.5, 7.5, 16 * 512).astype(np.float32)
    x[:8] = [0.0, 0.5, 1.0, 1.5, 3.0, -4.0, 6.0, -6.0]        # grid points stay put
    x[8:12] = [6.5, -9.0, 100.0, -0.0]                      # saturation; signed zero
    xs, sc = _unit_scale_input(x)
    for visit in range(4):
        v = _values(orc, orc.sr_requant(orc.NVFP4, xs, sc, 1.0, 42, visit))[0]
        assert np.array_equal(v[:8], x[:8])
        assert np.array_equal(v[8:11], [6.0, -6.0, 6.0])
        m = np.abs(x)
        lo = MAGS[np.clip(np.searchsorted(MAGS, m, side="right") - 1, 0, 7)]
        hi = MAGS[np.clip(np.searchsorted(MAGS, m, side="right"), 0, 7)]
        inside = m < 6
        assert np.all((np.abs(v) == lo) | (np.abs(v) == hi) | ~inside)
        assert np.all((np.signbit(v) == np.signbit(x)) | (v == 0))


def test_sr_unbiased_and_visit_dependent(orc):
    """Averaged over visits the decoded code approaches x (within 5 sigma of the
    Bernoulli spread), and different visits draw different codes."""
    x = np.array([0.1, 0.3, 0.74, 1.2, 1.9, 2.25, 2.9, 3.6, 4.5, 5.9, -0.2, -1.3, -2.6, -3.3, -4.2, -5.5],
                 np.float32)
    xs, sc = _unit_scale_input(x)
    V = 2000
    acc = np.zeros(16)
    first = orc.sr_requant(orc.NVFP4, xs, sc, 1.0, 7, 0)
    differ = 0
    for visit in range(V):
        c = orc.sr_requant(orc.NVFP4, xs, sc, 1.0, 7, visit)
        differ += int(not np.array_equal(c, first))
        acc += _values(orc, c)[0]
    mean = acc / V
    m = np.abs(x)
    gap = MAGS[np.searchsorted(MAGS, m, side="right")] - MAGS[np.searchsorted(MAGS, m, side="right") - 1]
    sigma = gap / 2 / np.sqrt(V)
    assert np.all(np.abs(mean - x) <= 5 * sigma)
    assert differ > V // 2
    # the same seed and visit reproduce the same codes
    assert np.array_equal(orc.sr_requant(orc.NVFP4, xs, sc, 1.0, 7, 3), orc.sr_requant(orc.NVFP4, xs, sc, 1.0, 7, 3))


def test_sr_uses_the_sigma_delta_normalisation(orc):
    """x = W / S with the fixed RU block scales, as the Sigma-Delta step: a
    weight whose normalised value is on the grid is reproduced exactly."""
    w = synth.small_like("weight", 2, 8, 64)
    s_t = orc.tensor_scale(orc.amax(w), 1536.0)
    codes, sc = orc.nvfp4_quantize(w, s_t, round_up=True)
    deq = orc.dequantize(orc.NVFP4, codes, sc, s_t, 8, 64).astype(np.float32)
    # W := its own RTN dequantization: every normalised value is a grid point
    again = orc.sr_requant(orc.NVFP4, deq, sc, s_t, 42, 5)
    assert np.array_equal(_values(orc, again), _values(orc, codes))
