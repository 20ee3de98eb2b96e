"""Pins for the oracle's scalar codecs (E2M1, E4M3, E8M0).

The expectations come from the format definitions the pages give (bit
layout, grid size, range), from torch's independent float8 codecs, and from
brute force over every code.
"""
import json
import math
from pathlib import Path

import numpy as np
import pytest
import torch

FACTS = json.loads((Path(__file__).parent / "golden" / "page_facts.json").read_text())


def e2m1_from_bits(code: int) -> float:
    """Value of an E2M1 code from its bit fields alone (1 sign, 2 exponent
    with bias 1, 1 mantissa; exponent field 0 is subnormal)."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = (m / 2.0) if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)
    return -mag if s else mag


def test_e2m1_grid_matches_bit_definition(orc):
    assert FACTS["e2m1_bits"]["value"] == [1, 2, 1]
    vals = [orc.e2m1_decode(c) for c in range(16)]
    assert vals == [e2m1_from_bits(c) for c in range(16)]
    assert len(vals) == FACTS["e2m1_codes"]["value"]
    assert len(set(vals)) == FACTS["e2m1_distinct_values"]["value"]
    pos = sorted(set(v for v in vals if v >= 0))
    assert len(pos) == FACTS["e2m1_positive_points"]["value"]
    assert [min(vals), max(vals)] == FACTS["e2m1_range"]["value"]
    assert max(np.diff(sorted(set(vals)))) == FACTS["e2m1_max_gap"]["value"]


def test_e2m1_encode_roundtrip_all_codes(orc):
    for c in range(16):
        v = orc.e2m1_decode(c)
        if c == 8:
            v = -0.0
        assert orc.e2m1_encode(v) == c


def test_e2m1_encode_is_nearest_brute_force(orc):
    grid = np.array([e2m1_from_bits(c) for c in range(16)])
    rng = np.random.default_rng(11)
    sweep = np.concatenate([
        np.arange(-8.0, 8.0, 1.0 / 256),
        rng.uniform(-9, 9, 4000),
        rng.standard_normal(2000) * 1e-3,
    ]).astype(np.float32)
    for v in sweep:
        c = orc.e2m1_encode(float(v))
        d = np.abs(grid - np.float64(v))
        if abs(v) > 6:
            assert c & 7 == 7 and (c >> 3) == (1 if np.signbit(v) else 0)
            continue
        assert d[c] == d.min(), (v, c)
        # sign bit follows the input sign bit
        assert (c >> 3) == (1 if np.signbit(v) else 0)


@pytest.mark.parametrize("v,expect", [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
    (-0.25, -0.0), (-0.75, -1.0), (-5.0, -4.0),
])
def test_e2m1_ties_to_even_mantissa(orc, v, expect):
    c = orc.e2m1_encode(v)
    assert orc.e2m1_decode(c) == expect and (c & 1) == 0


@pytest.mark.parametrize("v", [6.0, 6.5, 7.0, 100.0, float("inf")])
def test_e2m1_saturates_at_codebook_end(orc, v):
    assert orc.e2m1_encode(v) == 0x7
    assert orc.e2m1_encode(-v) == 0xF


def test_e2m1_negative_underflow_keeps_sign(orc):
    assert orc.e2m1_encode(-0.1) == 0x8
    assert orc.e2m1_encode(0.1) == 0x0


def test_e4m3_decode_matches_torch_all_codes(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for b in range(256):
        v = orc.e4m3_decode(b)
        if math.isnan(ref[b]):
            assert math.isnan(v)
        else:
            assert v == ref[b], b


def test_e4m3_encode_rn_matches_torch(orc):
    rng = np.random.default_rng(3)
    codes = np.arange(0, 0x7F)
    vals = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    mids = (vals[:-1] + vals[1:]) / 2.0
    sweep = np.concatenate([
        np.exp(rng.uniform(np.log(1e-4), np.log(447.0), 20000)),
        mids, vals[1:], np.nextafter(mids, 0), np.nextafter(mids, 1000),
    ]).astype(np.float32)
    sweep = sweep[(sweep > 0) & (sweep < 448)]
    ref = torch.from_numpy(sweep).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(v)) for v in sweep], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_ru_is_smallest_code_above(orc):
    rng = np.random.default_rng(4)
    sweep = np.exp(rng.uniform(np.log(1e-4), np.log(447.0), 5000)).astype(np.float32)
    for v in sweep:
        b = orc.e4m3_encode(float(v), round_up=True)
        assert orc.e4m3_decode(b) >= v
        if b > 0:
            assert orc.e4m3_decode(b - 1) < v
    # exact code values map to themselves
    for b in range(1, 0x7F):
        assert orc.e4m3_encode(orc.e4m3_decode(b), round_up=True) == b


def test_e4m3_saturation_and_zero(orc):
    for mode in (False, True):
        assert orc.e4m3_encode(1e6, mode) == 0x7E
        assert orc.e4m3_encode(448.0, mode) == 0x7E
        assert orc.e4m3_encode(0.0, mode) == 0x00
    assert orc.e4m3_decode(0x7E) == 448.0


def test_e8m0_decode_matches_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for b in range(255):
        assert orc.e8m0_decode(b) == ref[b]
    assert math.isnan(orc.e8m0_decode(255))


def test_mx_exponent_floor_and_round_up(orc):
    rng = np.random.default_rng(5)
    amaxes = np.exp(rng.uniform(np.log(1e-30), np.log(1e30), 3000)).astype(np.float32)
    for a in amaxes:
        a64 = float(a)
        e = orc.mx_exponent(a64)
        # OCP rule: the block max lands in [4, 8) after scaling by 2^-e
        assert 4.0 <= a64 * 2.0 ** (-e) < 8.0
        eu = orc.mx_exponent(a64, round_up=True)
        # smallest exponent with amax <= 6 * 2^e, by brute force over e
        brute = min(k for k in range(-140, 140) if a64 <= 6.0 * 2.0 ** k)
        assert eu == brute
    assert orc.mx_exponent(0.0) == -127
    # subnormal block maxima clamp to the smallest E8M0 exponent
    assert orc.mx_exponent(1e-42) == -127
