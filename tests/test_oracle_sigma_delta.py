"""Pins for the Sigma-Delta oracle.

"Looped Transformer quantization" sec. 2.1 (recursion, telescoping, the x = 0.3
integer-grid example) and sec. 2.2 (residue bound |r_k| <= d/2 for x inside the
codebook hull, the divergent counter-example, |r| <= 1 for E2M1 with the
rounded-up 4/6 scale).  The integer-grid sequence is checked against the closed
form sum_{i<=k} q_i = floor(k x + 1/2), which follows from the telescoping sum
and the half-open residue range of floor(v + 1/2), not from the recursion.
"""
import json
from fractions import Fraction
from pathlib import Path

import numpy as np
import pytest
import torch

import synth
from oracle import sigma_delta_exact as sde

FACTS = json.loads((Path(__file__).parent / "golden" / "page_facts.json").read_text())
E2M1 = [Fraction(v) for v in (-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6)]
# points whose E2M1 mantissa bit is 0 (0 and 2^(e-1) for e = 1..3)
EVEN_MANTISSA = {Fraction(0), Fraction(1), Fraction(2), Fraction(4)}


def even_mantissa(p):
    return abs(p) in EVEN_MANTISSA


def test_x03_integer_grid_closed_form():
    x = Fraction(3, 10)
    m = 40
    vs, qs, rs = sde.sequence(x, sde.floor_half_up, m)
    cum = 0
    for k in range(1, m + 1):
        cum += qs[k - 1]
        assert cum == Fraction((k * x + Fraction(1, 2)).__floor__())
        prefix_err = cum - k * x
        assert prefix_err == -rs[k - 1]
        assert abs(prefix_err) <= FACTS["x03_prefix_error_bound"]["value"]
    # a 1 every few steps: 3 ones in every 10
    assert sum(qs[:10]) == 3
    # the first eight steps, as the closed form gives them
    assert qs[:8] == [0, 1, 0, 0, 1, 0, 0, 0]
    # static RTN returns 0 each visit, a constant error of -0.3
    assert sde.floor_half_up(x) == 0
    assert float(sde.floor_half_up(x) - x) == FACTS["x03_rtn_step_error"]["value"]


def test_residue_bound_random_codebooks():
    rng = np.random.default_rng(0)
    for trial in range(60):
        pts = sorted(set(Fraction(int(v), 8) for v in rng.integers(-64, 64, size=rng.integers(2, 9))))
        if len(pts) < 2:
            continue
        d = max(b - a for a, b in zip(pts, pts[1:]))
        x = pts[0] + (pts[-1] - pts[0]) * Fraction(int(rng.integers(0, 1001)), 1000)
        q = sde.nearest(pts, tie="up" if trial % 2 else (lambda p: p < 0))
        vs, qs, rs = sde.sequence(x, q, 120)
        assert all(abs(r) <= d / 2 for r in rs)
        # telescoping: sum(q_k - x) = -r_m
        assert sum(qs) - len(qs) * x == -rs[-1]


def test_divergence_outside_hull():
    ex = FACTS["divergence_example"]["value"]
    q = sde.nearest([Fraction(c) for c in ex["codebook"]])
    _, _, rs = sde.sequence(ex["x"], q, 20)
    assert rs == [Fraction(k) for k in range(1, 21)]


def test_e2m1_bound_is_one():
    assert FACTS["e2m1_residue_bound"]["value"] == FACTS["e2m1_max_gap"]["value"] / 2
    q = sde.nearest(E2M1, tie=even_mantissa)
    rng = np.random.default_rng(1)
    for _ in range(40):
        x = Fraction(int(rng.integers(-6000, 6001)), 1000)
        vs, _, rs = sde.sequence(x, q, 64)
        assert all(abs(r) <= 1 for r in rs)
        lo, hi = FACTS["feedback_input_range"]["value"]
        assert all(lo <= v <= hi for v in vs)


def _unit_scale_block(rows, cols):
    """NVFP4 scales of exactly 1.0 (E4M3 0x38) with s_t = 1, so x = w exactly."""
    return np.full((rows, cols // 16), 0x38, np.uint8)


def test_c_oracle_equals_exact_recursion_on_dyadic_inputs(orc):
    rng = np.random.default_rng(2)
    rows, cols = 4, 64
    w = (rng.integers(-6 * 4096, 6 * 4096 + 1, size=(rows, cols)) / 4096.0).astype(np.float32)
    scales = _unit_scale_block(rows, cols)
    r = np.zeros_like(w)
    q = sde.nearest(E2M1, tie=even_mantissa)
    exact = [sde.sequence(Fraction(float(v)), q, 24) for v in w.reshape(-1)]
    for k in range(24):
        codes = orc.sigma_delta_step(orc.NVFP4, w, scales, 1.0, r)
        dec = np.array([orc.e2m1_decode(int(c)) for c in orc.unpack_codes(codes).reshape(-1)])
        assert np.array_equal(dec, np.array([float(e[1][k]) for e in exact]))
        assert np.array_equal(r.reshape(-1).astype(np.float64),
                              np.array([float(e[2][k]) for e in exact]))


def test_c_oracle_divergence_outside_range(orc):
    w = np.full((1, 16), 7.0, np.float32)
    r = np.zeros_like(w)
    for k in range(1, 9):
        codes = orc.sigma_delta_step(orc.NVFP4, w, _unit_scale_block(1, 16), 1.0, r)
        assert np.all(orc.unpack_codes(codes) == 7)
        assert np.all(r == k)


def e4m3_torch(b):
    return torch.from_numpy(np.asarray(b, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_looped_weights_bound_telescoping_first_visit(orc, fmt):
    w = synth.small_like("weight", 8, 32, 256)
    R = 8
    if fmt == "nvfp4":
        f = orc.NVFP4
        s_t = np.float32(np.abs(w).max()) / np.float32(1536)
        rtn_codes, scales = orc.nvfp4_quantize(w, s_t, round_up=True)
        S = np.repeat((e4m3_torch(scales).astype(np.float32) * s_t).astype(np.float32), 16, axis=1)
    else:
        f = orc.MXFP4
        s_t = np.float32(0)
        rtn_codes, scales = orc.mxfp4_quantize(w, round_up=True)
        S = np.repeat((2.0 ** (scales.astype(np.float64) - 127)).astype(np.float32), 32, axis=1)
    x = (w / S).astype(np.float32).astype(np.float64)       # sec. 2.5: x = W / s
    r = np.zeros_like(w)
    cum = np.zeros_like(x)
    for k in range(1, R + 1):
        codes = orc.sigma_delta_step(f, w, scales, s_t, r)
        if k == 1:
            assert np.array_equal(codes, rtn_codes)      # first visit = RTN codes
        assert np.abs(r).max() <= FACTS["e2m1_residue_bound"]["value"] * (1 + 2 ** -20)
        q = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, 0, -0.5, -1, -1.5, -2, -3, -4, -6])[orc.unpack_codes(codes)]
        cum += q - x
        # telescoping sum(q_k - x) = -r_k, up to binary32 rounding of v = x + r
        assert np.abs(cum + r).max() <= k * 2.0 ** -20 * 8
    # mean error after R visits is within d / (2R)
    assert np.abs(cum / R).max() <= 2.0 / (2 * R) * (1 + 1e-5)


def test_codebanks_reverse_tail_schedule(orc):
    """Codebanks of a K-step chain ("Looped Transformer quantization", sec. 2.3):
    the chain starts from r_0 = 0, so bank 0 -- the code of the LAST tail visit
    in the reverse schedule -- is the plain round-to-nearest code; every later
    bank is the next Sigma-Delta step; the mean of the K decoded codes tracks x
    within the first-order bound d / (2K) (largest gap d = 2 on E2M1)."""
    import synth
    w = synth.small_like("weight", 11, 48, 64)
    s_t = orc.tensor_scale(orc.amax(w), 1536.0)
    rtn, sc = orc.nvfp4_quantize(w, s_t, round_up=True)
    K = 12
    banks, rK = orc.sigma_delta_codebanks(orc.NVFP4, w, sc, s_t, K)
    assert banks.shape == (K, 48, 32)
    assert np.array_equal(banks[0], rtn)
    r = np.zeros_like(w)
    for k in range(K):
        assert np.array_equal(orc.sigma_delta_step(orc.NVFP4, w, sc, s_t, r), banks[k])
    assert np.array_equal(r.view(np.uint32), rK.view(np.uint32))
    # mean decoded code vs the normalised weight x = w / S
    S = orc.dequantize(orc.NVFP4, np.full_like(rtn, 0x22), sc, s_t, 48, 64)   # code 1.0 -> S per element
    x = w.astype(np.float64) / S
    mean = np.mean([orc.dequantize(orc.NVFP4, banks[k], sc, 1.0, 48, 64) / (S / s_t) for k in range(K)], axis=0)
    assert np.max(np.abs(mean - x)) <= 2.0 / (2 * K) + 1e-6
