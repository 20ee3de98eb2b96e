"""Pins for the oracle's block quantizers, dequantizer and scale layout.

Each check uses an independent route: torch's float8 decoders, numpy brute
force over the 16 codes, the scale rule the pages state (block max / 6), and
hand-computed layout offsets.
"""
import json
from pathlib import Path

import numpy as np
import pytest
import torch

import synth

FACTS = json.loads((Path(__file__).parent / "golden" / "page_facts.json").read_text())
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def e4m3_torch(b):
    return torch.from_numpy(np.asarray(b, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def unpack(codes):
    c = np.asarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 15
    out[..., 1::2] = c >> 4
    return out


def check_nearest(v32: np.ndarray, codes: np.ndarray):
    """Every code is a nearest E2M1 point to v (saturating), ties to even."""
    v = v32.astype(np.float64)
    d = np.abs(GRID[None, :] - v[:, None])
    dmin = d.min(axis=1)
    ok_near = d[np.arange(v.size), codes] == dmin
    sat = np.abs(v) > 6
    ok_sat = (codes & 7) == 7
    assert np.all(np.where(sat, ok_sat, ok_near))
    ties = (np.sum(d == dmin[:, None], axis=1) > 1) & ~sat
    assert np.all((codes[ties] & 1) == 0)


def test_nvfp4_scale_is_block_max_over_six(orc):
    """Block scale ~ amax / 6 in E4M3 (RN error <= 2^-4 relative in the normal range)."""
    x = synth.small_like("gauss", 1, 64, 256)
    codes, scales = orc.nvfp4_quantize(x, 1.0)
    assert FACTS["nvfp4_block"]["value"] == 16
    amax = np.abs(x.reshape(64, 16, 16)).max(axis=2)
    target = amax / FACTS["nvfp4_block_scale_divisor"]["value"]
    got = e4m3_torch(scales)
    assert np.all(np.abs(got - target) <= target * 2.0 ** -4 + 1e-12)
    # the RN scale is exactly torch's E4M3 rounding of amax/(6*s_t)
    ref = torch.from_numpy((amax / np.float32(6.0)).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(ref.view(torch.uint8).numpy(), scales)


@pytest.mark.parametrize("kind,round_up", [("gauss", False), ("heavy", False),
                                           ("outlier", True), ("weight", True)])
def test_nvfp4_codes_are_nearest(orc, kind, round_up):
    x = synth.small_like(kind, 7, 48, 160)
    s_t = np.float32(np.abs(x).max()) / np.float32(6 * 448)
    codes, scales = orc.nvfp4_quantize(x, s_t, round_up=round_up)
    # x / S ("Looped Transformer quantization" sec. 2.5: x = W / s), numpy's binary32 division
    S = (e4m3_torch(scales).astype(np.float32) * np.float32(s_t)).astype(np.float32)
    v = (x.reshape(48, 10, 16) / S[:, :, None]).astype(np.float32).reshape(-1)
    check_nearest(v, unpack(codes).reshape(-1))


def test_nvfp4_hand_example(orc):
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 6.0
    x[0, 3] = -1.4
    x[0, 5] = 0.25            # tie between 0 and 0.5 -> 0
    x[0, 16] = 3.0            # second block: max 3 -> scale 0.5
    x[0, 17] = -1.0
    codes, scales = orc.nvfp4_quantize(x, 1.0)
    assert list(scales[0]) == [0x38, 0x30]      # E4M3 1.0 and 0.5
    c = unpack(codes)[0]
    assert c[0] == 7 and c[3] == 0xB and c[5] == 0  # 6 -> 6, -1.4 -> -1.5, 0.25 -> 0
    assert c[16] == 7 and c[17] == 0xC              # 3/0.5 = 6, -1/0.5 = -2


def test_nvfp4_round_up_scale_never_saturates(orc):
    """[LT] sec. 2.2: with s_t = max|W|/(6*256) and the scale rounded up, |x| <= 6."""
    assert FACTS["looped_tensor_scale_divisor"]["value"] == 6 * 256
    w = synth.small_like("outlier", 9, 64, 512)
    s_t = np.float32(np.abs(w).max()) / np.float32(1536)
    codes, scales = orc.nvfp4_quantize(w, s_t, round_up=True)
    S = (e4m3_torch(scales).astype(np.float32) * s_t).astype(np.float32)
    v = (w.reshape(64, 32, 16) / S[:, :, None]).astype(np.float32)
    assert np.abs(v).max() <= 6.0


def test_dequantize_matches_independent_decode_and_input(orc):
    x = synth.small_like("heavy", 2, 40, 96)
    s_t = np.float32(np.abs(x).max()) / np.float32(2688)
    codes, scales = orc.nvfp4_quantize(x, s_t)
    deq = orc.dequantize(orc.NVFP4, codes, scales, s_t, 40, 96)
    ref = GRID[unpack(codes)] * np.repeat(e4m3_torch(scales), 16, axis=1) * np.float64(s_t)
    assert np.array_equal(deq, ref)
    # each element lands within the largest half-gap (1.0 in normalised units)
    # of its input: catches swapped nibbles, rows or blocks
    S = np.repeat(e4m3_torch(scales) * np.float64(s_t), 16, axis=1)
    unsat = np.abs(x) <= 6 * S
    assert np.all(np.abs(deq - x)[unsat] <= S[unsat] * 1.0 + 1e-30)
    # MXFP4 path
    c2, s2 = orc.mxfp4_quantize(x)
    deq2 = orc.dequantize(orc.MXFP4, c2, s2, 0.0, 40, 96)
    sc = np.repeat(2.0 ** (s2.astype(np.float64) - 127), 32, axis=1)
    assert np.array_equal(deq2, GRID[unpack(c2)] * sc)


def test_degenerate_blocks(orc):
    z = np.zeros((3, 32), np.float32)
    codes, scales = orc.nvfp4_quantize(z, 0.0)
    assert not codes.any() and not scales.any()
    x = synth.small_like("gauss", 4, 3, 32)
    x[1, :16] = 0.0
    x[2, 16:] = -0.0
    s_t = np.float32(np.abs(x).max()) / np.float32(2688)
    codes, scales = orc.nvfp4_quantize(x, s_t)
    assert scales[1, 0] == 0 and not unpack(codes)[1, :16].any()
    assert scales[2, 1] == 0 and not unpack(codes)[2, 16:].any()
    c2, s2 = orc.mxfp4_quantize(z)
    assert not c2.any() and not s2.any()


@pytest.mark.parametrize("hadamard,use_chan,round_up", [(False, False, False), (True, False, False),
                                                       (True, True, False), (False, True, True)])
def test_mxfp4_exponent_and_codes(orc, hadamard, use_chan, round_up):
    assert FACTS["mxfp4_block"]["value"] == 32
    rows, cols = 24, 128
    x = synth.small_like("heavy", 5, rows, cols)
    chan = np.linspace(0.5, 2.0, cols).astype(np.float32) if use_chan else None
    codes, scales = orc.mxfp4_quantize(x, chan, hadamard=hadamard, round_up=round_up)
    y = orc.mx_transform(x, chan, hadamard) if (hadamard or use_chan) else x
    amax = np.abs(y.reshape(rows, 4, 32)).max(axis=2).astype(np.float64)
    e = scales.astype(np.int64) - 127
    scaled = amax * 2.0 ** (-e)
    if round_up:
        assert np.all(scaled <= 6.0) and np.all((scaled > 3.0) | (amax == 0))
    else:
        assert np.all((scaled >= 4.0) & (scaled < 8.0))
    v = (y.reshape(rows, 4, 32) * (2.0 ** (-e))[:, :, None].astype(np.float32)).astype(np.float32)
    check_nearest(v.reshape(-1), unpack(codes).reshape(-1))


def test_mxfp4_bits_per_element():
    # 32 four-bit codes plus one 8-bit scale per block
    assert (32 * 4 + 8) / 32 == FACTS["mxfp4_bits_per_element"]["value"]


def test_tc_scale_layout_offsets(orc):
    scols = 8
    # hand-computed from: atom (r/128, c/4) of 512 B, atom-row-major;
    # inside, byte (r%32)*16 + ((r/32)%4)*4 + c%4
    cases = {(0, 0): 0, (1, 0): 16, (32, 0): 4, (0, 1): 1, (33, 3): 16 + 4 + 3,
             (0, 4): 512, (127, 7): 512 + 31 * 16 + 3 * 4 + 3, (128, 0): 1024, (130, 5): 1024 + 512 + 32 + 1}
    for (r, c), off in cases.items():
        assert orc.tc_scale_offset(r, c, scols) == off
    assert orc.tc_scale_bytes(130, 5) == 256 * 8
    rng = np.random.default_rng(0)
    s = rng.integers(1, 255, size=(130, 5), dtype=np.uint8)
    tc = orc.scales_to_tc(s)
    assert np.array_equal(orc.scales_from_tc(tc, 130, 5), s)
    assert np.count_nonzero(tc) == s.size   # padding is zero, the map is injective


def _block_sse(orc, x, codes, scales, s_t):
    """Per-block sum of squared errors in the input's units, recomputed in numpy."""
    deq = orc.dequantize(orc.NVFP4, codes, scales, s_t, *x.shape)
    d = x.astype(np.float64) - deq
    return (d * d).reshape(x.shape[0], -1, 16).sum(axis=2)


def test_scale46_picks_the_better_rounded_up_candidate(orc):
    """4/6 block scaling ("Looped Transformer quantization", sec. 2.2): every
    block's scale is one of the two rounded-up E4M3 candidates (block max -> 6 or
    -> 4), the choice never has a larger squared error than the other candidate
    (numpy recomputation), and so it is never worse than plain round-up scaling."""
    import synth
    w = synth.small_like("weight", 21, 64, 256)
    s_t = orc.tensor_scale(orc.amax(w), 1536.0)
    c46, s46 = orc.nvfp4_quantize46(w, s_t)
    c6, s6 = orc.nvfp4_quantize(w, s_t, round_up=True)
    amax = np.abs(w.astype(np.float32)).reshape(64, -1, 16).max(axis=2)
    cand4 = np.vectorize(lambda a: orc.e4m3_encode(float(np.float32(a) / np.float32(np.float32(4.0) * s_t)),
                                                   round_up=True))(amax)
    assert np.all((s46 == s6) | (s46 == cand4))
    e46 = _block_sse(orc, w, c46, s46, s_t)
    e6 = _block_sse(orc, w, c6, s6, s_t)
    assert np.all(e46 <= e6)
    assert np.any(s46 != s6)                     # the 4-candidate wins somewhere on real data
    # where the 4-candidate was chosen it was strictly better
    four = s46 != s6
    assert np.all(e46[four] < e6[four])


def test_scale46_keeps_normalised_weights_in_range(orc):
    """With s_t = max|W| / (6 * 256) both rounded-up candidates keep |x| <= 6
    (page fact), so no code of a 4/6-scaled weight saturates beyond the grid."""
    import synth
    w = synth.small_like("weight", 22, 32, 512)
    s_t = orc.tensor_scale(orc.amax(w), 1536.0)
    codes, scales = orc.nvfp4_quantize46(w, s_t)
    S = orc.dequantize(orc.NVFP4, np.full_like(codes, 0x22), scales, s_t, 32, 512)
    x = w.astype(np.float64) / S
    assert np.abs(x).max() <= 6.0 * (1 + 2 ** -20)
