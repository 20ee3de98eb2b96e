"""Pins for the oracle's normalisation step x = W / s.

"Looped Transformer quantization" sec. 2.5 gives the Sigma-Delta forward as a
short PyTorch sketch: the block scales s are fixed (block_scale_46), the
weight is normalised by one division x = W / s, the residue starts at zero,
and every visit does v = x + r, q = e2m1_round(v), r = v - q.  The tests here
evaluate that sketch with torch's own binary32 tensor operations (a division,
an add and a subtract per element, and an E2M1 rounding written below from the
grid's definition) and require the oracle's codes and residues to equal it bit
for bit over R = 32 visits of a looped-core weight, on non-unit scales.

A step that normalises by a reciprocal, x = W * (1 / s), is a different
function: it rounds twice.  Each pin below also shows that this other step
fails it, so the pins can tell the two apart.
"""
import numpy as np
import pytest
import torch

import synth

MAGS = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=torch.float64)
EVEN = torch.arange(8) % 2 == 0          # code index with mantissa bit 0


def e2m1_round(v: torch.Tensor):
    """Nearest E2M1 value of each binary32 v and its 4-bit code.

    Nearest point of {0, .5, 1, 1.5, 2, 3, 4, 6} to |v|, magnitudes above 6
    saturating to 6; of two equally near points the one whose code has mantissa
    bit 0 (codes 0, 2, 4, 6); the sign is v's, so a negative v that rounds to 0
    gives -0 and code 8."""
    a = v.double().abs().clamp(max=6.0)
    d = (a.unsqueeze(-1) - MAGS).abs()
    tied = d == d.min(-1, keepdim=True).values
    pref = tied & EVEN
    idx = torch.where(pref.any(-1), pref.to(torch.int8).argmax(-1), tied.to(torch.int8).argmax(-1))
    q = torch.copysign(MAGS[idx].float(), v)
    code = idx.to(torch.uint8) | (torch.signbit(v).to(torch.uint8) << 3)
    return q, code


def e4m3_values(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b, np.uint8)).view(torch.float8_e4m3fn).float()


def block_scale(scales: np.ndarray, s_t: np.float32) -> torch.Tensor:
    """s = dec(s_b) * s_t per element, one binary32 product (torch)."""
    s = e4m3_values(scales) * torch.tensor(s_t, dtype=torch.float32)
    return s.repeat_interleave(16, dim=1)


def sketch_chain(w: torch.Tensor, s: torch.Tensor, visits: int, reciprocal: bool = False):
    """The sec. 2.5 recursion in torch binary32; `reciprocal` swaps the division
    for x = W * (1 / s), the form this file shows to be different."""
    x = w * (1.0 / s) if reciprocal else w / s
    r = torch.zeros_like(x)
    out = []
    for _ in range(visits):
        v = x + r
        q, code = e2m1_round(v)
        r = v - q
        out.append((code, r.clone()))
    return out


def codes_of(orc, packed: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(orc.unpack_codes(packed))


@pytest.fixture(scope="module")
def looped_weight():
    # one looped-core weight: 1024 x 1024 ~ N(0, 0.02^2) (the shape of the four
    # square matrices of the looped core)
    w = synth.small_like("weight", 31, 1024, 1024)
    s_t = np.float32(np.abs(w).max()) / np.float32(6 * 256)      # sec. 2.2: max|W| / (6 * 256)
    return w, np.float32(s_t)


@pytest.mark.parametrize("rule", ["round_up", "block_scale_46"])
def test_sigma_delta_chain_equals_the_sketch(orc, looped_weight, rule):
    """32 visits of the oracle's step equal the sec. 2.5 sketch bit for bit, and
    the reciprocal form does not."""
    w, s_t = looped_weight
    if rule == "round_up":
        _, scales = orc.nvfp4_quantize(w, s_t, round_up=True)
    else:
        _, scales = orc.nvfp4_quantize46(w, s_t)
    s = block_scale(scales, s_t)
    assert not torch.all(s == s[0, 0])                    # non-unit, varying scales
    R = 32
    want = sketch_chain(torch.from_numpy(w), s, R)
    recip = sketch_chain(torch.from_numpy(w), s, R, reciprocal=True)
    r = np.zeros_like(w)
    code_flips = 0
    for k in range(R):
        codes = codes_of(orc, orc.sigma_delta_step(orc.NVFP4, w, scales, s_t, r))
        assert torch.equal(codes, want[k][0]), f"visit {k + 1}: codes"
        assert np.array_equal(r.view(np.uint32), want[k][1].numpy().view(np.uint32)), f"visit {k + 1}: residue"
        code_flips += int((recip[k][0] != want[k][0]).sum())
    # the reciprocal form changes codes over the chain, and its final residues
    assert code_flips > 0
    assert not torch.equal(recip[-1][1].view(torch.int32), want[-1][1].view(torch.int32))


def _step_ulps(x: np.float32, k: int) -> np.float32:
    """The binary32 value k representable steps from x."""
    toward = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
    for _ in range(abs(k)):
        x = np.nextafter(x, toward).astype(np.float32)
    return x


def _split_values(orc, s_t: np.float32, b: int, targets):
    """Binary32 values x near t * S (S = dec(b) * s_t, one binary32 product),
    for each target t, with RN(x / S) = t exactly but RN(x * RN(1 / S)) != t."""
    S = np.float32(np.float32(orc.e4m3_decode(b)) * s_t)
    rS = np.float32(np.float32(1.0) / S)
    found = []
    for t in targets:
        x0 = np.float32(np.float32(t) * S)
        for k in range(-4, 5):
            x = _step_ulps(x0, k)
            if np.float32(x / S) == np.float32(t) and np.float32(x * rS) != np.float32(t):
                found.append(x)
    return found


def _near_tie_blocks(orc, s_t: np.float32, sbytes):
    """Blocks whose normalised values sit on an E2M1 rounding boundary under the
    division but not under the reciprocal form.

    For a scale byte b, element 0 of the block is the value that selects b as
    the block scale (dec(b) * 6 s_t); the other 15 are values whose division
    by S lands exactly on a midpoint between grid points, signs alternating.
    Returns the blocks and their intended scale bytes."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    blocks, bytes_ = [], []
    for b in sbytes:
        found = _split_values(orc, s_t, b, mids)
        if len(found) < 4:
            continue
        lead = np.float32(np.float32(orc.e4m3_decode(b)) * np.float32(np.float32(6.0) * s_t))
        vals = np.asarray((found * 4)[:15], np.float32)
        signs = np.where(np.arange(15) % 2 == 0, 1, -1).astype(np.float32)
        blocks.append(np.concatenate([[lead], vals * signs]).astype(np.float32))
        bytes_.append(b)
    return np.stack(blocks), np.array(bytes_, np.uint8)


def test_nvfp4_quantize_near_ties_follow_the_division(orc):
    """NVFP4 codes are E2M1(RN(x / S)) on values where the division lands on a
    rounding boundary and the reciprocal form does not."""
    s_t = np.float32(0.0123)
    blocks, sbytes = _near_tie_blocks(orc, s_t, range(0x10, 0x77))
    assert len(blocks) >= 16
    codes, scales = orc.nvfp4_quantize(blocks, s_t)
    got = codes_of(orc, codes)
    keep = scales[:, 0] == sbytes                       # blocks whose scale is the intended byte
    assert keep.sum() >= 16
    S = block_scale(scales, s_t)
    x = torch.from_numpy(blocks)
    _, want = e2m1_round(x / S)
    _, recip = e2m1_round(x * (1.0 / S))
    assert torch.equal(got, want)
    assert int((recip[torch.from_numpy(keep)] != want[torch.from_numpy(keep)]).sum()) >= 32


GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def sr_code(x: np.float32, u: float) -> int:
    """Stochastic rounding of one normalised value (the rule of the SR baseline):
    between neighbouring magnitudes a <= |x| < b the magnitude is b when
    u < (|x| - a) / (b - a), else a; |x| >= 6 gives 6; the sign bit is x's.
    Evaluated in binary64, where every step is exact."""
    m = abs(float(x))
    if m >= 6.0:
        i = 7
    else:
        i = int(np.searchsorted(GRID, m, side="right")) - 1
        a, b = GRID[i], GRID[i + 1]
        i = i + 1 if u < (m - a) / (b - a) else i
    return i | (8 if np.signbit(x) else 0)


def test_sr_decisions_follow_the_division(orc):
    """Stochastic-rounding codes are decided on x = RN(w / S).

    For each element the uniform u of its (seed, visit, index) is computed from
    the Philox4x32-10 generator (pinned by its published known-answer vectors),
    and w is chosen so that u lies between the thresholds of RN(w / S) and of
    the reciprocal form's RN(w * RN(1 / S)) one unit lower: the two forms then
    give different codes, and the oracle must give the division's."""
    s_t = np.float32(0.0123)
    seed, visit = 42, 3
    rows, cols = 24, 16
    w = np.zeros((rows, cols), np.float32)
    sc = np.zeros((rows, 1), np.uint8)
    built = np.zeros((rows, cols), bool)
    want = np.zeros((rows, cols), np.uint8)
    for i in range(rows):
        b = 0x30 + 2 * i
        sc[i, 0] = b
        S = np.float32(np.float32(orc.e4m3_decode(b)) * s_t)
        rS = np.float32(np.float32(1.0) / S)
        for j in range(cols):
            e = i * cols + j
            g = e // 4
            word = orc.philox4x32_10([g & 0xFFFFFFFF, g >> 32, visit, 0], [seed & 0xFFFFFFFF, seed >> 32])[e % 4]
            u = float(int(word) >> 8) * 2.0 ** -24
            # x in [a, b) with (x - a) / (b - a) the smallest binary32-reachable
            # fraction above u, for a few of the grid's intervals
            for a, bb in ((1.0, 1.5), (1.5, 2.0), (2.0, 3.0), (3.0, 4.0), (0.5, 1.0)):
                ulp = float(np.spacing(np.float32(a)))
                step = ulp / (bb - a)
                x = np.float32(a + (np.floor(u / step) + 1) * step * (bb - a))
                if not (a <= x < bb):
                    continue
                hit = None
                x0 = np.float32(x * S)
                for k in range(-6, 7):
                    wv = _step_ulps(x0, k) * np.float32(1 if j % 2 == 0 else -1)
                    xd, xr = np.float32(wv / S), np.float32(wv * rS)
                    if abs(xd) == x and sr_code(xd, u) != sr_code(xr, u):
                        hit = wv
                        break
                if hit is not None:
                    w[i, j] = hit
                    want[i, j] = sr_code(np.float32(hit / S), u)
                    built[i, j] = True
                    break
    assert built.sum() >= 64
    got = orc.unpack_codes(orc.sr_requant(orc.NVFP4, w, sc, s_t, seed, visit))
    # elements not built are 0 and round to code 0 (or 8) either way
    assert np.array_equal(got[built], want[built])
