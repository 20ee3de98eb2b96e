"""The library's binary32 quotient helpers against CUDA's correctly rounded
division.

Every normalisation x = W / S of the path ("Looped Transformer quantization",
sec. 2.5) is formed on the device from y = RN(1 / S) by one Markstein
correction step (q4_codec.cuh).  These tests compare it with __fdiv_rn:

* on significand pairs: every one of the 2^23 significands of S against a
  grid of 4096 significands of w (the full 2^46 pairs when
  Q4_QUOTIENT_EXHAUSTIVE=1 is set; a full run takes about a minute);
* elementwise through the guarded form on zeros, subnormals, tiny and huge w,
  and S at and beyond the ends of the fast range: bit for bit, signs of zeros
  included;
* through the quantizer's block form: the E2M1 codes of whole 16-blocks whose
  quotients land on and next to every rounding midpoint.
"""
import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parent.parent
CSRC = ROOT / "mxfp4_w4a4_block_b200" / "csrc"


@pytest.fixture(scope="module")
def qc(tmp_path_factory):
    from mxfp4_w4a4_block_b200 import build
    out = tmp_path_factory.mktemp("qc") / "libquotient_check.so"
    cmd = [build.nvcc(), *build.NVCC_FLAGS, "-shared", "-I", str(CSRC),
           str(Path(__file__).parent / "quotient_check.cu"), "-o", str(out)]
    subprocess.run(cmd, check=True)
    lib = ctypes.CDLL(str(out))
    P, i64, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32
    lib.qc_pairs.argtypes = [u32, u32, u32, u32, P, P]
    lib.qc_elems.argtypes = [P, P, i64, P, P]
    lib.qc_codes.argtypes = [P, P, i64, P, P]
    return lib


def _pairs(qc, a_off, a_step, b_chunk=1 << 16):
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(3, dtype=torch.int32, device="cuda")
    for b0 in range(0, 1 << 23, b_chunk):
        assert qc.qc_pairs(b0, b_chunk, a_off, a_step, count.data_ptr(), first.data_ptr()) == 0
    torch.cuda.synchronize()
    return int(count.item()), first.cpu().numpy()


def test_correction_step_on_significand_pairs(qc):
    if os.environ.get("Q4_QUOTIENT_EXHAUSTIVE") == "1":
        n, first = _pairs(qc, 0, 1)
    else:
        n, first = 0, None
        for off in (0, 1, 977, 2047):
            k, f = _pairs(qc, off, 2048)
            n += k
            first = f if first is None or k else first
    assert n == 0, f"{n} mismatches, first w = 1.{first[0]:06x}, S = 1.{first[1]:06x}"


def _edge_values():
    rng = np.random.default_rng(7)
    tiny = np.array([0.0, -0.0, 1e-45, -1e-45, 2.0 ** -149, 2.0 ** -126, -(2.0 ** -126), 2.0 ** -100,
                     2.0 ** -97, 2.0 ** -96, 3.0 * 2.0 ** -97, -5.0 * 2.0 ** -99], np.float32)
    mags = (2.0 ** rng.uniform(-149, 127, 4000)).astype(np.float32)
    w = np.concatenate([tiny, mags, -mags, rng.standard_normal(4000).astype(np.float32)])
    S_list = np.array([2.0 ** -96, 2.0 ** 96, 2.0 ** -97, 2.0 ** 97, 1.5 * 2.0 ** -96, 1.75 * 2.0 ** 95,
                       2.0 ** -120, 2.0 ** 120, 0.0123, 448.0 * 0.0123, 1.0, 3.0], np.float32)
    S_rand = (rng.uniform(1, 2, 64) * 2.0 ** rng.integers(-100, 100, 64)).astype(np.float32)
    S_all = np.concatenate([S_list, S_rand])
    ww = np.tile(w, S_all.size)
    SS = np.repeat(S_all, w.size)
    return ww, SS


def test_guarded_quotient_matches_division_bitwise(qc):
    w, S = _edge_values()
    wt, St = torch.from_numpy(w).cuda(), torch.from_numpy(S).cuda()
    rn, dv = torch.empty_like(wt), torch.empty_like(wt)
    assert qc.qc_elems(wt.data_ptr(), St.data_ptr(), w.size, rn.data_ptr(), dv.data_ptr()) == 0
    torch.cuda.synchronize()
    a = rn.cpu().numpy().view(np.uint32)
    b = dv.cpu().numpy().view(np.uint32)
    bad = np.nonzero(a != b)[0]
    assert bad.size == 0, [(float(w[i]), float(S[i]), hex(a[i]), hex(b[i])) for i in bad[:5]]
    # and the division is the one numpy computes on the host (IEEE binary32)
    with np.errstate(over="ignore"):
        host = (w / S).astype(np.float32).view(np.uint32)
    assert np.array_equal(b, host)


def test_block_form_codes_at_midpoints(qc):
    """Blocks with S in and out of the fast range whose values sit on, and one
    and two units either side of, every E2M1 rounding midpoint (and 6 S, so
    the block maximum is what a quantizer block would have)."""
    rng = np.random.default_rng(11)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.0, 6.0, 7.0], np.float32)
    blocks, scales = [], []
    for _ in range(20000):
        S = np.float32(rng.uniform(1, 2) * 2.0 ** rng.integers(-110, 100))
        t = rng.choice(mids, 15)
        x0 = (t * S).astype(np.float32)
        k = rng.integers(-2, 3, 15)
        x = np.array([np.float32(v) for v in x0])
        for i in range(15):
            for _ in range(abs(int(k[i]))):
                x[i] = np.nextafter(x[i], np.float32(np.inf) if k[i] > 0 else np.float32(-np.inf))
        x *= np.where(rng.random(15) < 0.5, -1, 1).astype(np.float32)
        blocks.append(np.concatenate([[np.float32(6.0) * S], x]).astype(np.float32))
        scales.append(S)
    xb = torch.from_numpy(np.stack(blocks).reshape(-1)).cuda()
    Sb = torch.from_numpy(np.array(scales, np.float32)).cuda()
    n = len(scales)
    got = torch.empty(2 * n, dtype=torch.int32, device="cuda")
    want = torch.empty_like(got)
    assert qc.qc_codes(xb.data_ptr(), Sb.data_ptr(), n, got.data_ptr(), want.data_ptr()) == 0
    torch.cuda.synchronize()
    assert torch.equal(got, want)
