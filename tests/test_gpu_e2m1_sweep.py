"""The library's E2M1 conversion on every binary32 value with |v| <= 8, both
signs, against the oracle's encoder.

The oracle is scanned over the same 2 x (0x41000000 + 1) bit patterns on the
host (the e2m1_oracle_runs fixture, pinned to round-to-nearest-even on the
grid by tests/test_oracle_e2m1_sweep.py); the GPU kernel converts every
pattern with the two helpers the quantizers use and compares each code with
the oracle's run table.  Bit for bit, no sampling.
"""
import ctypes
import subprocess
from pathlib import Path

import numpy as np
import pytest
import torch

from conftest import E2M1_SWEEP_HI

pytestmark = pytest.mark.gpu

CSRC = Path(__file__).resolve().parent.parent / "mxfp4_w4a4_block_b200" / "csrc"


@pytest.fixture(scope="module")
def sweep(tmp_path_factory):
    from mxfp4_w4a4_block_b200 import build
    out = tmp_path_factory.mktemp("e2m1") / "libe2m1_sweep.so"
    subprocess.run([build.nvcc(), *build.NVCC_FLAGS, "-shared", "-I", str(CSRC),
                    str(Path(__file__).parent / "e2m1_sweep.cu"), "-o", str(out)], check=True)
    lib = ctypes.CDLL(str(out))
    P, u32 = ctypes.c_void_p, ctypes.c_uint32
    lib.e2m1_sweep.argtypes = [u32, u32, P, P, ctypes.c_int, P, P]
    return lib


@pytest.mark.parametrize("sign", [0, 1])
def test_e2m1_conversion_every_binary32_up_to_8(sweep, e2m1_oracle_runs, sign):
    starts, codes = e2m1_oracle_runs[sign]
    s = torch.from_numpy(starts.astype(np.uint32).view(np.int32)).cuda()
    c = torch.from_numpy(codes).cuda()
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert sweep.e2m1_sweep(sign, E2M1_SWEEP_HI, s.data_ptr(), c.data_ptr(), len(starts), bad.data_ptr(),
                            first.data_ptr()) == 0
    torch.cuda.synchronize()
    f = first.cpu().numpy().view(np.uint32)
    assert int(bad.item()) == 0, f"first mismatch: bits {(sign << 31) | int(f[0]):#010x} got {f[1]} want {f[2]}"
