import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


# Every binary32 value with |v| <= 8 (bit patterns 0 .. 0x41000000 of each sign)
E2M1_SWEEP_HI = 0x41000000


@pytest.fixture(scope="session")
def e2m1_oracle_runs(orc, tmp_path_factory):
    """The oracle's E2M1 encoder over every binary32 value with |v| <= 8, as
    runs of equal codes per sign: {sign: (starts uint32[], codes uint8[])}.
    Built from a full scan (tests/e2m1_runs.c, OpenMP over the host cores)."""
    import ctypes
    import subprocess

    import numpy as np
    out = tmp_path_factory.mktemp("e2m1") / "libe2m1_runs.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(out),
                    str(Path(__file__).parent / "e2m1_runs.c")], check=True)
    helper = ctypes.CDLL(str(out))
    helper.e2m1_runs.restype = ctypes.c_int
    helper.e2m1_runs.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_int]
    enc = ctypes.cast(orc._load().q4o_e2m1_encode, ctypes.c_void_p)
    runs = {}
    for sign in (0, 1):
        starts = np.zeros(64, np.uint32)
        codes = np.zeros(64, np.uint8)
        n = helper.e2m1_runs(enc, sign, E2M1_SWEEP_HI, starts.ctypes.data, codes.ctypes.data, 64)
        assert n > 0
        runs[sign] = (starts[:n].copy(), codes[:n].copy())
    return runs
