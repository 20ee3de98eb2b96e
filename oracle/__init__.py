"""CPU oracle for 4-bit block-scaled quantization, Sigma-Delta requantization
and the W4A4 GEMM.

TEST INFRASTRUCTURE ONLY: the reference that the CUDA path is checked
against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package.  The product package never imports
it and shares no code with it.

The arithmetic lives in ``q4_oracle.c`` (plain scalar C, binary32 steps in the
order the pages give, binary64 GEMM); this module only builds it with gcc,
loads it with ctypes and marshals numpy arrays.  The citations and the
readings taken where the pages are silent are in the C file's header.

Pins (tests/test_oracle_*.py) tie every function here to something other than
itself: the E2M1 grid and its 15 distinct values, torch's float8 codecs, scipy's
Sylvester Hadamard matrix, exact rational Sigma-Delta sequences, the residue
bound and telescoping identity, brute force over all codes, closed-form GEMMs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

NVFP4 = 0
MXFP4 = 1

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "q4_oracle.c"
_LIB = _HERE / "_build" / "libq4_oracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    _LIB.parent.mkdir(parents=True, exist_ok=True)
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".{os.getpid()}.tmp")
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(str(build()))
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    f32 = ctypes.c_float
    i32 = ctypes.c_int
    u8 = ctypes.c_uint8
    sig = {
        "q4o_e2m1_decode": (ctypes.c_double, [u8]),
        "q4o_e2m1_encode": (u8, [f32]),
        "q4o_e4m3_decode": (ctypes.c_double, [u8]),
        "q4o_e4m3_encode": (u8, [f32, i32]),
        "q4o_e8m0_decode": (ctypes.c_double, [u8]),
        "q4o_mx_exponent": (i32, [f32, i32]),
        "q4o_amax": (f32, [P, i64]),
        "q4o_tensor_scale": (f32, [f32, f32]),
        "q4o_nvfp4_quantize": (i32, [P, i64, i64, f32, i32, P, P]),
        "q4o_fwht32": (None, [P]),
        "q4o_mx_transform": (None, [P, P, i32, P]),
        "q4o_mxfp4_quantize": (i32, [P, i64, i64, P, i32, i32, P, P]),
        "q4o_tc_scale_bytes": (i64, [i64, i64]),
        "q4o_tc_scale_offset": (i64, [i64, i64, i64]),
        "q4o_scales_to_tc": (None, [P, i64, i64, P]),
        "q4o_scales_from_tc": (None, [P, i64, i64, P]),
        "q4o_dequantize": (i32, [i32, P, P, f32, i64, i64, P]),
        "q4o_sigma_delta_step": (i32, [i32, P, i64, i64, P, f32, P, P]),
        "q4o_gemm": (i32, [i32, i64, i64, i64, P, P, f32, P, P, f32, P, i64, P]),
        "q4o_gemm_w4a16": (i32, [i32, i64, i64, i64, P, P, P, f32, P, i64, P]),
        "q4o_philox4x32_10": (None, [P, P, P]),
        "q4o_nvfp4_quantize46": (i32, [P, i64, i64, f32, P, P]),
        "q4o_sr_requant": (i32, [i32, P, i64, i64, P, f32, ctypes.c_uint64, ctypes.c_uint32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    return a


# ---------------------------------------------------------------- scalar codecs
def e2m1_decode(code: int) -> float:
    return _load().q4o_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return _load().q4o_e2m1_encode(float(np.float32(v)))


def e4m3_decode(b: int) -> float:
    return _load().q4o_e4m3_decode(b)


def e4m3_encode(v: float, round_up: bool = False) -> int:
    return _load().q4o_e4m3_encode(float(np.float32(v)), int(round_up))


def e8m0_decode(b: int) -> float:
    return _load().q4o_e8m0_decode(b)


def mx_exponent(amax: float, round_up: bool = False) -> int:
    return _load().q4o_mx_exponent(float(np.float32(amax)), int(round_up))


# ---------------------------------------------------------------- tensor ops
def amax(x) -> np.float32:
    a = _f32(x)
    return np.float32(_load().q4o_amax(_ptr(a), a.size))


def tensor_scale(amax_value, denom) -> np.float32:
    return np.float32(_load().q4o_tensor_scale(float(np.float32(amax_value)),
                                               float(np.float32(denom))))


def nvfp4_quantize(x, s_t, round_up: bool = False):
    """x [rows, cols] (cast to float32) -> (codes u8 [rows, cols/2], scales u8 [rows, cols/16])."""
    a = _f32(x)
    rows, cols = a.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    rc = _load().q4o_nvfp4_quantize(_ptr(a), rows, cols, float(np.float32(s_t)),
                                    int(round_up), _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("nvfp4_quantize: cols must be a multiple of 16")
    return codes, scales


def nvfp4_quantize46(x, s_t):
    """NVFP4 with 4/6 block scaling: per block the rounded-up E4M3 candidate
    mapping the block max to 6 or to 4, whichever quantizes the block with the
    smaller squared error (ties: 6).  Returns (codes, row-major scales)."""
    a = _f32(x)
    rows, cols = a.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    rc = _load().q4o_nvfp4_quantize46(_ptr(a), rows, cols, float(np.float32(s_t)), _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("nvfp4_quantize46: cols must be a multiple of 16")
    return codes, scales


def fwht32(v) -> np.ndarray:
    a = _f32(v).copy()
    assert a.shape == (32,)
    _load().q4o_fwht32(_ptr(a))
    return a


def mx_transform(x, chan=None, hadamard: bool = True) -> np.ndarray:
    """Pre-quantization transform of every 32-block of the rows of x (no rounding to FP4)."""
    a = _f32(x)
    rows, cols = a.shape
    assert cols % 32 == 0
    c = None if chan is None else _f32(chan)
    out = np.zeros_like(a)
    lib = _load()
    for i in range(rows):
        for b in range(cols // 32):
            xb = np.ascontiguousarray(a[i, b * 32:(b + 1) * 32])
            yb = np.zeros(32, np.float32)
            cb = None if c is None else np.ascontiguousarray(c[b * 32:(b + 1) * 32])
            lib.q4o_mx_transform(_ptr(xb), None if cb is None else _ptr(cb), int(hadamard), _ptr(yb))
            out[i, b * 32:(b + 1) * 32] = yb
    return out


def mxfp4_quantize(x, chan=None, hadamard: bool = False, round_up: bool = False):
    """x [rows, cols] -> (codes [rows, cols/2], E8M0 scales [rows, cols/32])."""
    a = _f32(x)
    rows, cols = a.shape
    c = None if chan is None else _f32(chan)
    if c is not None:
        assert c.shape == (cols,)
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    rc = _load().q4o_mxfp4_quantize(_ptr(a), rows, cols, None if c is None else _ptr(c),
                                    int(hadamard), int(round_up), _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("mxfp4_quantize: cols must be a multiple of 32")
    return codes, scales


def tc_scale_bytes(rows: int, scols: int) -> int:
    return int(_load().q4o_tc_scale_bytes(rows, scols))


def tc_scale_offset(r: int, c: int, scols: int) -> int:
    return int(_load().q4o_tc_scale_offset(r, c, scols))


def scales_to_tc(rowmajor) -> np.ndarray:
    s = np.ascontiguousarray(rowmajor, dtype=np.uint8)
    rows, scols = s.shape
    out = np.zeros(tc_scale_bytes(rows, scols), np.uint8)
    _load().q4o_scales_to_tc(_ptr(s), rows, scols, _ptr(out))
    return out


def scales_from_tc(tc, rows: int, scols: int) -> np.ndarray:
    t = np.ascontiguousarray(tc, dtype=np.uint8)
    out = np.zeros((rows, scols), np.uint8)
    _load().q4o_scales_from_tc(_ptr(t), rows, scols, _ptr(out))
    return out


def dequantize(fmt: int, codes, scales, s_t, rows: int, cols: int) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), np.float64)
    rc = _load().q4o_dequantize(fmt, _ptr(c), _ptr(s), float(np.float32(s_t)),
                                rows, cols, _ptr(out))
    if rc != 0:
        raise ValueError("dequantize: bad shape")
    return out


def sigma_delta_step(fmt: int, w, scales, s_t, r: np.ndarray) -> np.ndarray:
    """One loop visit; updates the float32 residue ``r`` in place, returns codes."""
    a = _f32(w)
    rows, cols = a.shape
    assert r.dtype == np.float32 and r.shape == a.shape and r.flags["C_CONTIGUOUS"]
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    codes = np.zeros((rows, cols // 2), np.uint8)
    rc = _load().q4o_sigma_delta_step(fmt, _ptr(a), rows, cols, _ptr(s),
                                      float(np.float32(s_t)), _ptr(r), _ptr(codes))
    if rc != 0:
        raise ValueError("sigma_delta_step: bad shape")
    return codes


def philox4x32_10(ctr, key) -> np.ndarray:
    """The Philox4x32-10 block function: 4 counter words, 2 key words -> 4 words."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, np.uint32)
    _load().q4o_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sr_requant(fmt: int, w, scales, s_t, seed: int, visit: int) -> np.ndarray:
    """Stochastic-rounding requant of W at one loop visit with fixed (row-major)
    block scales; returns the codes [rows, cols/2]."""
    a = _f32(w)
    rows, cols = a.shape
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    codes = np.zeros((rows, cols // 2), np.uint8)
    rc = _load().q4o_sr_requant(fmt, _ptr(a), rows, cols, _ptr(s), float(np.float32(s_t)), int(seed), int(visit),
                                _ptr(codes))
    if rc != 0:
        raise ValueError("sr_requant: bad shape")
    return codes


def sigma_delta_codebanks(fmt: int, w, scales, s_t, visits: int):
    """The Sigma-Delta chain of `visits` steps from r_0 = 0 ("Looped Transformer
    quantization", sec. 2.3 / sec. 4: the tail restarts a chain and stores its
    codes as codebanks): `visits` applications of sigma_delta_step.  Returns
    (banks [visits, rows, cols/2], r_visits)."""
    a = _f32(w)
    r = np.zeros(a.shape, np.float32)
    banks = np.stack([sigma_delta_step(fmt, a, scales, s_t, r) for _ in range(visits)])
    return banks, r


def gemm(fmt: int, a_codes, a_scales, a_st, b_codes, b_scales, b_st, M, N, K, rows=None):
    """Y = alpha * dec(A) dec(B)^T in binary64; optionally only the listed rows."""
    ac = np.ascontiguousarray(a_codes, dtype=np.uint8)
    asc = np.ascontiguousarray(a_scales, dtype=np.uint8)
    bc = np.ascontiguousarray(b_codes, dtype=np.uint8)
    bsc = np.ascontiguousarray(b_scales, dtype=np.uint8)
    if rows is None:
        idx, n_rows = None, M
    else:
        idx = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = idx.size
    y = np.zeros((n_rows, N), np.float64)
    rc = _load().q4o_gemm(fmt, M, N, K, _ptr(ac), _ptr(asc), float(np.float32(a_st)),
                          _ptr(bc), _ptr(bsc), float(np.float32(b_st)),
                          None if idx is None else _ptr(idx), n_rows, _ptr(y))
    if rc != 0:
        raise ValueError("gemm: bad shape")
    return y


def gemm_w4a16(fmt: int, x, b_codes, b_scales, b_st, M, N, K, rows=None):
    """Y = alpha * X dec(W)^T in binary64 with X given as float32 (bf16 values);
    optionally only the listed rows."""
    xa = _f32(x)
    bc = np.ascontiguousarray(b_codes, dtype=np.uint8)
    bsc = np.ascontiguousarray(b_scales, dtype=np.uint8)
    if rows is None:
        idx, n_rows = None, M
    else:
        idx = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = idx.size
    y = np.zeros((n_rows, N), np.float64)
    rc = _load().q4o_gemm_w4a16(fmt, M, N, K, _ptr(xa), _ptr(bc), _ptr(bsc), float(np.float32(b_st)),
                                None if idx is None else _ptr(idx), n_rows, _ptr(y))
    if rc != 0:
        raise ValueError("gemm_w4a16: bad shape")
    return y


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """Packed bytes [rows, cols/2] -> one code per entry [rows, cols] (low nibble first)."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 0x0F
    out[..., 1::2] = c >> 4
    return out
