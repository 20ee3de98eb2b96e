"""mxfp4_w4a4_block_b200 -- 4-bit block-scaled quantization and the W4A4 GEMM
on B200 (sm_100a).

This module is a thin ctypes binding of the C-ABI library ``libq4.so``
(declared in ``include/q4.h``): it marshals torch tensors (device memory and
the current CUDA stream) into pointers and sizes and checks the returned
status.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU fallback, and importing fails loudly if the library has not
been built (``python -m mxfp4_w4a4_block_b200.build``).

Function names mirror the C entry points: q4_amax, q4_quantize,
q4_dequantize, q4_sigma_delta_step, q4_sigma_delta_codebanks, q4_sr_requant,
q4_sigma_delta_gemm, q4_gemm,
q4_gemm_workspace_size, q4_get_device_error, q4_scale_bytes (tail_bank is a
pure indexing helper of the reverse-order codebank schedule).
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

NVFP4 = 0
MXFP4 = 1
F32 = 0
BF16 = 1

SCALE_RU = 1
LAYOUT_TC = 2
HADAMARD32 = 4
SCALE_46 = 8
INJECT_STALL = 1 << 16

A_QUANTIZED = 0
A_BF16 = 1
A_BF16_W4A16 = 2

BLOCK = {NVFP4: 16, MXFP4: 32}

STATUS = {0: "ok", 1: "invalid argument", 2: "alignment", 3: "shape", 4: "unsupported",
          5: "CUDA error", 6: "device wait timed out", 7: "workspace"}

LIB_PATH = Path(__file__).resolve().parent / "libq4.so"

# ctypes signatures of include/q4.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "q4_version": (_I, []),
    "q4_status_string": (ctypes.c_char_p, [_I]),
    "q4_last_error": (ctypes.c_char_p, []),
    "q4_scale_bytes": (_SZ, [_I, _I64, _I64, _I]),
    "q4_amax": (_I, [_I, _P, _I64, _F, _P, _P]),
    "q4_quantize": (_I, [_I, _I, _I, _P, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P]),
    "q4_dequantize": (_I, [_I, _I, _P, _P, _P, _I64, _I64, _I, _I, _P, _P]),
    "q4_sigma_delta_step": (_I, [_I, _I, _P, _I64, _I64, _P, _P, _P, _P, _I, _P]),
    "q4_sigma_delta_codebanks": (_I, [_I, _I, _P, _I64, _I64, _P, _P, _I, _P, _P, _I, _P]),
    "q4_sigma_delta_gemm": (_I, [_I, _I, _I64, _I64, _I64, _P, _P, _P, _P, _P, _I, _P, _I, _P]),
    "q4_sr_requant": (_I, [_I, _I, _P, _I64, _I64, _P, _P, ctypes.c_uint64, ctypes.c_uint32, _P, _I, _P]),
    "q4_gemm": (_I, [_I, _I, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "q4_gemm_workspace_size": (_SZ, [_I, _I64, _I64, _I64, _I]),
    "q4_get_device_error": (_I, [_P]),
    "q4_gemm_a_bf16_noalloc": (_I, [_I64, _I64, _I64, _P, _P, _P, _P, _P, _I, _P, _P]),
    "q4_set_wait_limit": (_I, [_I64]),
    "q4_amax_quantize": (_I, [_I, _P, _I64, _I64, _I64, ctypes.c_float, _P, _P, _P, _I, _P]),
    "q4_gemm_shared_a": (_I, [_I, _I, _I64, _I64, _P, _P, _P, _P, _I, _I, _P]),
    "q4_quantize_grouped": (_I, [_I, _I, _I, _P, _I, _I, _P]),
    "q4_sigma_delta_step_grouped": (_I, [_I, _I, _P, _I, _I, _P]),
    "q4_sr_requant_grouped": (_I, [_I, _I, _P, _I, ctypes.c_uint64, ctypes.c_uint32, _I, _P]),
    "q4_sigma_delta_codebanks_grouped": (_I, [_I, _I, _P, _I, _I, _I, _P]),
    "q4_sigma_delta_gemm_grouped": (_I, [_I, _I, _I64, _I64, _P, _I, _I, _I, _P]),
}

MAX_GROUP = 32


class Q4SdGemmEntry(ctypes.Structure):
    """struct q4_sd_gemm_entry of include/q4.h."""
    _fields_ = [("x", _P), ("w", _P), ("scales", _P), ("d_gscale", _P), ("residue", _P), ("y", _P),
                ("N", _I64)]


class Q4GemmWeight(ctypes.Structure):
    """struct q4_gemm_weight of include/q4.h (one weight of q4_gemm_shared_a)."""
    _fields_ = [("b_codes", _P), ("b_scales", _P), ("d_b_gscale", _P), ("y", _P), ("N", _I64)]


class Q4Matrix(ctypes.Structure):
    """struct q4_matrix of include/q4.h (one entry of a grouped call)."""
    _fields_ = [("w", _P), ("rows", _I64), ("cols", _I64), ("scales", _P), ("d_gscale", _P),
                ("residue", _P), ("codes", _P)]

_lib = None


class Q4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = STATUS.get(status, str(status))
        if status == 5 and _lib is not None:
            msg += ": " + _lib.q4_last_error().decode()
        super().__init__(f"{fn} failed: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it is missing (there is no fallback)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mxfp4_w4a4_block_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Q4Error(fn, status)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ sizes
def q4_scale_bytes(fmt: int, rows: int, cols: int, flags: int = LAYOUT_TC) -> int:
    return int(lib().q4_scale_bytes(fmt, rows, cols, flags))


def q4_gemm_workspace_size(fmt: int, M: int, N: int, K: int, a_kind: int) -> int:
    return int(lib().q4_gemm_workspace_size(fmt, M, N, K, a_kind))


# ------------------------------------------------------------------ ops
def q4_amax(x: torch.Tensor, denom: float, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[0] = max|x|, out[1] = out[0] / denom (device float32[2])."""
    if out is None:
        out = torch.empty(2, dtype=torch.float32, device=x.device)
    _check("q4_amax", lib().q4_amax(_dtype_code(x), _ptr(x), x.numel(), float(denom), _ptr(out),
                                    _stream(stream)))
    return out


def q4_amax_quantize(x: torch.Tensor, denom: float = 2688.0, out: torch.Tensor | None = None,
                     flags: int = LAYOUT_TC, codes: torch.Tensor | None = None,
                     scales: torch.Tensor | None = None, stream=None):
    """Tensor amax, s_t = amax / denom and NVFP4 quantize in one launch;
    returns (codes, scales, out) with out = [amax, s_t, scratch, scratch]."""
    rows, cols = x.shape
    ld = x.stride(0) if x.stride(1) == 1 else cols
    if out is None:
        out = torch.empty(4, dtype=torch.float32, device=x.device)
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(q4_scale_bytes(NVFP4, rows, cols, flags), 1), dtype=torch.uint8, device=x.device)
    _check("q4_amax_quantize", lib().q4_amax_quantize(_dtype_code(x), _ptr(x), rows, cols, ld, float(denom), _ptr(out),
                                                     _ptr(codes), _ptr(scales), flags, _stream(stream)))
    return codes, scales, out


def q4_quantize(fmt: int, x: torch.Tensor, gscale: torch.Tensor | None = None,
                chan: torch.Tensor | None = None, flags: int = LAYOUT_TC,
                codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                stream=None, block: int | None = None):
    """Quantize a 2-D bf16/fp32 tensor; returns (codes, scales)."""
    rows, cols = x.shape
    ld = x.stride(0) if x.dim() == 2 and x.stride(1) == 1 else cols
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(q4_scale_bytes(fmt, rows, cols, flags), 1), dtype=torch.uint8,
                             device=x.device)
    blk = BLOCK[fmt] if block is None else block
    st = lib().q4_quantize(fmt, blk, _dtype_code(x), _ptr(x), rows, cols, ld, _ptr(gscale), _ptr(chan),
                           _ptr(codes), _ptr(scales), flags, _stream(stream))
    _check("q4_quantize", st)
    return codes, scales


def q4_dequantize(fmt: int, codes: torch.Tensor, scales: torch.Tensor, rows: int, cols: int,
                  gscale: torch.Tensor | None = None, flags: int = LAYOUT_TC,
                  out_dtype=torch.float32, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype, device=codes.device)
    st = lib().q4_dequantize(fmt, BLOCK[fmt], _ptr(codes), _ptr(scales), _ptr(gscale), rows, cols, flags,
                             _dtype_code(out), _ptr(out), _stream(stream))
    _check("q4_dequantize", st)
    return out


def q4_sigma_delta_step(fmt: int, w: torch.Tensor, scales: torch.Tensor, residue: torch.Tensor,
                        gscale: torch.Tensor | None = None, flags: int = LAYOUT_TC,
                        codes: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One loop visit: updates `residue` in place and returns the visit's codes."""
    rows, cols = w.shape
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    st = lib().q4_sigma_delta_step(fmt, BLOCK[fmt], _ptr(w), rows, cols, _ptr(scales), _ptr(gscale),
                                   _ptr(residue), _ptr(codes), flags, _stream(stream))
    _check("q4_sigma_delta_step", st)
    return codes


def q4_sigma_delta_codebanks(fmt: int, w: torch.Tensor, scales: torch.Tensor, visits: int,
                             gscale: torch.Tensor | None = None, flags: int = LAYOUT_TC,
                             codes: torch.Tensor | None = None, residue_out: torch.Tensor | None = None,
                             stream=None) -> torch.Tensor:
    """The Sigma-Delta chain of `visits` steps from a zero residue in one pass;
    returns the codebanks [visits, rows, cols/2] (bank k = chain step k + 1)."""
    rows, cols = w.shape
    if codes is None:
        codes = torch.empty((visits, rows, cols // 2), dtype=torch.uint8, device=w.device)
    st = lib().q4_sigma_delta_codebanks(fmt, BLOCK[fmt], _ptr(w), rows, cols, _ptr(scales), _ptr(gscale), visits,
                                        _ptr(codes), _ptr(residue_out), flags, _stream(stream))
    _check("q4_sigma_delta_codebanks", st)
    return codes


def q4_sr_requant(fmt: int, w: torch.Tensor, scales: torch.Tensor, seed: int, visit: int,
                  gscale: torch.Tensor | None = None, flags: int = LAYOUT_TC, codes: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """Stochastic-rounding requant of w at one loop visit; returns the codes."""
    rows, cols = w.shape
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    st = lib().q4_sr_requant(fmt, BLOCK[fmt], _ptr(w), rows, cols, _ptr(scales), _ptr(gscale), int(seed), int(visit),
                             _ptr(codes), flags, _stream(stream))
    _check("q4_sr_requant", st)
    return codes


# ------------------------------------------------------------------ grouped calls
def _group(ws, scales=None, gscales=None, residues=None, codes=None):
    """The host array of q4_matrix entries for a grouped call."""
    n = len(ws)
    arr = (Q4Matrix * max(n, 1))()
    for i, w in enumerate(ws):
        rows, cols = w.shape
        arr[i] = Q4Matrix(_ptr(w), rows, cols, _ptr(scales[i]) if scales is not None else None,
                          _ptr(gscales[i]) if gscales is not None else None,
                          _ptr(residues[i]) if residues is not None else None,
                          _ptr(codes[i]) if codes is not None else None)
    return arr, n


def q4_quantize_grouped(fmt: int, ws, gscales=None, flags: int = LAYOUT_TC, codes=None, scales=None,
                        stream=None):
    """q4_quantize of every 2-D tensor in ws (one dtype) in one launch; returns (codes, scales) lists."""
    if codes is None:
        codes = [torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=w.device) for w in ws]
    if scales is None:
        scales = [torch.empty(max(q4_scale_bytes(fmt, w.shape[0], w.shape[1], flags), 1), dtype=torch.uint8,
                              device=w.device) for w in ws]
    arr, n = _group(ws, scales, gscales, None, codes)
    dt = _dtype_code(ws[0]) if n else F32
    st = lib().q4_quantize_grouped(fmt, BLOCK[fmt], dt, ctypes.addressof(arr), n, flags, _stream(stream))
    _check("q4_quantize_grouped", st)
    return codes, scales


def q4_sigma_delta_step_grouped(fmt: int, ws, scales, residues, gscales=None, flags: int = LAYOUT_TC,
                                codes=None, stream=None):
    """q4_sigma_delta_step on every (w, scales, residue) in one launch; returns the codes list."""
    if codes is None:
        codes = [torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=w.device) for w in ws]
    arr, n = _group(ws, scales, gscales, residues, codes)
    st = lib().q4_sigma_delta_step_grouped(fmt, BLOCK[fmt], ctypes.addressof(arr), n, flags, _stream(stream))
    _check("q4_sigma_delta_step_grouped", st)
    return codes


def q4_sr_requant_grouped(fmt: int, ws, scales, seed: int, visit: int, gscales=None, flags: int = LAYOUT_TC,
                          codes=None, stream=None):
    """q4_sr_requant on every (w, scales) in one launch; returns the codes list."""
    if codes is None:
        codes = [torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=w.device) for w in ws]
    arr, n = _group(ws, scales, gscales, None, codes)
    st = lib().q4_sr_requant_grouped(fmt, BLOCK[fmt], ctypes.addressof(arr), n, int(seed), int(visit), flags,
                                     _stream(stream))
    _check("q4_sr_requant_grouped", st)
    return codes


def q4_sigma_delta_codebanks_grouped(fmt: int, ws, scales, visits: int, gscales=None, flags: int = LAYOUT_TC,
                                     codes=None, residue_out=None, stream=None):
    """q4_sigma_delta_codebanks on every (w, scales) in one launch; returns the bank tensors
    ([visits, rows, cols/2] each)."""
    if codes is None:
        codes = [torch.empty((visits, w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=w.device)
                 for w in ws]
    arr, n = _group(ws, scales, gscales, residue_out, codes)
    st = lib().q4_sigma_delta_codebanks_grouped(fmt, BLOCK[fmt], ctypes.addressof(arr), n, int(visits), flags,
                                                _stream(stream))
    _check("q4_sigma_delta_codebanks_grouped", st)
    return codes


def q4_sigma_delta_gemm_grouped(fmt: int, xs, ws, scales, residues, gscales, out_dtype=torch.bfloat16, ys=None,
                                flags: int = LAYOUT_TC, stream=None):
    """q4_sigma_delta_gemm on every (x, w, scales, residue, gscale) in one launch; the
    entries share M and K.  Returns the list of outputs [M, N_i]."""
    n = len(ws)
    M, K = (xs[0].shape if n else (0, 0))
    if ys is None:
        ys = [torch.empty((M, w.shape[0]), dtype=out_dtype, device=w.device) for w in ws]
    arr = (Q4SdGemmEntry * max(n, 1))()
    for i in range(n):
        arr[i] = Q4SdGemmEntry(_ptr(xs[i]), _ptr(ws[i]), _ptr(scales[i]), _ptr(gscales[i]), _ptr(residues[i]),
                               _ptr(ys[i]), ws[i].shape[0])
    dt = _dtype_code(ys[0]) if n else BF16
    st = lib().q4_sigma_delta_gemm_grouped(fmt, BLOCK[fmt], M, K, ctypes.addressof(arr), n, dt, flags,
                                           _stream(stream))
    _check("q4_sigma_delta_gemm_grouped", st)
    return ys


def q4_sigma_delta_gemm(fmt: int, x: torch.Tensor, w: torch.Tensor, scales: torch.Tensor, residue: torch.Tensor,
                        gscale: torch.Tensor, out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
                        flags: int = LAYOUT_TC, stream=None) -> torch.Tensor:
    """One looped-core visit with the Sigma-Delta codes generated inside the
    GEMM: updates `residue` in place and returns Y = s_t X (q s_b)^T."""
    M, K = x.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    st = lib().q4_sigma_delta_gemm(fmt, BLOCK[fmt], M, N, K, _ptr(x), _ptr(w), _ptr(scales), _ptr(gscale),
                                   _ptr(residue), _dtype_code(y), _ptr(y), flags, _stream(stream))
    _check("q4_sigma_delta_gemm", st)
    return y


def tail_bank(banks: torch.Tensor, j: int) -> torch.Tensor:
    """The codes of tail visit j (1-based) in the reverse-order schedule: the
    K-step chain's codes are used last-first, so visit j reads bank K - j."""
    K = banks.shape[0]
    if not 1 <= j <= K:
        raise ValueError(f"tail visit {j} outside 1..{K}")
    return banks[K - j]


def q4_gemm(fmt: int, M: int, N: int, K: int, a: torch.Tensor, a_scales, a_gscale,
            b_codes: torch.Tensor, b_scales: torch.Tensor, b_gscale,
            out_dtype=torch.bfloat16, a_kind: int = A_QUANTIZED, y: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y[M, N] = alpha * dec(A) dec(B)^T on the tensor cores."""
    dev = b_codes.device
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=dev)
    ws_need = q4_gemm_workspace_size(fmt, M, N, K, a_kind)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().q4_gemm(fmt, BLOCK[fmt], M, N, K, a_kind, _ptr(a), _ptr(a_scales), _ptr(a_gscale),
                       _ptr(b_codes), _ptr(b_scales), _ptr(b_gscale), _dtype_code(y), _ptr(y),
                       _ptr(workspace), ws_bytes, _stream(stream))
    _check("q4_gemm", st)
    return y


def q4_gemm_shared_a(fmt: int, M: int, K: int, a: torch.Tensor, a_scales: torch.Tensor, a_gscale, weights,
                     out_dtype=torch.bfloat16, ys=None, stream=None):
    """Y_w = alpha_w dec(A) dec(B_w)^T for each weight (b_codes, b_scales, b_gscale, N) of
    `weights`, in one launch; returns the list of Y_w."""
    dev = a.device
    if ys is None:
        ys = [torch.empty((M, w[3]), dtype=out_dtype, device=dev) for w in weights]
    arr = (Q4GemmWeight * len(weights))()
    for i, (bc, bs, bg, n) in enumerate(weights):
        arr[i] = Q4GemmWeight(_ptr(bc), _ptr(bs), _ptr(bg), _ptr(ys[i]), n)
    st = lib().q4_gemm_shared_a(fmt, BLOCK[fmt], M, K, _ptr(a), _ptr(a_scales), _ptr(a_gscale),
                                ctypes.cast(arr, ctypes.c_void_p), len(weights), _dtype_code(ys[0]), _stream(stream))
    _check("q4_gemm_shared_a", st)
    return ys


def q4_gemm_a_bf16_noalloc(M: int, N: int, K: int, a: torch.Tensor, a_gscale, b_codes: torch.Tensor,
                           b_scales: torch.Tensor, b_gscale, out_dtype=torch.bfloat16,
                           y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """q4_gemm with bf16 activations using the library's fixed scratch array
    instead of a workspace (for callers that cannot allocate at call time).
    The call runs with the operands' device current, since the library picks
    the scratch array of the current device."""
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=b_codes.device)
    with torch.cuda.device(b_codes.device):
        st = lib().q4_gemm_a_bf16_noalloc(M, N, K, _ptr(a), _ptr(a_gscale), _ptr(b_codes), _ptr(b_scales),
                                          _ptr(b_gscale), _dtype_code(y), _ptr(y), _stream(stream))
    _check("q4_gemm_a_bf16_noalloc", st)
    return y


def q4_set_wait_limit(cycles: int = 0) -> None:
    """Bounded-wait limit of the kernels in SM clock cycles (0: the default)."""
    _check("q4_set_wait_limit", lib().q4_set_wait_limit(int(cycles)))


def q4_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(lib().q4_get_device_error(_stream(stream)))
