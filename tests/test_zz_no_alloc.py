"""q4_gemm_a_bf16_noalloc -- the GEMM variant for callers that cannot allocate
device memory at call time -- against q4_gemm (Q4_A_BF16, caller workspace).

The variant keeps the quantized activations in one fixed array inside the
library, so this file is collected last: a failure here still leaves every other
test run first.  It calls the entry point through the C ABI (ctypes on
libq4.so), twice in a row with different inputs, and compares each result with
q4_gemm within the GEMM tolerance the other tests use."""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_w4a4_block_b200 as q4
import synth
from gpu_util import DEV, GEMM_F32_TOL, rel_fro

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024


def weight(seed, N, K):
    w = torch.from_numpy(synth.small_like("weight", seed, N, K)).to(DEV)
    g = q4.q4_amax(w, 2688.0)[1:2].clone()
    wc, ws = q4.q4_quantize(q4.NVFP4, w, gscale=g)
    return wc, ws, g


def activation(seed, M, K):
    x = synth.to_bf16(synth.small_like("heavy", seed, M, K)).to(DEV)
    return x, q4.q4_amax(x, 2688.0)[1:2].clone()


def call_noalloc(M, N, K, x, gx, wc, ws, gw, y):
    L = q4.lib()
    fn = L.q4_gemm_a_bf16_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    return fn(M, N, K, x.data_ptr(), gx.data_ptr(), wc.data_ptr(), ws.data_ptr(), gw.data_ptr(),
              q4.F32, y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_gemm_twice_in_a_row():
    cases = [(300, 264, 640, 11), (8192, 256, 512, 12), (17, 392, 1088, 13)]
    for M, N, K, seed in cases:
        x, gx = activation(seed, M, K)
        wc, ws, gw = weight(seed + 100, N, K)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
        assert call_noalloc(M, N, K, x, gx, wc, ws, gw, y) == 0
        ref = q4.q4_gemm(q4.NVFP4, M, N, K, x, None, gx, wc, ws, gw, out_dtype=torch.float32, a_kind=q4.A_BF16)
        torch.cuda.synchronize()
        got, want = y.cpu().numpy(), ref.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_fro(got, want) <= GEMM_F32_TOL
    assert q4.q4_get_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_array():
    M, K, N = 16384, 5120, 256          # codes alone are 40 MiB > 32 MiB
    assert M * K // 2 > SCRATCH_BYTES
    x = torch.zeros(8, dtype=torch.bfloat16, device=DEV)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    y = torch.zeros(8, dtype=torch.float32, device=DEV)
    # rejected on the host before any launch, so the small dummy buffers are never touched
    assert call_noalloc(M, N, K, x, g, x, x, g, y) == 7
