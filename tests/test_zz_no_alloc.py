"""q4_gemm_a_bf16_noalloc -- the GEMM variant for callers that cannot allocate
device memory at call time -- against q4_gemm (Q4_A_BF16, caller workspace)
and against the oracle.

The variant keeps the quantized activations in one fixed array inside the
library, so this file is collected last: a failure here still leaves every other
test run first.  It calls the entry point through the C ABI (ctypes on
libq4.so), twice in a row with different inputs.  Above M = 16 both entry
points run the same quantize and GEMM kernels on the same inputs, so their
outputs must agree bit for bit; at M <= 16 q4_gemm takes the fused decode
kernel (another summation order), so there both are held to the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_w4a4_block_b200 as q4
import oracle
import synth
from gpu_util import DEV, GEMM_F32_TOL, rel_fro

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024


def weight(seed, N, K):
    w32 = synth.small_like("weight", seed, N, K)
    w = torch.from_numpy(w32).to(DEV)
    g = q4.q4_amax(w, 2688.0)[1:2].clone()
    wc, ws = q4.q4_quantize(q4.NVFP4, w, gscale=g, flags=q4.LAYOUT_TC)
    return w32, wc, ws, g


def activation(seed, M, K):
    x_t = synth.to_bf16(synth.small_like("heavy", seed, M, K))
    x = x_t.to(DEV)
    return synth.bf16_to_f32(x_t), x, q4.q4_amax(x, 2688.0)[1:2].clone()


def call_noalloc(M, N, K, x, gx, wc, ws, gw, y):
    L = q4.lib()
    fn = L.q4_gemm_a_bf16_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    dt = q4.BF16 if y.dtype == torch.bfloat16 else q4.F32
    return fn(M, N, K, x.data_ptr(), gx.data_ptr(), wc.data_ptr(), ws.data_ptr(), gw.data_ptr(),
              dt, y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def oracle_rows(x32, w32, gx, gw, rows):
    """Binary64 oracle GEMM of the sampled rows on oracle-made operands."""
    s_a, s_b = np.float32(gx.item()), np.float32(gw.item())
    ac, asc = oracle.nvfp4_quantize(x32, s_a)
    bc, bsc = oracle.nvfp4_quantize(w32, s_b)
    M, K = x32.shape
    return oracle.gemm(oracle.NVFP4, ac, asc, s_a, bc, bsc, s_b, M, w32.shape[0], K, rows=rows)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_workspace_gemm_twice_in_a_row(out_dtype):
    cases = [(300, 264, 640, 11), (8192, 256, 512, 12), (17, 392, 1088, 13)]
    for M, N, K, seed in cases:
        x32, x, gx = activation(seed, M, K)
        w32, wc, ws, gw = weight(seed + 100, N, K)
        y = torch.full((M, N), float("nan"), dtype=out_dtype, device=DEV)
        assert call_noalloc(M, N, K, x, gx, wc, ws, gw, y) == 0
        ref = q4.q4_gemm(q4.NVFP4, M, N, K, x, None, gx, wc, ws, gw, out_dtype=out_dtype, a_kind=q4.A_BF16)
        torch.cuda.synchronize()
        # same kernels, same inputs: the same bits
        assert torch.equal(y.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                           ref.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32))
        if out_dtype == torch.float32 and M == 300:
            rows = np.arange(0, M, 7)
            want = oracle_rows(x32, w32, gx, gw, rows)
            assert rel_fro(y.cpu().numpy()[rows], want) <= GEMM_F32_TOL
    assert q4.q4_get_device_error() == 0


def test_noalloc_small_m_against_the_oracle():
    """M <= 16, where q4_gemm runs the fused decode kernel instead: both entry
    points against the binary64 oracle, and two calls in a row (the second with
    other inputs) through the Python binding."""
    for M, N, K, seed in [(16, 256, 512, 21), (3, 136, 1024, 22)]:
        x32, x, gx = activation(seed, M, K)
        w32, wc, ws, gw = weight(seed + 100, N, K)
        y = q4.q4_gemm_a_bf16_noalloc(M, N, K, x, gx, wc, ws, gw, out_dtype=torch.float32)
        ref = q4.q4_gemm(q4.NVFP4, M, N, K, x, None, gx, wc, ws, gw, out_dtype=torch.float32, a_kind=q4.A_BF16)
        want = oracle_rows(x32, w32, gx, gw, np.arange(M))
        torch.cuda.synchronize()
        assert rel_fro(y.cpu().numpy(), want) <= GEMM_F32_TOL
        assert rel_fro(ref.cpu().numpy(), want) <= GEMM_F32_TOL
        assert rel_fro(y.cpu().numpy(), ref.cpu().numpy()) <= GEMM_F32_TOL


def test_noalloc_k_zero_fills_and_bounds():
    w = torch.zeros(8, dtype=torch.uint8, device=DEV)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    y = torch.full((4, 16), 3.0, dtype=torch.float32, device=DEV)
    # K = 0: the empty sum, as q4_gemm gives it
    assert call_noalloc(4, 16, 0, w, g, w, w, g, y) == 0
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    # N beyond 2^31 is a shape error found on the host, before any launch
    assert call_noalloc(4, (1 << 31) + 8, 64, w, g, w, w, g, y) == 3


def test_noalloc_rejects_sizes_beyond_its_array():
    M, K, N = 16384, 5120, 256          # codes alone are 40 MiB > 32 MiB
    assert M * K // 2 > SCRATCH_BYTES
    x = torch.zeros(8, dtype=torch.bfloat16, device=DEV)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    y = torch.zeros(8, dtype=torch.float32, device=DEV)
    # rejected on the host before any launch, so the small dummy buffers are never touched
    assert call_noalloc(M, N, K, x, g, x, x, g, y) == 7
