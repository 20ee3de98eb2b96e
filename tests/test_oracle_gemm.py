"""Pins for the oracle's W4A4 GEMM (binary64 triple loop over decoded operands).

Checked against numpy's binary64 matmul of independently decoded operands and
against a closed form where every decoded value is known.
"""
import numpy as np
import pytest

import synth


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_gemm_matches_numpy_matmul(orc, fmt):
    M, N, K = 24, 40, 96
    x = synth.small_like("heavy", 1, M, K)
    w = synth.small_like("weight", 2, N, K)
    if fmt == "nvfp4":
        f = orc.NVFP4
        sa = np.float32(np.abs(x).max()) / np.float32(2688)
        sb = np.float32(np.abs(w).max()) / np.float32(2688)
        ac, asc = orc.nvfp4_quantize(x, sa)
        bc, bsc = orc.nvfp4_quantize(w, sb)
    else:
        f = orc.MXFP4
        sa = sb = np.float32(0)
        ac, asc = orc.mxfp4_quantize(x)
        bc, bsc = orc.mxfp4_quantize(w)
    y = orc.gemm(f, ac, asc, sa, bc, bsc, sb, M, N, K)
    da = orc.dequantize(f, ac, asc, 1.0, M, K)
    db = orc.dequantize(f, bc, bsc, 1.0, N, K)
    alpha = float(sa) * float(sb) if fmt == "nvfp4" else 1.0
    ref = alpha * (da @ db.T)
    assert y.shape == (M, N)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-300)
    # the product approximates the unquantised one (sanity on operand order)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(y - exact) / np.linalg.norm(exact) < 0.2
    # row sampling returns the same rows
    rows = np.array([0, 5, 23])
    ys = orc.gemm(f, ac, asc, sa, bc, bsc, sb, M, N, K, rows=rows)
    assert np.array_equal(ys, y[rows])


def test_gemm_closed_form(orc):
    M, N, K = 3, 5, 64
    a_codes = np.full((M, K // 2), 0x22, np.uint8)      # every element 1.0
    b_codes = np.full((N, K // 2), 0x11, np.uint8)      # every element 0.5
    a_sc = np.full((M, K // 16), 0x38, np.uint8)        # E4M3 1.0
    b_sc = np.full((N, K // 16), 0x40, np.uint8)        # E4M3 2.0
    y = orc.gemm(orc.NVFP4, a_codes, a_sc, 0.5, b_codes, b_sc, 3.0, M, N, K)
    # sum_k 1 * (0.5 * 2) = K, times alpha = 0.5 * 3
    assert np.all(y == K * 1.5)
    # a single non-zero pair picks out one term
    b2 = np.zeros((N, K // 2), np.uint8)
    b2[2, 7] = 0x70                                     # element k = 15 of row 2 is 6.0
    y2 = orc.gemm(orc.NVFP4, a_codes, a_sc, 1.0, b2, b_sc, 1.0, M, N, K)
    assert np.all(y2[:, 2] == 12.0) and np.count_nonzero(y2) == M


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_gemm_w4a16_matches_numpy_matmul(orc, fmt):
    """W4A16 (bf16 activations x 4-bit weights): numpy binary64 matmul of the
    activations with the independently dequantized weight."""
    M, N, K = 20, 36, 128
    x = synth.bf16_to_f32(synth.to_bf16(synth.small_like("heavy", 3, M, K)))
    w = synth.small_like("weight", 4, N, K)
    if fmt == "nvfp4":
        f = orc.NVFP4
        st = np.float32(np.abs(w).max()) / np.float32(1536)
        bc, bsc = orc.nvfp4_quantize(w, st, round_up=True)
    else:
        f = orc.MXFP4
        st = np.float32(0)
        bc, bsc = orc.mxfp4_quantize(w, round_up=True)
    y = orc.gemm_w4a16(f, x, bc, bsc, st, M, N, K)
    dw = orc.dequantize(f, bc, bsc, st if fmt == "nvfp4" else 0.0, N, K)
    ref = x.astype(np.float64) @ dw.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-300)
    # activations not quantized: close to the full-precision product
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(y - exact) / np.linalg.norm(exact) < 0.15
    rows = np.array([1, 19])
    assert np.array_equal(orc.gemm_w4a16(f, x, bc, bsc, st, M, N, K, rows=rows), y[rows])


def test_gemm_w4a16_closed_form(orc):
    M, N, K = 2, 3, 32
    x = np.full((M, K), 0.25, np.float32)
    x[1, 5] = -8.0
    codes = np.full((N, K // 2), 0x33, np.uint8)        # every element 1.5
    sc = np.full((N, K // 16), 0x40, np.uint8)          # E4M3 2.0
    y = orc.gemm_w4a16(orc.NVFP4, x, codes, sc, 0.5, M, N, K)
    # row 0: K * 0.25 * 1.5 * 2 * 0.5 ; row 1 replaces one 0.25 by -8
    assert np.all(y[0] == K * 0.375)
    assert np.all(y[1] == (K - 1) * 0.375 + (-8.0) * 1.5)
