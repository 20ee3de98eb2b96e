"""GPU parity of the Sigma-Delta step: codes and FP32 residues bit for bit
against the oracle on every loop visit, through the C-ABI library."""
import numpy as np
import pytest
import torch

import oracle
import synth
import mxfp4_w4a4_block_b200 as q4
from gpu_util import DEV, GEMM_F32_TOL, dev, gscale_dev, host, rel_fro

pytestmark = pytest.mark.gpu


def setup_scales(fmt, w32, tc=True):
    """Fixed per-block scales (RU) on both sides; returns GPU and oracle views."""
    flags_tc = q4.LAYOUT_TC if tc else 0
    if fmt == q4.NVFP4:
        s_t = oracle.tensor_scale(oracle.amax(w32), 1536.0)
        g_t = gscale_dev(s_t)
        _, g_sc = q4.q4_quantize(fmt, dev(w32), gscale=g_t, flags=q4.SCALE_RU | flags_tc)
        _, o_sc = oracle.nvfp4_quantize(w32, s_t, round_up=True)
    else:
        s_t, g_t = np.float32(0), None
        _, g_sc = q4.q4_quantize(fmt, dev(w32), flags=q4.SCALE_RU | flags_tc)
        _, o_sc = oracle.mxfp4_quantize(w32, round_up=True)
    return s_t, g_t, g_sc, o_sc


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("tc", [True, False])
@pytest.mark.parametrize("shape", [(200, 352), (512, 512), (1, 64), (70, 208), (33, 1040)])
def test_sigma_delta_visits_bit_exact(fmt, tc, shape):
    rows, cols = shape
    if fmt == q4.MXFP4 and cols % 32:
        pytest.skip("MXFP4 needs whole 32-blocks")
    w = synth.small_like("weight", rows + cols, rows, cols)
    s_t, g_t, g_sc, o_sc = setup_scales(fmt, w, tc)
    r_gpu = torch.zeros((rows, cols), dtype=torch.float32, device=DEV)
    r_orc = np.zeros((rows, cols), np.float32)
    flags = q4.LAYOUT_TC if tc else 0
    w_d = dev(w)
    for k in range(8):
        gc = q4.q4_sigma_delta_step(fmt, w_d, g_sc, r_gpu, gscale=g_t, flags=flags)
        oc = oracle.sigma_delta_step(fmt, w, o_sc, s_t, r_orc)
        assert np.array_equal(host(gc), oc), f"codes differ at visit {k + 1}"
        assert np.array_equal(host(r_gpu).view(np.uint32), r_orc.view(np.uint32)), f"residue differs at visit {k + 1}"
    assert np.abs(r_orc).max() <= 1.0 + 2 ** -20


def test_sigma_delta_first_visit_equals_rtn():
    w = synth.small_like("weight", 3, 256, 256)
    s_t, g_t, g_sc, _ = setup_scales(q4.NVFP4, w)
    rtn, _ = q4.q4_quantize(q4.NVFP4, dev(w), gscale=g_t, flags=q4.SCALE_RU | q4.LAYOUT_TC)
    r = torch.zeros_like(dev(w))
    c1 = q4.q4_sigma_delta_step(q4.NVFP4, dev(w), g_sc, r, gscale=g_t)
    assert torch.equal(c1, rtn)


def test_sigma_delta_resume_from_saved_residue():
    """Checkpoint/resume: restarting a chain from a saved residue reproduces it."""
    w = synth.small_like("weight", 4, 128, 256)
    s_t, g_t, g_sc, _ = setup_scales(q4.NVFP4, w)
    w_d = dev(w)
    r = torch.zeros_like(w_d)
    for _ in range(3):
        q4.q4_sigma_delta_step(q4.NVFP4, w_d, g_sc, r, gscale=g_t)
    saved = r.clone()
    run1 = [q4.q4_sigma_delta_step(q4.NVFP4, w_d, g_sc, r, gscale=g_t).clone() for _ in range(4)]
    r2 = saved.clone()
    run2 = [q4.q4_sigma_delta_step(q4.NVFP4, w_d, g_sc, r2, gscale=g_t).clone() for _ in range(4)]
    assert all(torch.equal(a, b) for a, b in zip(run1, run2))
    assert torch.equal(r, r2)


def test_looped_core_full_size_sampled_rows():
    """The 13 looped-core weights (41,943,040 weights), R = 32 visits on the GPU;
    the oracle follows every 61st row of each matrix (the step is elementwise,
    so sampled rows are exact) through all 32 visits."""
    d = synth.looped()
    R = 32
    for mi, w in enumerate(d["w"]):
        rows, cols = w.shape
        s_t, g_t, g_sc, _ = setup_scales(q4.NVFP4, w)
        sel = np.arange(mi % 61, rows, 61)
        ws = np.ascontiguousarray(w[sel])
        # oracle scales of the selected rows: quantize only those rows with the same s_t
        _, o_sc = oracle.nvfp4_quantize(ws, s_t, round_up=True)
        w_d = dev(w)
        r_gpu = torch.zeros_like(w_d)
        r_orc = np.zeros_like(ws)
        for k in range(R):
            gc = q4.q4_sigma_delta_step(q4.NVFP4, w_d, g_sc, r_gpu, gscale=g_t)
            oc = oracle.sigma_delta_step(q4.NVFP4, ws, o_sc, s_t, r_orc)
            if k in (0, R // 2, R - 1):
                assert np.array_equal(host(gc)[sel], oc)
        assert np.array_equal(host(r_gpu)[sel].view(np.uint32), r_orc.view(np.uint32))
        assert float(r_gpu.abs().max()) <= 1.0 + 2 ** -20


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("tc", [True, False])
@pytest.mark.parametrize("shape,K", [((200, 352), 1), ((64, 512), 5), ((33, 1024), 32)])
def test_codebanks_bit_exact(fmt, tc, shape, K):
    """The one-pass K-step chain: every bank and the final residue bit for bit
    against the oracle (K successive steps from r_0 = 0)."""
    rows, cols = shape
    w = synth.small_like("weight", rows * 3 + K, rows, cols)
    s_t, g_t, g_sc, o_sc = setup_scales(fmt, w, tc)
    flags = q4.LAYOUT_TC if tc else 0
    r_out = torch.empty((rows, cols), dtype=torch.float32, device=DEV)
    banks = q4.q4_sigma_delta_codebanks(fmt, dev(w), g_sc, K, gscale=g_t, flags=flags, residue_out=r_out)
    o_banks, o_r = oracle.sigma_delta_codebanks(fmt, w, o_sc, s_t, K)
    assert np.array_equal(host(banks), o_banks)
    assert np.array_equal(host(r_out).view(np.uint32), o_r.view(np.uint32))


def test_codebanks_match_successive_steps_and_reverse_tail():
    """On the GPU the one-pass banks equal K successive q4_sigma_delta_step
    calls, and tail visit K (the last) of the reverse schedule reads the
    round-to-nearest codes."""
    w = synth.small_like("weight", 5, 256, 768)
    s_t, g_t, g_sc, _ = setup_scales(q4.NVFP4, w)
    K = 8
    banks = q4.q4_sigma_delta_codebanks(q4.NVFP4, dev(w), g_sc, K, gscale=g_t)
    r = torch.zeros((256, 768), dtype=torch.float32, device=DEV)
    for k in range(K):
        c = q4.q4_sigma_delta_step(q4.NVFP4, dev(w), g_sc, r, gscale=g_t)
        assert torch.equal(c, banks[k])
    rtn, _ = q4.q4_quantize(q4.NVFP4, dev(w), gscale=g_t, flags=q4.SCALE_RU | q4.LAYOUT_TC)
    assert torch.equal(q4.tail_bank(banks, K), rtn)
    assert torch.equal(q4.tail_bank(banks, 1), banks[K - 1])


@pytest.mark.parametrize("M,N,K", [(1, 392, 320), (16, 1024, 1024), (5, 4096, 1024), (16, 136, 64), (12, 256, 2048)])
def test_sigma_delta_gemm_fused_producer(M, N, K):
    """Sigma-Delta fused into the GEMM's weight producer: three visits; the
    residue bit for bit against the oracle step, Y against the binary64 W4A16
    oracle on the oracle's own codes of that visit."""
    w = synth.small_like("weight", M + N + K, N, K)
    x = synth.to_bf16(synth.small_like("gauss", 3 * M + K, M, K))
    x32 = synth.bf16_to_f32(x)
    s_t, g_t, g_sc, o_sc = setup_scales(q4.NVFP4, w)
    r_gpu = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    r_orc = np.zeros((N, K), np.float32)
    w_d, x_d = dev(w), dev(x)
    for visit in range(3):
        y = q4.q4_sigma_delta_gemm(q4.NVFP4, x_d, w_d, g_sc, r_gpu, g_t, out_dtype=torch.float32)
        oc = oracle.sigma_delta_step(q4.NVFP4, w, o_sc, s_t, r_orc)
        assert np.array_equal(host(r_gpu).view(np.uint32), r_orc.view(np.uint32)), f"residue, visit {visit + 1}"
        ref = oracle.gemm_w4a16(q4.NVFP4, x32, oc, o_sc, s_t, M, N, K)
        assert rel_fro(host(y), ref) <= GEMM_F32_TOL


def test_sigma_delta_gemm_matches_unfused_path():
    """The fused visit equals q4_sigma_delta_step followed by the W4A16 q4_gemm
    (residue bit for bit, outputs to FP32 summation order)."""
    M, N, K = 16, 4096, 1024
    w = synth.looped()["w"][-1]
    x = synth.to_bf16(synth.small_like("gauss", 9, M, K))
    s_t, g_t, g_sc, _ = setup_scales(q4.NVFP4, w)
    w_d, x_d = dev(w), dev(x)
    r1 = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    r2 = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    for _ in range(2):
        y1 = q4.q4_sigma_delta_gemm(q4.NVFP4, x_d, w_d, g_sc, r1, g_t, out_dtype=torch.float32)
        c = q4.q4_sigma_delta_step(q4.NVFP4, w_d, g_sc, r2, gscale=g_t)
        y2 = q4.q4_gemm(q4.NVFP4, M, N, K, x_d, None, None, c, g_sc, g_t, out_dtype=torch.float32,
                        a_kind=q4.A_BF16_W4A16)
        assert torch.equal(r1, r2)
        assert rel_fro(host(y1), host(y2).astype(np.float64)) <= 1e-6


@pytest.mark.parametrize("M,K", [(16, 1024), (5, 320)])
def test_sigma_delta_gemm_grouped(M, K):
    """The fused step + GEMM over several weights in one launch (shared M and K,
    each weight its own activations, N ragged against the 128-row bands): three
    visits, every residue bit for bit against the oracle step and every Y against
    the W4A16 oracle on the oracle's codes of that visit."""
    Ns = [392, 1024, 136, 4096][: (4 if K == 1024 else 3)]
    E = []
    for i, N in enumerate(Ns):
        w = synth.small_like("weight", 31 * i + N + K, N, K)
        x = synth.to_bf16(synth.small_like("gauss", 7 * i + M + K, M, K))
        s_t, g_t, g_sc, o_sc = setup_scales(q4.NVFP4, w)
        E.append(dict(w=w, x32=synth.bf16_to_f32(x), wd=dev(w), xd=dev(x), s_t=s_t, g_t=g_t, g_sc=g_sc, o_sc=o_sc,
                      r_gpu=torch.zeros((N, K), dtype=torch.float32, device=DEV), r_orc=np.zeros((N, K), np.float32)))
    for visit in range(3):
        ys = q4.q4_sigma_delta_gemm_grouped(q4.NVFP4, [e["xd"] for e in E], [e["wd"] for e in E],
                                            [e["g_sc"] for e in E], [e["r_gpu"] for e in E], [e["g_t"] for e in E],
                                            out_dtype=torch.float32)
        for i, (e, N) in enumerate(zip(E, Ns)):
            oc = oracle.sigma_delta_step(q4.NVFP4, e["w"], e["o_sc"], e["s_t"], e["r_orc"])
            assert np.array_equal(host(e["r_gpu"]).view(np.uint32), e["r_orc"].view(np.uint32)), \
                f"residue of entry {i}, visit {visit + 1}"
            ref = oracle.gemm_w4a16(q4.NVFP4, e["x32"], oc, e["o_sc"], e["s_t"], M, N, K)
            assert rel_fro(host(ys[i]), ref) <= GEMM_F32_TOL, f"Y of entry {i}, visit {visit + 1}"
