"""GPU parity of the block-scaled FP4 GEMM (tcgen05) against the binary64 oracle
on the same decoded operands, through the C-ABI library.

Operands are quantized on both sides from the same synthetic inputs (the
quantizers agree bit for bit, checked here again); the oracle GEMM only ever
sees oracle-made codes and scales."""
import numpy as np
import pytest
import torch

import oracle
import synth
import mxfp4_w4a4_block_b200 as q4
from gpu_util import DEV, GEMM_BF16_TOL, GEMM_F32_TOL, dev, gscale_dev, host, rel_fro

pytestmark = pytest.mark.gpu


class Operand:
    """One GEMM operand quantized on the GPU and by the oracle."""

    def __init__(self, fmt, x32, x_t=None, chan=None, had=False, denom=2688.0):
        self.fmt = fmt
        self.rows, self.cols = x32.shape
        x_t = dev(x32) if x_t is None else x_t
        if fmt == q4.NVFP4:
            self.s_t = oracle.tensor_scale(oracle.amax(x32), denom)
            self.g_t = gscale_dev(self.s_t)
            self.codes, self.scales = q4.q4_quantize(fmt, x_t, gscale=self.g_t, flags=q4.LAYOUT_TC)
            self.o_codes, self.o_scales = oracle.nvfp4_quantize(x32, self.s_t)
        else:
            self.s_t, self.g_t = np.float32(0), None
            flags = q4.LAYOUT_TC | (q4.HADAMARD32 if had else 0)
            self.codes, self.scales = q4.q4_quantize(fmt, x_t, chan=None if chan is None else dev(chan),
                                                     flags=flags)
            self.o_codes, self.o_scales = oracle.mxfp4_quantize(x32, chan, hadamard=had)
        assert np.array_equal(host(self.codes), self.o_codes)

    def rows_subset(self, idx):
        return np.ascontiguousarray(self.o_codes[idx]), np.ascontiguousarray(self.o_scales[idx])


def run_gemm(A: Operand, B: Operand, out_dtype):
    M, K = A.rows, A.cols
    N = B.rows
    return q4.q4_gemm(A.fmt, M, N, K, A.codes, A.scales, A.g_t, B.codes, B.scales, B.g_t, out_dtype=out_dtype)


def oracle_gemm(A: Operand, B: Operand, rows=None, cols=None):
    M, K = A.rows, A.cols
    if cols is None:
        bc, bs, N = B.o_codes, B.o_scales, B.rows
    else:
        bc, bs = B.rows_subset(cols)
        N = len(cols)
    return oracle.gemm(A.fmt, A.o_codes, A.o_scales, A.s_t, bc, bs, B.s_t, M, N, K, rows=rows)


def check(y: torch.Tensor, ref: np.ndarray, out_dtype):
    got = host(y.float())
    if out_dtype == torch.float32:
        assert rel_fro(got, ref) <= GEMM_F32_TOL
    else:
        assert rel_fro(got, ref) <= GEMM_BF16_TOL
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mnk", [(128, 256, 256), (64, 512, 512), (200, 328, 320), (384, 768, 1024),
                                 (1, 8, 64), (130, 264, 576)])
def test_gemm_parity_small(fmt, out_dtype, mnk):
    M, N, K = mnk
    x = synth.small_like("heavy", M + K, M, K)
    w = synth.small_like("weight", N + K, N, K)
    A, B = Operand(fmt, x), Operand(fmt, w)
    y = run_gemm(A, B, out_dtype)
    check(y, oracle_gemm(A, B), out_dtype)


def test_gemm_tiny_linear_config():
    """X 64x512 and W 512x512 fp32 (1% x50 outliers), s_t = amax/(6*448), BF16 out."""
    d = synth.tiny()
    A, B = Operand(q4.NVFP4, d["x"]), Operand(q4.NVFP4, d["w"])
    for od in (torch.float32, torch.bfloat16):
        check(run_gemm(A, B, od), oracle_gemm(A, B), od)


def test_gemm_closed_form_integer_case():
    """All scales 1 and every element 1.0 x 0.5: every output is K/2 exactly."""
    M, N, K = 130, 264, 512
    a = np.ones((M, K), np.float32)
    b = np.full((N, K), 0.5, np.float32)
    A = Operand(q4.MXFP4, a)
    B = Operand(q4.MXFP4, b)
    y = host(run_gemm(A, B, torch.float32))
    assert np.all(y == K * 0.5)


@pytest.mark.parametrize("M,K", [(1, 1088), (16, 1088), (33, 1216), (64, 1152), (65, 1088), (128, 1088), (5, 192)])
def test_fused_activation_quant_decode_small(M, K):
    """a_kind = A_BF16 for small M: the GEMM launch quantizes the bf16
    activations itself (M <= 16 and K of at least one 256-element k-block;
    larger M, or K = 192, quantizes once into the workspace).  K leaves partial
    last k-blocks of 64, 192 and 128 elements; N a partial tile."""
    N = 392
    x = synth.to_bf16(synth.small_like("heavy", M, M, K))
    x32 = synth.bf16_to_f32(x)
    w = synth.small_like("weight", 9, N, K)
    A = Operand(q4.NVFP4, x32, x_t=dev(x))
    B = Operand(q4.NVFP4, w)
    for od in (torch.float32, torch.bfloat16):
        y = q4.q4_gemm(q4.NVFP4, M, N, K, dev(x), None, A.g_t, B.codes, B.scales, B.g_t, out_dtype=od,
                       a_kind=q4.A_BF16)
        check(y, oracle_gemm(A, B), od)


@pytest.mark.parametrize("M,K,many_tiles", [(3, 320, True), (16, 8256, False), (16, 16384, False),
                                             (16, 20480, False)])
def test_fused_decode_more_tiles_than_sms_and_long_k(M, K, many_tiles):
    """Fused decode with more 128-row weight tiles than SMs (CTAs take a second
    tile and reuse their resident quantized activations for it), with 33 and 64
    k-blocks (K = 16384: the resident activations leave room for 3 weight stages),
    and K = 20480, past what fits, which takes the quantize-once workspace path;
    called twice with new activations on the second call."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    N = (sms + 4) * 128 + 64 if many_tiles else 392
    w = synth.small_like("weight", 6, N, K)
    B = Operand(q4.NVFP4, w)
    for seed in (5, 7):
        x = synth.to_bf16(synth.small_like("heavy", seed, M, K))
        A = Operand(q4.NVFP4, synth.bf16_to_f32(x), x_t=dev(x))
        y = q4.q4_gemm(q4.NVFP4, M, N, K, dev(x), None, A.g_t, B.codes, B.scales, B.g_t,
                       out_dtype=torch.float32, a_kind=q4.A_BF16)
        check(y, oracle_gemm(A, B), torch.float32)


def test_fused_activation_quant_prefill_path():
    """a_kind = A_BF16 with M above the fused limit: quantize-once into the workspace."""
    M, N, K = 300, 264, 640
    x = synth.to_bf16(synth.small_like("heavy", 1, M, K))
    x32 = synth.bf16_to_f32(x)
    w = synth.small_like("weight", 2, N, K)
    A = Operand(q4.NVFP4, x32, x_t=dev(x))
    B = Operand(q4.NVFP4, w)
    assert q4.q4_gemm_workspace_size(q4.NVFP4, M, N, K, q4.A_BF16) > 0
    y = q4.q4_gemm(q4.NVFP4, M, N, K, dev(x), None, A.g_t, B.codes, B.scales, B.g_t,
                   out_dtype=torch.float32, a_kind=q4.A_BF16)
    check(y, oracle_gemm(A, B), torch.float32)


def test_decode_config_full_size_sampled_columns():
    """Decode shape 16 x 17408 x 5120 with the fused activation quantizer; the
    oracle computes 1024 sampled output columns (all 16 rows)."""
    d = synth.decode()
    x32 = synth.bf16_to_f32(d["x"])
    A = Operand(q4.NVFP4, x32, x_t=dev(d["x"]))
    B = Operand(q4.NVFP4, d["w"])
    M, N, K = 16, 17408, 5120
    y = q4.q4_gemm(q4.NVFP4, M, N, K, dev(d["x"]), None, A.g_t, B.codes, B.scales, B.g_t,
                   out_dtype=torch.float32, a_kind=q4.A_BF16)
    cols = np.sort(np.random.default_rng(0).choice(N, 1024, replace=False))
    ref = oracle_gemm(A, B, cols=cols)
    check_sub = host(y)[:, cols]
    assert rel_fro(check_sub, ref) <= GEMM_F32_TOL


@pytest.mark.parametrize("n", [5120, 17408])
def test_prefill_config_full_size_sampled(n):
    """Prefill 8192 x n x 5120 (quantized A), the launch the benchmark times;
    oracle on 2 rows per 128-row tile and 1024 sampled columns.  FP32 output is
    held to the relative Frobenius bar 1e-4; BF16 output is compared with the
    oracle rounded to bf16, which it matches except where the FP32 sum and the
    binary64 sum fall either side of a bf16 rounding boundary."""
    d = synth.prefill(n_list=(n,))
    x32 = synth.bf16_to_f32(d["x"])
    A = Operand(q4.NVFP4, x32, x_t=dev(d["x"]))
    B = Operand(q4.NVFP4, d["w"][0])
    rng = np.random.default_rng(n)
    rows = np.array([t * 128 + r for t in range(64) for r in sorted(rng.choice(128, 2, replace=False))])
    cols = np.sort(rng.choice(n, 1024, replace=False))
    ref = oracle_gemm(A, B, rows=rows, cols=cols)
    y32 = run_gemm(A, B, torch.float32)
    assert rel_fro(host(y32)[np.ix_(rows, cols)], ref) <= GEMM_F32_TOL
    y16 = run_gemm(A, B, torch.bfloat16)
    got16 = host(y16.float())[np.ix_(rows, cols)]
    ref16 = torch.from_numpy(ref).to(torch.bfloat16).float().numpy()
    assert rel_fro(got16, ref16) <= GEMM_F32_TOL
    # the two outputs of the same launch shape: bf16 is the fp32 result rounded
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_mxfp4_config_full_size_sampled():
    """MXFP4 4096 x 14336 x 4096 with t and Hadamard-32 on both operands."""
    d = synth.mxfp4()
    x32 = synth.bf16_to_f32(d["x"])
    A = Operand(q4.MXFP4, x32, x_t=dev(d["x"]), chan=d["t"], had=True)
    B = Operand(q4.MXFP4, d["w"], chan=d["inv_t"], had=True)
    y = run_gemm(A, B, torch.float32)
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(4096, 64, replace=False))
    cols = np.sort(rng.choice(14336, 1024, replace=False))
    ref = oracle_gemm(A, B, rows=rows, cols=cols)
    got = host(y)[np.ix_(rows, cols)]
    assert rel_fro(got, ref) <= GEMM_F32_TOL


def test_gemm_k_zero_and_empty():
    B = Operand(q4.NVFP4, synth.small_like("weight", 1, 64, 64))
    y = torch.full((4, 64), 7.0, device=DEV)
    a = torch.zeros((4, 32), dtype=torch.uint8, device=DEV)
    q4.q4_gemm(q4.NVFP4, 4, 64, 0, a, B.scales, B.g_t, B.codes, B.scales, B.g_t, out_dtype=torch.float32, y=y)
    assert float(y.abs().max()) == 0.0
    q4.q4_gemm(q4.NVFP4, 0, 64, 64, a, B.scales, B.g_t, B.codes, B.scales, B.g_t, out_dtype=torch.float32)
    assert q4.q4_get_device_error() == 0


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mnk", [(128, 256, 64), (200, 392, 320), (300, 136, 1088), (64, 512, 192)])
def test_w4a16_gemm_parity(fmt, out_dtype, mnk):
    """a_kind = A_BF16_W4A16: bf16 activations times the weight dequantized to
    bf16 on the fly; ragged M, partial weight tiles and bands, odd k-stage counts."""
    M, N, K = mnk
    x = synth.to_bf16(synth.small_like("heavy", M + K, M, K))
    x32 = synth.bf16_to_f32(x)
    B = Operand(fmt, synth.small_like("weight", N + 7, N, K), denom=1536.0)
    y = q4.q4_gemm(fmt, M, N, K, dev(x), None, None, B.codes, B.scales, B.g_t, out_dtype=out_dtype,
                   a_kind=q4.A_BF16_W4A16)
    ref = oracle.gemm_w4a16(fmt, x32, B.o_codes, B.o_scales, B.s_t, M, N, K)
    check(y, ref, out_dtype)


def test_w4a16_looped_core_full_size_sampled_rows():
    """Looped-core shape: X 4096 x 1024 bf16 times a 4096 x 1024 weight whose codes
    come from three Sigma-Delta visits (RU scales, s_t = max|W| / 1536); the
    oracle follows 96 sampled rows of Y with its own Sigma-Delta codes."""
    d = synth.looped()
    w = d["w"][-1]
    N, K = w.shape
    M = d["x"].shape[0]
    x32 = synth.bf16_to_f32(d["x"])
    s_t = oracle.tensor_scale(oracle.amax(w), 1536.0)
    g_t = gscale_dev(s_t)
    _, g_sc = q4.q4_quantize(q4.NVFP4, dev(w), gscale=g_t, flags=q4.SCALE_RU | q4.LAYOUT_TC)
    _, o_sc = oracle.nvfp4_quantize(w, s_t, round_up=True)
    r_gpu = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    r_orc = np.zeros((N, K), np.float32)
    w_d = dev(w)
    for _ in range(3):
        g_codes = q4.q4_sigma_delta_step(q4.NVFP4, w_d, g_sc, r_gpu, gscale=g_t)
        o_codes = oracle.sigma_delta_step(q4.NVFP4, w, o_sc, s_t, r_orc)
    y = q4.q4_gemm(q4.NVFP4, M, N, K, dev(d["x"]), None, None, g_codes, g_sc, g_t, out_dtype=torch.float32,
                   a_kind=q4.A_BF16_W4A16)
    rows = np.sort(np.random.default_rng(1).choice(M, 96, replace=False))
    ref = oracle.gemm_w4a16(q4.NVFP4, x32, o_codes, o_sc, s_t, M, N, K, rows=rows)
    assert rel_fro(host(y)[rows], ref) <= GEMM_F32_TOL


def test_w4a16_repeatable_full_size():
    """Eight launches of the looped-core W4A16 GEMM (4096 x 4096 x 1024) give the
    same Y bit for bit (the accumulation order is fixed), and the first agrees with
    the oracle on sampled rows: a converter reading a weight stage that is already
    being refilled would show up as run-to-run differences."""
    d = synth.looped()
    w = d["w"][-1]
    N, K = w.shape
    M = d["x"].shape[0]
    B = Operand(q4.NVFP4, w, denom=1536.0)
    x = dev(d["x"])
    ys = [host(q4.q4_gemm(q4.NVFP4, M, N, K, x, None, None, B.codes, B.scales, B.g_t, out_dtype=torch.float32,
                          a_kind=q4.A_BF16_W4A16)) for _ in range(8)]
    for k in range(1, 8):
        assert np.array_equal(ys[k].view(np.uint32), ys[0].view(np.uint32)), f"launch {k} differs"
    rows = np.sort(np.random.default_rng(2).choice(M, 64, replace=False))
    ref = oracle.gemm_w4a16(q4.NVFP4, synth.bf16_to_f32(d["x"]), B.o_codes, B.o_scales, B.s_t, M, N, K, rows=rows)
    assert rel_fro(ys[0][rows], ref) <= GEMM_F32_TOL


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_shared_a_equals_separate_gemms(fmt, out_dtype):
    """q4_gemm_shared_a: every Y_w is bit for bit the single-weight q4_gemm
    (same tiles, same arithmetic), with ragged M and N, a skipped N = 0 entry,
    and the first weight also checked against the oracle."""
    M, K = 300, 640
    A = Operand(fmt, synth.small_like("heavy", 41, M, K))
    Bs = [Operand(fmt, synth.small_like("weight", 50 + i, n, K)) for i, n in enumerate((264, 392, 136))]
    ws = [(B.codes, B.scales, B.g_t, B.rows) for B in Bs]
    ws.insert(1, (Bs[0].codes, Bs[0].scales, Bs[0].g_t, 0))
    ys = q4.q4_gemm_shared_a(fmt, M, K, A.codes, A.scales, A.g_t, ws, out_dtype=out_dtype)
    view = torch.int16 if out_dtype == torch.bfloat16 else torch.int32
    for y, B in zip([ys[0]] + ys[2:], Bs):
        ref = run_gemm(A, B, out_dtype)
        assert torch.equal(y.view(view), ref.view(view))
    check(ys[0], oracle_gemm(A, Bs[0]), out_dtype)


def test_shared_a_prefill_pair_bitwise():
    """The benchmark's step: the prefill activation (8192 x 5120) times both
    prefill weights (N = 5120 and 17408) in one launch equals the two q4_gemm
    calls bit for bit (each of those is held to the oracle above)."""
    d = synth.prefill()
    x32 = synth.bf16_to_f32(d["x"])
    A = Operand(q4.NVFP4, x32, x_t=dev(d["x"]))
    Bs = [Operand(q4.NVFP4, w) for w in d["w"]]
    ys = q4.q4_gemm_shared_a(q4.NVFP4, 8192, 5120, A.codes, A.scales, A.g_t,
                             [(B.codes, B.scales, B.g_t, B.rows) for B in Bs])
    for y, B in zip(ys, Bs):
        assert torch.equal(y.view(torch.int16), run_gemm(A, B, torch.bfloat16).view(torch.int16))
    assert q4.q4_get_device_error() == 0
