"""GPU parity: amax, NVFP4 / MXFP4 quantize, dequantize -- bit for bit against
the CPU oracle, through the C-ABI library."""
import numpy as np
import pytest
import torch

import oracle
import synth
import mxfp4_w4a4_block_b200 as q4
from gpu_util import DEV, dev, gscale_dev, host

pytestmark = pytest.mark.gpu


def gpu_nvfp4(x_t, s_t, flags):
    codes, scales = q4.q4_quantize(q4.NVFP4, x_t, gscale=gscale_dev(s_t), flags=flags)
    return host(codes), host(scales)


def check_nvfp4(x32: np.ndarray, x_t: torch.Tensor, s_t, ru: bool, tc: bool):
    rows, cols = x32.shape
    flags = (q4.SCALE_RU if ru else 0) | (q4.LAYOUT_TC if tc else 0)
    gc, gs = gpu_nvfp4(x_t, s_t, flags)
    oc, os_ = oracle.nvfp4_quantize(x32, s_t, round_up=ru)
    assert np.array_equal(gc, oc)
    if tc:
        assert np.array_equal(gs, oracle.scales_to_tc(os_))
    else:
        assert np.array_equal(gs.reshape(os_.shape), os_)


def test_e2m1_decisions_exhaustive_near_grid():
    """Every binary32 value in [-6, 6] with its 8 low mantissa bits clear, plus
    every neighbourhood of a rounding midpoint, through the NVFP4 kernel with
    block scale exactly 1 (each 16-block starts with 6.0 and s_t = 1)."""
    pos = np.arange(0, 0x40C00001, 256, dtype=np.uint32).view(np.float32)   # 0 .. 6
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([np.nextafter(np.repeat(mids, 1), np.float32(np.inf)),
                           np.nextafter(mids, np.float32(0)), mids])
    vals = np.concatenate([pos, -pos, near, -near, np.array([0.0, -0.0, 1e-30, -1e-30], np.float32)])
    vals = vals[np.abs(vals) <= 6.0]
    pad = (-len(vals)) % 15
    vals = np.concatenate([vals, np.zeros(pad, np.float32)]).reshape(-1, 15)
    blocks = np.concatenate([np.full((vals.shape[0], 1), 6.0, np.float32), vals], axis=1)
    nblk = blocks.shape[0]
    cols = 16 * 64
    nrows = (nblk + 63) // 64
    x = np.zeros((nrows * 64, 16), np.float32)
    x[:nblk] = blocks
    x[nblk:, 0] = 6.0
    x = x.reshape(nrows, cols)
    check_nvfp4(x, dev(x), 1.0, ru=False, tc=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("ru", [False, True])
@pytest.mark.parametrize("tc", [False, True])
@pytest.mark.parametrize("shape", [(200, 336), (128, 64), (1, 16), (257, 1040), (300, 1056), (513, 2080)])
def test_nvfp4_quantize_parity(dtype, ru, tc, shape):
    rows, cols = shape
    x = synth.small_like("heavy", rows * 7 + cols, rows, cols)
    if dtype == "bf16":
        xt = synth.to_bf16(x)
        x32 = synth.bf16_to_f32(xt)
        x_t = dev(xt)
    else:
        x32 = x
        x_t = dev(x)
    s_t = oracle.tensor_scale(oracle.amax(x32), 1536.0 if ru else 2688.0)
    check_nvfp4(x32, x_t, s_t, ru, tc)


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,cols,ld", [(130, 320, 384), (257, 96, 1000), (64, 1024, 1032)])
def test_quantize_strided_rows(fmt, dtype, rows, cols, ld):
    """Rows `ld` elements apart (a column slice of a wider tensor)."""
    full = synth.small_like("heavy", rows * 3 + ld, rows, ld)
    if dtype == "bf16":
        xt = synth.to_bf16(full)
        x32 = np.ascontiguousarray(synth.bf16_to_f32(xt)[:, :cols])
        x_t = dev(xt)[:, :cols]
    else:
        x32 = np.ascontiguousarray(full[:, :cols])
        x_t = dev(full)[:, :cols]
    assert x_t.stride(0) == ld
    if fmt == q4.NVFP4:
        s_t = oracle.tensor_scale(oracle.amax(x32), 2688.0)
        gc, gs = q4.q4_quantize(fmt, x_t, gscale=gscale_dev(s_t), flags=q4.LAYOUT_TC)
        oc, os_ = oracle.nvfp4_quantize(x32, s_t)
    else:
        gc, gs = q4.q4_quantize(fmt, x_t, flags=q4.LAYOUT_TC | q4.HADAMARD32)
        oc, os_ = oracle.mxfp4_quantize(x32, hadamard=True)
    assert np.array_equal(host(gc), oc)
    assert np.array_equal(host(gs), oracle.scales_to_tc(os_))


def test_nvfp4_degenerate_and_saturating_blocks():
    x = np.zeros((4, 64), np.float32)
    x[1, :16] = 6.35          # RN scale 1.0 -> 6.35 saturates to 6
    x[1, 16:32] = -6.35
    x[2, 0] = -1e-3           # negative values that round to zero keep the sign
    x[2, 1] = 3.0
    x[3, :] = -0.0
    check_nvfp4(x, dev(x), 1.0, ru=False, tc=True)
    # zero tensor scale: every block degenerate
    check_nvfp4(x, dev(x), 0.0, ru=False, tc=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("had,chan,ru", [(False, False, False), (True, False, False),
                                         (True, True, False), (False, True, True), (True, True, True)])
@pytest.mark.parametrize("shape", [(200, 352), (128, 128), (3, 32), (390, 1312)])
def test_mxfp4_quantize_parity(dtype, had, chan, ru, shape):
    rows, cols = shape
    x = synth.small_like("outlier", rows + 3 * cols, rows, cols)
    if dtype == "bf16":
        xt = synth.to_bf16(x)
        x32 = synth.bf16_to_f32(xt)
        x_t = dev(xt)
    else:
        x32 = x
        x_t = dev(x)
    c = np.exp(np.random.default_rng(cols).uniform(-2, 2, cols)).astype(np.float32) if chan else None
    flags = q4.LAYOUT_TC | (q4.HADAMARD32 if had else 0) | (q4.SCALE_RU if ru else 0)
    gc, gs = q4.q4_quantize(q4.MXFP4, x_t, chan=None if c is None else dev(c), flags=flags)
    oc, os_ = oracle.mxfp4_quantize(x32, c, hadamard=had, round_up=ru)
    assert np.array_equal(host(gc), oc)
    assert np.array_equal(host(gs), oracle.scales_to_tc(os_))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n", [0, 1, 7, 8, 1000, 123457])
def test_amax_parity(dtype, n):
    x = synth.small_like("heavy", n + 1, 1, max(n, 1) * 1).reshape(-1)[:n] if n else np.zeros(0, np.float32)
    if dtype == "bf16":
        xt = synth.to_bf16(x)
        x32 = synth.bf16_to_f32(xt)
        x_t = dev(xt) if n else torch.zeros(8, dtype=torch.bfloat16, device=DEV)[:0]
    else:
        x32 = x
        x_t = dev(x) if n else torch.zeros(8, dtype=torch.float32, device=DEV)[:0]
    out = host(q4.q4_amax(x_t, 2688.0))
    am = oracle.amax(x32) if n else np.float32(0)
    assert out[0] == am
    assert out[1] == oracle.tensor_scale(am, 2688.0)


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("tc", [False, True])
@pytest.mark.parametrize("shape", [(130, 224), (4097, 4160)])
def test_dequantize_parity(fmt, out_dtype, tc, shape):
    """Bit for bit against the oracle; the larger ragged shape gives every thread
    of the persistent grid several blocks / unit groups."""
    rows, cols = shape
    x = synth.small_like("heavy", 5, rows, cols)
    flags = q4.LAYOUT_TC if tc else 0
    if fmt == q4.NVFP4:
        s_t = oracle.tensor_scale(oracle.amax(x), 2688.0)
        gs_t = gscale_dev(s_t)
        codes, scales = q4.q4_quantize(fmt, dev(x), gscale=gs_t, flags=flags)
        oc, os_ = oracle.nvfp4_quantize(x, s_t)
    else:
        s_t, gs_t = 0.0, None
        codes, scales = q4.q4_quantize(fmt, dev(x), flags=flags)
        oc, os_ = oracle.mxfp4_quantize(x)
    out = host(q4.q4_dequantize(fmt, codes, scales, rows, cols, gscale=gs_t, flags=flags,
                                out_dtype=out_dtype).float())
    ref = oracle.dequantize(fmt, oc, os_, s_t, rows, cols)
    ref_t = torch.from_numpy(ref).float()
    if out_dtype == torch.bfloat16:
        ref_t = ref_t.bfloat16().float()
    assert np.array_equal(out, ref_t.numpy())


def test_prefill_activation_quantize_full_size():
    """The prefill activation (8192 x 5120 bf16) quantized in full, bit for bit."""
    d = synth.prefill(n_list=())
    x32 = synth.bf16_to_f32(d["x"])
    am = host(q4.q4_amax(dev(d["x"]), 2688.0))
    assert am[0] == oracle.amax(x32)
    s_t = oracle.tensor_scale(oracle.amax(x32), 2688.0)
    assert am[1] == s_t
    gc, gs = q4.q4_quantize(q4.NVFP4, dev(d["x"]), gscale=torch.tensor(am[1:2], device=DEV), flags=q4.LAYOUT_TC)
    oc, os_ = oracle.nvfp4_quantize(x32, s_t)
    assert np.array_equal(host(gc), oc)
    assert np.array_equal(host(gs), oracle.scales_to_tc(os_))


def test_amax_quantize_prefill_full_size():
    """amax, s_t and NVFP4 quantize of the prefill activation in one launch
    (the benchmark's step): bit for bit against the oracle and equal to the two
    separate launches, on two launches in a row."""
    d = synth.prefill(n_list=())
    x32 = synth.bf16_to_f32(d["x"])
    x = dev(d["x"])
    amax = oracle.amax(x32)
    s_t = oracle.tensor_scale(amax, 2688.0)
    oc, os_ = oracle.nvfp4_quantize(x32, s_t)
    for _ in range(2):
        gc, gs, out = q4.q4_amax_quantize(x, 2688.0)
        o = host(out)
        assert o[0] == amax and o[1] == s_t
        assert np.array_equal(host(gc), oc)
        assert np.array_equal(host(gs), oracle.scales_to_tc(os_))
    assert q4.q4_get_device_error() == 0


@pytest.mark.parametrize("rows,cols,ld,bf16,ru,tc", [
    (300, 400, 400, False, False, False),
    (300, 400, 416, True, True, True),
    (1, 16, 16, True, False, True),
    (4097, 160, 176, False, True, True),
    (130, 5120, 5120, True, False, False)])
def test_amax_quantize_parity(rows, cols, ld, bf16, ru, tc):
    """Ragged, strided, fp32 and bf16, RN and RU scales, both layouts."""
    full = synth.small_like("heavy", rows + cols, rows, ld)
    if bf16:
        xt = synth.to_bf16(full)
        full = synth.bf16_to_f32(xt)
        x = dev(xt)[:, :cols]
    else:
        x = dev(full)[:, :cols]
    x32 = np.ascontiguousarray(full[:, :cols])
    flags = (q4.SCALE_RU if ru else 0) | (q4.LAYOUT_TC if tc else 0)
    gc, gs, out = q4.q4_amax_quantize(x, 2688.0, flags=flags)
    amax = oracle.amax(x32)
    s_t = oracle.tensor_scale(amax, 2688.0)
    o = host(out)
    assert o[0] == amax and o[1] == s_t
    oc, os_ = oracle.nvfp4_quantize(x32, s_t, round_up=ru)
    assert np.array_equal(host(gc), oc)
    if tc:
        assert np.array_equal(host(gs), oracle.scales_to_tc(os_))
    else:
        assert np.array_equal(host(gs).reshape(os_.shape), os_)


def test_amax_quantize_empty():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    out = torch.full((4,), 7.0, device=DEV)
    q4.q4_amax_quantize(x, 2688.0, out=out)
    assert np.array_equal(host(out), np.zeros(4, np.float32))


def test_mxfp4_activation_quantize_full_size():
    """The MXFP4 activation (4096 x 4096 bf16) with t and Hadamard-32, bit for bit."""
    d = synth.mxfp4(n=256)
    x32 = synth.bf16_to_f32(d["x"])
    flags = q4.LAYOUT_TC | q4.HADAMARD32
    gc, gs = q4.q4_quantize(q4.MXFP4, dev(d["x"]), chan=dev(d["t"]), flags=flags)
    oc, os_ = oracle.mxfp4_quantize(x32, d["t"], hadamard=True)
    assert np.array_equal(host(gc), oc)
    assert np.array_equal(host(gs), oracle.scales_to_tc(os_))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("tc", [False, True])
@pytest.mark.parametrize("shape", [(200, 336), (128, 1024), (1, 16), (300, 1056)])
def test_nvfp4_scale46_parity(dtype, tc, shape):
    """4/6 block scaling: codes and the chosen scales bit for bit (the choice is
    a binary64 squared-error comparison on both sides)."""
    rows, cols = shape
    x = synth.small_like("weight", rows * 5 + cols, rows, cols)
    if dtype == "bf16":
        xt = synth.to_bf16(x)
        x32 = synth.bf16_to_f32(xt)
        x_t = dev(xt)
    else:
        x32 = x
        x_t = dev(x)
    s_t = oracle.tensor_scale(oracle.amax(x32), 1536.0)
    flags = q4.SCALE_46 | (q4.LAYOUT_TC if tc else 0)
    gc, gs = q4.q4_quantize(q4.NVFP4, x_t, gscale=gscale_dev(s_t), flags=flags)
    oc, os_ = oracle.nvfp4_quantize46(x32, s_t)
    assert np.array_equal(host(gc), oc)
    if tc:
        assert np.array_equal(host(gs), oracle.scales_to_tc(os_))
    else:
        assert np.array_equal(host(gs).reshape(os_.shape), os_)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_repeated_launches_full_size(dtype):
    """Ten launches of the tiled quantizer on 4097 x 4160 (ragged last row tile),
    both scale layouts, each bit for bit against the oracle: consumer warps run
    unsynchronised across tiles, so an input stage released before all of its
    shared-memory reads completed would be refilled under them (seen as a few
    wrong codes and scales in some launches)."""
    rows, cols = 4097, 4160
    x = synth.small_like("heavy", 5, rows, cols)
    if dtype == "bf16":
        xt = synth.to_bf16(x)
        x = synth.bf16_to_f32(xt)
        xd = dev(xt)
    else:
        xd = dev(x)
    s_t = oracle.tensor_scale(oracle.amax(x), 2688.0)
    oc, os_ = oracle.nvfp4_quantize(x, s_t)
    for flags, o_sc in ((0, os_.reshape(-1)), (q4.LAYOUT_TC, oracle.scales_to_tc(os_))):
        for k in range(10):
            gc, gs = q4.q4_quantize(q4.NVFP4, xd, gscale=gscale_dev(s_t), flags=flags)
            assert np.array_equal(host(gc), oc), f"codes, flags {flags}, launch {k}"
            assert np.array_equal(host(gs).reshape(-1), o_sc), f"scales, flags {flags}, launch {k}"


def test_scale46_ties_and_near_ties():
    """4/6 blocks whose two candidates tie or nearly tie (the kernels then take
    the binary64 comparison): with s_t = 1 a block of values from {0, +-12, +-24}
    with max 24 is exact under both scales (4 = 24/6 and 6 = 24/4), so both
    squared errors are 0 and the 6 candidate wins; all-zero blocks give equal
    scale bytes; blocks one ulp away from those give errors of nearly equal
    size.  Random blocks fill the rest; single and grouped launches agree with
    the oracle."""
    rng = np.random.default_rng(46)
    rows, cols = 256, 256
    x = synth.small_like("weight", 461, rows, cols)
    blocks = x.reshape(rows, cols // 16, 16)
    exact = rng.choice(np.array([0, 12, -12, 24, -24], np.float32), size=(64, cols // 16, 16))
    exact[:, :, 0] = 24.0
    blocks[:64] = exact
    blocks[64:96] = 0.0
    near = rng.choice(np.array([0, 12, -12, 24, -24], np.float32), size=(32, cols // 16, 16))
    near[:, :, 0] = 24.0
    j = rng.integers(1, 16, size=(32, cols // 16))
    sel = np.take_along_axis(near, j[..., None], axis=2)
    np.put_along_axis(near, j[..., None], np.nextafter(sel, np.float32(np.inf)), axis=2)
    blocks[96:128] = near
    x = blocks.reshape(rows, cols).astype(np.float32)
    s_t = np.float32(1.0)
    oc, os_ = oracle.nvfp4_quantize46(x, s_t)
    assert (os_[:64] == oracle.e4m3_encode(4.0)).all()       # the 6 candidate on exact ties
    gc, gs = q4.q4_quantize(q4.NVFP4, dev(x), gscale=gscale_dev(s_t), flags=q4.SCALE_46 | q4.LAYOUT_TC)
    assert np.array_equal(host(gc), oc)
    assert np.array_equal(host(gs), oracle.scales_to_tc(os_))
    gcs, gss = q4.q4_quantize_grouped(q4.NVFP4, [dev(x)], gscales=[gscale_dev(s_t)],
                                      flags=q4.SCALE_46 | q4.LAYOUT_TC)
    assert np.array_equal(host(gcs[0]), oc)
    assert np.array_equal(host(gss[0]), oracle.scales_to_tc(os_))


def test_scale46_sigma_delta_chain():
    """Sigma-Delta on 4/6 block scales (the page's block_scale_46(W) feeding the
    loop): eight visits bit for bit, residues within |r| <= 1."""
    w = synth.small_like("weight", 77, 256, 512)
    s_t = oracle.tensor_scale(oracle.amax(w), 1536.0)
    g_t = gscale_dev(s_t)
    _, g_sc = q4.q4_quantize(q4.NVFP4, dev(w), gscale=g_t, flags=q4.SCALE_46 | q4.LAYOUT_TC)
    _, o_sc = oracle.nvfp4_quantize46(w, s_t)
    r_g = torch.zeros((256, 512), dtype=torch.float32, device=DEV)
    r_o = np.zeros((256, 512), np.float32)
    for _ in range(8):
        gc = q4.q4_sigma_delta_step(q4.NVFP4, dev(w), g_sc, r_g, gscale=g_t)
        oc = oracle.sigma_delta_step(q4.NVFP4, w, o_sc, s_t, r_o)
        assert np.array_equal(host(gc), oc)
    assert np.array_equal(host(r_g).view(np.uint32), r_o.view(np.uint32))
    assert np.abs(r_o).max() <= 1.0 + 2 ** -20
