"""GPU parity of the grouped calls (one launch over a list of matrices): every
entry bit for bit against the oracle, with ragged shapes (rows not a multiple
of 128, block columns not a multiple of 4), a 1-row matrix and an empty entry
in the list, and the 13 looped-core weights at full size."""
import numpy as np
import pytest
import torch

import oracle
import synth
import mxfp4_w4a4_block_b200 as q4
from gpu_util import DEV, dev, gscale_dev, host
from test_gpu_sigma_delta import setup_scales

pytestmark = pytest.mark.gpu

SHAPES = [(200, 352), (1, 64), (130, 1040), (0, 64), (33, 1024), (256, 512)]


def weights(fmt, seed):
    out = []
    for i, (r, c) in enumerate(SHAPES):
        if fmt == q4.MXFP4 and c % 32:
            continue
        out.append(synth.small_like("weight", seed + 7 * i, r, c) if r else np.zeros((0, c), np.float32))
    return out


def oracle_scales(fmt, o_sc, tc):
    return oracle.scales_to_tc(o_sc) if tc else o_sc.reshape(-1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("tc", [True, False])
@pytest.mark.parametrize("fmt,mode", [(q4.NVFP4, "rn"), (q4.NVFP4, "ru"), (q4.NVFP4, "46"),
                                      (q4.MXFP4, "rn"), (q4.MXFP4, "ru"), (q4.MXFP4, "had")])
def test_quantize_grouped_parity(dtype, tc, fmt, mode):
    ws = weights(fmt, 11)
    if dtype == "bf16":
        xs = [synth.to_bf16(w) for w in ws]
        x32 = [synth.bf16_to_f32(x) for x in xs]
    else:
        xs, x32 = ws, ws
    flags = (q4.LAYOUT_TC if tc else 0) | {"rn": 0, "ru": q4.SCALE_RU, "46": q4.SCALE_46,
                                           "had": q4.HADAMARD32}[mode]
    s_ts = [oracle.tensor_scale(oracle.amax(w) if w.size else np.float32(1), 1536.0) for w in x32]
    g_ts = [gscale_dev(s) for s in s_ts] if fmt == q4.NVFP4 else None
    gc, gs = q4.q4_quantize_grouped(fmt, [dev(x) for x in xs], gscales=g_ts, flags=flags)
    for i, w in enumerate(x32):
        if w.size == 0:
            continue
        if fmt == q4.NVFP4:
            if mode == "46":
                oc, os_ = oracle.nvfp4_quantize46(w, s_ts[i])
            else:
                oc, os_ = oracle.nvfp4_quantize(w, s_ts[i], round_up=mode == "ru")
        else:
            oc, os_ = oracle.mxfp4_quantize(w, None, hadamard=mode == "had", round_up=mode == "ru")
        assert np.array_equal(host(gc[i]), oc), f"codes of entry {i}"
        assert np.array_equal(host(gs[i]), oracle_scales(fmt, os_, tc)), f"scales of entry {i}"


def prepared(fmt, tc, seed):
    """Weights with fixed RU scales on both sides, one tuple per non-empty entry."""
    out = []
    for w in weights(fmt, seed):
        if w.size == 0:
            continue
        s_t, g_t, g_sc, o_sc = setup_scales(fmt, w, tc)
        out.append((w, dev(w), s_t, g_t, g_sc, o_sc))
    return out


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("tc", [True, False])
def test_sigma_delta_step_grouped_visits(fmt, tc):
    P = prepared(fmt, tc, 3)
    flags = q4.LAYOUT_TC if tc else 0
    r_gpu = [torch.zeros(p[1].shape, dtype=torch.float32, device=DEV) for p in P]
    r_orc = [np.zeros(p[0].shape, np.float32) for p in P]
    g_ts = [p[3] for p in P] if fmt == q4.NVFP4 else None
    for k in range(4):
        gc = q4.q4_sigma_delta_step_grouped(fmt, [p[1] for p in P], [p[4] for p in P], r_gpu, gscales=g_ts,
                                            flags=flags)
        for i, p in enumerate(P):
            oc = oracle.sigma_delta_step(fmt, p[0], p[5], p[2], r_orc[i])
            assert np.array_equal(host(gc[i]), oc), f"codes of entry {i}, visit {k + 1}"
            assert np.array_equal(host(r_gpu[i]).view(np.uint32), r_orc[i].view(np.uint32)), \
                f"residue of entry {i}, visit {k + 1}"


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("tc", [True, False])
def test_sr_requant_grouped(fmt, tc):
    P = prepared(fmt, tc, 5)
    flags = q4.LAYOUT_TC if tc else 0
    g_ts = [p[3] for p in P] if fmt == q4.NVFP4 else None
    for seed, visit in [(42, 0), (2**40 + 5, 9)]:
        gc = q4.q4_sr_requant_grouped(fmt, [p[1] for p in P], [p[4] for p in P], seed, visit, gscales=g_ts,
                                      flags=flags)
        for i, p in enumerate(P):
            assert np.array_equal(host(gc[i]), oracle.sr_requant(fmt, p[0], p[5], p[2], seed, visit)), \
                f"entry {i}, seed {seed}, visit {visit}"


@pytest.mark.parametrize("fmt", [q4.NVFP4, q4.MXFP4])
@pytest.mark.parametrize("tc", [True, False])
def test_codebanks_grouped(fmt, tc):
    P = prepared(fmt, tc, 7)
    flags = q4.LAYOUT_TC if tc else 0
    g_ts = [p[3] for p in P] if fmt == q4.NVFP4 else None
    K = 6
    # the final residue is asked for on every other entry only
    r_out = [torch.empty(p[1].shape, dtype=torch.float32, device=DEV) if i % 2 == 0 else None
             for i, p in enumerate(P)]
    banks = q4.q4_sigma_delta_codebanks_grouped(fmt, [p[1] for p in P], [p[4] for p in P], K, gscales=g_ts,
                                                flags=flags, residue_out=r_out)
    for i, p in enumerate(P):
        o_banks, o_r = oracle.sigma_delta_codebanks(fmt, p[0], p[5], p[2], K)
        assert np.array_equal(host(banks[i]), o_banks), f"banks of entry {i}"
        if r_out[i] is not None:
            assert np.array_equal(host(r_out[i]).view(np.uint32), o_r.view(np.uint32)), f"residue of entry {i}"


def test_looped_core_grouped_full_size():
    """The 13 looped-core weights (41,943,040 weights) in one grouped launch per
    call: 4/6 quantize, two Sigma-Delta visits and one SR requant.  The oracle
    follows every 61st row of each matrix for the row-local steps (exact: the
    steps are per block / per element) and two whole matrices for SR (its
    counters number the elements of the whole matrix)."""
    d = synth.looped()
    ws = d["w"]
    P = []
    for w in ws:
        s_t, g_t, g_sc, _ = setup_scales(q4.NVFP4, w)
        P.append((w, dev(w), s_t, g_t, g_sc))
    W = [p[1] for p in P]
    G = [p[3] for p in P]
    S = [p[4] for p in P]
    c46, s46 = q4.q4_quantize_grouped(q4.NVFP4, W, gscales=G, flags=q4.SCALE_46 | q4.LAYOUT_TC)
    r_gpu = [torch.zeros_like(w) for w in W]
    codes = [q4.q4_sigma_delta_step_grouped(q4.NVFP4, W, S, r_gpu, gscales=G) for _ in range(2)]
    sr = q4.q4_sr_requant_grouped(q4.NVFP4, W, S, 42, 3, gscales=G)
    for mi, (w, _, s_t, _, _) in enumerate(P):
        rows = w.shape[0]
        sel = np.arange(mi % 61, rows, 61)
        wsel = np.ascontiguousarray(w[sel])
        oc, os_ = oracle.nvfp4_quantize46(wsel, s_t)
        assert np.array_equal(host(c46[mi])[sel], oc)
        got_sc = oracle.scales_from_tc(host(s46[mi]), rows, w.shape[1] // 16)[sel]
        assert np.array_equal(got_sc, os_)
        _, o_sc = oracle.nvfp4_quantize(wsel, s_t, round_up=True)
        r = np.zeros_like(wsel)
        for k in range(2):
            assert np.array_equal(host(codes[k][mi])[sel], oracle.sigma_delta_step(q4.NVFP4, wsel, o_sc, s_t, r))
        assert np.array_equal(host(r_gpu[mi])[sel].view(np.uint32), r.view(np.uint32))
    for mi in (0, len(P) - 1):
        w, _, s_t, _, _ = P[mi]
        _, o_sc = oracle.nvfp4_quantize(w, s_t, round_up=True)
        assert np.array_equal(host(sr[mi]), oracle.sr_requant(q4.NVFP4, w, o_sc, s_t, 42, 3))
