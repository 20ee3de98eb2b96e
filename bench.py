"""Benchmark of the 4-bit block-scaled W4A4 path on B200.

One step = one pass of the prefill-shaped W4A4 linear over one batch:
    tensor amax of X (8192 x 5120 bf16, heavy-tailed) -> s_t,
    then NVFP4 quantize of X (codes + tensor-core scales),  one launch
    W4A4 GEMM of X with W1 (5120 x 5120) and W2 (17408 x 5120),
    both weights in one launch                             (the GEMM TFLOP/s)
with the weights quantized once beforehand and resident in HBM.  `value` is
the GEMM FLOPs of the step divided by the step's device time.  The other
rows of the path are timed on their own workloads under "rows": MXFP4
quantize with per-channel scale and Hadamard-32 plus the MXFP4 GEMM
(4096 x 14336 x 4096), one Sigma-Delta visit over the 13 looped-core weights
(41,943,040 weights), the decode-shaped GEMM with fused activation quantize
(16 x 17408 x 5120), and dequantization.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
N > 1 runs under torchrun, one process per GPU, each rank running the same
workload on its own GPU (the problems are independent: weak scaling, no
collective on the data path; NCCL only for the barrier and the max-over-ranks
timing).  L2 is flushed (a 256 MiB write, then a 256 MiB read, so that no
dirty line is left) before every timed step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import synth  # noqa: E402

METRIC = "W4A4 GEMM TFLOP/s + quantize GB/s on 1 B200, as % of FP4/HBM roofline"
UNIT = "TFLOP/s"
M, K, N1, N2 = 8192, 5120, 5120, 17408
GEMM_FLOPS = 2.0 * M * K * (N1 + N2)
WORKLOAD = ("prefill NVFP4 W4A4 linear: X 8192x5120 bf16 (0.02*Student-t(3), 20% one-hot 16-blocks x100) "
            "-> amax -> NVFP4 quantize -> GEMM with W 5120x5120 and 17408x5120 (N(0,0.02^2), pre-quantized), "
            "bf16 out")
# algorithmic bytes per element (see the design notes)
B_W4A16_GEMM_NOTE = "2*M*N*K FLOP on the bf16 tensor pipe"
B_QUANT_BF16 = 2 + 0.5 + 1 / 16          # read bf16, write codes + E4M3 scale
B_AMAX_BF16 = 2
B_SIGMA_DELTA = 4 + 4 + 4 + 0.5 + 1 / 16  # w, r in, r out, codes, scale
B_SR = 4 + 0.5 + 1 / 16                   # w, codes, scale (the random numbers are computed)
B_MX_QUANT_BF16 = 2 + 0.5 + 1 / 32       # read bf16, write codes + E8M0 scale
B_DEQUANT_BF16 = 0.5 + 1 / 16 + 2


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sus": d["bf16_tflops_sustained"],
                "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}


# dram__bytes_read.sum + dram__bytes_write.sum of one launch of the roofline
# kernel (gemm_kernel<NVFP4>, one launch over both weights: 8192 x (5120 +
# 17408) x 5120) from one ncu capture, with
# the SHA-256 (first 16 hex digits) of the GEMM source file it was built from:
# the bench reports the figure only while that file is unchanged.
GEMM_TRAFFIC = {"bytes": 92923136 + 325975808, "source_sha256_16": "4aa354952cce7c86"}
GEMM_SOURCE = ROOT / "mxfp4_w4a4_block_b200" / "csrc" / "q4_gemm.cu"


def gemm_source_hash() -> str:
    """SHA-256 (16 hex digits) of what the roofline GEMM is built from: the W4A4
    GEMM section of q4_gemm.cu (from its namespace to the W4A16 section) and the
    PTX wrapper header."""
    import hashlib
    text = GEMM_SOURCE.read_text()
    a, b = text.index("namespace gemm {"), text.index("// ------------------------------------------------------------------ W4A16")
    h = hashlib.sha256(text[a:b].encode())
    h.update((GEMM_SOURCE.parent / "q4_ptx.cuh").read_bytes())
    return h.hexdigest()[:16]


def roofline_traffic(override):
    """(bytes or None, note): the captured DRAM traffic of the roofline kernel,
    None once the GEMM source differs from the one the capture was made of."""
    if override is not None:
        return override, "given on the command line"
    cur = gemm_source_hash()
    if GEMM_TRAFFIC["bytes"] is not None and GEMM_TRAFFIC["source_sha256_16"] == cur:
        return GEMM_TRAFFIC["bytes"], f"ncu capture of the kernel built from the GEMM source with sha256 {cur}"
    return None, f"no capture of the current kernel (GEMM source sha256 {cur})"

# Warp instructions executed by one launch of the three issue-bound grouped
# kernels (smsp__inst_executed.sum from one ncu capture each), with the
# SHA-256 (first 16 hex digits) of the quantizer sources they were built from;
# a row reports its issue bound only while those files are unchanged.
ISSUE_COUNTS = {"sources_sha256_16": "2f0ecddb833cf9bf",
                "sr_requant_visit": 96292792, "nvfp4_quantize46_looped_weights": 50849394,
                "sigma_delta_codebanks_K32": 239890479}
ISSUE_SOURCES = [ROOT / "mxfp4_w4a4_block_b200" / "csrc" / n for n in ("q4_quant.cu", "q4_codec.cuh", "q4_ptx.cuh")]
SM_CLOCK_MAX_MHZ = 1965.0      # clocks.max.sm of this B200
ISSUE_PER_SM_CYCLE = 4         # schedulers per SM, one warp instruction each per cycle


def issue_sources_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ISSUE_SOURCES:
        h.update(f.read_bytes())
    return h.hexdigest()[:16]


def issue_bound(row: str, us: float, n_sms: int):
    """Issue-rate bound of an instruction-bound row: the captured warp
    instructions over 4 per SM per cycle at the maximum SM clock."""
    if ISSUE_COUNTS.get("sources_sha256_16") != issue_sources_hash() or row not in ISSUE_COUNTS:
        return {"bound": "alu", "note": "no capture of the current build"}
    t = ISSUE_COUNTS[row] / (n_sms * ISSUE_PER_SM_CYCLE * SM_CLOCK_MAX_MHZ * 1e6) * 1e6
    return {"bound": "alu", "warp_instructions": ISSUE_COUNTS[row], "issue_bound_us": t, "frac": t / us}


# dense FP4 over dense bf16 on B200, nominal (9 / 2.25 PFLOP/s)
FP4_OVER_BF16 = 4.0


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, out_path: Path | None = None):
        self.gpu = gpu_id
        self.proc = None
        self.lines = []
        self.out_path = out_path

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if self.out_path is not None:
            self.out_path.write_text("\n".join(self.lines) + "\n")
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        maxc = max(r[1] for r in rows)
        load = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        active = sorted({names[i] for r in load for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": maxc, "reasons": active,
                "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r[2] for r in rows)}


def gpu_uuid(dev) -> str:
    """nvidia-smi id of the physical GPU behind a torch device (CUDA_VISIBLE_DEVICES aware)."""
    u = str(torch.cuda.get_device_properties(dev).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


# ------------------------------------------------------------------ our arm
class Prefill:
    """Device-resident inputs of the prefill workload and one step over them."""

    def __init__(self, q4, dev):
        self.q4 = q4
        d = synth.prefill()
        self.x_host = d["x"]                                  # bf16 CPU
        self.x = d["x"].to(dev)
        self.amax = torch.zeros(4, dtype=torch.float32, device=dev)
        self.xc = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        self.xs = torch.empty(q4.q4_scale_bytes(q4.NVFP4, M, K), dtype=torch.uint8, device=dev)
        self.w = []
        for w in d["w"]:
            wt = torch.from_numpy(w).to(dev)
            g = q4.q4_amax(wt, 2688.0)
            wc, ws = q4.q4_quantize(q4.NVFP4, wt, gscale=g[1:2])
            self.w.append((w.shape[0], wc, ws, g[1:2].clone()))
            del wt
        self.y = [torch.empty((M, n), dtype=torch.bfloat16, device=dev) for n, *_ in self.w]
        torch.cuda.synchronize()

    def step(self, ev=None, x=None, y=None):
        q4 = self.q4
        x = self.x if x is None else x
        y = self.y if y is None else y
        if ev is not None:
            ev[0].record()
        q4.q4_amax_quantize(x, 2688.0, out=self.amax, codes=self.xc, scales=self.xs)
        if ev is not None:
            ev[1].record()
        q4.q4_gemm_shared_a(q4.NVFP4, M, K, self.xc, self.xs, self.amax[1:2],
                            [(wc, ws, wg, n) for n, wc, ws, wg in self.w], ys=y)
        if ev is not None:
            ev[2].record()

    def two_launch_quantize(self):
        """The same activation quantize as q4_amax then q4_quantize (for comparison)."""
        q4 = self.q4
        q4.q4_amax(self.x, 2688.0, out=self.amax)
        q4.q4_quantize(q4.NVFP4, self.x, gscale=self.amax[1:2], codes=self.xc, scales=self.xs)

    LAUNCHES_PER_STEP = 2   # amax + quantize (one cooperative launch), the two GEMMs (one launch)
    SEGMENTS = 2


def e2e_pipelined(P, steps: int):
    """End to end through the public API with the host copies pipelined: every
    step uploads its X from pinned host memory and reads both Y back to pinned
    host memory, on three streams -- uploads, compute, downloads -- with the
    device X and Y double-buffered, so the next step's upload and this step's
    downloads overlap the compute.
    Returns ms per step (device time from the first upload to the last download)."""
    xh = P.x_host.pin_memory()
    yh = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in P.y]
    xd = [P.x, torch.empty_like(P.x)]
    yd = [P.y, [torch.empty_like(y) for y in P.y]]
    s_up, s_cmp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    E = lambda: torch.cuda.Event()
    up_done, cmp_done, down_done = [E(), E()], [E(), E()], [E(), E()]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    torch.cuda.synchronize()
    start.record(cur)
    for st in (s_up, s_cmp, s_down):
        st.wait_stream(cur)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(cmp_done[b])          # step i - 2 has read X[b]
            xd[b].copy_(xh, non_blocking=True)
            up_done[b].record(s_up)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(up_done[b])
            if i >= 2:
                s_cmp.wait_event(down_done[b])        # step i - 2's results have left Y[b]
            P.step(ev=[E(), E(), cmp_done[b]], x=xd[b], y=yd[b])
        with torch.cuda.stream(s_down):
            s_down.wait_event(cmp_done[b])
            yh[0].copy_(yd[b][0], non_blocking=True)
            yh[1].copy_(yd[b][1], non_blocking=True)
            down_done[b].record(s_down)
    for st in (s_up, s_cmp, s_down):
        cur.wait_stream(st)
    end.record(cur)
    end.synchronize()
    return start.elapsed_time(end) / steps


def time_fn(fn, reps, flush, warm=3):
    """Device time per call (ms) with L2 flushed before each timed call."""
    for _ in range(warm):
        fn()
    ts = []
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        flush()
        s.record()
        fn()
        e.record()
        e.synchronize()
        ts.append(s.elapsed_time(e))
    return statistics.mean(ts), min(ts)


def sigma_delta_quality(q4, mats, visits=32):
    """Weight representation error of R Sigma-Delta visits against static RTN
    ("Looped Transformer quantization", sec. 2.1-2.2): per weight, the mean of
    the R decoded codes against w, and the RTN code (the first visit from
    r_0 = 0) against w, both from the GPU codes.  Also the largest mean error in
    normalised units (|mean_k dec(q_k) / S - w / S|), which the page bounds by
    d / (2R) = 1 / R on E2M1 (largest gap d = 2) in exact arithmetic.  Binary32
    adds at most 6 * 2^-24 (rounding of each decoded code times S) + 2^-22 (x =
    W / S rounded) + 2^-22 (the average of the residue updates' roundings, each
    at most half an ulp of |x + r| < 8): the line reports both."""
    err_sd = err_rtn = 0.0
    worst = 0.0
    fp32_slack = 6 * 2.0 ** -24 + 2 * 2.0 ** -22
    n = 0
    for wt, sc, g, r, c, _ in mats:
        rows, cols = wt.shape
        r.zero_()
        acc = torch.zeros_like(wt, dtype=torch.float64)
        rtn = None
        for k in range(visits):
            q4.q4_sigma_delta_step(q4.NVFP4, wt, sc, r, gscale=g, codes=c)
            dq = q4.q4_dequantize(q4.NVFP4, c, sc, rows, cols, gscale=g)
            acc += dq
            if k == 0:
                rtn = dq.double()
        one = torch.full_like(c, 0x22)                       # code 1.0 in both nibbles: dequantizes to S
        S = q4.q4_dequantize(q4.NVFP4, one, sc, rows, cols, gscale=g).double()
        w64 = wt.double()
        mean = acc / visits
        err_sd += float((mean - w64).abs().sum())
        err_rtn += float((rtn - w64).abs().sum())
        worst = max(worst, float(((mean - w64).abs() / S).max()))
        n += wt.numel()
        r.zero_()
    return {"visits": visits, "weights": n, "mean_abs_err_sigma_delta": err_sd / n, "mean_abs_err_rtn": err_rtn / n,
            "ratio_sigma_delta_over_rtn": err_sd / err_rtn, "max_normalised_mean_err": worst,
            "bound_d_over_2R": 2.0 / (2 * visits), "binary32_allowance": fp32_slack,
            "within_bound": worst <= 2.0 / (2 * visits) + fp32_slack}


def tiny_rows(q4, dev, reps=200):
    """The tiny NVFP4 W4A4 linear (X 64 x 512, W 512 x 512 fp32, 1 % x50
    outliers): amax and quantize of both operands + GEMM with bf16 out, and a
    Sigma-Delta chain of W over R = 8 visits.  Latency-bound: microseconds per
    call with warm L2, eager and as one CUDA graph replay."""
    d = synth.tiny()
    x = torch.from_numpy(d["x"]).to(dev)
    w = torch.from_numpy(d["w"]).to(dev)
    ax = torch.zeros(2, dtype=torch.float32, device=dev)
    aw = torch.zeros(2, dtype=torch.float32, device=dev)
    xc = torch.empty((64, 256), dtype=torch.uint8, device=dev)
    xs = torch.empty(q4.q4_scale_bytes(q4.NVFP4, 64, 512), dtype=torch.uint8, device=dev)
    wc = torch.empty((512, 256), dtype=torch.uint8, device=dev)
    ws = torch.empty(q4.q4_scale_bytes(q4.NVFP4, 512, 512), dtype=torch.uint8, device=dev)
    y = torch.empty((64, 512), dtype=torch.bfloat16, device=dev)
    gw = q4.q4_amax(w, 1536.0)[1:2].clone()
    _, sw = q4.q4_quantize(q4.NVFP4, w, gscale=gw, flags=q4.SCALE_RU | q4.LAYOUT_TC)
    r = torch.zeros_like(w)
    cw = torch.empty((512, 256), dtype=torch.uint8, device=dev)
    ax4 = torch.zeros(4, dtype=torch.float32, device=dev)
    aw4 = torch.zeros(4, dtype=torch.float32, device=dev)
    banks8 = torch.empty((8, 512, 256), dtype=torch.uint8, device=dev)

    def linear():
        q4.q4_amax(x, 2688.0, out=ax)
        q4.q4_quantize(q4.NVFP4, x, gscale=ax[1:2], codes=xc, scales=xs)
        q4.q4_amax(w, 2688.0, out=aw)
        q4.q4_quantize(q4.NVFP4, w, gscale=aw[1:2], codes=wc, scales=ws)
        q4.q4_gemm(q4.NVFP4, 64, 512, 512, xc, xs, ax[1:2], wc, ws, aw[1:2], y=y)

    def linear_fused():
        q4.q4_amax_quantize(x, 2688.0, out=ax4, codes=xc, scales=xs)
        q4.q4_amax_quantize(w, 2688.0, out=aw4, codes=wc, scales=ws)
        q4.q4_gemm(q4.NVFP4, 64, 512, 512, xc, xs, ax4[1:2], wc, ws, aw4[1:2], y=y)

    def chain8():
        r.zero_()
        for _ in range(8):
            q4.q4_sigma_delta_step(q4.NVFP4, w, sw, r, gscale=gw, codes=cw)

    def chain8_banks():
        q4.q4_sigma_delta_codebanks(q4.NVFP4, w, sw, 8, gscale=gw, codes=banks8)

    def per_call(fn):
        for _ in range(10):
            fn()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        e.synchronize()
        return s.elapsed_time(e) * 1e3 / reps

    out = {"linear_us": per_call(linear), "sigma_delta_R8_us": per_call(chain8),
           "linear_fused_us": per_call(linear_fused), "sigma_delta_R8_banks_us": per_call(chain8_banks),
           "launches": {"linear": 5, "linear_fused": 3, "sigma_delta_R8": 9, "sigma_delta_R8_banks": 1},
           "note": "linear_fused: amax and quantize of each operand in one cooperative launch; "
                   "sigma_delta_R8_banks: the 8-visit chain as one codebank launch (same codes)",
           "l2": "warm (latency row)"}
    for name, fn in (("linear", linear), ("sigma_delta_R8", chain8), ("linear_fused", linear_fused),
                     ("sigma_delta_R8_banks", chain8_banks)):
        try:
            g = torch.cuda.CUDAGraph()
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                fn()
            torch.cuda.current_stream().wait_stream(st)
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                fn()
            out[name + "_graph_us"] = per_call(g.replay)
            del g
        except Exception as ex:                  # report, do not hide, a capture that fails
            out[name + "_graph_us"] = None
            out[name + "_graph_error"] = str(ex)[:200]
    out["gemm_TFLOP/s"] = 2.0 * 64 * 512 * 512 / (out["linear_us"] * 1e-6) / 1e12
    return out


def rows_bench(q4, dev, flush, pk, reps=30):
    """Per-row measurements on their own workloads (see module docstring)."""
    out = {}
    hbm = pk["hbm_gbs"]
    fp4 = pk["bf16"] * FP4_OVER_BF16
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out["tiny_linear"] = tiny_rows(q4, dev)

    # a3 + a5 (MXFP4): quantize X with t and Hadamard-32, GEMM with pre-quantized W'
    d = synth.mxfp4()
    xm = d["x"].to(dev)
    t = torch.from_numpy(d["t"]).to(dev)
    wm = torch.from_numpy(d["w"]).to(dev)
    inv_t = torch.from_numpy(d["inv_t"]).to(dev)
    flags = q4.LAYOUT_TC | q4.HADAMARD32
    wc, ws = q4.q4_quantize(q4.MXFP4, wm, chan=inv_t, flags=flags)
    del wm
    Mx, Kx, Nx = 4096, 4096, 14336
    xc = torch.empty((Mx, Kx // 2), dtype=torch.uint8, device=dev)
    xs = torch.empty(q4.q4_scale_bytes(q4.MXFP4, Mx, Kx), dtype=torch.uint8, device=dev)
    ym = torch.empty((Mx, Nx), dtype=torch.bfloat16, device=dev)
    ms_q, _ = time_fn(lambda: q4.q4_quantize(q4.MXFP4, xm, chan=t, flags=flags, codes=xc, scales=xs), reps, flush)
    gbs = Mx * Kx * B_MX_QUANT_BF16 / (ms_q * 1e-3) / 1e9
    out["mxfp4_quantize_t_hadamard"] = {"shape": [Mx, Kx], "us": ms_q * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm}
    ms_g, _ = time_fn(lambda: q4.q4_gemm(q4.MXFP4, Mx, Nx, Kx, xc, xs, None, wc, ws, None, y=ym), reps, flush)
    tf = 2.0 * Mx * Nx * Kx / (ms_g * 1e-3) / 1e12
    out["mxfp4_gemm"] = {"mnk": [Mx, Nx, Kx], "us": ms_g * 1e3, "TFLOP/s": tf, "frac_fp4": tf / fp4,
                         "online_transform_overhead": ms_q / ms_g}
    del xm, t, inv_t, wc, ws, xc, xs, ym

    # a4 + a7: one looped-core visit -- a Sigma-Delta requant of the 13 weights
    # (41,943,040 weights) and the W4A16 GEMM of X (4096 x 1024 bf16) with each
    dl = synth.looped()
    xl = dl["x"].to(dev)
    Ml, Kl = xl.shape
    mats = []
    for w in dl["w"]:
        wt = torch.from_numpy(w).to(dev)
        g = q4.q4_amax(wt, 1536.0)
        _, sc = q4.q4_quantize(q4.NVFP4, wt, gscale=g[1:2], flags=q4.SCALE_RU | q4.LAYOUT_TC)
        mats.append((wt, sc, g[1:2].clone(), torch.zeros_like(wt),
                     torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=dev),
                     torch.empty((Ml, w.shape[0]), dtype=torch.bfloat16, device=dev)))
    nw = sum(w.size for w in dl["w"])
    w16_flops = sum(2.0 * Ml * w.shape[0] * Kl for w in dl["w"])

    # the per-visit requant steps run as one grouped launch over the 13 matrices
    gW = [m[0] for m in mats]
    gS = [m[1] for m in mats]
    gG = [m[2] for m in mats]
    gR = [m[3] for m in mats]
    gC = [m[4] for m in mats]

    def sd_visit():
        q4.q4_sigma_delta_step_grouped(q4.NVFP4, gW, gS, gR, gscales=gG, codes=gC)

    def w16_visit():
        for wt, sc, g, r, c, y in mats:
            q4.q4_gemm(q4.NVFP4, Ml, wt.shape[0], Kl, xl, None, None, c, sc, g, y=y, a_kind=q4.A_BF16_W4A16)

    def visit():
        sd_visit()
        w16_visit()
    ms_sd, _ = time_fn(sd_visit, reps, flush)
    gbs = nw * B_SIGMA_DELTA / (ms_sd * 1e-3) / 1e9
    out["sigma_delta_visit"] = {"weights": nw, "matrices": 13, "us": ms_sd * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm,
                                "us_R32": ms_sd * 1e3 * 32}
    ms_w, _ = time_fn(w16_visit, reps, flush)
    tf = w16_flops / (ms_w * 1e-3) / 1e12
    out["w4a16_visit"] = {"gemms": 13, "M": Ml, "K": Kl, "us": ms_w * 1e3, "TFLOP/s": tf,
                          "frac_bf16": tf / pk["bf16"]}
    banks = [torch.empty((32, wt.shape[0], wt.shape[1] // 2), dtype=torch.uint8, device=dev)
             for wt, *_ in mats]

    def codebanks():
        q4.q4_sigma_delta_codebanks_grouped(q4.NVFP4, gW, gS, 32, gscales=gG, codes=banks)
    ms_cb, _ = time_fn(codebanks, max(5, reps // 3), flush)
    gbs = nw * (4 + 32 * 0.5) / (ms_cb * 1e-3) / 1e9
    out["sigma_delta_codebanks_K32"] = {"weights": nw, "visits": 32, "us": ms_cb * 1e3, "GB/s": gbs,
                                        "frac_hbm": gbs / hbm, "B_per_weight": 4 + 32 * 0.5,
                                        "vs_32_separate_visits": ms_sd * 32 / ms_cb}
    out["sigma_delta_codebanks_K32"]["issue"] = issue_bound("sigma_delta_codebanks_K32", ms_cb * 1e3, n_sms)
    del banks

    q46_c = [torch.empty_like(c) for c in gC]
    q46_s = [torch.empty_like(sc) for sc in gS]

    def q46():
        q4.q4_quantize_grouped(q4.NVFP4, gW, gscales=gG, flags=q4.SCALE_46 | q4.LAYOUT_TC, codes=q46_c, scales=q46_s)
    ms_46, _ = time_fn(q46, reps, flush)
    gbs = nw * (4 + 0.5 + 1 / 16) / (ms_46 * 1e-3) / 1e9
    out["nvfp4_quantize46_looped_weights"] = {"weights": nw, "matrices": 13, "us": ms_46 * 1e3, "GB/s": gbs,
                                              "frac_hbm": gbs / hbm}
    out["nvfp4_quantize46_looped_weights"]["issue"] = issue_bound("nvfp4_quantize46_looped_weights", ms_46 * 1e3, n_sms)
    del q46_c, q46_s

    def sr_visit():
        q4.q4_sr_requant_grouped(q4.NVFP4, gW, gS, 42, 7, gscales=gG, codes=gC)
    ms_sr, _ = time_fn(sr_visit, reps, flush)
    gbs = nw * B_SR / (ms_sr * 1e-3) / 1e9
    out["sr_requant_visit"] = {"weights": nw, "matrices": 13, "us": ms_sr * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm}
    out["sr_requant_visit"]["issue"] = issue_bound("sr_requant_visit", ms_sr * 1e3, n_sms)
    # a decode-shaped visit (M = 16) with the Sigma-Delta codes generated inside the
    # GEMM producer, against the same visit as a separate step + W4A16 GEMM
    xd16 = xl[:16].contiguous()
    yd16 = [torch.empty((16, wt.shape[0]), dtype=torch.bfloat16, device=dev) for wt, *_ in mats]

    def fused16():
        q4.q4_sigma_delta_gemm_grouped(q4.NVFP4, [xd16] * len(mats), gW, gS, gR, gG, ys=yd16)

    def unfused16():
        q4.q4_sigma_delta_step_grouped(q4.NVFP4, gW, gS, gR, gscales=gG, codes=gC)
        for (wt, sc, g, r, c, _), yy in zip(mats, yd16):
            q4.q4_gemm(q4.NVFP4, 16, wt.shape[0], Kl, xd16, None, None, c, sc, g, y=yy, a_kind=q4.A_BF16_W4A16)
    ms_f, _ = time_fn(fused16, reps, flush)
    ms_u, _ = time_fn(unfused16, reps, flush)
    gbs = nw * 12.0 / (ms_f * 1e-3) / 1e9
    out["sigma_delta_fused_gemm_m16"] = {"weights": nw, "matrices": 13, "M": 16, "us": ms_f * 1e3, "GB/s": gbs,
                                         "frac_hbm": gbs / hbm, "B_per_weight": 12.0,
                                         "unfused_us": ms_u * 1e3, "speedup_vs_unfused": ms_u / ms_f}
    del xd16, yd16
    ms_v, _ = time_fn(visit, max(5, reps // 3), flush)
    out["looped_visit"] = {"us": ms_v * 1e3, "us_R32": ms_v * 1e3 * 32,
                           "note": "Sigma-Delta requant of all 13 weights + 13 W4A16 GEMMs"}
    out["sigma_delta_vs_rtn"] = sigma_delta_quality(q4, mats, visits=32)
    del mats, xl

    # a6: decode-shaped GEMM with fused activation quantize
    dd = synth.decode()
    xd = dd["x"].to(dev)
    wt = torch.from_numpy(dd["w"]).to(dev)
    gw = q4.q4_amax(wt, 2688.0)[1:2].clone()
    wc, ws = q4.q4_quantize(q4.NVFP4, wt, gscale=gw)
    del wt
    gx = q4.q4_amax(xd, 2688.0)[1:2].clone()
    Md, Nd, Kd = 16, 17408, 5120
    yd = torch.empty((Md, Nd), dtype=torch.bfloat16, device=dev)
    ms_d, _ = time_fn(lambda: q4.q4_gemm(q4.NVFP4, Md, Nd, Kd, xd, None, gx, wc, ws, gw, y=yd, a_kind=q4.A_BF16),
                      reps * 3, flush)
    byts = Nd * Kd * (0.5 + 1 / 16) + 2 * Md * Kd + 2 * Md * Nd
    gbs = byts / (ms_d * 1e-3) / 1e9
    out["decode_fused_gemm"] = {"mnk": [Md, Nd, Kd], "us": ms_d * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm,
                                "TFLOP/s": 2.0 * Md * Nd * Kd / (ms_d * 1e-3) / 1e12}
    # a8: dequantize (fake quant) of the decode weight, 17408 x 5120 -> bf16
    dq = torch.empty((Nd, Kd), dtype=torch.bfloat16, device=dev)
    ms_dq, _ = time_fn(lambda: q4.q4_dequantize(q4.NVFP4, wc, ws, Nd, Kd, gscale=gw, out_dtype=torch.bfloat16, out=dq),
                       reps, flush)
    gbs = Nd * Kd * B_DEQUANT_BF16 / (ms_dq * 1e-3) / 1e9
    out["dequantize_bf16"] = {"shape": [Nd, Kd], "us": ms_dq * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm}
    del xd, wc, ws, yd, dq
    torch.cuda.empty_cache()
    return out


def rank_env():
    """(rank, world size, local rank) as the launcher sets them; a plain
    single-process run is rank 0 of 1."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's figure.  Every rank calls this at the same point (the
    collective order is the same on all ranks); `dist` None = one process."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: float, step_ms: float) -> float:
    """Whole-job throughput: every rank runs its own copy of the step (weak
    scaling), so the job does world x the step's FLOPs in the slowest rank's
    step time."""
    return world * flops_per_rank_step / (step_ms * 1e-3) / 1e12


def run_ours(args):
    import mxfp4_w4a4_block_b200 as q4
    rank, world, local = rank_env()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q4.lib()
    pk = peaks()
    hbm = pk["hbm_gbs"]
    fp4_burst = pk["bf16"] * FP4_OVER_BF16
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    def flush():
        # write 256 MiB (evicts everything), then read another 256 MiB so that the
        # L2 holds no dirty lines whose write-back the next kernel would pay for
        flush_buf.fill_(1)
        flush_rd.sum()

    P = Prefill(q4, dev)
    # the achieved heavy-tail statistic of the synthetic X: median over rows of max|x| / rms(x)
    xf = P.x.float()
    ratio = xf.abs().amax(dim=1) / xf.pow(2).mean(dim=1).sqrt()
    x_stat = {"row_max_over_rms_median": float(ratio.median()),
              "one_hot_block_fraction_recipe": 0.2}
    del xf, ratio
    for _ in range(max(args.warmup, 3)):
        P.step()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(Prefill.SEGMENTS + 1)] for _ in range(args.steps)]
    clock_path = Path(args.clocks_csv) if args.clocks_csv else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with ClockSampler(gpu_uuid(dev), clock_path) as cs:
        for i in range(args.steps):
            flush()
            P.step(evs[i])
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    wall = time.perf_counter() - wall0
    seg = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(Prefill.SEGMENTS)]
                    for i in range(args.steps)])
    step_ms = max_over_ranks(float(seg.sum(axis=1).mean()), dist, dev)
    clocks = cs.summary()
    k_ms = seg.mean(axis=0)          # amax + quantize, the shared-A GEMM launch
    gemm_tf = GEMM_FLOPS / (k_ms[1] * 1e-3) / 1e12
    # the fused launch reads X from HBM once (the second pass mostly hits L2):
    # its algorithmic bytes are those of the quantize alone
    q_gbs = M * K * B_QUANT_BF16 / (k_ms[0] * 1e-3) / 1e9
    value = whole_job_tflops(world, GEMM_FLOPS, step_ms)

    # end to end through the C ABI with host buffers: pinned X in, both Y out
    e2e = None
    if not args.no_e2e:
        xh = P.x_host.pin_memory()
        yh = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in P.y]
        reps = max(3, args.e2e_steps)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for i in range(reps + 2):
            flush()
            s.record()
            P.x.copy_(xh, non_blocking=True)
            P.step()
            for y, h in zip(P.y, yh):
                h.copy_(y, non_blocking=True)
            e.record()
            e.synchronize()
            if i >= 2:
                ts.append(s.elapsed_time(e))
        serial_ms = max_over_ranks(statistics.mean(ts), dist, dev)
        pipe_err = None
        try:
            e2e_pipelined(P, 2)                              # warm-up of the streams and buffers
            pipe_ms = e2e_pipelined(P, max(4, args.e2e_steps))
        except Exception as ex:                              # report it; the serial figure stands
            pipe_err, pipe_ms = str(ex)[:200], serial_ms
        e2e_ms = max_over_ranks(pipe_ms, dist, dev)
        e2e = {"value": whole_job_tflops(world, GEMM_FLOPS, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(P.x_host.numel() * 2),
               "d2h_bytes_per_step": int(sum(y.numel() * 2 for y in P.y)), "ms_per_step": e2e_ms,
               "note": ("copies pipelined over steps on three streams (uploads, compute, downloads)"
                        if pipe_err is None else "pipelined run failed (" + pipe_err + "); serial figure"),
               "serial": {"value": whole_job_tflops(world, GEMM_FLOPS, serial_ms), "ms_per_step": serial_ms,
                          "note": "upload, step, downloads back to back, L2 flushed before each step"}}

    rows = None
    if not args.no_rows:
        # the prefill activation quantize alone after a cold, clean L2, and the
        # same work as two launches (amax, then quantize)
        xq_ms, _ = time_fn(lambda: q4.q4_quantize(q4.NVFP4, P.x, gscale=P.amax[1:2], codes=P.xc, scales=P.xs), 30,
                           flush)
        xq_gbs = M * K * B_QUANT_BF16 / (xq_ms * 1e-3) / 1e9
        iso_quant = {"shape": [M, K], "us": xq_ms * 1e3, "GB/s": xq_gbs, "frac_hbm": xq_gbs / hbm}
        am_ms, _ = time_fn(lambda: q4.q4_amax(P.x, 2688.0, out=P.amax), 30, flush)
        two_ms, _ = time_fn(P.two_launch_quantize, 30, flush)
        fused_ms, _ = time_fn(lambda: q4.q4_amax_quantize(P.x, 2688.0, out=P.amax, codes=P.xc, scales=P.xs), 30,
                              flush)
        a_gbs = M * K * B_AMAX_BF16 / (am_ms * 1e-3) / 1e9
        rows = {}
        rows["amax_quantize_prefill_x"] = {"shape": [M, K], "us": k_ms[0] * 1e3, "GB/s": q_gbs,
                                           "frac_hbm": q_gbs / hbm, "B_per_element": B_QUANT_BF16,
                                           "note": "in the step: one cooperative launch, amax then quantize"}
        fused_gbs = M * K * B_QUANT_BF16 / (fused_ms * 1e-3) / 1e9
        rows["amax_quantize_prefill_x_cold"] = {"us": fused_ms * 1e3, "GB/s": fused_gbs, "frac_hbm": fused_gbs / hbm,
                                                "two_launches_us": two_ms * 1e3,
                                                "speedup_vs_two_launches": two_ms / fused_ms}
        rows["nvfp4_quantize_prefill_x_cold"] = iso_quant
        rows["amax_prefill_x_cold"] = {"us": am_ms * 1e3, "GB/s": a_gbs, "frac_hbm": a_gbs / hbm}
        rows["gemm_prefill_shared_a"] = {"us": k_ms[1] * 1e3, "TFLOP/s": gemm_tf, "frac_fp4": gemm_tf / fp4_burst,
                                         "note": "in the step: both weights in one launch"}
        for n, wc, ws, wg in P.w:
            yy = torch.empty((M, n), dtype=torch.bfloat16, device=dev)
            g_ms, _ = time_fn(lambda: q4.q4_gemm(q4.NVFP4, M, n, K, P.xc, P.xs, P.amax[1:2], wc, ws, wg, y=yy), 20,
                              flush)
            tf = 2.0 * M * n * K / (g_ms * 1e-3) / 1e12
            rows[f"gemm_prefill_n{n}_cold"] = {"us": g_ms * 1e3, "TFLOP/s": tf, "frac_fp4": tf / fp4_burst,
                                               "note": "the single-weight launch alone, after a cold, clean L2"}
            del yy
        del P
        torch.cuda.empty_cache()
        rows.update(rows_bench(q4, dev, flush, pk, reps=args.rows_reps))

    cpu = None if args.no_cpu_baseline or rank != 0 else cpu_baseline(budget_s=args.cpu_seconds)
    traffic, traffic_note = roofline_traffic(args.traffic)
    # a timed region of a second or more runs the GEMM under the power cap: its
    # peak is then the sustained (seconds-long loop) figure, else the burst one
    fp4_sus = pk["bf16_sus"] * FP4_OVER_BF16
    sustained = wall >= 1.0
    fp4_peak = fp4_sus if sustained else fp4_burst
    peak_note = (f"dense FP4 = {pk['src']} bf16 {'sustained' if sustained else 'burst'} "
                 f"{pk['bf16_sus'] if sustained else pk['bf16']} x 4 (nominal 9/2.25); "
                 f"{'sustained' if sustained else 'burst'}: the timed region lasted {wall:.2f} s")

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1 x e2m1 -> f32 (NVFP4 block-scaled)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": [N1, N2], "x_stat": x_stat, "quantize_GB/s": q_gbs,
                   "quantize_frac_hbm": q_gbs / hbm, "l2": "flushed before every timed step: 256 MiB write, then a 256 MiB read (cold, clean L2)",
                   "parallelism": f"replicas x{world} (independent problems per GPU)"},
        "roofline": {"kernel": "gemm_kernel<NVFP4>, one launch over W1 and W2: 8192 x (5120 + 17408) x 5120",
                     "bound": "tensor", "achieved": gemm_tf,
                     "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tf / fp4_peak,
                     "peak_note": peak_note,
                     "frac_vs_burst": gemm_tf / fp4_burst,
                     "frac_vs_sustained": gemm_tf / fp4_sus,
                     "traffic": traffic, "traffic_note": traffic_note,
                     "algorithmic_bytes": M * K / 2 + M * K / 16 + (N1 + N2) * K * (0.5 + 1 / 16) + 2 * M * (N1 + N2)},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": Prefill.LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks,
        "timed_wall_s": wall,
        "rows": rows,
    }
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ oracle arm
class OracleSample:
    """A bounded sample of the prefill workload for the CPU oracle: the first
    `rows` rows of X and `cols` rows of each weight, quantized by the oracle."""

    def __init__(self, rows: int = 64, cols: int = 256):
        import oracle
        self.oracle = oracle
        d = synth.prefill()
        x32 = synth.bf16_to_f32(d["x"])
        self.rows, self.cols = rows, cols
        self.s_t = oracle.tensor_scale(oracle.amax(x32), 2688.0)
        self.x = np.ascontiguousarray(x32[:rows])
        self.w = []
        for w in d["w"]:
            w_t = oracle.tensor_scale(oracle.amax(w), 2688.0)
            self.w.append([np.ascontiguousarray(w[j * cols:(j + 1) * cols]) for j in range(w.shape[0] // cols)]
                          + [w_t])

    def quantize(self):
        o = self.oracle
        t0 = time.perf_counter()
        o.amax(self.x)
        c, s = o.nvfp4_quantize(self.x, self.s_t)
        return c, s, time.perf_counter() - t0

    def gemm_chunk(self, xc, xs, wi: int, j: int):
        """One (rows x cols x K) oracle GEMM; returns (flops, seconds)."""
        o = self.oracle
        chunks, w_t = self.w[wi][:-1], self.w[wi][-1]
        wc, wsc = o.nvfp4_quantize(chunks[j % len(chunks)], w_t)
        t0 = time.perf_counter()
        o.gemm(o.NVFP4, xc, xs, self.s_t, wc, wsc, w_t, self.rows, self.cols, K)
        return 2.0 * self.rows * self.cols * K, time.perf_counter() - t0


def _row_ranges(n: int, parts: int):
    step = max(1, (n + parts - 1) // parts)
    return [(i, min(n, i + step)) for i in range(0, n, step)]


def _on_threads(fn, items, threads: int):
    """fn over items on `threads` host threads.  The oracle's arithmetic runs
    in C behind ctypes, which releases the GIL, so the calls run in parallel."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


def cpu_baseline(budget_s: float = 10.0):
    """The CPU oracle as it stands, on the machine's host cores: single-threaded and
    row-parallel over every core the process may use (the same oracle calls on
    row ranges, one host thread each).

    * NVFP4 quantize of the full prefill X (8192 x 5120, amax included);
    * one Sigma-Delta visit over all 13 looped-core weights (41,943,040);
    * the binary64 GEMM on a sample: 64 rows of X against 256-row chunks of
      W1 / W2 (K = 5120), for about budget_s / 2 seconds each way.
    `value` is the all-core GEMM throughput in the line's unit."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    smp = OracleSample()
    x32 = synth.bf16_to_f32(synth.prefill(n_list=())["x"])

    def quant(rng):
        i0, i1 = rng
        oracle.amax(x32[i0:i1])
        oracle.nvfp4_quantize(x32[i0:i1], smp.s_t)
    t0 = time.perf_counter()
    quant((0, M))
    q1 = time.perf_counter() - t0
    t0 = time.perf_counter()
    _on_threads(quant, _row_ranges(M, 4 * threads), threads)
    qn = time.perf_counter() - t0
    qbytes = M * K * (B_QUANT_BF16 + B_AMAX_BF16)
    del x32

    dl = synth.looped(m=16)
    mats = []

    def prep(w):
        s_t = oracle.tensor_scale(oracle.amax(w), 1536.0)
        _, sc = oracle.nvfp4_quantize(w, s_t, round_up=True)
        return w, sc, s_t, np.zeros_like(w)
    mats = _on_threads(prep, dl["w"], threads)
    nw = sum(w.size for w, *_ in mats)

    def sd(item):
        w, sc, s_t, r, (i0, i1) = item
        oracle.sigma_delta_step(oracle.NVFP4, w[i0:i1], sc[i0:i1], s_t, r[i0:i1])
    t0 = time.perf_counter()
    for w, sc, s_t, r in mats:
        sd((w, sc, s_t, r, (0, w.shape[0])))
    s1 = time.perf_counter() - t0
    items = [(w, sc, s_t, r, rr) for w, sc, s_t, r in mats for rr in _row_ranges(w.shape[0], threads)]
    t0 = time.perf_counter()
    _on_threads(sd, items, threads)
    sn = time.perf_counter() - t0
    del mats, dl

    xc, xs, _ = smp.quantize()
    f1, g1, j = 0.0, 0.0, 0
    while g1 < budget_s / 2:
        f, t = smp.gemm_chunk(xc, xs, j % 2, j // 2)
        f1, g1, j = f1 + f, g1 + t, j + 1
    n_chunks = max(threads, 2 * threads)
    t0 = time.perf_counter()
    fn = 0.0
    while time.perf_counter() - t0 < budget_s / 2:
        res = _on_threads(lambda jj: smp.gemm_chunk(xc, xs, jj % 2, jj // 2)[0], range(n_chunks), threads)
        fn += sum(res)
    gn = time.perf_counter() - t0
    return {"value": fn / gn / 1e12, "unit": UNIT, "cores": threads, "host_cpu_count": os.cpu_count(),
            "kind": "oracle",
            "sample": (f"GEMM: binary64 oracle on {smp.rows} rows of X against {smp.cols}-row chunks of W1/W2 "
                       f"(K = {K}), ~{budget_s / 2:.0f} s single-threaded and ~{budget_s / 2:.0f} s on all "
                       f"{threads} threads; quantize: the full 8192 x 5120 X (amax + NVFP4); Sigma-Delta: one "
                       f"visit over the full looped core ({nw} weights)"),
            "gemm_TFLOP/s_1thread": f1 / g1 / 1e12,
            "quantize_GB/s_1thread": qbytes / q1 / 1e9, "quantize_GB/s_all": qbytes / qn / 1e9,
            "sigma_delta_GB/s_1thread": nw * B_SIGMA_DELTA / s1 / 1e9,
            "sigma_delta_GB/s_all": nw * B_SIGMA_DELTA / sn / 1e9}


def run_reference(args):
    """The oracle arm: each step is a bounded sample of the prefill workload
    sized so that warm-up + timed steps take about two minutes in total."""
    rank, _, _ = rank_env()
    if rank != 0:
        return
    smp = OracleSample(rows=16, cols=64)
    xc, xs, tq = smp.quantize()
    budget = min(1.0, 120.0 / max(1, args.steps + args.warmup))
    flops, secs, times, j = 0.0, 0.0, [], 0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        f_step, t_step = 0.0, 0.0
        while True:
            f, t = smp.gemm_chunk(xc, xs, j % 2, j // 2)
            f_step += f
            t_step += t
            j += 1
            if time.perf_counter() - t0 >= budget:
                break
        if i >= args.warmup:
            flops += f_step
            secs += t_step
            times.append(time.perf_counter() - t0)
    val = flops / secs / 1e12
    cpu = {"value": val, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"per step: binary64 GEMMs of {smp.rows} rows of X against {smp.cols}-row chunks of "
                     f"W1/W2 (K = {K}) for ~{budget * 1e3:.0f} ms, operands quantized by the oracle"}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": statistics.mean(times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": cpu["sample"]},
        "cpu_baseline": cpu,
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


PROFILE_ROWS = ("mxfp4_quantize", "amax_quantize", "nvfp4_quantize", "gemm_n5120", "gemm_n17408", "gemm_shared",
                "decode",
                "sigma_delta_visit", "sd_gemm_m16", "w4a16_4096", "sr_visit", "q46_visit", "codebanks_visit")


def run_profile(row: str, launches: int):
    """Launch one row's kernel `launches` times on its workload, untimed: the
    program a profiler capture of that kernel runs."""
    import mxfp4_w4a4_block_b200 as q4
    dev = torch.device("cuda", 0)
    if row == "mxfp4_quantize":
        d = synth.mxfp4(n=256)
        x, t = d["x"].to(dev), torch.from_numpy(d["t"]).to(dev)
        c = torch.empty((4096, 2048), dtype=torch.uint8, device=dev)
        sc = torch.empty(q4.q4_scale_bytes(q4.MXFP4, 4096, 4096), dtype=torch.uint8, device=dev)
        fn = lambda: q4.q4_quantize(q4.MXFP4, x, chan=t, flags=q4.LAYOUT_TC | q4.HADAMARD32, codes=c, scales=sc)
    elif row in ("amax_quantize", "nvfp4_quantize", "gemm_n5120", "gemm_n17408", "gemm_shared"):
        n_list = {"gemm_n5120": (N1,), "gemm_n17408": (N2,), "gemm_shared": (N1, N2)}.get(row, ())
        d = synth.prefill(n_list=n_list)
        x = d["x"].to(dev)
        out = torch.zeros(4, dtype=torch.float32, device=dev)
        c = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty(q4.q4_scale_bytes(q4.NVFP4, M, K), dtype=torch.uint8, device=dev)
        q4.q4_amax_quantize(x, 2688.0, out=out, codes=c, scales=sc)
        if row == "amax_quantize":
            fn = lambda: q4.q4_amax_quantize(x, 2688.0, out=out, codes=c, scales=sc)
        elif row == "nvfp4_quantize":
            fn = lambda: q4.q4_quantize(q4.NVFP4, x, gscale=out[1:2], codes=c, scales=sc)
        else:
            wts = []
            for wn in d["w"]:
                w = torch.from_numpy(wn).to(dev)
                g = q4.q4_amax(w, 2688.0)[1:2].clone()
                wc, ws = q4.q4_quantize(q4.NVFP4, w, gscale=g)
                del w
                wts.append((wc, ws, g, wn.shape[0]))
            ys = [torch.empty((M, n), dtype=torch.bfloat16, device=dev) for n in n_list]
            if row == "gemm_shared":
                fn = lambda: q4.q4_gemm_shared_a(q4.NVFP4, M, K, c, sc, out[1:2], wts, ys=ys)
            else:
                wc, ws, g, n = wts[0]
                fn = lambda: q4.q4_gemm(q4.NVFP4, M, n, K, c, sc, out[1:2], wc, ws, g, y=ys[0])
    elif row == "decode":
        dd = synth.decode()
        xd = dd["x"].to(dev)
        wt = torch.from_numpy(dd["w"]).to(dev)
        gw = q4.q4_amax(wt, 2688.0)[1:2].clone()
        wc, ws = q4.q4_quantize(q4.NVFP4, wt, gscale=gw)
        del wt
        gx = q4.q4_amax(xd, 2688.0)[1:2].clone()
        yd = torch.empty((16, 17408), dtype=torch.bfloat16, device=dev)
        fn = lambda: q4.q4_gemm(q4.NVFP4, 16, 17408, 5120, xd, None, gx, wc, ws, gw, y=yd, a_kind=q4.A_BF16)
    else:
        dl = synth.looped()
        xl = dl["x"].to(dev)
        mats = []
        for w in dl["w"]:
            wt = torch.from_numpy(w).to(dev)
            g = q4.q4_amax(wt, 1536.0)[1:2].clone()
            _, scl = q4.q4_quantize(q4.NVFP4, wt, gscale=g, flags=q4.SCALE_RU | q4.LAYOUT_TC)
            mats.append((wt, scl, g, torch.zeros_like(wt),
                         torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=dev)))
        gW, gS, gG, gR, gC = ([m[i] for m in mats] for i in range(5))
        if row == "sigma_delta_visit":
            fn = lambda: q4.q4_sigma_delta_step_grouped(q4.NVFP4, gW, gS, gR, gscales=gG, codes=gC)
        elif row == "sr_visit":
            fn = lambda: q4.q4_sr_requant_grouped(q4.NVFP4, gW, gS, 42, 7, gscales=gG, codes=gC)
        elif row == "q46_visit":
            q46_s = [torch.empty_like(sc) for sc in gS]
            fn = lambda: q4.q4_quantize_grouped(q4.NVFP4, gW, gscales=gG, flags=q4.SCALE_46 | q4.LAYOUT_TC,
                                                codes=gC, scales=q46_s)
        elif row == "codebanks_visit":
            banks = [torch.empty((32, w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=dev) for w in gW]
            fn = lambda: q4.q4_sigma_delta_codebanks_grouped(q4.NVFP4, gW, gS, 32, gscales=gG, codes=banks)
        elif row == "sd_gemm_m16":
            x16 = xl[:16].contiguous()
            ys = [torch.empty((16, w.shape[0]), dtype=torch.bfloat16, device=dev) for w in gW]
            fn = lambda: q4.q4_sigma_delta_gemm_grouped(q4.NVFP4, [x16] * len(gW), gW, gS, gR, gG, ys=ys)
        else:
            wt, scl, g, _, c = mats[4]                           # a 4096 x 1024 looped-core weight
            q4.q4_sigma_delta_step(q4.NVFP4, wt, scl, torch.zeros_like(wt), gscale=g, codes=c)
            y = torch.empty((xl.shape[0], wt.shape[0]), dtype=torch.bfloat16, device=dev)
            fn = lambda: q4.q4_gemm(q4.NVFP4, xl.shape[0], wt.shape[0], xl.shape[1], xl, None, None, c, scl, g, y=y,
                                    a_kind=q4.A_BF16_W4A16)
    torch.cuda.synchronize()
    for _ in range(launches):
        fn()
    torch.cuda.synchronize()
    print(f"profiled row {row}: {launches} launches")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write the clock samples taken during the timed steps to this CSV file")
    ap.add_argument("--rows-reps", type=int, default=30,
                    help="timed calls per kernel row (small values for profiler captures)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the roofline kernel from an ncu capture (overrides the stored one)")
    ap.add_argument("--profile", choices=PROFILE_ROWS, default=None,
                    help="only launch this row's kernel --profile-launches times, untimed (for profiler captures)")
    ap.add_argument("--profile-launches", type=int, default=4)
    args = ap.parse_args()
    if args.profile:
        run_profile(args.profile, args.profile_launches)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
