"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and arranges them; it holds none of the
quantization, Sigma-Delta or GEMM arithmetic.  Both the CUDA path (through the
product package) and the CPU oracle consume exactly the arrays made here.

Recipes (numpy ``default_rng(seed)``, float32 draws, bf16 by round-to-nearest-
even where an input is bf16):

* ``tiny``      (seed 0): X 64x512 and W 512x512 ~ N(0, 1); 1% of entries
  (Bernoulli) multiplied by 50; float32.
* ``decode``    (seed 1): X 16x5120 = 0.02 * Student-t(3); 20% of the 16-element
  blocks, chosen at random, get one random entry multiplied by 100; bf16.
  W 17408x5120 ~ N(0, 0.02^2).
* ``prefill``   (seed 2): X 8192x5120 drawn like ``decode``; W 5120x5120 and
  17408x5120 ~ N(0, 0.02^2).
* ``looped``    (seed 3): 13 master weights ~ N(0, 0.02^2), four 1024x1024 and
  nine 4096x1024 (41,943,040 weights); X 4096x1024 ~ N(0, 1), bf16.
* ``mxfp4``     (seed 4): X 4096x4096 = the Student-t recipe above plus 10 random
  columns multiplied by 50, bf16; W 14336x4096 ~ N(0, 0.02^2).  The per-channel
  balancing scale t is a calibration output, outside the hot path; it is
  synthesised from a separate calibration draw (seed 5, 1024 rows of the same
  activation recipe) as t_j = sigma_W_j^0.75 / rms_x_j^0.25, clipped to
  [1e-3, 1e3], and 1/t is rounded to float32 on the host.

These stand in for the real captured activations and trained weights that the
pages measure on (heavy-tailed rows, one-hot 16-blocks, outlier channels).
"""
from __future__ import annotations

import numpy as np
import torch

CONFIGS = ("tiny", "decode", "prefill", "looped", "mxfp4")

LOOPED_SHAPES = [(1024, 1024)] * 4 + [(4096, 1024)] * 9


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 numpy -> bf16 torch CPU tensor (round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_to_f32(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> float32 numpy (exact widening)."""
    return t.float().numpy()


def gaussian(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def bernoulli_outliers(rng, x: np.ndarray, p: float, factor: float) -> np.ndarray:
    mask = rng.random(x.shape) < p
    x = x.copy()
    x[mask] *= np.float32(factor)
    return x


def heavy_tailed(rng, rows: int, cols: int, one_hot_frac: float = 0.2,
                 factor: float = 100.0, block: int = 16) -> np.ndarray:
    """0.02 * Student-t(3), plus one entry x100 in a random 20% of 16-blocks."""
    x = (rng.standard_t(3.0, size=(rows, cols)) * 0.02).astype(np.float32)
    nblk = rows * (cols // block)
    chosen = rng.random(nblk) < one_hot_frac
    idx = np.nonzero(chosen)[0]
    within = rng.integers(0, block, size=idx.size)
    flat = x.reshape(-1)
    flat_idx = (idx // (cols // block)) * cols + (idx % (cols // block)) * block + within
    flat[flat_idx] *= np.float32(factor)
    return x


def outlier_channels(rng, x: np.ndarray, n: int, factor: float) -> np.ndarray:
    cols = rng.choice(x.shape[1], size=n, replace=False)
    x = x.copy()
    x[:, cols] *= np.float32(factor)
    return x


def tiny(seed: int = 0):
    rng = np.random.default_rng(seed)
    x = bernoulli_outliers(rng, gaussian(rng, (64, 512)), 0.01, 50.0)
    w = bernoulli_outliers(rng, gaussian(rng, (512, 512)), 0.01, 50.0)
    return {"x": x, "w": w}


def decode(seed: int = 1, n: int = 17408, k: int = 5120, m: int = 16):
    rng = np.random.default_rng(seed)
    x = heavy_tailed(rng, m, k)
    w = gaussian(rng, (n, k), 0.02)
    return {"x": to_bf16(x), "w": w}


def prefill(seed: int = 2, m: int = 8192, k: int = 5120, n_list=(5120, 17408)):
    rng = np.random.default_rng(seed)
    x = heavy_tailed(rng, m, k)
    ws = [gaussian(rng, (n, k), 0.02) for n in n_list]
    return {"x": to_bf16(x), "w": ws}


def looped(seed: int = 3, shapes=None, m: int = 4096):
    rng = np.random.default_rng(seed)
    shapes = LOOPED_SHAPES if shapes is None else shapes
    ws = [gaussian(rng, s, 0.02) for s in shapes]
    x = gaussian(rng, (m, shapes[0][1]))
    return {"w": ws, "x": to_bf16(x)}


def balancing_scale(w: np.ndarray, xcal: np.ndarray, alpha: float = 0.75,
                    lo: float = 1e-3, hi: float = 1e3):
    """Synthetic calibration output t (float32) and its host-rounded inverse."""
    sig_w = np.sqrt(np.mean(w.astype(np.float64) ** 2, axis=0))
    rms_x = np.sqrt(np.mean(xcal.astype(np.float64) ** 2, axis=0))
    t = np.clip(sig_w ** alpha / np.maximum(rms_x, 1e-30) ** (1.0 - alpha), lo, hi)
    t32 = t.astype(np.float32)
    inv_t = (1.0 / t32.astype(np.float64)).astype(np.float32)
    return t32, inv_t


def mxfp4(seed: int = 4, m: int = 4096, k: int = 4096, n: int = 14336, calib_seed: int = 5,
          calib_rows: int = 1024):
    rng = np.random.default_rng(seed)
    x = outlier_channels(rng, heavy_tailed(rng, m, k), 10, 50.0)
    w = gaussian(rng, (n, k), 0.02)
    crng = np.random.default_rng(calib_seed)
    xcal = outlier_channels(crng, heavy_tailed(crng, calib_rows, k), 10, 50.0)
    t, inv_t = balancing_scale(w, xcal)
    return {"x": to_bf16(x), "w": w, "t": t, "inv_t": inv_t}


def small_like(kind: str, seed: int, rows: int, cols: int) -> np.ndarray:
    """Small float32 draws with a given recipe, for parity cases at odd sizes."""
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        return gaussian(rng, (rows, cols))
    if kind == "heavy":
        return heavy_tailed(rng, rows, cols)
    if kind == "outlier":
        return bernoulli_outliers(rng, gaussian(rng, (rows, cols)), 0.01, 50.0)
    if kind == "weight":
        return gaussian(rng, (rows, cols), 0.02)
    raise ValueError(kind)
