"""Pins for the oracle's block-Hadamard-32 and per-channel transform.

MACaQ, core method step (ii): x' = (x.t)B, W' = (W/t)B with B orthogonal, so
the unquantised product XW^T is unchanged.  The matrix is checked against
scipy's Sylvester-order Hadamard matrix.
"""
import numpy as np
import scipy.linalg

import synth


def oracle_matrix(orc):
    """Columns are the oracle's unnormalised FWHT of the unit vectors."""
    return np.stack([orc.fwht32(np.eye(32, dtype=np.float32)[j]) for j in range(32)], axis=1)


def test_fwht_is_sylvester_hadamard(orc):
    H = oracle_matrix(orc)
    assert np.array_equal(H, scipy.linalg.hadamard(32).astype(np.float32))


def test_hadamard_orthogonal(orc):
    H = oracle_matrix(orc).astype(np.float64)
    assert np.array_equal(H @ H.T, 32.0 * np.eye(32))


def test_one_hot_spreads_flat(orc):
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = 1.0
    y = orc.mx_transform(x, None, True)
    assert np.allclose(np.abs(y), 1 / np.sqrt(32), rtol=1e-7, atol=0)


def test_transform_is_linear_in_blocks(orc):
    """Blocks are transformed independently: a one-hot in block 1 leaves block 0 at zero."""
    x = np.zeros((1, 64), np.float32)
    x[0, 40] = 2.0
    y = orc.mx_transform(x, None, True)
    assert not y[0, :32].any() and np.all(y[0, 32:] != 0)


def test_product_invariance_unquantised(orc):
    """X' W'^T == X W^T with c = t for X and c = 1/t for W (binary32 rounding only)."""
    x = synth.small_like("heavy", 3, 16, 128)
    w = synth.small_like("weight", 4, 24, 128)
    t = np.exp(np.random.default_rng(6).uniform(-1, 1, 128)).astype(np.float32)
    inv_t = (1.0 / t.astype(np.float64)).astype(np.float32)
    xp = orc.mx_transform(x, t, True).astype(np.float64)
    wp = orc.mx_transform(w, inv_t, True).astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    got = xp @ wp.T
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-6
    # without the rotation the scale alone also cancels
    xs = orc.mx_transform(x, t, False).astype(np.float64)
    ws = orc.mx_transform(w, inv_t, False).astype(np.float64)
    assert np.linalg.norm(xs @ ws.T - ref) / np.linalg.norm(ref) < 1e-6
