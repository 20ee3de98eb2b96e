"""First-order Sigma-Delta over an arbitrary finite codebook, in exact rational
arithmetic (TEST INFRASTRUCTURE ONLY; see the package docstring).

Follows "Looped Transformer quantization: error propagation, NVFP4 and
Sigma-Delta modulation", sec. 2.1 (the recursion with a fixed scale:
r_0 = 0, v_k = x + r_{k-1}, q_k = Q(v_k), r_k = v_k - q_k) and sec. 2.2 (Q is
nearest rounding onto a codebook C = {c_0 < ... < c_N}, saturating to the end
points outside [c_0, c_N]).  Pure-Python loops: small cases only.
"""
from __future__ import annotations

from fractions import Fraction
from typing import Callable, Sequence


def nearest(codebook: Sequence[Fraction], tie="up") -> Callable[[Fraction], Fraction]:
    """Nearest-point quantizer with end-point saturation.

    tie="up": ties go to the larger point (the integer-grid example's
    floor(v + 1/2)); otherwise ``tie`` is a predicate on points, and a tie goes
    to the point for which it is true (for E2M1: the even mantissa bit).
    """
    cb = sorted(Fraction(c) for c in codebook)

    def q(v: Fraction) -> Fraction:
        if v <= cb[0]:
            return cb[0]
        if v >= cb[-1]:
            return cb[-1]
        best, best_d = cb[0], abs(v - cb[0])
        for c in cb[1:]:
            d = abs(v - c)
            if d < best_d:
                best, best_d = c, d
            elif d == best_d and (tie == "up" or (callable(tie) and tie(c))):
                best = c
        return best

    return q


def floor_half_up(v: Fraction) -> Fraction:
    """Q(v) = floor(v + 1/2) on the unbounded integer grid."""
    return Fraction((v + Fraction(1, 2)).__floor__())


def sequence(x, quantizer: Callable[[Fraction], Fraction], m: int):
    """Return lists (v_k, q_k, r_k) for k = 1..m, starting from r_0 = 0."""
    x = Fraction(x)
    r = Fraction(0)
    vs, qs, rs = [], [], []
    for _ in range(m):
        v = x + r
        qv = quantizer(v)
        r = v - qv
        vs.append(v)
        qs.append(qv)
        rs.append(r)
    return vs, qs, rs
