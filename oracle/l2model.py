"""Eq.(1) of "Fleet: Hierarchical Task-based Abstraction for Megakernels on
Multi-Die GPUs" (reading notes, section 3f "Solution Justification"), written
out as plain arithmetic.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Under M-major cooperative traversal, R workers share one weight column tile:

    m_tiles = ceil(B / T_M),   R = min(W, m_tiles)
    hit_weight = (R - 1) / R = 1 - 1 / R                      (Eq. 1)

and the effective arithmetic intensity against HBM (same section, Figure 7
discussion) is

    AI_eff = B / (1 - hit).

``B`` is the batch (the GEMM's M), ``W`` the number of workers that can share a
column at once and ``T_M`` the M-tile height.  On B200 the library applies it
with W = the number of CTAs that can run the m-tiles of one column
concurrently, which is never the binding term at M <= 64.
"""
from __future__ import annotations

from fractions import Fraction


def m_tiles(B: int, T_M: int) -> int:
    if B < 1 or T_M < 1:
        raise ValueError("B and T_M must be positive")
    return -(-B // T_M)


def sharers(B: int, W: int, T_M: int) -> int:
    """R = min(W, ceil(B / T_M))."""
    if W < 1:
        raise ValueError("W must be positive")
    return min(W, m_tiles(B, T_M))


def weight_hit(B: int, W: int, T_M: int) -> Fraction:
    """Eq.(1): predicted L2 hit fraction of weight reads, as an exact fraction."""
    R = sharers(B, W, T_M)
    return Fraction(R - 1, R)


def ai_eff(B: int, hit) -> float:
    """AI_eff = B / (1 - hit); infinite when every weight read hits."""
    hit = Fraction(hit)
    if hit >= 1:
        return float("inf")
    return float(Fraction(B) / (1 - hit))


def hbm_weight_bytes(weight_bytes: int, B: int, W: int, T_M: int) -> Fraction:
    """Weight bytes that still come from HBM when R sharers read each column:
    (1 - hit) * R * weight_bytes = weight_bytes (one fetch per column)."""
    R = sharers(B, W, T_M)
    return (1 - weight_hit(B, W, T_M)) * R * weight_bytes
