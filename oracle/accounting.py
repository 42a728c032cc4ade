"""Storage accounting for BenQ and MDBF: CPU oracle (test infrastructure only).

* BenQ: "Qwen3.8-27B -- BenQ 6-bit", bits/weight table under "What BenQ
  stores": 6.000 bits of code plus a 64-entry bf16 table per output row,
  amortised over the row's K columns (64 * 16 / K bits per weight).
* MDBF: "MDBF (Multi-Envelope Double Binary Factorization)", section
  "Bit-width and rank" (effective BPW and its inversion for the rank) and the
  note "The matrix shape caps the reachable BPW" (rank clamp and b_max).
"""
from __future__ import annotations

import math
import warnings
from fractions import Fraction


def benq_bits_per_weight(K: int, code_bits: int = 6) -> float:
    """Code bits plus the per-row table (64 bf16 entries) spread over K columns."""
    return code_bits + 64 * 16 / K


def benq_packed_bytes_per_row(K: int) -> int:
    """Bytes of one packed code row: 6 bits per code, 4 codes per 3 bytes."""
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    return 3 * K // 4


def mdbf_b_eff(n: int, m: int, r: int, P: int, l: int, scale_bits: int = 16) -> Fraction:
    """b_eff = P [ r (n+m) + scale_bits * l (n + m + 2r) ] / (n m), exactly."""
    return Fraction(P * (r * (n + m) + scale_bits * l * (n + m + 2 * r)), n * m)


def mdbf_b_max(n: int, m: int, P: int, l: int, scale_bits: int = 16) -> Fraction:
    """b_max = P [ s (s + t) + scale_bits * l (t + 3s) ] / (s t), s = min, t = max."""
    s, t = min(n, m), max(n, m)
    return Fraction(P * (s * (s + t) + scale_bits * l * (t + 3 * s)), s * t)


def mdbf_rank_real(n: int, m: int, b: float, P: int, l: int, scale_bits: int = 16) -> Fraction:
    """r = (b n m / P - scale_bits l (n+m)) / ((n+m) + 2 scale_bits l), as an exact rational."""
    bq = Fraction(b)
    return (bq * n * m / P - scale_bits * l * (n + m)) / ((n + m) + 2 * scale_bits * l)


def mdbf_select_rank(n: int, m: int, b: float, P: int, l: int, scale_bits: int = 16):
    """Integer rank for a target BPW: floor of the inverted formula, clamped to [1, min(n, m)].

    Returns (r, clamped).  A target above b_max lands on r = min(n, m) with a
    warning; a target too small for rank 1 raises ValueError.
    """
    s = min(n, m)
    rr = mdbf_rank_real(n, m, b, P, l, scale_bits)
    r = math.floor(rr)
    if rr > s:
        warnings.warn(f"target {b} bpw exceeds b_max {float(mdbf_b_max(n, m, P, l, scale_bits)):.6f}; "
                      f"rank clamped to {s}")
        return s, True
    if r < 1:
        raise ValueError(f"target {b} bpw is below the cost of rank 1")
    return r, False
