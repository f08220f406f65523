"""Pure-Python brute force of the block-scaled FP8 NT GEMM, for tiny shapes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  A second statement of
the definition (DeepGEMM pages, page 2 "技术特性": per-K-block partial sums
promoted with the fine-grained scales), written independently of
``oracle.c``: the E4M3 value of a byte comes from Python's own float
arithmetic on the bit fields as exact fractions, and every sum is an explicit
Python loop over exact ``fractions.Fraction`` values, so the result carries
no rounding at all.
"""
from __future__ import annotations

from fractions import Fraction


def e4m3_value(code: int) -> Fraction:
    """Exact value of an E4M3 ("fn") byte; raises on the NaN codes."""
    s, e, m = code >> 7, (code >> 3) & 0xF, code & 7
    if e == 15 and m == 7:
        raise ValueError("NaN code")
    if e == 0:
        mag = Fraction(m, 8) * Fraction(2) ** (-6)
    else:
        mag = (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -mag if s else mag


def gemm(a, sa, b, sb, M: int, N: int, K: int):
    """Exact D (list of lists of Fraction).

    a: [M][K] bytes, sa: [M][KB] floats (row-major per row!), b: [N][K] bytes,
    sb: [NB][KB] floats.  Note the row-major sa here, unlike the C ABI's
    MN-major storage, so a mix-up of the two shows up as a mismatch."""
    KB = K // 128
    out = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            total = Fraction(0)
            for kb in range(KB):
                part = Fraction(0)
                for k in range(kb * 128, kb * 128 + 128):
                    part += e4m3_value(int(a[m][k])) * e4m3_value(int(b[n][k]))
                total += Fraction(float(sa[m][kb])) * Fraction(float(sb[n // 128][kb])) * part
            out[m][n] = total
    return out
