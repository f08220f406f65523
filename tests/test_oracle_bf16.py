"""Pins of the oracle's BF16 NT GEMM (no block scales).

Checked against an exact-fraction brute force written here (BF16 values from
their bit fields), exact integer cases against int64 arithmetic, and the
grouped layouts against per-group dense calls.
"""
from fractions import Fraction

import numpy as np
import pytest

import workloads as W


def _bf16_fraction(bits: int) -> Fraction:
    """Exact value of a finite BF16 bit pattern from its fields."""
    s, e, m = bits >> 15, (bits >> 7) & 0xFF, bits & 0x7F
    assert e != 0xFF
    mag = Fraction(m, 128) * Fraction(2) ** -126 if e == 0 else (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
    return -mag if s else mag


def test_bf16_matches_exact_brute_force(oracle_lib):
    p = W.make_bf16_dense(3, 5, 96, seed=1)
    d = oracle_lib.gemm_bf16("dense", p.a, p.b[0], 3, 5, 96)
    for m in range(3):
        for n in range(5):
            exact = sum(_bf16_fraction(int(x)) * _bf16_fraction(int(y)) for x, y in zip(p.a[m], p.b[0, n]))
            assert abs(d[m, n] - float(exact)) <= 1e-14 * max(1.0, abs(float(exact)))


def test_bf16_exact_integers(oracle_lib):
    rng = np.random.default_rng(2)
    M, N, K = 33, 70, 640
    ai = rng.integers(-8, 9, size=(M, K))
    bi = rng.integers(-8, 9, size=(N, K))
    to_bits = lambda v: W._bf16_bits(v.astype(np.float32))
    d = oracle_lib.gemm_bf16("dense", to_bits(ai), to_bits(bi), M, N, K)
    assert np.array_equal(d, (ai @ bi.T).astype(np.float64))


def test_bf16_subnormal_and_signs(oracle_lib):
    # smallest subnormal times 2^126 is 2^-7; signs multiply
    a = np.array([[0x0001, 0x8000, 0x3F80]], np.uint16)      # 2^-133, -0, 1
    b = np.array([[0x7E80, 0x3F80, 0xBF80]], np.uint16)      # 2^126, 1, -1
    d = oracle_lib.gemm_bf16("dense", a, b, 1, 1, 3)
    assert d[0, 0] == 2.0 ** -7 - 1.0


def test_bf16_grouped_equal_per_group_dense(oracle_lib):
    pc = W.make_bf16_contiguous([5, 0, 130], 48, 256, seed=3)
    dc = oracle_lib.gemm_bf16("contiguous", pc.a, pc.b, pc.M, pc.N, pc.K, G=pc.G, m_indices=pc.m_indices)
    for g in range(pc.G):
        rows = np.flatnonzero(pc.m_indices == g)
        if len(rows):
            ref = oracle_lib.gemm_bf16("dense", pc.a[rows], pc.b[g], len(rows), pc.N, pc.K)
            assert np.array_equal(dc[rows], ref)
    assert np.isnan(dc[pc.m_indices < 0]).all()
    pm = W.make_bf16_masked([3, 0, 17], 20, 64, 128, seed=4)
    dm = oracle_lib.gemm_bf16("masked", pm.a, pm.b, pm.M, pm.N, pm.K, G=pm.G, masked_m=pm.masked_m)
    for g in range(pm.G):
        m = pm.masked_m[g]
        if m:
            assert np.array_equal(dm[g, :m], oracle_lib.gemm_bf16("dense", pm.a[g, :m], pm.b[g], m, pm.N, pm.K))
        assert np.isnan(dm[g, m:]).all()
