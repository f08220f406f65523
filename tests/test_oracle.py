"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle (oracle/oracle.c through oracle/__init__.py)
against something independent: torch's float8 cast, closed-form E4M3 values,
an exact-fraction brute force, a float64 library matmul, exact integer
arithmetic, identity/zero operands, scale linearity and the grouped ==
per-group-dense invariant.  Shapes are chosen so that a dropped K-block, a
wrong sign, a transposed operand, a row-major/MN-major scale mix-up or an
n % 128 vs n / 128 mix-up fails at least one test.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import brute

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _dequant_torch(q: np.ndarray) -> np.ndarray:
    """E4M3 bytes -> float64 via torch's float8 cast (a library routine)."""
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _rand_bytes(rng, shape):
    """Uniform over all finite E4M3 codes (NaN codes 0x7F / 0xFF excluded)."""
    q = rng.integers(0, 256, size=shape, dtype=np.int64)
    q = np.where((q & 0x7F) == 0x7F, q ^ 0x01, q)
    return q.astype(np.uint8)


def _int_bytes(vals: np.ndarray) -> np.ndarray:
    """Small integers -> E4M3 bytes (exact for |v| <= 16)."""
    return torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# --------------------------------------------------------------------------- decode table
def test_e4m3_table_matches_torch_cast(oracle_lib):
    lut = oracle_lib.e4m3_table()
    ref = _dequant_torch(np.arange(256, dtype=np.uint8))
    nan_l, nan_r = np.isnan(lut), np.isnan(ref)
    assert (nan_l == nan_r).all()
    assert np.array_equal(lut[~nan_l], ref[~nan_r])
    assert np.array_equal(np.signbit(lut[~nan_l]), np.signbit(ref[~nan_r]))


def test_e4m3_table_closed_forms(oracle_lib):
    lut = oracle_lib.e4m3_table()
    assert lut[0x7E] == 448.0 and lut[0xFE] == -448.0          # largest finite
    assert lut[0x01] == 2.0 ** -9                               # smallest subnormal
    assert lut[0x07] == 7 * 2.0 ** -9                           # largest subnormal
    assert lut[0x08] == 2.0 ** -6                               # smallest normal
    assert lut[0x38] == 1.0 and lut[0xB8] == -1.0
    assert lut[0x40] == 2.0 and lut[0x3C] == 1.5
    assert lut[0x00] == 0.0 and not math.copysign(1, lut[0x00]) < 0
    assert lut[0x80] == 0.0 and math.copysign(1, lut[0x80]) < 0
    assert sorted(np.flatnonzero(np.isnan(lut)).tolist()) == [0x7F, 0xFF]
    assert np.isfinite(lut[[c for c in range(256) if c not in (0x7F, 0xFF)]]).all()


# --------------------------------------------------------------------------- brute force
@pytest.mark.parametrize("M,N,K,seed", [(3, 5, 128, 0), (4, 6, 256, 1), (2, 130, 256, 2)])
def test_dense_matches_exact_brute_force(oracle_lib, M, N, K, seed):
    rng = np.random.default_rng(100 + seed)
    a, b = _rand_bytes(rng, (M, K)), _rand_bytes(rng, (N, K))
    KB, NB = K // 128, (N + 127) // 128
    sa = rng.uniform(0.01, 2.0, size=(M, KB)).astype(np.float32)
    sb = rng.uniform(0.01, 2.0, size=(NB, KB)).astype(np.float32)
    d = oracle_lib.gemm_dense(a, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb, M, N, K)
    ref = brute.gemm(a, sa, b, sb, M, N, K)
    for m in range(M):
        for n in range(N):
            exact = float(ref[m][n])
            assert abs(d[m, n] - exact) <= 1e-13 * max(1.0, abs(exact)), (m, n)


# --------------------------------------------------------------------------- textbook reduction
@pytest.mark.parametrize("M,N,K", [(17, 40, 512), (128, 256, 384)])
def test_unit_scales_equal_float64_matmul(oracle_lib, M, N, K):
    """All scales 1: D = dequant(A) @ dequant(B)^T.  Every partial sum is a
    multiple of 2^-18 below 2^27, so both sides are exact and must be equal."""
    rng = np.random.default_rng(7)
    a, b = _rand_bytes(rng, (M, K)), _rand_bytes(rng, (N, K))
    KB, NB = K // 128, (N + 127) // 128
    d = oracle_lib.gemm_dense(a, np.ones((KB, W.tma_aligned(M)), np.float32), W.tma_aligned(M),
                              b, np.ones((NB, KB), np.float32), M, N, K)
    ref = _dequant_torch(a) @ _dequant_torch(b).T
    assert np.array_equal(d, ref)


# --------------------------------------------------------------------------- exact integers
def _exact_case(seed, M, N, K):
    rng = np.random.default_rng(seed)
    KB, NB = K // 128, (N + 127) // 128
    ai = rng.integers(-2, 3, size=(M, K))
    bi = rng.integers(-2, 3, size=(N, K))
    ea = rng.integers(-3, 4, size=(M, KB))          # distinct powers of two per (m, kb)
    eb = rng.integers(-3, 4, size=(NB, KB))         # and per (n-block, kb)
    sa = np.ldexp(1.0, ea).astype(np.float32)
    sb = np.ldexp(1.0, eb).astype(np.float32)
    exact = np.zeros((M, N), dtype=np.float64)
    for kb in range(KB):
        sl = slice(kb * 128, kb * 128 + 128)
        p = ai[:, sl] @ bi[:, sl].T                                   # int64, exact
        scale = sa[:, kb].astype(np.float64)[:, None] * sb[np.arange(N) // 128, kb].astype(np.float64)[None, :]
        exact += scale * p
    return _int_bytes(ai), sa, _int_bytes(bi), sb, exact


@pytest.mark.parametrize("M,N,K", [(5, 200, 384), (130, 72, 256)])
def test_exact_integer_operands_power_of_two_scales(oracle_lib, M, N, K):
    a, sa, b, sb, exact = _exact_case(11, M, N, K)
    d = oracle_lib.gemm_dense(a, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb, M, N, K)
    assert np.array_equal(d, exact)


def test_identity_and_zero(oracle_lib):
    K = N = 256
    M = 256
    rng = np.random.default_rng(3)
    b = _rand_bytes(rng, (N, K))
    sa = rng.uniform(0.5, 2, size=(M, K // 128)).astype(np.float32)
    sb = rng.uniform(0.5, 2, size=(N // 128, K // 128)).astype(np.float32)
    eye = np.zeros((M, K), np.uint8)
    eye[np.arange(M), np.arange(M)] = 0x38                      # E4M3 1.0
    d = oracle_lib.gemm_dense(eye, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb, M, N, K)
    bd = _dequant_torch(b)
    m = np.arange(M)[:, None]
    n = np.arange(N)[None, :]
    expect = sa[m, m // 128].astype(np.float64) * sb[n // 128, m // 128].astype(np.float64) * bd[n, m]
    assert np.array_equal(d, expect)
    z = oracle_lib.gemm_dense(np.zeros((M, K), np.uint8), W.sfa_mn_major(sa), W.tma_aligned(M),
                              b, sb, M, N, K)
    assert (z == 0).all() and not np.signbit(z).any()


# --------------------------------------------------------------------------- scale linearity
def test_scale_linearity(oracle_lib):
    M, N, K = 6, 300, 384
    rng = np.random.default_rng(5)
    a, b = _rand_bytes(rng, (M, K)), _rand_bytes(rng, (N, K))
    sa = rng.uniform(0.1, 1, size=(M, 3)).astype(np.float32)
    sb = rng.uniform(0.1, 1, size=(3, 3)).astype(np.float32)
    base = oracle_lib.gemm_dense(a, W.sfa_mn_major(sa), 8, b, sb, M, N, K)
    sa2 = sa.copy()
    sa2[2] *= 2
    d2 = oracle_lib.gemm_dense(a, W.sfa_mn_major(sa2), 8, b, sb, M, N, K)
    assert np.array_equal(d2[2], 2 * base[2])
    assert np.array_equal(np.delete(d2, 2, 0), np.delete(base, 2, 0))
    # scaling sB[j=1, kb=2] by c changes only columns 128..255, by (c-1)*sA*sB*P_kb
    c = 3.0
    sb3 = sb.copy()
    sb3[1, 2] *= c
    d3 = oracle_lib.gemm_dense(a, W.sfa_mn_major(sa), 8, b, sb3, M, N, K)
    cols = np.arange(N)
    out = (cols < 128) | (cols >= 256)
    assert np.array_equal(d3[:, out], base[:, out])
    p = _dequant_torch(a[:, 256:384]) @ _dequant_torch(b[128:256, 256:384]).T
    want = (c - 1) * sa[:, 2:3].astype(np.float64) * np.float64(sb[1, 2]) * p
    np.testing.assert_allclose(d3[:, 128:256] - base[:, 128:256], want, rtol=1e-9, atol=1e-9)


# --------------------------------------------------------------------------- grouped layouts
def test_contiguous_equals_per_group_dense(oracle_lib):
    prob = W.make_contiguous([130, 0, 5, 256], N=192, K=256, seed=9)
    d = oracle_lib.solve(prob)
    for g in range(prob.G):
        rows = np.flatnonzero(prob.m_indices == g)
        if len(rows) == 0:
            continue
        sa_rows = prob.sfa[:, rows]
        ref = oracle_lib.gemm_dense(prob.a[rows], np.ascontiguousarray(sa_rows), len(rows),
                                    prob.b[g], prob.sfb[g], len(rows), prob.N, prob.K)
        assert np.array_equal(d[rows], ref)
    pad = prob.m_indices < 0
    assert np.isnan(d[pad]).all()                  # padding rows are not written
    assert np.isfinite(d[~pad]).all()              # NaN padding never leaks


def test_contiguous_with_whole_padding_blocks(oracle_lib):
    """Whole padding blocks between groups change nothing for the groups' rows:
    the same groups without the gaps give the same outputs, and padding rows
    stay unwritten."""
    gapped = W.make_contiguous([200, 100, 300], N=136, K=256, seed=6, gaps=[2, 0, 1])
    plain = W.make_contiguous([200, 100, 300], N=136, K=256, seed=6)
    d, e = oracle_lib.solve(gapped), oracle_lib.solve(plain)
    for g in range(3):
        assert np.array_equal(d[gapped.m_indices == g], e[plain.m_indices == g])
    assert np.isnan(d[gapped.m_indices < 0]).all()


def test_masked_equals_per_group_dense(oracle_lib):
    prob = W.make_masked([0, 7, 64, 65], Mmax=64 + 16, N=160, K=256, seed=4)
    d = oracle_lib.solve(prob)
    for g in range(prob.G):
        m = int(prob.masked_m[g])
        if m:
            ref = oracle_lib.gemm_dense(prob.a[g, :m], np.ascontiguousarray(prob.sfa[g][:, :m]), m,
                                        prob.b[g], prob.sfb[g], m, prob.N, prob.K)
            assert np.array_equal(d[g, :m], ref)
            assert np.isfinite(d[g, :m]).all()
        assert np.isnan(d[g, m:]).all()


def test_points_equal_full(oracle_lib):
    for prob in (W.make_dense(40, 200, 256, seed=1),
                 W.make_contiguous([3, 200], N=136, K=128, seed=2),
                 W.make_masked([5, 0, 33], Mmax=48, N=64, K=256, seed=3)):
        full = oracle_lib.solve(prob)
        rng = np.random.default_rng(0)
        n = 50
        row = rng.integers(0, prob.M, n)
        col = rng.integers(0, prob.N, n)
        grp = rng.integers(0, prob.G, n)
        pts = oracle_lib.points(prob, grp, row, col)
        ref = full[grp, row, col] if prob.layout == "masked" else full[row, col]
        assert np.array_equal(np.isnan(pts), np.isnan(ref))
        assert np.array_equal(pts[~np.isnan(pts)], ref[~np.isnan(ref)])


def test_oracle_rejects_bad_shapes(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.gemm_dense(np.zeros((2, 100), np.uint8), np.zeros((1, 4), np.float32), 4,
                              np.zeros((2, 100), np.uint8), np.zeros((1, 1), np.float32), 2, 2, 100)


# --------------------------------------------------------------------------- k-grouped
def test_k_grouped_brute_force(oracle_lib):
    """Each group equals the exact brute force over its own K columns (a
    second statement of the definition, with the K slicing done here)."""
    rng = np.random.default_rng(301)
    M, N, ks = 3, 130, np.array([128, 0, 256], np.int32)
    K = int(ks.sum())
    a, b = _rand_bytes(rng, (M, K)), _rand_bytes(rng, (N, K))
    KB, NB = K // 128, (N + 127) // 128
    sa = rng.uniform(0.01, 2.0, size=(M, KB)).astype(np.float32)
    sb = rng.uniform(0.01, 2.0, size=(NB, KB)).astype(np.float32)
    d = oracle_lib.gemm_k_grouped(a, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb, ks, M, N, K)
    off = 0
    for g, kg in enumerate(ks):
        c0, c1, b0, b1 = off, off + kg, off // 128, (off + kg) // 128
        if kg == 0:
            assert (d[g] == 0).all()
        else:
            ref = brute.gemm(a[:, c0:c1], sa[:, b0:b1], b[:, c0:c1], sb[:, b0:b1], M, N, int(kg))
            for m in range(M):
                for n in range(N):
                    assert abs(d[g, m, n] - float(ref[m][n])) <= 1e-13 * max(1.0, abs(float(ref[m][n])))
        off += kg


def test_k_grouped_sums_to_dense_exactly(oracle_lib):
    """Linearity over K: the groups' outputs add up to the dense GEMM over all
    of K -- exactly, with integer operands and power-of-two scales."""
    M, N, K = 6, 136, 768
    a, sa, b, sb, exact = _exact_case(23, M, N, K)
    ks = np.array([256, 128, 0, 384], np.int32)
    d = oracle_lib.gemm_k_grouped(a, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb, ks, M, N, K)
    assert d.shape == (4, M, N)
    assert np.array_equal(d.sum(axis=0), exact)
    assert (d[2] == 0).all()
    one = oracle_lib.gemm_k_grouped(a, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb,
                                    np.array([K], np.int32), M, N, K)
    assert np.array_equal(one[0], oracle_lib.gemm_dense(a, W.sfa_mn_major(sa), W.tma_aligned(M), b, sb, M, N, K))


def test_k_grouped_points_and_rejections(oracle_lib):
    p = W.make_k_grouped([256, 128, 384], 40, 200, seed=5)
    full = oracle_lib.solve(p)
    rng = np.random.default_rng(0)
    g, r, c = rng.integers(0, 3, 50), rng.integers(0, 40, 50), rng.integers(0, 200, 50)
    assert np.array_equal(oracle_lib.points(p, g, r, c), full[g, r, c])
    with pytest.raises(ValueError):      # group sizes must be multiples of 128
        oracle_lib.gemm_k_grouped(p.a, p.sfa, p.ld_sfa, p.b[0], p.sfb[0], [200, 184, 384], 40, 200, 768)
    with pytest.raises(ValueError):      # and add up to K
        oracle_lib.gemm_k_grouped(p.a, p.sfa, p.ld_sfa, p.b[0], p.sfb[0], [256, 128, 256], 40, 200, 768)
