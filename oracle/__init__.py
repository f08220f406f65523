"""CPU oracle for the FP8 block-scaled NT GEMM (dense / contiguous / masked /
K-grouped) and the per-token 1x128 activation quantiser.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA path.  The arithmetic lives in ``oracle.c`` (plain C, FP64,
OpenMP over output rows); this module compiles it with gcc and marshals numpy
arrays.  ``brute.py`` is a second, pure-Python statement of the same
definition for tiny shapes.

Definition (DeepGEMM pages, page 2 "技术特性" and page 3 "核心功能"):
    D[m,n] = sum_kb sA[m,kb] * sB[n//128,kb] * sum_{k in kb} A[m,k] * B[n,k]
BF16 GEMM (page 3 "核心功能"): D = sum_k A[m,k] * B[n,k], no block scales.
K-grouped (page 3 "核心功能", k_grouped_gemm): group g sums only over its own
ks[g] consecutive K columns, D[g] = the same sum over those K-blocks.
Fused expert FFN (page 5 "03", Mega MoE without its communication): GEMM1 ->
SwiGLU (FP64, rounded to FP32) -> per-token 1x128 quantiser -> GEMM2.
Quantiser (page 2 "技术特性", dynamic fine-grained scaling): per row and
128-wide K-block, s = amax / 448 in FP32, q = E4M3_RNE(clamp(x / s, +-448)).
Every function is pinned (tests/test_oracle.py, tests/test_oracle_quant.py,
tests/test_oracle_mutants.py); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into _oracle.so (gcc, -O3, OpenMP, portable x86-64)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # ORACLE_SO lets the mutation test point the wrapper at a deliberately
        # broken build of oracle.c; it is never set otherwise.
        lib = ctypes.CDLL(os.environ.get("ORACLE_SO") or build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        lib.oracle_e4m3_table.argtypes = [P]
        lib.oracle_e4m3_table.restype = None
        lib.oracle_fp8_gemm_nt.argtypes = [P, P, L, P, P, L, L, L, P]
        lib.oracle_m_grouped_contiguous.argtypes = [P, P, L, P, P, P, L, L, L, L, P]
        lib.oracle_m_grouped_masked.argtypes = [P, P, L, P, P, P, L, L, L, L, P]
        lib.oracle_points.argtypes = [ctypes.c_int, P, P, L, P, P, P, P, L, L, L, L,
                                      L, P, P, P, P]
        for f in ("oracle_fp8_gemm_nt", "oracle_m_grouped_contiguous",
                  "oracle_m_grouped_masked", "oracle_points"):
            getattr(lib, f).restype = ctypes.c_int
        lib.oracle_k_grouped.argtypes = [P, P, L, P, P, P, L, L, L, L, P]
        lib.oracle_k_grouped.restype = ctypes.c_int
        lib.oracle_k_grouped_points.argtypes = [P, P, L, P, P, P, L, L, L, L, L, P, P, P, P]
        lib.oracle_k_grouped_points.restype = ctypes.c_int
        lib.oracle_bf16_gemm_nt.argtypes = [ctypes.c_int, P, P, P, P, L, L, L, L, P]
        lib.oracle_bf16_gemm_nt.restype = ctypes.c_int
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_quantize_1x128.argtypes = [P, L, L, P, P, L]
        lib.oracle_quantize_1x128.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(x: Optional[np.ndarray]):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _c(x, dtype):
    return np.ascontiguousarray(x, dtype=dtype)


def e4m3_table() -> np.ndarray:
    """The oracle's 256-entry E4M3 decode table (float64)."""
    out = np.empty(256, dtype=np.float64)
    _load().oracle_e4m3_table(_p(out))
    return out


def gemm_dense(a, sfa, ld_sfa, b, sfb, M, N, K) -> np.ndarray:
    """Dense D = A * B^T with block scales; returns float64 [M, N]."""
    a, b = _c(a, np.uint8), _c(b, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    d = np.empty((M, N), dtype=np.float64)
    rc = _load().oracle_fp8_gemm_nt(_p(a), _p(sfa), ld_sfa, _p(b), _p(sfb), M, N, K, _p(d))
    if rc:
        raise ValueError(f"oracle_fp8_gemm_nt rejected the shape (rc={rc})")
    return d


def gemm_contiguous(a, sfa, ld_sfa, b, sfb, m_indices, M_total, N, K, G,
                    fill: float = np.nan) -> np.ndarray:
    """M-grouped contiguous; padding rows (m_indices < 0) hold ``fill``."""
    a, b = _c(a, np.uint8), _c(b, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    mi = _c(m_indices, np.int32)
    d = np.full((M_total, N), fill, dtype=np.float64)
    rc = _load().oracle_m_grouped_contiguous(_p(a), _p(sfa), ld_sfa, _p(b), _p(sfb),
                                             _p(mi), M_total, N, K, G, _p(d))
    if rc:
        raise ValueError(f"oracle_m_grouped_contiguous rejected the input (rc={rc})")
    return d


def gemm_masked(a, sfa, ld_sfa, b, sfb, masked_m, G, Mmax, N, K,
                fill: float = np.nan) -> np.ndarray:
    """M-grouped masked; rows >= masked_m[g] hold ``fill``.  Returns [G, Mmax, N]."""
    a, b = _c(a, np.uint8), _c(b, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    mm = _c(masked_m, np.int32)
    d = np.full((G, Mmax, N), fill, dtype=np.float64)
    rc = _load().oracle_m_grouped_masked(_p(a), _p(sfa), ld_sfa, _p(b), _p(sfb), _p(mm),
                                         G, Mmax, N, K, _p(d))
    if rc:
        raise ValueError(f"oracle_m_grouped_masked rejected the input (rc={rc})")
    return d


def gemm_k_grouped(a, sfa, ld_sfa, b, sfb, ks, M, N, K) -> np.ndarray:
    """K-grouped: group g reduces over its ks[g] K columns only; returns
    float64 [G, M, N] (zeros for an empty group)."""
    a, b = _c(a, np.uint8), _c(b, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    ks = _c(ks, np.int32)
    G = len(ks)
    d = np.empty((G, M, N), dtype=np.float64)
    rc = _load().oracle_k_grouped(_p(a), _p(sfa), ld_sfa, _p(b), _p(sfb), _p(ks), G, M, N, K, _p(d))
    if rc:
        raise ValueError(f"oracle_k_grouped rejected the input (rc={rc})")
    return d


def gemm_bf16(layout: str, a_bits, b_bits, M, N, K, G=1, m_indices=None, masked_m=None,
              fill: float = np.nan) -> np.ndarray:
    """BF16 NT GEMM on raw BF16 bit patterns (uint16): dense [M,N],
    contiguous [M_total,N] (padding rows = fill), masked [G,Mmax,N] (rows past
    masked_m = fill).  FP64 accumulation of exact products."""
    a, b = _c(a_bits, np.uint16), _c(b_bits, np.uint16)
    mi = None if m_indices is None else _c(m_indices, np.int32)
    mm = None if masked_m is None else _c(masked_m, np.int32)
    shape = (G, M, N) if layout == "masked" else (M, N)
    d = np.full(shape, fill, dtype=np.float64)
    rc = _load().oracle_bf16_gemm_nt(_LAYOUT_CODE[layout], _p(a), _p(b), _p(mi), _p(mm),
                                     G, M, N, K, _p(d))
    if rc:
        raise ValueError(f"oracle_bf16_gemm_nt rejected the input (rc={rc})")
    return d


def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x) = x / (1 + exp(-x)), float64."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def ffn_rows(prob, rows) -> dict:
    """Fused expert FFN (contiguous layout) for the given valid rows:
    h = block-scaled GEMM1 (FP64), act = silu(gate) * up in FP64, rounded to
    FP32, quantised per 128 columns (s = amax/448, E4M3 codes), y = block-scaled
    GEMM2 of the codes.  Returns h, act (FP32), q, s ([IB, len(rows)]) and y."""
    rows = np.asarray(rows)
    I, H = prob.I, prob.H
    out = {"h": np.empty((len(rows), 2 * I)), "act": np.empty((len(rows), I), np.float32),
           "q": np.empty((len(rows), I), np.uint8), "s": np.empty((I // 128, len(rows)), np.float32),
           "y": np.empty((len(rows), H))}
    groups = prob.m_indices[rows]
    assert (groups >= 0).all(), "padding rows have no FFN output"
    for g in np.unique(groups):
        sel = np.flatnonzero(groups == g)
        r = rows[sel]
        n = len(r)
        ld = (n + 3) // 4 * 4
        sfa = np.zeros((H // 128, ld), np.float32)
        sfa[:, :n] = prob.sfa[:, r]
        h = gemm_dense(prob.a[r], sfa, ld, prob.w1[g], prob.sfb1[g], n, 2 * I, H)
        hb = h.reshape(n, I // 128, 2, 128)
        act = (silu(hb[:, :, 0, :]) * hb[:, :, 1, :]).reshape(n, I).astype(np.float32)
        q, s = quantize_1x128(act, ld_sfa=ld)
        y = gemm_dense(q, s, ld, prob.w2[g], prob.sfb2[g], n, H, I)
        out["h"][sel], out["act"][sel], out["q"][sel], out["s"][:, sel], out["y"][sel] = h, act, q, s[:, :n], y
    return out


_LAYOUT_CODE = {"dense": 0, "contiguous": 1, "masked": 2}


def points(prob, grp, row, col) -> np.ndarray:
    """Sampled outputs D[grp, row, col] of a ``workloads.Problem``."""
    if prob.layout == "k_grouped":
        a, b = _c(prob.a, np.uint8), _c(prob.b[0], np.uint8)
        sfa, sfb = _c(prob.sfa, np.float32), _c(prob.sfb[0], np.float32)
        ks = _c(prob.ks, np.int32)
        grp, row, col = (_c(x, np.int32) for x in (grp, row, col))
        out = np.empty(len(row), dtype=np.float64)
        rc = _load().oracle_k_grouped_points(_p(a), _p(sfa), prob.ld_sfa, _p(b), _p(sfb), _p(ks),
                                             len(ks), prob.M, prob.N, prob.K, len(row),
                                             _p(grp), _p(row), _p(col), _p(out))
        if rc:
            raise ValueError(f"oracle_k_grouped_points rejected the input (rc={rc})")
        return out
    a, b = _c(prob.a, np.uint8), _c(prob.b, np.uint8)
    sfa, sfb = _c(prob.sfa, np.float32), _c(prob.sfb, np.float32)
    mi = None if prob.m_indices is None else _c(prob.m_indices, np.int32)
    mm = None if prob.masked_m is None else _c(prob.masked_m, np.int32)
    grp, row, col = (_c(x, np.int32) for x in (grp, row, col))
    out = np.empty(len(row), dtype=np.float64)
    rc = _load().oracle_points(_LAYOUT_CODE[prob.layout], _p(a), _p(sfa), prob.ld_sfa,
                               _p(b), _p(sfb), _p(mi), _p(mm), prob.G, prob.M, prob.N,
                               prob.K, len(row), _p(grp), _p(row), _p(col), _p(out))
    if rc:
        raise ValueError(f"oracle_points rejected the input (rc={rc})")
    return out


def solve(prob) -> np.ndarray:
    """Full oracle output for a ``workloads.Problem`` (float64, NaN where unwritten)."""
    if prob.layout == "dense":
        return gemm_dense(prob.a, prob.sfa, prob.ld_sfa, prob.b[0], prob.sfb[0],
                          prob.M, prob.N, prob.K)
    if prob.layout == "contiguous":
        return gemm_contiguous(prob.a, prob.sfa, prob.ld_sfa, prob.b, prob.sfb,
                               prob.m_indices, prob.M, prob.N, prob.K, prob.G)
    if prob.layout == "k_grouped":
        return gemm_k_grouped(prob.a, prob.sfa, prob.ld_sfa, prob.b[0], prob.sfb[0], prob.ks,
                              prob.M, prob.N, prob.K)
    return gemm_masked(prob.a, prob.sfa, prob.ld_sfa, prob.b, prob.sfb, prob.masked_m,
                       prob.G, prob.M, prob.N, prob.K)


def e4m3_encode(values) -> np.ndarray:
    """The oracle's E4M3 round-to-nearest-even encoder, element by element."""
    lib = _load()
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib.oracle_e4m3_encode(float(x)) for x in v], dtype=np.uint8)


def quantize_1x128(x: np.ndarray, ld_sfa: Optional[int] = None):
    """Per-token 1x128 quantisation of float32 x [M, K] (the exact BF16 inputs):
    returns (q uint8 [M, K], sfa float32 [KB, ld_sfa])."""
    x = _c(x, np.float32)
    M, K = x.shape
    ld = ld_sfa if ld_sfa is not None else (M + 3) // 4 * 4
    q = np.empty((M, K), dtype=np.uint8)
    sfa = np.zeros((K // 128, ld), dtype=np.float32)
    rc = _load().oracle_quantize_1x128(_p(x), M, K, _p(q), _p(sfa), ld)
    if rc:
        raise ValueError(f"oracle_quantize_1x128 rejected the shape (rc={rc})")
    return q, sfa
