"""Seeded synthetic inputs for the FP8 block-scaled NT GEMM.

This module is shared by the oracle side and the CUDA side of the tests and by
``bench.py``.  It draws random numbers and packs them into the storage formats
the library consumes; it holds none of the GEMM's arithmetic (no E4M3 decode,
no dot products, no promotion).  The FP8 encoding of a float uses torch's own
``float8_e4m3fn`` cast (round-to-nearest-even, OCP E4M3 "fn" format), a library
primitive.

Storage formats (shared with the C ABI):

* ``a``   uint8 E4M3 bytes, [rows, K] row-major (K-major).
* ``sfa`` float32 [KB, ld_sfa] "MN-major": for K-block kb, one float per row;
  ``ld_sfa`` = rows rounded up to a multiple of 4 (16-byte TMA alignment).
  Masked layout: [G, KB, ld_sfa].
* ``b``   uint8 E4M3 bytes, [G, N, K] row-major (G = 1 for dense).
* ``sfb`` float32 [G, NB, KB] row-major, one float per 128x128 block.

Quantisation recipe (the pages only say "fine-grained" / "block-wise" scaling,
DeepGEMM pages 2 and 3 "技术特性" / "精细粒度缩放"; the 1x128 and 128x128 block
shapes come from the workload definitions): per block, s = amax / 448 in FP32
(s = 1 when the block is all zero), q = e4m3_rne(clamp(x / s, -448, 448)).

Random streams use ``numpy.random.default_rng`` (PCG64).  Dense: A, then B,
then the outlier columns, all from ``seed``.  Grouped layouts: the structure
(multinomial token counts, masked counts) comes from ``seed`` because it fixes
the operand shapes; A and then B come from ``seed + 1000``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

BLOCK = 128            # K-block and weight-block edge
E4M3_MAX = 448.0
NAN_BYTE = 0x7F        # an E4M3 NaN code, used to poison padding rows
ALIGN_M = 128          # row alignment of the contiguous layout


def tma_aligned(n: int, elem_bytes: int = 4) -> int:
    """Round n up so that n * elem_bytes is a multiple of 16 bytes."""
    q = 16 // elem_bytes
    return (n + q - 1) // q * q


def _to_e4m3_bytes(x: torch.Tensor) -> torch.Tensor:
    x = torch.clamp(x, -E4M3_MAX, E4M3_MAX)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def quantize_rows_1x128(x: np.ndarray):
    """Per-row, per-128-K block quantisation.  x: float32 [R, K].

    Returns (q uint8 [R, K], s float32 [R, KB])."""
    R, K = x.shape
    assert K % BLOCK == 0
    t = torch.from_numpy(x).view(R, K // BLOCK, BLOCK)
    amax = t.abs().amax(dim=2)
    s = amax / E4M3_MAX
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = _to_e4m3_bytes(t / s.unsqueeze(2)).reshape(R, K)
    return q.numpy(), s.numpy().astype(np.float32)


def quantize_blocks_128x128(x: np.ndarray):
    """Per-128x128 block quantisation.  x: float32 [N, K] (N may have a tail).

    Returns (q uint8 [N, K], s float32 [NB, KB])."""
    N, K = x.shape
    assert K % BLOCK == 0
    NB, KB = (N + BLOCK - 1) // BLOCK, K // BLOCK
    t = torch.from_numpy(x)
    pad = NB * BLOCK - N
    tp = torch.nn.functional.pad(t, (0, 0, 0, pad)) if pad else t
    blk = tp.view(NB, BLOCK, KB, BLOCK)
    amax = blk.abs().amax(dim=(1, 3))                  # [NB, KB]
    s = amax / E4M3_MAX
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = _to_e4m3_bytes(blk / s[:, None, :, None]).reshape(NB * BLOCK, K)[:N]
    return q.contiguous().numpy(), s.numpy().astype(np.float32)


def sfa_mn_major(s_rows: np.ndarray, ld: Optional[int] = None) -> np.ndarray:
    """[R, KB] per-row scales -> [KB, ld] MN-major storage (padding = 0)."""
    R, KB = s_rows.shape
    ld = tma_aligned(R) if ld is None else ld
    out = np.zeros((KB, ld), dtype=np.float32)
    out[:, :R] = s_rows.T
    return out


@dataclasses.dataclass
class Problem:
    """One GEMM problem in the library's storage formats (host numpy arrays)."""
    layout: str                    # "dense" | "contiguous" | "masked" | "k_grouped"
    M: int                         # dense, k_grouped: rows; contiguous: M_total; masked: Mmax
    N: int
    K: int
    G: int
    a: np.ndarray                  # uint8
    sfa: np.ndarray                # float32
    ld_sfa: int
    b: np.ndarray                  # uint8 [G, N, K]
    sfb: np.ndarray                # float32 [G, NB, KB]
    m_indices: Optional[np.ndarray] = None   # int32 [M_total] (contiguous)
    masked_m: Optional[np.ndarray] = None    # int32 [G] (masked)
    name: str = ""
    ks: Optional[np.ndarray] = None          # int32 [G] (k_grouped: K columns per group)

    @property
    def KB(self) -> int:
        return self.K // BLOCK

    @property
    def NB(self) -> int:
        return (self.N + BLOCK - 1) // BLOCK

    def valid_rows(self) -> int:
        if self.layout in ("dense", "k_grouped"):
            return self.M
        if self.layout == "contiguous":
            return int((self.m_indices >= 0).sum())
        return int(self.masked_m.sum())

    def groups_touched(self) -> int:
        if self.layout in ("dense", "k_grouped"):
            return 1
        if self.layout == "contiguous":
            return int(len(np.unique(self.m_indices[self.m_indices >= 0])))
        return int((self.masked_m > 0).sum())

    def flops(self) -> float:
        """Algorithmic FLOP: 2 * valid rows * N * K."""
        return 2.0 * self.valid_rows() * self.N * self.K

    def bytes(self) -> float:
        """Algorithmic bytes: A + B + sA + sB + D over valid rows / touched groups
        (k_grouped: A, B and their scales once, one D per group)."""
        rows, g = self.valid_rows(), self.groups_touched()
        if self.layout == "k_grouped":
            return float(rows * self.K + self.N * self.K + rows * self.KB * 4
                         + self.NB * self.KB * 4 + self.G * rows * self.N * 2)
        return float(rows * self.K + g * self.N * self.K + rows * self.KB * 4
                     + g * self.NB * self.KB * 4 + rows * self.N * 2)

    def d_shape(self):
        if self.layout in ("masked", "k_grouped"):
            return (self.G, self.M, self.N)
        return (self.M, self.N)


def _normal(rng, shape):
    return rng.standard_normal(shape, dtype=np.float32)


def make_dense(M: int, N: int, K: int, seed: int, outliers: bool = False,
               name: str = "") -> Problem:
    """Dense problem: A ~ N(0,1) [M,K], B ~ N(0,1) [N,K].

    With ``outliers``, one fixed set of floor(0.01*K) K-columns of A (drawn
    after A and B) is multiplied by 20 before quantisation."""
    rng = np.random.default_rng(seed)
    a32 = _normal(rng, (M, K))
    b32 = _normal(rng, (N, K))
    if outliers:
        cols = rng.choice(K, size=K // 100, replace=False)
        a32[:, cols] *= 20.0
    qa, sa = quantize_rows_1x128(a32) if M > 0 else (np.zeros((0, K), np.uint8),
                                                     np.zeros((0, K // BLOCK), np.float32))
    qb, sb = quantize_blocks_128x128(b32)
    ld = tma_aligned(max(M, 1))
    return Problem("dense", M, N, K, 1, qa, sfa_mn_major(sa, ld), ld,
                   qb[None], sb[None], name=name)


def make_contiguous(counts, N: int, K: int, seed: int, name: str = "",
                    poison: bool = True, gaps=None) -> Problem:
    """M-grouped contiguous problem with explicit per-group token counts.

    Group g's rows are packed back to back and padded to a multiple of 128;
    padding rows carry m_indices = -1, NaN bytes in A and NaN scales.
    ``gaps[g]`` whole 128-row blocks of padding follow group g's rows (a
    caller's fixed-size buffer with unused blocks)."""
    rng = np.random.default_rng(seed)
    counts = [int(c) for c in counts]
    G = len(counts)
    gaps = [0] * G if gaps is None else [int(x) for x in gaps]
    padded = [(c + ALIGN_M - 1) // ALIGN_M * ALIGN_M + ALIGN_M * x for c, x in zip(counts, gaps)]
    M_total = int(sum(padded))
    a32 = _normal(rng, (sum(counts), K))
    b32 = _normal(rng, (G * N, K))
    m_idx = np.full((M_total,), -1, dtype=np.int32)
    qa_all, sa_all = (quantize_rows_1x128(a32) if a32.shape[0] else
                      (np.zeros((0, K), np.uint8), np.zeros((0, K // BLOCK), np.float32)))
    a = np.full((M_total, K), NAN_BYTE if poison else 0, dtype=np.uint8)
    sa = np.full((M_total, K // BLOCK), np.nan if poison else 0.0, dtype=np.float32)
    src = dst = 0
    for g, (c, p) in enumerate(zip(counts, padded)):
        a[dst:dst + c] = qa_all[src:src + c]
        sa[dst:dst + c] = sa_all[src:src + c]
        m_idx[dst:dst + c] = g
        src += c
        dst += p
    qb = np.empty((G, N, K), dtype=np.uint8)
    NB = (N + BLOCK - 1) // BLOCK
    sb = np.empty((G, NB, K // BLOCK), dtype=np.float32)
    for g in range(G):
        qb[g], sb[g] = quantize_blocks_128x128(b32[g * N:(g + 1) * N])
    ld = tma_aligned(max(M_total, 1))
    sfa = sfa_mn_major(sa, ld)
    if poison:
        sfa[:, M_total:] = np.nan
    return Problem("contiguous", M_total, N, K, G, a, sfa, ld, qb, sb,
                   m_indices=m_idx, name=name)


def make_contiguous_multinomial(G: int, tokens: int, N: int, K: int, seed: int,
                                name: str = "") -> Problem:
    """Token counts per expert from multinomial(tokens, [1/G]*G) drawn from a
    generator seeded with ``seed`` before the operands (structure first here
    because the counts fix the operand shapes); operands then come from
    ``seed + 1000``."""
    rng = np.random.default_rng(seed)
    counts = rng.multinomial(tokens, [1.0 / G] * G)
    return make_contiguous(counts, N, K, seed + 1000, name=name)


def make_masked(masked_m, Mmax: int, N: int, K: int, seed: int, name: str = "",
                poison: bool = True) -> Problem:
    """M-grouped masked problem: A [G, Mmax, K], valid rows m < masked_m[g].

    Rows >= masked_m[g] carry NaN bytes and NaN scales."""
    rng = np.random.default_rng(seed)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = len(masked_m)
    a32 = _normal(rng, (G * Mmax, K))
    b32 = _normal(rng, (G * N, K))
    qa, sa = quantize_rows_1x128(a32)
    qa = qa.reshape(G, Mmax, K)
    sa = sa.reshape(G, Mmax, K // BLOCK)
    ld = tma_aligned(Mmax)
    sfa = np.zeros((G, K // BLOCK, ld), dtype=np.float32)
    for g in range(G):
        sfa[g, :, :Mmax] = sa[g].T
        if poison:
            qa[g, masked_m[g]:] = NAN_BYTE
            sfa[g, :, masked_m[g]:] = np.nan
    qb = np.empty((G, N, K), dtype=np.uint8)
    NB = (N + BLOCK - 1) // BLOCK
    sb = np.empty((G, NB, K // BLOCK), dtype=np.float32)
    for g in range(G):
        qb[g], sb[g] = quantize_blocks_128x128(b32[g * N:(g + 1) * N])
    return Problem("masked", Mmax, N, K, G, qa, sfa, ld, qb, sb,
                   masked_m=masked_m, name=name)


def make_masked_uniform(G: int, Mmax: int, N: int, K: int, seed: int,
                        name: str = "") -> Problem:
    """masked_m[g] ~ Uniform{0..Mmax} from ``seed``; operands from seed+1000."""
    rng = np.random.default_rng(seed)
    masked_m = rng.integers(0, Mmax + 1, size=G).astype(np.int32)
    return make_masked(masked_m, Mmax, N, K, seed + 1000, name=name)


def make_k_grouped(ks, M: int, N: int, seed: int, name: str = "", outliers: bool = False) -> Problem:
    """K-grouped problem: group g owns ks[g] consecutive K columns (multiples
    of 128) of A [M, K] and B [N, K], K = sum(ks); D is [G, M, N].  A and B ~
    N(0,1), quantised like the dense layout (1x128 rows of A, 128x128 blocks
    of B), so each group's K-blocks carry their own scales."""
    ks = np.asarray(ks, dtype=np.int32)
    K = int(ks.sum())
    assert K > 0 and (ks % BLOCK == 0).all() and (ks >= 0).all()
    p = make_dense(M, N, K, seed, outliers=outliers, name=name)
    return Problem("k_grouped", M, N, K, len(ks), p.a, p.sfa, p.ld_sfa, p.b, p.sfb,
                   name=name, ks=ks)


def make_k_grouped_multinomial(G: int, tokens: int, M: int, N: int, seed: int,
                               name: str = "") -> Problem:
    """Tokens per expert from multinomial(tokens, [1/G]*G) drawn from ``seed``,
    each rounded up to a multiple of 128 (the K alignment); operands from
    seed+1000."""
    rng = np.random.default_rng(seed)
    counts = rng.multinomial(tokens, [1.0 / G] * G)
    ks = ((counts + BLOCK - 1) // BLOCK * BLOCK).astype(np.int32)
    return make_k_grouped(ks, M, N, seed + 1000, name=name)


# The five workloads of the method's benchmark set (shapes from the pages'
# benchmark table, DeepGEMM page 2 "性能实测", plus the expert counts).
WORKLOADS = {
    "dense_tiny": dict(kind="dense", M=128, N=256, K=512, seed=0),
    "dense_decode_m64": dict(kind="dense", M=64, N=2112, K=7168, seed=1, outliers=True),
    "dense_decode_m128": dict(kind="dense", M=128, N=2112, K=7168, seed=2, outliers=True),
    "dense_large": dict(kind="dense", M=4096, N=7168, K=16384, seed=3),
    "contiguous_g4": dict(kind="contiguous", G=4, tokens=32768, N=4096, K=7168, seed=4),
    "masked_g16": dict(kind="masked", G=16, Mmax=256, N=4096, K=7168, seed=5),
    # weight-gradient shape of MoE training: 4 experts, 32768 tokens along K
    "kgrouped_g4": dict(kind="k_grouped", G=4, tokens=32768, M=4096, N=7168, seed=9),
}


def make_workload(name: str) -> Problem:
    w = dict(WORKLOADS[name])
    kind = w.pop("kind")
    if kind == "dense":
        return make_dense(name=name, **w)
    if kind == "contiguous":
        return make_contiguous_multinomial(w["G"], w["tokens"], w["N"], w["K"], w["seed"], name=name)
    if kind == "k_grouped":
        return make_k_grouped_multinomial(w["G"], w["tokens"], w["M"], w["N"], w["seed"], name=name)
    return make_masked_uniform(w["G"], w["Mmax"], w["N"], w["K"], w["seed"], name=name)


# ----------------------------------------------------------------------------- quantiser inputs
@dataclasses.dataclass
class QuantProblem:
    """Inputs of the per-token 1x128 quantiser: BF16 activations, held here as
    their exact float32 values.  Dense: x [M, K]; masked: x [G, Mmax, K] with
    valid rows m < masked_m[g] (the other rows hold NaN, which the quantiser
    must never read)."""
    layout: str
    x: np.ndarray
    masked_m: Optional[np.ndarray] = None
    name: str = ""

    @property
    def K(self) -> int:
        return int(self.x.shape[-1])

    @property
    def KB(self) -> int:
        return self.K // BLOCK

    @property
    def G(self) -> int:
        return 1 if self.layout == "dense" else int(self.x.shape[0])

    @property
    def M(self) -> int:
        """Rows per group (dense: M; masked: Mmax)."""
        return int(self.x.shape[-2])

    @property
    def ld_sfa(self) -> int:
        return tma_aligned(max(self.M, 1))

    def valid_rows(self) -> int:
        return self.M if self.layout == "dense" else int(self.masked_m.sum())

    def bytes(self) -> float:
        """Algorithmic bytes: BF16 in, E4M3 out, one FP32 scale per 128 out."""
        return float(self.valid_rows()) * (2 * self.K + self.K + 4 * self.KB)

    def x_bf16(self) -> torch.Tensor:
        return torch.from_numpy(np.ascontiguousarray(self.x)).to(torch.bfloat16)


def _bf16_exact(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x32).to(torch.bfloat16).to(torch.float32).numpy()


def _activations(rng, rows: int, K: int, outliers: bool) -> np.ndarray:
    x = _normal(rng, (rows, K))
    if outliers:
        cols = rng.choice(K, size=K // 100, replace=False)
        x[:, cols] *= 20.0
    return _bf16_exact(x)


def make_activations(M: int, K: int, seed: int, outliers: bool = True, name: str = "") -> QuantProblem:
    """Dense activations x [M, K]: N(0,1), one fixed set of floor(0.01*K)
    outlier columns x20 (as the GEMM workloads' A), rounded to BF16."""
    rng = np.random.default_rng(seed)
    return QuantProblem("dense", _activations(rng, M, K, outliers), name=name)


def make_activations_masked(masked_m, Mmax: int, K: int, seed: int, outliers: bool = True,
                            name: str = "", poison: bool = True) -> QuantProblem:
    """Masked activations x [G, Mmax, K]; rows >= masked_m[g] are NaN."""
    rng = np.random.default_rng(seed)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = len(masked_m)
    x = _activations(rng, G * Mmax, K, outliers).reshape(G, Mmax, K)
    if poison:
        for g in range(G):
            x[g, masked_m[g]:] = np.nan
    return QuantProblem("masked", x, masked_m=masked_m, name=name)


def make_activations_masked_uniform(G: int, Mmax: int, K: int, seed: int,
                                    name: str = "") -> QuantProblem:
    """masked_m[g] ~ Uniform{0..Mmax} from ``seed``; values from seed+1000."""
    rng = np.random.default_rng(seed)
    masked_m = rng.integers(0, Mmax + 1, size=G).astype(np.int32)
    return make_activations_masked(masked_m, Mmax, K, seed + 1000, name=name)


# Quantiser workloads: the activations that feed the contiguous prefill GEMM
# (32768 tokens, K = 7168) and the masked decode GEMM (16 groups, Mmax 256).
QUANT_WORKLOADS = {
    "quant_tiny": dict(kind="dense", M=130, K=640, seed=8),
    "quant_tokens_32768": dict(kind="dense", M=32768, K=7168, seed=6),
    "quant_masked_g16": dict(kind="masked", G=16, Mmax=256, K=7168, seed=7),
}


def make_quant_workload(name: str, seed_offset: int = 0) -> QuantProblem:
    w = dict(QUANT_WORKLOADS[name])
    kind = w.pop("kind")
    seed = w.pop("seed") + seed_offset
    if kind == "dense":
        return make_activations(w["M"], w["K"], seed, name=name)
    return make_activations_masked_uniform(w["G"], w["Mmax"], w["K"], seed, name=name)


# ----------------------------------------------------------------------------- BF16 GEMM inputs
BF16_NAN_BITS = 0x7FC0    # a BF16 NaN pattern, used to poison rows that must not be read


@dataclasses.dataclass
class BF16Problem:
    """One BF16 NT GEMM problem (no block scales): raw BF16 bit patterns.
    a: uint16 [rows, K] (masked: [G, Mmax, K]); b: uint16 [G, N, K]."""
    layout: str                    # "dense" | "contiguous" | "masked"
    M: int                         # dense: rows; contiguous: M_total; masked: Mmax
    N: int
    K: int
    G: int
    a: np.ndarray
    b: np.ndarray
    m_indices: Optional[np.ndarray] = None
    masked_m: Optional[np.ndarray] = None
    name: str = ""

    def valid_rows(self) -> int:
        if self.layout == "dense":
            return self.M
        if self.layout == "contiguous":
            return int((self.m_indices >= 0).sum())
        return int(self.masked_m.sum())

    def groups_touched(self) -> int:
        if self.layout == "dense":
            return 1
        if self.layout == "contiguous":
            return int(len(np.unique(self.m_indices[self.m_indices >= 0])))
        return int((self.masked_m > 0).sum())

    def flops(self) -> float:
        return 2.0 * self.valid_rows() * self.N * self.K

    def bytes(self) -> float:
        """Algorithmic bytes: A and D over valid rows, B of the touched groups."""
        rows, g = self.valid_rows(), self.groups_touched()
        return float(2 * rows * self.K + 2 * g * self.N * self.K + 2 * rows * self.N)

    def d_shape(self):
        if self.layout == "masked":
            return (self.G, self.M, self.N)
        return (self.M, self.N)


def _bf16_bits(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def make_bf16_dense(M: int, N: int, K: int, seed: int, name: str = "") -> BF16Problem:
    """A ~ N(0,1) [M,K], B ~ N(0,1) [N,K], rounded to BF16."""
    rng = np.random.default_rng(seed)
    a = _bf16_bits(_normal(rng, (M, K)))
    b = _bf16_bits(_normal(rng, (N, K)))
    return BF16Problem("dense", M, N, K, 1, a, b[None], name=name)


def make_bf16_contiguous(counts, N: int, K: int, seed: int, name: str = "", gaps=None) -> BF16Problem:
    """Contiguous layout: groups packed back to back, each padded to 128 rows;
    padding rows hold BF16 NaN and m_indices -1.  ``gaps[g]`` whole 128-row
    blocks of padding follow group g's rows."""
    rng = np.random.default_rng(seed)
    counts = [int(c) for c in counts]
    G = len(counts)
    gaps = [0] * G if gaps is None else [int(x) for x in gaps]
    padded = [(c + ALIGN_M - 1) // ALIGN_M * ALIGN_M + ALIGN_M * x for c, x in zip(counts, gaps)]
    M_total = int(sum(padded))
    a_all = _bf16_bits(_normal(rng, (sum(counts), K)))
    b = _bf16_bits(_normal(rng, (G * N, K))).reshape(G, N, K)
    a = np.full((M_total, K), BF16_NAN_BITS, dtype=np.uint16)
    m_idx = np.full((M_total,), -1, dtype=np.int32)
    src = dst = 0
    for g, (c, p) in enumerate(zip(counts, padded)):
        a[dst:dst + c] = a_all[src:src + c]
        m_idx[dst:dst + c] = g
        src += c
        dst += p
    return BF16Problem("contiguous", M_total, N, K, G, a, b, m_indices=m_idx, name=name)


def make_bf16_masked(masked_m, Mmax: int, N: int, K: int, seed: int, name: str = "") -> BF16Problem:
    """Masked layout: a [G, Mmax, K]; rows >= masked_m[g] hold BF16 NaN."""
    rng = np.random.default_rng(seed)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    G = len(masked_m)
    a = _bf16_bits(_normal(rng, (G * Mmax, K))).reshape(G, Mmax, K)
    b = _bf16_bits(_normal(rng, (G * N, K))).reshape(G, N, K)
    for g in range(G):
        a[g, masked_m[g]:] = BF16_NAN_BITS
    return BF16Problem("masked", Mmax, N, K, G, a, b, masked_m=masked_m, name=name)


BF16_WORKLOADS = {
    "bf16_dense_large": dict(kind="dense", M=4096, N=7168, K=16384, seed=11),
    "bf16_dense_decode_m64": dict(kind="dense", M=64, N=2112, K=7168, seed=12),
    "bf16_contiguous_g4": dict(kind="contiguous", G=4, tokens=32768, N=4096, K=7168, seed=13),
    "bf16_masked_g16": dict(kind="masked", G=16, Mmax=256, N=4096, K=7168, seed=14),
}


def make_bf16_workload(name: str, seed_offset: int = 0) -> BF16Problem:
    w = dict(BF16_WORKLOADS[name])
    kind = w.pop("kind")
    seed = w.pop("seed") + seed_offset
    if kind == "dense":
        return make_bf16_dense(w["M"], w["N"], w["K"], seed, name=name)
    rng = np.random.default_rng(seed)
    if kind == "contiguous":
        counts = rng.multinomial(w["tokens"], [1.0 / w["G"]] * w["G"])
        return make_bf16_contiguous(counts, w["N"], w["K"], seed + 1000, name=name)
    masked_m = rng.integers(0, w["Mmax"] + 1, size=w["G"]).astype(np.int32)
    return make_bf16_masked(masked_m, w["Mmax"], w["N"], w["K"], seed + 1000, name=name)


# ----------------------------------------------------------------------------- fused expert FFN inputs
@dataclasses.dataclass
class FFNProblem:
    """Single-GPU expert FFN in the contiguous layout: tokens a [M_total, H]
    (E4M3, 1x128 scales), w1 [G, 2I, H] with gate and up rows interleaved per
    128 rows (block 2j = gate rows 128j.., block 2j+1 = the matching up rows),
    w2 [G, H, I]; both weights with 128x128 scales."""
    M: int                     # M_total (groups padded to 128 rows)
    H: int
    I: int
    G: int
    a: np.ndarray
    sfa: np.ndarray
    ld_sfa: int
    w1: np.ndarray
    sfb1: np.ndarray
    w2: np.ndarray
    sfb2: np.ndarray
    m_indices: np.ndarray
    name: str = ""
    layout: str = "ffn_contiguous"

    def valid_rows(self) -> int:
        return int((self.m_indices >= 0).sum())

    def groups_touched(self) -> int:
        return int(len(np.unique(self.m_indices[self.m_indices >= 0])))

    def flops(self) -> float:
        """Both GEMMs: 2 * rows * (2I * H + H * I)."""
        return 2.0 * self.valid_rows() * (2 * self.I * self.H + self.H * self.I)

    def bytes(self) -> float:
        """A, the touched experts' weights, the intermediate codes (written and
        read) with their scales, and y."""
        r, g = self.valid_rows(), self.groups_touched()
        kb, ib = self.H // BLOCK, self.I // BLOCK
        return float(r * self.H + r * kb * 4 + g * 3 * self.I * self.H
                     + g * (2 * ib * kb + kb * ib) * 4 + 2 * (r * self.I + r * ib * 4) + 2 * r * self.H)


def make_ffn_contiguous(counts, H: int, I: int, seed: int, name: str = "") -> FFNProblem:
    """Token rows as the contiguous GEMM's A (N(0,1), 1x128 scales, padding rows
    NaN); weights N(0,1)/sqrt(fan-in) quantised per 128x128 block; gate and up
    interleaved per 128 rows in w1."""
    assert H % BLOCK == 0 and I % BLOCK == 0
    base = make_contiguous(counts, 2 * I, H, seed, name=name)     # a, sfa, m_indices (w unused)
    rng = np.random.default_rng(seed + 500)
    G = len(counts)
    gate = _normal(rng, (G, I, H)) / np.float32(np.sqrt(H))
    up = _normal(rng, (G, I, H)) / np.float32(np.sqrt(H))
    down = _normal(rng, (G, H, I)) / np.float32(np.sqrt(I))
    w1_32 = np.empty((G, 2 * I, H), np.float32)
    for j in range(I // BLOCK):
        w1_32[:, 2 * j * BLOCK:(2 * j + 1) * BLOCK] = gate[:, j * BLOCK:(j + 1) * BLOCK]
        w1_32[:, (2 * j + 1) * BLOCK:(2 * j + 2) * BLOCK] = up[:, j * BLOCK:(j + 1) * BLOCK]
    w1 = np.empty((G, 2 * I, H), np.uint8)
    sfb1 = np.empty((G, 2 * I // BLOCK, H // BLOCK), np.float32)
    w2 = np.empty((G, H, I), np.uint8)
    sfb2 = np.empty((G, H // BLOCK, I // BLOCK), np.float32)
    for g in range(G):
        w1[g], sfb1[g] = quantize_blocks_128x128(w1_32[g])
        w2[g], sfb2[g] = quantize_blocks_128x128(down[g])
    return FFNProblem(base.M, H, I, G, base.a, base.sfa, base.ld_sfa, w1, sfb1, w2, sfb2,
                      base.m_indices, name=name)


def make_ffn_multinomial(G: int, tokens: int, H: int, I: int, seed: int, name: str = "") -> FFNProblem:
    rng = np.random.default_rng(seed)
    counts = rng.multinomial(tokens, [1.0 / G] * G)
    return make_ffn_contiguous(counts, H, I, seed + 1000, name=name)


# an expert FFN of a DeepSeek-V3-sized MoE layer on 4 experts: hidden 7168,
# intermediate 2048, 32768 routed tokens (the contiguous workload's tokens)
FFN_WORKLOADS = {
    "ffn_g4": dict(G=4, tokens=32768, H=7168, I=2048, seed=15),
}


def make_ffn_workload(name: str, seed_offset: int = 0) -> FFNProblem:
    w = dict(FFN_WORKLOADS[name])
    return make_ffn_multinomial(w["G"], w["tokens"], w["H"], w["I"], w["seed"] + seed_offset, name=name)
