"""Python binding of the B200 GEMM library (``_dg.so``): FP8 block-scaled NT
GEMMs (dense, M-grouped contiguous and masked, K-grouped), the fused expert
FFN, BF16 GEMMs in the same layouts, and the per-token 1x128 quantiser.

Argument marshalling only: every function below checks dtypes and shapes of
torch CUDA tensors, reads their raw pointers and calls the C function of the
same name declared in ``include/dg.h``.  All arithmetic runs in the CUDA
kernels of ``_dg.so``.  There is no fallback: if the shared library is missing
or fails to load, importing the library handle raises.

Storage formats (see ``include/dg.h``): FP8 A/B are uint8 E4M3 bytes, K-major;
sfa is float32 [KB, ld_sfa] ("MN-major"; [G, KB, ld_sfa] for the masked
layout); sfb is float32 [G, NB, KB]; D is bfloat16.  BF16 GEMM operands and
quantiser inputs are bfloat16 rows.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_dg.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "dg.h")

DG_SUCCESS = 0
# size of the fixed device array of dg_m_grouped_fp8_ffn_contiguous_noalloc (DG_NOALLOC_SCRATCH_BYTES)
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
STATUS_NAMES = {0: "DG_SUCCESS", 1: "DG_ERR_INVALID_VALUE", 2: "DG_ERR_MISALIGNED",
                3: "DG_ERR_UNSUPPORTED_SHAPE", 4: "DG_ERR_UNSUPPORTED_DEVICE",
                5: "DG_ERR_CUDA", 6: "DG_ERR_TIMEOUT"}

_lib = None


class DGError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


def exported_names():
    """Names of the functions that include/dg.h declares."""
    text = open(HEADER).read()
    return re.findall(r"DG_API\s+[\w\s\*]+?\b(dg_\w+)\s*\(", text)


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m moe_grouped_gemm_fp32_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I = ctypes.c_void_p, ctypes.c_int
    L.dg_fp8_gemm_nt.argtypes = [P, P, I, P, P, P, I, I, I, P]
    L.dg_m_grouped_fp8_gemm_nt_contiguous.argtypes = [P, P, I, P, P, P, P, I, I, I, I, P]
    L.dg_m_grouped_fp8_gemm_nt_masked.argtypes = [P, P, I, P, P, P, P, I, I, I, I, P]
    L.dg_k_grouped_fp8_gemm_nt_contiguous.argtypes = [P, P, I, P, P, P, P, I, I, I, I, P]
    L.dg_m_grouped_fp8_gemm_swiglu_quant_contiguous.argtypes = [P, P, I, P, P, P, P, I, P, I, I, I, I, P]
    L.dg_m_grouped_fp8_ffn_contiguous.argtypes = [P, P, I, P, P, P, P, P, P, I, P, P, I, I, I, I, P]
    L.dg_m_grouped_fp8_ffn_contiguous_noalloc.argtypes = [P, P, I, P, P, P, P, P, P, I, I, I, I, P]
    L.dg_bf16_gemm_nt.argtypes = [P, P, P, I, I, I, P]
    L.dg_m_grouped_bf16_gemm_nt_contiguous.argtypes = [P, P, P, P, I, I, I, I, P]
    L.dg_m_grouped_bf16_gemm_nt_masked.argtypes = [P, P, P, P, I, I, I, I, P]
    L.dg_per_token_cast_to_fp8.argtypes = [P, P, P, I, I, I, P]
    L.dg_per_token_cast_to_fp8_masked.argtypes = [P, P, P, I, P, I, I, I, P]
    for f in ("dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
              "dg_m_grouped_fp8_gemm_nt_masked", "dg_k_grouped_fp8_gemm_nt_contiguous",
              "dg_m_grouped_fp8_gemm_swiglu_quant_contiguous", "dg_m_grouped_fp8_ffn_contiguous",
              "dg_bf16_gemm_nt", "dg_m_grouped_bf16_gemm_nt_contiguous",
              "dg_m_grouped_bf16_gemm_nt_masked",
              "dg_per_token_cast_to_fp8",
              "dg_per_token_cast_to_fp8_masked"):
        getattr(L, f).restype = I
    L.dg_get_m_alignment_for_contiguous_layout.argtypes = []
    L.dg_get_m_alignment_for_contiguous_layout.restype = I
    L.dg_get_tma_aligned_size.argtypes = [ctypes.c_size_t, ctypes.c_size_t]
    L.dg_get_tma_aligned_size.restype = ctypes.c_size_t
    L.dg_get_device_status.argtypes = [ctypes.POINTER(I), I]
    L.dg_get_device_status.restype = I
    L.dg_status_string.argtypes = [I]
    L.dg_status_string.restype = ctypes.c_char_p
    L.dg_last_cuda_error.argtypes = []
    L.dg_last_cuda_error.restype = ctypes.c_char_p
    L.dg_debug_set_flags.argtypes = [I]
    L.dg_debug_set_flags.restype = None
    _lib = L
    return L


def _check(status: int, where: str):
    if status != DG_SUCCESS:
        detail = lib().dg_last_cuda_error().decode() if status == 5 else ""
        raise DGError(status, where, detail)


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _req(t, dtype, name, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() not in ((ndim,) if isinstance(ndim, int) else ndim):
        raise ValueError(f"{name} has {t.dim()} dims")
    return t.data_ptr()


def _shape(t, want, name):
    """Raise ValueError unless ``t`` has exactly the shape ``want``; a None
    entry is a size this call cannot know (left to the C call's own checks).
    The C functions receive only pointers and sizes, so a buffer smaller than
    its sizes imply must be caught here."""
    got = tuple(t.shape)
    if len(got) != len(want) or any(w is not None and g != w for g, w in zip(got, want)):
        shown = tuple("*" if w is None else w for w in want)
        raise ValueError(f"{name} has shape {got}, expected {shown}")


def _blocks(n):
    """Number of 128-wide blocks of a size that must be a multiple of 128
    (None otherwise: the C call rejects such a size itself)."""
    return n // 128 if n % 128 == 0 else None


def _ceil_blocks(n):
    return (n + 127) // 128


def _call(where, fn, tensors, stream, *args):
    """Call ``fn(*args, stream_handle)`` and raise on a non-success status.
    The C library launches on the current CUDA device, so every tensor (and
    the stream, if given) must live on that device."""
    import torch
    devs = {t.device for t in tensors}
    if len(devs) != 1:
        raise ValueError(f"{where}: all tensors must be on one CUDA device, got {sorted(map(str, devs))}")
    dev = devs.pop()
    if dev.type == "cuda" and dev.index != torch.cuda.current_device():
        raise ValueError(f"{where}: tensors are on {dev} but the current device is "
                         f"cuda:{torch.cuda.current_device()} (select it with torch.cuda.device)")
    if stream is not None and stream.device != dev:
        raise ValueError(f"{where}: stream is on {stream.device}, tensors on {dev}")
    _check(fn(*args, _stream_handle(stream)), where)


# --------------------------------------------------------------------------- GEMMs
def dg_fp8_gemm_nt(a, sfa, b, sfb, d, stream=None):
    """D[M,N] (bf16) = block-scaled A[M,K] * B[N,K]^T.

    a uint8 [M,K]; sfa float32 [KB, ld_sfa]; b uint8 [N,K] (or [1,N,K]);
    sfb float32 [NB,KB] (or [1,NB,KB]); d bfloat16 [M,N]."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 2), _req(sfa, torch.float32, "sfa", 2),
            _req(b, torch.uint8, "b", (2, 3)), _req(sfb, torch.float32, "sfb", (2, 3)),
            _req(d, torch.bfloat16, "d", 2))
    M, K = a.shape
    N = b.shape[-2]
    ld = sfa.shape[-1]
    KB = _blocks(K)
    _shape(b, (1,) * (b.dim() - 2) + (N, K), "b")
    _shape(sfa, (KB, ld), "sfa")
    _shape(sfb, (1,) * (sfb.dim() - 2) + (_ceil_blocks(N), KB), "sfb")
    _shape(d, (M, N), "d")
    _call("dg_fp8_gemm_nt", lib().dg_fp8_gemm_nt, (a, sfa, b, sfb, d), stream,
          ptrs[0], ptrs[1], ld, ptrs[2], ptrs[3], ptrs[4], M, N, K)
    return d


def dg_m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, m_indices, stream=None):
    """Contiguous M-grouped GEMM.  a uint8 [M_total,K]; b uint8 [G,N,K];
    sfb float32 [G,NB,KB]; d bfloat16 [M_total,N]; m_indices int32 [M_total]."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 2), _req(sfa, torch.float32, "sfa", 2),
            _req(b, torch.uint8, "b", 3), _req(sfb, torch.float32, "sfb", 3),
            _req(d, torch.bfloat16, "d", 2), _req(m_indices, torch.int32, "m_indices", 1))
    M_total, K = a.shape
    G, N, _ = b.shape
    KB = _blocks(K)
    _shape(b, (G, N, K), "b")
    _shape(sfa, (KB, None), "sfa")
    _shape(sfb, (G, _ceil_blocks(N), KB), "sfb")
    _shape(d, (M_total, N), "d")
    _shape(m_indices, (M_total,), "m_indices")
    _call("dg_m_grouped_fp8_gemm_nt_contiguous", lib().dg_m_grouped_fp8_gemm_nt_contiguous,
          (a, sfa, b, sfb, d, m_indices), stream,
          ptrs[0], ptrs[1], sfa.shape[-1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], M_total, N, K, G)
    return d


def dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, masked_m, stream=None):
    """Masked M-grouped GEMM.  a uint8 [G,Mmax,K]; sfa float32 [G,KB,ld_sfa];
    b uint8 [G,N,K]; sfb float32 [G,NB,KB]; d bfloat16 [G,Mmax,N];
    masked_m int32 [G] (device).  Rows >= masked_m[g] of d are not written."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 3), _req(sfa, torch.float32, "sfa", 3),
            _req(b, torch.uint8, "b", 3), _req(sfb, torch.float32, "sfb", 3),
            _req(d, torch.bfloat16, "d", 3), _req(masked_m, torch.int32, "masked_m", 1))
    G, Mmax, K = a.shape
    N = b.shape[1]
    KB = _blocks(K)
    _shape(b, (G, N, K), "b")
    _shape(sfa, (G, KB, None), "sfa")
    _shape(sfb, (G, _ceil_blocks(N), KB), "sfb")
    _shape(d, (G, Mmax, N), "d")
    _shape(masked_m, (G,), "masked_m")
    _call("dg_m_grouped_fp8_gemm_nt_masked", lib().dg_m_grouped_fp8_gemm_nt_masked,
          (a, sfa, b, sfb, d, masked_m), stream,
          ptrs[0], ptrs[1], sfa.shape[-1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], G, Mmax, N, K)
    return d



def dg_k_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, ks, stream=None):
    """K-grouped GEMM (groups contiguous along K).  a uint8 [M,K]; sfa float32
    [KB, ld_sfa]; b uint8 [N,K]; sfb float32 [NB,KB]; d bfloat16 [G,M,N];
    ks int32 [G] (device), multiples of 128 adding up to K."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 2), _req(sfa, torch.float32, "sfa", 2),
            _req(b, torch.uint8, "b", (2, 3)), _req(sfb, torch.float32, "sfb", (2, 3)),
            _req(d, torch.bfloat16, "d", 3), _req(ks, torch.int32, "ks", 1))
    M, K = a.shape
    N = b.shape[-2]
    G = ks.shape[0]
    KB = _blocks(K)
    _shape(b, (1,) * (b.dim() - 2) + (N, K), "b")
    _shape(sfa, (KB, None), "sfa")
    _shape(sfb, (1,) * (sfb.dim() - 2) + (_ceil_blocks(N), KB), "sfb")
    _shape(d, (G, M, N), "d")
    _call("dg_k_grouped_fp8_gemm_nt_contiguous", lib().dg_k_grouped_fp8_gemm_nt_contiguous,
          (a, sfa, b, sfb, d, ks), stream,
          ptrs[0], ptrs[1], sfa.shape[-1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], G, M, N, K)
    return d



# --------------------------------------------------------------------------- fused expert FFN
def dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(a, sfa, b, sfb, q_out, s_out, m_indices, stream=None):
    """First FFN stage: contiguous FP8 GEMM with gate/up weights b [G, 2I, K]
    (interleaved per 128 rows) whose epilogue writes E4M3 codes q_out
    [M_total, I] and scales s_out [I/128, ld] of silu(gate) * up."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 2), _req(sfa, torch.float32, "sfa", 2),
            _req(b, torch.uint8, "b", 3), _req(sfb, torch.float32, "sfb", 3),
            _req(q_out, torch.uint8, "q_out", 2), _req(s_out, torch.float32, "s_out", 2),
            _req(m_indices, torch.int32, "m_indices", 1))
    M_total, K = a.shape
    G, N, _ = b.shape
    KB = _blocks(K)
    I = N // 2 if N % 2 == 0 else None
    _shape(b, (G, N, K), "b")
    _shape(sfa, (KB, None), "sfa")
    _shape(sfb, (G, _ceil_blocks(N), KB), "sfb")
    _shape(q_out, (M_total, I), "q_out")
    _shape(s_out, (_blocks(I) if I is not None else None, None), "s_out")
    _shape(m_indices, (M_total,), "m_indices")
    _call("dg_m_grouped_fp8_gemm_swiglu_quant_contiguous",
          lib().dg_m_grouped_fp8_gemm_swiglu_quant_contiguous,
          (a, sfa, b, sfb, q_out, s_out, m_indices), stream,
          ptrs[0], ptrs[1], sfa.shape[-1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], s_out.shape[-1],
          ptrs[6], M_total, N, K, G)
    return q_out, s_out


def dg_m_grouped_fp8_ffn_contiguous(a, sfa, w1, sfb1, w2, sfb2, q_mid, s_mid, y, m_indices, stream=None):
    """Fused expert FFN on one GPU: y [M_total, H] (bfloat16) from tokens a
    [M_total, H], w1 [G, 2I, H] (gate/up interleaved per 128 rows), w2 [G, H, I];
    q_mid [M_total, I] / s_mid [I/128, ld] are the caller's intermediate buffers."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 2), _req(sfa, torch.float32, "sfa", 2),
            _req(w1, torch.uint8, "w1", 3), _req(sfb1, torch.float32, "sfb1", 3),
            _req(w2, torch.uint8, "w2", 3), _req(sfb2, torch.float32, "sfb2", 3),
            _req(q_mid, torch.uint8, "q_mid", 2), _req(s_mid, torch.float32, "s_mid", 2),
            _req(y, torch.bfloat16, "y", 2), _req(m_indices, torch.int32, "m_indices", 1))
    M_total, H = a.shape
    G, I2, _ = w1.shape
    I = I2 // 2
    HB, IB = _blocks(H), _blocks(I)
    _shape(sfa, (HB, None), "sfa")
    _shape(w1, (G, 2 * I, H), "w1")
    _shape(sfb1, (G, _ceil_blocks(2 * I), HB), "sfb1")
    _shape(w2, (G, H, I), "w2")
    _shape(sfb2, (G, _ceil_blocks(H), IB), "sfb2")
    _shape(q_mid, (M_total, I), "q_mid")
    _shape(s_mid, (IB, None), "s_mid")
    _shape(y, (M_total, H), "y")
    _shape(m_indices, (M_total,), "m_indices")
    _call("dg_m_grouped_fp8_ffn_contiguous", lib().dg_m_grouped_fp8_ffn_contiguous,
          (a, sfa, w1, sfb1, w2, sfb2, q_mid, s_mid, y, m_indices), stream,
          ptrs[0], ptrs[1], sfa.shape[-1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], ptrs[6], ptrs[7],
          s_mid.shape[-1], ptrs[8], ptrs[9], M_total, H, I, G)
    return y


def dg_m_grouped_fp8_ffn_contiguous_noalloc(a, sfa, w1, sfb1, w2, sfb2, y, m_indices, stream=None):
    """The fused expert FFN for callers that cannot allocate device memory: as
    dg_m_grouped_fp8_ffn_contiguous, but the intermediate codes and scales live
    in the library's own fixed device array (DG_NOALLOC_SCRATCH_BYTES, 16 MiB),
    so nothing is allocated, here or in the C call.  Calls that overlap on the
    GPU share that array and race; order them."""
    import torch
    ptrs = (_req(a, torch.uint8, "a", 2), _req(sfa, torch.float32, "sfa", 2),
            _req(w1, torch.uint8, "w1", 3), _req(sfb1, torch.float32, "sfb1", 3),
            _req(w2, torch.uint8, "w2", 3), _req(sfb2, torch.float32, "sfb2", 3),
            _req(y, torch.bfloat16, "y", 2), _req(m_indices, torch.int32, "m_indices", 1))
    M_total, H = a.shape
    G, I2, _ = w1.shape
    I = I2 // 2
    HB, IB = _blocks(H), _blocks(I)
    _shape(sfa, (HB, None), "sfa")
    _shape(w1, (G, 2 * I, H), "w1")
    _shape(sfb1, (G, _ceil_blocks(2 * I), HB), "sfb1")
    _shape(w2, (G, H, I), "w2")
    _shape(sfb2, (G, _ceil_blocks(H), IB), "sfb2")
    _shape(y, (M_total, H), "y")
    _shape(m_indices, (M_total,), "m_indices")
    _call("dg_m_grouped_fp8_ffn_contiguous_noalloc", lib().dg_m_grouped_fp8_ffn_contiguous_noalloc,
          (a, sfa, w1, sfb1, w2, sfb2, y, m_indices), stream,
          ptrs[0], ptrs[1], sfa.shape[-1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], ptrs[6], ptrs[7],
          M_total, H, I, G)
    return y

# --------------------------------------------------------------------------- BF16 GEMMs
def dg_bf16_gemm_nt(a, b, d, stream=None):
    """D[M,N] = A[M,K] * B[N,K]^T, all bfloat16 (FP32 accumulation)."""
    import torch
    ptrs = (_req(a, torch.bfloat16, "a", 2), _req(b, torch.bfloat16, "b", (2, 3)),
            _req(d, torch.bfloat16, "d", 2))
    M, K = a.shape
    N = b.shape[-2]
    _shape(b, (1,) * (b.dim() - 2) + (N, K), "b")
    _shape(d, (M, N), "d")
    _call("dg_bf16_gemm_nt", lib().dg_bf16_gemm_nt, (a, b, d), stream, *ptrs, M, N, K)
    return d


def dg_m_grouped_bf16_gemm_nt_contiguous(a, b, d, m_indices, stream=None):
    """Contiguous M-grouped BF16 GEMM: a [M_total,K], b [G,N,K], d [M_total,N]."""
    import torch
    ptrs = (_req(a, torch.bfloat16, "a", 2), _req(b, torch.bfloat16, "b", 3),
            _req(d, torch.bfloat16, "d", 2), _req(m_indices, torch.int32, "m_indices", 1))
    M_total, K = a.shape
    G, N, _ = b.shape
    _shape(b, (G, N, K), "b")
    _shape(d, (M_total, N), "d")
    _shape(m_indices, (M_total,), "m_indices")
    _call("dg_m_grouped_bf16_gemm_nt_contiguous", lib().dg_m_grouped_bf16_gemm_nt_contiguous,
          (a, b, d, m_indices), stream, *ptrs, M_total, N, K, G)
    return d


def dg_m_grouped_bf16_gemm_nt_masked(a, b, d, masked_m, stream=None):
    """Masked M-grouped BF16 GEMM: a [G,Mmax,K], b [G,N,K], d [G,Mmax,N]."""
    import torch
    ptrs = (_req(a, torch.bfloat16, "a", 3), _req(b, torch.bfloat16, "b", 3),
            _req(d, torch.bfloat16, "d", 3), _req(masked_m, torch.int32, "masked_m", 1))
    G, Mmax, K = a.shape
    N = b.shape[1]
    _shape(b, (G, N, K), "b")
    _shape(d, (G, Mmax, N), "d")
    _shape(masked_m, (G,), "masked_m")
    _call("dg_m_grouped_bf16_gemm_nt_masked", lib().dg_m_grouped_bf16_gemm_nt_masked,
          (a, b, d, masked_m), stream, *ptrs, G, Mmax, N, K)
    return d

# --------------------------------------------------------------------------- quantisers
def dg_per_token_cast_to_fp8(x, q, sfa, stream=None):
    """Per-token 1x128 quantisation.  x bfloat16 [M,K]; q uint8 [M,K];
    sfa float32 [KB, ld_sfa] with ld_sfa >= M, a multiple of 4."""
    import torch
    ptrs = (_req(x, torch.bfloat16, "x", 2), _req(q, torch.uint8, "q", 2),
            _req(sfa, torch.float32, "sfa", 2))
    M, K = x.shape
    _shape(q, (M, K), "q")
    _shape(sfa, (_blocks(K), None), "sfa")
    _call("dg_per_token_cast_to_fp8", lib().dg_per_token_cast_to_fp8, (x, q, sfa), stream,
          *ptrs, sfa.shape[-1], M, K)
    return q, sfa


def dg_per_token_cast_to_fp8_masked(x, q, sfa, masked_m, stream=None):
    """Quantiser fused with the masked layout.  x bfloat16 [G,Mmax,K]; q uint8
    [G,Mmax,K]; sfa float32 [G,KB,ld_sfa]; masked_m int32 [G] (device).  Only
    rows < masked_m[g] are read and written."""
    import torch
    ptrs = (_req(x, torch.bfloat16, "x", 3), _req(q, torch.uint8, "q", 3),
            _req(sfa, torch.float32, "sfa", 3), _req(masked_m, torch.int32, "masked_m", 1))
    G, Mmax, K = x.shape
    _shape(q, (G, Mmax, K), "q")
    _shape(sfa, (G, _blocks(K), None), "sfa")
    _shape(masked_m, (G,), "masked_m")
    _call("dg_per_token_cast_to_fp8_masked", lib().dg_per_token_cast_to_fp8_masked,
          (x, q, sfa, masked_m), stream, ptrs[0], ptrs[1], ptrs[2], sfa.shape[-1], ptrs[3], G, Mmax, K)
    return q, sfa


# --------------------------------------------------------------------------- helpers
def dg_get_m_alignment_for_contiguous_layout() -> int:
    return lib().dg_get_m_alignment_for_contiguous_layout()


def dg_get_tma_aligned_size(n: int, elem_bytes: int = 4) -> int:
    return lib().dg_get_tma_aligned_size(n, elem_bytes)


def dg_get_device_status(clear: bool = True) -> int:
    code = ctypes.c_int(0)
    _check(lib().dg_get_device_status(ctypes.byref(code), int(clear)), "dg_get_device_status")
    return code.value


def dg_status_string(status: int) -> str:
    return lib().dg_status_string(status).decode()


def dg_debug_set_flags(flags: int) -> None:
    lib().dg_debug_set_flags(flags)
