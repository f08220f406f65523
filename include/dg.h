/*
 * dg.h -- C ABI of the B200 (sm_100a) FP8 block-scaled NT GEMM library.
 *
 * The operation (DeepGEMM pages: page 2 "技术特性" -- FP8 GEMM with
 * fine-grained scaling, each K-block's tensor-core sum promoted into an FP32
 * accumulator on CUDA cores; page 3 "核心功能" -- "fp8_gemm_nt", block-wise
 * scaling, m-grouped GEMMs):
 *
 *   D[m,n] = sum_kb  sA[m,kb] * sB[n/128,kb] * sum_{k in block kb} A[m,k] * B[n,k]
 *
 * promoted to FP32 per 128-wide K-block and stored as BF16 (round to nearest
 * even).  "NT": A [M,K] and B [N,K] are both K-major, D = A * B^T.
 *
 * Common conventions for every GEMM entry point:
 *   - All pointers are DEVICE memory owned by the caller, 16-byte aligned.
 *     The library allocates nothing and keeps no reference after the call
 *     returns; the caller keeps the buffers alive until the stream work ends.
 *   - E4M3 bytes are OCP FP8 E4M3 ("fn": no infinities, 0x7F/0xFF are NaN,
 *     largest finite 448).
 *   - KB = K / 128 and NB = ceil(N / 128).
 *   - sfa ("MN-major"): the scale of row r for K-block kb is
 *     sfa[kb * ld_sfa + r]; ld_sfa >= rows and ld_sfa % 4 == 0.
 *   - sfb: the scale of weight block j (rows 128j..128j+127) for K-block kb is
 *     sfb[j * KB + kb]; grouped calls hold one such [NB][KB] array per group,
 *     back to back.
 *   - d: BF16 [rows, N] row-major (row stride N elements).
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on it and never synchronise the host.
 *   - Shape rules: K > 0, K % 128 == 0; N > 0, N % 16 == 0; M >= 0.
 *   - Errors: every argument is validated before anything is enqueued; on an
 *     error nothing is launched and d is untouched.  DG_ERR_CUDA reports a
 *     failed launch or a CUDA runtime error (text via dg_last_cuda_error()).
 *     A kernel that gives up on a bounded wait records DG_ERR_TIMEOUT in the
 *     device status word (dg_get_device_status) instead of hanging.  The call
 *     that launched it has already returned DG_SUCCESS, and d may be partly
 *     written.  The status word is one per device, shared by every call on
 *     every stream: a caller that needs to know which call failed reads (and
 *     clears) it between calls.
 *   - Thread safety: calls on different streams may run concurrently.
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DG_API __attribute__((visibility("default")))
#else
#define DG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DG_SUCCESS = 0,
    DG_ERR_INVALID_VALUE = 1,      /* null pointer, negative size, bad index table */
    DG_ERR_MISALIGNED = 2,         /* pointer or leading dimension not 16-byte aligned */
    DG_ERR_UNSUPPORTED_SHAPE = 3,  /* K % 128, N % 16, or a size beyond the limits */
    DG_ERR_UNSUPPORTED_DEVICE = 4, /* no CUDA device, or not compute capability 10.0 */
    DG_ERR_CUDA = 5,               /* CUDA runtime / launch failure */
    DG_ERR_TIMEOUT = 6             /* a kernel's bounded wait ran out (device status) */
} dg_status_t;

/*
 * Dense GEMM (page 3 "核心功能" / "快速开始": fp8_gemm_nt).
 *   a   [M, K] E4M3;  sfa [KB, ld_sfa] FP32, ld_sfa >= M
 *   b   [N, K] E4M3;  sfb [NB, KB] FP32
 *   d   [M, N] BF16, fully written.
 * M == 0 is a no-op.
 */
DG_API dg_status_t dg_fp8_gemm_nt(const uint8_t *a, const float *sfa, int ld_sfa,
                           const uint8_t *b, const float *sfb,
                           void *d, int M, int N, int K, void *stream);

/*
 * M-grouped GEMM, contiguous layout (page 2 "MoE模型专属优化"; page 5 "02",
 * prefill).  The rows of all groups are packed back to back in a; each
 * group's rows are padded to a multiple of
 * dg_get_m_alignment_for_contiguous_layout() (128).
 *   a         [M_total, K] E4M3;  sfa [KB, ld_sfa] FP32, ld_sfa >= M_total
 *   b         [G, N, K] E4M3;     sfb [G, NB, KB] FP32
 *   d         [M_total, N] BF16
 *   m_indices [M_total] int32 on the device: the group of each row, -1 for
 *             padding.  Precondition: the rows of each 128-row block carry
 *             one group index or -1, and the block's first row is not -1
 *             unless the whole block is padding (a block whose first row is
 *             -1 is skipped).  Outputs of padding rows are unspecified (they
 *             may be written).  An index >= G makes the kernel skip the block
 *             and record DG_ERR_INVALID_VALUE in the device status word.
 *             The layout packs each group's rows as one run of blocks; runs
 *             may also repeat or alternate, within one limit: large calls
 *             (N > 128, K >= 4096, G < 1024) compute 256-row block pairs,
 *             and at most 1024 pairs may hold two different groups.  Past
 *             that the excess pairs' second blocks are not written and
 *             DG_ERR_INVALID_VALUE is recorded.  One run per group keeps the
 *             count below G.
 * M_total % 128 == 0; M_total == 0 is a no-op.
 */
DG_API dg_status_t dg_m_grouped_fp8_gemm_nt_contiguous(const uint8_t *a, const float *sfa, int ld_sfa,
                                                const uint8_t *b, const float *sfb,
                                                void *d, const int32_t *m_indices,
                                                int M_total, int N, int K, int G,
                                                void *stream);

/*
 * M-grouped GEMM, masked layout (page 2 "MoE模型专属优化"; page 5 "02",
 * decode): a fixed [G, Mmax, K] buffer and a per-group valid-row count that
 * only the device reads, so the call works unchanged inside a CUDA graph.
 *   a        [G, Mmax, K] E4M3;   sfa [G, KB, ld_sfa] FP32, ld_sfa >= Mmax
 *   b        [G, N, K] E4M3;      sfb [G, NB, KB] FP32
 *   d        [G, Mmax, N] BF16
 *   masked_m [G] int32 on the device, 0 <= masked_m[g] <= Mmax.
 * Rows m < masked_m[g] of group g are computed; rows >= masked_m[g] of d are
 * never written (bit-for-bit untouched).  Groups with masked_m[g] == 0 read
 * nothing.  A count outside [0, Mmax] is clamped and recorded as
 * DG_ERR_INVALID_VALUE in the device status word.  G <= 1024 and
 * G * Mmax < 2^31 (32-bit tensor-map row coordinates), else
 * DG_ERR_UNSUPPORTED_SHAPE.
 */
DG_API dg_status_t dg_m_grouped_fp8_gemm_nt_masked(const uint8_t *a, const float *sfa, int ld_sfa,
                                            const uint8_t *b, const float *sfb,
                                            void *d, const int32_t *masked_m,
                                            int G, int Mmax, int N, int K, void *stream);

/*
 * K-grouped GEMM, groups contiguous along K (page 3 "核心功能": the
 * k_grouped_gemm family -- the weight-gradient shape of MoE training, where
 * the reduced dimension is each expert's tokens).  Group g owns ks[g]
 * consecutive K columns of A and B (and the matching K-blocks of sfa / sfb);
 * its output is the block-scaled sum over those K-blocks only:
 *   D[g][m][n] = sum_{kb in group g} sA[m,kb] * sB[n/128,kb] * (A_kb . B_kb)
 *   a   [M, K] E4M3;  sfa [KB, ld_sfa] FP32, ld_sfa >= M   (dense layout)
 *   b   [N, K] E4M3;  sfb [NB, KB] FP32                     (dense layout)
 *   d   [G, M, N] BF16, fully written (zeros for a group with ks[g] == 0)
 *   ks  [G] int32 on the device, each a multiple of 128, sum == K.  Only the
 *       device reads it (graph-compatible).  A size that is negative, not a
 *       multiple of 128, or a total other than K is recorded as
 *       DG_ERR_INVALID_VALUE in the device status word; the kernel then uses
 *       the K-blocks that exist (rounded down, clipped at K).
 * 1 <= G <= 1024; M == 0 is a no-op.  G * M < 2^31 (the output's stacked
 * rows are addressed by 32-bit tensor-map coordinates), else
 * DG_ERR_UNSUPPORTED_SHAPE.
 */
DG_API dg_status_t dg_k_grouped_fp8_gemm_nt_contiguous(const uint8_t *a, const float *sfa,
                                                       int ld_sfa, const uint8_t *b,
                                                       const float *sfb, void *d,
                                                       const int32_t *ks, int G, int M, int N,
                                                       int K, void *stream);

/*
 * Fused expert FFN, first stage (page 5 "03" -- Mega MoE fuses the first
 * layer's GEMM, the SwiGLU activation and the second layer into one MoE
 * kernel; here on one GPU, without the expert-parallel dispatch and combine):
 * the contiguous M-grouped FP8 GEMM of the gate and up projections, whose
 * epilogue applies SwiGLU and re-quantises the activation per token and
 * 128-column block, writing the second GEMM's A operand directly (the FP32
 * accumulators never go to memory).
 *   a, sfa, m_indices: as for dg_m_grouped_fp8_gemm_nt_contiguous (K = hidden size)
 *   b   [G, N, K] E4M3, N = 2 * I: for each 128-column block j of the
 *       intermediate size I, weight rows [256 j, 256 j + 128) are the gate
 *       projection and rows [256 j + 128, 256 j + 256) the up projection
 *       ("interleaved by 128"); sfb [G, N/128, K/128] FP32.
 *   With h = the promoted FP32 product (as in the GEMMs above):
 *     act[m, 128 j + c] = silu(h[m, 256 j + c]) * h[m, 256 j + 128 + c],
 *     silu(x) = x / (1 + exp(-x)), in FP32;
 *     per row and 128-column block: s = amax / 448 (1 if amax == 0),
 *     q = E4M3_RNE(act / s) (IEEE quotient; values saturate at +-448).
 *   q_out [M_total, I] E4M3; s_out [I/128, ld_s_out] FP32 (MN-major,
 *       ld_s_out >= M_total, a multiple of 4).  Rows of 128-row blocks whose
 *       first row is padding are not written; padding rows inside a block may be.
 * M_total % 128 == 0, N % 256 == 0.
 */
DG_API dg_status_t dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(
    const uint8_t *a, const float *sfa, int ld_sfa, const uint8_t *b, const float *sfb,
    uint8_t *q_out, float *s_out, int ld_s_out, const int32_t *m_indices, int M_total, int N, int K,
    int G, void *stream);

/*
 * Fused expert FFN on one GPU: the first stage above, then the contiguous
 * M-grouped FP8 GEMM of the down projection on its output:
 *   y = dg_m_grouped_fp8_gemm_nt_contiguous(q_mid, s_mid, w2 [G, H, I], sfb2 [G, H/128, I/128])
 * a [M_total, H] E4M3 with sfa; w1 [G, 2I, H] (interleaved by 128) with sfb1;
 * q_mid [M_total, I] and s_mid [I/128, ld_mid] are caller-owned intermediate
 * buffers; y [M_total, H] BF16.  Two launches on the stream, no host sync.
 */
DG_API dg_status_t dg_m_grouped_fp8_ffn_contiguous(const uint8_t *a, const float *sfa, int ld_sfa,
                                                   const uint8_t *w1, const float *sfb1,
                                                   const uint8_t *w2, const float *sfb2,
                                                   uint8_t *q_mid, float *s_mid, int ld_mid, void *y,
                                                   const int32_t *m_indices, int M_total, int H,
                                                   int I, int G, void *stream);

/*
 * The fused expert FFN above for callers that cannot allocate device memory.
 * The pages have no counterpart: this entry point exists for users of this
 * library, not for the method.  Some callers cannot call cudaMalloc at the
 * point where they run the FFN: a plugin that runs inside another runtime's
 * execution step, where the host runtime owns all device memory and forbids
 * allocation; a serving loop that freezes its memory after warm-up so that
 * it can never fail or stall on an allocation mid-request; a plain C program
 * with no device allocator of its own.  Such a caller still passes its inputs
 * and its output, but not the intermediate buffers q_mid and s_mid: the call
 * keeps them in one file-scope device array of DG_NOALLOC_SCRATCH_BYTES bytes,
 * which every GPU that loads this library holds until the process exits.
 *   Arguments: as for dg_m_grouped_fp8_ffn_contiguous, without q_mid, s_mid
 *   and ld_mid.
 *   Size limit: the intermediate takes M_total * I bytes of E4M3 codes
 *   (rounded up to 256) plus (I / 128) * ld * 4 bytes of scales, with ld =
 *   M_total rounded up to a multiple of 4 (at least 4).  A call that needs
 *   more than DG_NOALLOC_SCRATCH_BYTES returns DG_ERR_UNSUPPORTED_SHAPE before
 *   enqueueing anything.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents.  Nothing in it has to start at zero: the second GEMM reads
 *   only intermediate rows that the first GEMM wrote in the same call.  Calls
 *   that overlap on the GPU (on different streams, or from different threads
 *   without ordering) race on the array and give wrong results; the caller
 *   must order them.
 *   The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library routine.
 */
#define DG_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
DG_API dg_status_t dg_m_grouped_fp8_ffn_contiguous_noalloc(const uint8_t *a, const float *sfa,
                                                           int ld_sfa, const uint8_t *w1,
                                                           const float *sfb1, const uint8_t *w2,
                                                           const float *sfb2, void *y,
                                                           const int32_t *m_indices, int M_total,
                                                           int H, int I, int G, void *stream);

/*
 * BF16 GEMMs (page 3 "核心功能": FP8, FP4 and BF16 GEMM operations, in the same
 * dense and m-grouped layouts):
 *   D[m,n] = sum_k A[m,k] * B[n,k]    accumulated in FP32, stored as BF16 (RNE)
 * A and B are BF16 (raw 16-bit patterns), K-major; no block scales.  Shape
 * rules: K > 0, K % 8 == 0; N > 0, N % 8 == 0 (16-byte rows); M >= 0.
 * Pointers, stream and error conventions as for the FP8 GEMMs.
 *
 * Dense: a [M, K], b [N, K], d [M, N].
 */
DG_API dg_status_t dg_bf16_gemm_nt(const void *a, const void *b, void *d, int M, int N, int K,
                                   void *stream);

/* Contiguous M-grouped BF16: a [M_total, K] (groups packed, each padded to 128
 * rows), b [G, N, K], d [M_total, N], m_indices [M_total] int32 on the device
 * with the same precondition and padding rules as the FP8 contiguous call.
 * Here the 256-row block pairs (and their limit of 1024 pairs holding two
 * different groups) apply to every call with N > 128, at least two blocks and
 * G < 1024, whatever K.  M_total % 128 == 0. */
DG_API dg_status_t dg_m_grouped_bf16_gemm_nt_contiguous(const void *a, const void *b, void *d,
                                                        const int32_t *m_indices, int M_total,
                                                        int N, int K, int G, void *stream);

/* Masked M-grouped BF16: a [G, Mmax, K], b [G, N, K], d [G, Mmax, N]; rows
 * m < masked_m[g] computed, the others never written (graph-compatible, as for
 * the FP8 masked call).  G <= 1024 and G * Mmax < 2^31, else
 * DG_ERR_UNSUPPORTED_SHAPE (as for the FP8 masked call). */
DG_API dg_status_t dg_m_grouped_bf16_gemm_nt_masked(const void *a, const void *b, void *d,
                                                    const int32_t *masked_m, int G, int Mmax,
                                                    int N, int K, void *stream);

/*
 * Per-token 1x128 activation quantiser (page 2 "技术特性": fine-grained
 * dynamic scaling; page 3 "核心功能": block-wise scaling): produces the A
 * operand and sfa of the GEMMs above from BF16 activations.  For each row m
 * and K-block kb:
 *   amax = max |x[m, 128kb .. 128kb+127]|
 *   s    = amax / 448 in FP32 (IEEE division), or 1 when amax == 0
 *   q[m,k] = E4M3 round-to-nearest-even of clamp(x[m,k] / s, -448, 448),
 *            with x / s the correctly rounded FP32 quotient
 *   sfa[kb * ld_sfa + m] = s
 * The codes are therefore a deterministic function of the inputs, identical
 * on every run and to any IEEE reference.
 *   x   [M, K] BF16 row-major (device);  q [M, K] E4M3 (device)
 *   sfa [KB, ld_sfa] FP32 (device), ld_sfa >= M, ld_sfa % 4 == 0 (so each
 *       K-block's column starts 16-byte aligned, as the GEMMs' TMA wants);
 *       entries m >= M are not written.
 * Inputs must be finite (NaN or infinity gives unspecified codes and scales).
 * K % 128 == 0; M == 0 is a no-op.  Same pointer, stream and error
 * conventions as the GEMMs.
 */
DG_API dg_status_t dg_per_token_cast_to_fp8(const void *x, uint8_t *q, float *sfa, int ld_sfa,
                                            int M, int K, void *stream);

/*
 * The quantiser fused with the masked layout's packing (page 2
 * "MoE模型专属优化"; page 5 "02", decode): x [G, Mmax, K] BF16, q
 * [G, Mmax, K] E4M3, sfa [G, KB, ld_sfa] FP32 with ld_sfa >= Mmax -- exactly
 * the a / sfa operands of dg_m_grouped_fp8_gemm_nt_masked.  Only rows
 * m < masked_m[g] (device int32 [G]) are read and written; the other rows of
 * q and sfa are untouched, so the call works unchanged inside a CUDA graph.  A
 * count outside [0, Mmax] is clamped and recorded as DG_ERR_INVALID_VALUE in
 * the device status word.  1 <= G <= 1024, G * Mmax < 2^31.
 */
DG_API dg_status_t dg_per_token_cast_to_fp8_masked(const void *x, uint8_t *q, float *sfa,
                                                   int ld_sfa, const int32_t *masked_m, int G,
                                                   int Mmax, int K, void *stream);

/* Row alignment of the contiguous layout (page 2 "MoE模型专属优化":
 * get_m_alignment_for_contiguous_layout).  Returns 128. */
DG_API int dg_get_m_alignment_for_contiguous_layout(void);

/* Smallest count >= n whose size n * elem_bytes is a multiple of 16 bytes,
 * the TMA alignment (page 2 "快速实践指南": get_tma_aligned_size).
 * elem_bytes must divide 16 (1, 2, 4, 8, 16); otherwise returns 0. */
DG_API size_t dg_get_tma_aligned_size(size_t n, size_t elem_bytes);

/* Reads the current device's status word, which kernels set when a bounded
 * wait runs out (DG_ERR_TIMEOUT) or a device-side index is out of range
 * (DG_ERR_INVALID_VALUE).  Synchronises the device.  *code receives the raw
 * word (0 = clean; low 8 bits = dg_status_t, upper bits = where).  When
 * clear != 0 the word is reset to 0 afterwards. */
DG_API dg_status_t dg_get_device_status(int *code, int clear);

/* Static text for a status code. */
DG_API const char *dg_status_string(dg_status_t status);

/* Text of the last CUDA error seen by this library on the calling thread
 * (empty string if none). */
DG_API const char *dg_last_cuda_error(void);

/* Test hook, not part of the GEMM contract (the pages have no counterpart):
 * kernels launched afterwards by this process run with the given debug flags.
 * Flag 1 makes the producer warp issue no loads, so the consumers' bounded
 * waits run out and the kernel records DG_ERR_TIMEOUT in the device status
 * word and returns instead of hanging.  Flag 2 makes the quantisers take the
 * IEEE division for every element instead of the reciprocal fast path (the
 * results are identical).  0 restores normal operation.  The
 * wait limit in clock cycles comes from the environment variable
 * DG_WAIT_TIMEOUT_CYCLES, read once (default 2^32). */
DG_API void dg_debug_set_flags(int flags);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
