/*
 * oracle.c -- CPU oracle for the FP8 (E4M3) block-scaled NT GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes (DeepGEMM pages: page 2 "技术特性" -- FP8 GEMM with
 * fine-grained scaling and two-level accumulation, the tensor-core partial sum
 * of each K-block promoted into an FP32 accumulator on CUDA cores; page 3
 * "核心功能" -- "fp8_gemm_nt", block-wise scaling, m-grouped GEMM; page 5
 * "02" -- contiguous and masked MoE layouts):
 *
 *   D[m,n] = sum_kb  sA[m,kb] * sB[n/128,kb] * ( sum_{k in block kb} A[m,k] * B[n,k] )
 *
 * with A [M,K] and B [N,K] both K-major E4M3 ("NT": D = A * B^T), one FP32
 * scale per row per 128-wide K-block for A and one per 128x128 block for B.
 * The oracle evaluates this definition directly in FP64:
 *   - E4M3 bytes are decoded through a 256-entry table built from the bit-field
 *     definition (sign, 4-bit exponent with bias 7, 3-bit mantissa,
 *     subnormals at exponent 0, NaN at S.1111.111, no infinities);
 *   - each 128-wide block sum is accumulated in FP64.  Every product of two
 *     E4M3 values has at most 8 significant bits and lies in [2^-18, 2^17.6],
 *     so 128 of them span fewer than 44 bits and the block sum is EXACT;
 *   - the block sum is then scaled by (double)sA * (double)sB and added to an
 *     FP64 accumulator.
 * The result is FP64 (no BF16 rounding); callers round or compare with a
 * tolerance.
 *
 * Layout conventions (the C ABI's):
 *   sfa: element (row r, K-block kb) at sfa[kb * ld_sfa + r]  ("MN-major");
 *        masked layout: group g at sfa + g * KB * ld_sfa.
 *   sfb: element (N-block j, K-block kb) at sfb[(g * NB + j) * KB + kb].
 *   b:   group g at b + g * N * K.
 *
 * Pins (tests/test_oracle.py): the decode table against torch's float8 cast
 * and closed-form values; brute force on tiny shapes; the all-ones-scale case
 * against a float64 matmul; exact integer cases with power-of-two scales
 * against exact integer arithmetic; identity and zero operands; scale
 * linearity; grouped == per-group dense; K-grouped: the groups' outputs sum
 * to the dense GEMM over all of K (exactly, for integer cases), one group ==
 * dense, an empty group gives zeros, brute force on tiny shapes.  BF16 GEMM:
 * exact brute force, exact integer cases, grouped == per-group dense.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define ORC_BLOCK 128

/* E4M3 ("fn") decode table from the bit-field definition. */
void oracle_e4m3_table(double lut[256])
{
    for (int code = 0; code < 256; ++code) {
        int sign = (code >> 7) & 1;
        int exponent = (code >> 3) & 0xF;
        int mantissa = code & 0x7;
        double v;
        if (exponent == 0xF && mantissa == 0x7) {
            v = NAN;
        } else if (exponent == 0) {
            v = ldexp((double)mantissa / 8.0, 1 - 7);          /* subnormal */
        } else {
            v = ldexp(1.0 + (double)mantissa / 8.0, exponent - 7);
        }
        lut[code] = sign ? -v : v;
    }
}

/* One output element by the definition above.
 *   arow: K bytes of A's row; sa: that row's scale for K-block 0, with
 *   consecutive K-blocks sa_stride apart; brow: K bytes of B's row; sb: the
 *   scale of B's 128-row block for K-block 0, consecutive K-blocks 1 apart. */
static double block_scaled_dot(const uint8_t *arow, const float *sa, long sa_stride,
                               const uint8_t *brow, const float *sb, long K,
                               const double *lut)
{
    double acc = 0.0;
    long KB = K / ORC_BLOCK;
    for (long kb = 0; kb < KB; ++kb) {
        double p = 0.0;
        const uint8_t *ak = arow + kb * ORC_BLOCK;
        const uint8_t *bk = brow + kb * ORC_BLOCK;
        for (int i = 0; i < ORC_BLOCK; ++i)
            p += lut[ak[i]] * lut[bk[i]];
        acc += ((double)sa[kb * sa_stride] * (double)sb[kb]) * p;
    }
    return acc;
}

static int check_shape(long M, long N, long K)
{
    if (M < 0 || N <= 0 || K <= 0 || K % ORC_BLOCK != 0) return 1;
    return 0;
}

/* Dense: d[m*N + n] for all m < M, n < N.  Returns 0 on success. */
int oracle_fp8_gemm_nt(const uint8_t *a, const float *sfa, long ld_sfa,
                       const uint8_t *b, const float *sfb,
                       long M, long N, long K, double *d)
{
    if (check_shape(M, N, K)) return 1;
    double lut[256];
    oracle_e4m3_table(lut);
    long KB = K / ORC_BLOCK;
    #pragma omp parallel for schedule(dynamic, 1)
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n)
            d[m * N + n] = block_scaled_dot(a + m * K, sfa + m, ld_sfa,
                                            b + n * K, sfb + (n / ORC_BLOCK) * KB, K, lut);
    return 0;
}

/* M-grouped contiguous: row m belongs to group m_indices[m]; rows with a
 * negative index are padding and their outputs are not written. */
int oracle_m_grouped_contiguous(const uint8_t *a, const float *sfa, long ld_sfa,
                                const uint8_t *b, const float *sfb,
                                const int32_t *m_indices,
                                long M_total, long N, long K, long G, double *d)
{
    if (check_shape(M_total, N, K) || G <= 0) return 1;
    double lut[256];
    oracle_e4m3_table(lut);
    long KB = K / ORC_BLOCK, NB = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    for (long m = 0; m < M_total; ++m)
        if (m_indices[m] >= G) return 2;
    #pragma omp parallel for schedule(dynamic, 1)
    for (long m = 0; m < M_total; ++m) {
        long g = m_indices[m];
        if (g < 0) continue;
        for (long n = 0; n < N; ++n)
            d[m * N + n] = block_scaled_dot(a + m * K, sfa + m, ld_sfa,
                                            b + (g * N + n) * K,
                                            sfb + (g * NB + n / ORC_BLOCK) * KB, K, lut);
    }
    return 0;
}

/* M-grouped masked: a is [G, Mmax, K]; group g's rows m < masked_m[g] are
 * computed into d[(g*Mmax + m)*N + n]; other rows are not written. */
int oracle_m_grouped_masked(const uint8_t *a, const float *sfa, long ld_sfa,
                            const uint8_t *b, const float *sfb,
                            const int32_t *masked_m,
                            long G, long Mmax, long N, long K, double *d)
{
    if (check_shape(Mmax, N, K) || G <= 0) return 1;
    double lut[256];
    oracle_e4m3_table(lut);
    long KB = K / ORC_BLOCK, NB = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    for (long g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > Mmax) return 2;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long g = 0; g < G; ++g)
        for (long m = 0; m < Mmax; ++m) {
            if (m >= masked_m[g]) continue;
            const uint8_t *arow = a + (g * Mmax + m) * K;
            const float *sa = sfa + g * KB * ld_sfa + m;
            for (long n = 0; n < N; ++n)
                d[(g * Mmax + m) * N + n] =
                    block_scaled_dot(arow, sa, ld_sfa, b + (g * N + n) * K,
                                     sfb + (g * NB + n / ORC_BLOCK) * KB, K, lut);
        }
    return 0;
}

/* Sampled outputs, for problems too large to evaluate in full.
 * Point i is (grp[i], row[i], col[i]); the meaning of grp/row follows the
 * layout:  layout 0 dense (grp ignored, row < M), 1 contiguous (grp ignored,
 * the group is m_indices[row]; padding rows give NaN), 2 masked (group grp,
 * row < Mmax; rows >= masked_m[grp] give NaN).  rows_a is M (dense),
 * M_total (contiguous) or Mmax (masked). */
int oracle_points(int layout, const uint8_t *a, const float *sfa, long ld_sfa,
                  const uint8_t *b, const float *sfb, const int32_t *m_indices,
                  const int32_t *masked_m, long G, long rows_a, long N, long K,
                  long npts, const int32_t *grp, const int32_t *row,
                  const int32_t *col, double *out)
{
    if (check_shape(rows_a, N, K)) return 1;
    double lut[256];
    oracle_e4m3_table(lut);
    long KB = K / ORC_BLOCK, NB = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    for (long i = 0; i < npts; ++i) {
        long r = row[i], n = col[i];
        if (r < 0 || r >= rows_a || n < 0 || n >= N) return 2;
        if (layout == 2 && (grp[i] < 0 || grp[i] >= G)) return 2;
    }
    #pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < npts; ++i) {
        long r = row[i], n = col[i], g;
        const uint8_t *arow;
        const float *sa;
        if (layout == 0) {
            g = 0; arow = a + r * K; sa = sfa + r;
        } else if (layout == 1) {
            g = m_indices[r];
            if (g < 0 || g >= G) { out[i] = NAN; continue; }
            arow = a + r * K; sa = sfa + r;
        } else {
            g = grp[i];
            if (r >= masked_m[g]) { out[i] = NAN; continue; }
            arow = a + (g * rows_a + r) * K; sa = sfa + g * KB * ld_sfa + r;
        }
        out[i] = block_scaled_dot(arow, sa, ld_sfa, b + (g * N + n) * K,
                                  sfb + (g * NB + n / ORC_BLOCK) * KB, K, lut);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * K-grouped GEMM (DeepGEMM page 3 "核心功能": the k_grouped_gemm family next to
 * the m-grouped one -- groups laid out along K, the weight-gradient shape of
 * MoE training, where the reduced dimension is each expert's tokens).
 *
 * Group g owns ks[g] consecutive K columns (ks[g] % 128 == 0, sum = K), i.e.
 * the K-blocks [o_g, o_g + ks[g]/128) with o_g the exclusive prefix of
 * ks/128, of both A [M,K] and B [N,K] and of their scales (the dense layout's
 * sfa [KB][ld_sfa] and sfb [NB][KB]).  Each group has its own output:
 *
 *   D[g][m][n] = sum_{kb in group g} sA[m,kb] * sB[n/128,kb] * (A_blk . B_blk)
 *
 * -- the dense definition restricted to the group's K-blocks; an empty group
 * gives zeros.
 * ------------------------------------------------------------------------ */
static int check_ks(const int32_t *ks, long G, long K)
{
    long sum = 0;
    for (long g = 0; g < G; ++g) {
        if (ks[g] < 0 || ks[g] % ORC_BLOCK != 0) return 2;
        sum += ks[g];
    }
    return sum == K ? 0 : 2;
}

int oracle_k_grouped(const uint8_t *a, const float *sfa, long ld_sfa,
                     const uint8_t *b, const float *sfb, const int32_t *ks,
                     long G, long M, long N, long K, double *d)
{
    if (check_shape(M, N, K) || G <= 0) return 1;
    if (check_ks(ks, G, K)) return 2;
    double lut[256];
    oracle_e4m3_table(lut);
    long KB = K / ORC_BLOCK;
    long off = 0;
    for (long g = 0; g < G; ++g) {
        const long kb0 = off / ORC_BLOCK, Kg = ks[g];
        #pragma omp parallel for schedule(dynamic, 1)
        for (long m = 0; m < M; ++m)
            for (long n = 0; n < N; ++n)
                d[(g * M + m) * N + n] =
                    Kg == 0 ? 0.0
                            : block_scaled_dot(a + m * K + kb0 * ORC_BLOCK, sfa + kb0 * ld_sfa + m, ld_sfa,
                                               b + n * K + kb0 * ORC_BLOCK,
                                               sfb + (n / ORC_BLOCK) * KB + kb0, Kg, lut);
        off += Kg;
    }
    return 0;
}

/* Sampled outputs D[grp[i]][row[i]][col[i]] of the K-grouped GEMM. */
int oracle_k_grouped_points(const uint8_t *a, const float *sfa, long ld_sfa,
                            const uint8_t *b, const float *sfb, const int32_t *ks,
                            long G, long M, long N, long K, long npts,
                            const int32_t *grp, const int32_t *row, const int32_t *col,
                            double *out)
{
    if (check_shape(M, N, K) || G <= 0) return 1;
    if (check_ks(ks, G, K)) return 2;
    for (long i = 0; i < npts; ++i)
        if (grp[i] < 0 || grp[i] >= G || row[i] < 0 || row[i] >= M || col[i] < 0 || col[i] >= N)
            return 3;
    double lut[256];
    oracle_e4m3_table(lut);
    long KB = K / ORC_BLOCK;
    #pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < npts; ++i) {
        long g = grp[i], m = row[i], n = col[i], off = 0;
        for (long h = 0; h < g; ++h) off += ks[h];
        const long kb0 = off / ORC_BLOCK, Kg = ks[g];
        out[i] = Kg == 0 ? 0.0
                         : block_scaled_dot(a + m * K + kb0 * ORC_BLOCK, sfa + kb0 * ld_sfa + m, ld_sfa,
                                            b + n * K + kb0 * ORC_BLOCK,
                                            sfb + (n / ORC_BLOCK) * KB + kb0, Kg, lut);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * BF16 GEMM (DeepGEMM page 3 "核心功能": FP8, FP4 and BF16 GEMMs), NT like
 * the FP8 one, no block scales:
 *
 *   D[m,n] = sum_k A[m,k] * B[n,k]          (A [M,K], B [N,K] BF16, K-major)
 *
 * evaluated in FP64 (the BF16 values widened exactly; each product of two
 * BF16 values is exact in FP64, the sum is FP64); callers round to BF16 or
 * compare with a tolerance.  Layouts as for FP8: dense; M-grouped contiguous
 * (row m uses B[m_indices[m]], rows with a negative index untouched); masked
 * (a [G][Mmax][K], rows m < masked_m[g]).
 * ------------------------------------------------------------------------ */
static double bf16_value(uint16_t bits)
{
    union { uint32_t u; float f; } v;
    v.u = (uint32_t)bits << 16;
    return (double)v.f;
}

static double bf16_dot(const uint16_t *arow, const uint16_t *brow, long K)
{
    double acc = 0.0;
    for (long k = 0; k < K; ++k)
        acc += bf16_value(arow[k]) * bf16_value(brow[k]);
    return acc;
}

/* layout 0 dense, 1 contiguous (m_indices), 2 masked (masked_m); rows_a is M,
 * M_total or Mmax.  Output d [rows][N] (masked: [G][Mmax][N]); rows that the
 * layout does not compute are left as they are. */
int oracle_bf16_gemm_nt(int layout, const uint16_t *a, const uint16_t *b,
                        const int32_t *m_indices, const int32_t *masked_m,
                        long G, long rows_a, long N, long K, double *d)
{
    if (rows_a < 0 || N <= 0 || K <= 0 || G <= 0) return 1;
    if (layout == 1)
        for (long m = 0; m < rows_a; ++m)
            if (m_indices[m] >= G) return 2;
    if (layout == 2)
        for (long g = 0; g < G; ++g)
            if (masked_m[g] < 0 || masked_m[g] > rows_a) return 2;
    long groups = layout == 2 ? G : 1;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long g = 0; g < groups; ++g)
        for (long m = 0; m < rows_a; ++m) {
            long bg = 0;
            if (layout == 1) {
                if (m_indices[m] < 0) continue;
                bg = m_indices[m];
            } else if (layout == 2) {
                if (m >= masked_m[g]) continue;
                bg = g;
            }
            const uint16_t *arow = a + (g * rows_a + m) * K;
            for (long n = 0; n < N; ++n)
                d[(g * rows_a + m) * N + n] = bf16_dot(arow, b + (bg * N + n) * K, K);
        }
    return 0;
}

/* ------------------------------------------------------------------------
 * Per-token 1x128 activation quantiser (the step that produces A and sA;
 * DeepGEMM page 2 "技术特性": fine-grained scaling, each small block with its
 * own scale; page 3 "精细粒度缩放": block-wise instead of tensor-wise).
 *
 * For row m and K-block kb of x [M][K] (values given as FP32, the exact BF16
 * inputs widened):
 *   amax = max |x[m, kb*128 .. kb*128+127]|          (exact)
 *   s    = fl32(amax / 448), or 1 when amax == 0     (one FP32 rounding)
 *   q    = E4M3_RNE(clamp(fl32(x / s), -448, 448))   (FP32 division, then RNE)
 * s is stored at sfa[kb * ld_sfa + m] (MN-major), q at q[m * K + k].
 * ------------------------------------------------------------------------ */

/* Round a finite float to the nearest E4M3 ("fn") value, ties to even; the
 * input must already lie in [-448, 448].  From the bit-field definition: a
 * value with exponent e >= -6 has 3 fraction bits (spacing 2^(e-3)); below
 * 2^-6 the spacing is the subnormal step 2^-9. */
uint8_t oracle_e4m3_encode(float x)
{
    uint8_t sign = (x < 0.0f || (x == 0.0f && signbit(x))) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) -> exponent e-1 */
    int exp2 = e - 1;
    if (exp2 < -6) exp2 = -6;     /* subnormal range: fixed spacing 2^-9 */
    double spacing = ldexp(1.0, exp2 - 3);
    double units = a / spacing;   /* exact: a power-of-two rescale */
    double lo = floor(units);
    double frac = units - lo;
    double r = lo;
    if (frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0)) r = lo + 1.0;
    if (r == 0.0) return sign;    /* rounds to a signed zero */
    double v = r * spacing;       /* may carry into the next binade: still exact */
    /* encode v (0 < v <= 448) */
    int ve;
    frexp(v, &ve);
    int vexp = ve - 1;
    uint8_t code;
    if (vexp < -6) {
        code = (uint8_t)(v / ldexp(1.0, -9));                 /* subnormal mantissa */
    } else {
        int mant = (int)((v / ldexp(1.0, vexp) - 1.0) * 8.0);
        code = (uint8_t)(((vexp + 7) << 3) | mant);
    }
    return (uint8_t)(sign | code);
}

int oracle_quantize_1x128(const float *x, long M, long K, uint8_t *q, float *sfa, long ld_sfa)
{
    if (M < 0 || K <= 0 || K % ORC_BLOCK != 0 || ld_sfa < M) return 1;
    long KB = K / ORC_BLOCK;
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        for (long kb = 0; kb < KB; ++kb) {
            const float *xb = x + m * K + kb * ORC_BLOCK;
            float amax = 0.0f;
            for (int i = 0; i < ORC_BLOCK; ++i) {
                float v = fabsf(xb[i]);
                if (v > amax) amax = v;
            }
            float s = amax / 448.0f;
            if (amax == 0.0f) s = 1.0f;
            sfa[kb * ld_sfa + m] = s;
            for (int i = 0; i < ORC_BLOCK; ++i) {
                float t = xb[i] / s;
                if (t > 448.0f) t = 448.0f;
                if (t < -448.0f) t = -448.0f;
                q[m * K + kb * ORC_BLOCK + i] = oracle_e4m3_encode(t);
            }
        }
    }
    return 0;
}
