/*
 * oracle.c -- CPU oracle for microscaling FP4 quantization and the W4A4
 * block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this file.  Only the test suite, the smoke check of the entry
 * module and the CPU-baseline leg of the benchmark use it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Every routine is the plain definition, written element by element in the
 * order the pages state it.  Floating point follows IEEE-754 binary32/64 with
 * round-to-nearest-even; the file must be compiled with -ffp-contract=off and
 * without -ffast-math so that each float expression is rounded exactly once.
 *
 * Sources (web pages, by title and section):
 *  [NVFP4-Arch]  "NVFP4 Architecture: Microscaling & 4-Bit LLMs on Blackwell"
 *                - "1. The E2M1 Floating-Point Format" (value set, code table)
 *                - "2. Micro-Block Exponent Scaling: E8M0 Format" (S = 2^(E-127))
 *                - "1. The Dual-Level Mathematical Formulation" (S_global,
 *                  S_block,j, q_i, reconstruction x_hat)
 *                - "2. Hardware-Managed Tensor Core Dot-Products" (16-element
 *                  dot products scaled by S_u*S_v, FP32 accumulation)
 *                - "End-to-End Implementation: Emulating NVFP4 & Microscaling
 *                  in PyTorch" (block amax, 1e-8 clamp, ceil(log2(amax/6)),
 *                  nearest-value quantization, naive per-tensor baseline)
 *  [ia4pymes]    "NVIDIA NVFP4 quantization ..." - "The Physics of NVFP4:
 *                Block-Wise Microscaling Quantization" (16-element blocks,
 *                8-bit shared scale)
 *  [MXFP4-BW]    "How Microscaling FP4 (MXFP4) Halves Memory Bandwidth in
 *                Frontier Models Without Training Divergence"
 *                - "The Representation Dilemma: E2M1 vs. E3M0" (saturation at 6)
 *                - "The Microscaling Breakthrough: 32-Element Blocks"
 *                - "Silicon Execution: Tensor Cores & Register Fusing"
 *  [MXFP4-kc]    "MXFP4" - "Core Facts" (E8M0 scale, block size 32)
 *
 * Readings where the pages are silent or disagree (each one is listed with its
 * reason in the design notes of the repository):
 *  - NVFP4 block scale is an unsigned E4M3 byte under an FP32 per-tensor scale
 *    S_global; it is rounded to nearest-even with saturation at 448.
 *  - S_global = amax(tensor) / (6 * 448) in FP32 (1 for an all-zero tensor).
 *  - Element rounding onto the E2M1 grid is round-to-nearest, ties to the code
 *    with an even mantissa bit, saturating at +-6; the sign bit of x is kept
 *    (so -0 and negative underflow encode as 0x8).
 *  - NVFP4 elements are multiplied by RN(1 / (E4M3(sb) * S_global)) rather than
 *    divided; MXFP4 elements are multiplied by the exact power of two 2^-e.
 *  - Two nibbles per byte, the even index in the low nibble.
 *  - Scales are stored in 128-row x 4-column tiles of 512 bytes (the layout
 *    the block-scaled tensor-core MMA reads); padding bytes are zero.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>
#include <float.h>

#define ORC_NVFP4 0     /* k = 16, unsigned E4M3 block scale, FP32 S_global */
#define ORC_MXFP4 1     /* k = 32, E8M0 block scale                        */
#define ORC_P1E8  2     /* k = 16, E8M0 block scale under S_global (the
                           dual-level formula exactly as [NVFP4-Arch] prints it) */

/* ------------------------------------------------------------------------ */
/* BF16 / FP32 bit helpers                                                   */
/* ------------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* E2M1 -- [NVFP4-Arch] "1. The E2M1 Floating-Point Format":                 */
/* 1 sign bit, 2 exponent bits, 1 mantissa bit; exponent field 0 encodes the */
/* subnormal m * 2^-1, otherwise (1 + m/2) * 2^(e-1).  Zero is signed.       */
/* ------------------------------------------------------------------------ */
double orc_e2m1_decode(uint8_t nib)
{
    int s = (nib >> 3) & 1;
    int e = (nib >> 1) & 3;
    int m = nib & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Round |v| to the nearest of the eight E2M1 magnitudes; on an exact tie pick
 * the code whose mantissa bit is 0 (round-to-nearest-even); |v| >= 6 (and
 * infinity) saturates to 6 ([MXFP4-BW] "E2M1 vs. E3M0": values beyond 6
 * saturate).  The sign bit of v is copied into bit 3. */
uint8_t orc_e2m1_encode(float v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (!(a < 6.0))
        return sign | 7;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - orc_e2m1_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* The rounding of the emulation script in [NVFP4-Arch] "End-to-End
 * Implementation": argmin over the codebook keeps the first (smaller)
 * magnitude on a tie.  Used only to count where it differs from the
 * nearest-even rule above. */
uint8_t orc_e2m1_encode_first_index_tie(float v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - orc_e2m1_decode((uint8_t)c));
        if (d < bestd) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------ */
/* E8M0 -- [NVFP4-Arch] "2. Micro-Block Exponent Scaling: E8M0 Format":      */
/* S = 2^(E - 127), E in [0, 255].                                          */
/* ------------------------------------------------------------------------ */
double orc_e8m0_decode(uint8_t byte)
{
    return ldexp(1.0, (int)byte - 127);
}

/* Block exponent of the emulation script ("Step 2"): amax is clamped to at
 * least 1e-8 (FP32), then e = ceil(log2(amax / 6)), i.e. the smallest integer
 * e with 6 * 2^e >= amax.  Searched directly, in exact double arithmetic. */
int orc_mx_exponent(float amax)
{
    float a = amax < 1e-8f ? 1e-8f : amax;
    for (int e = -200; e <= 200; ++e)
        if (ldexp(6.0, e) >= (double)a)
            return e;
    return 200; /* not reached for finite input */
}

uint8_t orc_e8m0_encode_block(float amax)
{
    return (uint8_t)(orc_mx_exponent(amax) + 127);
}

/* ------------------------------------------------------------------------ */
/* E4M3 (unsigned use as the NVFP4 block scale; [ia4pymes] "8-bit" scale).   */
/* 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0 encodes the   */
/* subnormal m/8 * 2^-6; code 0x7F is NaN; largest finite value 448.         */
/* ------------------------------------------------------------------------ */
double orc_e4m3_decode(uint8_t byte)
{
    int s = (byte >> 7) & 1;
    int e = (byte >> 3) & 15;
    int m = byte & 7;
    if (e == 15 && m == 7)
        return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest non-negative finite E4M3 value to t >= 0, ties to the even code
 * (even mantissa LSB), saturating at 448: plain search over all 127 codes. */
uint8_t orc_e4m3_encode_unsigned(float t)
{
    double a = (double)t;
    if (!(a < 448.0))
        return 0x7E;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(a - orc_e4m3_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* S_global -- [NVFP4-Arch] "1. The Dual-Level Mathematical Formulation",    */
/* item 1: a per-tensor scale representing the tensor's dynamic ceiling.    */
/* Reading: S_global = amax / (6 * 448) in FP32, so that the block with the  */
/* tensor's amax gets block scale 448 (the E4M3 maximum); 1 if amax == 0.    */
/* ------------------------------------------------------------------------ */
float orc_amax_bf16(const uint16_t* x, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_f32(x[i]));
        if (a > amax)
            amax = a;
    }
    return amax;
}

float orc_global_scale_from_amax(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    return amax / 2688.0f; /* 2688 = 6 * 448, exact in FP32 */
}

float orc_global_scale(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r) {
        float a = orc_amax_bf16(x + r * ld, cols);
        if (a > amax)
            amax = a;
    }
    return orc_global_scale_from_amax(amax);
}

/* ------------------------------------------------------------------------ */
/* Per-block scale.  Returns the stored scale byte and writes the multiplier */
/* applied to each element of the block.                                     */
/* ------------------------------------------------------------------------ */
static uint8_t block_scale(int fmt, float amax, float gs, float* inv_out)
{
    if (fmt == ORC_MXFP4) {
        /* S_block = 2^ceil(log2(amax / 6)) (no global scale in MXFP4). */
        int e = orc_mx_exponent(amax);
        *inv_out = ldexpf(1.0f, -e); /* exact: e in [-29, 126] */
        return (uint8_t)(e + 127);
    }
    if (fmt == ORC_P1E8) {
        /* S_block = 2^ceil(log2(amax / (6 * S_global))), exactly as printed:
         * the ratio amax / (6 * S_global) is formed in FP32 and the smallest
         * e with 2^e >= ratio is taken (ratio clamped like the script). */
        float denom = 6.0f * gs;
        float ratio = amax / denom;
        float a = ratio < 1e-8f ? 1e-8f : ratio;
        int e = -200;
        while (ldexp(1.0, e) < (double)a)
            ++e;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
        float eff = (float)ldexp(1.0, e) * gs;
        *inv_out = (eff == 0.0f) ? 0.0f : 1.0f / eff;
        if (isinf(*inv_out)) *inv_out = FLT_MAX;
        return (uint8_t)(e + 127);
    }
    /* NVFP4: t = amax / (6 * S_global) rounded to unsigned E4M3; the
     * effective block scale is E4M3(sb) * S_global; elements are multiplied
     * by its FP32 reciprocal (0 for an all-zero block). */
    float denom = 6.0f * gs;
    float t = amax / denom;
    uint8_t sb = orc_e4m3_encode_unsigned(t);
    float eff = (float)orc_e4m3_decode(sb) * gs;
    float inv;
    if (eff == 0.0f) {
        inv = 0.0f;
    } else {
        inv = 1.0f / eff;
        if (isinf(inv))
            inv = FLT_MAX;
    }
    *inv_out = inv;
    return sb;
}

int orc_block_size(int fmt)
{
    return fmt == ORC_MXFP4 ? 32 : 16;
}

/* Offset of scale (row, col) inside the tiled scale buffer: 128-row x 4-col
 * tiles of 512 bytes, column tiles fastest; inside a tile the byte for
 * (r, c) sits at (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4). */
int64_t orc_scale_offset(int64_t row, int64_t col, int64_t n_scale_cols)
{
    int64_t col_tiles = (n_scale_cols + 3) / 4;
    int64_t tile = (row / 128) * col_tiles + col / 4;
    return tile * 512 + (row % 32) * 16 + ((row / 32) % 4) * 4 + (col % 4);
}

int64_t orc_scale_bytes(int64_t rows, int64_t n_scale_cols)
{
    return ((rows + 127) / 128) * ((n_scale_cols + 3) / 4) * 512;
}

/* ------------------------------------------------------------------------ */
/* Quantizer.  axis 0 (rowwise): blocks of k consecutive elements along each */
/* row of x[rows x cols] (leading dimension ld); output row r holds row r.   */
/* axis 1 (colwise): blocks of k consecutive elements down each column;      */
/* output row c holds column c, i.e. the result is the transpose.           */
/* Outputs: packed[out_rows x K/2] (K = blocked length), scales in the tiled */
/* layout (zero padding), and optionally scales_rm[out_rows x K/k].          */
/* Steps follow the emulation script: block amax (Step 1), block scale       */
/* (Step 2), normalise (Step 3), nearest E2M1 value (Step 4).                */
/* ------------------------------------------------------------------------ */
int orc_quantize(int fmt, int axis, const uint16_t* x, int64_t rows, int64_t cols,
                 int64_t ld, float gs, uint8_t* packed, uint8_t* scales,
                 uint8_t* scales_rm)
{
    int k = orc_block_size(fmt);
    int64_t out_rows = axis == 0 ? rows : cols;
    int64_t K = axis == 0 ? cols : rows;
    if (K % k != 0 || K % 2 != 0)
        return -1;
    int64_t nsc = K / k;
    if (scales)
        memset(scales, 0, (size_t)orc_scale_bytes(out_rows, nsc));

    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < out_rows; ++i) {
        for (int64_t b = 0; b < nsc; ++b) {
            float xs[32];
            float amax = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t kk = b * k + j;
                uint16_t h = axis == 0 ? x[i * ld + kk] : x[kk * ld + i];
                xs[j] = bf16_to_f32(h);
                float a = fabsf(xs[j]);
                if (a > amax)
                    amax = a;
            }
            float inv;
            uint8_t sbyte = block_scale(fmt, amax, gs, &inv);
            if (scales)
                scales[orc_scale_offset(i, b, nsc)] = sbyte;
            if (scales_rm)
                scales_rm[i * nsc + b] = sbyte;
            for (int j = 0; j < k; j += 2) {
                uint8_t lo = orc_e2m1_encode(xs[j] * inv);
                uint8_t hi = orc_e2m1_encode(xs[j + 1] * inv);
                packed[i * (K / 2) + (b * k + j) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return 0;
}

/* Value of one stored block scale (without S_global). */
static double scale_value(int fmt, uint8_t byte)
{
    if (fmt == ORC_NVFP4)
        return orc_e4m3_decode(byte);
    return orc_e8m0_decode(byte);
}

/* Reconstruction x_hat = q * S_block (* S_global when gs != 0) of one
 * quantized row-major operand [rows x K] -- [NVFP4-Arch] "1. The Dual-Level
 * Mathematical Formulation", reconstruction line.  Output in FP64 (exact). */
void orc_dequantize(int fmt, const uint8_t* packed, const uint8_t* scales,
                    int64_t rows, int64_t K, double gs, double* out)
{
    int k = orc_block_size(fmt);
    int64_t nsc = K / k;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t kk = 0; kk < K; ++kk) {
            uint8_t byte = packed[i * (K / 2) + kk / 2];
            uint8_t nib = (kk & 1) ? (byte >> 4) : (byte & 15);
            double s = scale_value(fmt, scales[orc_scale_offset(i, kk / k, nsc)]);
            double v = orc_e2m1_decode(nib) * s;
            out[i * K + kk] = gs != 0.0 ? v * gs : v;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* GEMM -- [NVFP4-Arch] "2. Hardware-Managed Tensor Core Dot-Products" and   */
/* [MXFP4-BW] "Silicon Execution": per-block products of the E2M1 values,    */
/* scaled by the product of the two block scales, summed in high precision.  */
/* D[m,n] = alpha * sum_k (qA*SA)[m,k] * (qB*SB)[n,k], accumulated in FP64.  */
/* Also S[m,n] = |alpha| * sum_k |(qA*SA)[m,k] * (qB*SB)[n,k]| (tolerance).  */
/* A is [M x K] packed, B is [N x K] packed (both K-major), scales tiled.    */
/* Only the listed (m, n) pairs are computed.                               */
/* ------------------------------------------------------------------------ */
static double deq_elem(int fmt, const uint8_t* packed, const uint8_t* scales,
                       int64_t row, int64_t kk, int64_t K)
{
    int k = orc_block_size(fmt);
    uint8_t byte = packed[row * (K / 2) + kk / 2];
    uint8_t nib = (kk & 1) ? (byte >> 4) : (byte & 15);
    double s = scale_value(fmt, scales[orc_scale_offset(row, kk / k, K / k)]);
    return orc_e2m1_decode(nib) * s;
}

void orc_gemm_pairs(int fmt, const uint8_t* A, const uint8_t* sA,
                    const uint8_t* B, const uint8_t* sB, int64_t K, double alpha,
                    const int64_t* ms, const int64_t* ns, int64_t count,
                    double* D, double* S)
{
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t p = 0; p < count; ++p) {
        double acc = 0.0, mag = 0.0;
        for (int64_t kk = 0; kk < K; ++kk) {
            double prod = deq_elem(fmt, A, sA, ms[p], kk, K) *
                          deq_elem(fmt, B, sB, ns[p], kk, K);
            acc += prod;
            mag += fabs(prod);
        }
        D[p] = alpha * acc;
        S[p] = fabs(alpha) * mag;
    }
}

/* Full product over all (m, n) for small problems: the operands are first
 * reconstructed (same per-element definition as above), then each output is
 * one FP64 dot product. */
void orc_gemm(int fmt, const uint8_t* A, const uint8_t* sA, const uint8_t* B,
              const uint8_t* sB, int64_t M, int64_t N, int64_t K, double alpha,
              double* Adq, double* Bdq, double* D, double* S)
{
    orc_dequantize(fmt, A, sA, M, K, 0.0, Adq);
    orc_dequantize(fmt, B, sB, N, K, 0.0, Bdq);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t kk = 0; kk < K; ++kk) {
                double prod = Adq[m * K + kk] * Bdq[n * K + kk];
                acc += prod;
                mag += fabs(prod);
            }
            D[m * N + n] = alpha * acc;
            S[m * N + n] = fabs(alpha) * mag;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Naive per-tensor FP4 baseline of [NVFP4-Arch] "1. The Catastrophic Impact */
/* of Coarse-Grained 4-Bit Quantization" and the emulation script: one scale */
/* s = max(amax, 1e-8) / 6 for the whole tensor; returns q * s in FP64.      */
/* ------------------------------------------------------------------------ */
void orc_naive_per_tensor(const float* x, int64_t n, double* out)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i)
        if (fabsf(x[i]) > amax)
            amax = fabsf(x[i]);
    if (amax < 1e-8f)
        amax = 1e-8f;
    float s = amax / 6.0f;
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_e2m1_decode(orc_e2m1_encode(x[i] / s)) * (double)s;
}

/* Block quantize-dequantize of an FP32 vector with power-of-two block scales
 * (the emulation script's mxfp4_block_quantize / dequantize at any block
 * size; the vector is zero-padded to a whole number of blocks). */
void orc_block_pow2_roundtrip(const float* x, int64_t n, int k, int page_tie,
                              double* out)
{
    for (int64_t b0 = 0; b0 < n; b0 += k) {
        float amax = 0.0f;
        for (int j = 0; j < k && b0 + j < n; ++j)
            if (fabsf(x[b0 + j]) > amax)
                amax = fabsf(x[b0 + j]);
        int e = orc_mx_exponent(amax);
        float inv = ldexpf(1.0f, -e);
        for (int j = 0; j < k && b0 + j < n; ++j) {
            float v = x[b0 + j] * inv;
            uint8_t q = page_tie ? orc_e2m1_encode_first_index_tie(v) : orc_e2m1_encode(v);
            out[b0 + j] = orc_e2m1_decode(q) * ldexp(1.0, e);
        }
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Element-wise batch forms of the scalar encoders above (plain loops), so
 * that exhaustive checks do not pay one foreign call per value. */
void orc_e2m1_encode_n(const float* v, int64_t n, uint8_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_unsigned_n(const float* t, int64_t n, uint8_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_e4m3_encode_unsigned(t[i]);
}

void orc_mx_exponent_n(const float* a, int64_t n, int32_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_mx_exponent(a[i]);
}
