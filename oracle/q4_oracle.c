/*
 * Q4 oracle: plain, slow, scalar CPU implementation of the 4-bit symmetric
 * group-32 weight format and of the products against it.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no source with the CUDA library.
 *
 * What the pages fix (QORA-4B thread on zingnex.cn, section "量化与内存管理";
 * QORA-LLM-0.8B model card, section "Weight Format"): weights are quantised to
 * 4 bits, symmetrically, in groups of 32 along the reduction axis, with one
 * scale per group, and GEMV/GEMM run against the dequantised values.  What
 * they leave open (divisor, rounding, storage) is fixed by the format
 * definition this library implements:
 *
 *   amax  = max_j |w_j| over the 32 f32 values of a group     (exact)
 *   s32   = amax / 7                                          (f32, round-to-nearest-even)
 *   s     = binary16(s32)                                     (round-to-nearest-even)
 *   s == 0           -> every code is 8 (bytes 0x88), scale bits 0x0000
 *   otherwise q_j    = clamp(rint(w_j / f32(s)), -8, 7)       (f32 division, ties to even)
 *   stored nibble    = q_j + 8, byte k/2 = nib[2i] | nib[2i+1] << 4 (low nibble = even k)
 *   dequantised w'_j = (nib_j - 8) * f32(s)
 *
 * The quotient uses the STORED binary16 scale, so |w - w'| <= s/2 holds against
 * the scale that is actually stored.  A group holding a NaN or an infinity, or
 * whose scale overflows binary16, is encoded as a zero group and reported in a
 * flag word (bit 0: non-finite input, bit 1: scale overflow).
 *
 * Products (QORA-LLM-0.8B model card, "Weight Format" and "File Structure":
 * GEMV/GEMM against Q4 weights): y[m,n] = sum_k x[m,k] * w'[n,k], every term
 * and the running sum in IEEE binary64, k in increasing order.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 * No SIMD intrinsics; the only parallelism is an OpenMP loop over output rows,
 * which does not change any result.
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_FLAG_NONFINITE 1u
#define ORACLE_FLAG_SCALE_OVERFLOW 2u

/* ---- IEEE-754 binary16 <-> binary32, written out from the bit layouts ----
 * binary32: 1 sign, 8 exponent (bias 127), 23 fraction bits.
 * binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits; subnormal unit 2^-24.
 */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t bexp = (x >> 23) & 0xFFu;
    uint32_t frac = x & 0x7FFFFFu;

    if (bexp == 0xFFu) {                      /* infinity or NaN */
        if (frac == 0) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | 0x7E00u | (frac >> 13));   /* quiet NaN */
    }
    if (bexp == 0) return (uint16_t)sign;     /* |f| < 2^-126: far below half of 2^-24 */

    int e = (int)bexp - 127;                  /* value = 1.frac * 2^e */
    if (e > 15) return (uint16_t)(sign | 0x7C00u);

    if (e >= -14) {                           /* binary16 normal range */
        uint32_t h = ((uint32_t)(e + 15) << 10) | (frac >> 13);
        uint32_t rem = frac & 0x1FFFu;        /* 13 dropped bits; half = 0x1000 */
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1;  /* carry may reach inf */
        return (uint16_t)(sign | h);
    }

    /* binary16 subnormal: count of 2^-24 units = m * 2^(e+1), m the 24-bit significand */
    uint32_t m = frac | 0x800000u;
    int shift = -(e + 1);                     /* >= 14 here */
    if (shift > 24) return (uint16_t)sign;    /* below 2^-25: rounds to zero */
    uint32_t h = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (h & 1u))) h += 1;   /* may become the smallest normal */
    return (uint16_t)(sign | h);
}

float oracle_f16_to_f32(uint16_t h)
{
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t bexp = ((uint32_t)h >> 10) & 0x1Fu;
    uint32_t frac = (uint32_t)h & 0x3FFu;
    float out;
    if (bexp == 0) {
        out = ldexpf((float)frac, -24);       /* exact: frac < 2^10 */
        if (sign) out = -out;
        return out;
    }
    uint32_t x;
    if (bexp == 0x1Fu) x = sign | 0x7F800000u | (frac << 13);
    else x = sign | ((bexp - 15u + 127u) << 23) | (frac << 13);
    memcpy(&out, &x, sizeof out);
    return out;
}

/* bfloat16 is the top half of a binary32. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t x = (uint32_t)b << 16;
    float out;
    memcpy(&out, &x, sizeof out);
    return out;
}

void oracle_f32_to_f16_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(in[i]);
}

void oracle_f16_to_f32_array(const uint16_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(in[i]);
}

/* ---- quantiser ---- */

static void encode_zero_group(uint8_t* bytes, uint16_t* scale)
{
    for (int i = 0; i < 16; ++i) bytes[i] = 0x88u;   /* nibble 8 == code 0 */
    *scale = 0;
}

/* Quantise one group of 32 consecutive weights; returns flag bits. */
static uint32_t quantize_group(const float* w, uint8_t* bytes, uint16_t* scale)
{
    int nonfinite = 0;
    float amax = 0.0f;
    for (int j = 0; j < 32; ++j) {
        if (!isfinite(w[j])) nonfinite = 1;
        float a = fabsf(w[j]);
        if (a > amax) amax = a;
    }
    if (nonfinite) { encode_zero_group(bytes, scale); return ORACLE_FLAG_NONFINITE; }

    volatile float s32 = amax / 7.0f;         /* one IEEE f32 division */
    uint16_t sbits = oracle_f32_to_f16(s32);
    if ((sbits & 0x7FFFu) == 0x7C00u) { encode_zero_group(bytes, scale); return ORACLE_FLAG_SCALE_OVERFLOW; }
    if ((sbits & 0x7FFFu) == 0) { encode_zero_group(bytes, scale); return 0; }

    float sf = oracle_f16_to_f32(sbits);
    int nib[32];
    for (int j = 0; j < 32; ++j) {
        volatile float t = w[j] / sf;         /* f32 quotient by the stored scale */
        float r = nearbyintf(t);              /* current mode: to nearest, ties to even */
        int q = (int)r;
        if (q < -8) q = -8;
        if (q > 7) q = 7;
        nib[j] = q + 8;
    }
    for (int i = 0; i < 16; ++i) bytes[i] = (uint8_t)(nib[2 * i] | (nib[2 * i + 1] << 4));
    *scale = sbits;
    return 0;
}

/* W: f32 [N,K] row-major; packed: [N,K/2]; scales: binary16 bits [N,K/32].
 * Returns -1 if K is not a multiple of 32, else 0.  *flags gets the OR of all groups' flags. */
int oracle_q4_quantize(const float* W, int64_t N, int64_t K,
                       uint8_t* packed, uint16_t* scales, uint32_t* flags)
{
    if (K % 32 != 0 || N < 0) return -1;
    fesetround(FE_TONEAREST);
    uint32_t f = 0;
    int64_t G = K / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            f |= quantize_group(W + n * K + g * 32, packed + n * (K / 2) + g * 16, scales + n * G + g);
    if (flags) *flags = f;
    return 0;
}

/* Dequantised weight of row n, column k, exactly: (nibble - 8) * f32(scale). */
static double dequant_one(const uint8_t* packed, const uint16_t* scales, int64_t K, int64_t n, int64_t k)
{
    uint8_t byte = packed[n * (K / 2) + k / 2];
    int nibble = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    double s = (double)oracle_f16_to_f32(scales[n * (K / 32) + k / 32]);
    return (double)(nibble - 8) * s;
}

void oracle_q4_dequant(const uint8_t* packed, const uint16_t* scales, int64_t N, int64_t K, double* Wd)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            Wd[n * K + k] = dequant_one(packed, scales, K, n, k);
}

static double x_value(const void* x, int x_is_bf16, int64_t idx)
{
    if (x_is_bf16) return (double)oracle_bf16_to_f32(((const uint16_t*)x)[idx]);
    return (double)((const float*)x)[idx];
}

/* y[m, j] = sum_k x[m,k] * w'[rows[j], k] in binary64, k ascending.
 * x: [M,K] f32 (x_is_bf16 == 0) or bfloat16 bits (x_is_bf16 == 1), row-major.
 * rows: output rows to compute (NULL = all N rows, then nrows must equal N).
 * y: binary64 [M, nrows] row-major.  Each weight row is dequantised once into a
 * binary64 buffer and then dotted with every x row.  Returns -1 on allocation
 * failure, else 0. */
int oracle_q4_matmul_rows(const void* x, int x_is_bf16, int64_t M, int64_t K,
                          const uint8_t* packed, const uint16_t* scales,
                          const int64_t* rows, int64_t nrows, double* y, int nthreads)
{
    int failed = 0;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
    #pragma omp parallel num_threads(nthreads)
#else
    (void)nthreads;
#endif
    {
        double* wrow = (double*)malloc((size_t)(K > 0 ? K : 1) * sizeof(double));
        if (!wrow) {
#ifdef _OPENMP
            #pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
        #pragma omp for schedule(dynamic, 16)
#endif
        for (int64_t j = 0; j < nrows; ++j) {
            if (!wrow) continue;
            int64_t n = rows ? rows[j] : j;
            for (int64_t k = 0; k < K; ++k) wrow[k] = dequant_one(packed, scales, K, n, k);
            for (int64_t m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += x_value(x, x_is_bf16, m * K + k) * wrow[k];
                y[m * nrows + j] = acc;
            }
        }
        free(wrow);
    }
    return failed ? -1 : 0;
}

int oracle_q4_matmul(const void* x, int x_is_bf16, int64_t M, int64_t K,
                     const uint8_t* packed, const uint16_t* scales, int64_t N,
                     double* y, int nthreads)
{
    return oracle_q4_matmul_rows(x, x_is_bf16, M, K, packed, scales, NULL, N, y, nthreads);
}

/* Fused gate+up of the MLP (QORA-LLM-0.8B model card, section "AVX-512 SIMD
 * Acceleration": "Fused gate+up", the gate and up projections decoded in one pass).
 * The activation is not named there; the model card's only activation is SiLU, so
 * the gated product is taken as SwiGLU's:
 *     y[m, j] = silu(g[m, j]) * u[m, j],   silu(g) = g / (1 + exp(-g)),
 * with g = x . dequant(Wg)^T and u = x . dequant(Wu)^T from oracle_q4_matmul_rows,
 * everything in binary64.  rows, nrows, y and nthreads as for oracle_q4_matmul_rows.
 * Returns -1 on allocation failure, else 0. */
int oracle_q4_gate_up_rows(const void* x, int x_is_bf16, int64_t M, int64_t K,
                           const uint8_t* gate_packed, const uint16_t* gate_scales,
                           const uint8_t* up_packed, const uint16_t* up_scales,
                           const int64_t* rows, int64_t nrows, double* y, int nthreads)
{
    const size_t count = (size_t)(M * nrows > 0 ? M * nrows : 1);
    double* g = (double*)malloc(count * sizeof(double));
    double* u = (double*)malloc(count * sizeof(double));
    int rc = (g && u) ? 0 : -1;
    if (rc == 0) rc = oracle_q4_matmul_rows(x, x_is_bf16, M, K, gate_packed, gate_scales, rows, nrows, g, nthreads);
    if (rc == 0) rc = oracle_q4_matmul_rows(x, x_is_bf16, M, K, up_packed, up_scales, rows, nrows, u, nthreads);
    if (rc == 0)
        for (int64_t i = 0; i < M * nrows; ++i) y[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
    free(g);
    free(u);
    return rc;
}

/* F16-weight GEMV, the pages' second weight format (QORA-LLM-0.8B model card, section
 * "AVX-512 SIMD Acceleration": "F16 GEMV", binary16 weights widened to f32 and
 * multiply-added; section "File Structure": Q4/F16 GEMV kernels):
 *     y[m, n] = sum_k x[m, k] * w[n, k],   w binary16 bits [N, K] row-major,
 * every term and the running sum in binary64, k ascending (binary16 widens exactly).
 * x, M, K, y and nthreads as for oracle_q4_matmul. */
int oracle_f16_matmul(const void* x, int x_is_bf16, int64_t M, int64_t K, const uint16_t* w, int64_t N,
                      double* y, int nthreads)
{
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
    #pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads)
#else
    (void)nthreads;
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += x_value(x, x_is_bf16, m * K + k) * (double)oracle_f16_to_f32(w[n * K + k]);
            y[m * N + n] = acc;
        }
    }
    return 0;
}

/* ---- INT8 weights: the second half of a mixed INT8/INT4 model ----
 * The QKV-Core thread (zingnex.cn, section "自适应混合量化") quantises per layer: layers
 * that are sensitive to precision (attention) in INT8, the feed-forward layers in INT4.
 * It gives no encoding.  The reading taken here is the Q4 format above with 8-bit codes:
 *
 *   s32 = amax / 127                                  (f32, round-to-nearest-even)
 *   s   = binary16(s32)                               (round-to-nearest-even)
 *   s == 0            -> every code 0, scale bits 0x0000
 *   otherwise q_j     = clamp(rint(w_j / f32(s)), -128, 127)   (f32 division, ties to even)
 *   stored byte k     = q_k as a two's-complement int8, codes [N, K] row-major
 *   dequantised w'_j  = q_j * f32(s)
 *
 * The divisor is the largest positive code and the clamp is the whole code range, as
 * 7 and [-8, 7] are for Q4: -128 is reached only when rounding the scale to binary16
 * lowers it by more than half a code (subnormal scales).  Non-finite input and scale
 * overflow give a zero group and the same flag bits as Q4. */
static uint32_t quantize_group_q8(const float* w, int8_t* codes, uint16_t* scale)
{
    int nonfinite = 0;
    float amax = 0.0f;
    for (int j = 0; j < 32; ++j) {
        if (!isfinite(w[j])) nonfinite = 1;
        float a = fabsf(w[j]);
        if (a > amax) amax = a;
    }
    uint32_t flag = 0;
    uint16_t sbits = 0;
    if (nonfinite) {
        flag = ORACLE_FLAG_NONFINITE;
    } else {
        volatile float s32 = amax / 127.0f;   /* one IEEE f32 division */
        sbits = oracle_f32_to_f16(s32);
        if ((sbits & 0x7FFFu) == 0x7C00u) flag = ORACLE_FLAG_SCALE_OVERFLOW;
    }
    if (flag || (sbits & 0x7FFFu) == 0) {
        for (int j = 0; j < 32; ++j) codes[j] = 0;
        *scale = 0;
        return flag;
    }
    float sf = oracle_f16_to_f32(sbits);
    for (int j = 0; j < 32; ++j) {
        volatile float t = w[j] / sf;         /* f32 quotient by the stored scale */
        int q = (int)nearbyintf(t);           /* current mode: to nearest, ties to even */
        if (q < -128) q = -128;
        if (q > 127) q = 127;
        codes[j] = (int8_t)q;
    }
    *scale = sbits;
    return 0;
}

/* W: f32 [N,K] row-major; codes: int8 [N,K]; scales: binary16 bits [N,K/32].
 * Returns -1 if K is not a multiple of 32, else 0.  *flags gets the OR of all groups' flags. */
int oracle_q8_quantize(const float* W, int64_t N, int64_t K, int8_t* codes, uint16_t* scales, uint32_t* flags)
{
    if (K % 32 != 0 || N < 0) return -1;
    fesetround(FE_TONEAREST);
    uint32_t f = 0;
    int64_t G = K / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            f |= quantize_group_q8(W + n * K + g * 32, codes + n * K + g * 32, scales + n * G + g);
    if (flags) *flags = f;
    return 0;
}

/* y[m, n] = sum_k x[m,k] * w'[n,k] with w' = code * f32(scale), every term and the running
 * sum in binary64, k ascending.  x, M, K, y and nthreads as for oracle_q4_matmul. */
int oracle_q8_matmul(const void* x, int x_is_bf16, int64_t M, int64_t K, const int8_t* codes,
                     const uint16_t* scales, int64_t N, double* y, int nthreads)
{
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
    #pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads)
#else
    (void)nthreads;
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const double s = (double)oracle_f16_to_f32(scales[n * (K / 32) + k / 32]);
                acc += x_value(x, x_is_bf16, m * K + k) * ((double)codes[n * K + k] * s);
            }
            y[m * N + n] = acc;
        }
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
