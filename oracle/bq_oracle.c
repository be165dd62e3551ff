/*
 * bq_oracle.c -- plain CPU oracle for weight-only block-quantized matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this code:
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * load it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (every step spelled out, no blocking, no fusion):
 *   y[M,N] = x[M,K] . dequant(Wq)[N,K]^T,  x and dequant(W) in bf16,
 *   accumulated in float64.
 * The equivalence "quantized_matmul(x, wq, ...) == x @ dequantize(wq, ...).T"
 * is the premise of "quantized_matmul takes 14-41% longer than dequantize +
 * bf16 matmul at prefill sizes (> 512 tokens)" (Summary, Repro).
 *
 * Formats:
 *  - Q4_0, the format of "et-backend: Q4_0 matrix-engine GEMM rewrite for
 *    prefill" (Overview) and "2026-05-06 Q4 sync-after focused repro"
 *    (Important source touch points).  The pages name it but do not print its
 *    layout; the ggml block format is used: 32 weights along K share one fp16
 *    scale d, w = d * (q - 8), q in [0, 15]; byte j of a block holds element
 *    j in its low nibble and element j + 16 in its high nibble.  Stored as two
 *    planes ("reordered" layout): wq u8 [N][K/2], d fp16 [N][K/32].
 *  - Affine b-bit (b in {4, 8}), the format of mx.quantize / mx.dequantize /
 *    mx.quantized_matmul on the MLX issue page (Repro): per group of
 *    `group` weights along K a scale and a bias, w = scale * q + bias,
 *    q in [0, 2^b - 1], packed 32/b per uint32, lowest bits first.
 *    scales and biases are bf16 [N][K/group], wq is u32 [N][K*b/32].
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (no FMA
 * contraction: every product and sum below rounds exactly as written).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Scalar bit conversions, written out from the IEEE-754 definitions. */
/* ------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bf16 -> fp32: bf16 is the top half of an fp32 word. */
float oracle_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even.  NaN stays NaN (quiet). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u = f32_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u)            /* NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))
        keep += 1u;                                  /* may carry into exponent */
    return (uint16_t)keep;
}

/* fp16 -> fp32, exact (normals, subnormals, zeros, inf, NaN). */
float oracle_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1fu;
    uint32_t m = h & 0x3ffu;
    if (e == 0x1fu)                                  /* inf / NaN */
        return bits_f32(sign | 0x7f800000u | (m << 13));
    if (e == 0) {
        if (m == 0) return bits_f32(sign);           /* +-0 */
        /* subnormal: value = m * 2^-24 */
        float v = (float)m * 0x1p-24f;               /* exact: m < 2^10 */
        return sign ? -v : v;
    }
    return bits_f32(sign | ((e + 112u) << 23) | (m << 13));
}

/* fp32 -> fp16, round to nearest, ties to even, with subnormals and
 * overflow to infinity. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u)                             /* NaN: keep it quiet */
        return (uint16_t)(sign | 0x7e00u | ((a >> 13) & 0x3ffu));
    if (a == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);
    uint32_t e = a >> 23;                            /* biased fp32 exponent */
    uint32_t m = (a & 0x7fffffu) | 0x800000u;        /* 24-bit significand */
    if (e == 0) m = a;                               /* fp32 subnormal: far below fp16 range */
    if (e >= 113u) {                                 /* fp16 normal range or overflow */
        uint32_t he = e - 112u;                      /* fp16 biased exponent */
        uint32_t q = (he << 10) | ((m >> 13) & 0x3ffu);
        uint32_t rest = m & 0x1fffu;
        if (rest > 0x1000u || (rest == 0x1000u && (q & 1u))) q += 1u;
        if (q >= 0x7c00u) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | q);
    }
    /* fp16 subnormal or zero: result = round(m * 2^(e-150) / 2^-24) = round(m * 2^(e-126)) */
    uint32_t shift = 126u - e;                       /* >= 14 */
    if (shift > 25u) return sign;                    /* below half of the smallest subnormal */
    uint32_t q = m >> shift;
    uint32_t rest = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1u);
    if (rest > half || (rest == half && (q & 1u))) q += 1u;
    return (uint16_t)(sign | q);                     /* q == 0x400 is the smallest normal */
}

void oracle_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(in[i]); }
void oracle_bf16_to_f32_array(const uint16_t* in, float* out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_f32(in[i]); }
void oracle_f32_to_f16_array(const float* in, uint16_t* out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(in[i]); }
void oracle_f16_to_f32_array(const uint16_t* in, float* out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(in[i]); }

/* ------------------------------------------------------------------ */
/* Q4_0                                                                */
/* ------------------------------------------------------------------ */

/* Quantize one row-major fp32 matrix w[N][K] (K % 32 == 0) to Q4_0.
 * Per block of 32 weights along K:
 *   1. m = the weight with the largest |w| (first index wins a tie);
 *   2. d = m / -8 in fp32, so that m itself maps to q = 0;
 *   3. q_j = clamp(trunc(w_j / d + 8.5), 0, 15) with an IEEE fp32 division and
 *      addition (q_j = 8 when d == 0: the block is all zeros);
 *   4. the stored scale is fp16(d); byte j = q_j | q_{j+16} << 4.
 * Reading (the pages print no quantizer; the Q4_0 workload statement gives
 * "d = signed max-abs / -8 as fp16" and "q = clamp(int(w/d + 8.5), 0, 15)"):
 * w/d is a true division by the unrounded fp32 d, and fp16(d) is what is
 * stored. */
void oracle_q4_0_quantize(const float* w, int64_t N, int64_t K, uint8_t* wq, uint16_t* d16)
{
    const int64_t nb = K / 32;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* blk = w + n * K + b * 32;
            float amax = 0.0f, mx = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float v = blk[j];
                if (fabsf(v) > amax) { amax = fabsf(v); mx = v; }
            }
            float d = mx / -8.0f;
            d16[n * nb + b] = oracle_f32_to_f16(d);
            uint8_t* out = wq + n * (K / 2) + b * 16;
            for (int j = 0; j < 16; ++j) {
                float t0 = (d != 0.0f) ? blk[j] / d : 0.0f;
                float t1 = (d != 0.0f) ? blk[j + 16] / d : 0.0f;
                t0 = t0 + 8.5f;
                t1 = t1 + 8.5f;
                int q0 = (int)t0, q1 = (int)t1;
                if (q0 > 15) q0 = 15;
                if (q1 > 15) q1 = 15;
                if (q0 < 0) q0 = 0;
                if (q1 < 0) q1 = 0;
                out[j] = (uint8_t)(q0 | (q1 << 4));
            }
        }
    }
}

/* Dequantize Q4_0 to bf16 bit patterns: out = bf16(fp32(d) * fp32(q - 8)).
 * The fp32 product is exact (11-bit times 4-bit significand), so the only
 * rounding is the final round-to-nearest-even to bf16. */
void oracle_q4_0_dequantize(const uint8_t* wq, const uint16_t* d16, int64_t N, int64_t K, uint16_t* out)
{
    const int64_t nb = K / 32;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            float d = oracle_f16_to_f32(d16[n * nb + b]);
            const uint8_t* in = wq + n * (K / 2) + b * 16;
            uint16_t* o = out + n * K + b * 32;
            for (int j = 0; j < 16; ++j) {
                int lo = in[j] & 0x0f;
                int hi = in[j] >> 4;
                o[j]      = oracle_f32_to_bf16(d * (float)(lo - 8));
                o[j + 16] = oracle_f32_to_bf16(d * (float)(hi - 8));
            }
        }
    }
}

/* Split array-of-structs Q4_0 blocks into the separate code and scale arrays.
 * Block layout (ggml's Q4_0 block, which the SYCL page's "reordered" Q4_0
 * kernels start from): the fp16 scale d (2 bytes, little-endian), then the 16
 * code bytes in the same nibble order as wq.  Row n holds K/32 consecutive
 * 18-byte blocks. */
void oracle_q4_0_import_aos(const uint8_t* blocks, int64_t N, int64_t K, uint8_t* wq, uint16_t* d16)
{
    const int64_t nb = K / 32;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t* blk = blocks + (n * nb + b) * 18;
            d16[n * nb + b] = (uint16_t)(blk[0] | (blk[1] << 8));
            for (int j = 0; j < 16; ++j) wq[n * (K / 2) + b * 16 + j] = blk[2 + j];
        }
    }
}

/* ------------------------------------------------------------------ */
/* Quantized activations (Q8_1 style) for the Q4_0 decode path         */
/* ------------------------------------------------------------------ */

/* Per block of 32 consecutive elements of a token row: amax = max |x|,
 * d = amax / 127 in fp32, id = d != 0 ? 1 / d : 0, q = roundf(x * id) (half away
 * from zero, in [-127, 127]), qsum = the sum of the block's q. */
void oracle_q8_1_quantize(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* dx, int32_t* qsum)
{
    const int64_t nb = K / 32;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint16_t* xb = x + m * K + b * 32;
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float v = fabsf(oracle_bf16_to_f32(xb[j]));
                if (v > amax) amax = v;
            }
            const float d = amax / 127.0f;
            const float id = d != 0.0f ? 1.0f / d : 0.0f;
            int32_t sum = 0;
            for (int j = 0; j < 32; ++j) {
                const int q = (int)roundf(oracle_bf16_to_f32(xb[j]) * id);
                xq[m * K + b * 32 + j] = (int8_t)q;
                sum += q;
            }
            dx[m * nb + b] = d;
            qsum[m * nb + b] = sum;
        }
    }
}

/* y[m][n] = sum over blocks b of d_w[n][b] * dx[m][b] * sum_j xq[m][32b+j] * (q_w[n][32b+j] - 8),
 * in float64 from the integer codes; a[m][n] = the same sum of absolute values of the
 * block terms (for the tolerance). */
void oracle_q4_0_q8_matmul(const int8_t* xq, const float* dx, const uint8_t* wq, const uint16_t* d16,
                           int64_t M, int64_t N, int64_t K, double* y, double* a)
{
    const int64_t nb = K / 32;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                const uint8_t* in = wq + n * (K / 2) + b * 16;
                const int8_t* xb = xq + m * K + b * 32;
                int64_t dot = 0;
                for (int j = 0; j < 16; ++j) {
                    dot += (int64_t)xb[j] * ((in[j] & 0x0f) - 8);
                    dot += (int64_t)xb[j + 16] * ((in[j] >> 4) - 8);
                }
                const double term = (double)oracle_f16_to_f32(d16[n * nb + b]) * (double)dx[m * nb + b] * (double)dot;
                acc += term;
                abs_acc += fabs(term);
            }
            y[m * N + n] = acc;
            a[m * N + n] = abs_acc;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Affine (MLX-style) b-bit, b in {2, 3, 4, 6, 8}                      */
/* ------------------------------------------------------------------ */

/* Codes of a row form a little-endian bit stream over its 32-bit words: code k
 * occupies stream bits bits*k .. bits*k + bits - 1, lowest first, and stream
 * bit i is bit (i mod 32) of word i / 32.  For 2, 4 and 8 bits a code never
 * crosses a word (32 / bits codes per word, lowest bits first); 3- and 6-bit
 * codes may.  Rows hold K * bits / 32 whole words (K is a multiple of 32). */
static int64_t affine_words_per_row(int64_t K, int bits) { return K * bits / 32; }

static void put_code(uint32_t* row, int64_t k, int bits, uint32_t q)
{
    for (int i = 0; i < bits; ++i) {
        const int64_t bit = k * bits + i;
        if ((q >> i) & 1u) row[bit / 32] |= 1u << (int)(bit % 32);
    }
}

static uint32_t get_code(const uint32_t* row, int64_t k, int bits)
{
    uint32_t q = 0;
    for (int i = 0; i < bits; ++i) {
        const int64_t bit = k * bits + i;
        q |= ((row[bit / 32] >> (int)(bit % 32)) & 1u) << i;
    }
    return q;
}

/* Quantize w[N][K] (values already bf16-representable) per group:
 *   scale = bf16((max - min) / L), bias = bf16(min), L = 2^bits - 1;
 *   q = clamp(round_half_even((w - bias) / scale), 0, L), computed in fp32 from
 *   the STORED (bf16) scale and bias; a group with scale == 0 gets q = 0. */
void oracle_affine_quantize(const float* w, int64_t N, int64_t K, int group, int bits,
                            uint32_t* wq, uint16_t* scales, uint16_t* biases)
{
    const int L = (1 << bits) - 1;
    const int64_t ng = K / group;
    const int64_t wpr = affine_words_per_row(K, bits);
    memset(wq, 0, (size_t)(N * wpr) * sizeof(uint32_t));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < ng; ++g) {
            const float* grp = w + n * K + g * group;
            float mn = grp[0], mx = grp[0];
            for (int j = 1; j < group; ++j) {
                if (grp[j] < mn) mn = grp[j];
                if (grp[j] > mx) mx = grp[j];
            }
            float range = mx - mn;
            float scale_f = range / (float)L;
            uint16_t s16 = oracle_f32_to_bf16(scale_f);
            uint16_t b16 = oracle_f32_to_bf16(mn);
            scales[n * ng + g] = s16;
            biases[n * ng + g] = b16;
            float s = oracle_bf16_to_f32(s16);
            float bb = oracle_bf16_to_f32(b16);
            for (int j = 0; j < group; ++j) {
                int q = 0;
                if (s != 0.0f) {
                    float t = grp[j] - bb;
                    t = t / s;
                    float r = nearbyintf(t);           /* default mode: ties to even */
                    if (r < 0.0f) r = 0.0f;
                    if (r > (float)L) r = (float)L;
                    q = (int)r;
                }
                put_code(wq + n * wpr, g * group + j, bits, (uint32_t)q);
            }
        }
    }
}

/* Dequantize affine to bf16 bit patterns: out = bf16(fmaf(scale, q, bias)),
 * one fp32 fused multiply-add, then one round-to-nearest-even to bf16. */
void oracle_affine_dequantize(const uint32_t* wq, const uint16_t* scales, const uint16_t* biases,
                              int64_t N, int64_t K, int group, int bits, uint16_t* out)
{
    const int64_t ng = K / group;
    const int64_t wpr = affine_words_per_row(K, bits);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint32_t q = get_code(wq + n * wpr, k, bits);
            float s = oracle_bf16_to_f32(scales[n * ng + k / group]);
            float b = oracle_bf16_to_f32(biases[n * ng + k / group]);
            out[n * K + k] = oracle_f32_to_bf16(fmaf(s, (float)q, b));
        }
    }
}

/* ------------------------------------------------------------------ */
/* Reference matmul, float64                                           */
/* ------------------------------------------------------------------ */

typedef struct {
    const uint16_t* x; const uint16_t* w;
    int64_t M, N, K;
    const int64_t* rows; int64_t nrows;
    double* y; double* a;
    int64_t begin, end;             /* range of (selected row, n) work items */
} mm_job;

static void* mm_worker(void* arg)
{
    mm_job* j = (mm_job*)arg;
    for (int64_t it = j->begin; it < j->end; ++it) {
        int64_t r = it / j->N, n = it % j->N;
        int64_t m = j->rows ? j->rows[r] : r;
        const uint16_t* xr = j->x + m * j->K;
        const uint16_t* wr = j->w + n * j->K;
        double s = 0.0, sa = 0.0;
        for (int64_t k = 0; k < j->K; ++k) {
            double p = (double)oracle_bf16_to_f32(xr[k]) * (double)oracle_bf16_to_f32(wr[k]);
            s += p;
            sa += fabs(p);
        }
        j->y[r * j->N + n] = s;
        j->a[r * j->N + n] = sa;
    }
    return NULL;
}

/* y[r][n] = sum_k x[m_r][k] * w[n][k] and a[r][n] = sum_k |x[m_r][k] * w[n][k]|,
 * for the selected rows m_r (rows == NULL: all M rows), in float64, k ascending.
 * x is bf16 [M][K], w is bf16 [N][K] (the transpose=True convention: W stored
 * with one output per row).  Work items are split over nthreads host threads;
 * the order of the sum within one dot product is fixed. */
int oracle_matmul_ref(const uint16_t* x, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                      const int64_t* rows, int64_t nrows, double* y, double* a, int nthreads)
{
    if (!rows) nrows = M;
    if (nthreads < 1) nthreads = 1;
    int64_t total = nrows * N;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > total) nthreads = (int)(total > 0 ? total : 1);
    mm_job jobs[256];
    pthread_t tids[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = (mm_job){x, w, M, N, K, rows, nrows, y, a,
                           total * t / nthreads, total * (t + 1) / nthreads};
    }
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&tids[t], NULL, mm_worker, &jobs[t]) != 0) break;
        started = t;
    }
    mm_worker(&jobs[0]);
    for (int t = 1; t <= started; ++t) pthread_join(tids[t], NULL);
    for (int t = started + 1; t < nthreads; ++t) mm_worker(&jobs[t]);   /* thread creation failed */
    return nthreads;
}
