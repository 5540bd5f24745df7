/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for block-quantised
 * weight GEMV (decode step).  TEST INFRASTRUCTURE ONLY: nothing on the product
 * path may include, link or call this file.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg use it.  It shares no code, header or
 * table with the CUDA library.
 *
 * What it computes (BaseRT: Best-in-Class LLM Inference on Apple Silicon via
 * Native Metal, gist.science technical summary, "Methodologie" /
 * "Specialisatie"): decode is a GEMV per quantisation format, with the
 * dequantisation done inside the dot-product loop.  The result that method
 * reaches is, up to rounding order, the plain definition
 *
 *      y[b][n] = sum_k  deq(W)[n][k] * x[b][k]
 *
 * which this file evaluates in fp64 straight from the packed bytes.  The block
 * formats themselves (32-element blocks along K, one fp16 scale per block,
 * Q8: int8 q = round(w/d), d = absmax/127; Q4: q = clamp(round(w/d)+8, 0, 15),
 * d = absmax/7, element j in the low nibble and element j+16 in the high nibble
 * of byte j) are not printed on those pages: the pages only name the Q4/Q8
 * formats (abstract; technical summary "Belangrijkste Bijdragen").  The
 * definitions used here are the workload definitions that accompany them.
 *
 * Q6 (a third format of the same family; the pages list formats from Q2 to
 * FP16 without defining them): 32-element blocks along K, one fp16 scale
 * d = absmax/31, code q = clamp(round(w/d)+32, 0, 63), weight d*(q-32).  A
 * row of codes is 3K/4 bytes: first a low-nibble plane laid out exactly as Q4
 * (block j at byte 16j; byte i holds the low 4 bits of element i, and in its
 * high nibble those of element i+16), then a 2-bit plane (block j at byte
 * K/2 + 8j; byte i holds the top 2 bits of elements i, i+8, i+16 and i+24 in
 * bits 0-1, 2-3, 4-5 and 6-7).
 *
 * Q5 (the same construction with one top bit): d = absmax/15, q =
 * clamp(round(w/d)+16, 0, 31), weight d*(q-16); a row of codes is 5K/8 bytes:
 * the low-nibble plane as Q4, then a 1-bit plane (block j at byte K/2 + 4j;
 * byte i (0..3) holds the top bit of element i + 4p in bit p, p = 0..7).
 *
 * Q3 (the 3-bit member): d = absmax/3, q = clamp(round(w/d)+4, 0, 7), weight
 * d*(q-4); a row of codes is 3K/8 bytes: a 2-bit plane holding the low 2 bits
 * of each code (block j at byte 8j; byte i holds elements i, i+8, i+16 and
 * i+24 in bits 0-1, 2-3, 4-5 and 6-7, the layout of Q6's top plane), then a
 * 1-bit plane holding bit 2 (block j at byte K/4 + 4j; byte i (0..3) holds
 * element i + 4p in bit p, the layout of Q5's top plane).
 *
 * Q2 (the 2-bit member): d = absmax/1, q = clamp(round(w/d)+2, 0, 3), weight
 * d*(q-2); a row of codes is K/4 bytes, the 2-bit plane alone (laid out as
 * Q3's).  The quantiser never emits code 0 (|w/d| <= 1), but the format and
 * its dequantisation define it.
 *
 * Readings taken where the definition is silent (each is also listed in the
 * design notes of the repository):
 *   - blocks run along K (the reduction axis), consecutive within a row;
 *   - round() is round-half-away-from-zero (C roundf);
 *   - w is divided by the *stored* fp16 scale, and Q8 codes are clamped to
 *     [-127, 127];
 *   - a block whose fp16 scale is zero (all-zero block, or a scale that
 *     rounds to zero) gets the zero-point code (0 for Q8, 8 for Q4);
 *   - the scale plane has rows of ldS = roundup(K/32, 8) entries; the extra
 *     entries are zero.
 *
 * Every function here is pinned by tests/test_oracle_pins.py against closed
 * forms, library conversions, exhaustive enumeration or brute force.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BLOCK 32

/* ---------------------------------------------------------------------------
 * IEEE 754 binary16 <-> binary64, written out from the format definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * ------------------------------------------------------------------------ */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);  /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Nearest binary16 to v (ties to even), for finite or infinite v. */
uint16_t oracle_double_to_half(double v)
{
    uint16_t sign = 0;
    if (isnan(v))
        return 0x7e00;
    if (signbit(v)) {
        sign = 0x8000;
        v = -v;
    }
    /* 65520 is the midpoint between 65504 (largest finite) and 2^16: the
     * tie goes to the even neighbour, which is the overflow to infinity. */
    if (v >= 65520.0)
        return sign | 0x7c00;
    if (v < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; rint() rounds half to even */
        double q = rint(v * ldexp(1.0, 24));
        return sign | (uint16_t)q;              /* q == 1024 encodes 2^-14 */
    }
    int E;
    (void)frexp(v, &E);                         /* v = f * 2^E, f in [0.5,1) */
    int e = E - 1;                              /* v in [2^e, 2^(e+1)) */
    double q = rint(ldexp(v, 10 - e));          /* in [1024, 2048] */
    if (q >= 2048.0) {
        q = 1024.0;
        e += 1;
    }
    if (e + 15 >= 31)
        return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

int oracle_scales_ld(int K)
{
    int nb = K / ORACLE_BLOCK;
    return (nb + 7) / 8 * 8;
}

/* ---------------------------------------------------------------------------
 * Quantisers (fp32 arithmetic, as the format definition fixes the scale from
 * an fp32 absmax).  Returns 0 on success, -1 on bad shape, -2 if a block's
 * scale overflows fp16 or the input holds a non-finite value.
 * ------------------------------------------------------------------------ */
static int oracle_quantize(const float *w, int N, int K, int levels_half,
                           int fmt, uint8_t *codes, uint16_t *scales)
{
    /* zero-point code: 2, 4, 16, 32 or 8 for Q2, Q3, Q5, Q6 or Q4; Q8 has none */
    const int zero = fmt == 2 ? 2 : fmt == 3 ? 4 : fmt == 4 ? 8 : fmt == 5 ? 16 : fmt == 6 ? 32 : 0;
    if (N < 1 || K < ORACLE_BLOCK || K % ORACLE_BLOCK)
        return -1;
    int nb = K / ORACLE_BLOCK;
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++) {
        for (int j = 0; j < ldS; j++)
            scales[(size_t)n * ldS + j] = 0;
        for (int j = 0; j < nb; j++) {
            const float *blk = w + (size_t)n * K + (size_t)j * ORACLE_BLOCK;
            float a = 0.0f;
            for (int i = 0; i < ORACLE_BLOCK; i++) {
                if (!isfinite(blk[i]))
                    return -2;
                float m = fabsf(blk[i]);
                if (m > a)
                    a = m;
            }
            float d32 = a / (float)levels_half;    /* fp32 division */
            uint16_t dh = oracle_double_to_half((double)d32);
            if ((dh & 0x7c00) == 0x7c00)
                return -2;
            float d = (float)oracle_half_to_double(dh);
            scales[(size_t)n * ldS + j] = dh;
            int q[ORACLE_BLOCK];
            for (int i = 0; i < ORACLE_BLOCK; i++) {
                if (d == 0.0f) {
                    q[i] = zero;
                    continue;
                }
                float r = roundf(blk[i] / d);      /* fp32 division, half away */
                if (fmt != 8) {
                    float t = r + (float)zero;
                    float top = (float)(2 * zero - 1);   /* 3, 7, 15, 31 or 63 */
                    q[i] = t < 0.0f ? 0 : (t > top ? (int)top : (int)t);
                } else {
                    q[i] = r < -127.0f ? -127 : (r > 127.0f ? 127 : (int)r);
                }
            }
            if (fmt == 4) {
                uint8_t *dst = codes + (size_t)n * (K / 2) + (size_t)j * 16;
                for (int i = 0; i < 16; i++)
                    dst[i] = (uint8_t)(q[i] | (q[i + 16] << 4));
            } else if (fmt == 5) {
                uint8_t *row = codes + (size_t)n * (5 * (size_t)K / 8);
                uint8_t *lo = row + (size_t)j * 16;
                uint8_t *hi = row + (size_t)K / 2 + (size_t)j * 4;
                for (int i = 0; i < 16; i++)
                    lo[i] = (uint8_t)((q[i] & 15) | ((q[i + 16] & 15) << 4));
                for (int i = 0; i < 4; i++) {
                    int b = 0;
                    for (int p = 0; p < 8; p++)
                        b |= (q[i + 4 * p] >> 4) << p;
                    hi[i] = (uint8_t)b;
                }
            } else if (fmt == 2 || fmt == 3) {
                uint8_t *row = codes + (size_t)n * (fmt == 2 ? (size_t)K / 4 : 3 * (size_t)K / 8);
                uint8_t *lo = row + (size_t)j * 8;
                for (int i = 0; i < 8; i++)
                    lo[i] = (uint8_t)((q[i] & 3) | ((q[i + 8] & 3) << 2) |
                                      ((q[i + 16] & 3) << 4) | ((q[i + 24] & 3) << 6));
                if (fmt == 3) {
                    uint8_t *hi = row + (size_t)K / 4 + (size_t)j * 4;
                    for (int i = 0; i < 4; i++) {
                        int b = 0;
                        for (int p = 0; p < 8; p++)
                            b |= (q[i + 4 * p] >> 2) << p;
                        hi[i] = (uint8_t)b;
                    }
                }
            } else if (fmt == 6) {
                uint8_t *row = codes + (size_t)n * (3 * (size_t)K / 4);
                uint8_t *lo = row + (size_t)j * 16;
                uint8_t *hi = row + (size_t)K / 2 + (size_t)j * 8;
                for (int i = 0; i < 16; i++)
                    lo[i] = (uint8_t)((q[i] & 15) | ((q[i + 16] & 15) << 4));
                for (int i = 0; i < 8; i++)
                    hi[i] = (uint8_t)((q[i] >> 4) | ((q[i + 8] >> 4) << 2) |
                                      ((q[i + 16] >> 4) << 4) | ((q[i + 24] >> 4) << 6));
            } else {
                int8_t *dst = (int8_t *)codes + (size_t)n * K + (size_t)j * ORACLE_BLOCK;
                for (int i = 0; i < ORACLE_BLOCK; i++)
                    dst[i] = (int8_t)q[i];
            }
        }
    }
    return 0;
}

int oracle_quantize_q8(const float *w, int N, int K, int8_t *codes, uint16_t *scales)
{
    return oracle_quantize(w, N, K, 127, 8, (uint8_t *)codes, scales);
}

int oracle_quantize_q4(const float *w, int N, int K, uint8_t *codes, uint16_t *scales)
{
    return oracle_quantize(w, N, K, 7, 4, codes, scales);
}

/* codes: N rows of K/4 bytes (see the header) */
int oracle_quantize_q2(const float *w, int N, int K, uint8_t *codes, uint16_t *scales)
{
    return oracle_quantize(w, N, K, 1, 2, codes, scales);
}

/* codes: N rows of 3K/8 bytes (see the header) */
int oracle_quantize_q3(const float *w, int N, int K, uint8_t *codes, uint16_t *scales)
{
    return oracle_quantize(w, N, K, 3, 3, codes, scales);
}

/* codes: N rows of 5K/8 bytes (see the header) */
int oracle_quantize_q5(const float *w, int N, int K, uint8_t *codes, uint16_t *scales)
{
    return oracle_quantize(w, N, K, 15, 5, codes, scales);
}

/* codes: N rows of 3K/4 bytes (see the header) */
int oracle_quantize_q6(const float *w, int N, int K, uint8_t *codes, uint16_t *scales)
{
    return oracle_quantize(w, N, K, 31, 6, codes, scales);
}

/* ---------------------------------------------------------------------------
 * Dequantisation of one element, straight from the packed planes.
 * ------------------------------------------------------------------------ */
static double deq_q4(const uint8_t *codes, const uint16_t *scales, int K, int ldS,
                     int n, int k)
{
    int j = k / ORACLE_BLOCK;          /* block index along K */
    int i = k % ORACLE_BLOCK;          /* position inside the block */
    uint8_t byte = codes[(size_t)n * (K / 2) + (size_t)j * 16 + (i % 16)];
    int q = (i < 16) ? (byte & 0x0f) : (byte >> 4);
    double d = oracle_half_to_double(scales[(size_t)n * ldS + j]);
    return d * (double)(q - 8);
}

static double deq_q2(const uint8_t *codes, const uint16_t *scales, int K, int ldS,
                     int n, int k)
{
    int j = k / ORACLE_BLOCK;
    int i = k % ORACLE_BLOCK;
    uint8_t byte = codes[(size_t)n * ((size_t)K / 4) + (size_t)j * 8 + (i % 8)];
    int q = (byte >> (2 * (i / 8))) & 3;
    double d = oracle_half_to_double(scales[(size_t)n * ldS + j]);
    return d * (double)(q - 2);
}

static double deq_q3(const uint8_t *codes, const uint16_t *scales, int K, int ldS,
                     int n, int k)
{
    int j = k / ORACLE_BLOCK;
    int i = k % ORACLE_BLOCK;
    const uint8_t *row = codes + (size_t)n * (3 * (size_t)K / 8);
    uint8_t lo_byte = row[(size_t)j * 8 + (i % 8)];
    uint8_t hi_byte = row[(size_t)K / 4 + (size_t)j * 4 + (i % 4)];
    int lo = (lo_byte >> (2 * (i / 8))) & 3;
    int hi = (hi_byte >> (i / 4)) & 1;
    int q = lo | (hi << 2);
    double d = oracle_half_to_double(scales[(size_t)n * ldS + j]);
    return d * (double)(q - 4);
}

static double deq_q5(const uint8_t *codes, const uint16_t *scales, int K, int ldS,
                     int n, int k)
{
    int j = k / ORACLE_BLOCK;
    int i = k % ORACLE_BLOCK;
    const uint8_t *row = codes + (size_t)n * (5 * (size_t)K / 8);
    uint8_t lo_byte = row[(size_t)j * 16 + (i % 16)];
    uint8_t hi_byte = row[(size_t)K / 2 + (size_t)j * 4 + (i % 4)];
    int lo = (i < 16) ? (lo_byte & 0x0f) : (lo_byte >> 4);
    int hi = (hi_byte >> (i / 4)) & 1;
    int q = lo | (hi << 4);
    double d = oracle_half_to_double(scales[(size_t)n * ldS + j]);
    return d * (double)(q - 16);
}

static double deq_q6(const uint8_t *codes, const uint16_t *scales, int K, int ldS,
                     int n, int k)
{
    int j = k / ORACLE_BLOCK;
    int i = k % ORACLE_BLOCK;
    const uint8_t *row = codes + (size_t)n * (3 * (size_t)K / 4);
    uint8_t lo_byte = row[(size_t)j * 16 + (i % 16)];
    uint8_t hi_byte = row[(size_t)K / 2 + (size_t)j * 8 + (i % 8)];
    int lo = (i < 16) ? (lo_byte & 0x0f) : (lo_byte >> 4);
    int hi = (hi_byte >> (2 * (i / 8))) & 3;
    int q = lo | (hi << 4);
    double d = oracle_half_to_double(scales[(size_t)n * ldS + j]);
    return d * (double)(q - 32);
}

static double deq_q8(const int8_t *codes, const uint16_t *scales, int K, int ldS,
                     int n, int k)
{
    int j = k / ORACLE_BLOCK;
    double d = oracle_half_to_double(scales[(size_t)n * ldS + j]);
    return d * (double)codes[(size_t)n * K + k];
}

void oracle_dequantize_q4(const uint8_t *codes, const uint16_t *scales, int N, int K,
                          double *w)
{
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++)
            w[(size_t)n * K + k] = deq_q4(codes, scales, K, ldS, n, k);
}

void oracle_dequantize_q2(const uint8_t *codes, const uint16_t *scales, int N, int K,
                          double *w)
{
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++)
            w[(size_t)n * K + k] = deq_q2(codes, scales, K, ldS, n, k);
}

void oracle_dequantize_q3(const uint8_t *codes, const uint16_t *scales, int N, int K,
                          double *w)
{
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++)
            w[(size_t)n * K + k] = deq_q3(codes, scales, K, ldS, n, k);
}

void oracle_dequantize_q5(const uint8_t *codes, const uint16_t *scales, int N, int K,
                          double *w)
{
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++)
            w[(size_t)n * K + k] = deq_q5(codes, scales, K, ldS, n, k);
}

void oracle_dequantize_q6(const uint8_t *codes, const uint16_t *scales, int N, int K,
                          double *w)
{
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++)
            w[(size_t)n * K + k] = deq_q6(codes, scales, K, ldS, n, k);
}

void oracle_dequantize_q8(const int8_t *codes, const uint16_t *scales, int N, int K,
                          double *w)
{
    int ldS = oracle_scales_ld(K);
    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++)
            w[(size_t)n * K + k] = deq_q8(codes, scales, K, ldS, n, k);
}

/* ---------------------------------------------------------------------------
 * GEMV: y[b][n] = sum_k deq(W)[n][k] * x[b][k], and the tolerance reference
 * absy[b][n] = sum_k |deq(W)[n][k] * x[b][k]|, both in fp64.  x is fp16 bits,
 * row b at x + b*ldx.  Rows are split over nthreads POSIX threads; each
 * output is still one plain sequential sum.
 * ------------------------------------------------------------------------ */
typedef struct {
    int fmt;                  /* 2, 3, 4, 5, 6 or 8 */
    const void *codes;
    const uint16_t *scales;
    int N, K, ldS;
    const uint16_t *x;
    int B, ldx;
    double *y, *absy;
    int n0, n1;
} gemv_job;

static void gemv_rows(const gemv_job *t)
{
    for (int n = t->n0; n < t->n1; n++) {
        for (int b = 0; b < t->B; b++) {
            double s = 0.0, sa = 0.0;
            for (int k = 0; k < t->K; k++) {
                double w = (t->fmt == 2)   ? deq_q2((const uint8_t *)t->codes, t->scales, t->K, t->ldS, n, k)
                           : (t->fmt == 3) ? deq_q3((const uint8_t *)t->codes, t->scales, t->K, t->ldS, n, k)
                           : (t->fmt == 4) ? deq_q4((const uint8_t *)t->codes, t->scales, t->K, t->ldS, n, k)
                           : (t->fmt == 5) ? deq_q5((const uint8_t *)t->codes, t->scales, t->K, t->ldS, n, k)
                           : (t->fmt == 6) ? deq_q6((const uint8_t *)t->codes, t->scales, t->K, t->ldS, n, k)
                                           : deq_q8((const int8_t *)t->codes, t->scales, t->K, t->ldS, n, k);
                double p = w * oracle_half_to_double(t->x[(size_t)b * t->ldx + k]);
                s += p;
                sa += fabs(p);
            }
            t->y[(size_t)b * t->N + n] = s;
            if (t->absy)
                t->absy[(size_t)b * t->N + n] = sa;
        }
    }
}

static void *gemv_thread(void *arg)
{
    gemv_rows((const gemv_job *)arg);
    return NULL;
}

static int oracle_gemv(int fmt, const void *codes, const uint16_t *scales, int N, int K,
                       const uint16_t *x, int B, int ldx, double *y, double *absy,
                       int nthreads)
{
    if (N < 1 || K < ORACLE_BLOCK || K % ORACLE_BLOCK || B < 1 || ldx < K)
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > N)
        nthreads = N;
    gemv_job *jobs = (gemv_job *)calloc((size_t)nthreads, sizeof(gemv_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return -3;
    }
    for (int i = 0; i < nthreads; i++) {
        gemv_job j = {fmt, codes, scales, N, K, oracle_scales_ld(K), x, B, ldx, y, absy,
                      (int)((long long)N * i / nthreads), (int)((long long)N * (i + 1) / nthreads)};
        jobs[i] = j;
    }
    int started = 0;
    for (int i = 1; i < nthreads; i++)
        if (pthread_create(&th[i], NULL, gemv_thread, &jobs[i]) == 0)
            started = i;
        else
            break;
    gemv_rows(&jobs[0]);
    for (int i = 1; i <= started; i++)
        pthread_join(th[i], NULL);
    /* any job whose thread could not be created runs here */
    for (int i = started + 1; i < nthreads; i++)
        gemv_rows(&jobs[i]);
    free(jobs);
    free(th);
    return 0;
}

int oracle_gemv_q4(const uint8_t *codes, const uint16_t *scales, int N, int K,
                   const uint16_t *x, int B, int ldx, double *y, double *absy, int nthreads)
{
    return oracle_gemv(4, codes, scales, N, K, x, B, ldx, y, absy, nthreads);
}

int oracle_gemv_q2(const uint8_t *codes, const uint16_t *scales, int N, int K,
                   const uint16_t *x, int B, int ldx, double *y, double *absy, int nthreads)
{
    return oracle_gemv(2, codes, scales, N, K, x, B, ldx, y, absy, nthreads);
}

int oracle_gemv_q3(const uint8_t *codes, const uint16_t *scales, int N, int K,
                   const uint16_t *x, int B, int ldx, double *y, double *absy, int nthreads)
{
    return oracle_gemv(3, codes, scales, N, K, x, B, ldx, y, absy, nthreads);
}

int oracle_gemv_q5(const uint8_t *codes, const uint16_t *scales, int N, int K,
                   const uint16_t *x, int B, int ldx, double *y, double *absy, int nthreads)
{
    return oracle_gemv(5, codes, scales, N, K, x, B, ldx, y, absy, nthreads);
}

int oracle_gemv_q6(const uint8_t *codes, const uint16_t *scales, int N, int K,
                   const uint16_t *x, int B, int ldx, double *y, double *absy, int nthreads)
{
    return oracle_gemv(6, codes, scales, N, K, x, B, ldx, y, absy, nthreads);
}

int oracle_gemv_q8(const int8_t *codes, const uint16_t *scales, int N, int K,
                   const uint16_t *x, int B, int ldx, double *y, double *absy, int nthreads)
{
    return oracle_gemv(8, codes, scales, N, K, x, B, ldx, y, absy, nthreads);
}

/* ---------------------------------------------------------------------------
 * Routed-expert (MoE) decode GEMV, Q4.  The technical summary's results
 * ("Prefill Throughput", Mixture-of-Experts models such as Qwen3-30B-A3B) and
 * the follow-up paper's method paragraph name expert GEMMs; at decode each
 * token's routed experts are applied as GEMVs:
 *
 *   per-slot (route_w == NULL):  y[b][s][n] = sum_k deq(W_e)[n][k] * x_bs[k]
 *   combined:                    y[b][n]    = sum_s route_w[b][s] * (that)
 *
 * with e = expert_idx[b][s], expert e's planes at codes + e*codes_stride and
 * scales + e*scales_stride, and x_bs = x[b] (x_per_slot == 0) or x[b][s].
 * A slot whose index is outside [0, E) contributes zero (its per-slot output
 * is zero) and the return value has bit 1 set.  absy gets the matching sums
 * of |.| (weighted by |route_w| in the combined form).
 * ------------------------------------------------------------------------ */
int oracle_moe_gemv_q4(const uint8_t *codes, const uint16_t *scales, int E, int N, int K,
                       long long codes_stride, long long scales_stride,
                       const uint16_t *x, int x_per_slot, const int32_t *expert_idx,
                       const float *route_w, int B, int topk, double *y, double *absy,
                       int nthreads)
{
    if (N < 1 || K < ORACLE_BLOCK || K % ORACLE_BLOCK || B < 1 || topk < 1 || E < 1)
        return -1;
    int bad = 0;
    size_t out_rows = route_w ? (size_t)B : (size_t)B * topk;
    for (size_t i = 0; i < out_rows * N; i++) {
        y[i] = 0.0;
        if (absy)
            absy[i] = 0.0;
    }
    double *tmp = (double *)malloc(sizeof(double) * (size_t)N * 2);
    if (!tmp)
        return -3;
    for (int b = 0; b < B; b++) {
        for (int s = 0; s < topk; s++) {
            int e = expert_idx[b * topk + s];
            if (e < 0 || e >= E) {
                bad = 1;
                continue;
            }
            const uint16_t *xv = x + (size_t)(x_per_slot ? (b * topk + s) : b) * K;
            int rc = oracle_gemv_q4(codes + (size_t)e * codes_stride,
                                    scales + (size_t)e * scales_stride, N, K, xv, 1, K,
                                    tmp, tmp + N, nthreads);
            if (rc) {
                free(tmp);
                return rc;
            }
            if (route_w) {
                double r = (double)route_w[b * topk + s];
                for (int n = 0; n < N; n++) {
                    y[(size_t)b * N + n] += r * tmp[n];
                    if (absy)
                        absy[(size_t)b * N + n] += fabs(r) * tmp[N + n];
                }
            } else {
                for (int n = 0; n < N; n++) {
                    y[((size_t)b * topk + s) * N + n] = tmp[n];
                    if (absy)
                        absy[((size_t)b * topk + s) * N + n] = tmp[N + n];
                }
            }
        }
    }
    free(tmp);
    return bad ? 2 : 0;
}

/*
 * Feed-forward activation between the fused gate|up projection and the down
 * projection.  The pages' runtime fuses operator sequences inside
 * feed-forward blocks (gist.science technical summary, "Methodologie" ->
 * "Kernel Fusie en Specialisatie"); the activation of the model families they
 * evaluate (Qwen3, Llama 3.2) is SwiGLU:
 *
 *      h[i] = silu(g[i]) * u[i],    silu(z) = z / (1 + e^-z)
 *
 * evaluated here in fp64 and rounded once to the nearest fp16 (ties to even),
 * the type the down projection consumes.
 */
double oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

void oracle_swiglu_f16(const double *g, const double *u, int n, uint16_t *h)
{
    for (int i = 0; i < n; i++)
        h[i] = oracle_double_to_half(oracle_silu(g[i]) * u[i]);
}

/* ---------------------------------------------------------------------------
 * Decode attention over a block-quantised KV cache.  The pages' runtime keeps
 * its KV cache preallocated for the whole decode loop (gist.science technical
 * summary, "Methodologie" -> "Zero-Allocation Decode Loop"), and at decode
 * runs a specialised decode-attention kernel beside the GEMV (romaanj.github.io
 * review of the M5 follow-up paper, "Method").  One new token per sequence
 * attends to the positions t < lens[b] of its cache:
 *
 *      s_t  = scale * sum_d q[d] * K[t][d]
 *      p_t  = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)
 *      o[d] = sum_t p_t * V[t][d]
 *
 * with K[t][d] = dK(t, d/32) * k(t, d) and V[t][d] = dV(t, d/32) * v(d, t):
 * the cache rows are Q8 blocks of 32 along the head dimension (fp16 scale
 * d = absmax/127, int8 codes -- the Q8 format of the weights, applied to each
 * position's key and value vectors).  Query head i of a sequence uses KV head
 * i / G (grouped-query attention).  Everything is evaluated in fp64.
 *
 * Layouts (all row-major):
 *   k_codes   int8  [B][Hkv][Tmax][D]          key codes, one row per position
 *   k_scales  fp16  [B][Hkv][Tmax][D/32]
 *   vt_codes  int8  [B][Hkv][D][Tmax]          value codes transposed: row d
 *                                              holds component d of every
 *                                              position
 *   v_scales  fp16  [B][Hkv][Tmax][D/32]       scale of position t's block j
 *   q         fp16  [B][Hkv*G][D]
 *   lens      int32 [B]                        0 <= lens[b] <= Tmax
 *   o, abso   fp64  [B][Hkv*G][D]              abso[d] = sum_t p_t |V[t][d]|
 * A sequence with lens[b] == 0 attends to nothing: its outputs are zero and
 * the return value has bit 1 set.  Positions t >= lens[b] are never read.
 * ------------------------------------------------------------------------ */
int oracle_attn_decode_q8(const int8_t *k_codes, const uint16_t *k_scales,
                          const int8_t *vt_codes, const uint16_t *v_scales, const uint16_t *q,
                          const int32_t *lens, int B, int Hkv, int G, int D, int Tmax,
                          double scale, double *o, double *abso)
{
    if (B < 1 || Hkv < 1 || G < 1 || D < ORACLE_BLOCK || D % ORACLE_BLOCK || Tmax < 1)
        return -1;
    const int nb = D / ORACLE_BLOCK, H = Hkv * G;
    int empty = 0;
    double *s = (double *)malloc(sizeof(double) * (size_t)Tmax);
    double *qd = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !qd) {
        free(s);
        free(qd);
        return -3;
    }
    for (int b = 0; b < B; b++) {
        const int L = lens[b];
        if (L < 0 || L > Tmax) {
            free(s);
            free(qd);
            return -1;
        }
        for (int i = 0; i < H; i++) {
            const int h = i / G;
            const size_t kv = (size_t)b * Hkv + h;
            double *oo = o + ((size_t)b * H + i) * D;
            double *aa = abso + ((size_t)b * H + i) * D;
            for (int d = 0; d < D; d++)
                oo[d] = aa[d] = 0.0;
            if (L == 0) {
                empty = 1;
                continue;
            }
            for (int d = 0; d < D; d++)
                qd[d] = oracle_half_to_double(q[((size_t)b * H + i) * D + d]);
            /* scores */
            double m = -INFINITY;
            for (int t = 0; t < L; t++) {
                const int8_t *kr = k_codes + (kv * Tmax + t) * D;
                const uint16_t *ksr = k_scales + (kv * Tmax + t) * nb;
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qd[d] * (oracle_half_to_double(ksr[d / ORACLE_BLOCK]) * (double)kr[d]);
                s[t] = scale * acc;
                if (s[t] > m)
                    m = s[t];
            }
            /* softmax weights */
            double l = 0.0;
            for (int t = 0; t < L; t++) {
                s[t] = exp(s[t] - m);
                l += s[t];
            }
            /* o = sum_t p_t V[t] */
            for (int t = 0; t < L; t++) {
                const double p = s[t] / l;
                const uint16_t *vsr = v_scales + (kv * Tmax + t) * nb;
                for (int d = 0; d < D; d++) {
                    const double v = oracle_half_to_double(vsr[d / ORACLE_BLOCK]) *
                                     (double)vt_codes[(kv * D + d) * Tmax + t];
                    oo[d] += p * v;
                    aa[d] += p * fabs(v);
                }
            }
        }
    }
    free(s);
    free(qd);
    return empty ? 2 : 0;
}
