/*
 * Plain CPU oracle for the W4A16 group-128 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's compute path may call,
 * link or include this file; only the tests, the smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code with the CUDA library.
 *
 * What it computes (tiny-llm, "Week 2 Day 6: SIMD-Matrix Prefill": the
 * introduction fixes 4-bit weights, group size 128, BF16 activations, BF16
 * quantisation parameters, BF16 output and FP32 accumulators; Task 3 fixes one
 * scale and one bias per 128 reduction values):
 *
 *   1. unpack   q[n,k] = (wq[n*(K/8) + k/8] >> (4*(k%8))) & 15
 *   2. dequant  w[n,k] = float(s[n,k/128]) * float(q[n,k]) + float(b[n,k/128])
 *               (two FP32 roundings: the product, then the sum)
 *   3. dot      acc = 0; for k = 0..K-1: acc = acc + float(x[m,k]) * w[n,k]
 *               (FP32, product and sum rounded separately, k ascending)
 *   4. store    y[m,n] = bf16_round_to_nearest_even(acc)
 *
 * This is the plain definition; it must be compiled without contraction of
 * a*b+c into fused multiply-adds (-ffp-contract=off) and without fast-math.
 * Outputs are independent, so they may be computed by several threads; the
 * arithmetic of each output is the sequence above regardless.
 *
 * The quantiser (w4a16_oracle_quantize) produces the packed format above from
 * FP32 or BF16 weights.  Its recipe is the one the reference problem's inputs
 * are made with (affine min/max quantisation per 128-group: scale = (max - min)
 * / 15, bias = min, q = round and clamp to 0..15, eight codes per uint32 low
 * nibble first); the steps are spelled out above the function.
 *
 * The same layer with 2- or 8-bit codes (w4a16_oracle_matmul_bits; the
 * "Route affine qmv_wide by bit-width and batch size" PR routes the affine
 * format by its bit width b): 32 / b codes per uint32, the lowest code in the
 * lowest bits, so step 1 reads
 *   q[n,k] = (wq[n*(K*b/32) + k/(32/b)] >> (b*(k%(32/b)))) & (2^b - 1)
 * and steps 2-4 are unchanged.
 *
 * BF16 values are passed as uint16_t bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#if defined(__FAST_MATH__)
#error "the oracle must not be built with fast-math"
#endif

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u) {          /* inf or nan */
        if (u & 0x007fffffu)
            return (uint16_t)((u >> 16) | 0x0040u);  /* quiet nan */
        return (uint16_t)(u >> 16);
    }
    /* add half an ulp of bf16, plus one more when the kept lsb is odd: ties go to even */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static unsigned unpack_code(const uint32_t *wq, int64_t K, int64_t n, int64_t k)
{
    uint32_t word = wq[n * (K / 8) + k / 8];
    return (unsigned)((word >> (4 * (k % 8))) & 15u);
}

static float dot_fp32(const uint16_t *x, const uint32_t *wq, const uint16_t *s,
                      const uint16_t *b, int64_t K, int64_t m, int64_t n)
{
    const int64_t G = K / 128;
    float acc = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        const float sc = bf16_to_f32(s[n * G + k / 128]);
        const float bi = bf16_to_f32(b[n * G + k / 128]);
        const float q = (float)unpack_code(wq, K, n, k);
        const float sq = sc * q;
        const float w = sq + bi;
        const float xv = bf16_to_f32(x[m * K + k]);
        const float p = xv * w;
        acc = acc + p;
    }
    return acc;
}

/* Status: 0 ok, 1 bad argument (null pointer, negative size, K % 128 != 0). */
static int check(const void *x, const void *wq, const void *s, const void *b,
                 const void *y, int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0 || K % 128 != 0)
        return 1;
    if (M > 0 && N > 0 && (!x || !wq || !s || !b || !y))
        return 1;
    return 0;
}

/* y[M,N] bf16 bits = x[M,K] . dequant(wq)^T, steps 1-4 above. */
int w4a16_oracle_matmul(const uint16_t *x, const uint32_t *wq, const uint16_t *s,
                        const uint16_t *b, uint16_t *y, int64_t M, int64_t N,
                        int64_t K)
{
    if (check(x, wq, s, b, y, M, N, K))
        return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = f32_to_bf16_rne(dot_fp32(x, wq, s, b, K, m, n));
    return 0;
}

/* Same as above but stops before step 4: the FP32 accumulator itself. */
int w4a16_oracle_matmul_f32(const uint16_t *x, const uint32_t *wq, const uint16_t *s,
                            const uint16_t *b, float *acc, int64_t M, int64_t N,
                            int64_t K)
{
    if (check(x, wq, s, b, acc, M, N, K))
        return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            acc[m * N + n] = dot_fp32(x, wq, s, b, K, m, n);
    return 0;
}

/*
 * Fused gate/up projection with the SwiGLU product.  wq, s, b hold 2 N2 rows, the
 * gate and up layers interleaved in blocks of 8: rows 16 (j / 8) + j % 8 (gate j) and
 * 16 (j / 8) + 8 + j % 8 (up j).  For each output:
 *   g, u = the plain dots of the gate and up rows (steps 1-3 above, FP32)
 *   h    = bf16_rne((float)(silu(g) * u)), silu(g) = g / (1 + exp(-g)) in double
 * (the product is rounded to FP32, then to BF16).
 */
static double silu(double g)
{
    return g / (1.0 + exp(-g));
}

int w4a16_oracle_gate_up(const uint16_t *x, const uint32_t *wq, const uint16_t *s,
                         const uint16_t *b, uint16_t *h, int64_t M, int64_t N2, int64_t K)
{
    if (N2 < 0 || N2 % 8 != 0 || check(x, wq, s, b, h, M, 2 * N2, K))
        return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N2; ++j) {
            const int64_t gate_row = 16 * (j / 8) + j % 8;
            const int64_t up_row = gate_row + 8;
            const double gv = (double)dot_fp32(x, wq, s, b, K, m, gate_row);
            const double uv = (double)dot_fp32(x, wq, s, b, K, m, up_row);
            h[m * N2 + j] = f32_to_bf16_rne((float)(silu(gv) * uv));
        }
    return 0;
}

/*
 * b-bit codes (b = 2, 4 or 8): step 1 with 32 / b codes per word, then steps 2-4 exactly
 * as dot_fp32 takes them.
 */
static unsigned unpack_code_bits(const uint32_t *wq, int64_t K, int64_t n, int64_t k, int bits)
{
    const int64_t per_word = 32 / bits;
    const uint32_t word = wq[n * (K / per_word) + k / per_word];
    return (unsigned)((word >> (bits * (k % per_word))) & ((1u << bits) - 1u));
}

static float dot_fp32_bits(const uint16_t *x, const uint32_t *wq, const uint16_t *s,
                           const uint16_t *b, int64_t K, int64_t m, int64_t n, int bits)
{
    const int64_t G = K / 128;
    float acc = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        const float sc = bf16_to_f32(s[n * G + k / 128]);
        const float bi = bf16_to_f32(b[n * G + k / 128]);
        const float q = (float)unpack_code_bits(wq, K, n, k, bits);
        const float sq = sc * q;
        const float w = sq + bi;
        const float xv = bf16_to_f32(x[m * K + k]);
        const float p = xv * w;
        acc = acc + p;
    }
    return acc;
}

/* y[M,N] bf16 bits = x[M,K] . dequant(wq)^T with b-bit codes; status 1 also for b not 2, 4, 8. */
int w4a16_oracle_matmul_bits(const uint16_t *x, const uint32_t *wq, const uint16_t *s,
                             const uint16_t *b, uint16_t *y, int64_t M, int64_t N,
                             int64_t K, int bits)
{
    if ((bits != 2 && bits != 4 && bits != 8) || check(x, wq, s, b, y, M, N, K))
        return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = f32_to_bf16_rne(dot_fp32_bits(x, wq, s, b, K, m, n, bits));
    return 0;
}

/* Step 1 alone for b-bit codes: q[N,K] as bytes. */
int w4a16_oracle_unpack_bits(const uint32_t *wq, uint8_t *q, int64_t N, int64_t K, int bits)
{
    if ((bits != 2 && bits != 4 && bits != 8) || N < 0 || K < 0 || K % (32 / bits) != 0 ||
        (N > 0 && K > 0 && (!wq || !q)))
        return 1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (uint8_t)unpack_code_bits(wq, K, n, k, bits);
    return 0;
}

/* Step 1 alone: q[N,K] codes as bytes. */
int w4a16_oracle_unpack(const uint32_t *wq, uint8_t *q, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 8 != 0 || (N > 0 && K > 0 && (!wq || !q)))
        return 1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (uint8_t)unpack_code(wq, K, n, k);
    return 0;
}

/* Step 4 alone, for the rounding pins: float32 -> bf16 bits. */
void w4a16_oracle_round_bf16(const float *a, uint16_t *out, int64_t count)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = f32_to_bf16_rne(a[i]);
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int w4a16_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Cap the threads later parallel regions use (no effect without OpenMP). */
void w4a16_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Quantiser, one 128-group v[0..127] of one weight row:
 *   1. lo = min, hi = max of the 128 values (compared in k order); a zero lo or hi
 *      is taken as +0, so the result does not depend on the order of the values
 *   2. scale = bf16_rne((hi - lo) / 15)    FP32 subtraction, FP32 division
 *      bias  = bf16_rne(lo)
 *   3. with sc, bi the BF16 scale and bias widened to FP32:
 *      q[k] = 0 when sc == 0 (a constant group), else
 *      q[k] = clamp(nearbyint((v[k] - bi) / sc), 0, 15)   FP32 subtraction and
 *             division, nearbyint in the default rounding mode (half to even)
 *   4. word j of the group = sum over i < 8 of q[8 j + i] << (4 i)
 * Inputs must be finite.
 */
static void quantize_group(const float *v, uint32_t *words, uint16_t *scale, uint16_t *bias)
{
    float lo = v[0], hi = v[0];
    for (int j = 1; j < 128; ++j) {
        if (v[j] < lo)
            lo = v[j];
        if (v[j] > hi)
            hi = v[j];
    }
    if (lo == 0.0f)
        lo = 0.0f;
    if (hi == 0.0f)
        hi = 0.0f;
    const float range = hi - lo;
    const float step = range / 15.0f;
    *scale = f32_to_bf16_rne(step);
    *bias = f32_to_bf16_rne(lo);
    const float sc = bf16_to_f32(*scale);
    const float bi = bf16_to_f32(*bias);
    for (int j = 0; j < 16; ++j)
        words[j] = 0u;
    for (int j = 0; j < 128; ++j) {
        uint32_t code = 0u;
        if (sc != 0.0f) {
            const float d = v[j] - bi;
            const float t = d / sc;
            const float r = nearbyintf(t);
            code = r < 0.0f ? 0u : (r > 15.0f ? 15u : (uint32_t)r);
        }
        words[j / 8] |= code << (4 * (j % 8));
    }
}

static int quantize_check(const void *w, const void *wq, const void *s, const void *b, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 128 != 0)
        return 1;
    if (N > 0 && K > 0 && (!w || !wq || !s || !b))
        return 1;
    return 0;
}

/* W [N,K] FP32 -> wq [N,K/8], scales and biases [N,K/128] BF16 bits. */
int w4a16_oracle_quantize(const float *w, uint32_t *wq, uint16_t *s, uint16_t *b, int64_t N, int64_t K)
{
    if (quantize_check(w, wq, s, b, N, K))
        return 1;
    const int64_t G = K / 128;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            quantize_group(w + n * K + g * 128, wq + n * (K / 8) + g * 16, s + n * G + g, b + n * G + g);
    return 0;
}

/* The same from BF16 weights: each value widened to FP32 (exactly), then as above. */
int w4a16_oracle_quantize_bf16(const uint16_t *w, uint32_t *wq, uint16_t *s, uint16_t *b, int64_t N, int64_t K)
{
    if (quantize_check(w, wq, s, b, N, K))
        return 1;
    const int64_t G = K / 128;
    float v[128];
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            for (int j = 0; j < 128; ++j)
                v[j] = bf16_to_f32(w[n * K + g * 128 + j]);
            quantize_group(v, wq + n * (K / 8) + g * 16, s + n * G + g, b + n * G + g);
        }
    return 0;
}
