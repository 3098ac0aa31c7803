/*
 * fp8bq oracle: a plain, slow, obviously-correct CPU statement of the
 * block-wise FP8 (E4M3) linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant generator with the CUDA path, and the
 * CUDA path never calls it.
 *
 * What the method is, by source passage (page: "NVIDIA NeMo RL Achieves 48%
 * Speedup With End-to-End FP8 Precision Training", three translations of one
 * article):
 *   - section "Technical breakthrough": block-wise quantized FP8 in the E4M3
 *     format, 128x128 tiles for weights and 1x128 tiles for activations; the
 *     linear layers do FP8 math;
 *   - section "Real-world performance gains": the scales are recalibrated
 *     after every training step (so quantization is a pure function of W);
 *   - section "Why this matters for AI economics": power-of-2 scaling factors
 *     are an option.
 * The pages fix nothing else.  The readings taken where they are silent are
 * stated beside each function (scale = amax/448, round-to-nearest-even with
 * saturation at +-448, the power-of-2 exponent rule, FP64 accumulation of the
 * dequantized operands as the GEMM definition).
 *
 * Pins (tests/test_oracle_*.py): every one of the 256 codes; two independent
 * encoders compared over all 2^32 fp32 bit patterns; the encoder compared with
 * torch's float8_e4m3fn cast where that cast is defined; scales against a
 * closed form; quantization against numpy float32 division + torch's cast;
 * GEMM against an exact integer matmul and numpy float64 matmul on cases
 * where the double sum is exact.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 * No FMA contraction, no flush-to-zero: float division is IEEE-754 binary32
 * division, correctly rounded, denormals kept.
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>
#include <omp.h>

#define O_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------- */
/* E4M3 (OCP 8-bit floating point, "E4M3" variant: 1 sign, 4 exponent bits   */
/* with bias 7, 3 mantissa bits, no infinities, NaN = S.1111.111).           */
/* The pages name only "E4M3"; the bit layout is the OCP definition.         */
/* ------------------------------------------------------------------------- */

/* Value of one code, exactly, in double.  NaN for S.1111.111. */
O_API double o_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int E = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0)
        v = ldexp((double)m, -9);                 /* subnormal: m * 2^-9 */
    else
        v = ldexp(1.0 + (double)m / 8.0, E - 7);  /* normal: 1.m * 2^(E-7) */
    return s ? -v : v;
}

/*
 * Encoder A (arithmetic).  Round-to-nearest-even onto the E4M3 grid, then
 * saturate: anything at or above 448 in magnitude becomes 448 (0x7E).  The
 * sign bit is kept for zero results (-0.0 and negative underflow give 0x80).
 * Every step is exact in double for a float input.
 */
O_API uint8_t o_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a;
    if (isnan(v)) return (uint8_t)(0x7F | sign);
    a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(0x7E | sign);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: grid step 2^-9; m == 8 is the smallest normal. */
        double m = nearbyint(a * 512.0);          /* default mode: to nearest, ties to even */
        return (uint8_t)((int)m | sign);
    } else {
        int ex;
        int E, f;
        (void)frexp(a, &ex);                      /* a = g * 2^ex, g in [0.5, 1) */
        E = ex - 1;                               /* a in [2^E, 2^(E+1)) */
        f = (int)nearbyint(ldexp(a, 3 - E) - 8.0);/* 3-bit fraction, ties to even */
        if (f == 8) { E += 1; f = 0; }            /* rounded up into the next binade */
        return (uint8_t)((((E + 7) << 3) | f) | sign);
    }
}

/* The 127 non-negative finite values, built from o_e4m3_decode. */
static double g_pos[127];
static int g_pos_ready = 0;
static void o_init_pos(void)
{
    int c;
    if (g_pos_ready) return;
    for (c = 0; c < 127; ++c) g_pos[c] = o_e4m3_decode((uint8_t)c);
    g_pos_ready = 1;
}

/*
 * Encoder B (brute force by definition).  The nearest of the 127
 * non-negative finite E4M3 values by absolute difference; on an exact tie the
 * code with an even last bit.  Magnitudes >= 448 saturate to 0x7E.  A
 * bisection finds the bracketing pair; the choice between the two is made by
 * comparing distances, not by any rounding instruction.
 */
O_API uint8_t o_e4m3_encode_nearest(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a, dlo, dhi;
    int lo, hi;
    if (isnan(v)) return (uint8_t)(0x7F | sign);
    if (!g_pos_ready) o_init_pos();
    a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(0x7E | sign);
    /* largest code lo with value <= a (g_pos is increasing, g_pos[0] = 0) */
    lo = 0; hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (g_pos[mid] <= a) lo = mid; else hi = mid - 1;
    }
    if (lo == 126) return (uint8_t)(126 | sign);
    hi = lo + 1;
    dlo = a - g_pos[lo];
    dhi = g_pos[hi] - a;
    if (dlo < dhi) return (uint8_t)(lo | sign);
    if (dhi < dlo) return (uint8_t)(hi | sign);
    return (uint8_t)(((lo & 1) == 0 ? lo : hi) | sign);
}

static float o_bits_to_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }

/*
 * Compare encoder A with encoder B over the fp32 bit patterns
 * [start, start+count) (NaN patterns are skipped).  Returns the number of
 * disagreements and the first one in *first_bad.
 */
O_API uint64_t o_sweep_encoders(uint64_t start, uint64_t count, uint32_t *first_bad)
{
    uint64_t bad = 0;
    uint64_t first = UINT64_MAX;
    int64_t i;
    o_init_pos();
#pragma omp parallel for schedule(static) reduction(+:bad) reduction(min:first)
    for (i = 0; i < (int64_t)count; ++i) {
        uint32_t b = (uint32_t)(start + (uint64_t)i);
        float v = o_bits_to_f32(b);
        if (isnan(v)) continue;
        if (o_e4m3_encode(v) != o_e4m3_encode_nearest(v)) {
            bad += 1;
            if ((uint64_t)b < first) first = b;
        }
    }
    if (first_bad) *first_bad = (first == UINT64_MAX) ? 0u : (uint32_t)first;
    return bad;
}

/* Encoder A applied to the fp32 bit patterns [start, start+count). */
O_API void o_encode_patterns(uint64_t start, uint64_t count, uint8_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < (int64_t)count; ++i)
        out[i] = o_e4m3_encode(o_bits_to_f32((uint32_t)(start + (uint64_t)i)));
}

/* Encoder A applied to an array of floats. */
O_API void o_encode_array(const float *v, int64_t n, uint8_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) out[i] = o_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------------- */
/* Scales                                                                    */
/* ------------------------------------------------------------------------- */

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
static float o_bf16(uint16_t h) { return o_bits_to_f32((uint32_t)h << 16); }

O_API float o_bf16_to_f32(uint16_t h) { return o_bf16(h); }

/*
 * Scale of one tile from its amax.
 *   mode 0 (fp32):  s = amax / 448, one IEEE binary32 division.  448 is the
 *                   largest E4M3 magnitude, so the tile's amax lands on it.
 *   mode 1 (pow2):  s = 2^e with e the smallest integer such that
 *                   amax <= 448 * 2^e (the exact form of 2^ceil(log2(amax/448))),
 *                   clamped to [-127, 127] so that s is a UE8M0 value.
 *   amax == 0:      s = 1 in both modes (an all-zero tile; avoids 0/0).
 * The option of power-of-2 scaling factors is named in section "Why this
 * matters for AI economics"; the formulae are the plainest full-range reading.
 */
O_API float o_scale(float amax, int mode)
{
    if (!(amax > 0.0f)) return 1.0f;
    if (mode == 0) return amax / 448.0f;
    {
        double a = (double)amax;
        int e;
        (void)frexp(a / 448.0, &e);               /* first guess, corrected below */
        while (a > ldexp(448.0, e)) e += 1;       /* exact comparisons in double */
        while (a <= ldexp(448.0, e - 1)) e -= 1;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
        return ldexpf(1.0f, e);                   /* 2^-127 is a binary32 denormal: exact */
    }
}

/* One quantized element: the fp32 quotient x/s (correctly rounded), then E4M3. */
static uint8_t o_qelem(float x, float s) { return o_e4m3_encode(x / s); }

/*
 * Activation quantization over 1x128 tiles (section "Technical breakthrough").
 * x: bf16 bits [M][ldx]; q: codes [M][ldq]; sa: scales [KB][ldsa], i.e. the
 * scale of tile (m, kb) is sa[kb*ldsa + m].  The last tile of a row may be
 * shorter than 128 (only in-bounds elements enter the amax).
 */
O_API void o_quant_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                       uint8_t *q, int64_t ldq, float *sa, int64_t ldsa, int mode)
{
    int64_t KB = (K + 127) / 128;
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int64_t kb;
        for (kb = 0; kb < KB; ++kb) {
            int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K, k;
            float amax = 0.0f, s;
            for (k = k0; k < k1; ++k) {
                float a = fabsf(o_bf16(x[m * ldx + k]));
                if (a > amax) amax = a;
            }
            s = o_scale(amax, mode);
            sa[kb * ldsa + m] = s;
            for (k = k0; k < k1; ++k) q[m * ldq + k] = o_qelem(o_bf16(x[m * ldx + k]), s);
        }
    }
}

/*
 * Weight quantization over 128x128 tiles (section "Technical breakthrough"),
 * which is also what the per-step recalibration computes for every weight
 * tensor (section "Real-world performance gains").
 * w: bf16 bits [N][ldw]; q: codes [N][ldq]; sw: scales [NB][KB] row-major.
 * Edge tiles are clipped to the tensor.
 */
O_API void o_quant_weight(const uint16_t *w, int64_t N, int64_t K, int64_t ldw,
                          uint8_t *q, int64_t ldq, float *sw, int mode)
{
    int64_t NB = (N + 127) / 128, KB = (K + 127) / 128;
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < NB * KB; ++t) {
        int64_t nb = t / KB, kb = t % KB;
        int64_t n0 = nb * 128, n1 = n0 + 128 < N ? n0 + 128 : N;
        int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
        int64_t n, k;
        float amax = 0.0f, s;
        for (n = n0; n < n1; ++n)
            for (k = k0; k < k1; ++k) {
                float a = fabsf(o_bf16(w[n * ldw + k]));
                if (a > amax) amax = a;
            }
        s = o_scale(amax, mode);
        sw[nb * KB + kb] = s;
        for (n = n0; n < n1; ++n)
            for (k = k0; k < k1; ++k) q[n * ldq + k] = o_qelem(o_bf16(w[n * ldw + k]), s);
    }
}

/* Dequantization: code value times its tile scale, exact in double. */
O_API void o_dequant_act(const uint8_t *q, int64_t M, int64_t K, int64_t ldq,
                         const float *sa, int64_t ldsa, double *out /* [M][K] */)
{
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int64_t k;
        for (k = 0; k < K; ++k)
            out[m * K + k] = o_e4m3_decode(q[m * ldq + k]) * (double)sa[(k / 128) * ldsa + m];
    }
}

O_API void o_dequant_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq,
                            const float *sw, double *out /* [N][K] */)
{
    int64_t KB = (K + 127) / 128;
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        int64_t k;
        for (k = 0; k < K; ++k)
            out[n * K + k] = o_e4m3_decode(q[n * ldq + k]) * (double)sw[(n / 128) * KB + (k / 128)];
    }
}

/*
 * Block-scaled GEMM, by definition: Y[m][n] = sum_k deq_a[m][k] * deq_w[n][k]
 * accumulated in double in ascending k, for the rows listed in rows[0..R)
 * (rows == NULL: all M rows, R ignored).  y is [R or M][N].
 * The linear layer computes Y = X W^T with both operands quantized
 * (section "Technical breakthrough"); the reference output is this FP64 sum
 * of the dequantized operands.
 */
O_API void o_gemm_rows(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                       const uint8_t *qw, int64_t ldw, const float *sw,
                       int64_t M, int64_t N, int64_t K,
                       const int64_t *rows, int64_t R, double *y)
{
    int64_t KB = (K + 127) / 128;
    int64_t nrows = rows ? R : M;
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        int64_t n;
        for (n = 0; n < N; ++n) {
            double acc = 0.0;
            int64_t k;
            for (k = 0; k < K; ++k) {
                double a = o_e4m3_decode(qa[m * lda + k]) * (double)sa[(k / 128) * ldsa + m];
                double b = o_e4m3_decode(qw[n * ldw + k]) * (double)sw[(n / 128) * KB + (k / 128)];
                acc += a * b;
            }
            y[i * N + n] = acc;
        }
    }
}

/*
 * Second formulation of the same GEMM: per 128-deep K block the exact integer
 * dot product of the codes scaled by 2^9 (every E4M3 value times 2^9 is an
 * integer), then the block sum times 2^-18 * sa * sw, accumulated over blocks
 * in double.  Agrees with o_gemm_rows to rounding of the double sums.
 */
O_API void o_gemm_blockint_rows(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                const uint8_t *qw, int64_t ldw, const float *sw,
                                int64_t M, int64_t N, int64_t K,
                                const int64_t *rows, int64_t R, double *y)
{
    int64_t KB = (K + 127) / 128;
    int64_t nrows = rows ? R : M;
    int64_t i;
    int64_t ival[256];
    int c;
    for (c = 0; c < 256; ++c) {
        double d = o_e4m3_decode((uint8_t)c);
        ival[c] = isnan(d) ? 0 : (int64_t)ldexp(d, 9);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        int64_t n;
        for (n = 0; n < N; ++n) {
            double acc = 0.0;
            int64_t kb;
            for (kb = 0; kb < KB; ++kb) {
                int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K, k;
                int64_t p = 0;
                for (k = k0; k < k1; ++k) p += ival[qa[m * lda + k]] * ival[qw[n * ldw + k]];
                acc += ldexp((double)p, -18) * (double)sa[kb * ldsa + m] * (double)sw[(n / 128) * KB + kb];
            }
            y[i * N + n] = acc;
        }
    }
}

/*
 * Grouped (mixture-of-experts) GEMM: rows [offsets[e], offsets[e+1]) of the
 * row-sorted activations use expert e's weight qw[e] ([N][K], codes) and
 * scales sw[e] ([NB][KB]).  Each expert's rows are o_gemm_rows with that
 * expert's operands.  Only rows listed in rows[0..R) are computed
 * (rows == NULL: all rows).  Section "Real-world performance gains" reports
 * the recipe on a mixture-of-experts model.
 */
O_API void o_grouped_gemm_rows(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                               const uint8_t *qw, const float *sw, const int64_t *offsets, int64_t E,
                               int64_t N, int64_t K, const int64_t *rows, int64_t R, double *y)
{
    int64_t NB = (N + 127) / 128, KB = (K + 127) / 128;
    int64_t total = offsets[E];
    int64_t nrows = rows ? R : total;
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        int64_t e = 0, n;
        while (e + 1 < E && offsets[e + 1] <= m) ++e;
        for (n = 0; n < N; ++n) {
            const uint8_t *w = qw + e * N * K;
            const float *s = sw + e * NB * KB;
            double acc = 0.0;
            int64_t k;
            for (k = 0; k < K; ++k) {
                double a = o_e4m3_decode(qa[m * lda + k]) * (double)sa[(k / 128) * ldsa + m];
                double b = o_e4m3_decode(w[n * K + k]) * (double)s[(n / 128) * KB + (k / 128)];
                acc += a * b;
            }
            y[i * N + n] = acc;
        }
    }
}

/*
 * The weight-gradient GEMM of a linear layer's backward pass, by definition:
 * dW[n][k] = sum over tokens m of dY[m][n] X[m][k], both operands quantized
 * over 1x128 tiles along the token axis (the contraction), given transposed:
 * a = codes of dY^T [N][lda] with scales sa[mb*ldsa + n], b = codes of X^T
 * [K][ldb] with scales sb[mb*ldsb + k].  Accumulated in double in ascending m,
 * for the rows listed in rows[0..R) (rows == NULL: all N rows).  y is [R or N][K].
 * Training in FP8 (section "Technical breakthrough": FP8 in both generation and
 * training) multiplies activations and gradients block-wise in the backward
 * pass as well; the 1x128 activation granularity is applied along the
 * contraction, the plainest reading for two activation-like operands.
 */
O_API void o_gemm_wgrad_rows(const uint8_t *a, int64_t lda, const float *sa, int64_t ldsa,
                             const uint8_t *b, int64_t ldb, const float *sb, int64_t ldsb,
                             int64_t N, int64_t K, int64_t M,
                             const int64_t *rows, int64_t R, double *y)
{
    int64_t nrows = rows ? R : N;
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < nrows; ++i) {
        int64_t n = rows ? rows[i] : i;
        int64_t k;
        for (k = 0; k < K; ++k) {
            double acc = 0.0;
            int64_t m;
            for (m = 0; m < M; ++m) {
                double da = o_e4m3_decode(a[n * lda + m]) * (double)sa[(m / 128) * ldsa + n];
                double db = o_e4m3_decode(b[k * ldb + m]) * (double)sb[(m / 128) * ldsb + k];
                acc += da * db;
            }
            y[i * K + k] = acc;
        }
    }
}

/* bf16 round-to-nearest-even of a double (single rounding).  NaN -> 0x7FC0. */
O_API uint16_t o_f64_to_bf16(double v)
{
    uint16_t sign;
    double a, m;
    int ex, E;
    if (isnan(v)) return 0x7FC0;
    sign = signbit(v) ? 0x8000 : 0;
    a = fabs(v);
    if (a == 0.0) return sign;
    /* largest finite bf16 = (2 - 2^-7) * 2^127; half a step above rounds to inf */
    if (a >= ldexp(2.0 - ldexp(1.0, -8), 127)) return (uint16_t)(sign | 0x7F80);
    (void)frexp(a, &ex);
    E = ex - 1;                                   /* a in [2^E, 2^(E+1)) */
    if (E < -126) E = -126;                       /* subnormal: fixed step 2^-133 */
    m = nearbyint(ldexp(a, 7 - E));               /* 8 significant bits, ties to even */
    if (E == -126 && m < 128.0) return (uint16_t)(sign | (uint16_t)m);
    if (m >= 256.0) { m /= 2.0; E += 1; }
    if (E > 127) return (uint16_t)(sign | 0x7F80);
    return (uint16_t)(sign | (uint16_t)(((E + 127) << 7) | ((int)m - 128)));
}

O_API void o_f64_to_bf16_array(const double *v, int64_t n, uint16_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) out[i] = o_f64_to_bf16(v[i]);
}

/*
 * The gated feed-forward activation between the gate+up projection and the
 * down projection of a Llama-style block.  The pages name Llama 3.1 8B
 * (section "Technical breakthrough"), whose feed-forward block is SwiGLU
 * (N. Shazeer, "GLU Variants Improve Transformer", 2020):
 *     h = silu(g) * u,   silu(g) = g * sigmoid(g) = g / (1 + e^-g),
 * with g the gate projection and u the up projection.  The same section keeps
 * non-linear functions in BF16: g and u are the BF16 outputs of the FP8 GEMM
 * and h is rounded to BF16 once; the arithmetic here is double.
 */
O_API double o_silu(double g) { return g / (1.0 + exp(-g)); }

O_API void o_swiglu_bf16(const uint16_t *g, const uint16_t *u, int64_t n, uint16_t *h)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) h[i] = o_f64_to_bf16(o_silu((double)o_bf16(g[i])) * (double)o_bf16(u[i]));
}

/*
 * Decode attention over an FP8 KV cache (section "Real-world performance
 * gains": an FP8 KV cache and FP8 attention take the speedup from the linear
 * layers' 15-25% to about 48%).  The cache holds E4M3 codes of every key and
 * value head vector with one scale per vector: the head dimension D = 128 is
 * exactly one 1x128 tile, the activation granularity of section "Technical
 * breakthrough".  For batch entry b, query head h and its key/value head
 * g = h / (Hq / Hkv) (grouped-query attention), over the cached tokens
 * t < lens[b]:
 *     s_t = scale * sum_d q[b][h][d] * dec(kq[b][t][g][d]) * ks[b][t][g]
 *     p_t = exp(s_t - max_t s_t) / sum_t exp(s_t - max_t s_t)
 *     o[b][h][d] = sum_t p_t * dec(vq[b][t][g][d]) * vs[b][t][g]
 * in double (q is bf16; out is double).  lens[b] = 0 gives o = 0.
 * Layouts: q [B][Hq][D]; kq, vq [B][S][Hkv][D]; ks, vs [B][S][Hkv].
 */
O_API void o_decode_attention(const uint16_t *q, const uint8_t *kq, const float *ks, const uint8_t *vq,
                              const float *vs, const int32_t *lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t S,
                              int64_t D, double scale, double *out)
{
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < B * Hq; ++bh) {
        int64_t b = bh / Hq, h = bh % Hq, g = h / (Hq / Hkv);
        int64_t L = lens[b], t, d;
        double mx = -HUGE_VAL, den = 0.0;
        double *o = out + bh * D;
        double *sc = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        for (d = 0; d < D; ++d) o[d] = 0.0;
        for (t = 0; t < L; ++t) {
            const uint8_t *k = kq + ((b * S + t) * Hkv + g) * D;
            double dot = 0.0;
            for (d = 0; d < D; ++d) dot += (double)o_bf16(q[bh * D + d]) * o_e4m3_decode(k[d]);
            sc[t] = scale * dot * (double)ks[(b * S + t) * Hkv + g];
            if (sc[t] > mx) mx = sc[t];
        }
        for (t = 0; t < L; ++t) {
            const uint8_t *v = vq + ((b * S + t) * Hkv + g) * D;
            double p = exp(sc[t] - mx), sv = (double)vs[(b * S + t) * Hkv + g];
            den += p;
            for (d = 0; d < D; ++d) o[d] += p * o_e4m3_decode(v[d]) * sv;
        }
        if (L > 0)
            for (d = 0; d < D; ++d) o[d] /= den;
        free(sc);
    }
}

/*
 * Causal (prefill) attention over FP8 queries, keys and values: the "FP8 KV
 * cache and attention" of section "Real-world performance gains", for the
 * many-query case.  Every query, key and value head vector (D = 128) is one
 * 1x128 tile of section "Technical breakthrough": E4M3 codes and one scale.
 * Query row i of sequence b (i < lens[b]) attends the keys j <= i of its own
 * sequence; query head h reads key/value head h / (Hq / Hkv):
 *   s_j   = scale * qs[b,i,h] * ks[b,j,g] * sum_d dec(qq[b,i,h,d]) dec(kq[b,j,g,d])
 *   p_j   = exp(s_j - max_j s) / sum_j exp(s_j - max_j s)
 *   o[d]  = sum_j p_j * vs[b,j,g] * dec(vq[b,j,g,d])
 * everything in double.  Rows i >= lens[b] are 0.  When `mag` is not NULL it
 * also receives sum_j p_j |vs[b,j,g] dec(vq[b,j,g,d])|, the size of the terms
 * of o[d] (an error bound of a kernel that rounds the weights p_j is
 * proportional to it).
 * rows: the query rows to compute (indices b * S + i), or NULL for all; out
 * (and mag) are [R][Hq][D] for R = nrows (or B * S).
 */
O_API void o_prefill_attention(const uint8_t *qq, const float *qs, const uint8_t *kq, const float *ks,
                               const uint8_t *vq, const float *vs, const int32_t *lens, int64_t B, int64_t S,
                               int64_t Hq, int64_t Hkv, int64_t D, double scale, const int64_t *rows, int64_t nrows,
                               double *out, double *mag)
{
    const int64_t R = rows ? nrows : B * S;
    int64_t rh;
#pragma omp parallel for schedule(dynamic, 1)
    for (rh = 0; rh < R * Hq; ++rh) {
        const int64_t r = rh / Hq, h = rh % Hq, g = h / (Hq / Hkv);
        const int64_t bi = rows ? rows[r] : r;
        const int64_t b = bi / S, i = bi % S;
        int64_t L = lens[b] < S ? lens[b] : S, j, d;
        double mx = -HUGE_VAL, den = 0.0;
        double *o = out + rh * D;
        double *m = mag ? mag + rh * D : NULL;
        double *sc;
        for (d = 0; d < D; ++d) {
            o[d] = 0.0;
            if (m) m[d] = 0.0;
        }
        if (i >= L) continue;
        sc = (double *)malloc(sizeof(double) * (size_t)(i + 1));
        for (j = 0; j <= i; ++j) {
            const uint8_t *qv = qq + ((b * S + i) * Hq + h) * D;
            const uint8_t *kv = kq + ((b * S + j) * Hkv + g) * D;
            double dot = 0.0;
            for (d = 0; d < D; ++d) dot += o_e4m3_decode(qv[d]) * o_e4m3_decode(kv[d]);
            sc[j] = scale * (double)qs[(b * S + i) * Hq + h] * (double)ks[(b * S + j) * Hkv + g] * dot;
            if (sc[j] > mx) mx = sc[j];
        }
        for (j = 0; j <= i; ++j) den += exp(sc[j] - mx);
        for (j = 0; j <= i; ++j) {
            const uint8_t *vv = vq + ((b * S + j) * Hkv + g) * D;
            const double p = exp(sc[j] - mx) / den, sv = (double)vs[(b * S + j) * Hkv + g];
            for (d = 0; d < D; ++d) {
                const double t = p * sv * o_e4m3_decode(vv[d]);
                o[d] += t;
                if (m) m[d] += fabs(t);
            }
        }
        free(sc);
    }
}

/*
 * One optimizer step of an FP32 master weight, the step after which the
 * scales are recalibrated (section "Real-world performance gains": the policy
 * weights change every training step).  The pages do not name the optimizer;
 * the reading is AdamW (I. Loshchilov, F. Hutter, "Decoupled Weight Decay
 * Regularization", ICLR 2019, Algorithm 2, with Adam's bias-corrected moments
 * of D. Kingma, J. Ba, "Adam", ICLR 2015) on binary32 state, the usual
 * mixed-precision recipe.  Every operation below is one IEEE binary32
 * operation, in this order (no contraction, -ffp-contract=off):
 *   m' = b1 m + (1 - b1) g
 *   v' = b2 v + ((1 - b2) g) g
 *   m^ = m' / bc1,  v^ = v' / bc2,   bc_i = 1 - b_i^t  (double pow, rounded to binary32)
 *   p' = p - lr (m^ / (sqrt(v^) + eps) + wd p)
 */
O_API void o_adamw_step(float *p, const float *g, float *m, float *v, int64_t n, float lr, float b1, float b2,
                        float eps, float wd, int64_t step)
{
    const float bc1 = (float)(1.0 - pow((double)b1, (double)step));
    const float bc2 = (float)(1.0 - pow((double)b2, (double)step));
    const float c1 = 1.0f - b1, c2 = 1.0f - b2;
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) {
        float mi = b1 * m[i] + c1 * g[i];
        float vi = b2 * v[i] + (c2 * g[i]) * g[i];
        float mh = mi / bc1;
        float vh = vi / bc2;
        float d = sqrtf(vh) + eps;
        float u = mh / d + wd * p[i];
        p[i] = p[i] - lr * u;
        m[i] = mi;
        v[i] = vi;
    }
}

/* binary32 -> bf16, round to nearest even (exact through double). */
O_API void o_f32_to_bf16_array(const float *x, int64_t n, uint16_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) out[i] = o_f64_to_bf16((double)x[i]);
}

O_API int o_num_threads(void) { return omp_get_max_threads(); }
