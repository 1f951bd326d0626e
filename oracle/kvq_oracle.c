/*
 * kvq_oracle.c -- the plain, slow, obviously correct CPU oracle for the KV-cache
 * compression path.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the
 * smoke check and by the CPU-baseline leg of the benchmark, never by the product
 * path.  It shares no source with the CUDA library (no header, no helper, no table).
 *
 * Every function is the definition written out with scalar loops, in the order the
 * pages state it.  Build flags: -O2 -fno-fast-math -ffp-contract=off, so each fp32
 * operation below is one IEEE-754 operation rounded to nearest-even, exactly as written
 * (x86-64 SSE arithmetic, FLT_EVAL_METHOD == 0).
 *
 * Sources (web pages; cited by title and section):
 *  [INT8]  "Q-TensorFormer" model card, section 6 "Adaptive KV Cache Quantization &
 *          Attention-Sink Eviction", Symmetric Channel-Wise INT8 equation:
 *          X_hat = clamp(round(X / s8), -128, 127) * s8,  s8 = max|X| / 127.
 *  [PAPER] "GPU-Accelerated INT8 Quantization for KV Cache Compression in Large
 *          Language Models" (arXiv 2601.04719), abstract: INT8 KV-cache quantization,
 *          reconstruction error and attention-score error.
 *  [QJL]   "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
 *          Overhead" (arXiv 2406.03482), abstract: a JL transform followed by sign-bit
 *          quantization of one vector, an unquantized JL transform of the other, and an
 *          asymmetric unbiased inner-product estimator.
 *  [GQA]   "Q-TensorFormer" model card, section 4 "Grouped-Query Attention (GQA) &
 *          Multi-Query Attention (MQA)": KV head broadcast by unsqueeze/expand/reshape.
 *  [INT4]  "Q-TensorFormer" model card, section 6, Asymmetric Group-Wise INT4 equations:
 *          X_hat = clamp(round((X - z4) / s4), 0, 15) * s4 + z4,
 *          s4 = (max X - min X) / 15,  z4 = min X.
 *  [RES]   "Кризис отменяется: Google изобрел квантовый алгоритм сокращения объема памяти
 *          для ИИ в 6 раз" (news page on TurboQuant): a first quantizer does
 *          most of the compression and a 1-bit QJL layer then corrects its residual
 *          error, one sign bit per sketch coordinate, for better attention scores.  The
 *          first stage here is [INT4]; the residual is the key minus its INT4
 *          reconstruction, and the score is the reconstruction's dot product plus the
 *          [QJL] estimate of the residual's.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - granularity is one scale per row of head_dim ("per token");
 *  - round() is round-half-to-even of the fp32 quotient x / s, with s the STORED fp32
 *    scale fl32(a / 127) and IEEE division;
 *  - a row whose scale is 0 (absmax 0, or absmax so small that a/127 underflows) gets
 *    codes 0;
 *  - QJL: bit i = [ (S k)_i >= 0 ], packed LSB-first, 32 coordinates per uint32 word;
 *    the key norm is stored as fp16 (round to nearest even of the fp64 norm);
 *  - estimator: sqrt(pi/2)/m * ||k|| * sum_i (S q)_i * (2 bit_i - 1)  (unbiased for
 *    Gaussian S with unit-variance entries), using the stored fp16 norm and the fp32
 *    stored query sketch;
 *  - decode attends to every cached token (no mask), logits = sm_scale * score with
 *    sm_scale = 1/sqrt(D) by default, softmax and value sum accumulated in fp32 in
 *    token order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORA_F32 0
#define ORA_F16 1
#define ORA_KEYS_INT8 0
#define ORA_KEYS_QJL 1
#define ORA_KEYS_QJLRES 2

/* ---------------------------------------------------------------------------------
 * IEEE-754 binary16 <-> binary64, written from the format's definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits).
 * ------------------------------------------------------------------------------- */
/* The all-cores build (-fopenmp) runs the outer loops over rows, keys or (batch, head)
 * units in parallel; every row, key or unit is computed by one thread exactly as in the
 * plain build, so the results are identical.  Threads the all-cores build uses (1 in
 * the plain build). */
int ora_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

double ora_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);              /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25);  /* (1.f) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round a binary64 value to the nearest binary16 value, ties to even. */
uint16_t ora_double_to_half(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    if (a >= 65520.0) return sign | 0x7c00;     /* halfway to 2^16 and beyond -> inf */
    if (a < ldexp(1.0, -14)) {                  /* subnormal range, quantum 2^-24 */
        double q = nearbyint(ldexp(a, 24));     /* exact scaling, then RNE */
        return sign | (uint16_t)q;              /* q == 1024 encodes 2^-14 correctly */
    }
    int E;
    frexp(a, &E);                               /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;                              /* a in [2^e, 2^(e+1)) */
    double q = nearbyint(ldexp(a, 10 - e));     /* significand in [1024, 2048] */
    if (q == 2048.0) { q = 1024.0; e += 1; }
    if (e > 15) return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

static float load_elem(const void* x, int dtype, int64_t i) {
    if (dtype == ORA_F16) return (float)ora_half_to_double(((const uint16_t*)x)[i]);
    return ((const float*)x)[i];
}

/* ---------------------------------------------------------------------------------
 * [INT8] quantize: per row r,  a = max_j |x_rj|,  s = fl32(a / 127),
 *        c_rj = clamp(round_half_even(fl32(x_rj / s)), -128, 127);  s == 0 -> c = 0.
 * x is fp32 or fp16 (widened exactly), row-major [n_rows][d].
 * ------------------------------------------------------------------------------- */
int ora_quantize_int8(const void* x, int dtype, int64_t n_rows, int64_t d,
                      int8_t* codes, float* scales) {
    if (n_rows < 0 || d <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        float a = 0.0f;
        for (int64_t j = 0; j < d; ++j) {
            float v = fabsf(load_elem(x, dtype, r * d + j));
            if (v > a) a = v;
        }
        float s = a / 127.0f;
        scales[r] = s;
        for (int64_t j = 0; j < d; ++j) {
            int8_t c = 0;
            if (s != 0.0f) {
                float qt = load_elem(x, dtype, r * d + j) / s;
                float rq = nearbyintf(qt);             /* default mode: ties to even */
                if (rq < -128.0f) rq = -128.0f;
                if (rq > 127.0f) rq = 127.0f;
                c = (int8_t)rq;
            }
            codes[r * d + j] = c;
        }
    }
    return 0;
}

/* [INT8] dequantize: x_hat = fl32(c * s); fp16 output is the fp32 value rounded to
 * nearest-even fp16. */
int ora_dequantize_int8(const int8_t* codes, const float* scales, int64_t n_rows,
                        int64_t d, void* out, int out_dtype) {
    if (n_rows < 0 || d <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        for (int64_t j = 0; j < d; ++j) {
            float v = (float)codes[r * d + j] * scales[r];
            if (out_dtype == ORA_F16)
                ((uint16_t*)out)[r * d + j] = ora_double_to_half((double)v);
            else
                ((float*)out)[r * d + j] = v;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------------
 * [INT8] channel-wise: the same equation with one scale per column.  x holds n_blocks
 * blocks of [rows][d] (row-major, blocks one after another); for block b and column j:
 *   a = max_r |x_brj|,  s_bj = fl32(a / 127),
 *   c_brj = clamp(round_half_even(fl32(x_brj / s_bj)), -128, 127);  s_bj == 0 -> c = 0.
 * scales: [n_blocks][d].
 * ------------------------------------------------------------------------------- */
int ora_quantize_int8_channelwise(const void* x, int dtype, int64_t n_blocks, int64_t rows,
                                  int64_t d, int8_t* codes, float* scales) {
    if (n_blocks < 0 || rows <= 0 || d <= 0) return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < n_blocks; ++b) {
        for (int64_t j = 0; j < d; ++j) {
            float a = 0.0f;
            for (int64_t r = 0; r < rows; ++r) {
                float v = fabsf(load_elem(x, dtype, (b * rows + r) * d + j));
                if (v > a) a = v;
            }
            float s = a / 127.0f;
            scales[b * d + j] = s;
            for (int64_t r = 0; r < rows; ++r) {
                int8_t c = 0;
                if (s != 0.0f) {
                    float qt = load_elem(x, dtype, (b * rows + r) * d + j) / s;
                    float rq = nearbyintf(qt);
                    if (rq < -128.0f) rq = -128.0f;
                    if (rq > 127.0f) rq = 127.0f;
                    c = (int8_t)rq;
                }
                codes[(b * rows + r) * d + j] = c;
            }
        }
    }
    return 0;
}

/* [INT8] channel-wise dequantize: x_hat_brj = fl32(c_brj * s_bj). */
int ora_dequantize_int8_channelwise(const int8_t* codes, const float* scales, int64_t n_blocks,
                                    int64_t rows, int64_t d, void* out, int out_dtype) {
    if (n_blocks < 0 || rows <= 0 || d <= 0) return 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < n_blocks; ++b)
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t j = 0; j < d; ++j) {
                int64_t i = (b * rows + r) * d + j;
                float v = (float)codes[i] * scales[b * d + j];
                if (out_dtype == ORA_F16) ((uint16_t*)out)[i] = ora_double_to_half((double)v);
                else ((float*)out)[i] = v;
            }
    return 0;
}

/* ---------------------------------------------------------------------------------
 * [INT4] asymmetric group-wise: each row of d is cut into groups of g consecutive
 * elements.  Per group:  mn = min x,  mx = max x,  s4 = fl32(fl32(mx - mn) / 15),
 * z4 = mn,  c = clamp(round_half_even(fl32(fl32(x - z4) / s4)), 0, 15)  (s4 == 0 ->
 * c = 0).  Codes are packed two per byte: element 2i in bits 0-3, element 2i+1 in
 * bits 4-7 (packed: [n_rows][d/2]); scales and zeros: [n_rows][d/g] fp32.
 * ------------------------------------------------------------------------------- */
int ora_quantize_int4_group(const void* x, int dtype, int64_t n_rows, int64_t d, int g,
                            uint8_t* packed, float* scales, float* zeros) {
    if (n_rows < 0 || d <= 0 || g <= 0 || (d % g) != 0 || (g % 2) != 0) return 1;
    int64_t ng = d / g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        for (int64_t k = 0; k < ng; ++k) {
            int64_t o = r * d + k * g;
            float mn = load_elem(x, dtype, o), mx = mn;
            for (int e = 1; e < g; ++e) {
                float v = load_elem(x, dtype, o + e);
                if (v < mn) mn = v;
                if (v > mx) mx = v;
            }
            float s = (mx - mn) / 15.0f;
            scales[r * ng + k] = s;
            zeros[r * ng + k] = mn;
            for (int e = 0; e < g; ++e) {
                int c = 0;
                if (s != 0.0f) {
                    float qt = (load_elem(x, dtype, o + e) - mn) / s;
                    float rq = nearbyintf(qt);
                    if (rq < 0.0f) rq = 0.0f;
                    if (rq > 15.0f) rq = 15.0f;
                    c = (int)rq;
                }
                int64_t i = o + e;
                uint8_t* byte = &packed[i / 2];
                if ((i % 2) == 0) *byte = (uint8_t)((*byte & 0xF0) | c);
                else *byte = (uint8_t)((*byte & 0x0F) | (c << 4));
            }
        }
    }
    return 0;
}

/* [INT4] dequantize: x_hat = fl32(fl32(c * s4) + z4). */
static float int4_value(const uint8_t* packed, const float* scales, const float* zeros,
                        int64_t r, int64_t d, int g, int64_t j) {
    int64_t i = r * d + j;
    int c = (packed[i / 2] >> ((i % 2) * 4)) & 0xF;
    int64_t k = r * (d / g) + j / g;
    float cs = (float)c * scales[k];
    return cs + zeros[k];
}

int ora_dequantize_int4_group(const uint8_t* packed, const float* scales, const float* zeros,
                              int64_t n_rows, int64_t d, int g, void* out, int out_dtype) {
    if (n_rows < 0 || d <= 0 || g <= 0 || (d % g) != 0 || (g % 2) != 0) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int64_t j = 0; j < d; ++j) {
            float v = int4_value(packed, scales, zeros, r, d, g, j);
            if (out_dtype == ORA_F16) ((uint16_t*)out)[r * d + j] = ora_double_to_half((double)v);
            else ((float*)out)[r * d + j] = v;
        }
    return 0;
}

/* [PAPER] attention score against an INT8 row: score = sum_j q_j * x_hat_j, with
 * x_hat_j = fl32(c_j * s), accumulated in fp32 in index order. */
static float int8_row_score(const float* q, const int8_t* c, float s, int64_t d) {
    float acc = 0.0f;
    for (int64_t j = 0; j < d; ++j) {
        float xh = (float)c[j] * s;
        float prod = q[j] * xh;
        acc = acc + prod;
    }
    return acc;
}

/* Scores of one query (fp32 or fp16, length d) against every row of an INT8 matrix. */
int ora_int8_scores(const void* q, int q_dtype, const int8_t* codes, const float* scales,
                    int64_t n_rows, int64_t d, float* scores) {
    if (n_rows < 0 || d <= 0) return 1;
    float* qf = (float*)malloc(sizeof(float) * (size_t)d);
    if (!qf) return 2;
    for (int64_t j = 0; j < d; ++j) qf[j] = load_elem(q, q_dtype, j);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        scores[r] = int8_row_score(qf, codes + r * d, scales[r], d);
    free(qf);
    return 0;
}

/* ---------------------------------------------------------------------------------
 * [QJL] sketch of keys: u = S k (S is m x d, row-major, any real entries; the fp16
 * sketch matrix is passed widened to fp64), computed in fp64;
 * bit i = [u_i >= 0], word w bit j <-> coordinate i = 32 w + j;
 * norm = fp16(||k||_2) with the sum of squares and the root in fp64.
 * u_out (optional, [n_keys][m]) receives the fp64 projections.
 * ------------------------------------------------------------------------------- */
int ora_qjl_encode(const uint16_t* keys_f16, int64_t n_keys, int d, const double* S,
                   int m, uint32_t* words, uint16_t* norms_f16, double* u_out) {
    if (n_keys < 0 || d <= 0 || m <= 0 || (m % 32) != 0) return 1;
    int nw = m / 32;
    int fail = 0;
#pragma omp parallel
    {
        double* k = (double*)malloc(sizeof(double) * (size_t)d);   /* one per thread */
        if (!k) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(static)
        for (int64_t n = 0; n < n_keys; ++n) {
            if (!k) continue;
            double ss = 0.0;
            for (int j = 0; j < d; ++j) {
                k[j] = ora_half_to_double(keys_f16[n * d + j]);
                ss += k[j] * k[j];
            }
            for (int w = 0; w < nw; ++w) words[n * nw + w] = 0u;
            for (int i = 0; i < m; ++i) {
                double u = 0.0;
                for (int j = 0; j < d; ++j) u += S[(int64_t)i * d + j] * k[j];
                if (u_out) u_out[n * m + i] = u;
                if (u >= 0.0) words[n * nw + i / 32] |= (1u << (i % 32));
            }
            norms_f16[n] = ora_double_to_half(sqrt(ss));
        }
        free(k);
    }
    return fail ? 2 : 0;
}

/* [QJL] the query side: the plain (unquantized) JL transform v = S q, fp64, returned in
 * fp64 (v64) and as the stored fp32 value (v32).  Either output may be NULL. */
int ora_qjl_query_sketch(const void* q, int q_dtype, int64_t n_q, int d, const double* S,
                         int m, double* v64, float* v32) {
    if (n_q < 0 || d <= 0 || m <= 0) return 1;
    for (int64_t n = 0; n < n_q; ++n) {
        for (int i = 0; i < m; ++i) {
            double v = 0.0;
            for (int j = 0; j < d; ++j)
                v += S[(int64_t)i * d + j] * (double)load_elem(q, q_dtype, n * d + j);
            if (v64) v64[n * m + i] = v;
            if (v32) v32[n * m + i] = (float)v;
        }
    }
    return 0;
}

/* [QJL] asymmetric estimator of <q, k> from the query sketch v (length m), the key's
 * sign bits and its stored norm:
 *     s_hat = sqrt(pi/2) / m * ||k|| * sum_i v_i * (2 b_i - 1).
 * For a row g of S with i.i.d. N(0,1) entries, E[sign(<g,k>) <g,q>] =
 * sqrt(2/pi) <k,q> / ||k||, which makes s_hat unbiased.  Evaluated in fp64. */
double ora_qjl_estimate(const double* v, const uint32_t* key_words, double key_norm, int m) {
    double acc = 0.0;
    for (int i = 0; i < m; ++i) {
        int b = (key_words[i / 32] >> (i % 32)) & 1u;
        acc += b ? v[i] : -v[i];
    }
    return sqrt(M_PI / 2.0) / (double)m * key_norm * acc;
}

/* Estimator scores of n_q queries' sketches (fp64, [n_q][m]) against n_keys keys,
 * output fp32 [n_q][n_keys]. */
int ora_qjl_scores(const double* v, int64_t n_q, const uint32_t* words,
                   const uint16_t* norms_f16, int64_t n_keys, int m, float* scores) {
    if (n_q < 0 || n_keys < 0 || m <= 0 || (m % 32) != 0) return 1;
    int nw = m / 32;
    for (int64_t a = 0; a < n_q; ++a)
        for (int64_t t = 0; t < n_keys; ++t)
            scores[a * n_keys + t] = (float)ora_qjl_estimate(
                v + a * m, words + t * nw, ora_half_to_double(norms_f16[t]), m);
    return 0;
}

/* ---------------------------------------------------------------------------------
 * [RES] encode of keys (fp16, [n_keys][d]) as INT4 groups of g plus the 1-bit QJL sketch
 * of the residual.  Per key:
 *   packed, scales, zeros = [INT4] of the key (groups of g);
 *   k_hat_j = fl32(fl32(c_j * s4) + z4), the INT4 reconstruction;
 *   r_j     = fp16(fl32(k_j - k_hat_j)), the residual in the key's own precision;
 *   words, rnorm = [QJL] encode of r (sign bits of S r in fp64; fp16 of the fp64 norm).
 * r_out_f16 ([n_keys][d]) and u_out ([n_keys][m], the fp64 projections of r) are
 * optional.
 * ------------------------------------------------------------------------------- */
int ora_qjlres_encode(const uint16_t* keys_f16, int64_t n_keys, int d, int g, const double* S, int m,
                      uint8_t* packed, float* scales, float* zeros, uint32_t* words,
                      uint16_t* rnorms_f16, uint16_t* r_out_f16, double* u_out) {
    if (n_keys < 0 || d <= 0 || g <= 0 || (d % g) != 0 || (g % 2) != 0 || (d % 2) != 0) return 1;
    if (m <= 0 || (m % 32) != 0) return 1;
    int nw = m / 32, ng = d / g;
    uint16_t* r16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)d);
    if (!r16) return 2;
    for (int64_t n = 0; n < n_keys; ++n) {
        const uint16_t* k = keys_f16 + n * d;
        uint8_t* pk = packed + n * (d / 2);
        float* sc = scales + n * ng;
        float* zr = zeros + n * ng;
        int rc = ora_quantize_int4_group(k, ORA_F16, 1, d, g, pk, sc, zr);
        if (rc) { free(r16); return rc; }
        for (int j = 0; j < d; ++j) {
            float k_hat = int4_value(pk, sc, zr, 0, d, g, j);
            float kj = (float)ora_half_to_double(k[j]);
            float diff = kj - k_hat;
            r16[j] = ora_double_to_half((double)diff);
            if (r_out_f16) r_out_f16[n * d + j] = r16[j];
        }
        rc = ora_qjl_encode(r16, 1, d, S, m, words + n * nw, rnorms_f16 + n, u_out ? u_out + n * m : NULL);
        if (rc) { free(r16); return rc; }
    }
    free(r16);
    return 0;
}

/* [RES] score of a query against key `row` of a residual-format cache:
 *   sum_j q_j k_hat_j (fp64, the INT4 reconstruction) + the [QJL] estimate with the
 *   residual's sign bits and stored norm, from the fp32 stored query sketch vst. */
static double qjlres_score(const float* qf, const uint8_t* packed, const float* s4, const float* z4,
                           int64_t row, int d, int g, const double* vst, const uint32_t* words,
                           double rnorm, int m) {
    double base = 0.0;
    for (int j = 0; j < d; ++j)
        base += (double)qf[j] * (double)int4_value(packed, s4, z4, row, d, g, j);
    return base + ora_qjl_estimate(vst, words + row * (m / 32), rnorm, m);
}

/* ---------------------------------------------------------------------------------
 * One decode step over a compressed cache.
 *   q:        fp16 [B][Hq][D]
 *   keys:     INT8 codes [B][Hkv][T][D] + fp32 scales [B][Hkv][T], or
 *             QJL words [B][Hkv][T][m/32] + fp16 norms [B][Hkv][T] + sketch S (fp64 m x D), or
 *             [RES] INT4 codes [B][Hkv][T][D/2] + scales, zeros [B][Hkv][T][D/k_group] and
 *             the residual's words and fp16 norms (k_words, k_norms_f16) + S
 *   values:   INT8 codes [B][Hkv][T][D] + fp32 scales [B][Hkv][T], or (when v_packed4
 *             is given) [INT4] group-wise codes [B][Hkv][T][D/2] + scales and zeros
 *             [B][Hkv][T][D/v_group], x_hat = fl32(fl32(c * s4) + z4)
 *   [GQA]     query head h reads KV head h / (Hq / Hkv)  (expand along a new group axis
 *             after the KV-head axis, then merge the two axes).
 *   score_t   = INT8: sum_j q_j x_hat_tj (fp32, index order); QJL: the estimator, fp32;
 *               RES: qjlres_score, rounded to fp32.
 *   logit_t   = fl32(sm_scale * score_t), sm_scale = fl32(1/sqrt(D)) when 0 is given.
 *   p_t       = expf(logit_t - max logit) / sum_t expf(...), fp32 in token order.
 *   out_j     = sum_t p_t * x_hat_v_tj, fp32 accumulation in token order.
 * Outputs (each may be NULL): out fp32 [B][Hq][D], scores_out fp32 [B][Hq][T] (raw
 * scores before sm_scale), probs_out fp32 [B][Hq][T].
 * ------------------------------------------------------------------------------- */
int ora_decode_attention(int64_t B, int64_t Hq, int64_t Hkv, int64_t T, int D,
                         const uint16_t* q_f16, int key_format,
                         const int8_t* k_codes, const float* k_scales,
                         const uint32_t* k_words, const uint16_t* k_norms_f16,
                         const double* S, int m,
                         const uint8_t* k_packed4, const float* k_scales4, const float* k_zeros4,
                         int k_group,
                         const int8_t* v_codes, const float* v_scales,
                         const uint8_t* v_packed4, const float* v_scales4, const float* v_zeros4,
                         int v_group, float sm_scale,
                         float* out, float* scores_out, float* probs_out) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || D <= 0 || (Hq % Hkv) != 0) return 1;
    int sketched = key_format == ORA_KEYS_QJL || key_format == ORA_KEYS_QJLRES;
    if (sketched && (m <= 0 || (m % 32) != 0)) return 1;
    if (key_format == ORA_KEYS_QJLRES && (k_group <= 0 || (D % k_group) != 0)) return 1;
    int64_t G = Hq / Hkv;
    int nw = m / 32;
    float sigma = sm_scale != 0.0f ? sm_scale : 1.0f / sqrtf((float)D);
    int fail = 0;
#pragma omp parallel
    {
    /* scratch, one set per thread */
    float* qf = (float*)malloc(sizeof(float) * (size_t)D);
    float* score = (float*)malloc(sizeof(float) * (size_t)T);
    float* e = (float*)malloc(sizeof(float) * (size_t)T);
    double* v64 = (double*)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
    double* vst = (double*)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
    int ok = qf && score && e && v64 && vst;
    if (!ok) {
#pragma omp atomic write
        fail = 2;
    }
    /* one (batch, query head) pair per iteration */
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * Hq; ++bh) {
        if (!ok) continue;
        {
            int64_t b = bh / Hq, h = bh % Hq;
            int64_t kvh = h / G;
            int64_t qo = (b * Hq + h) * D;
            int64_t base = (b * Hkv + kvh) * T;   /* first token row of this KV head */
            for (int j = 0; j < D; ++j) qf[j] = (float)ora_half_to_double(q_f16[qo + j]);
            if (sketched) {
                for (int i = 0; i < m; ++i) {
                    double v = 0.0;
                    for (int j = 0; j < D; ++j) v += S[(int64_t)i * D + j] * (double)qf[j];
                    v64[i] = v;
                    vst[i] = (double)(float)v;     /* the stored fp32 sketch */
                }
            }
            for (int64_t t = 0; t < T; ++t) {
                if (key_format == ORA_KEYS_QJL)
                    score[t] = (float)ora_qjl_estimate(vst, k_words + (base + t) * nw,
                                                       ora_half_to_double(k_norms_f16[base + t]), m);
                else if (key_format == ORA_KEYS_QJLRES)
                    score[t] = (float)qjlres_score(qf, k_packed4, k_scales4, k_zeros4, base + t, D, k_group,
                                                   vst, k_words, ora_half_to_double(k_norms_f16[base + t]), m);
                else
                    score[t] = int8_row_score(qf, k_codes + (base + t) * D, k_scales[base + t], D);
            }
            float mx = -INFINITY;
            for (int64_t t = 0; t < T; ++t) {
                float lg = sigma * score[t];
                if (lg > mx) mx = lg;
            }
            float sum = 0.0f;
            for (int64_t t = 0; t < T; ++t) {
                e[t] = expf(sigma * score[t] - mx);
                sum = sum + e[t];
            }
            for (int64_t t = 0; t < T; ++t) {
                float p = e[t] / sum;
                if (scores_out) scores_out[(b * Hq + h) * T + t] = score[t];
                if (probs_out) probs_out[(b * Hq + h) * T + t] = p;
                e[t] = p;
            }
            if (out) {
                for (int j = 0; j < D; ++j) {
                    float acc = 0.0f;
                    for (int64_t t = 0; t < T; ++t) {
                        float xv = v_packed4
                                       ? int4_value(v_packed4, v_scales4, v_zeros4, base + t, D, v_group, j)
                                       : (float)v_codes[(base + t) * D + j] * v_scales[base + t];
                        float prod = e[t] * xv;
                        acc = acc + prod;
                    }
                    out[qo + j] = acc;
                }
            }
        }
    }
    free(qf); free(score); free(e); free(v64); free(vst);
    }
    return fail;
}
