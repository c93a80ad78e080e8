/*
 * mq_oracle.c -- plain, slow CPU oracle for the Mix-Quant prefill linear layer
 * (NVFP4 activation quantization + block-scaled FP4 x FP4 GEMM) and for the
 * BF16 decode linear on the same weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg may load or call this library.
 * The product library (libmq, CUDA) never calls it and shares no source,
 * header, table or helper with it.
 *
 * Sources (the pages describing "Mix-Quant: Quantized Prefilling, Precise
 * Decoding for Agentic LLMs", arXiv 2605.20315):
 *   - gist.science technical summary, section 2 "Hybrid Precision Strategy":
 *     prefill uses NVFP4 for weights AND activations; NVFP4 has a local scale
 *     per group of 16 elements plus a tensor-level scale; quantization is plain
 *     round-to-nearest (RTN).  Decode keeps BF16.
 *   - same page, "System-Level Deployment": prefill runs the W4A4 path.
 *   - zingnex.cn forum post, section "动态精度切换": weights are stored in a
 *     quickly convertible form and activations are converted at the phase
 *     boundary.
 * The pages do not give the element / scale types or the tie rule; the
 * standard NVFP4 encoding is used: E2M1 elements, one E4M3 scale per 16
 * contiguous K-elements, one FP32 tensor scale, round-to-nearest-even.
 * Readings of points the pages leave open are marked [reading] below.
 *
 * Every floating-point step is written as an explicit binary32 or binary64
 * operation; build with -ffp-contract=off and without fast-math so that no
 * step is fused or reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 0; /* 0 = OpenMP default */

void mqo_set_threads(int n) { g_threads = n; }

int mqo_threads_used(void) {
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

#ifdef _OPENMP
#define MQO_NT (g_threads > 0 ? g_threads : omp_get_max_threads())
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* E2M1 (4 bits: sign, 2 exponent bits with bias 1, 1 mantissa bit, no
 * Inf/NaN).  Exponent field 0 is subnormal: value = m * 2^-1. */
double mqo_e2m1_decode(int code) {
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag;
    if (e == 0)
        mag = ldexp((double)m, -1);
    else
        mag = ldexp(1.0 + (double)m / 2.0, e - 1);
    return s ? -mag : mag;
}

/* E4M3, the "FN" variant (bias 7, no Inf; S.1111.111 is NaN; max 448).
 * Exponent field 0 is subnormal: value = (m/8) * 2^-6. */
double mqo_e4m3_decode(int byte) {
    int s = (byte >> 7) & 1;
    int e = (byte >> 3) & 15;
    int m = byte & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* BF16 is the upper half of a binary32. */
float mqo_bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even: choose between the two
 * bf16 values that bracket f (truncation and truncation + 1 ulp). */
uint16_t mqo_float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
    uint16_t lo = (uint16_t)(u >> 16);
    uint16_t hi = (uint16_t)(lo + 1);
    double dlo = (double)mqo_bf16_to_float(lo);
    double dhi = (double)mqo_bf16_to_float(hi);
    double d = (double)f;
    double elo = fabs(d - dlo), ehi = fabs(dhi - d);
    if (elo < ehi) return lo;
    if (ehi < elo) return hi;
    return (lo & 1) ? hi : lo;
}

/* Non-negative binary32 -> E4M3 byte, round to nearest with ties to the even
 * code, saturating to the largest finite value 448 (0x7E).  Written as the
 * definition: the nearest of the 127 finite non-negative E4M3 values. */
int mqo_e4m3_encode_satfinite(float v) {
    double x = (double)v;
    if (x >= 448.0) return 0x7E; /* saturate (distances lose meaning far out) */
    int best = 0;
    double best_err = fabs(x - mqo_e4m3_decode(0));
    for (int b = 1; b <= 0x7E; ++b) {
        double err = fabs(x - mqo_e4m3_decode(b));
        if (err < best_err || (err == best_err && (b & 1) == 0 && (best & 1) == 1)) {
            best = b;
            best_err = err;
        }
    }
    return best;
}

/* binary32 -> E2M1 code: the magnitude is the nearest of the 8 finite E2M1
 * magnitudes (ties to the even code, saturating at 6); the sign bit is the
 * sign bit of v, so a negative value that rounds to zero keeps its sign
 * [reading: the pages do not discuss signed zero]. */
int mqo_e2m1_encode_satfinite(float v) {
    double a = fabs((double)v);
    if (a >= 6.0) return (signbit(v) ? 8 : 0) | 7; /* saturate */
    int best = 0;
    double best_err = fabs(a - mqo_e2m1_decode(0));
    for (int c = 1; c <= 7; ++c) {
        double err = fabs(a - mqo_e2m1_decode(c));
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return (signbit(v) ? 8 : 0) | best;
}

/* ------------------------------------------------------------------------ */
/* Tensor-level scale                                                        */
/* ------------------------------------------------------------------------ */

/* amax_t = max |x| over a BF16 matrix [rows, cols] with leading dimension ld
 * (elements).  Max is exact, so the order does not matter. */
float mqo_tensor_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld) {
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(mqo_bf16_to_float(x[r * ld + c]));
            if (a > amax) amax = a;
        }
    return amax;
}

/* Tensor-level encode scale.  The pages only say "a tensor-level scale".
 * [reading] s_enc = 2688 / amax_t with 2688 = 6 * 448 (largest E2M1 magnitude
 * times largest E4M3 value), so that the block holding amax_t gets the block
 * scale 448; the decode factor is 1/s_enc.  An all-zero tensor (or a quotient
 * that is not finite) uses s_enc = 1. */
float mqo_tensor_scale(float amax) {
    float s = 2688.0f / amax;
    if (amax == 0.0f || !isfinite(s)) s = 1.0f;
    return s;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantization (the "groups of 16" local scale + tensor scale, RTN)  */
/* ------------------------------------------------------------------------ */

/* Quantize rows of a BF16 matrix [rows, cols] (cols % 16 == 0).
 *   per 16-block b of row r:
 *     amax_b = max |x|
 *     sb     = E4M3( fp32( fp32(amax_b / 6) * s_enc ) )        (block scale)
 *     f      = dec(sb) == 0 ? 0 : fp32( s_enc / dec(sb) )       [reading:
 *              multiply by the per-block factor rather than divide by the
 *              dequantization scale]
 *     q      = E2M1( fp32(x * f) )
 * codes: [rows, cols/2] bytes, element 2j in bits 3:0, element 2j+1 in bits
 * 7:4.  sf: row-major [rows, cols/16] E4M3 bytes (not swizzled). */
void mqo_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, float s_enc,
                  uint8_t *codes, uint8_t *sf) {
    int64_t nblk = cols / 16;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(MQO_NT)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const uint16_t *xb = x + r * ld + b * 16;
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(mqo_bf16_to_float(xb[i]));
                if (a > amax_b) amax_b = a;
            }
            float sb_f = (amax_b / 6.0f) * s_enc;
            int sbyte = mqo_e4m3_encode_satfinite(sb_f);
            sf[r * nblk + b] = (uint8_t)sbyte;
            float dec = (float)mqo_e4m3_decode(sbyte);
            float f = (dec == 0.0f) ? 0.0f : s_enc / dec;
            for (int i = 0; i < 16; i += 2) {
                float v0 = mqo_bf16_to_float(xb[i]) * f;
                float v1 = mqo_bf16_to_float(xb[i + 1]) * f;
                int c0 = mqo_e2m1_encode_satfinite(v0);
                int c1 = mqo_e2m1_encode_satfinite(v1);
                codes[r * (cols / 2) + b * 8 + i / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
}

/* Dequantize one element back to real units: e2m1 * dec(sb) / s_enc. */
double mqo_dequant(const uint8_t *codes, const uint8_t *sf, int64_t cols, float s_enc,
                   int64_t r, int64_t c) {
    uint8_t byte = codes[r * (cols / 2) + c / 2];
    int code = (c & 1) ? (byte >> 4) : (byte & 15);
    double s = mqo_e4m3_decode(sf[r * (cols / 16) + c / 16]);
    return mqo_e2m1_decode(code) * s / (double)s_enc;
}

/* ------------------------------------------------------------------------ */
/* Scale-factor layout                                                       */
/* ------------------------------------------------------------------------ */

/* [reading] The pages are silent on memory layout.  The block-scaled tensor
 * core consumes scales in 128-row x 4-column tiles of 512 bytes; within a
 * tile, scale (r, c) sits at byte (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4.
 * Tiles are stored with the column-tile index fastest.  Rows are padded to a
 * multiple of 128 and columns to a multiple of 4 with zero bytes. */
int64_t mqo_sf_swizzled_bytes(int64_t rows, int64_t kblocks) {
    int64_t rp = (rows + 127) / 128 * 128;
    int64_t cp = (kblocks + 3) / 4 * 4;
    return rp * cp;
}

int64_t mqo_sf_swizzled_offset(int64_t r, int64_t c, int64_t kblocks) {
    int64_t ctiles = (kblocks + 3) / 4;
    int64_t tile = (r / 128) * ctiles + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
}

void mqo_sf_swizzle(const uint8_t *sf, int64_t rows, int64_t kblocks, uint8_t *out) {
    int64_t rp = (rows + 127) / 128 * 128;
    int64_t cp = (kblocks + 3) / 4 * 4;
    for (int64_t r = 0; r < rp; ++r)
        for (int64_t c = 0; c < cp; ++c) {
            uint8_t v = (r < rows && c < kblocks) ? sf[r * kblocks + c] : 0;
            out[mqo_sf_swizzled_offset(r, c, kblocks)] = v;
        }
}

void mqo_sf_unswizzle(const uint8_t *swz, int64_t rows, int64_t kblocks, uint8_t *sf) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < kblocks; ++c)
            sf[r * kblocks + c] = swz[mqo_sf_swizzled_offset(r, c, kblocks)];
}

/* ------------------------------------------------------------------------ */
/* Block-scaled GEMM  Y = X * W^T  on NVFP4 operands                         */
/* ------------------------------------------------------------------------ */

/* 2 * e2m1 is an integer in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}; 2^9 * E4M3
 * is an integer in [0, 229376] (E4M3 values are multiples of 2^-9).  So every
 * dequantized product is an integer times 2^-20 and the sum over K is exact
 * in int64 (max term ~7.6e12; K = 28672 stays below 2^58). */
static int64_t mqo_e2m1_times2(int code) { return (int64_t)(2.0 * mqo_e2m1_decode(code)); }
static int64_t mqo_e4m3_times512(int byte) { return (int64_t)ldexp(mqo_e4m3_decode(byte), 9); }

/* int64 value times 2^-20 as a double, splitting so both parts convert
 * exactly; one rounding in the final add. */
static double mqo_scaled_i64(int64_t v) {
    int64_t hi = v >> 20;         /* floor */
    int64_t lo = v - hi * (1 << 20); /* in [0, 2^20) */
    return (double)hi + ldexp((double)lo, -20);
}

/* For each sampled row index rows_idx[i] of A and each n in [0, N):
 *   S = sum_k e2m1(qa) dec(sa) e2m1(qb) dec(sb)   (exact)
 *   y[i, n] = alpha * S,  alpha = 1 / (s_enc_a * s_enc_b)   (binary64)
 *   p[i, n] = alpha * sum_k |product|  (for the error bound)
 * Operands use row-major (unswizzled) scale matrices. */
void mqo_gemm_nvfp4(const uint8_t *a_codes, const uint8_t *a_sf, float a_s_enc,
                    const int64_t *rows_idx, int64_t n_rows,
                    const uint8_t *b_codes, const uint8_t *b_sf, float b_s_enc,
                    int64_t N, int64_t K, double *y, double *p) {
    double alpha = 1.0 / ((double)a_s_enc * (double)b_s_enc);
    int64_t kb = K / 16;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(MQO_NT)
#endif
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t m = rows_idx[i];
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0, asum = 0;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t ab = a_codes[m * (K / 2) + k / 2];
                uint8_t bb = b_codes[n * (K / 2) + k / 2];
                int ca = (k & 1) ? (ab >> 4) : (ab & 15);
                int cb = (k & 1) ? (bb >> 4) : (bb & 15);
                int64_t t = mqo_e2m1_times2(ca) * mqo_e4m3_times512(a_sf[m * kb + k / 16]) *
                            mqo_e2m1_times2(cb) * mqo_e4m3_times512(b_sf[n * kb + k / 16]);
                sum += t;
                asum += (t < 0) ? -t : t;
            }
            y[i * N + n] = alpha * mqo_scaled_i64(sum);
            p[i * N + n] = alpha * mqo_scaled_i64(asum);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* BF16 decode linear (gist.science §2: decoding keeps BF16)                 */
/* ------------------------------------------------------------------------ */

/* y[m, n] = sum_k x[m, k] * w[n, k] in binary64 (each product of two BF16
 * values is exact in binary64), p[m, n] = sum_k |x w|. */
void mqo_decode_linear(const uint16_t *x, int64_t M, const uint16_t *w, int64_t N, int64_t K,
                       double *y, double *p) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(MQO_NT)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double s = 0.0, a = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double t = (double)mqo_bf16_to_float(x[m * K + k]) *
                           (double)mqo_bf16_to_float(w[n * K + k]);
                s += t;
                a += fabs(t);
            }
            y[m * N + n] = s;
            p[m * N + n] = a;
        }
}

/* ------------------------------------------------------------------------ */
/* SwiGLU between the gate/up and down projections                          */
/* ------------------------------------------------------------------------ */

/* h = bf16( (g / (1 + exp(-g))) * u ) evaluated in binary32 from the BF16
 * values g and u, with the C library's expf. */
void mqo_swiglu(const uint16_t *g, const uint16_t *u, int64_t n, uint16_t *h) {
    for (int64_t i = 0; i < n; ++i) {
        float gf = mqo_bf16_to_float(g[i]);
        float uf = mqo_bf16_to_float(u[i]);
        float den = 1.0f + expf(-gf);
        float silu = gf / den;
        float hv = silu * uf;
        h[i] = mqo_float_to_bf16_rne(hv);
    }
}

/* ------------------------------------------------------------------------ */
/* RMSNorm in front of a prefill linear                                     */
/* ------------------------------------------------------------------------ */

/* Round a binary64 value to the nearest BF16 (ties to even), directly --
 * not through binary32, so there is one rounding. */
uint16_t mqo_double_to_bf16_rne(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return 0x7FC0u;
    const int neg = v < 0.0;
    double a = neg ? -v : v;
    if (isinf(a)) return (uint16_t)(neg ? 0xFF80u : 0x7F80u);
    int e;
    (void)frexp(a, &e);              /* a = m 2^e, 0.5 <= m < 1 */
    int ulp_exp = e - 8;             /* 8 significant bits */
    if (ulp_exp < -133) ulp_exp = -133; /* BF16 subnormal spacing 2^-133 */
    double q = rint(ldexp(a, -ulp_exp)); /* round half to even */
    double r = ldexp(q, ulp_exp);
    if (r > 3.38953138925153547590470800371487866880e+38) return (uint16_t)(neg ? 0xFF80u : 0x7F80u);
    uint16_t b = mqo_float_to_bf16_rne((float)r);  /* exact: r has <= 8 significant bits */
    return (uint16_t)(neg ? (b | 0x8000u) : b);
}

/* [reading] The pages do not define the normalisation that produces the
 * prefill linear's input (the step before the QKV and gate/up projections);
 * the Llama-family RMSNorm is used, evaluated in binary64 from the BF16 row x
 * and BF16 gain gamma:
 *   r   = 1 / sqrt( sum_k x_k^2 / K + eps )
 *   t_k = bf16_RNE(x_k * r)          (the normalised row in the input type)
 *   y_k = bf16_RNE(gamma_k * t_k)    (the learned per-channel gain)        */
void mqo_rmsnorm(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, const uint16_t *gamma,
                 double eps, uint16_t *y) {
#pragma omp parallel for schedule(static) num_threads(MQO_NT)
    for (int64_t m = 0; m < rows; ++m) {
        const uint16_t *xr = x + m * ld;
        double ss = 0.0;
        for (int64_t k = 0; k < cols; ++k) {
            double v = (double)mqo_bf16_to_float(xr[k]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / (double)cols + eps);
        for (int64_t k = 0; k < cols; ++k) {
            double t = (double)mqo_bf16_to_float(mqo_double_to_bf16_rne((double)mqo_bf16_to_float(xr[k]) * r));
            double gk = (double)mqo_bf16_to_float(gamma[k]);
            y[m * cols + k] = mqo_double_to_bf16_rne(gk * t);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Attention of the prefill layer and of the decode step                   */
/* ------------------------------------------------------------------------ */

/* [reading] The pages name the KV cache that prefill builds and decode
 * consumes (zingnex.cn forum thread, section "动态精度切换"; gist.science
 * technical summary, section 2 "System-Level Deployment") but do not define
 * the attention itself.  The plain causal softmax attention of the Llama
 * family's layer is used, with grouped KV heads and no positional rotation:
 *
 *   o[i, h, :] = sum_{j <= pos0 + i} w_j v[j, g, :] / sum_j w_j,
 *   w_j = exp(s_j - max_j s_j),  s_j = scale * sum_d q[i, h, d] k[j, g, d],
 *   g = h / (H / Hkv)   (query heads h share KV head g in groups of H/Hkv),
 *
 * evaluated in binary64 from the BF16 inputs (each product q k is exact in
 * binary64).  Query i sits at absolute position pos0 + i; keys 0..pos0+i
 * are visible to it.  q[i, h, d] is at q[i * q_tok + h * D + d], k[j, g, d]
 * at k[j * k_tok + g * k_head + d], v likewise.  For the requested query
 * rows, out[r][h][d] = o and a[r][h][d] = sum_j w_j |v[j, g, d]| / sum_j w_j
 * (the weighted magnitude that bounds rounding errors of a GPU evaluation). */
void mqo_attention(const uint16_t *q, int64_t q_tok, const uint16_t *k, int64_t k_tok,
                   int64_t k_head, const uint16_t *v, int64_t v_tok, int64_t v_head,
                   int64_t pos0, int64_t H, int64_t Hkv, int64_t D, double scale,
                   const int64_t *rows, int64_t n_rows, double *out, double *a) {
    const int64_t group = H / Hkv;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic) num_threads(MQO_NT)
#endif
    for (int64_t t = 0; t < n_rows * H; ++t) {
        const int64_t r = t / H, h = t % H, i = rows[r], g = h / group;
        const int64_t n_keys = pos0 + i + 1;
        double *s = (double *)malloc(sizeof(double) * (size_t)n_keys);
        double smax = -INFINITY;
        for (int64_t j = 0; j < n_keys; ++j) {
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d)
                acc += (double)mqo_bf16_to_float(q[i * q_tok + h * D + d]) *
                       (double)mqo_bf16_to_float(k[j * k_tok + g * k_head + d]);
            s[j] = scale * acc;
            if (s[j] > smax) smax = s[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j < n_keys; ++j) {
            s[j] = exp(s[j] - smax);
            z += s[j];
        }
        for (int64_t d = 0; d < D; ++d) {
            double o = 0.0, m = 0.0;
            for (int64_t j = 0; j < n_keys; ++j) {
                const double vv = (double)mqo_bf16_to_float(v[j * v_tok + g * v_head + d]);
                o += s[j] * vv;
                m += s[j] * fabs(vv);
            }
            out[(r * H + h) * D + d] = o / z;
            a[(r * H + h) * D + d] = m / z;
        }
        free(s);
    }
}
