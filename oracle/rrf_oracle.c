/*
 * rrf_oracle.c -- the oracle for the fused "R-way bf16 sum + residual +
 * RMSNorm + dynamic per-row FP8 (e4m3fn) quantisation" operation.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, single-threaded CPU
 * statement of what the operation computes.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark may build, load or call it.
 * It shares no code, header, table or constant with the CUDA library, and the
 * library never calls it: a missing CUDA extension is an error, not a reason
 * to fall back to this file.
 *
 * Sources (web pages, cited by title and section):
 *  - Modular docs, Mojo function `allreduce_rmsnorm_fp8` (module
 *    nn/allreduce_residual_rmsnorm_fp8), "Args": per-GPU input buffers with
 *    last dim = cols, FP8 output of the input's shape, 1-D gamma of length
 *    cols, epsilon, weight_offset ("additive offset for gamma weights"),
 *    scale_ub ("upper bound for FP8 scale clamping"), per-row scales with last
 *    dim 1; in_dtype bfloat16, out_dtype float8_e4m3fn, scales float32.
 *  - local-inference-lab/b12x PR #283 "PCIeTwoShotBF16", opening description
 *    and "Behavior": the partials are accumulated in fp32 in a fixed rank
 *    order and the result is rounded to bf16 once, so it is deterministic and
 *    lies within one bf16 rounding of the exact sum.
 *  - NVIDIA/TensorRT-LLM PR #19836, "Description": the RESIDUAL_RMS_NORM
 *    epilogue adds a residual before the norm.
 *  - Tenstorrent rmsnorm_2d.py, `_resolve_2d_config` (add_unit_offset adds
 *    1.0 to the weight): weight_offset is added to gamma before it scales.
 *  - Huawei Ascend aclnnAlltoAllQuantMatmul, quant-mode list, mode 7
 *    "per-token dynamic quantization": one scale per row, from the row's data.
 *
 * The pages name the parameters but print no formula.  This file takes the
 * plainest reading, the textbook RMSNorm followed by amax-scaled FP8
 * quantisation.  Per row i, with x_r the R bf16 inputs:
 *   1. acc_j = f32(x_0[i,j]); acc_j = acc_j + f32(x_r[i,j]) for r = 1..R-1,
 *      each an IEEE fp32 add (no fused multiply-add); s_j = RN_bf16(acc_j).
 *   2. with a residual: h_j = RN_bf16(f32(s_j) + f32(res_in[i,j])), written
 *      to res_out; without one: h_j = s_j.
 *   3. ss = sum_j h_j^2 in float64 (each term and, at these sizes, the sum
 *      are exact); ms = f32(ss) / f32(cols); r = 1 / sqrtf(ms + eps), all fp32.
 *   4. y_j = (f32(h_j) * r) * (f32(gamma_j) + weight_offset), fp32.
 *   5. amax = max_j |y_j|; scale = max(min(amax, scale_ub), 1e-12) / 448.
 *   6. q_j = e4m3fn(y_j / scale), round to nearest even, finite values and
 *      infinities beyond 448 saturate to +-448, NaN gives 0x7F.
 *      scales[i] = scale (the dequantisation multiplier: y ~ f32(q) * scale).
 *
 * Build with -ffp-contract=off (no FMA contraction) and without fast-math, so
 * every fp32 operation above is one IEEE-rounded operation.
 *
 * The FP8 GEMM that consumes the per-row scales (oracle_scaled_mm, at the
 * end) follows the Huawei Ascend aclnnAlltoAllQuantMatmul page, the formula
 * of its per-token dynamic quantisation scenario: out = (x1_q @ x2) *
 * x1Scale * x2Scale + bias, one x1Scale per row of x1 and one x2Scale per
 * output column.
 *
 * The same page's mx scenario carries x1Scale of shape (BS, ceil(H/64), 2):
 * one scale per 32 elements of a row.  oracle_sum_rmsnorm_mxfp8_rows gives
 * the norm's output in that form, following the OCP Microscaling Formats
 * (MX) v1.0 specification (conversion to MX, section 6.3): a block of 32
 * elements shares the scale X = 2^(floor(log2(max |V|)) - 8), 8 being the
 * exponent of e4m3's largest normal (448 = 1.75 * 2^8), stored as an E8M0
 * code (the exponent biased by 127); each element is V / X rounded to
 * e4m3fn, nearest even, saturating.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define E4M3_MAX 448.0
#define SCALE_FLOOR 1e-12f

/* ---------------------------------------------------------------- bf16 --- */

/* bf16 is the top 16 bits of an IEEE binary32. */
float oracle_bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static double bf16_magnitude_for_rounding(uint16_t b) {
    /* Rounding behaves as if the exponent range were unbounded and then
     * overflows to infinity, so the encoding 0x7F80 (infinity) stands for
     * 2^128 while the nearest neighbour is chosen. */
    if ((b & 0x7FFF) == 0x7F80) return ldexp(1.0, 128);
    return fabs((double)oracle_bf16_to_float(b));
}

/* Round an fp32 value to the nearest bf16, ties to the even encoding (IEEE
 * round-to-nearest-even).  The candidates are the bf16 value nearer zero
 * (truncation of the low 16 bits) and the next one away from zero. */
uint16_t oracle_bf16_round(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040); /* stays a quiet NaN */
    uint16_t lo = (uint16_t)(u >> 16);
    if ((lo & 0x7FFF) >= 0x7F80) return lo; /* infinity stays infinity */
    uint16_t hi = (uint16_t)(lo + 1);
    double a = fabs((double)f);
    double dlo = a - bf16_magnitude_for_rounding(lo);
    double dhi = bf16_magnitude_for_rounding(hi) - a;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1) ? hi : lo;
}

/* -------------------------------------------------------------- e4m3fn --- */

/* Value of an e4m3fn code: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 holds subnormals m * 2^-9; S.1111.111 is NaN; there
 * is no infinity, so S.1111.110 = 1.75 * 2^8 = 448 is the largest finite. */
double oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 0x7;
    if (e == 0xF && m == 0x7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return s ? -mag : mag;
}

/* Nearest e4m3fn code to v, ties to the even code, saturating: any finite or
 * infinite magnitude above 448 becomes +-448; NaN becomes 0x7F.  The search
 * runs over all 127 non-negative finite codes, which is slow on purpose. */
uint8_t oracle_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a > E4M3_MAX) return (uint8_t)(sign | 0x7E);
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* ---------------------------------------------------------- vectorised --- */

void oracle_bf16_round_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_bf16_round(in[k]);
}

void oracle_e4m3_encode_array(const float* in, uint8_t* out, int64_t n) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_e4m3_encode(in[k]);
}

/* ------------------------------------------------------------ the sum --- */

/* Step 1 for one element: fp32 accumulation in the fixed order 0..R-1,
 * starting from the first input (not from +0, so all -0 inputs give -0),
 * then a single rounding to bf16. */
static uint16_t sum_element(const uint16_t* const* x, int R, int64_t k) {
    float acc = oracle_bf16_to_float(x[0][k]);
    for (int r = 1; r < R; ++r) acc = acc + oracle_bf16_to_float(x[r][k]);
    return oracle_bf16_round(acc);
}

/* The bf16 sum alone: out[i, j] = RN_bf16(sum over r in order of x_r[i, j]).
 * All arrays are row-major [rows, cols] of bf16 bit patterns. */
void oracle_sum(const uint16_t* const* x, int R, int64_t rows, int64_t cols,
                uint16_t* out) {
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j) out[i * cols + j] = sum_element(x, R, i * cols + j);
}

/* ---------------------------------------------------------- fused row --- */

/* Steps 1-6 for the rows [row0, row0 + nrows).  res_in / res_out are both
 * NULL (no residual) or both non-NULL; they may be the same array.  The
 * optional outputs h_out (the bf16 norm input, [rows, cols]) and v_out (the
 * fp32 pre-quantisation value y / scale, [rows, cols]) serve the tests. */
void oracle_sum_rmsnorm_fp8_rows(const uint16_t* const* x, int R, int64_t row0,
                                 int64_t nrows, int64_t cols, const uint16_t* res_in,
                                 uint16_t* res_out, const uint16_t* gamma, float eps,
                                 float weight_offset, float scale_ub, uint8_t* q,
                                 float* scales, uint16_t* h_out, float* v_out) {
    for (int64_t i = row0; i < row0 + nrows; ++i) {
        const int64_t base = i * cols;

        /* steps 1-2: the norm input h, one bf16 per element */
        double ss = 0.0;
        for (int64_t j = 0; j < cols; ++j) {
            uint16_t s = sum_element(x, R, base + j);
            uint16_t h = s;
            if (res_in != NULL) {
                float t = oracle_bf16_to_float(s) + oracle_bf16_to_float(res_in[base + j]);
                h = oracle_bf16_round(t);
                res_out[base + j] = h;
            }
            if (h_out != NULL) h_out[base + j] = h;
            double hd = (double)oracle_bf16_to_float(h);
            ss += hd * hd; /* step 3, float64 */
        }
        const uint16_t* hrow = (h_out != NULL) ? h_out + base
                              : (res_out != NULL) ? res_out + base
                                                  : NULL;

        /* step 3: r = 1 / sqrt(mean(h^2) + eps) in fp32 */
        float ms = (float)ss / (float)cols;
        float r = 1.0f / sqrtf(ms + eps);

        /* steps 4-5: y and its absolute maximum */
        float amax = 0.0f;
        for (int64_t j = 0; j < cols; ++j) {
            float h = hrow ? oracle_bf16_to_float(hrow[j])
                           : oracle_bf16_to_float(sum_element(x, R, base + j));
            float g = oracle_bf16_to_float(gamma[j]) + weight_offset;
            float y = (h * r) * g;
            float ay = fabsf(y);
            if (ay > amax) amax = ay;
        }
        float scale = fmaxf(fminf(amax, scale_ub), SCALE_FLOOR) / 448.0f;
        scales[i] = scale;

        /* step 6: quantise */
        for (int64_t j = 0; j < cols; ++j) {
            float h = hrow ? oracle_bf16_to_float(hrow[j])
                           : oracle_bf16_to_float(sum_element(x, R, base + j));
            float g = oracle_bf16_to_float(gamma[j]) + weight_offset;
            float y = (h * r) * g;
            float v = y / scale;
            if (v_out != NULL) v_out[base + j] = v;
            q[base + j] = oracle_e4m3_encode(v);
        }
    }
}

/* The whole operation over all rows. */
void oracle_sum_rmsnorm_fp8(const uint16_t* const* x, int R, int64_t rows, int64_t cols,
                            const uint16_t* res_in, uint16_t* res_out,
                            const uint16_t* gamma, float eps, float weight_offset,
                            float scale_ub, uint8_t* q, float* scales) {
    oracle_sum_rmsnorm_fp8_rows(x, R, 0, rows, cols, res_in, res_out, gamma, eps,
                                weight_offset, scale_ub, q, scales, NULL, NULL);
}

/* ------------------------------------------------------- the FP8 GEMM --- */

/* Round a float64 value to the nearest bf16 (ties to the even encoding),
 * without passing through fp32 (which would round twice).  bf16 holds 8
 * significant bits; below 2^-126 the spacing stays 2^-133 (subnormals).
 * Magnitudes that round to 2^128 or beyond become infinity. */
uint16_t oracle_bf16_round_double(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e); /* a = f * 2^e, 0.5 <= f < 1 */
    int q_exp = e - 8; /* spacing of the 8-bit significands in [2^(e-1), 2^e) */
    if (q_exp < -133) q_exp = -133;
    double quantum = ldexp(1.0, q_exp);
    double k = floor(a / quantum); /* a / quantum is exact: a power-of-two scaling */
    double lo = k * quantum, hi = (k + 1.0) * quantum;
    double pick;
    if (a - lo < hi - a) pick = lo;
    else if (hi - a < a - lo) pick = hi;
    else pick = (fmod(k, 2.0) == 0.0) ? lo : hi;
    if (pick >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    float f = (float)pick; /* exact: 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* out[m][n] = RN_bf16(S * a_scale[m] * b_scale[n] + bias[n]) with
 * S = sum_k e4m3(a[m][k]) * e4m3(b[n][k]).  a is [M, K] and b is [N, K], both
 * row-major e4m3fn codes; bias (bf16 [N]) may be NULL.  Everything is float64:
 * each product of two e4m3 values is an integer multiple of 2^-18 below
 * 2^18, so for K below 2^17 the sum S is exact; the scaling and the bias add
 * two float64 roundings (relative 2^-53) before the one rounding to bf16.
 * exact (may be NULL) receives that float64 value. */
void oracle_scaled_mm(const uint8_t* a, const float* a_scale, const uint8_t* b,
                      const float* b_scale, const uint16_t* bias, int64_t M, int64_t N,
                      int64_t K, uint16_t* out, double* exact) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double S = 0.0;
            for (int64_t k = 0; k < K; ++k)
                S += oracle_e4m3_decode(a[m * K + k]) * oracle_e4m3_decode(b[n * K + k]);
            double y = S * (double)a_scale[m] * (double)b_scale[n];
            if (bias != NULL) y += (double)oracle_bf16_to_float(bias[n]);
            if (exact != NULL) exact[m * N + n] = y;
            out[m * N + n] = oracle_bf16_round_double(y);
        }
    }
}

/* ------------------------------------------- MX (block-scaled) output --- */

#define MX_BLOCK 32

/* E8M0 code of a block's shared scale from the block's max |V|: the biased
 * exponent of 2^(floor(log2(amax)) - 8), clamped to the codes of finite
 * scales (0..254).  An all-zero block takes code 0 (a reading: the
 * specification leaves the scale of a zero block free). */
uint8_t oracle_mx_scale_code(float amax) {
    if (!(amax > 0.0f)) return 0;
    int e;
    frexp((double)amax, &e); /* amax = f * 2^e with 0.5 <= f < 1: floor(log2(amax)) = e - 1 */
    int c = (e - 1) - 8 + 127;
    if (c < 0) c = 0;
    if (c > 254) c = 254;
    return (uint8_t)c;
}

/* Steps 1-4 of the fused operation (the sum, the residual, r and y = (h *
 * r) * g'), then per block of 32 columns: the E8M0 scale code from the
 * block's max |y| and the codes e4m3fn(y * 2^(127 - code)) (a power-of-two
 * scaling, exact in fp32 here).  scales_mx is [rows][cols / 32]; cols is a
 * multiple of 32.  v_out (may be NULL) receives y * 2^(127 - code). */
void oracle_sum_rmsnorm_mxfp8_rows(const uint16_t* const* x, int R, int64_t row0,
                                   int64_t nrows, int64_t cols, const uint16_t* res_in,
                                   uint16_t* res_out, const uint16_t* gamma, float eps,
                                   float weight_offset, uint8_t* q, uint8_t* scales_mx,
                                   uint16_t* h_out, float* v_out) {
    const int64_t nblocks = cols / MX_BLOCK;
    for (int64_t i = row0; i < row0 + nrows; ++i) {
        const int64_t base = i * cols;
        double ss = 0.0;
        for (int64_t j = 0; j < cols; ++j) {
            uint16_t h = sum_element(x, R, base + j);
            if (res_in != NULL) {
                float t = oracle_bf16_to_float(h) + oracle_bf16_to_float(res_in[base + j]);
                h = oracle_bf16_round(t);
                res_out[base + j] = h;
            }
            h_out[base + j] = h;
            double hd = (double)oracle_bf16_to_float(h);
            ss += hd * hd;
        }
        float ms = (float)ss / (float)cols;
        float r = 1.0f / sqrtf(ms + eps);

        for (int64_t b = 0; b < nblocks; ++b) {
            float y[MX_BLOCK];
            float amax = 0.0f;
            for (int k = 0; k < MX_BLOCK; ++k) {
                const int64_t j = b * MX_BLOCK + k;
                float g = oracle_bf16_to_float(gamma[j]) + weight_offset;
                y[k] = (oracle_bf16_to_float(h_out[base + j]) * r) * g;
                if (fabsf(y[k]) > amax) amax = fabsf(y[k]);
            }
            uint8_t c = oracle_mx_scale_code(amax);
            scales_mx[i * nblocks + b] = c;
            float inv_x = ldexpf(1.0f, 127 - (int)c);
            for (int k = 0; k < MX_BLOCK; ++k) {
                float v = y[k] * inv_x;
                if (v_out != NULL) v_out[base + b * MX_BLOCK + k] = v;
                q[base + b * MX_BLOCK + k] = oracle_e4m3_encode(v);
            }
        }
    }
}

/* ------------------------------------------------------ the MX GEMM --- */

/* Value of an E8M0 code: 2^(code - 127); 0xFF is NaN (OCP MX v1.0). */
double oracle_e8m0_decode(uint8_t c) {
    if (c == 0xFF) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* The mx scenario of the Ascend aclnnAlltoAllQuantMatmul page:
 * out = (x1 * x1Scale) @ (x2 * x2Scale) + bias with one scale per 32 values
 * of K on both sides.  Here a is [M, K] and b is [N, K] e4m3fn codes,
 * sa is [M, K / 32] and sb is [N, K / 32] E8M0 codes (row-major),
 *   out[m][n] = RN_bf16( sum_k (e4m3(a[m][k]) * 2^(sa[m][k/32] - 127))
 *                              * (e4m3(b[n][k]) * 2^(sb[n][k/32] - 127)) + bias[n] )
 * in float64: every term is an exact power-of-two multiple of a product of
 * two e4m3 values, and the sum is exact while the terms' exponents stay
 * within float64's 53 bits (checked by the tests' magnitudes); one rounding to
 * bf16.  exact (may be NULL) receives the float64 value before rounding. */
void oracle_scaled_mm_mx(const uint8_t* a, const uint8_t* sa, const uint8_t* b,
                         const uint8_t* sb, const uint16_t* bias, int64_t M, int64_t N,
                         int64_t K, uint16_t* out, double* exact) {
    const int64_t nb = K / MX_BLOCK;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double S = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double x = oracle_e4m3_decode(a[m * K + k]) * oracle_e8m0_decode(sa[m * nb + k / MX_BLOCK]);
                double y = oracle_e4m3_decode(b[n * K + k]) * oracle_e8m0_decode(sb[n * nb + k / MX_BLOCK]);
                S += x * y;
            }
            if (bias != NULL) S += (double)oracle_bf16_to_float(bias[n]);
            if (exact != NULL) exact[m * N + n] = S;
            out[m * N + n] = oracle_bf16_round_double(S);
        }
    }
}
