/*
 * NVFP4 scale-calibration ORACLE — plain, slow, scalar CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library and its
 * Python binding) may include, link, load or call this file.  Only the test
 * suite, the smoke check of the package entry point and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA path: every table below is written out here from the format
 * definitions, independently.
 *
 * Arithmetic: fp64 throughout (bf16 inputs are exact in double), except where
 * the method itself fixes an fp32 quantity (the tensor scale s_g, the
 * effective block scale s_eff and the dequantised value before its bf16
 * rounding); those are formed with single IEEE float operations.
 *
 * Sources (cited by page title and section):
 *   [QAD]   "為什么NVFP4推理精度會掉以及QAD到底在修什么" (czchanglian.com),
 *           sections 2.1, 2.3, 3.2, 4.2.
 *   [BT]    Baseten engineering blog, "What makes high-quality NVFP4"
 *           (Chinese copy on attain.fans), sections "Why do we need scales?",
 *           "Block scaling: one scale per 16 values", "Why blocks?",
 *           "Calibration".
 *   [LH]    "4 比特量化到底让模型笨了多少？" (2kiu.com), a write-up of NVIDIA
 *           Model Optimizer's "Improving NVFP4 Accuracy with Local-Hessian
 *           Weight Scales"; sections "The NVFP4 structure" and "A different
 *           objective: output error as the ruler", "Trying it" (Local-Hessian
 *           combined with GPTQ).
 *   [GPTQ]  Frantar, Ashkboos, Hoefler, Alistarh, "GPTQ: Accurate
 *           Post-Training Quantization for Generative Pre-trained
 *           Transformers" (the paper [LH] links): dampening, the Cholesky
 *           reformulation and the column-by-column rounding loop.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): the tensor scale s_g = fl32(amax / (6*448)) (1 when amax = 0);
 * round-to-nearest-even and saturation for both E2M1 and E4M3; the sign of
 * a value that rounds to zero is kept (code 0x8 for negative inputs); ties
 * in a scale search keep the smallest code; element 2j of a row goes into the
 * low nibble of byte j; dequantisation rounds v*s_eff to fp32 and then to
 * bf16, both to nearest even.
 *
 * Parity pins: every exported function is pinned by a test that does not go
 * through this file's arithmetic (brute-force enumeration with exact
 * rationals, the worked example of [BT], the trace identity of [LH], the
 * H = I and C = 16 special cases, library Gram products on tiny inputs).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_SHAPE 2
#define ORACLE_ERR_NONFINITE 4

/* ---------------------------------------------------------------- formats */

/* E2M1 magnitudes by 3-bit magnitude index k = code & 7 ([BT] "Why do we
 * need scales?" lists the 16 representable values; [LH] "The NVFP4
 * structure" gives the 1 sign / 2 exponent / 1 mantissa split). */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int code)
{
    double m = E2M1_MAGNITUDE[code & 7];
    return (code & 8) ? -m : m;
}

/* E4M3 (the FN variant: no infinities, 0x7F is NaN): 1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 is subnormal, m * 2^-9.
 * [LH] "The NVFP4 structure": each block carries one FP8 scale.  126 of the
 * codes (0x01..0x7E) are positive, finite and non-zero, which is the
 * candidate count of the MSE search in [LH]. */
double oracle_e4m3_value(int code)
{
    int e = (code >> 3) & 0xF;
    int m = code & 7;
    double v;
    if ((code & 0x7F) == 0x7F)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return (code & 0x80) ? -v : v;
}

double oracle_bf16_to_double(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* fp32 -> bf16, round to nearest even (finite inputs). */
uint16_t oracle_float_to_bf16(float f)
{
    uint32_t bits;
    memcpy(&bits, &f, 4);
    if ((bits & 0x7F800000u) == 0x7F800000u) /* inf / nan: truncate, keep nan quiet */
        return (uint16_t)((bits >> 16) | ((bits & 0xFFFF) ? 0x40 : 0));
    uint32_t lsb = (bits >> 16) & 1u;
    bits += 0x7FFFu + lsb;
    return (uint16_t)(bits >> 16);
}

/* The same rounding over an array (n values). */
void oracle_floats_to_bf16(const float *f, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_float_to_bf16(f[i]);
}

/* Effective block scale: the FP8 block scale times the FP32 tensor scale,
 * formed as one fp32 multiply ([BT] "Why do we need scales?": NVFP4 has a
 * tensor-level FP32 scale on top of the block scale). */
float oracle_effective_scale(float s_g, int code)
{
    float e = (float)oracle_e4m3_value(code); /* exact: <= 4 significant bits */
    return s_g * e;
}

/* --------------------------------------------------------- E2M1 rounding */

/* Round x / s onto the E2M1 grid: nearest magnitude, ties to the even
 * magnitude index (round-to-nearest-even on the 1-bit mantissa), saturating
 * at 6; s = 0 gives magnitude 0.  The decision compares |x| with each
 * midpoint times s; both products are exact in double (the midpoints have at
 * most 3 significant bits and s has 24), so the exact quotient is rounded,
 * not an fp32 approximation of it.  [QAD] section 2.1: a value between two
 * representable values goes to the nearer one.  [BT] "Why blocks?": with
 * scale 14, everything below 3.5 becomes 0. */
int oracle_e2m1_encode(double x, double s)
{
    int sign = signbit(x) ? 8 : 0;
    double a = fabs(x);
    int k = 0;
    if (s > 0.0) {
        for (int i = 0; i < 7; i++) {
            double mid = 0.5 * (E2M1_MAGNITUDE[i] + E2M1_MAGNITUDE[i + 1]);
            double thr = mid * s;
            /* between index i and i+1 a tie goes to the even index */
            int up = (i % 2 == 0) ? (a > thr) : (a >= thr);
            if (up)
                k = i + 1;
        }
    }
    return sign | k;
}

/* ------------------------------------------------------- E4M3 rounding */

/* Round the exact quotient num/den (num >= 0, den > 0) to E4M3 with
 * round-to-nearest-even and saturation to the largest finite value 448
 * (code 0x7E).  Ties between codes c and c+1 go to the even code.  The
 * caller guarantees that midpoint*den is exact in double (midpoints have at
 * most 5 significant bits). */
int oracle_e4m3_round_quotient(double num, double den)
{
    int code = 0;
    for (int c = 0; c < 126; c++) {
        double mid = 0.5 * (oracle_e4m3_value(c) + oracle_e4m3_value(c + 1));
        double thr = mid * den;
        int up = (c % 2 == 0) ? (num > thr) : (num >= thr);
        if (up)
            code = c + 1;
    }
    return code;
}

/* --------------------------------------------------------- global scale */

/* Tensor amax -> FP32 tensor scale s_g = fl32(amax / 2688), 2688 = 6 * 448,
 * so that the largest E4M3 block scale (448) maps the tensor's largest
 * value onto the largest E2M1 magnitude (6).  amax = 0 gives s_g = 1.
 * [BT] "Why do we need scales?" (the FP32 tensor scale exists; its formula
 * is this reading).  Non-finite input is an error. */
int oracle_global_scale(const uint16_t *x, int64_t n, float *s_g)
{
    double amax = 0.0;
    for (int64_t i = 0; i < n; i++) {
        double v = oracle_bf16_to_double(x[i]);
        if (!isfinite(v))
            return ORACLE_ERR_NONFINITE;
        if (fabs(v) > amax)
            amax = fabs(v);
    }
    if (amax == 0.0) {
        *s_g = 1.0f;
    } else {
        float a = (float)amax;        /* exact: a bf16 value */
        *s_g = a / 2688.0f;           /* one IEEE fp32 division */
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------ max rule */

/* Max scaling: block scale = block amax / 6 relative to s_g, rounded to
 * E4M3 (RNE, saturating at 448, which is the clamp to the FP8 maximum of
 * [QAD] section 4.2).  An all-zero block gets code 0.  [QAD] section 2.3
 * (step M/6); [BT] "Why blocks?" (84 / 6 = 14) and "Calibration"
 * (activations use the block max); [LH] "The NVFP4 structure" (max scaling
 * is the default). */
int oracle_max_rule_code(const uint16_t *blk, float s_g)
{
    double amax = 0.0;
    for (int i = 0; i < 16; i++) {
        double v = fabs(oracle_bf16_to_double(blk[i]));
        if (v > amax)
            amax = v;
    }
    if (amax == 0.0)
        return 0;
    return oracle_e4m3_round_quotient(amax, 6.0 * (double)s_g);
}

int oracle_scale_search_max(const uint16_t *w, int64_t R, int64_t C, float s_g,
                            uint8_t *codes)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < nb; b++)
            codes[r * nb + b] = (uint8_t)oracle_max_rule_code(w + r * C + b * 16, s_g);
    return ORACLE_OK;
}

/* ------------------------------------------------- objectives and searches */

/* Quantisation error of one block for candidate code c:
 * delta_i = w_i - v(q_i) * s_eff(c), with q_i the E2M1 code of w_i / s_eff. */
static void block_delta(const uint16_t *blk, float s_g, int c, double delta[16])
{
    double s = (double)oracle_effective_scale(s_g, c);
    for (int i = 0; i < 16; i++) {
        double w = oracle_bf16_to_double(blk[i]);
        int q = oracle_e2m1_encode(w, s);
        delta[i] = w - oracle_e2m1_value(q) * s;
    }
}

/* MSE objective: sum of squared weight errors ([LH] "The NVFP4 structure":
 * the MSE method tries all 126 positive non-zero FP8 scales and keeps the
 * one with the smallest weight error). */
double oracle_block_mse(const uint16_t *blk, float s_g, int c)
{
    double d[16], e = 0.0;
    block_delta(blk, s_g, c, d);
    for (int i = 0; i < 16; i++)
        e += d[i] * d[i];
    return e;
}

/* Local-Hessian objective E = delta H_b delta^T with the 16x16 diagonal block
 * H_b of the calibration Gram matrix ([LH] "A different objective":
 * E(s) = ||delta X||^2 = tr(delta X X^T delta^T), block-diagonal
 * approximation, exhaustive over the 126 candidates per block). */
double oracle_block_lh(const uint16_t *blk, float s_g, int c, const double *Hb)
{
    double d[16], e = 0.0;
    block_delta(blk, s_g, c, d);
    for (int j = 0; j < 16; j++)
        for (int k = 0; k < 16; k++)
            e += d[j] * Hb[j * 16 + k] * d[k];
    return e;
}

/* Exhaustive search over codes 1..126; the first (smallest) code reaching
 * the minimum wins.  Hb == NULL selects the MSE objective.  *second (if not
 * NULL) receives the smallest objective among the other 125 codes, which
 * tells a test whether the block is a near tie. */
static int search_block(const uint16_t *blk, float s_g, const double *Hb, double *best,
                        double *second)
{
    int best_c = 1;
    double best_e = INFINITY, second_e = INFINITY;
    for (int c = 1; c <= 126; c++) {
        double e = Hb ? oracle_block_lh(blk, s_g, c, Hb) : oracle_block_mse(blk, s_g, c);
        if (e < best_e) {
            second_e = best_e;
            best_e = e;
            best_c = c;
        } else if (e < second_e) {
            second_e = e;
        }
    }
    if (best)
        *best = best_e;
    if (second)
        *second = second_e;
    return best_c;
}

/* Objectives of all 126 candidates of one block (index c-1), for tie
 * analysis in the tests. */
void oracle_block_objectives(const uint16_t *blk, float s_g, const double *Hb, double *out126)
{
    for (int c = 1; c <= 126; c++)
        out126[c - 1] = Hb ? oracle_block_lh(blk, s_g, c, Hb) : oracle_block_mse(blk, s_g, c);
}

/* second_obj (nullable): the runner-up objective of every block. */
int oracle_scale_search_mse(const uint16_t *w, int64_t R, int64_t C, float s_g,
                            uint8_t *codes, double *best_obj, double *second_obj)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < nb; b++) {
            double e, e2;
            codes[r * nb + b] = (uint8_t)search_block(w + r * C + b * 16, s_g, NULL, &e, &e2);
            if (best_obj)
                best_obj[r * nb + b] = e;
            if (second_obj)
                second_obj[r * nb + b] = e2;
        }
    return ORACLE_OK;
}

/* H: [C/16][16][16] (row-major 16x16 per column block), shared by all rows.
 * second_obj (nullable): the runner-up objective of every block. */
int oracle_scale_search_lh(const uint16_t *w, int64_t R, int64_t C, float s_g,
                           const double *H, uint8_t *codes, double *best_obj,
                           double *second_obj)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < nb; b++) {
            double e, e2;
            codes[r * nb + b] =
                (uint8_t)search_block(w + r * C + b * 16, s_g, H + b * 256, &e, &e2);
            if (best_obj)
                best_obj[r * nb + b] = e;
            if (second_obj)
                second_obj[r * nb + b] = e2;
        }
    return ORACLE_OK;
}

/* Same search restricted to a list of (row, column-block) pairs, for parity
 * on samples of large layers. */
int oracle_scale_search_sampled(const uint16_t *w, int64_t C, float s_g, const double *H,
                                const int64_t *rows, const int64_t *blocks, int64_t n,
                                uint8_t *codes, double *best_obj)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; i++) {
        double e;
        const double *Hb = H ? H + blocks[i] * 256 : NULL;
        codes[i] = (uint8_t)search_block(w + rows[i] * C + blocks[i] * 16, s_g, Hb, &e, NULL);
        if (best_obj)
            best_obj[i] = e;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------- Four Over Six */

/* Four Over Six ([LH] "The NVFP4 structure": it chooses one of two
 * candidate scales).  The pages do not name the two; the reading here: the
 * max-rule scale, which puts the block amax on E2M1's largest magnitude 6,
 * and the scale that puts it on 4, E4M3(amax / (4 s_g)) -- whichever gives
 * the smaller block MSE, the smaller code on a tie.  An all-zero block gets
 * code 0. */
int oracle_four_over_six_code(const uint16_t *blk, float s_g)
{
    double amax = 0.0;
    for (int i = 0; i < 16; i++) {
        double v = fabs(oracle_bf16_to_double(blk[i]));
        if (v > amax)
            amax = v;
    }
    if (amax == 0.0)
        return 0;
    int c6 = oracle_e4m3_round_quotient(amax, 6.0 * (double)s_g);
    int c4 = oracle_e4m3_round_quotient(amax, 4.0 * (double)s_g);
    int lo = c4 < c6 ? c4 : c6, hi = c4 < c6 ? c6 : c4;
    double e_lo = oracle_block_mse(blk, s_g, lo), e_hi = oracle_block_mse(blk, s_g, hi);
    return e_hi < e_lo ? hi : lo;
}

int oracle_scale_search_four_over_six(const uint16_t *w, int64_t R, int64_t C, float s_g,
                                      uint8_t *codes)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < nb; b++)
            codes[r * nb + b] = (uint8_t)oracle_four_over_six_code(w + r * C + b * 16, s_g);
    return ORACLE_OK;
}

/* ------------------------------------------------------ W4A4 GEMM */

/* The matrix product both NVFP4 operands stand for: with A [M, K] and
 * B [N, K] (row-major, K contiguous) given as packed E2M1 codes, one E4M3
 * code per 16 consecutive values and an FP32 tensor scale each,
 *   Y[m][n] = s_ga s_gb sum_k (v(a_mk) e4m3(ca_m,k/16)) (v(b_nk) e4m3(cb_n,k/16))
 * in fp64 (every product is exact; the sum runs over k in order), and
 * absY[m][n] = the same sum of the terms' magnitudes (for tolerances).
 * [W4A4] (weights and activations both NVFP4); [BT] "Block scaling" (a value
 * is its E2M1 code times its block scale times the tensor scale). */
static double nvfp4_value(const uint8_t *packed, const uint8_t *codes, int64_t row, int64_t K,
                          int64_t k)
{
    uint8_t byte = packed[row * (K / 2) + k / 2];
    int q = (k & 1) ? (byte >> 4) : (byte & 15);
    return oracle_e2m1_value(q) * oracle_e4m3_value(codes[row * (K / 16) + k / 16]);
}

int oracle_gemm_nvfp4(const uint8_t *a_packed, const uint8_t *a_codes, float a_sg,
                      const uint8_t *b_packed, const uint8_t *b_codes, float b_sg, int64_t M,
                      int64_t N, int64_t K, double *Y, double *absY)
{
    if (K % 16)
        return ORACLE_ERR_SHAPE;
    double g = (double)a_sg * (double)b_sg;
#pragma omp parallel for collapse(2) schedule(dynamic, 64)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double t = nvfp4_value(a_packed, a_codes, m, K, k) *
                           nvfp4_value(b_packed, b_codes, n, K, k);
                acc += t;
                aacc += fabs(t);
            }
            Y[m * N + n] = acc * g;
            if (absY)
                absY[m * N + n] = aacc * fabs(g);
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------- Gram */

/* Block-diagonal Gram accumulation: for every column block j,
 * H[j] += sum_t x[t, 16j:16j+16]^T x[t, 16j:16j+16], in fp64.  x is
 * tokens-by-channels ([LH] writes Y = W X with X channels-by-tokens; this is
 * the same product with X transposed).  [LH] "A different objective": only
 * the 16x16 diagonal blocks of X X^T are kept. */
int oracle_gram_accumulate(const uint16_t *x, int64_t n_tok, int64_t C, double *H)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nb; j++) {
        double *Hj = H + j * 256;
        for (int64_t t = 0; t < n_tok; t++) {
            const uint16_t *row = x + t * C + j * 16;
            double v[16];
            for (int a = 0; a < 16; a++)
                v[a] = oracle_bf16_to_double(row[a]);
            for (int a = 0; a < 16; a++)
                for (int b = 0; b < 16; b++)
                    Hj[a * 16 + b] += v[a] * v[b];
        }
    }
    return ORACLE_OK;
}

/* Grouped form (experts): tokens offsets[g]..offsets[g+1] accumulate into
 * H[g]. */
int oracle_gram_accumulate_grouped(const uint16_t *x, const int64_t *offsets, int64_t G,
                                   int64_t C, double *H)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    for (int64_t g = 0; g < G; g++) {
        int64_t n = offsets[g + 1] - offsets[g];
        int st = oracle_gram_accumulate(x + offsets[g] * C, n, C, H + g * (C / 16) * 256);
        if (st)
            return st;
    }
    return ORACLE_OK;
}

/* ----------------------------------------------------- pack / dequant */

/* E2M1 codes of a row-major [R, C] tensor given block codes, two codes per
 * byte: element 2j in the low nibble of byte j, element 2j+1 in the high
 * nibble ([BT] "Where quantisation helps": FP4 takes half a byte per value;
 * the nibble order is this reading). */
int oracle_quantize_pack(const uint16_t *w, int64_t R, int64_t C, float s_g,
                         const uint8_t *codes, uint8_t *packed)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t i = 0; i < C; i += 2) {
            double s = (double)oracle_effective_scale(s_g, codes[r * nb + i / 16]);
            int q0 = oracle_e2m1_encode(oracle_bf16_to_double(w[r * C + i]), s);
            int q1 = oracle_e2m1_encode(oracle_bf16_to_double(w[r * C + i + 1]), s);
            packed[r * (C / 2) + i / 2] = (uint8_t)(q0 | (q1 << 4));
        }
    return ORACLE_OK;
}

/* y = bf16_rn(fl32(v(q) * s_eff)) ([QAD] section 3.2: the dequantised value
 * is the E2M1 value times the scale). */
int oracle_dequantize(const uint8_t *packed, const uint8_t *codes, float s_g, int64_t R,
                      int64_t C, uint16_t *out)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t i = 0; i < C; i++) {
            uint8_t byte = packed[r * (C / 2) + i / 2];
            int q = (i & 1) ? (byte >> 4) : (byte & 0xF);
            float s = oracle_effective_scale(s_g, codes[r * nb + i / 16]);
            float y = (float)oracle_e2m1_value(q) * s; /* one fp32 multiply */
            out[r * C + i] = oracle_float_to_bf16(y);
        }
    return ORACLE_OK;
}

/* Dynamic activation fake-quant (W4A4): tensor scale from the whole
 * activation, then per 16 consecutive channels of each token the max rule,
 * E2M1 encode and dequantise ([BT] "Calibration": activation blocks of 16
 * use their absolute maximum; [QAD] section 3.2: reshape into blocks of 16,
 * scale by the block max over 6, quantise, dequantise).  packed and codes
 * may be NULL. */
/* Fake-quant at a given tensor scale (a static, calibrated one): per block
 * the max rule, E2M1 encode and dequantise; values beyond 6 * 448 * s_g
 * saturate.  [BT] "Calibration" (block scales from the block maximum). */
int oracle_fake_quant_static(const uint16_t *x, int64_t rows, int64_t C, float s_g,
                             uint16_t *out, uint8_t *packed, uint8_t *codes)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < nb; b++) {
            const uint16_t *blk = x + r * C + b * 16;
            int c = oracle_max_rule_code(blk, s_g);
            float s = oracle_effective_scale(s_g, c);
            if (codes)
                codes[r * nb + b] = (uint8_t)c;
            for (int i = 0; i < 16; i++) {
                int q = oracle_e2m1_encode(oracle_bf16_to_double(blk[i]), (double)s);
                float y = (float)oracle_e2m1_value(q) * s;
                out[r * C + b * 16 + i] = oracle_float_to_bf16(y);
                if (packed) {
                    int64_t idx = r * (C / 2) + (b * 16 + i) / 2;
                    if (i & 1)
                        packed[idx] = (uint8_t)(packed[idx] | (q << 4));
                    else
                        packed[idx] = (uint8_t)q;
                }
            }
        }
    return ORACLE_OK;
}

int oracle_fake_quant(const uint16_t *x, int64_t rows, int64_t C, uint16_t *out,
                      uint8_t *packed, uint8_t *codes, float *s_g_out)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    float s_g;
    int st = oracle_global_scale(x, rows * C, &s_g);
    if (st)
        return st;
    *s_g_out = s_g;
    return oracle_fake_quant_static(x, rows, C, s_g, out, packed, codes);
}

/* ------------------------------------------- activation-range calibration */

/* [BT] "Calibration": the clipping range of an activation tensor comes from
 * calibration data -- the maximum avoids clipping, but percentile-,
 * histogram- and error-based ranges clip a few outliers so that the typical
 * values are represented more finely.  Reading: the range sets the static
 * tensor scale s_g = fl32(clip / 2688) of fake_quant_static (block scales
 * still follow each block's maximum).
 *
 * Histogram of |x| over the 32768 bf16 magnitude patterns (exact counts,
 * accumulated: call once per calibration chunk). */
void oracle_abs_histogram(const uint16_t *x, int64_t n, uint64_t *hist)
{
    for (int64_t i = 0; i < n; i++)
        hist[x[i] & 0x7FFF]++;
}

/* The p-quantile of |x| (0 < p <= 1): the smallest bf16 magnitude m with at
 * least ceil(p * N) of the N counted values at or below it.  Non-finite
 * magnitudes are counted but a quantile that lands on one is an error. */
int oracle_quantile_magnitude(const uint64_t *hist, double p, double *m_out)
{
    uint64_t n = 0;
    for (int k = 0; k < 32768; k++)
        n += hist[k];
    if (n == 0 || !(p > 0.0) || p > 1.0)
        return ORACLE_ERR_SHAPE;
    uint64_t need = (uint64_t)ceil(p * (double)n);
    if (need < 1)
        need = 1;
    uint64_t acc = 0;
    for (int k = 0; k < 32768; k++) {
        acc += hist[k];
        if (acc >= need) {
            double m = oracle_bf16_to_double((uint16_t)k);
            if (!isfinite(m))
                return ORACLE_ERR_NONFINITE;
            *m_out = m;
            return ORACLE_OK;
        }
    }
    return ORACLE_ERR_SHAPE;
}

/* Static tensor scale from a clipping range: fl32(clip / 2688), 1 for 0. */
float oracle_static_scale(double clip)
{
    if (clip == 0.0)
        return 1.0f;
    return (float)clip / 2688.0f;  /* clip is a bf16 value: exact in float */
}

/* Quantisation error of fake_quant_static: sum over all values of
 * (x - y)^2 with y the bf16 fake-quant output, in fp64 -- the measure the
 * error-based range minimises over candidate clips. */
double oracle_quant_error(const uint16_t *x, int64_t rows, int64_t C, float s_g)
{
    uint16_t *y = (uint16_t *)malloc(sizeof(uint16_t) * rows * C);
    if (!y)
        return NAN;
    if (oracle_fake_quant_static(x, rows, C, s_g, y, NULL, NULL)) {
        free(y);
        return NAN;
    }
    double e = 0.0;
    for (int64_t i = 0; i < rows * C; i++) {
        double d = oracle_bf16_to_double(x[i]) - oracle_bf16_to_double(y[i]);
        e += d * d;
    }
    free(y);
    return e;
}

/* ----------------------------------------------------- full Gram, GPTQ */

/* Full Gram accumulation H += X^T X over all C channels (C x C, row-major,
 * fp64).  [LH] "A different objective": the output-error Hessian is X X^T;
 * "Trying it": Local-Hessian can be combined with GPTQ, which needs the whole
 * matrix, not only its 16x16 diagonal blocks. */
int oracle_gram_full(const uint16_t *x, int64_t n_tok, int64_t C, double *H)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t a = 0; a < C; a++)
        for (int64_t b = 0; b < C; b++) {
            double acc = 0.0;
            for (int64_t t = 0; t < n_tok; t++)
                acc += oracle_bf16_to_double(x[t * C + a]) * oracle_bf16_to_double(x[t * C + b]);
            H[a * C + b] += acc;
        }
    return ORACLE_OK;
}

/* GPTQ (Frantar, Ashkboos, Hoefler, Alistarh, "GPTQ: Accurate Post-Training
 * Quantization for Generative Pre-trained Transformers"), as [LH] "Trying it"
 * combines it with Local-Hessian scales: the block scales are given (from any
 * scale rule) and GPTQ changes only the rounding.  The paper quantises the
 * columns of W one at a time, in order, and after column j moves the columns
 * not yet quantised to compensate its error, through the inverse Hessian:
 *   (dampening)  H <- H + lambda I, lambda = damp * mean(diag H)
 *   (Cholesky reformulation)  U = the upper Cholesky factor of H^-1
 *   for j = 0..C-1:  q_j = quant(w_j);  e = (w_j - q_j) / U_jj;
 *                    w_k <- w_k - e U_jk  for every k > j.
 * The factor step, once per Hessian: U (C x C upper, row-major) from H.
 * Plain fp64: H + lambda I = L L^T, H^-1 = L^-T L^-1, H^-1 = U^T U.
 * Returns ORACLE_ERR_NOT_SPD when a pivot is not positive. */
#define ORACLE_ERR_NOT_SPD 9
int oracle_gptq_factor(const double *H, int64_t C, double damp, double *U)
{
    double *L = (double *)calloc((size_t)(C * C), sizeof(double));
    double *Li = (double *)calloc((size_t)(C * C), sizeof(double));
    double *Hi = (double *)calloc((size_t)(C * C), sizeof(double));
    if (!L || !Li || !Hi) {
        free(L); free(Li); free(Hi);
        return ORACLE_ERR_SHAPE;
    }
    int st = ORACLE_OK;
    double mean = 0.0;
    for (int64_t i = 0; i < C; i++)
        mean += H[i * C + i];
    mean /= (double)C;
    double lambda = damp * mean;
    /* H + lambda I = L L^T (lower, column by column) */
    for (int64_t j = 0; j < C && st == ORACLE_OK; j++) {
        double d = H[j * C + j] + lambda;
        for (int64_t k = 0; k < j; k++)
            d -= L[j * C + k] * L[j * C + k];
        if (!(d > 0.0)) {
            st = ORACLE_ERR_NOT_SPD;
            break;
        }
        double ljj = sqrt(d);
        L[j * C + j] = ljj;
#pragma omp parallel for schedule(static)
        for (int64_t i = j + 1; i < C; i++) {
            double v = H[i * C + j];
            for (int64_t k = 0; k < j; k++)
                v -= L[i * C + k] * L[j * C + k];
            L[i * C + j] = v / ljj;
        }
    }
    if (st == ORACLE_OK) {
        /* L^-1 (lower), one column c per unit vector by forward substitution;
         * stored transposed (Li[c][i] = (L^-1)[i][c]) so the sums run along
         * rows */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t c = 0; c < C; c++)
            for (int64_t i = c; i < C; i++) {
                double v = (i == c) ? 1.0 : 0.0;
                for (int64_t k = c; k < i; k++)
                    v -= L[i * C + k] * Li[c * C + k];
                Li[c * C + i] = v / L[i * C + i];
            }
        /* H^-1 = L^-T L^-1: entry (a, b) = sum over k >= max(a, b) of
         * (L^-1)[k][a] (L^-1)[k][b] */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t a = 0; a < C; a++)
            for (int64_t b = 0; b < C; b++) {
                double v = 0.0;
                for (int64_t k = (a > b ? a : b); k < C; k++)
                    v += Li[a * C + k] * Li[b * C + k];
                Hi[a * C + b] = v;
            }
        /* H^-1 = U^T U (U upper), row i of U finished at step i; built as its
         * transpose Ut (lower, Ut[j][i] = U[i][j]) so the sums run along rows */
        double *Ut = L; /* L is no longer needed */
        memset(Ut, 0, sizeof(double) * (size_t)(C * C));
        for (int64_t i = 0; i < C && st == ORACLE_OK; i++) {
            double d = Hi[i * C + i];
            for (int64_t k = 0; k < i; k++)
                d -= Ut[i * C + k] * Ut[i * C + k];
            if (!(d > 0.0)) {
                st = ORACLE_ERR_NOT_SPD;
                break;
            }
            double uii = sqrt(d);
            Ut[i * C + i] = uii;
#pragma omp parallel for schedule(static)
            for (int64_t j = i + 1; j < C; j++) {
                double v = Hi[i * C + j];
                for (int64_t k = 0; k < i; k++)
                    v -= Ut[i * C + k] * Ut[j * C + k];
                Ut[j * C + i] = v / uii;
            }
        }
        for (int64_t i = 0; i < C; i++)
            for (int64_t j = 0; j < C; j++)
                U[i * C + j] = (j >= i) ? Ut[j * C + i] : 0.0;
    }
    free(L); free(Li); free(Hi);
    return st;
}

/* The column loop for a list of rows (rows are independent given U): packed
 * GPTQ codes of each listed row ([n_rows][C/2], nibble order of
 * oracle_quantize_pack) and, when wq is not NULL, the value each element
 * had when it was rounded ([n_rows][C]).  The quantised value q_j = v s_eff
 * is exact in fp64, and so is the rounding decision (oracle_e2m1_encode). */
int oracle_gptq_rows(const uint16_t *w, int64_t C, float s_g, const uint8_t *codes,
                     const double *U, const int64_t *rows, int64_t n_rows, uint8_t *packed,
                     double *wq)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nb = C / 16;
    int st = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_rows; n++) {
        int64_t r = rows[n];
        double *x = (double *)malloc(sizeof(double) * (size_t)C);
        if (!x) {
            st = ORACLE_ERR_SHAPE;
            continue;
        }
        for (int64_t i = 0; i < C; i++)
            x[i] = oracle_bf16_to_double(w[r * C + i]);
        for (int64_t j = 0; j < C; j++) {
            double s = (double)oracle_effective_scale(s_g, codes[r * nb + j / 16]);
            int q = oracle_e2m1_encode(x[j], s);
            if (wq)
                wq[n * C + j] = x[j];
            if (j & 1)
                packed[n * (C / 2) + j / 2] |= (uint8_t)(q << 4);
            else
                packed[n * (C / 2) + j / 2] = (uint8_t)q;
            double e = (x[j] - oracle_e2m1_value(q) * s) / U[j * C + j];
            for (int64_t k = j + 1; k < C; k++)
                x[k] -= e * U[j * C + k];
        }
        free(x);
    }
    return st;
}

/* Whole-matrix GPTQ rounding of W [R, C] with its Hessian H [C, C]. */
int oracle_gptq(const uint16_t *w, int64_t R, int64_t C, float s_g, const uint8_t *codes,
                const double *H, double damp, uint8_t *packed)
{
    if (C % 16)
        return ORACLE_ERR_SHAPE;
    double *U = (double *)malloc(sizeof(double) * (size_t)(C * C));
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(R > 0 ? R : 1));
    if (!U || !rows) {
        free(U); free(rows);
        return ORACLE_ERR_SHAPE;
    }
    int st = oracle_gptq_factor(H, C, damp, U);
    if (st == ORACLE_OK) {
        for (int64_t r = 0; r < R; r++)
            rows[r] = r;
        st = oracle_gptq_rows(w, C, s_g, codes, U, rows, R, packed, NULL);
    }
    free(U); free(rows);
    return st;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
