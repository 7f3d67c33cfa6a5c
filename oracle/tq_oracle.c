/*
 * tq_oracle.c -- plain, slow, single-threaded CPU oracle for the ternary
 * (BitNet b1.58 style) linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never
 * calls it.
 *
 * Every function follows the definition on the pages in the order the pages
 * give it, with no blocking, fusion or reordering:
 *
 *   [F]  Foundry, docs/quantization.md -- "Ternary Format / Encoding" and
 *        "Ternary Quantization (BitNet b1.58) / How It Works" (absmean gamma,
 *        round+clamp, 00=-1 01=0 10=+1 packing four per byte LSB-first,
 *        add/subtract/skip matmul scaled by gamma); "Ternary Training
 *        (Backward Pass + Stochastic Flip)" (backward_input, xorshift64
 *        stochastic flip, seed).
 *   [H]  Hetman-2b, src/quantization.py -- section 1 (FWHT B=512: nine
 *        butterfly stages h = 1..256, then 1/sqrt(512)), section 2
 *        (AbsmeanWeightQuantizer.forward, SymmetricActivationQuantizer.forward),
 *        section 4 (SubLayerRMSNorm.forward), section 5 (BitLinear.forward
 *        steps 0-6), section 7 (simulate_hardware_bitnet_gemv); section 2
 *        AbsmeanWeightQuantizer.backward (the STE) for training.
 *   [B]  BitRASP, core_math.py -- additive_ternary_linear_int8
 *        (y[o] = sum of x where W=+1 minus sum of x where W=-1).
 *
 * Precision: the pages compute in fp32 ([H] says so for FWHT, gamma and the
 * activation scale), so every step whose result decides an integer code is
 * done in fp32 exactly as written.  gamma is the real-valued mean of |w|
 * rounded once to the nearest fp32 (ties to even) -- computed here with an
 * exact integer sum, so it does not depend on any summation order.  The
 * RMSNorm sum of squares and the output rescale are computed in fp64 and
 * rounded once to fp32.
 *
 * Compile: gcc -O2 -std=gnu99 -fPIC -shared -ffp-contract=off (no fast-math:
 * the fp32 divides and rint() below must be IEEE round-to-nearest-even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define TQO_EPS 1e-6f /* [H] section 2: eps = 1e-6 for gamma and for the activation absmax */

/* ------------------------------------------------------------------------ */
/* Exact mean of |w| rounded to fp32                                          */
/* ------------------------------------------------------------------------ */

/* The sum is held as an unsigned integer in units of 2^-213 (the smallest
 * fp32 subnormal 2^-149, shifted up by 64 more bits so the quotient by n
 * keeps at least 25 significant bits).  14 x 32-bit limbs = 448 bits, enough
 * for 2^40 terms of magnitude below 2^128. */
#define TQO_LIMBS 14
#define TQO_UNIT_EXP (-213)

static void big_add_shifted(uint32_t *limb, uint64_t v, int bitpos)
{
    /* limb += v << bitpos */
    int li = bitpos / 32, off = bitpos % 32;
    unsigned __int128 t = ((unsigned __int128)v) << off;
    uint64_t carry = 0;
    for (int i = li; i < TQO_LIMBS; ++i) {
        uint64_t piece = (uint64_t)(t & 0xffffffffu);
        t >>= 32;
        uint64_t s = (uint64_t)limb[i] + piece + carry;
        limb[i] = (uint32_t)s;
        carry = s >> 32;
        if (t == 0 && carry == 0) break;
    }
}

static int big_bit(const uint32_t *limb, int i)
{
    return (int)((limb[i / 32] >> (i % 32)) & 1u);
}

static int big_any_below(const uint32_t *limb, int i)
{
    /* any bit set in positions [0, i) */
    for (int j = 0; j < i; ++j)
        if (big_bit(limb, j)) return 1;
    return 0;
}

static int big_bitlen(const uint32_t *limb)
{
    for (int i = TQO_LIMBS - 1; i >= 0; --i)
        if (limb[i]) {
            int b = 31;
            while (!((limb[i] >> b) & 1u)) --b;
            return i * 32 + b + 1;
        }
    return 0;
}

/* Round-to-nearest-even fp32 of mean(|w|) over n values, then max(eps).
 * [F] "How It Works" step 1: gamma = mean(|weights|);
 * [H] section 2 AbsmeanWeightQuantizer.forward: mean(|W|).clamp(min=eps).
 * Non-finite inputs are outside this function's contract (see
 * tqo_sanitize_weights). */
float tqo_absmean_gamma(const float *w, int64_t n, float eps)
{
    /* Bucket the integer significands by binary exponent: |w| = m * 2^(s-149),
     * m < 2^24, s in [0, 253].  Each bucket sum is exact in 64 bits. */
    uint64_t bucket[256];
    memset(bucket, 0, sizeof bucket);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits;
        memcpy(&bits, &w[i], 4);
        uint32_t e = (bits >> 23) & 0xffu;
        uint32_t f = bits & 0x7fffffu;
        if (e == 0) {
            bucket[0] += f; /* subnormal: f * 2^-149 */
        } else {
            bucket[e - 1] += (uint64_t)(f | 0x800000u); /* (f+2^23) * 2^(e-150) */
        }
    }
    uint32_t sum[TQO_LIMBS];
    memset(sum, 0, sizeof sum);
    for (int s = 0; s < 256; ++s)
        if (bucket[s]) big_add_shifted(sum, bucket[s], s + 64);

    /* Long division by n: q = floor(sum / n), r = sum mod n. */
    uint32_t q[TQO_LIMBS];
    unsigned __int128 r = 0;
    for (int i = TQO_LIMBS - 1; i >= 0; --i) {
        unsigned __int128 cur = (r << 32) | sum[i];
        q[i] = (uint32_t)(cur / (unsigned __int128)n);
        r = cur % (unsigned __int128)n;
    }

    float mean;
    int b = big_bitlen(q);
    if (b == 0 && r == 0) {
        mean = 0.0f;
    } else {
        /* Value = (q + r/n) * 2^-213.  Keep 24 significant bits for a normal
         * result; a subnormal result has a fixed resolution of 2^-149, i.e. it
         * drops exactly the 64 pre-shift bits. */
        int d = b - 24;
        if (d < 64) d = 64;
        uint64_t kept = 0;
        for (int i = b - 1; i >= d; --i) kept = (kept << 1) | (uint64_t)big_bit(q, i);
        int half = big_bit(q, d - 1);
        int sticky = big_any_below(q, d - 1) || (r != 0);
        if (half && (sticky || (kept & 1u))) kept += 1;
        mean = (float)ldexp((double)kept, d + TQO_UNIT_EXP);
    }
    return mean > eps ? mean : eps;
}

/* ------------------------------------------------------------------------ */
/* Weight quantisation and packing                                            */
/* ------------------------------------------------------------------------ */

/* [H] section 2 AbsmeanWeightQuantizer.forward quarantines corrupted weights
 * with nan -> 0, +inf -> +1, -inf -> -1 before the absmean. */
void tqo_sanitize_weights(const float *w, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) {
        float v = w[i];
        if (isnan(v)) v = 0.0f;
        else if (isinf(v)) v = v > 0 ? 1.0f : -1.0f;
        out[i] = v;
    }
}

/* q = clamp(round(w / gamma), -1, 1), fp32 divide, round half to even.
 * [F] "How It Works" step 2; [H] section 2 (W_tilde = Clip(Round(W/gamma))).
 * gamma has one entry (per_row == 0) or N entries (per_row != 0, the
 * per-output-channel granularity of [F] fq_quantize_ternary_per_channel).
 * A NaN quotient maps to 0. */
void tqo_ternary_codes(const float *w, int64_t N, int64_t K, const float *gamma,
                       int per_row, int8_t *q)
{
    for (int64_t n = 0; n < N; ++n) {
        float g = per_row ? gamma[n] : gamma[0];
        for (int64_t k = 0; k < K; ++k) {
            float r = w[n * K + k] / g;
            float t = rintf(r);
            int8_t c;
            if (isnan(t)) c = 0;
            else if (t > 1.0f) c = 1;
            else if (t < -1.0f) c = -1;
            else c = (int8_t)t;
            q[n * K + k] = c;
        }
    }
}

/* Threshold ternarisation: tau = fp32(ratio * gamma), code = +1 if w > tau,
 * -1 if w < -tau, else 0 (strict comparisons).  ratio = 1 is [F] "Absmean
 * Thresholding (BitNet b1.58)" (threshold = mean |w|); ratio = 0.55 with
 * per-row gamma is [B] ternarize_weight (w > threshold * scale, scale = the
 * row's mean |w|).  gamma as for tqo_ternary_codes. */
void tqo_ternary_codes_threshold(const float *w, int64_t N, int64_t K, const float *gamma,
                                 int per_row, float ratio, int8_t *q)
{
    for (int64_t n = 0; n < N; ++n) {
        float g = per_row ? gamma[n] : gamma[0];
        float tau = ratio * g;
        for (int64_t k = 0; k < K; ++k) {
            float v = w[n * K + k];
            q[n * K + k] = (int8_t)(v > tau ? 1 : (v < -tau ? -1 : 0));
        }
    }
}

/* byte[n][j] = (v3 << 6) | (v2 << 4) | (v1 << 2) | v0 with v = code + 1,
 * i.e. -1 -> 0b00, 0 -> 0b01, +1 -> 0b10, value 4j+i in bits 2i..2i+1.
 * [F] "Ternary Format / Encoding".  Rows are K-contiguous, K % 4 == 0. */
void tqo_pack(const int8_t *q, int64_t N, int64_t K, uint8_t *packed)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 4; ++j) {
            unsigned v0 = (unsigned)(q[n * K + 4 * j + 0] + 1);
            unsigned v1 = (unsigned)(q[n * K + 4 * j + 1] + 1);
            unsigned v2 = (unsigned)(q[n * K + 4 * j + 2] + 1);
            unsigned v3 = (unsigned)(q[n * K + 4 * j + 3] + 1);
            packed[n * (K / 4) + j] = (uint8_t)((v3 << 6) | (v2 << 4) | (v1 << 2) | v0);
        }
}

/* Inverse of tqo_pack.  The encoding leaves 0b11 unassigned; it decodes to 0
 * here and the return value counts how many were seen. */
int64_t tqo_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *q)
{
    int64_t reserved = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 4; ++j) {
            unsigned b = packed[n * (K / 4) + j];
            for (int i = 0; i < 4; ++i) {
                unsigned v = (b >> (2 * i)) & 3u;
                int8_t c;
                if (v == 0) c = -1;
                else if (v == 1) c = 0;
                else if (v == 2) c = 1;
                else { c = 0; ++reserved; }
                q[n * K + 4 * j + i] = c;
            }
        }
    return reserved;
}

/* The other two layouts of [H] section 3 (PackedTernaryStorage), four codes
 * per byte LSB-first as above:
 *   format 1 ("Format 0", the arithmetic-optimised default there): the low
 *            two bits of the int8 code, -1 -> 0b11, 0 -> 0b00, +1 -> 0b01;
 *   format 2 ("Format 1"): -1 -> 0b10, 0 -> 0b00, +1 -> 0b01.
 * format 0 is [F]'s layout (tqo_pack).  The numbering is this library's. */
void tqo_pack_format(const int8_t *q, int64_t N, int64_t K, int format, uint8_t *packed)
{
    if (format == 0) {
        tqo_pack(q, N, K, packed);
        return;
    }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 4; ++j) {
            unsigned b = 0;
            for (int i = 0; i < 4; ++i) {
                int c = q[n * K + 4 * j + i];
                unsigned v;
                if (format == 1) v = (unsigned)(c & 3); /* two's complement -1 = ...11 */
                else v = c == -1 ? 2u : (c == 1 ? 1u : 0u);
                b |= v << (2 * i);
            }
            packed[n * (K / 4) + j] = (uint8_t)b;
        }
}

/* Decoding of [H] section 3 unpack_torch, per 2-bit field f: P = f & 1,
 * N = (f >> 1) & 1; "Format 0": v = P - 2 (P & N); "Format 1": v = P - N.
 * The unassigned field (0b10, resp. 0b11) decodes to 0 by these formulas
 * (the page's "reserved / NOP").  format 0 ([F]) decodes as tqo_unpack. */
static int decode_field(unsigned f, int format)
{
    int P = (int)(f & 1u), Nb = (int)((f >> 1) & 1u);
    if (format == 1) return P - 2 * (P & Nb);
    if (format == 2) return P - Nb;
    return f == 0 ? -1 : (f == 2 ? 1 : 0);
}

void tqo_unpack_format(const uint8_t *packed, int64_t N, int64_t K, int format, int8_t *q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 4; ++j) {
            unsigned b = packed[n * (K / 4) + j];
            for (int i = 0; i < 4; ++i) q[n * K + 4 * j + i] = (int8_t)decode_field((b >> (2 * i)) & 3u, format);
        }
}

/* gamma (per tensor, or per row) then codes then packing: the export path of
 * [H] section 5 BitLinear.export_packed_weights, with the per-row gamma of
 * [F] fq_quantize_ternary_per_channel as the alternative granularity. */
void tqo_quantize_pack_threshold(const float *w_in, int64_t N, int64_t K, int per_row,
                                 int sanitize, int format, float ratio, uint8_t *packed,
                                 float *gamma)
{
    const float *w = w_in;
    float *tmp = NULL;
    if (sanitize) {
        tmp = (float *)malloc((size_t)(N * K) * sizeof(float));
        tqo_sanitize_weights(w_in, N * K, tmp);
        w = tmp;
    }
    if (per_row) {
        for (int64_t n = 0; n < N; ++n) gamma[n] = tqo_absmean_gamma(w + n * K, K, TQO_EPS);
    } else {
        gamma[0] = tqo_absmean_gamma(w, N * K, TQO_EPS);
    }
    int8_t *q = (int8_t *)malloc((size_t)(N * K));
    if (ratio > 0.0f)
        tqo_ternary_codes_threshold(w, N, K, gamma, per_row, ratio, q);
    else
        tqo_ternary_codes(w, N, K, gamma, per_row, q);
    tqo_pack_format(q, N, K, format, packed);
    free(q);
    free(tmp);
}

/* [F] "Ternary Quantization": the manual-threshold variant
 * fq_quantize_ternary_threshold(weights, shape, ndim, threshold).  The page
 * gives the absmean rule as "threshold = mean |w|; w > threshold -> +1,
 * w < -threshold -> -1, otherwise 0; scale = threshold" and says a manual
 * threshold replaces the automatic absmean one, so here the caller's threshold
 * takes mean |w|'s place in all three lines: codes by strict comparison with
 * +-thr, and the stored scale (gamma[0]) is thr itself.  One scale for the
 * tensor, as the page's call takes one threshold.  thr >= 0, finite. */
void tqo_quantize_pack_abs_threshold(const float *w_in, int64_t N, int64_t K, int sanitize, int format,
                                     float thr, uint8_t *packed, float *gamma)
{
    const float *w = w_in;
    float *tmp = NULL;
    if (sanitize) {
        tmp = (float *)malloc((size_t)(N * K) * sizeof(float));
        tqo_sanitize_weights(w_in, N * K, tmp);
        w = tmp;
    }
    int8_t *q = (int8_t *)malloc((size_t)(N * K));
    for (int64_t i = 0; i < N * K; ++i) {
        float v = w[i];
        q[i] = (int8_t)(v > thr ? 1 : (v < -thr ? -1 : 0));
    }
    gamma[0] = thr;
    tqo_pack_format(q, N, K, format, packed);
    free(q);
    free(tmp);
}

/* ratio 0: the round/clamp rule of tqo_ternary_codes. */
void tqo_quantize_pack_format(const float *w_in, int64_t N, int64_t K, int per_row,
                              int sanitize, int format, uint8_t *packed, float *gamma)
{
    tqo_quantize_pack_threshold(w_in, N, K, per_row, sanitize, format, 0.0f, packed, gamma);
}

void tqo_quantize_pack(const float *w_in, int64_t N, int64_t K, int per_row,
                       int sanitize, uint8_t *packed, float *gamma)
{
    tqo_quantize_pack_format(w_in, N, K, per_row, sanitize, 0, packed, gamma);
}

/* ------------------------------------------------------------------------ */
/* Activation quantisation                                                    */
/* ------------------------------------------------------------------------ */

/* Per token m ([H] section 2 SymmetricActivationQuantizer.forward, which
 * reduces over the last dimension):
 *   eta   = max(max_k |x|, eps)                 (optionally clamped to
 *                                                [eta_min, eta_max], the
 *                                                Hadamard gain clamp)
 *   scale = 127 / eta                          (fp32)
 *   x_q   = clamp(round(x * scale), -127, 127)  (fp32 product, half to even)
 *   s_x   = eta / 127                           (fp32; y = acc * gamma * s_x)
 *   rowsum= sum_k x_q                           (int32)
 * rowsum is not a quantity of the pages; the CUDA path uses it to correct
 * an offset encoding of the codes and exposes it, so the oracle defines it
 * here by its plain sum. */
void tqo_act_quant(const float *x, int64_t M, int64_t K, int clamp_eta, float eta_min,
                   float eta_max, int8_t *xq, float *s_x, int32_t *rowsum)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *row = x + m * K;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(row[k]);
            if (v > a) a = v;
        }
        float eta = a > TQO_EPS ? a : TQO_EPS;
        if (clamp_eta) {
            if (eta < eta_min) eta = eta_min;
            if (eta > eta_max) eta = eta_max;
        }
        float scale = 127.0f / eta;
        int32_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float p = row[k] * scale;
            float t = rintf(p);
            int32_t c;
            if (isnan(t)) c = 0;
            else if (t > 127.0f) c = 127;
            else if (t < -127.0f) c = -127;
            else c = (int32_t)t;
            xq[m * K + k] = (int8_t)c;
            sum += c;
        }
        s_x[m] = eta / 127.0f;
        if (rowsum) rowsum[m] = sum;
    }
}

/* ------------------------------------------------------------------------ */
/* Integer contraction                                                        */
/* ------------------------------------------------------------------------ */

/* acc[m][n] = sum_k x_q[m][k] * q[n][k], the dense integer definition
 * ([H] section 5 step 5, y_int32 = x_q @ w_ternary^T).  Accumulated in 64
 * bits; |acc| <= 127 * K fits int32 for every K this library accepts. */
void tqo_matmul_dense(const int8_t *xq, const int8_t *q, int64_t M, int64_t N, int64_t K,
                      int32_t *acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)xq[m * K + k] * (int64_t)q[n * K + k];
            acc[m * N + n] = (int32_t)s;
        }
}

/* The multiply-free form: decode each packed byte ([F] encoding) and add x
 * where the code is +1, subtract where it is -1, skip 0 ([F] "Native Matmul
 * Kernel"; [B] additive_ternary_linear_int8; [H] section 7 walks the packed
 * row byte by byte the same way). */
void tqo_matmul_addsub(const int8_t *xq, const uint8_t *packed, int64_t M, int64_t N,
                       int64_t K, int32_t *acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t plus = 0, minus = 0;
            for (int64_t j = 0; j < K / 4; ++j) {
                unsigned b = packed[n * (K / 4) + j];
                for (int i = 0; i < 4; ++i) {
                    unsigned v = (b >> (2 * i)) & 3u;
                    int64_t xv = xq[m * K + 4 * j + i];
                    if (v == 2) plus += xv;       /* +1 */
                    else if (v == 0) minus += xv; /* -1 */
                }
            }
            acc[m * N + n] = (int32_t)(plus - minus);
        }
}

/* The same add/subtract/skip walk for a packed row in any of the three
 * layouts, each field decoded by the layout's own rule (decode_field). */
void tqo_matmul_addsub_format(const int8_t *xq, const uint8_t *packed, int64_t M, int64_t N,
                              int64_t K, int format, int32_t *acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t plus = 0, minus = 0;
            for (int64_t j = 0; j < K / 4; ++j) {
                unsigned b = packed[n * (K / 4) + j];
                for (int i = 0; i < 4; ++i) {
                    int v = decode_field((b >> (2 * i)) & 3u, format);
                    int64_t xv = xq[m * K + 4 * j + i];
                    if (v == 1) plus += xv;
                    else if (v == -1) minus += xv;
                }
            }
            acc[m * N + n] = (int32_t)(plus - minus);
        }
}

/* y[m][n] = acc[m][n] * gamma_n * s_x[m], computed in fp64 and rounded once
 * to fp32 ([H] section 5 step 6 and section 7's single scale fusion,
 * written as y = acc * gamma * s_x with s_x = eta / 127). */
void tqo_dequant(const int32_t *acc, const float *gamma, int per_row, const float *s_x,
                 int64_t M, int64_t N, float *y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double g = per_row ? (double)gamma[n] : (double)gamma[0];
            y[m * N + n] = (float)((double)acc[m * N + n] * g * (double)s_x[m]);
        }
}

/* Epilogue variants.
 * [H] section 5 BitLinear.forward step 6: y = y_int32 * scale_fusion, then
 * "+ self.bias" when the layer has one: here y = acc * gamma_n * s_x[m] +
 * bias[n], computed in fp64 and rounded once (bias may be NULL).
 * [B] additive_ternary_linear_int8: acc += bias[o] (int32), then, for
 * out_shift > 0, acc >>= out_shift (arithmetic shift): the integer output. */
void tqo_dequant_bias(const int32_t *acc, const float *gamma, int per_row, const float *s_x,
                      const float *bias, int64_t M, int64_t N, float *y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double g = per_row ? (double)gamma[n] : (double)gamma[0];
            double b = bias ? (double)bias[n] : 0.0;
            y[m * N + n] = (float)((double)acc[m * N + n] * g * (double)s_x[m] + b);
        }
}

void tqo_int_epilogue(const int32_t *acc, const int32_t *bias, int out_shift, int64_t M, int64_t N,
                      int32_t *out)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t v = (int64_t)acc[m * N + n] + (bias ? (int64_t)bias[n] : 0);
            if (out_shift > 0) {
                /* floor division by 2^out_shift: the arithmetic right shift */
                int64_t d = (int64_t)1 << out_shift;
                v = v >= 0 ? v / d : -((-v + d - 1) / d);
            }
            out[m * N + n] = (int32_t)v;
        }
}

/* [H] section 6 SwiGLUClamped.forward, between the projections:
 *   activated = SiLU(gate) * up,  SiLU(v) = v * sigmoid(v) = v / (1 + e^-v),
 *   clamped   = clamp(activated, -clamp_val, +clamp_val)   (10.0 on the page).
 * Computed in fp64 and rounded once to fp32. */
void tqo_swiglu_act(const float *gate, const float *up, int64_t n, float clamp_val, float *out)
{
    for (int64_t i = 0; i < n; ++i) {
        double g = (double)gate[i];
        double a = g / (1.0 + exp(-g)) * (double)up[i];
        if (a > (double)clamp_val) a = (double)clamp_val;
        if (a < -(double)clamp_val) a = -(double)clamp_val;
        out[i] = (float)a;
    }
}

/* ------------------------------------------------------------------------ */
/* Prologue: quench, RMSNorm, FWHT-512                                        */
/* ------------------------------------------------------------------------ */

/* [H] section 5 BitLinear.forward step 0: nan -> 0, +inf -> eta_max,
 * -inf -> -eta_max. */
void tqo_sanitize_acts(const float *x, int64_t n, float eta_max, float *out)
{
    for (int64_t i = 0; i < n; ++i) {
        float v = x[i];
        if (isnan(v)) v = 0.0f;
        else if (isinf(v)) v = v > 0 ? eta_max : -eta_max;
        out[i] = v;
    }
}

/* x * rsqrt(mean(x^2) + eps) * g per token ([H] section 4
 * SubLayerRMSNorm.forward).  gain == NULL means unit gain. */
void tqo_rmsnorm(const float *x, const float *gain, int64_t M, int64_t K, float eps,
                 float *out)
{
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += (double)x[m * K + k] * (double)x[m * K + k];
        double r = 1.0 / sqrt(ss / (double)K + (double)eps);
        for (int64_t k = 0; k < K; ++k) {
            double g = gain ? (double)gain[k] : 1.0;
            out[m * K + k] = (float)((double)x[m * K + k] * r * g);
        }
    }
}

/* Blockwise FWHT over 512-element blocks of each row, in fp32 ([H] section 1
 * fast_walsh_hadamard_transform_512 and blockwise_fwht_forward): for
 * h = 1, 2, 4, ..., 256, every pair (i, i+h) with bit h of i clear becomes
 * (a + b, a - b); then, if normalize, every element is multiplied by the
 * fp32 value of 1/sqrt(512).  K % 512 == 0.  x and y may alias. */
void tqo_fwht512(const float *x, float *y, int64_t rows, int64_t K, int normalize)
{
    const float norm = (float)(1.0 / sqrt(512.0));
    float buf[512];
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t blk = 0; blk < K / 512; ++blk) {
            const float *src = x + r * K + blk * 512;
            float *dst = y + r * K + blk * 512;
            for (int i = 0; i < 512; ++i) buf[i] = src[i];
            for (int h = 1; h < 512; h *= 2)
                for (int i = 0; i < 512; ++i)
                    if ((i & h) == 0) {
                        float a = buf[i], b = buf[i + h];
                        buf[i] = a + b;
                        buf[i + h] = a - b;
                    }
            for (int i = 0; i < 512; ++i) dst[i] = normalize ? buf[i] * norm : buf[i];
        }
}

/* [H] section 1 FastWalshHadamardTransform.forward (the quantisation round
 * trip of the module, per row of K, K % 512 == 0):
 *   0. nan -> 0, +inf -> eta_max, -inf -> -eta_max (nan_to_num);
 *   1. x_rot = FWHT-512 (normalised) of every block;
 *   2. eta = max_k |x_rot| + 1e-5 (fp32), clamped to [eta_min, eta_max];
 *   3. x_q = clamp(round(x_rot * (127 / eta)), -127, 127) (fp32, half to even),
 *      dequantised as x_q * fp32(eta / 127) -- the straight-through form
 *      x_s + (x_q - x_s) is exactly x_q in fp32, since x_q - x_s is exact;
 *   4. y = FWHT-512 (normalised) of the dequantised row.
 * eta_out[row] receives the clamped eta (the module reports their mean). */
void tqo_fwht_roundtrip(const float *x, int64_t rows, int64_t K, float eta_min, float eta_max,
                        float *y, float *eta_out)
{
    float *t = (float *)malloc((size_t)K * sizeof(float));
    float *u = (float *)malloc((size_t)K * sizeof(float));
    for (int64_t r = 0; r < rows; ++r) {
        tqo_sanitize_acts(x + r * K, K, eta_max, t);
        tqo_fwht512(t, u, 1, K, 1);
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(u[k]);
            if (v > a) a = v;
        }
        float eta = a + 1e-5f;
        if (eta < eta_min) eta = eta_min;
        if (eta > eta_max) eta = eta_max;
        float scale = 127.0f / eta;
        float back = eta / 127.0f;
        for (int64_t k = 0; k < K; ++k) {
            float q = rintf(u[k] * scale);
            if (q > 127.0f) q = 127.0f;
            if (q < -127.0f) q = -127.0f;
            t[k] = q * back;
        }
        tqo_fwht512(t, y + r * K, 1, K, 1);
        if (eta_out) eta_out[r] = eta;
    }
    free(t);
    free(u);
}

/* ------------------------------------------------------------------------ */
/* Whole layer                                                                */
/* ------------------------------------------------------------------------ */

/* [H] section 5 BitLinear.forward on pre-packed weights:
 *   0. optional quench (sanitize)          3. per-token int8 quantisation
 *   1. optional RMSNorm (eps, gain)        5. integer contraction (add/sub)
 *   2. optional blockwise FWHT-512         6. y = acc * gamma * s_x
 * Steps 1-2 run in the pages' order.  xq_out / s_x_out / acc_out may be NULL. */
void tqo_bitlinear(const float *x, const float *rms_gain, float rms_eps, int use_rmsnorm,
                   int use_fwht, int sanitize, int clamp_eta, float eta_min, float eta_max,
                   const uint8_t *packed, const float *gamma, int per_row, int64_t M,
                   int64_t N, int64_t K, float *y, int8_t *xq_out, float *s_x_out,
                   int32_t *acc_out)
{
    float *a = (float *)malloc((size_t)(M * K) * sizeof(float));
    if (sanitize) tqo_sanitize_acts(x, M * K, eta_max, a);
    else memcpy(a, x, (size_t)(M * K) * sizeof(float));
    if (use_rmsnorm) tqo_rmsnorm(a, rms_gain, M, K, rms_eps, a);
    if (use_fwht) tqo_fwht512(a, a, M, K, 1);
    int8_t *xq = (int8_t *)malloc((size_t)(M * K));
    float *sx = (float *)malloc((size_t)M * sizeof(float));
    tqo_act_quant(a, M, K, clamp_eta, eta_min, eta_max, xq, sx, NULL);
    int32_t *acc = (int32_t *)malloc((size_t)(M * N) * sizeof(int32_t));
    tqo_matmul_addsub(xq, packed, M, N, K, acc);
    tqo_dequant(acc, gamma, per_row, sx, M, N, y);
    if (xq_out) memcpy(xq_out, xq, (size_t)(M * K));
    if (s_x_out) memcpy(s_x_out, sx, (size_t)M * sizeof(float));
    if (acc_out) memcpy(acc_out, acc, (size_t)(M * N) * sizeof(int32_t));
    free(acc);
    free(sx);
    free(xq);
    free(a);
}

/* ------------------------------------------------------------------------ */
/* Training: gradient through the layer, STE, stochastic flip               */
/* ------------------------------------------------------------------------ */

/* [F] "Ternary Training (Backward Pass + Stochastic Flip) / Backward Pass",
 * fq_matmul_ternary_backward_input: the gradient of Y = scale * X W_ternary
 * with respect to X, formed with the same unpacking as the forward and summed
 * over the output features.  W is stored [N][K] here (row = output feature n),
 * so, with scale_n = gamma_n (per row) or gamma_0 (per tensor),
 *
 *   g[m][n]  = fp32(dY[m][n] * scale_n)                 (one fp32 product)
 *   dX[m][k] = fp32( (accumulate ? dX[m][k] : 0) + row_scale[m] * sum_n g[m][n] q[n][k] )
 *
 * The sum is taken in fp64 (terms are fp32 values times -1, 0 or +1) and the
 * result rounded once.  accumulate = 1 is the page's "+=" (the caller zeroes
 * d_input first); row_scale (NULL = 1) is the per-token factor of [H]
 * section 5 BitLinear.forward step 6 (y_int32 * gamma / scale_x): the
 * gradient reaching x_q there is dY * gamma * s_x W, which section 2's
 * identity STE passes on unchanged. */
void tqo_backward_input(const float *dY, const uint8_t *packed, int format, const float *gamma,
                        int per_row, const float *row_scale, int accumulate, int64_t M, int64_t N,
                        int64_t K, float *dX)
{
    int8_t *q = (int8_t *)malloc((size_t)(N * K));
    double *s = (double *)malloc((size_t)K * sizeof(double));
    tqo_unpack_format(packed, N, K, format, q);
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) s[k] = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            float sc = per_row ? gamma[n] : gamma[0];
            float g = dY[m * N + n] * sc;
            for (int64_t k = 0; k < K; ++k) s[k] += (double)g * (double)q[n * K + k];
        }
        double rs = row_scale ? (double)row_scale[m] : 1.0;
        for (int64_t k = 0; k < K; ++k) {
            double v = rs * s[k];
            if (accumulate) v += (double)dX[m * K + k];
            dX[m * K + k] = (float)v;
        }
    }
    free(s);
    free(q);
}

/* [H] section 2, AbsmeanWeightQuantizer.backward.  The forward saved
 * w_scaled = w / gamma (fp32, after the quarantine nan -> 0, +inf -> 1,
 * -inf -> -1 when the weights held any); the gradient of the latent weights is
 *
 *   grad_w = (grad_w_ternary / gamma) * (|w_scaled| <= tau ? 1 : 0.1)
 *
 * every operation in fp32 as the page computes it (0.1 is the fp32 constant).
 * gamma per tensor on the page; per row as the per-channel variant. */
void tqo_ste_backward(const float *grad, const float *w, const float *gamma, int per_row, float tau,
                      int sanitize, int64_t N, int64_t K, float *out)
{
    for (int64_t n = 0; n < N; ++n) {
        float gm = per_row ? gamma[n] : gamma[0];
        for (int64_t k = 0; k < K; ++k) {
            float wv = w[n * K + k];
            if (sanitize) {
                if (isnan(wv)) wv = 0.0f;
                else if (isinf(wv)) wv = wv > 0 ? 1.0f : -1.0f;
            }
            float ws = wv / gm;
            float damp = fabsf(ws) <= tau ? 1.0f : 0.1f;
            float gw = grad[n * K + k] / gm;
            out[n * K + k] = gw * damp;
        }
    }
}

/* [F] "Stochastic Weight Flip": the generator is xorshift64 on a 64-bit
 * state the caller owns.  G. Marsaglia, "Xorshift RNGs", Journal of
 * Statistical Software 8(14), 2003: the 64-bit generator with the shift
 * triple (13, 7, 17) -- x ^= x << 13; x ^= x >> 7; x ^= x << 17 -- whose
 * new state is also the output. */
uint64_t tqo_xorshift64(uint64_t *state)
{
    uint64_t x = *state;
    x ^= x << 13;
    x ^= x >> 7;
    x ^= x << 17;
    *state = x;
    return x;
}

/* [F] fq_seed.  The page does not say how the seed becomes the state; here
 * the state is the seed itself, except that 0 (a fixed point of xorshift)
 * becomes 0x9E3779B97F4A7C15. */
void tqo_seed(uint64_t *state, uint64_t seed)
{
    *state = seed ? seed : 0x9E3779B97F4A7C15ull;
}

/* [F] fq_ternary_stochastic_flip, for every weight in storage order (row n,
 * then k), one draw each:
 *   x = xorshift64(state), u = (x >> 40) * 2^-24      (a uniform fp32 in [0, 1))
 *   p = clamp(|grad| * temperature, 0, 1)              (fp32; NaN never flips)
 *   if u < p: q = clamp(q - sign(grad), -1, 1)         (one step toward -grad)
 * Codes are read and written in `format` (see tqo_pack_format); the state is
 * left after the last draw. */
void tqo_stochastic_flip(uint8_t *packed, int format, const float *grad, float temperature,
                         int64_t N, int64_t K, uint64_t *state)
{
    int8_t *q = (int8_t *)malloc((size_t)(N * K));
    tqo_unpack_format(packed, N, K, format, q);
    for (int64_t i = 0; i < N * K; ++i) {
        uint64_t x = tqo_xorshift64(state);
        float u = (float)(x >> 40) * 0x1p-24f;
        float a = fabsf(grad[i]) * temperature;
        float p = a > 1.0f ? 1.0f : a; /* a >= 0 or NaN; NaN stays NaN and u < NaN is false */
        if (u < p) {
            int c = q[i] - (grad[i] > 0.0f ? 1 : (grad[i] < 0.0f ? -1 : 0));
            q[i] = (int8_t)(c > 1 ? 1 : (c < -1 ? -1 : c));
        }
    }
    tqo_pack_format(q, N, K, format, packed);
    free(q);
}
