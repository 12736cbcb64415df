/*
 * wq_oracle.c -- plain, slow, fp64 CPU oracle for group-wise 4-bit weight coding
 * and its W4A16 consumption.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call this
 * file: only the test suite, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (cited below by their key and section):
 *   [DG]  "MiniCPM5-1B 验证: 6× 压缩, ppl 反超 fp, 1.2GB 显存, 50ms Triton 推理"
 *         (the DyadicGumbel 4-bit article), wmrh.cn/news/898890
 *   [KM]  "K-Means量化技术：突破LLM低比特部署瓶颈", mhpn.cn/news/872954
 *   [G32] "int4-g32+warm 裸量化：原理与实验报告", 0539edu.com/news/5477008
 *   [BX]  "同一个 1B 模型，我上了三种压缩方案：无损的、4bit 的、还有没跑通的",
 *         bjdmk.com.cn/news/3920032, section "第一剑·完美主义：BF16X" (lossless codec)
 *
 * Conventions
 *   - W is row-major [n, k] (out x in), groups are runs of `group` consecutive
 *     columns of one row ([G32] §5.1: "for each group g along in").
 *   - bf16 / fp16 values travel as their bit patterns (uint16_t). They are widened
 *     exactly to double; rounding back uses round-to-nearest-even written out below.
 *   - Every function works on a row range [r0, r1) so that the caller can split a
 *     matrix across host threads. Returns 0 on success, <0 on invalid input.
 *   - All arithmetic is double precision. No blocking, fusion or reordering beyond the
 *     definitions.
 *
 * Parity status of each function (what pins it) is listed in the test suite; the
 * absolute MSE figures printed by [G32] §1.4 are "parity unpinned" (they need a real
 * model layer).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------- */
/* Binary16-style formats: decode exactly, encode with round-to-nearest-even.        */
/* ------------------------------------------------------------------------------- */

/* Decode a (1, ebits, mbits) IEEE-style bit pattern to double (exact). */
static double decode_ieee(uint32_t bits, int ebits, int mbits)
{
    uint32_t sign = (bits >> (ebits + mbits)) & 1u;
    uint32_t e = (bits >> mbits) & ((1u << ebits) - 1u);
    uint32_t m = bits & ((1u << mbits) - 1u);
    int bias = (1 << (ebits - 1)) - 1;
    double v;
    if (e == 0)
        v = ldexp((double)m, 1 - bias - mbits);                 /* zero / subnormal */
    else if (e == (1u << ebits) - 1u)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | (1u << mbits)), (int)e - bias - mbits);
    return sign ? -v : v;
}

/* Encode a double into a (1, ebits, mbits) format, rounding to nearest, ties to even.
 * The magnitude is divided by the quantum (a power of two: exact), split into an
 * integer part and a remainder (exact), and rounded by comparing the remainder with
 * one half. Overflow gives infinity, as IEEE rounding does. */
static uint32_t encode_ieee_rne(double v, int ebits, int mbits)
{
    uint32_t sign = signbit(v) ? 1u : 0u;
    uint32_t sbit = sign << (ebits + mbits);
    uint32_t emask = (1u << ebits) - 1u;
    int bias = (1 << (ebits - 1)) - 1;
    int emin = 1 - bias;                                         /* smallest normal exponent */
    int emax = bias;                                             /* largest finite exponent */
    if (isnan(v))
        return sbit | (emask << mbits) | (1u << (mbits - 1));
    double a = fabs(v);
    if (isinf(a))
        return sbit | (emask << mbits);
    if (a == 0.0)
        return sbit;
    int e2;
    frexp(a, &e2);                                               /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;
    if (E < emin)
        E = emin;                                                /* subnormal: fixed quantum */
    double quantum = ldexp(1.0, E - mbits);
    double q = a / quantum;
    double fl = floor(q);
    double rem = q - fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))
        fl += 1.0;
    double r = fl * quantum;                                     /* rounded magnitude */
    double maxfinite = ldexp((double)((2u << mbits) - 1u), emax - mbits);
    if (r > maxfinite)
        return sbit | (emask << mbits);
    if (r < ldexp(1.0, emin)) {
        /* subnormal; a carry up to 2^emin encodes as exponent field 1, mantissa 0 */
        uint32_t m = (uint32_t)(r / ldexp(1.0, emin - mbits));
        return sbit | m;
    }
    frexp(r, &e2);
    E = e2 - 1;
    uint32_t m = (uint32_t)(r / ldexp(1.0, E - mbits)) - (1u << mbits);
    return sbit | ((uint32_t)(E + bias) << mbits) | m;
}

double orc_bf16_to_double(uint16_t h) { return decode_ieee(h, 8, 7); }
uint16_t orc_double_to_bf16(double v) { return (uint16_t)encode_ieee_rne(v, 8, 7); }
double orc_fp16_to_double(uint16_t h) { return decode_ieee(h, 5, 10); }
uint16_t orc_double_to_fp16(double v) { return (uint16_t)encode_ieee_rne(v, 5, 10); }

void orc_bf16_to_double_array(const uint16_t* h, int64_t count, double* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = orc_bf16_to_double(h[i]);
}
void orc_double_to_bf16_array(const double* v, int64_t count, uint16_t* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = orc_double_to_bf16(v[i]);
}
void orc_fp16_to_double_array(const uint16_t* h, int64_t count, double* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = orc_fp16_to_double(h[i]);
}
void orc_double_to_fp16_array(const double* v, int64_t count, uint16_t* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = orc_double_to_fp16(v[i]);
}

/* ------------------------------------------------------------------------------- */
/* Dyadic 4-bit code ([DG] §2.1, §2.2, §2.3, §2.5)                                   */
/* ------------------------------------------------------------------------------- */

/* Per group: scale = max |w| (a bf16 value, so storing it as bf16 is exact; [DG] §2.2
 * "scale_i (bf16), the codebook half-range"); half = 2^(b-1) = 8, step = scale / half,
 * codebook = step * {-8, ..., 7} ([DG] §2.1); idx = argmin_j |w - (j - 8) * step|
 * ([DG] §2.3, §2.5 "hard argmin"), the lowest j winning a tie. The argmin is a plain
 * search over the 16 code values. */
int orc_dyadic_quantize(const uint16_t* w, int64_t n, int64_t k, int32_t group,
                        int64_t r0, int64_t r1, uint16_t* scale, uint8_t* codes)
{
    (void)n;
    if (group <= 0 || k % group != 0) return -1;
    const int64_t ng = k / group;
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const uint16_t* wg = w + r * k + g * group;
            double amax = 0.0;
            for (int32_t j = 0; j < group; ++j) {
                double v = orc_bf16_to_double(wg[j]);
                if (!isfinite(v)) return -2;
                if (fabs(v) > amax) amax = fabs(v);
            }
            scale[r * ng + g] = orc_double_to_bf16(amax);
            const double half = 8.0;
            const double step = amax / half;
            for (int32_t j = 0; j < group; ++j) {
                double v = orc_bf16_to_double(wg[j]);
                int best = 0;
                double bestd = fabs(v - (0 - 8) * step);
                for (int c = 1; c < 16; ++c) {
                    double d = fabs(v - (c - 8) * step);
                    if (d < bestd) { bestd = d; best = c; }
                }
                codes[r * k + g * group + j] = (uint8_t)best;
            }
        }
    }
    return 0;
}

/* STE fake quantisation, forward ([DG] §2.3 "STE"): on an fp32 latent z with the block's
 * bf16 scale, idx = argmin_j |z - step*(j-8)| over j = 0..15 (lowest j on a tie, the same
 * rule as the hard argmin above), step = scale/8, and the forward value is the code value
 * q = step*(idx-8) itself (exact in fp32: an 8-bit significand times an integer of
 * magnitude <= 8, over 8). The backward of STE is the identity and computes nothing. Every
 * distance is exact in double (z has 24 significant bits, a code value 11). z may lie
 * outside [-scale, scale] (the scale is a trained parameter): the argmin then picks the
 * end code. */
int orc_fake_quant_ste(const float* z, const uint16_t* scale, int64_t n, int64_t k, int32_t group,
                       int64_t r0, int64_t r1, float* q, uint8_t* codes)
{
    (void)n;
    if (group <= 0 || k % group != 0) return -1;
    const int64_t ng = k / group;
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t c = 0; c < k; ++c) {
            const double v = (double)z[r * k + c];
            const double step = orc_bf16_to_double(scale[r * ng + c / group]) / 8.0;
            if (!isfinite(v) || !isfinite(step)) return -2;
            int best = 0;
            double bestd = fabs(v - (0 - 8) * step);
            for (int j = 1; j < 16; ++j) {
                const double d = fabs(v - (j - 8) * step);
                if (d < bestd) { bestd = d; best = j; }
            }
            codes[r * k + c] = (uint8_t)best;
            q[r * k + c] = (float)((best - 8) * step);
        }
    }
    return 0;
}

/* Gumbel-ST soft assignment, backward ([DG] §2.3 "Gumbel-ST"). The page's training step:
 *   codes = step * {-8, ..., 7}, step = scale / 8     (a function of the trained scale)
 *   soft  = softmax(-dist / tau) . codes               (soft weighting)
 *   hard  = codes[argmin(dist)]                         (hard choice)
 *   q     = hard + (soft - soft.detach())               (hard forward, soft backward)
 * Readings: dist_j = (z - codes_j)^2 (the squared distance the page checkpoints as
 * "dist2" in §2.4); the printed softmax carries no noise term, so none is added; argmin
 * ties go to the lowest index. The forward value q is hard itself (soft - soft = 0), the
 * STE forward above. This function gives the backward for an upstream gradient gq:
 *   gz[i]       = gq[i] * d soft / d z
 *   gscale[g]   = sum over the group of gq[i] * (d hard / d scale + d soft / d scale)
 * by the chain rule written out term by term through the softmax, in double:
 *   l_j = -dist_j / tau,  d p_j / d t = p_j * sum_i p_i (d l_j / d t - d l_i / d t)
 *   (the softmax Jacobian p_j (delta_ji - p_i), with sum_i p_i = 1), where
 *   d l_j / d z - d l_i / d z         = 2 (codes_j - codes_i) / tau,
 *   d l_j / d scale - d l_i / d scale = 2 ((z - codes_j) a_j - (z - codes_i) a_i) / tau,
 *   a_j = d codes_j / d scale = (j - 8) / 8, d hard / d scale = a_idx, d hard / d z = 0
 *   (idx is piecewise constant in z).
 * Each difference of two logit derivatives is formed from its closed form, in which z
 * cancels exactly: subtracting the two large derivatives themselves loses most digits when
 * tau is small and z lies beyond the codes. gz_mag / gscale_mag (may be NULL) receive the
 * same sums taken over absolute values of every term, a scale for comparing a
 * lower-precision result with these. */
int orc_gumbel_st_backward(const float* z, const uint16_t* scale, const float* gq, int64_t n,
                           int64_t k, int32_t group, double tau, int64_t r0, int64_t r1,
                           float* gz, double* gscale, double* gz_mag, double* gscale_mag)
{
    (void)n;
    if (group <= 0 || k % group != 0) return -1;
    if (!(tau > 0.0) || !isfinite(tau)) return -3;
    const int64_t ng = k / group;
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const double s = orc_bf16_to_double(scale[r * ng + g]);
            const double step = s / 8.0;
            if (!isfinite(s)) return -2;
            double codes[16], a[16];
            for (int j = 0; j < 16; ++j) {
                codes[j] = step * (j - 8);
                a[j] = (j - 8) / 8.0;
            }
            double gs = 0.0, gs_mag = 0.0;
            for (int64_t c = g * group; c < (g + 1) * group; ++c) {
                const double v = (double)z[r * k + c], up = (double)gq[r * k + c];
                if (!isfinite(v) || !isfinite(up)) return -2;
                double dist[16], l[16], p[16];
                int idx = 0;
                for (int j = 0; j < 16; ++j) {
                    dist[j] = (v - codes[j]) * (v - codes[j]);
                    if (dist[j] < dist[idx]) idx = j;
                    l[j] = -dist[j] / tau;
                }
                double lmax = l[0];
                for (int j = 1; j < 16; ++j) lmax = l[j] > lmax ? l[j] : lmax;
                double den = 0.0;
                for (int j = 0; j < 16; ++j) { p[j] = exp(l[j] - lmax); den += p[j]; }
                for (int j = 0; j < 16; ++j) p[j] /= den;
                double dsoft_z = 0.0, dsoft_s = 0.0, mag_z = 0.0, mag_s = 0.0;
                for (int j = 0; j < 16; ++j) {
                    double dpz = 0.0, dps = 0.0, dpz_mag = 0.0, dps_mag = 0.0;
                    for (int i = 0; i < 16; ++i) {
                        const double ddz = 2.0 * (codes[j] - codes[i]) / tau;
                        const double dds = 2.0 * ((v - codes[j]) * a[j] - (v - codes[i]) * a[i]) / tau;
                        dpz += p[i] * ddz;
                        dps += p[i] * dds;
                        dpz_mag += p[i] * fabs(ddz);
                        dps_mag += p[i] * fabs(dds);
                    }
                    dpz *= p[j];
                    dps *= p[j];
                    dsoft_z += codes[j] * dpz;
                    dsoft_s += p[j] * a[j] + codes[j] * dps;
                    mag_z += fabs(codes[j]) * p[j] * dpz_mag;
                    mag_s += p[j] * fabs(a[j]) + fabs(codes[j]) * p[j] * dps_mag;
                }
                const double dhard_s = a[idx];
                gz[r * k + c] = (float)(up * dsoft_z);
                if (gz_mag) gz_mag[r * k + c] = fabs(up) * mag_z;
                gs += up * (dhard_s + dsoft_s);
                gs_mag += fabs(up) * (fabs(dhard_s) + mag_s);
            }
            if (gscale) gscale[r * ng + g] = gs;
            if (gscale_mag) gscale_mag[r * ng + g] = gs_mag;
        }
    }
    return 0;
}

/* Reconstruction w = step * (idx - 8) ([DG] §2.2), stored as bf16 (one rounding). */
int orc_dyadic_dequant(const uint8_t* codes, const uint16_t* scale, int64_t n, int64_t k,
                       int32_t group, int64_t r0, int64_t r1, uint16_t* out)
{
    (void)n;
    if (group <= 0 || k % group != 0) return -1;
    const int64_t ng = k / group;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = 0; c < k; ++c) {
            double step = orc_bf16_to_double(scale[r * ng + c / group]) / 8.0;
            out[r * k + c] = orc_double_to_bf16(step * ((double)codes[r * k + c] - 8.0));
        }
    return 0;
}

/* ------------------------------------------------------------------------------- */
/* Nibble packing ([DG] §2.5: two 4-bit indices to one byte, "lo | hi << 4")         */
/* ------------------------------------------------------------------------------- */

/* byte[r, j] = code[r, 2j] | code[r, 2j+1] << 4: the even column is the low nibble. */
int orc_pack(const uint8_t* codes, int64_t n, int64_t k, int64_t r0, int64_t r1, uint8_t* packed)
{
    (void)n;
    if (k % 2 != 0) return -1;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < k / 2; ++j) {
            uint8_t lo = codes[r * k + 2 * j], hi = codes[r * k + 2 * j + 1];
            if (lo > 15 || hi > 15) return -2;
            packed[r * (k / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
    return 0;
}

int orc_unpack(const uint8_t* packed, int64_t n, int64_t k, int64_t r0, int64_t r1, uint8_t* codes)
{
    (void)n;
    if (k % 2 != 0) return -1;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < k / 2; ++j) {
            uint8_t b = packed[r * (k / 2) + j];
            codes[r * k + 2 * j] = (uint8_t)(b & 15);
            codes[r * k + 2 * j + 1] = (uint8_t)(b >> 4);
        }
    return 0;
}

/* ------------------------------------------------------------------------------- */
/* Dequantised rows for the three formats, and the W4A16 product reference.          */
/* ------------------------------------------------------------------------------- */

enum { ORC_DYADIC4 = 0, ORC_LLOYD8S = 1, ORC_LUT16 = 2 };

/* One dequantised row as doubles.
 *   DYADIC4: bf16(step * (idx - 8)), step = scale / 8            ([DG] §2.2)
 *   LLOYD8S: bf16(sign ? -level[q] : level[q]), code = q | sign<<3, fp32 levels
 *            ([G32] §1.3 step 4 "w = sign * |w|", §2 "3-bit level + 1 sign bit")
 *   LUT16:   the fp16 centroid selected by the code, exactly      ([KM] §1.2, §2.2)  */
static int dequant_row(int fmt, const uint8_t* packed, const void* aux, int64_t k, int32_t group,
                       int64_t r, double* row)
{
    const uint8_t* p = packed + r * (k / 2);
    const int64_t ng = k / group;
    for (int64_t c = 0; c < k; ++c) {
        uint8_t b = p[c / 2];
        int code = (c % 2 == 0) ? (b & 15) : (b >> 4);
        int64_t g = r * ng + c / group;
        if (fmt == ORC_DYADIC4) {
            double step = orc_bf16_to_double(((const uint16_t*)aux)[g]) / 8.0;
            row[c] = orc_bf16_to_double(orc_double_to_bf16(step * (code - 8)));
        } else if (fmt == ORC_LLOYD8S) {
            double lv = (double)((const float*)aux)[g * 8 + (code & 7)];
            row[c] = orc_bf16_to_double(orc_double_to_bf16((code >> 3) ? -lv : lv));
        } else if (fmt == ORC_LUT16) {
            row[c] = orc_fp16_to_double(((const uint16_t*)aux)[g * 16 + code]);
        } else {
            return -1;
        }
    }
    return 0;
}

/* Dequantised weights as 16-bit patterns: bf16 for DYADIC4 and LLOYD8S, fp16 for LUT16
 * (the centroid itself, so that nothing is rounded). */
int orc_dequant(int32_t fmt, const uint8_t* packed, const void* aux, int64_t n, int64_t k,
                int32_t group, int64_t r0, int64_t r1, uint16_t* out)
{
    (void)n;
    if (group <= 0 || k % group != 0 || k % 2 != 0) return -1;
    double* row = (double*)malloc(sizeof(double) * (size_t)k);
    if (!row) return -3;
    int rc = 0;
    for (int64_t r = r0; r < r1 && rc == 0; ++r) {
        rc = dequant_row(fmt, packed, aux, k, group, r, row);
        for (int64_t c = 0; c < k && rc == 0; ++c)
            out[r * k + c] = (fmt == ORC_LUT16) ? orc_double_to_fp16(row[c]) : orc_double_to_bf16(row[c]);
    }
    free(row);
    return rc;
}

/* y[b, r] = sum_c Wdeq[r, c] * x[b, c] in double, over the output rows listed in
 * `rows` (all rows of a range, or a sample), together with the error scale
 * bound[b, r] = sum_c |Wdeq[r, c]| * |x[b, c]| that the parity tolerance is relative to.
 * x is bf16 [m, k]; y and bound are [m, nrows] (column j belongs to rows[j]). */
int orc_matmul_rows(int32_t fmt, const uint8_t* packed, const void* aux, int64_t k, int32_t group,
                    const uint16_t* x, int64_t m, const int64_t* rows, int64_t nrows,
                    int64_t j0, int64_t j1, double* y, double* bound)
{
    if (group <= 0 || k % group != 0 || k % 2 != 0) return -1;
    double* row = (double*)malloc(sizeof(double) * (size_t)k);
    double* xd = (double*)malloc(sizeof(double) * (size_t)(k * m));
    if (!row || !xd) { free(row); free(xd); return -3; }
    for (int64_t i = 0; i < k * m; ++i) xd[i] = orc_bf16_to_double(x[i]);
    int rc = 0;
    for (int64_t j = j0; j < j1 && rc == 0; ++j) {
        rc = dequant_row(fmt, packed, aux, k, group, rows[j], row);
        for (int64_t b = 0; b < m && rc == 0; ++b) {
            double s = 0.0, sa = 0.0;
            for (int64_t c = 0; c < k; ++c) {
                s += row[c] * xd[b * k + c];
                sa += fabs(row[c]) * fabs(xd[b * k + c]);
            }
            y[b * nrows + j] = s;
            bound[b * nrows + j] = sa;
        }
    }
    free(row);
    free(xd);
    return rc;
}

/* ------------------------------------------------------------------------------- */
/* Lloyd g32 producer with the 112-candidate warm start ([G32] §1.2, §1.3, §2, §5.1)  */
/* ------------------------------------------------------------------------------- */

/* The candidate grid, [G32] §1.2. Candidates are numbered c = 0..111:
 *   c = 7*r + t   (0 <= c < 105): bounded rational family f(a) = a / (b + a^beta),
 *                  b_rel = 10^(-3 + 5r/14) (logspace(-3, 2, 15)), beta = BETA[t];
 *   c = 105 + u  (105 <= c < 112): tanh family f(a) = tanh(a / b), b_rel = TANH_BREL[u].
 * In both, b = b_rel * gmax with gmax = max |w| of the group. The constant c of the
 * rational family cancels in f / fmax and is taken as 1. */
static const double BETA[7] = {0.50, 0.55, 0.65, 0.75, 0.85, 0.95, 1.00};
static const double TANH_BREL[7] = {0.25, 0.4, 0.6, 0.85, 1.2, 1.8, 3.0};

int orc_lloyd_num_candidates(void) { return 112; }

/* family (0 rational, 1 tanh), b_rel, beta (1 for tanh) of candidate c. */
int orc_lloyd_candidate(int32_t c, int32_t* family, double* b_rel, double* beta)
{
    if (c < 0 || c >= 112) return -1;
    if (c < 105) {
        int r = c / 7, t = c % 7;
        *family = 0;
        *b_rel = pow(10.0, -3.0 + 5.0 * r / 14.0);
        *beta = BETA[t];
    } else {
        *family = 1;
        *b_rel = TANH_BREL[c - 105];
        *beta = 1.0;
    }
    return 0;
}

/* Per-group parameter byte in the 1 + 4 + 3 bit split of [G32] §2:
 * family << 7 | b_rel index << 3 | beta index (tanh: b_rel index = u, beta index 0). */
int orc_lloyd_params_byte(int32_t c)
{
    if (c < 0 || c >= 112) return -1;
    if (c < 105) return ((c / 7) << 3) | (c % 7);
    return (1 << 7) | ((c - 105) << 3);
}

static double transform(int family, double a, double b, double beta)
{
    if (family == 0) return a / (b + pow(a, beta));
    return tanh(a / b);
}

/* Inverse of the transform at fd, [G32] §1.2: rational beta = 1 has the closed form
 * w = fd*b / (1 - fd); tanh has w = b * atanh(fd); rational beta < 1 has no closed form
 * (the page iterates w <- fd*b + fd*w^beta) and is solved here as the root of the
 * increasing function f(L) - fd on [0, hi] by bisection down to adjacent doubles. */
double orc_lloyd_inverse(int32_t family, double fd, double b, double beta, double hi)
{
    if (family == 1) return b * atanh(fd);
    if (beta == 1.0) return fd * b / (1.0 - fd);
    double lo = 0.0;
    if (fd <= 0.0) return 0.0;
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (transform(0, mid, b, beta) < fd) lo = mid; else hi = mid;
    }
    /* the root lies in [lo, hi], adjacent doubles: take the closer one */
    double glo = fabs(transform(0, lo, b, beta) - fd), ghi = fabs(transform(0, hi, b, beta) - fd);
    return (glo <= ghi) ? lo : hi;
}

/* [G32] §1.3 step 1 / §5.1, for one candidate: 8-level uniform quantisation in f-space,
 * q = clamp(round(f / fmax * 7), 0, 7) (round half to even), reconstruction through the
 * inverse at q / 7 * fmax, and the group MSE of the magnitudes. Levels 0 and 7 are the
 * exact images of 0 and gmax. Returns the MSE; writes the 8 levels and the q's. */
static double candidate_eval(int c, const double* a, int gsize, double gmax, double* levels, int* q)
{
    int family;
    double b_rel, beta;
    orc_lloyd_candidate(c, &family, &b_rel, &beta);
    double b = b_rel * gmax;
    double fmax = transform(family, gmax, b, beta);
    for (int i = 0; i < gsize; ++i) {
        double f = transform(family, a[i], b, beta);
        double qq = rint(f / fmax * 7.0);
        if (qq < 0.0) qq = 0.0;
        if (qq > 7.0) qq = 7.0;
        q[i] = (int)qq;
    }
    levels[0] = 0.0;
    levels[7] = gmax;
    for (int j = 1; j < 7; ++j)
        levels[j] = orc_lloyd_inverse(family, (double)j / 7.0 * fmax, b, beta, gmax);
    double se = 0.0;
    for (int i = 0; i < gsize; ++i) {
        double d = a[i] - levels[q[i]];
        se += d * d;
    }
    return se / gsize;
}

/* Nearest level, lowest index on a tie; also returns the gap to the runner-up. */
static int nearest_level(double a, const double* lv, int nl, double* gap)
{
    int best = 0;
    double bd = fabs(a - lv[0]), second = INFINITY;
    for (int j = 1; j < nl; ++j) {
        double d = fabs(a - lv[j]);
        if (d < bd) { second = bd; bd = d; best = j; }
        else if (d < second) second = d;
    }
    *gap = second - bd;
    return best;
}

/* The whole [G32] §1.3 pipeline for the groups of rows [r0, r1):
 *   1. a_i = |w_i|, sign s_i = (w_i < 0) stored apart (-0.0 counts as positive);
 *   2. evaluate the 112 candidates, keep the lowest-MSE one (lowest c on a tie) --
 *      or candidate force_cand[g] when force_cand is given;
 *   3. its 8 reconstruction values are the initial codebook; `rounds` Lloyd rounds
 *      (assign each a_i to its nearest level, lowest index on a tie; move each level
 *      to the mean of its members, an empty level keeping its value);
 *   4. a final assignment against the final levels; code = q | s << 3.
 * A group with gmax = 0 gets codes 0, levels 0, candidate 0 and MSE 0.
 * Outputs per group g (row-major over [n, k/group]):
 *   codes[n, k]; levels[g*8 + q]; params[g] (the [G32] §2 byte); cand[g];
 *   trace[g*(rounds+2) + t]: t=0 the candidate MSE, t=1..rounds+1 the MSE after each
 *   assignment (the last is the final one);
 *   cand_gap[g]: (second-best - best) candidate MSE; min_margin[g]: the smallest
 *   nearest-vs-runner-up distance gap over all assignments (both for margin-aware
 *   comparison). Any of the per-group outputs may be NULL. */
int orc_lloyd(const uint16_t* w, int64_t n, int64_t k, int32_t group, int32_t rounds,
              const int32_t* force_cand, const int32_t* init_mode,
              int64_t r0, int64_t r1, uint8_t* codes, double* levels, uint8_t* params,
              int32_t* cand, double* trace, double* cand_gap, double* min_margin)
{
    (void)n;
    if (group <= 0 || group > 256 || k % group != 0 || rounds < 0) return -1;
    const int64_t ng = k / group;
    double a[256], lv[8], best_lv[8];
    int s[256], q[256], qbest[256];
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t gi = 0; gi < ng; ++gi) {
            const int64_t g = r * ng + gi;
            const uint16_t* wg = w + r * k + gi * group;
            double gmax = 0.0;
            for (int i = 0; i < group; ++i) {
                double v = orc_bf16_to_double(wg[i]);
                if (!isfinite(v)) return -2;
                a[i] = fabs(v);
                s[i] = (v < 0.0) ? 1 : 0;
                if (a[i] > gmax) gmax = a[i];
            }
            double* tr = trace ? trace + g * (rounds + 2) : NULL;
            if (gmax == 0.0) {
                for (int i = 0; i < group; ++i) codes[r * k + gi * group + i] = 0;
                if (levels) for (int j = 0; j < 8; ++j) levels[g * 8 + j] = 0.0;
                if (params) params[g] = 0;
                if (cand) cand[g] = 0;
                if (tr) for (int t = 0; t < rounds + 2; ++t) tr[t] = 0.0;
                if (cand_gap) cand_gap[g] = INFINITY;
                if (min_margin) min_margin[g] = INFINITY;
                continue;
            }
            /* step 2: candidate search (or a forced candidate) */
            int cbest = -1;
            double mbest = INFINITY, msecond = INFINITY;
            if (init_mode && init_mode[0] == 1) {
                /* cold start for comparison: levels at the quantiles i/7 of the sorted
                 * magnitudes ("分位数初值", [G32] §1.4 decision 1) */
                double srt[256];
                memcpy(srt, a, sizeof(double) * group);
                for (int i = 1; i < group; ++i)
                    for (int j = i; j > 0 && srt[j - 1] > srt[j]; --j) {
                        double t = srt[j]; srt[j] = srt[j - 1]; srt[j - 1] = t;
                    }
                for (int j = 0; j < 8; ++j) best_lv[j] = srt[(int)((double)j / 7.0 * (group - 1) + 0.5)];
                double gap;
                double se = 0.0;
                for (int i = 0; i < group; ++i) {
                    qbest[i] = nearest_level(a[i], best_lv, 8, &gap);
                    double d = a[i] - best_lv[qbest[i]];
                    se += d * d;
                }
                mbest = se / group;
                cbest = 0;
            } else if (force_cand && force_cand[g] >= 0) {
                cbest = force_cand[g];
                mbest = candidate_eval(cbest, a, group, gmax, best_lv, qbest);
            } else {
                for (int c = 0; c < 112; ++c) {
                    double m = candidate_eval(c, a, group, gmax, lv, q);
                    if (m < mbest) {
                        msecond = mbest;
                        mbest = m;
                        cbest = c;
                        memcpy(best_lv, lv, sizeof lv);
                        memcpy(qbest, q, sizeof(int) * group);
                    } else if (m < msecond) {
                        msecond = m;
                    }
                }
            }
            if (tr) tr[0] = mbest;
            if (cand) cand[g] = cbest;
            if (params) params[g] = (uint8_t)orc_lloyd_params_byte(cbest);
            if (cand_gap) cand_gap[g] = msecond - mbest;
            /* step 3: Lloyd rounds */
            double margin = INFINITY;
            memcpy(lv, best_lv, sizeof lv);
            for (int t = 0; t <= rounds; ++t) {
                double sum[8] = {0}, se = 0.0;
                int cnt[8] = {0};
                for (int i = 0; i < group; ++i) {
                    double gap;
                    q[i] = nearest_level(a[i], lv, 8, &gap);
                    if (gap < margin) margin = gap;
                    double d = a[i] - lv[q[i]];
                    se += d * d;
                    sum[q[i]] += a[i];
                    cnt[q[i]] += 1;
                }
                if (tr) tr[t + 1] = se / group;
                if (t == rounds) break;              /* the final assignment: no update */
                for (int j = 0; j < 8; ++j)
                    if (cnt[j] > 0) lv[j] = sum[j] / cnt[j];
            }
            /* step 4: store */
            for (int i = 0; i < group; ++i) codes[r * k + gi * group + i] = (uint8_t)(q[i] | (s[i] << 3));
            if (levels) for (int j = 0; j < 8; ++j) levels[g * 8 + j] = lv[j];
            if (min_margin) min_margin[g] = margin;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------- */
/* LUT16 producer: per-block-64 1D k-means with 16 centroids ([KM] §1.2, §2.2)       */
/* ------------------------------------------------------------------------------- */

/* [KM] §1.2 gives kmeans(w_flat, k=16) and nearest_neighbor(w_flat, centroids) for each
 * block of 64 weights. The page leaves the initialisation, the number of rounds and
 * the centroid storage open; the readings taken are:
 *   init: centroid i = the (4i+2)-th smallest of the 64 values (i = 0..15);
 *   `rounds` Lloyd rounds on the signed values (nearest centroid, lowest index on a
 *   tie; centroid = mean of its members, an empty centroid keeps its value);
 *   centroids rounded to fp16 (round to nearest even), then a final nearest assignment
 *   against the fp16 centroids; no separate scale (the centroids are in weight units).
 * Outputs: codes[n, k]; lut[g*16 + i] fp16 bits; trace[g*(rounds+1) + t] the MSE after
 * each assignment (the last against the fp16 centroids); min_margin[g]. */
int orc_kmeans_lut16(const uint16_t* w, int64_t n, int64_t k, int32_t group, int32_t rounds,
                     int64_t r0, int64_t r1, uint8_t* codes, uint16_t* lut, double* trace,
                     double* min_margin)
{
    (void)n;
    if (group < 16 || group > 256 || k % group != 0 || rounds < 0) return -1;
    const int64_t ng = k / group;
    double v[256], srt[256], cen[16];
    int q[256];
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t gi = 0; gi < ng; ++gi) {
            const int64_t g = r * ng + gi;
            for (int i = 0; i < group; ++i) {
                v[i] = orc_bf16_to_double(w[r * k + gi * group + i]);
                if (!isfinite(v[i])) return -2;
                srt[i] = v[i];
            }
            for (int i = 1; i < group; ++i)                      /* insertion sort */
                for (int j = i; j > 0 && srt[j - 1] > srt[j]; --j) {
                    double t = srt[j]; srt[j] = srt[j - 1]; srt[j - 1] = t;
                }
            const int stride = group / 16;
            for (int i = 0; i < 16; ++i) cen[i] = srt[stride * i + stride / 2];
            double margin = INFINITY;
            double* tr = trace ? trace + g * (rounds + 1) : NULL;
            for (int t = 0; t <= rounds; ++t) {
                if (t == rounds)
                    for (int i = 0; i < 16; ++i) cen[i] = orc_fp16_to_double(orc_double_to_fp16(cen[i]));
                double sum[16] = {0}, se = 0.0;
                int cnt[16] = {0};
                for (int i = 0; i < group; ++i) {
                    double gap;
                    q[i] = nearest_level(v[i], cen, 16, &gap);
                    if (gap < margin) margin = gap;
                    double d = v[i] - cen[q[i]];
                    se += d * d;
                    sum[q[i]] += v[i];
                    cnt[q[i]] += 1;
                }
                if (tr) tr[t] = se / group;
                if (t == rounds) break;
                for (int i = 0; i < 16; ++i)
                    if (cnt[i] > 0) cen[i] = sum[i] / cnt[i];
            }
            for (int i = 0; i < group; ++i) codes[r * k + gi * group + i] = (uint8_t)q[i];
            if (lut) for (int i = 0; i < 16; ++i) lut[g * 16 + i] = orc_double_to_fp16(cen[i]);
            if (min_margin) min_margin[g] = margin;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------- */
/* Storage accounting ([DG] §2.5; [G32] §2)                                          */
/* ------------------------------------------------------------------------------- */

/* Bytes of the stored artefact for n*k weights: DYADIC4 = packed nibbles + one bf16
 * scale per group ([DG] §2.5: 679M x 4 bit / 8 = 340 MB, plus 21 MB of scales).
 * LLOYD8S as the page counts it = 4 bits per weight + one 8-bit parameter byte per
 * group ([G32] §2: 4 + 8/32 = 4.25 bit). LUT16 = packed nibbles + 16 fp16 centroids per
 * group. The LLOYD8S codebook actually kept for decoding (8 fp32 per group) is counted
 * separately by `orc_storage_lloyd_codebook_bytes`. */
double orc_storage_bytes(int32_t fmt, double nweights, int32_t group)
{
    double nib = nweights * 4.0 / 8.0;
    double groups = nweights / group;
    if (fmt == ORC_DYADIC4) return nib + groups * 2.0;
    if (fmt == ORC_LLOYD8S) return nib + groups * 1.0;
    if (fmt == ORC_LUT16) return nib + groups * 16.0 * 2.0;
    return -1.0;
}

double orc_storage_lloyd_codebook_bytes(double nweights, int32_t group)
{
    return nweights / group * 8.0 * 4.0;
}

/* ------------------------------------------------------------------------------- */
/* [BX] BF16X: lossless bf16 block codec                                             */
/* ------------------------------------------------------------------------------- */
/*
 * [BX] "第一剑·完美主义：BF16X": blocks of 16 bf16 weights share the largest exponent of
 * the block; each weight keeps a 3-bit difference to it; the few weights too far below
 * it go to an overflow table; decoding gives back every bit. The page fixes neither the
 * bit layout nor what happens to sign and mantissa; the reading taken here keeps both
 * verbatim (a lossless codec must), so:
 *
 *   weight j of block b (flat row-major index 16 b + j), bits h = s:1 | e:8 | m:7
 *   E_b      = max_j e_j                       (the shared exponent field)
 *   d_j      = E_b - e_j; stored as d_j if d_j <= 6, else 7 = "escaped"
 *   sm[i]    = s << 7 | m                      (one byte per weight, flat order)
 *   hdr[b]   = 64 bits: bit j of plane p (p = 0, 1, 2) at bit 16 p + j holds bit p of the
 *              stored 3-bit field of weight j; bits 48..55 = E_b; bits 56..63 = number of
 *              escaped weights in the earlier blocks of b's superblock
 *   superblock = 16 consecutive blocks (256 weights); sb_off[t] = escaped weights in all
 *              superblocks before t, sb_off[S] = total, S = ceil(blocks / 16)
 *   ovf[]    = the exponent fields e_j of the escaped weights, in flat index order
 *
 * Every bf16 pattern (zeros, subnormals, Inf, NaN payloads) round-trips.
 * The encoder below walks the weights in order with one running escape counter.
 */
int64_t orc_bf16x_superblocks(int64_t n, int64_t k)
{
    return (n * k / 16 + 15) / 16;
}

int orc_bf16x_encode(const uint16_t* w, int64_t n, int64_t k, uint8_t* sm, uint64_t* hdr,
                     uint32_t* sb_off, uint8_t* ovf, int64_t ovf_cap, int64_t* n_ovf)
{
    if (n < 0 || k < 0 || k % 16 != 0) return -1;
    int64_t nblocks = n * k / 16, escaped = 0;
    for (int64_t b = 0; b < nblocks; ++b) {
        if (b % 16 == 0) sb_off[b / 16] = (uint32_t)escaped;
        int emax = 0;
        for (int j = 0; j < 16; ++j) {
            int e = (w[16 * b + j] >> 7) & 0xFF;
            if (e > emax) emax = e;
        }
        uint64_t h = (uint64_t)emax << 48;
        h |= (uint64_t)(escaped - (int64_t)sb_off[b / 16]) << 56;
        for (int j = 0; j < 16; ++j) {
            uint16_t v = w[16 * b + j];
            int e = (v >> 7) & 0xFF;
            int d = emax - e;
            int field = d <= 6 ? d : 7;
            if (field == 7) {
                if (escaped >= ovf_cap) return -2;
                ovf[escaped++] = (uint8_t)e;
            }
            for (int p = 0; p < 3; ++p)
                if ((field >> p) & 1) h |= (uint64_t)1 << (16 * p + j);
            sm[16 * b + j] = (uint8_t)(((v >> 8) & 0x80) | (v & 0x7F));
        }
        hdr[b] = h;
    }
    sb_off[(nblocks + 15) / 16] = (uint32_t)escaped;
    *n_ovf = escaped;
    return 0;
}

/* Decoding reads the escape table with its own running counter, in flat order. The
 * superblock offsets and per-block prefixes are redundant random-access indexes; they
 * are checked against the counter (-3 if they disagree) and not otherwise used. */
int orc_bf16x_decode(const uint8_t* sm, const uint64_t* hdr, const uint32_t* sb_off,
                     const uint8_t* ovf, int64_t n_ovf, int64_t n, int64_t k, uint16_t* out)
{
    if (n < 0 || k < 0 || k % 16 != 0) return -1;
    int64_t nblocks = n * k / 16, next = 0;
    for (int64_t b = 0; b < nblocks; ++b) {
        uint64_t h = hdr[b];
        if ((int64_t)sb_off[b / 16] + (int64_t)(h >> 56) != next) return -3;
        int emax = (int)((h >> 48) & 0xFF);
        for (int j = 0; j < 16; ++j) {
            int field = 0;
            for (int p = 0; p < 3; ++p) field |= (int)((h >> (16 * p + j)) & 1) << p;
            int e;
            if (field == 7) {
                if (next >= n_ovf) return -2;
                e = ovf[next++];
            } else {
                e = emax - field;
                if (e < 0) return -4;
            }
            uint8_t c = sm[16 * b + j];
            out[16 * b + j] = (uint16_t)(((c & 0x80) << 8) | (e << 7) | (c & 0x7F));
        }
    }
    if (sb_off[(nblocks + 15) / 16] != (uint32_t)next || next != n_ovf) return -3;
    return 0;
}

/* ------------------------------------------------------------------------------- */
/* [DG] water-filling: 3/4/5-bit dyadic blocks in one level index space             */
/* ------------------------------------------------------------------------------- */
/*
 * [DG] §2.1: with half = 2^(b-1) and step = scale / half, the b-bit codebook is
 * step * {-half, ..., half - 1}; codebooks of different b line up, so when water-filling
 * changes one block's precision the 3/4/5-bit codes share one level index space and the
 * codebook need not be rebuilt. [DG] §6 leaves water-filling disabled and says no more.
 * Readings taken here (the page fixes neither the allocation rule nor the layout):
 *   block     64 consecutive weights of a row (the §2.2 block), scale = max |w| (bf16).
 *   codes     for b in {3, 4, 5}: idx_b = argmin_j |w - (j - half_b) * scale / half_b|
 *             over j = 0 .. 2^b - 1, lowest j on a tie (the 4-bit rule of §2.3).
 *   index     idx_5 = idx_b * 2^(5 - b): the same value step_5 * (idx_5 - 16).
 *   D_b       the block's squared error sum_j (w_j - code)^2. Each difference is exact in
 *             float and double (the code is zero, or within a factor of two of w), each
 *             square is exact in double; the sum runs over j = 0..63 in order, in double.
 *   width     the water level lambda (a distortion per weight, chosen by the caller):
 *             the smallest b in {3, 4, 5} with D_b <= 64 * lambda, else 5. Blocks whose
 *             3-bit error already lies under the water keep 3 bits; the others get bits
 *             until their error does, up to 5 (reverse water-filling with three rates).
 *   layout    scale bf16 [n, k/64]; width uint8 [n, k/64]; the blocks' bit streams back to
 *             back in row-major block order, block i taking 8 * width_i bytes, its code j
 *             in bits [b j, b j + b) counted from bit 0 of the block's first byte (for
 *             b = 4 this is the nibble layout of §2.5); blk_off uint32 [n k/64 + 1]: the
 *             byte offset of every block, and the total at the end.
 */

/* idx_b by a plain search over the 2^b codes (lowest index on a tie) */
static int wf_index(double w, double scale, int b)
{
    const int half = 1 << (b - 1);
    const double step = scale / half;
    int best = 0;
    double bestd = fabs(w - (0 - half) * step);
    for (int j = 1; j < (1 << b); ++j) {
        const double d = fabs(w - (j - half) * step);
        if (d < bestd) { bestd = d; best = j; }
    }
    return best;
}

/* Per block: scale, the three distortions (dist may be NULL: [n, k/64, 3] for b = 3, 4, 5),
 * the width for water level lambda, and blk_size = 8 * width bytes. */
int orc_wf_analyze(const uint16_t* w, int64_t n, int64_t k, double lambda, int64_t r0, int64_t r1,
                   uint16_t* scale, uint8_t* width, double* dist)
{
    (void)n;
    if (k % 64 != 0) return -1;
    if (!(lambda >= 0.0)) return -3;
    const int64_t nb = k / 64;
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t g = 0; g < nb; ++g) {
            const uint16_t* wg = w + r * k + g * 64;
            double amax = 0.0;
            for (int j = 0; j < 64; ++j) {
                const double v = orc_bf16_to_double(wg[j]);
                if (!isfinite(v)) return -2;
                if (fabs(v) > amax) amax = fabs(v);
            }
            scale[r * nb + g] = orc_double_to_bf16(amax);
            int chosen = 5;
            for (int b = 3; b <= 5; ++b) {
                const int half = 1 << (b - 1);
                double D = 0.0;
                for (int j = 0; j < 64; ++j) {
                    const double v = orc_bf16_to_double(wg[j]);
                    const int idx = wf_index(v, amax, b);
                    const double e = v - (idx - half) * (amax / half);
                    D += e * e;
                }
                if (dist) dist[(r * nb + g) * 3 + (b - 3)] = D;
                if (chosen == 5 && b < 5 && D <= 64.0 * lambda) chosen = b;
            }
            width[r * nb + g] = (uint8_t)chosen;
        }
    }
    return 0;
}

/* blk_off[0..nblocks] = exclusive prefix of 8 * width, total at the end */
int orc_wf_offsets(const uint8_t* width, int64_t nblocks, uint32_t* blk_off)
{
    uint64_t off = 0;
    for (int64_t i = 0; i < nblocks; ++i) {
        if (width[i] < 3 || width[i] > 5) return -2;
        blk_off[i] = (uint32_t)off;
        off += 8u * width[i];
        if (off >= ((uint64_t)1 << 32)) return -4;
    }
    blk_off[nblocks] = (uint32_t)off;
    return 0;
}

/* The blocks' codes at their widths, bit-packed (layout above). */
int orc_wf_pack(const uint16_t* w, int64_t n, int64_t k, const uint16_t* scale, const uint8_t* width,
                const uint32_t* blk_off, int64_t r0, int64_t r1, uint8_t* packed)
{
    (void)n;
    if (k % 64 != 0) return -1;
    const int64_t nb = k / 64;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t g = 0; g < nb; ++g) {
            const int b = width[r * nb + g];
            if (b < 3 || b > 5) return -2;
            const double s = orc_bf16_to_double(scale[r * nb + g]);
            uint8_t* out = packed + blk_off[r * nb + g];
            memset(out, 0, (size_t)(8 * b));
            for (int j = 0; j < 64; ++j) {
                const int idx = wf_index(orc_bf16_to_double(w[r * k + g * 64 + j]), s, b);
                for (int t = 0; t < b; ++t)
                    if ((idx >> t) & 1) out[(b * j + t) / 8] |= (uint8_t)(1u << ((b * j + t) % 8));
            }
        }
    return 0;
}

/* Reconstruction through the 5-bit index space: idx_5 = idx_b << (5 - b),
 * w = bf16((scale / 16) * (idx_5 - 16)). */
int orc_wf_dequant(const uint8_t* packed, const uint16_t* scale, const uint8_t* width,
                   const uint32_t* blk_off, int64_t n, int64_t k, int64_t r0, int64_t r1, uint16_t* out)
{
    (void)n;
    if (k % 64 != 0) return -1;
    const int64_t nb = k / 64;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t g = 0; g < nb; ++g) {
            const int b = width[r * nb + g];
            if (b < 3 || b > 5) return -2;
            const double s = orc_bf16_to_double(scale[r * nb + g]);
            const uint8_t* in = packed + blk_off[r * nb + g];
            for (int j = 0; j < 64; ++j) {
                int idx = 0;
                for (int t = 0; t < b; ++t)
                    idx |= ((in[(b * j + t) / 8] >> ((b * j + t) % 8)) & 1) << t;
                const int idx5 = idx << (5 - b);
                out[r * k + g * 64 + j] = orc_double_to_bf16(s / 16.0 * (idx5 - 16));
            }
        }
    return 0;
}
