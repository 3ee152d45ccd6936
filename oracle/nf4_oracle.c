/*
 * nf4_oracle.c -- plain, slow CPU oracle for the QLoRA linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA path.  All floating point is done in fp64 unless a step's definition
 * fixes a narrower rounding (noted where it happens).
 *
 * Sources (web pages; cited below by the short tag in brackets):
 *   [CSDN]  "大模型量化从0到1（十）：bitsandbytes——一行配置就量化的最省心方案"
 *           (aicoding.csdn.net) -- sections 5.2, 6.2, 7.1-7.2, 8.6, 12.2, 12.4
 *   [AIQZ]  "QLoRA：用4比特行李箱装下整个大模型，单卡微调不再是梦"
 *           (aiqz.cc) -- chapter 3 (NF4 by quantiles), chapter 4 (double quant)
 *   [BLOG]  "从 LoRA 到 QLoRA、QA-LoRA：低秩更新如何进入量化模型"
 *           (ludovicoyin.github.io) -- sections 1-5
 *   [CARD]  airsota "Science Depth" card on LoRA/QLoRA -- section 3
 *
 * Conventions (the plainest reading where the pages leave a step open):
 *   - x:[M,Din], A:[Din,r], B:[r,Dout], y:[M,Dout] with row-vector
 *     activations ([BLOG] section 1 shapes; [CSDN] 12.2 Y = XW + sXAB).
 *   - The frozen weight is stored transposed, Wt:[Dout,Din] row-major
 *     (nn.Linear layout); flattening it row-major and cutting it into blocks
 *     of 64 ([CSDN] 5.1) makes every block run along Din.
 *   - Two 4-bit indices per byte ([CSDN] 5.2, last paragraph): element 2i
 *     goes to the HIGH nibble of byte i, element 2i+1 to the low nibble.
 *   - Activations, adapters and the dequantized weight are bf16 values; the
 *     oracle reads them exactly as doubles and returns fp64 results.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_STATUS_NONFINITE 1
/* Double-quantization codes of the first-level scales (the `dq` argument). */
#define ORC_DQ_NONE 0
#define ORC_DQ_U8 1     /* unsigned, step = max / 255, codes 0..255 */
#define ORC_DQ_S8 2     /* signed INT8 absmax code of [CSDN] 4.1: step = max / 127, codes 0..127 */
#define ORC_DQ_MEAN 3   /* signed INT8 code of a_b minus the group mean; one mean per group */
#define ORC_DQ_F8 4     /* 8-bit float (E4M3) code of a_b / step, step = max / 448 */

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32 helpers (storage format of the inputs and of dequant out)  */
/* ------------------------------------------------------------------------ */

static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* IEEE binary16 bits -> double (exact): 1 sign, 5 exponent (bias 15) and 10
 * fraction bits; exponent 0 holds the subnormals f * 2^-24. */
static double fp16_to_double(uint16_t h) {
    const int sign = h >> 15, ex = (h >> 10) & 31, fr = h & 1023;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -24);
    else if (ex == 31)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + fr), ex - 25);
    return sign ? -v : v;
}

/* A 16-bit activation or weight element in the layer's compute dtype
 * ([CSDN] 8.3): dt 0 = bf16, 1 = fp16. */
static double dec16(uint16_t h, int dt) { return dt ? fp16_to_double(h) : bf16_to_double(h); }

/* Round an fp32 value to bf16, round-to-nearest-even on the bit pattern. */
static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* Standard normal CDF and its inverse                                      */
/* ------------------------------------------------------------------------ */

/* Phi(x) = P(Z <= x) for Z ~ N(0,1), written through the complementary
 * error function: Phi(x) = erfc(-x/sqrt(2)) / 2. */
double orc_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Phi^{-1}(p): the x with Phi(x) = p.  Found from the definition alone:
 * bisection on the monotone Phi over [-40, 40] until the bracket stops
 * shrinking, then two Newton steps x -= (Phi(x) - p) / phi(x) to polish the
 * last bits.  p must lie in (0, 1).  For p > 1/2 the symmetry
 * Phi^{-1}(p) = -Phi^{-1}(1-p) is used (1-p is exact there), so the search
 * always runs in the lower tail, where erfc keeps full relative precision. */
double orc_normal_ppf(double p) {
    if (!(p > 0.0 && p < 1.0)) return NAN;
    if (p > 0.5) return -orc_normal_ppf(1.0 - p);
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (orc_normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    for (int it = 0; it < 2; ++it) {
        double pdf = exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
        if (pdf <= 0.0) break;
        double step = (orc_normal_cdf(x) - p) / pdf;
        if (!isfinite(step)) break;
        x -= step;
    }
    return x;
}

/* ------------------------------------------------------------------------ */
/* The NF4 codebook                                                          */
/* ------------------------------------------------------------------------ */

/* [AIQZ] ch.3: levels are taken from standard-normal quantiles (Phi^{-1})
 * of equal-probability pieces of the CDF, 16 levels.  [CSDN] 6.2: the
 * levels are fixed (not per block), normalised to [-1,1], and the positive
 * and negative halves are built asymmetrically so that 0 is an exact level.
 *
 * Reading (the formula itself is missing from the pages): 8 positive and 7
 * negative levels plus an exact 0.  Positive side: Phi^{-1} of 9 probabilities
 * equally spaced from `delta` down to 1/2, the last (1/2 -> 0) dropped.
 * Negative side: the same with 8 probabilities, mirrored.  All values are
 * divided by Phi^{-1}(delta) so the extremes are exactly -1 and +1, then
 * rounded to fp32 and sorted ascending.  `delta` < 1 because Phi^{-1}(1) is
 * infinite; the library default is 1 - (1/32 + 1/30)/2, the mean of the
 * outermost interval-midpoint probabilities for 16 and for 15 equal pieces. */
void orc_nf4_codebook(double delta, float out[16]) {
    double v[16];
    int n = 0;
    double zmax = orc_normal_ppf(delta);
    for (int i = 0; i < 8; ++i) { /* linspace(delta, 1/2, 9), last dropped */
        double p = delta + (0.5 - delta) * (double)i / 8.0;
        v[n++] = orc_normal_ppf(p) / zmax;
    }
    for (int i = 0; i < 7; ++i) { /* linspace(delta, 1/2, 8), last dropped */
        double p = delta + (0.5 - delta) * (double)i / 7.0;
        v[n++] = -orc_normal_ppf(p) / zmax;
    }
    v[n++] = 0.0;
    /* insertion sort, ascending */
    for (int i = 1; i < 16; ++i) {
        double t = v[i];
        int j = i - 1;
        while (j >= 0 && v[j] > t) { v[j + 1] = v[j]; --j; }
        v[j + 1] = t;
    }
    for (int i = 0; i < 16; ++i) out[i] = (float)v[i];
}

/* The FP4 codebook ([CSDN] 6.4-6.5, 9.3: bitsandbytes' other 4-bit type, and
 * its configuration default, is a "4-bit float-style" table, not uniform
 * INT4; the pages print no values).  Reading: the FP4 E2M1 layout of the OCP
 * Microscaling formats -- 1 sign bit, 2 exponent bits with bias 1, 1 mantissa
 * bit, exponent field 0 holding the subnormals 0 and 0.5 -- divided by its
 * largest magnitude 6 so that absmax scaling maps the ends to -1 and +1.
 * Its 16 codes hold 15 distinct values: -0 and +0 are both kept, -0 first,
 * so the table is non-decreasing with one repeated level.  Rounded to fp32. */
void orc_fp4_codebook(float out[16]) {
    double mag[8];
    for (int code = 0; code < 8; ++code) {     /* exponent field e, mantissa bit m */
        const int e = code >> 1, m = code & 1;
        mag[code] = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    }
    for (int i = 0; i < 8; ++i) {
        out[7 - i] = (float)(-mag[i] / 6.0);   /* -0, -1/12, ..., -1 */
        out[8 + i] = (float)(mag[i] / 6.0);    /* +0, +1/12, ..., +1 */
    }
}

/* ------------------------------------------------------------------------ */
/* Blockwise quantization ([CSDN] 5.2) and double quantization ([CSDN] 7.2) */
/* ------------------------------------------------------------------------ */

static int zero_level_index(const float cb[16]) {
    for (int j = 0; j < 16; ++j)
        if (cb[j] == 0.0f) return j;
    return -1;
}

/* Knuth's TwoSum: s = fl(x + y) and e such that s + e == x + y exactly. */
static void two_sum(double x, double y, double *s, double *e) {
    double ss = x + y;
    double yy = ss - x;
    *e = (x - (ss - yy)) + (y - yy);
    *s = ss;
}

/* |w - p| held exactly as hi + lo (hi = fl(|w - p|)). */
static void abs_diff_exact(double w, double p, double *hi, double *lo) {
    double s, e;
    two_sum(w, -p, &s, &e);
    if (s < 0.0 || (s == 0.0 && e < 0.0)) { s = -s; e = -e; }
    *hi = s;
    *lo = e;
}

/* Nearest level of w in a block with absmax a: q = argmin_j |w/a - c_j|,
 * the first minimum on ties ([CSDN] 5.2).  Multiplying through by a > 0 the
 * rule is argmin_j |w - c_j a|, evaluated in exact real arithmetic: c_j a is
 * an exact fp64 product of two fp32 values, and w - c_j a is kept as an
 * unevaluated sum hi + lo of two doubles, so comparing (hi, lo) pairs
 * lexicographically compares the exact distances.  a == 0 (an all-zero
 * block) leaves u = w/a undefined; every weight then maps to the exact-zero
 * level, the only level that reproduces it. */
static int nearest_level(float w, float a, const float cb[16], int zero_idx) {
    if (a == 0.0f) return zero_idx;
    int best = 0;
    double bh, bl;
    abs_diff_exact((double)w, (double)cb[0] * (double)a, &bh, &bl);
    for (int j = 1; j < 16; ++j) {
        double h, l;
        abs_diff_exact((double)w, (double)cb[j] * (double)a, &h, &l);
        if (h < bh || (h == bh && l < bl)) { bh = h; bl = l; best = j; }
    }
    return best;
}

/* Double quantization with the group mean taken out first (a variant of
 * [CSDN] 7.2's structure, whose 8-bit code the pages do not give; reading:
 * centre the scales on their mean, then a symmetric INT8 code as in [CSDN]
 * 4.1).  Every step is one stated rounding:
 *   mu   = RN32(S / n), S the fp64 sum of the group's a_b in block order
 *   d_b  = RN32(a_b - mu)
 *   f    = RN32(max_b |d_b| / 127)
 *   code = clamp(round-half-even(d_b / f), -127, 127), stored as int8
 * decoded as a_hat = RN32(mu + RN32(code * f)); f = 0 gives codes of 0.
 * d_b / f is a ratio of two fp32 values of magnitude <= 127.5 (before the
 * clamp): unless it is a half-integer it lies at least 2^-32 (relative) away
 * from one, far above fp64 rounding, so rint of the fp64 quotient is the
 * exact rule.  In the decode, fp32 + fp32 done in fp64 and rounded to fp32 is
 * the correctly rounded fp32 sum (53 >= 2*24 + 2). */
static void dq_group_mean(const float *a, int64_t n, uint8_t *codes, float *step, float *offset) {
    double sum = 0.0;
    for (int64_t i = 0; i < n; ++i) sum += (double)a[i];
    const float mu = (float)(sum / (double)n);
    float mx = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        const float d = a[i] - mu;
        if (fabsf(d) > mx) mx = fabsf(d);
    }
    const float f = (float)((double)mx / 127.0);
    *step = f;
    *offset = mu;
    for (int64_t i = 0; i < n; ++i) {
        int code = 0;
        if (f > 0.0f) {
            const float d = a[i] - mu;
            double qd = rint((double)d / (double)f);
            if (qd < -127.0) qd = -127.0;
            if (qd > 127.0) qd = 127.0;
            code = (int)qd;
        }
        codes[i] = (uint8_t)(int8_t)code;
    }
}

/* The 8-bit float code of the scales.  [CSDN] 7.2 stores the first-level
 * scales in 8 bits without naming the code; an 8-bit float is one of the
 * readings.  Reading: the E4M3 layout (1 sign bit, 4 exponent bits biased by
 * 7, 3 mantissa bits, no infinity; exponent field 0 holds the subnormals
 * m * 2^-9, the largest finite value is 1.75 * 2^8 = 448).  Scales are >= 0,
 * so the sign bit is clear: codes 0 .. 0x7E. */
double orc_e4m3_value(int code) {
    const int e = (code >> 3) & 15, m = code & 7;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp(8.0 + (double)m, e - 10);
}

/* The E4M3 code nearest to x >= 0, ties to the even mantissa; x >= 448
 * gives 448 (the format has no infinity). */
int orc_e4m3_encode(double x) {
    if (!(x > 0.0)) return 0;
    if (x >= 448.0) return 0x7E;
    if (x < ldexp(1.0, -6)) return (int)rint(ldexp(x, 9)); /* a rounded-up 8 is the smallest normal */
    int e2;
    (void)frexp(x, &e2);
    const int e = e2 - 1;                                  /* 2^e <= x < 2^(e+1), e in -6..8 */
    const double m = rint((ldexp(x, -e) - 1.0) * 8.0);     /* exact scaling; rint ties to even */
    const int code = ((e + 7) << 3) + (int)m;              /* m = 8 carries into the exponent */
    return code > 0x7E ? 0x7E : code;
}

/* Quantize Wt:[rows, cols] (fp32, row-major) in blocks of `block` weights
 * (64 by default; 32, 128 or 256 trade scale resolution against metadata,
 * [CSDN] 5.1).  The row-major flattening is cut into consecutive blocks; cols
 * is a multiple of block, so every block lies inside one row.
 *   packed  [rows*cols/2]        two indices per byte, high nibble first
 *   absmax  [nb]                 fp32 block absmax (used when dq == 0)
 *   codes   [nb], steps [ceil(nb/dq_group)]   (used when dq != 0)
 * Returns a status word: ORC_STATUS_NONFINITE if any weight is NaN/Inf
 * (the pages are silent; such a block's outputs are unspecified).
 *
 * Double quantization reading ([CSDN] 7.2; [AIQZ] ch.4): the first-level
 * fp32 absmax values are quantized to 8 bits and each run of dq_group (256)
 * consecutive first-level scales shares one fp32 second-level constant.  The
 * pages give no 8-bit code; the only 8-bit quantizer they define is absmax
 * with rounding ([CSDN] 4.1).  Absmax values are >= 0, so the code is
 * unsigned with 255 as the top: the stored constant is the step
 * f = RN32(max_b a_b / 255) and code_b = round-half-even(a_b / f) in
 * [0,255] (f = 0 gives code 0).  The weights themselves are encoded once,
 * with the true a_b ([CSDN] 7: the second pass quantizes the scales, not
 * the weights). */
int orc_quantize(const float *W, int64_t rows, int64_t cols, int block, const float cb[16],
                 int dq, int dq_group, uint8_t *packed, float *absmax,
                 uint8_t *codes, float *steps, float *offsets) {
    const int64_t n = rows * cols;
    const int64_t nb = n / block;
    const int zero_idx = zero_level_index(cb);
    int status = 0;
    float *a_all = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
#pragma omp parallel for schedule(static) reduction(| : status)
    for (int64_t b = 0; b < nb; ++b) {
        const float *wb = W + b * block;
        double a = 0.0;
        for (int i = 0; i < block; ++i) {
            if (!isfinite(wb[i])) status |= ORC_STATUS_NONFINITE;
            double m = fabs((double)wb[i]);
            if (m > a) a = m;
        }
        float af = (float)a; /* exact: a is the magnitude of an fp32 value */
        a_all[b] = af;
        for (int i = 0; i < block; i += 2) {
            int q0 = nearest_level(wb[i], af, cb, zero_idx);
            int q1 = nearest_level(wb[i + 1], af, cb, zero_idx);
            packed[(b * block + i) / 2] = (uint8_t)((q0 << 4) | q1);
        }
        if (!dq) absmax[b] = af;
    }
    if (dq) {
        int64_t ng = (nb + dq_group - 1) / dq_group;
        for (int64_t g = 0; g < ng; ++g) {
            int64_t b0 = g * dq_group;
            int64_t b1 = b0 + dq_group < nb ? b0 + dq_group : nb;
            if (dq == ORC_DQ_MEAN) {
                dq_group_mean(a_all + b0, b1 - b0, codes + b0, steps + g, offsets + g);
                continue;
            }
            if (dq == ORC_DQ_F8) {
                /* step f = RN32(max / 448), the largest code's value; each
                 * scale's quotient is rounded to fp32 first, then to the
                 * nearest E4M3 value: code = E4M3(RN32(a_b / f)). */
                float mx = 0.0f;
                for (int64_t b = b0; b < b1; ++b)
                    if (a_all[b] > mx) mx = a_all[b];
                const float f = (float)((double)mx / 448.0);
                steps[g] = f;
                for (int64_t b = b0; b < b1; ++b) {
                    const float qf = f > 0.0f ? (float)((double)a_all[b] / (double)f) : 0.0f;
                    codes[b] = (uint8_t)orc_e4m3_encode((double)qf);
                }
                continue;
            }
            /* the top code: 255 for the unsigned code, 127 for the signed
             * INT8 code of [CSDN] 4.1 (absmax values are >= 0, so only its
             * codes 0..127 occur) */
            const double top = dq == ORC_DQ_S8 ? 127.0 : 255.0;
            float mx = 0.0f;
            for (int64_t b = b0; b < b1; ++b)
                if (a_all[b] > mx) mx = a_all[b];
            /* RN32(mx/top): fp64 division then one rounding to fp32 is the
             * correctly rounded fp32 quotient (53 >= 2*24+2). */
            float f = (float)((double)mx / top);
            steps[g] = f;
            for (int64_t b = b0; b < b1; ++b) {
                int code = 0;
                if (f > 0.0f) {
                    /* a/f is a ratio of two fp32 values below 256: when it is
                     * not a half-integer it sits at least 2^-33 (relative)
                     * away from one, far above fp64 rounding, so rint of the
                     * fp64 quotient is round-half-even of the exact ratio. */
                    double qd = rint((double)a_all[b] / (double)f);
                    if (qd < 0.0) qd = 0.0;
                    if (qd > top) qd = top;
                    code = (int)qd;
                }
                codes[b] = (uint8_t)code;
            }
        }
    }
    free(a_all);
    return status;
}

/* Decoded first-level scale of block b: a_b itself, or with double
 * quantization RN32(code_b * f_g) -- the product is exact in fp64 and is
 * rounded once to fp32 -- or, for the mean-offset variant with a signed
 * code, RN32(mu_g + RN32(code_b * f_g)), or for the 8-bit float code
 * RN32(E4M3(code_b) * f_g). */
static float block_scale(int64_t b, int dq, int dq_group, const float *absmax,
                         const uint8_t *codes, const float *steps, const float *offsets) {
    if (!dq) return absmax[b];
    const int64_t g = b / dq_group;
    if (dq == ORC_DQ_MEAN) {
        const float d = (float)((double)(int8_t)codes[b] * (double)steps[g]);
        return (float)((double)offsets[g] + (double)d);
    }
    if (dq == ORC_DQ_F8) return (float)(orc_e4m3_value(codes[b]) * (double)steps[g]);
    return (float)((double)codes[b] * (double)steps[g]);
}

/* Dequantize ([CSDN] 5.2 w_hat = a * c_q; 8.6 the result is in the compute
 * dtype, bf16 here): w_hat = RN_bf16(RN_fp32(a_hat * c_q)), element e taking
 * the scale of block e / block.  Output is bf16 bit patterns, [rows, cols]. */
void orc_dequantize(int64_t rows, int64_t cols, int block, const float cb[16], int dq,
                    int dq_group, const uint8_t *packed, const float *absmax,
                    const uint8_t *codes, const float *steps, const float *offsets, uint16_t *out) {
    const int64_t n = rows * cols;
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n; ++e) {
        int64_t b = e / block;
        uint8_t byte = packed[e / 2];
        int q = (e % 2 == 0) ? (byte >> 4) : (byte & 0x0f);
        float ah = block_scale(b, dq, dq_group, absmax, codes, steps, offsets);
        float w = (float)((double)ah * (double)cb[q]);
        out[e] = float_to_bf16_rne(w);
    }
}

/* Round a finite or infinite fp32 value to IEEE binary16, round to nearest
 * even, as bits.  binary16 keeps 11 significant bits; below 2^-14 its
 * spacing is fixed at 2^-24 (subnormals).  x is scaled so that the kept bits
 * are the integer part, rounded by rint (the default mode is to nearest
 * even) and scaled back, all exact in fp64; magnitudes past 65504 after
 * rounding are infinite. */
static uint16_t float_to_fp16_rne(float f) {
    double x = (double)f;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7e00u);
    x = fabs(x);
    if (isinf(x)) return (uint16_t)(sign | 0x7c00u);
    if (x == 0.0) return sign;
    int e;
    frexp(x, &e);                        /* x = m 2^e, m in [0.5, 1): leading bit 2^(e-1) */
    int q = e - 11;                      /* exponent of the last kept bit */
    if (q < -24) q = -24;                /* the subnormal spacing */
    double r = ldexp(rint(ldexp(x, -q)), q);
    if (r > 65504.0) return (uint16_t)(sign | 0x7c00u);
    if (r < ldexp(1.0, -14))             /* subnormal (or zero): mantissa in units of 2^-24 */
        return (uint16_t)(sign | (uint16_t)ldexp(r, 24));
    int er;
    double mr = frexp(r, &er);           /* r = mr 2^er; biased exponent er - 1 + 15 */
    uint16_t mant = (uint16_t)(ldexp(mr, 11) - 1024.0);
    return (uint16_t)(sign | (uint16_t)((er - 1 + 15) << 10) | mant);
}

/* Dequantize into a chosen compute dtype ([CSDN] 8.3: the dequantized
 * weights and the arithmetic are FP32, BF16 or FP16): w_hat =
 * RN_dtype(RN_fp32(a_hat * c_q)).  dtype 0 = bf16, 1 = fp16 (16-bit patterns
 * in out), 2 = fp32 (out holds fp32 values). */
void orc_dequantize_dt(int64_t rows, int64_t cols, int block, const float cb[16], int dq,
                       int dq_group, const uint8_t *packed, const float *absmax,
                       const uint8_t *codes, const float *steps, const float *offsets, int dtype,
                       void *out) {
    const int64_t n = rows * cols;
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n; ++e) {
        uint8_t byte = packed[e / 2];
        int q = (e % 2 == 0) ? (byte >> 4) : (byte & 0x0f);
        float ah = block_scale(e / block, dq, dq_group, absmax, codes, steps, offsets);
        float w = (float)((double)ah * (double)cb[q]);
        if (dtype == 2)
            ((float *)out)[e] = w;
        else if (dtype == 1)
            ((uint16_t *)out)[e] = float_to_fp16_rne(w);
        else
            ((uint16_t *)out)[e] = float_to_bf16_rne(w);
    }
}

/* binary16 bits -> double, exported so tests can pin the decoding alone. */
void orc_fp16_decode(const uint16_t *h, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = fp16_to_double(h[i]);
}

/* fp32 -> binary16 bits, exported so tests can pin the conversion alone. */
void orc_fp16_bits(const float *x, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_fp16_rne(x[i]);
}

/* ------------------------------------------------------------------------ */
/* The layer: forward and backward in fp64                                   */
/* ------------------------------------------------------------------------ */

/* Adapter input: x itself, or with pooling ([BLOG] sections 3-4) the mean of
 * each run of g consecutive input features: p[m,k'] = (1/g) sum_i x[m,k'g+i]. */
static double adapter_in(const uint16_t *X, int64_t Din, int64_t m, int64_t kp,
                         int g, int dt) {
    if (g == 1) return dec16(X[m * Din + kp], dt);
    double s = 0.0;
    for (int i = 0; i < g; ++i) s += dec16(X[m * Din + kp * g + i], dt);
    return s / (double)g;
}

/* T = adapter_in(x) . A   ->  T:[M, r]   ([BLOG] section 2; [CSDN] 12.2) */
void orc_adapter_down(const uint16_t *X, int64_t M, int64_t Din,
                      const uint16_t *A, int r, int g, double *T, int dt) {
    const int64_t Da = Din / g;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < r; ++j) {
            double s = 0.0;
            for (int64_t k = 0; k < Da; ++k)
                s += adapter_in(X, Din, m, k, g, dt) * dec16(A[k * r + j], dt);
            T[m * r + j] = s;
        }
}

/* Forward ([BLOG] section 2 W_eff = dequant(W4) + (alpha/r) A B;
 * [CSDN] 12.4 Y = X W_hat + s X A B with s = lora_alpha / r):
 *   y[m,n] = sum_k x[m,k] Wt[n,k] + s * sum_j T[m,j] B[j,n].
 * Wt is the dequantized weight ([Dout, Din]).  T may be NULL.  In every layer
 * function the 16-bit arrays (x, dY, Wt, A, B) hold bf16 (dt = 0) or fp16
 * (dt = 1) bit patterns, the compute dtype of [CSDN] 8.3; all arithmetic is
 * fp64 either way. */
void orc_forward(const uint16_t *X, int64_t M, int64_t Din, int64_t Dout,
                 const uint16_t *Wt, const uint16_t *A, const uint16_t *B,
                 int r, double alpha, int g, double *Y, double *T_out, int dt) {
    const double s = alpha / (double)r;
    double *T = (double *)malloc(sizeof(double) * (size_t)(M * r > 0 ? M * r : 1));
    orc_adapter_down(X, M, Din, A, r, g, T, dt);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < Dout; ++n) {
            double base = 0.0;
            for (int64_t k = 0; k < Din; ++k)
                base += dec16(X[m * Din + k], dt) * dec16(Wt[n * Din + k], dt);
            double ad = 0.0;
            for (int j = 0; j < r; ++j) ad += T[m * r + j] * dec16(B[(int64_t)j * Dout + n], dt);
            Y[m * Dout + n] = base + s * ad;
        }
    if (T_out) memcpy(T_out, T, sizeof(double) * (size_t)(M * r));
    free(T);
}

/* G = dY . B^T  ->  G:[M, r] */
void orc_grad_G(const uint16_t *dY, int64_t M, int64_t Dout, const uint16_t *B,
                int r, double *G, int dt) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < r; ++j) {
            double s = 0.0;
            for (int64_t n = 0; n < Dout; ++n)
                s += dec16(dY[m * Dout + n], dt) * dec16(B[(int64_t)j * Dout + n], dt);
            G[m * r + j] = s;
        }
}

/* Backward input gradient ([CSDN] 12.4: the chain rule runs through the
 * frozen base; W gets no gradient).  With y = x W + s adapter_in(x) A B:
 *   dX[m,k] = sum_n dY[m,n] Wt[n,k] + (s/g) sum_j G[m,j] A[k/g, j]. */
void orc_backward_dx(const uint16_t *dY, int64_t M, int64_t Din, int64_t Dout,
                     const uint16_t *Wt, const uint16_t *A, const uint16_t *B,
                     int r, double alpha, int g, double *dX, int dt) {
    const double s = alpha / (double)r;
    double *G = (double *)malloc(sizeof(double) * (size_t)(M * r > 0 ? M * r : 1));
    orc_grad_G(dY, M, Dout, B, r, G, dt);
    /* Each output dX[m,k] sums n = 0..Dout-1 in ascending order; the loops
     * run n outside k only so that Wt is read row by row. */
    const int64_t KC = 256;
    const int64_t nkc = (Din + KC - 1) / KC;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t c = 0; c < nkc; ++c) {
            double acc[256];
            const int64_t k0 = c * KC, k1 = k0 + KC < Din ? k0 + KC : Din;
            for (int64_t k = k0; k < k1; ++k) acc[k - k0] = 0.0;
            for (int64_t n = 0; n < Dout; ++n) {
                const double dy = dec16(dY[m * Dout + n], dt);
                for (int64_t k = k0; k < k1; ++k)
                    acc[k - k0] += dy * dec16(Wt[n * Din + k], dt);
            }
            for (int64_t k = k0; k < k1; ++k) {
                double ad = 0.0;
                for (int j = 0; j < r; ++j)
                    ad += G[m * r + j] * dec16(A[(k / g) * r + j], dt);
                dX[m * Din + k] = acc[k - k0] + s * ad / (double)g;
            }
        }
    free(G);
}

/* Backward adapter gradients:
 *   dA[k',j] = s sum_m adapter_in(x)[m,k'] G[m,j]      (dA:[Din/g, r])
 *   dB[j,n]  = s sum_m T[m,j] dY[m,n]                  (dB:[r, Dout]) */
void orc_backward_dadb(const uint16_t *X, const uint16_t *dY, int64_t M,
                       int64_t Din, int64_t Dout, const uint16_t *A,
                       const uint16_t *B, int r, double alpha, int g,
                       double *dA, double *dB, int dt) {
    const double s = alpha / (double)r;
    const int64_t Da = Din / g;
    double *G = (double *)malloc(sizeof(double) * (size_t)(M * r > 0 ? M * r : 1));
    double *T = (double *)malloc(sizeof(double) * (size_t)(M * r > 0 ? M * r : 1));
    orc_grad_G(dY, M, Dout, B, r, G, dt);
    orc_adapter_down(X, M, Din, A, r, g, T, dt);
    /* Each output sums m = 0..M-1 in ascending order; the loops run m
     * outside the output column so that x, dY are read row by row. */
    if (dA) {
        const int64_t KC = 64;
        const int64_t nkc = (Da + KC - 1) / KC;
#pragma omp parallel for schedule(dynamic)
        for (int64_t c = 0; c < nkc; ++c) {
            const int64_t k0 = c * KC, k1 = k0 + KC < Da ? k0 + KC : Da;
            for (int64_t k = k0; k < k1; ++k)
                for (int j = 0; j < r; ++j) dA[k * r + j] = 0.0;
            for (int64_t m = 0; m < M; ++m)
                for (int64_t k = k0; k < k1; ++k) {
                    const double u = adapter_in(X, Din, m, k, g, dt);
                    for (int j = 0; j < r; ++j) dA[k * r + j] += u * G[m * r + j];
                }
            for (int64_t k = k0; k < k1; ++k)
                for (int j = 0; j < r; ++j) dA[k * r + j] *= s;
        }
    }
    if (dB) {
        const int64_t NC = 1024;
        const int64_t nnc = (Dout + NC - 1) / NC;
#pragma omp parallel for collapse(2) schedule(dynamic)
        for (int j = 0; j < r; ++j)
            for (int64_t c = 0; c < nnc; ++c) {
                const int64_t n0 = c * NC, n1 = n0 + NC < Dout ? n0 + NC : Dout;
                double *row = dB + (int64_t)j * Dout;
                for (int64_t n = n0; n < n1; ++n) row[n] = 0.0;
                for (int64_t m = 0; m < M; ++m) {
                    const double t = T[m * r + j];
                    for (int64_t n = n0; n < n1; ++n) row[n] += t * dec16(dY[m * Dout + n], dt);
                }
                for (int64_t n = n0; n < n1; ++n) row[n] *= s;
            }
    }
    free(G);
    free(T);
}

/* Threads the OpenMP runtime will use for the parallel loops above. */
/* Adapter merge for inference: W_eff = dequant(W4) + s * (A . B), written in
 * the stored orientation [Dout][Din]:
 *   W_eff[n][k] = Wt[n][k] + s * sum_j A[k][j] B[j][n]               (g = 1)
 *   W_eff[n][k] = Wt[n][k] + (s/g) * sum_j A_p[k/g][j] B[j][n]       (pooled)
 * ([BLOG] section 2, W_eff = dequant(W4) + (alpha/r) A B; [CSDN] 12.10, merging
 * the adapter into the weight for deployment; [BLOG] section 5, every input of
 * a group shares the update (A_p B)/g.)  The pooled form is the one for which
 * x . W_eff^T equals the layer's forward, since pool(x) averages a group.
 * Wt is the bf16 dequantized weight; the result is exact fp64 arithmetic on it. */
void orc_merge(int64_t Din, int64_t Dout, const uint16_t *Wt, const uint16_t *A,
               const uint16_t *B, int r, double alpha, int g, double *out, int dt) {
    const double s = alpha / (double)r;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < Dout; ++n)
        for (int64_t k = 0; k < Din; ++k) {
            double ad = 0.0;
            for (int j = 0; j < r; ++j)
                ad += dec16(A[(k / g) * r + j], dt) * dec16(B[(int64_t)j * Dout + n], dt);
            out[n * Din + k] = dec16(Wt[n * Din + k], dt) + (s / (double)g) * ad;
        }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
