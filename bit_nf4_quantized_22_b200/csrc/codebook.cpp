// codebook.cpp -- step 1 of the method on the host: the 16 levels of the
// NF4 table, and of the FP4 table.
//
// "QLoRA：用4比特行李箱装下整个大模型" chapter 3 takes the levels from the
// standard normal distribution: the CDF is cut into equal-probability pieces
// and each level is a quantile Phi^-1 of that split.  The bitsandbytes article
// (CSDN) section 6.2 adds that the table is fixed (one for every block), lies
// in [-1, 1], and is built asymmetrically so that 0 is one of the levels.
//
// The formula itself did not survive on the pages.  The construction here:
// 8 positive and 7 negative levels and an exact 0.  The positive side takes
// Phi^-1 at 9 probabilities evenly spaced from `delta` down to 1/2 and drops
// the last (Phi^-1(1/2) = 0); the negative side takes 8 such probabilities,
// drops the last, and mirrors them.  Every quantile is divided by
// Phi^-1(delta), so the ends are exactly -1 and +1; the values are rounded
// once to fp32.  delta must lie in (1/2, 1): Phi^-1(1) is infinite, and at
// delta <= 1/2 the two sides would not be ordered.
//
// The inverse normal is Wichura's algorithm AS 241 (PPND16, Applied
// Statistics 37 (1988) 477-484): three rational approximations in
// q = p - 1/2 (central region) and in sqrt(-log(min(p, 1-p))) (tails),
// followed by one Halley step on Phi(x) = p, with Phi taken from the C
// library's erfc, to polish the last bits.
#include <cmath>

#include "../../include/qlora.h"

namespace {

double poly7(const double *c, double r) {
    double v = c[7];
    for (int i = 6; i >= 0; --i) v = v * r + c[i];
    return v;
}

// AS 241 coefficients, lowest order first.
const double kA[8] = {3.3871328727963666080e0, 1.3314166789178437745e+2,
                      1.9715909503065514427e+3, 1.3731693765509461125e+4,
                      4.5921953931549871457e+4, 6.7265770927008700853e+4,
                      3.3430575583588128105e+4, 2.5090809287301226727e+3};
const double kB[8] = {1.0, 4.2313330701600911252e+1, 6.8718700749205790830e+2,
                      5.3941960214247511077e+3, 2.1213794301586595867e+4,
                      3.9307895800092710610e+4, 2.8729085735721942674e+4,
                      5.2264952788528545610e+3};
const double kC[8] = {1.42343711074968357734e0, 4.63033784615654529590e0,
                      5.76949722146069140550e0, 3.64784832476320460504e0,
                      1.27045825245236838258e0, 2.41780725177450611770e-1,
                      2.27238449892691845833e-2, 7.74545014278341407640e-4};
const double kD[8] = {1.0, 2.05319162663775882187e0, 1.67638483018380384940e0,
                      6.89767334985100004550e-1, 1.48103976427480074590e-1,
                      1.51986665636164571966e-2, 5.47593808499534494600e-4,
                      1.05075007164441684324e-9};
const double kE[8] = {6.65790464350110377720e0, 5.46378491116411436990e0,
                      1.78482653991729133580e0, 2.96560571828504891230e-1,
                      2.65321895265761230930e-2, 1.24266094738807843860e-3,
                      2.71155556874348757815e-5, 2.01033439929228813265e-7};
const double kF[8] = {1.0, 5.99832206555887937690e-1, 1.36929880922735805310e-1,
                      1.48753612908506148525e-2, 7.86869131145613259100e-4,
                      1.84631831751005468180e-5, 1.42151175831644588870e-7,
                      2.04426310338993978564e-15};

// Phi^-1(p) for p in (0, 1) by AS 241.
double as241(double p) {
    const double q = p - 0.5;
    if (std::fabs(q) <= 0.425) {
        const double r = 0.180625 - q * q;
        return q * poly7(kA, r) / poly7(kB, r);
    }
    double r = std::sqrt(-std::log(q < 0 ? p : 1.0 - p));
    double x;
    if (r <= 5.0) {
        r -= 1.6;
        x = poly7(kC, r) / poly7(kD, r);
    } else {
        r -= 5.0;
        x = poly7(kE, r) / poly7(kF, r);
    }
    return q < 0 ? -x : x;
}

// Phi^-1(p), refined.  Works in the lower half, p <= 1/2, where
// Phi(x) = erfc(-x / sqrt 2) / 2 keeps full relative precision; the upper
// half follows from Phi^-1(p) = -Phi^-1(1 - p), and 1 - p is exact there.
double inv_normal(double p) {
    if (p > 0.5) return -inv_normal(1.0 - p);
    if (p == 0.5) return 0.0;
    double x = as241(p);
    // Halley's step on f(x) = Phi(x) - p: u = f / f', x -= u / (1 + x u / 2)
    // (f'' = -x f' for the normal density).
    const double e = 0.5 * std::erfc(-x * 0.70710678118654752440) - p;
    const double u = e * 2.50662827463100050242 * std::exp(0.5 * x * x);
    x -= u / (1.0 + 0.5 * x * u);
    return x;
}

}  // namespace

extern "C" int nf4_codebook(double delta, float out[16]) {
    if (!out || !(delta > 0.5 && delta < 1.0)) return QLORA_EINVAL;
    const double z = inv_normal(delta);
    // Probabilities fall from delta towards 1/2 as i grows, so the negative
    // side (i = 0..6) comes out ascending from -1, and the positive side is
    // written from i = 7 down to i = 0, ending at +1.
    double v[16];
    for (int i = 0; i < 7; ++i) v[i] = -inv_normal(delta + (0.5 - delta) * i / 7.0) / z;
    v[7] = 0.0;
    for (int i = 0; i < 8; ++i) v[15 - i] = inv_normal(delta + (0.5 - delta) * i / 8.0) / z;
    for (int i = 0; i < 16; ++i) out[i] = (float)v[i];
    return QLORA_OK;
}

// FP4 ("大模型量化从0到1（十）：bitsandbytes" 6.4-6.5 and 9.3: bitsandbytes' other
// 4-bit type is a float-style table, values not given).  The layout read for
// it is E2M1 of the OCP Microscaling formats: sign, two exponent bits with
// bias 1, one mantissa bit; exponent field 0 is subnormal (0 and 1/2).  Each
// value is divided by the largest, 6, and the 16 codes are listed in
// ascending order with -0 before +0.
extern "C" int fp4_codebook(float out[16]) {
    if (!out) return QLORA_EINVAL;
    float v[16];
    for (int code = 0; code < 16; ++code) {
        const int sign = code >> 3, e = (code >> 1) & 3, m = code & 1;
        const float mag = e ? std::ldexp(2.f + m, e - 2) : 0.5f * m;   // 2^(e-1) (1 + m/2)
        v[code] = (sign ? -mag : mag) / 6.f;
    }
    // negative codes 15..8 (largest magnitude first), then positive codes 0..7
    for (int i = 0; i < 8; ++i) {
        out[i] = v[15 - i];
        out[8 + i] = v[i];
    }
    return QLORA_OK;
}
