// quantize.cu -- blockwise NF4 quantization (+ double quantization) and
// dequantization kernels.
//
// Rule (bitsandbytes article (CSDN) section 5.2): per block of 64 weights
// a = max|w|; each weight takes the codebook index argmin_j |w/a - c_j|
// (exact arithmetic, first index on ties); two indices per byte, element 2i
// in the high nibble.  Double quantization (section 7.2): per 256 blocks,
// step f = RN32(max a / 255), code = round-half-even(a / f) in [0, 255].
#include <cmath>

#include "common.cuh"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kQuantThreads = 256;   // one thread per block, one CTA per DQ group

// The levels whose midpoint is decision threshold j: (c_j, c_{j+1}), or,
// where a level repeats (c_j == c_{j+1}, the FP4 table's -0 and +0), the next
// pair of distinct levels, so that threshold j equals threshold j + 1 and
// the repeated level's second copy is never chosen: the count of thresholds
// below w is then the first nearest level, as with distinct levels.  With no
// distinct pair above, both are +inf (a threshold never passed).
struct ThreshPairs {
    float lo[16];
    float hi[16];
};

// Tables of the fast kernel: T[bin] for 32 bins, four bits each, and the
// halved codebook midpoints h_k = (c_k + c_{k+1}) / 2 when each is exact in
// fp64 with at most 29 significant bits (then h_k * a is exact in fp64).
struct QuantBins {
    uint32_t nib[4];
    double half[15];
};

__device__ __forceinline__ float next_up(float x) {
    const uint32_t u = __float_as_uint(x);
    if ((u & 0x7fffffffu) == 0u) return __uint_as_float(1u);   // +-0 -> smallest subnormal
    return __uint_as_float(x > 0.f ? u + 1u : u - 1u);
}

// tau such that, for every fp32 w,  w >= tau  <=>  w > (c_lo + c_hi) * a / 2
// exactly.  c*a is an exact fp64 product of two fp32 values; TwoSum gives the
// midpoint sum as S + err exactly.  tau = smallest fp32 >= S/2, moved up one
// ulp when S/2 is itself an fp32 value and err >= 0 (then the exact midpoint
// is >= tau and w must exceed it).  In every other case the fp64 residue is
// far below the fp32 spacing, so no fp32 value lies between the midpoint and
// tau.
__device__ __forceinline__ float exact_threshold(float c_lo, float c_hi, float a) {
    const double p1 = __dmul_rn((double)c_lo, (double)a);
    const double p2 = __dmul_rn((double)c_hi, (double)a);
    const double s = __dadd_rn(p1, p2);
    const double bb = __dsub_rn(s, p1);
    const double err = __dadd_rn(__dsub_rn(p1, __dsub_rn(s, bb)), __dsub_rn(p2, bb));
    const double half = s * 0.5;
    float tau = __double2float_ru(half);
    if ((double)tau == half && err >= 0.0) tau = next_up(tau);
    return tau;
}

// Branch-free binary search over 15 sorted thresholds: the number of j with
// w >= t[j], i.e. the index of the nearest level.
__device__ __forceinline__ uint32_t level_index(float w, const float t[15]) {
    const bool b3 = w >= t[7];
    const float t2 = b3 ? t[11] : t[3];
    const bool b2 = w >= t2;
    const float t1 = b3 ? (b2 ? t[13] : t[9]) : (b2 ? t[5] : t[1]);
    const bool b1 = w >= t1;
    const float t0 = b3 ? (b2 ? (b1 ? t[14] : t[12]) : (b1 ? t[10] : t[8]))
                        : (b2 ? (b1 ? t[6] : t[4]) : (b1 ? t[2] : t[0]));
    const bool b0 = w >= t0;
    return (uint32_t(b3) << 3) | (uint32_t(b2) << 2) | (uint32_t(b1) << 1) | uint32_t(b0);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Double-quant code RNE(d / f) clamped to [-top, top] (d >= 0 for the
// unsigned and signed absmax codes, either sign for the mean-offset code).
// For f in [2^-100, 2^100]: an approximate quotient c (within one of the
// answer, as |d / f| <= 256 and the approximation errs by < 2^-14), then the
// signs of d - (c +- 1/2) f from one fma each -- a correctly rounded fma has
// the sign of the exact value and is zero only when it is -- decide c - 1, c
// or c + 1, ties to even.  Other f: the quotient in fp64, whose rint is exact
// for these ratios of fp32 values.
__device__ __forceinline__ int dq_code(float d, float f, int top) {
    if (!(f > 0.f)) return 0;
    float c;
    if (f >= 0x1p-100f && f <= 0x1p100f) {
        c = rintf(__fmul_rn(d, rcp_approx(f)));
        const float hi = fmaf(-(c + 0.5f), f, d);
        const float lo = fmaf(-(c - 0.5f), f, d);
        const bool odd = ((int)c & 1) != 0;
        if (hi > 0.f || (hi == 0.f && odd))
            c += 1.f;
        else if (lo < 0.f || (lo == 0.f && odd))
            c -= 1.f;
    } else {
        c = (float)rint(__ddiv_rn((double)d, (double)f));
    }
    return (int)fminf(fmaxf(c, -(float)top), (float)top);
}

// The E4M3 code nearest to x >= 0 (QLORA_DQ_F8): ties to the even code, 448
// (code 0x7E) for x >= 448.  Below 2^-6 the subnormal code is RNE(x * 2^9)
// (a power-of-two scaling, exact; 8 is also the smallest normal's code); above,
// the fp32 mantissa is rounded to 3 bits, the carry of m = 8 moving into the
// exponent field.
__device__ __forceinline__ uint32_t e4m3_encode(float x) {
    if (!(x > 0.f)) return 0u;
    if (x >= 448.f) return 0x7Eu;
    if (x < 0x1p-6f) return (uint32_t)rintf(__fmul_rn(x, 512.f));
    const uint32_t u = __float_as_uint(x);
    const uint32_t mant = u & 0x7FFFFFu, rem = mant & 0xFFFFFu;
    uint32_t q = mant >> 20;
    q += (rem > 0x80000u || (rem == 0x80000u && (q & 1u))) ? 1u : 0u;
    const uint32_t code = (((u >> 23) - 120u) << 3) + q;
    return code > 0x7Eu ? 0x7Eu : code;
}

// Double quantization of one group of first-level scales, one per thread of
// the CTA (a, valid for the first nvalid threads): writes the step, the
// codes and, for the mean-offset code, the group mean (the rules of
// QLORA_DQ_U8 / _S8 / _MEAN in qlora.h).  s_a: the CTA's shared buffer of
// kThreads floats; warp_max: kThreads / 32 floats; s_mu: one float.
template <int kThreads>
__device__ __forceinline__ void dq_group_encode(float a, bool valid, int nvalid, int dq, float *s_a,
                                                float *warp_max, float *s_mu, uint8_t *code_out,
                                                float *step_out, float *mean_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float v = valid ? a : 0.f, mu = 0.f;
    if (dq == QLORA_DQ_MEAN) {
        s_a[threadIdx.x] = v;
        __syncthreads();
        if (threadIdx.x == 0) {   // the fp64 sum in block order, then one division and one rounding
            double sum = 0.0;
            for (int i = 0; i < nvalid; ++i) sum = __dadd_rn(sum, (double)s_a[i]);
            *s_mu = __double2float_rn(__ddiv_rn(sum, (double)nvalid));
        }
        __syncthreads();
        mu = *s_mu;
        v = valid ? fabsf(__fsub_rn(a, mu)) : 0.f;
    }
    float m = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) warp_max[warp] = m;
    __syncthreads();
    float gm = warp_max[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) gm = fmaxf(gm, warp_max[i]);
    const int top = dq == QLORA_DQ_U8 ? 255 : 127;
    const float f = __fdiv_rn(gm, dq == QLORA_DQ_F8 ? 448.f : (float)top);
    if (threadIdx.x == 0) {
        *step_out = f;
        if (dq == QLORA_DQ_MEAN) *mean_out = mu;
    }
    if (valid) {
        if (dq == QLORA_DQ_F8) {
            *code_out = (uint8_t)(f > 0.f ? e4m3_encode(__fdiv_rn(a, f)) : 0u);
        } else {
            const float d = dq == QLORA_DQ_MEAN ? __fsub_rn(a, mu) : a;
            *code_out = (uint8_t)(int8_t)dq_code(d, f, top);
        }
    }
}

// One CTA per double-quant group of 256 blocks (64 KB of fp32 weights).
// The group is brought into shared memory by two TMA tile loads (columns
// 0-31 and 32-63 of the [nb, 64] view, 128-byte swizzle), so the DRAM stream
// is sequential and thread t -- owning block b0 + t -- reads its row with
// 16-byte loads that hit 8 different bank groups per 8 threads.
constexpr int kQuantSmem = 2 * 256 * 128 + 1024;

__global__ void __launch_bounds__(kQuantThreads, 2)
k_nf4_quantize(const __grid_constant__ CUtensorMap tW, int64_t nb, ThreshPairs tp, int zero_idx,
               int dq, uint8_t *__restrict__ packed, float *__restrict__ absmax,
               uint8_t *__restrict__ codes, float *__restrict__ steps, float *__restrict__ means,
               uint32_t *__restrict__ status) {
    extern __shared__ __align__(1024) uint8_t qsm_raw[];
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ int abort_flag;
    __shared__ float warp_max[kQuantThreads / 32];
    const uint32_t raw = smem_u32(qsm_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    const uint32_t bar = smem_u32(&bar_storage);
    const int64_t b0 = (int64_t)blockIdx.x * kQuantThreads;
    const int64_t b = b0 + threadIdx.x;
    const bool valid = b < nb;

    if (threadIdx.x == 0) {
        tc::mbar_init(bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        tc::fence_proxy_async();
        tc::mbar_expect_tx(bar, 2 * 256 * 128);
        tc::tma_load_2d(sbase, &tW, 0, (int)b0, bar);
        tc::tma_load_2d(sbase + 256 * 128, &tW, 32, (int)b0, bar);
    }
    __syncthreads();
    const bool arrived = tc::mbar_wait(bar, 0, &abort_flag);
    if (!arrived && status) atomicOr(status, QLORA_STATUS_TIMEOUT);

    float w[64];
    const uint32_t row = threadIdx.x, sw = row & 7;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 v = tc::lds128(sbase + h * 256 * 128 + row * 128 + ((c ^ sw) << 4));
            w[32 * h + 4 * c + 0] = __uint_as_float(v.x);
            w[32 * h + 4 * c + 1] = __uint_as_float(v.y);
            w[32 * h + 4 * c + 2] = __uint_as_float(v.z);
            w[32 * h + 4 * c + 3] = __uint_as_float(v.w);
        }
    float a = 0.f;
    uint32_t bad = 0;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        a = fmaxf(a, fabsf(w[i]));
        bad |= ((__float_as_uint(w[i]) & 0x7f800000u) == 0x7f800000u);
    }
    if (valid && bad && status) atomicOr(status, QLORA_STATUS_NONFINITE);
    if (!valid) a = 0.f;

    if (valid) {
        uint32_t out[8];
        if (a == 0.f) {
            const uint32_t z = (uint32_t)zero_idx * 0x11111111u;
#pragma unroll
            for (int i = 0; i < 8; ++i) out[i] = z;
        } else {
            float t[15];
#pragma unroll
            for (int j = 0; j < 15; ++j) t[j] = exact_threshold(tp.lo[j], tp.hi[j], a);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t word = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t q0 = level_index(w[8 * i + 2 * k], t);
                    const uint32_t q1 = level_index(w[8 * i + 2 * k + 1], t);
                    word |= ((q0 << 4) | q1) << (8 * k);
                }
                out[i] = word;
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(packed + b * 32);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        if (!dq) absmax[b] = a;
    }

    if (dq) {
        __shared__ float s_grp[kQuantThreads];
        __shared__ float s_mu;
        const int nvalid = (int)(nb - (int64_t)blockIdx.x * kQuantThreads < kQuantThreads
                                     ? nb - (int64_t)blockIdx.x * kQuantThreads : kQuantThreads);
        uint8_t code = 0;
        dq_group_encode<kQuantThreads>(a, valid, nvalid, dq, s_grp, warp_max, &s_mu, &code,
                                       steps + blockIdx.x, means + blockIdx.x);
        if (valid) codes[b] = code;
    }
}

// ------------------------------------------------------------------ fast path
// One CTA per group of 256 blocks.  Each warp reads its weights straight
// from global memory with 16-byte streaming loads, the four passes of a
// quarter issued together; four CTAs per SM keep enough loads in flight (in
// measurements this beat staging the group through shared memory with bulk
// copies).  A warp takes two blocks at a
// time: lanes 0-15 the first, 16-31 the second, V consecutive weights per
// lane (V = 4 for blocks of 64, 2 for blocks of 32).  Lane j of a half also holds the exact threshold tau_j of its block
// (lane 15: +inf).  A weight's index then costs one table lookup and one
// exact compare instead of a four-level search:
//   bin = RN(K * (w * RN(1/a)) + 16)          (approximate)
//   j~  = T[bin]                              (thresholds surely below the bin)
//   q   = j~ + (w >= tau_{j~})
// The host builds T for the codebook and proves that every bin, widened by a
// margin far above the error of the approximate w/a, holds at most one
// threshold; only then is this kernel used, and the one compare is exact.
// Blocks with a = 0, a tiny or huge a, or a non-finite weight take the
// branch-free search (warp-uniform branch).
// Every lane addresses its weights and packed bytes from two base pointers
// with constant offsets, and a full group (256 blocks, all but the last one)
// runs a copy of the loop without the per-block range tests: about 10% fewer
// issued instructions on this issue-bound kernel.
template <bool B> struct BoolTag { static constexpr bool value = B; };
constexpr float kBinK = 15.49f;
constexpr float kBinC = 12582928.0f;   // 1.5 * 2^23 + 16: the low 5 bits of the sum are the bin
constexpr int kQfThreads = 256;
constexpr int kQfSmem = 0;

// V weights per lane: 4 for blocks of 64, 2 for blocks of 32 (16 lanes per block either way).
template <bool kExactHalf, int V>
__global__ void __launch_bounds__(kQfThreads, 4)
k_nf4_quantize_fast(const float *__restrict__ W, int64_t nb, ThreshPairs tp, QuantBins bins,
                    int zero_idx, int dq, uint8_t *__restrict__ packed,
                    float *__restrict__ absmax, uint8_t *__restrict__ codes,
                    float *__restrict__ steps, float *__restrict__ means, uint32_t *__restrict__ status) {
    __shared__ float s_a[kQfThreads];
    __shared__ float s_lo[16], s_hi[16];
    __shared__ double s_half[16];
    __shared__ uint32_t s_lut[32];
    __shared__ float warp_max[kQfThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t b0 = (int64_t)blockIdx.x * 256;
    const int nblk = (int)(nb - b0 < 256 ? nb - b0 : 256);
    s_a[threadIdx.x] = 0.f;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) s_lo[j] = tp.lo[j], s_hi[j] = tp.hi[j];
#pragma unroll
        for (int j = 0; j < 15; ++j) s_half[j] = bins.half[j];
#pragma unroll
        for (int i = 0; i < 32; ++i) s_lut[i] = (bins.nib[i >> 3] >> (4 * (i & 7))) & 15u;
    }
    __syncthreads();
    const int j = lane & 15, half = lane >> 4;
    const float c_lo = s_lo[j < 15 ? j : 14], c_hi = s_hi[j < 15 ? j : 14];
    const double hk = s_half[j < 15 ? j : 14];
    const uint32_t lut = s_lut[lane];
    uint32_t bad_any = 0;
    // this lane's weights and packed bytes of block bl = 64 c + 16 i + 2 warp + half
    // are at constant offsets (c, i) from these
    const float *wlane = W + (b0 + 2 * warp + half) * (16 * V) + V * j;
    uint8_t *plane = packed + (b0 + 2 * warp + half) * (8 * V) + (V / 2) * j;
    auto run = [&](auto tag) {
        constexpr bool FULL = decltype(tag)::value;
        float nxt[4][V];
        auto load_quarter = [&](int c, float (&dst)[4][V]) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int bl = 64 * c + 16 * i + 2 * warp + half;
                const float *src = wlane + (64 * c + 16 * i) * (16 * V);
                const bool ld = FULL || bl < nblk;
                if (V == 4) {
                    const float4 v = ld ? __ldcs(reinterpret_cast<const float4 *>(src))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    dst[i][0] = v.x, dst[i][1] = v.y, dst[i][2] = v.z, dst[i][3] = v.w;
                } else {
                    const float2 v = ld ? __ldcs(reinterpret_cast<const float2 *>(src)) : make_float2(0.f, 0.f);
                    dst[i][0] = v.x, dst[i][1] = v.y;
                }
            }
        };
        load_quarter(0, nxt);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            if (!FULL && 64 * c >= nblk) break;
            float pre[4][V];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < V; ++k) pre[i][k] = nxt[i][k];
            if (c + 1 < 4 && (FULL || 64 * (c + 1) < nblk)) load_quarter(c + 1, nxt);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int bl = 64 * c + 16 * i + 2 * warp + half;   // block within the group
                const bool valid = FULL || bl < nblk;
                float w[V];
#pragma unroll
                for (int k = 0; k < V; ++k) w[k] = pre[i][k];
                // max |w|, NaN-propagating: a NaN or Inf weight makes a non-finite scale
                float fm = 0.f;
#pragma unroll
                for (int k = 0; k < V; ++k) asm("max.NaN.f32 %0, %1, %2;" : "=f"(fm) : "f"(fm), "f"(fabsf(w[k])));
                const uint32_t m = __float_as_uint(fm);
                const uint32_t m0 = __reduce_max_sync(0xffffffffu, half ? 0u : m);
                const uint32_t m1 = __reduce_max_sync(0xffffffffu, half ? m : 0u);
                const uint32_t ab = half ? m1 : m0;
                const float a = __uint_as_float(ab);
                const bool bad = ab >= 0x7f800000u;
                // tau_j: the smallest fp32 above the exact midpoint h_j * a
                float tau;
                if (kExactHalf)
                    tau = next_up(__double2float_rd(__dmul_rn(hk, (double)a)));
                else
                    tau = exact_threshold(c_lo, c_hi, a);
                if (j == 15) tau = __uint_as_float(0x7f800000u);
                const bool fast = ab >= 0x0d800000u && ab <= 0x71800000u;   // 2^-100 <= a <= 2^100
                uint32_t qv[V];
                if (__all_sync(0xffffffffu, fast || !valid)) {
                    const float kr = __fmul_rn(kBinK, rcp_approx(a));   // K / a, relative error < 2^-22
#pragma unroll
                    for (int k = 0; k < V; ++k) {
                        const float y = fmaf(w[k], kr, kBinC);
                        const uint32_t jt = __shfl_sync(0xffffffffu, lut, (int)__float_as_uint(y));
                        const float t = __shfl_sync(0xffffffffu, tau, (int)jt, 16);
                        qv[k] = jt + (w[k] >= t ? 1u : 0u);
                    }
                } else {
                    float t[15];
#pragma unroll
                    for (int k = 0; k < 15; ++k) t[k] = __shfl_sync(0xffffffffu, tau, k, 16);
#pragma unroll
                    for (int k = 0; k < V; ++k) qv[k] = ab == 0u ? (uint32_t)zero_idx : level_index(w[k], t);
                }
                if (valid) {
                    // weights V j .. V j + V-1 -> bytes (V/2) j ..; element 2i in the high nibble
                    uint8_t *dstp = plane + (64 * c + 16 * i) * (8 * V);
                    if (V == 4) {
                        const uint32_t v = (qv[2 % V] * 16u + qv[3 % V]) * 256u + (qv[0] * 16u + qv[1]);
                        *reinterpret_cast<uint16_t *>(dstp) = (uint16_t)v;
                    } else {
                        *dstp = (uint8_t)(qv[1] | (qv[0] << 4));
                    }
                    if (j == 0) {
                        s_a[bl] = a;
                        if (!dq) absmax[b0 + bl] = a;
                        bad_any |= bad;
                    }
                }
            }
        }
    };
    if (nblk == 256) run(BoolTag<true>{});
    else run(BoolTag<false>{});
    if (bad_any && status) atomicOr(status, QLORA_STATUS_NONFINITE);
    if (dq) {
        __shared__ float s_mu;
        __syncthreads();
        const bool valid = threadIdx.x < nblk;
        const float a = s_a[threadIdx.x];
        __syncthreads();   // s_a is reused as the encoder's buffer
        uint8_t code = 0;
        dq_group_encode<kQfThreads>(a, valid, nblk, dq, s_a, warp_max, &s_mu, &code,
                                    steps + blockIdx.x, means + blockIdx.x);
        if (valid) codes[b0 + threadIdx.x] = code;
    }
}

// ------------------------------------------------------------------ other block sizes
// Blocks of B = 32 V weights (V = 1, 4, 8: blocks of 32, 128, 256; the
// article's section 5.1 trade of scale resolution against metadata).  One
// CTA per double-quant group of 256 blocks; warp w takes blocks w, w + 8, ...
// of the group, one whole block per warp with V weights per lane, four
// blocks' loads issued together (for V <= 4 the next four blocks' loads are
// issued before these four are decided; a full group runs a copy of the loop
// without range tests).  The decision per weight is the fast
// kernel's (bin table, one exact compare against tau_j held by lane j) when
// the table is usable and a lies in [2^-100, 2^100], else the branch-free
// search; packing, absmax and double quantization as in the other kernels.
//   V = 1: lane l holds weight l; bytes are paired across lanes by shuffles.
//   V = 4: lane l holds weights 4l .. 4l+3 (bytes 2l, 2l+1).
//   V = 8: lane l holds weights 4l .. 4l+3 and 128 + 4l .. 131 + 4l.
constexpr int kQbThreads = 256, kQbUnroll = 4;

template <int V, bool kExactHalf>
__global__ void __launch_bounds__(kQbThreads)
k_nf4_quantize_blk(const float *__restrict__ W, int64_t nb, ThreshPairs tp, QuantBins bins, bool use_bins,
                   int zero_idx, int dq, uint8_t *__restrict__ packed, float *__restrict__ absmax,
                   uint8_t *__restrict__ codes, float *__restrict__ steps, float *__restrict__ means,
                   uint32_t *__restrict__ status) {
    constexpr int B = 32 * V;
    __shared__ float s_a[kQbThreads];
    __shared__ float s_lo[16], s_hi[16];
    __shared__ double s_half[16];
    __shared__ uint32_t s_lut[32];
    __shared__ float warp_max[kQbThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t b0 = (int64_t)blockIdx.x * 256;
    const int nblk = (int)(nb - b0 < 256 ? nb - b0 : 256);
    s_a[threadIdx.x] = 0.f;
    if (threadIdx.x == 0) {   // constant indices keep the parameters out of local memory
#pragma unroll
        for (int j = 0; j < 16; ++j) s_lo[j] = tp.lo[j], s_hi[j] = tp.hi[j];
#pragma unroll
        for (int j = 0; j < 15; ++j) s_half[j] = bins.half[j];
#pragma unroll
        for (int i = 0; i < 32; ++i) s_lut[i] = (bins.nib[i >> 3] >> (4 * (i & 7))) & 15u;
    }
    __syncthreads();
    const int j = lane < 15 ? lane : 14;
    const float c_lo = s_lo[j], c_hi = s_hi[j];
    const double hk = s_half[j];
    const uint32_t lut = s_lut[lane];
    uint32_t bad_any = 0;
    auto run = [&](auto tag) {
        constexpr bool FULL = decltype(tag)::value;
        constexpr int NC = 256 / (8 * kQbUnroll);
        float nxt[kQbUnroll][V];
        auto load_chunk = [&](int c, float (&w)[kQbUnroll][V]) {
#pragma unroll
            for (int i = 0; i < kQbUnroll; ++i) {
                const int bl = 8 * (kQbUnroll * c + i) + warp;
                const float *src = W + (b0 + bl) * B;
                if (FULL || bl < nblk) {
                    if (V == 1) {
                        w[i][0] = __ldcs(src + lane);
                    } else {
#pragma unroll
                        for (int h = 0; h < V / 4; ++h) {
                            const float4 v = __ldcs(reinterpret_cast<const float4 *>(src + 128 * h) + lane);
                            w[i][4 * h] = v.x, w[i][4 * h + 1] = v.y, w[i][4 * h + 2] = v.z, w[i][4 * h + 3] = v.w;
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < V; ++k) w[i][k] = 0.f;
                }
            }
        };
        load_chunk(0, nxt);
#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
            if (!FULL && 8 * kQbUnroll * c >= nblk) break;
            float w[kQbUnroll][V];
#pragma unroll
            for (int i = 0; i < kQbUnroll; ++i)
#pragma unroll
                for (int k = 0; k < V; ++k) w[i][k] = nxt[i][k];
            if (c + 1 < NC && (FULL || 8 * kQbUnroll * (c + 1) < nblk)) load_chunk(c + 1, nxt);
#pragma unroll
            for (int i = 0; i < kQbUnroll; ++i) {
                const int bl = 8 * (kQbUnroll * c + i) + warp;
                if (!FULL && bl >= nblk) break;                  // warp-uniform
                // max |w| on the bit patterns: NaN and Inf sort above every finite value
                uint32_t m = 0;
#pragma unroll
                for (int k = 0; k < V; ++k) m = max(m, __float_as_uint(w[i][k]) & 0x7fffffffu);
                const uint32_t ab = __reduce_max_sync(0xffffffffu, m);
                const float a = __uint_as_float(ab);
                float tau = kExactHalf ? next_up(__double2float_rd(__dmul_rn(hk, (double)a)))
                                       : exact_threshold(c_lo, c_hi, a);
                if (lane >= 15) tau = __uint_as_float(0x7f800000u);
                const bool fast = use_bins && ab >= 0x0d800000u && ab <= 0x71800000u;   // warp-uniform
                uint32_t qv[V];
                if (fast) {
                    const float kr = __fmul_rn(kBinK, rcp_approx(a));
#pragma unroll
                    for (int k = 0; k < V; ++k) {
                        const float y = fmaf(w[i][k], kr, kBinC);
                        const uint32_t jt = __shfl_sync(0xffffffffu, lut, (int)__float_as_uint(y));
                        const float t = __shfl_sync(0xffffffffu, tau, (int)jt);
                        qv[k] = jt + (w[i][k] >= t ? 1u : 0u);
                    }
                } else {
                    float t[15];
#pragma unroll
                    for (int k = 0; k < 15; ++k) t[k] = __shfl_sync(0xffffffffu, tau, k);
#pragma unroll
                    for (int k = 0; k < V; ++k) qv[k] = ab == 0u ? (uint32_t)zero_idx : level_index(w[i][k], t);
                }
                uint8_t *dst = packed + (b0 + bl) * (B / 2);
                if (V == 1) {
                    // even lane 2i: byte i = (q_2i << 4) | q_2i+1; lane 8k gathers bytes 4k .. 4k+3
                    const uint32_t nx = __shfl_down_sync(0xffffffffu, qv[0], 1);
                    const uint32_t byte = ((qv[0] << 4) | nx) & 0xffu;
                    const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 2);
                    const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 4);
                    const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 6);
                    if ((lane & 7) == 0)
                        *reinterpret_cast<uint32_t *>(dst + lane / 2) = byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
                } else {
#pragma unroll
                    for (int h = 0; h < V / 4; ++h) {
                        const uint32_t v = qv[4 * h + 1] | (qv[4 * h] << 4) | (qv[4 * h + 3] << 8) | (qv[4 * h + 2] << 12);
                        *reinterpret_cast<uint16_t *>(dst + 64 * h + 2 * lane) = (uint16_t)v;
                    }
                }
                if (lane == 0) {
                    s_a[bl] = a;
                    if (!dq) absmax[b0 + bl] = a;
                    bad_any |= ab >= 0x7f800000u;
                }
            }
        }
    };
    // blocks of 256: four blocks' loads (8 per lane) already keep enough bytes in
    // flight; loading the next four ahead measured slower
    if (V == 8) {
        for (int c = 0; 8 * kQbUnroll * c < nblk; ++c) {
            float w[kQbUnroll][V];
#pragma unroll
            for (int i = 0; i < kQbUnroll; ++i) {
                const int bl = 8 * (kQbUnroll * c + i) + warp;
                const float *src = W + (b0 + bl) * B;
                if (bl < nblk) {
                    if (V == 1) {
                        w[i][0] = __ldcs(src + lane);
                    } else {
#pragma unroll
                        for (int h = 0; h < V / 4; ++h) {
                            const float4 v = __ldcs(reinterpret_cast<const float4 *>(src + 128 * h) + lane);
                            w[i][4 * h] = v.x, w[i][4 * h + 1] = v.y, w[i][4 * h + 2] = v.z, w[i][4 * h + 3] = v.w;
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < V; ++k) w[i][k] = 0.f;
                }
            }
#pragma unroll
            for (int i = 0; i < kQbUnroll; ++i) {
                const int bl = 8 * (kQbUnroll * c + i) + warp;
                if (bl >= nblk) break;                           // warp-uniform
                // max |w| on the bit patterns: NaN and Inf sort above every finite value
                uint32_t m = 0;
#pragma unroll
                for (int k = 0; k < V; ++k) m = max(m, __float_as_uint(w[i][k]) & 0x7fffffffu);
                const uint32_t ab = __reduce_max_sync(0xffffffffu, m);
                const float a = __uint_as_float(ab);
                float tau = kExactHalf ? next_up(__double2float_rd(__dmul_rn(hk, (double)a)))
                                       : exact_threshold(c_lo, c_hi, a);
                if (lane >= 15) tau = __uint_as_float(0x7f800000u);
                const bool fast = use_bins && ab >= 0x0d800000u && ab <= 0x71800000u;   // warp-uniform
                uint32_t qv[V];
                if (fast) {
                    const float kr = __fmul_rn(kBinK, rcp_approx(a));
#pragma unroll
                    for (int k = 0; k < V; ++k) {
                        const float y = fmaf(w[i][k], kr, kBinC);
                        const uint32_t jt = __shfl_sync(0xffffffffu, lut, (int)__float_as_uint(y));
                        const float t = __shfl_sync(0xffffffffu, tau, (int)jt);
                        qv[k] = jt + (w[i][k] >= t ? 1u : 0u);
                    }
                } else {
                    float t[15];
#pragma unroll
                    for (int k = 0; k < 15; ++k) t[k] = __shfl_sync(0xffffffffu, tau, k);
#pragma unroll
                    for (int k = 0; k < V; ++k) qv[k] = ab == 0u ? (uint32_t)zero_idx : level_index(w[i][k], t);
                }
                uint8_t *dst = packed + (b0 + bl) * (B / 2);
                if (V == 1) {
                    // even lane 2i: byte i = (q_2i << 4) | q_2i+1; lane 8k gathers bytes 4k .. 4k+3
                    const uint32_t nx = __shfl_down_sync(0xffffffffu, qv[0], 1);
                    const uint32_t byte = ((qv[0] << 4) | nx) & 0xffu;
                    const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 2);
                    const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 4);
                    const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 6);
                    if ((lane & 7) == 0)
                        *reinterpret_cast<uint32_t *>(dst + lane / 2) = byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
                } else {
#pragma unroll
                    for (int h = 0; h < V / 4; ++h) {
                        const uint32_t v = qv[4 * h + 1] | (qv[4 * h] << 4) | (qv[4 * h + 3] << 8) | (qv[4 * h + 2] << 12);
                        *reinterpret_cast<uint16_t *>(dst + 64 * h + 2 * lane) = (uint16_t)v;
                    }
                }
                if (lane == 0) {
                    s_a[bl] = a;
                    if (!dq) absmax[b0 + bl] = a;
                    bad_any |= ab >= 0x7f800000u;
                }
            }
        }
    } else if (nblk == 256) {
        run(BoolTag<true>{});
    } else {
        run(BoolTag<false>{});
    }
    if (bad_any && status) atomicOr(status, QLORA_STATUS_NONFINITE);
    if (dq) {
        __shared__ float s_mu;
        __syncthreads();
        const float a = s_a[threadIdx.x];
        __syncthreads();   // s_a is reused as the encoder's buffer
        uint8_t code = 0;
        dq_group_encode<kQbThreads>(a, threadIdx.x < nblk, nblk, dq, s_a, warp_max, &s_mu, &code,
                                    steps + blockIdx.x, means + blockIdx.x);
        if (threadIdx.x < nblk) codes[b0 + threadIdx.x] = code;
    }
}

// Dequantize blocks of any supported size: a thread decodes 16 consecutive
// elements (two packed words, always inside one block) through the per-block
// product table; grid-stride over the weight.
__global__ void __launch_bounds__(256)
k_nf4_dequantize_blk(const uint8_t *__restrict__ packed, ScaleSrc sc, int64_t n16, int log2_b16,
                     Codebook cb, uint16_t *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float ah = load_scale(sc, i >> log2_b16);
        ProdTable tab;
        build_table(ah, cb, tab);
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(packed) + i);
        uint32_t o0[4], o1[4];
        decode8(w.x, tab, o0);
        decode8(w.y, tab, o1);
        uint4 *dst = reinterpret_cast<uint4 *>(out + 16 * i);
        dst[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
        dst[1] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
    }
}

// Dequantize into fp16: the per-block product table of binary16 patterns
// RN_fp16(RN32(a_hat * c_j)) (IEEE rounding of each half, subnormals kept),
// decoded by the same byte permutes as the bf16 table; 16 elements a thread.
__global__ void __launch_bounds__(256)
k_nf4_dequantize_f16(const uint8_t *__restrict__ packed, ScaleSrc sc, int64_t n16, int log2_b16,
                     Codebook cb, uint16_t *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float ah = load_scale(sc, i >> log2_b16);
        uint32_t p[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const __half2 h = __floats2half2_rn(__fmul_rn(ah, cb.c[2 * k]), __fmul_rn(ah, cb.c[2 * k + 1]));
            p[k] = *reinterpret_cast<const uint32_t *>(&h);
        }
        ProdTable tab;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            tab.lo[k] = __byte_perm(p[2 * k], p[2 * k + 1], 0x6420);
            tab.hi[k] = __byte_perm(p[2 * k], p[2 * k + 1], 0x7531);
        }
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(packed) + i);
        uint32_t o0[4], o1[4];
        decode8(w.x, tab, o0);
        decode8(w.y, tab, o1);
        uint4 *dst = reinterpret_cast<uint4 *>(out + 16 * i);
        dst[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
        dst[1] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
    }
}

// Dequantize into fp32: RN32(a_hat * c_q) itself; 8 elements (one packed
// word) a thread, the codebook in shared memory.
__global__ void __launch_bounds__(256)
k_nf4_dequantize_f32(const uint8_t *__restrict__ packed, ScaleSrc sc, int64_t n8, int log2_b8,
                     Codebook cb, float *__restrict__ out) {
    __shared__ float cbs[16];
    if (threadIdx.x == 0) {   // constant indices keep the parameter out of local memory
#pragma unroll
        for (int j = 0; j < 16; ++j) cbs[j] = cb.c[j];
    }
    __syncthreads();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float ah = load_scale(sc, i >> log2_b8);
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(packed) + i);
        float v[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // byte k: element 2k in the high nibble
            const uint32_t byte = (w >> (8 * k)) & 0xffu;
            v[2 * k] = __fmul_rn(ah, cbs[byte >> 4]);
            v[2 * k + 1] = __fmul_rn(ah, cbs[byte & 15]);
        }
        float4 *dst = reinterpret_cast<float4 *>(out + 8 * i);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// Dequantize: 4 threads per block; thread i of the 4 owns packed bytes
// [4i, 4i+4) and [16+4i, 16+4i+4) of its block, i.e. output elements
// [8i, 8i+8) and [32+8i, 32+8i+8), so each group of 4 threads reads 16
// contiguous bytes and writes 64 contiguous bytes per instruction.
__global__ void __launch_bounds__(256)
k_nf4_dequantize(const uint8_t *__restrict__ packed, ScaleSrc sc, int64_t nb, Codebook cb,
                 uint16_t *__restrict__ out) {
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = gt >> 2;
    const int part = (int)(gt & 3);
    if (b >= nb) return;
    const float ah = load_scale(sc, b);
    ProdTable tab;
    build_table(ah, cb, tab);
    const uint32_t *src = reinterpret_cast<const uint32_t *>(packed + b * 32);
    const uint32_t w0 = __ldg(src + part);
    const uint32_t w1 = __ldg(src + 4 + part);
    uint32_t o0[4], o1[4];
    decode8(w0, tab, o0);
    decode8(w1, tab, o1);
    uint4 *dst = reinterpret_cast<uint4 *>(out + b * 64);
    dst[part] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
    dst[4 + part] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
}

}  // namespace

ThreshPairs make_pairs(const Codebook &cb) {
    ThreshPairs tp{};
    for (int j = 0; j < 15; ++j) {
        int k = j;
        while (k < 15 && cb.c[k] == cb.c[k + 1]) ++k;
        tp.lo[j] = k < 15 ? cb.c[k] : INFINITY;
        tp.hi[j] = k < 15 ? cb.c[k + 1] : INFINITY;
    }
    tp.lo[15] = tp.hi[15] = INFINITY;
    return tp;
}

// T[bin] of the fast kernel for this codebook, or false when some bin,
// widened by the margin, holds two thresholds (levels closer than about
// 1/K apart): bin i holds every u with RN(K u + 16) = i.  The margin 2^-18
// bounds both the error of w * RN(1/a) against w/a (< 2^-22 for |w| <= a) and
// the distance of an exact threshold tau_k / a from its midpoint m_k.
bool make_quant_bins(const ThreshPairs &tp, QuantBins *out) {
    const double K = (double)kBinK, margin = std::ldexp(1.0, -18);
    double m[15];
    for (int k = 0; k < 15; ++k) m[k] = ((double)tp.lo[k] + (double)tp.hi[k]) * 0.5;
    QuantBins qb{};
    for (int i = 0; i < 32; ++i) {
        const double lo = (i - 16.5) / K - margin, hi = (i - 15.5) / K + margin;
        int below = 0, inside = 0;
        for (int k = 0; k < 15; ++k) {
            if (m[k] + margin < lo)
                ++below;
            else if (m[k] - margin <= hi)
                ++inside;
        }
        if (inside > 1) return false;
        qb.nib[i >> 3] |= (uint32_t)below << (4 * (i & 7));
    }
    *out = qb;
    return true;
}

// Fills bins->half; true when every (c_k + c_{k+1}) / 2 is exact in fp64 and
// has at most 29 significant bits, so that its product with any fp32 scale
// is exact in fp64.
bool make_exact_halves(const ThreshPairs &tp, QuantBins *bins) {
    bool ok = true;
    for (int k = 0; k < 15; ++k) {
        const double x = tp.lo[k], y = tp.hi[k];
        const double s = x + y;
        const double bb = s - x;
        const double err = (x - (s - bb)) + (y - bb);   // TwoSum: s + err == x + y
        const double h = s * 0.5;
        bins->half[k] = h;
        if (!(err == 0.0) || !std::isfinite(h)) ok = false;
        if (h != 0.0) {
            int e;
            const double m = std::frexp(std::fabs(h), &e);          // m in [0.5, 1)
            const uint64_t bits = (uint64_t)std::ldexp(m, 53);      // exact: 53-bit integer
            const int tz = __builtin_ctzll(bits);
            if (53 - tz > 29) ok = false;
        }
    }
    return ok;
}

namespace {

template <int V>
void launch_quantize_blk(const float *W, const nf4_weight_t &q, const Codebook &cb, int zero_idx,
                         uint32_t *d_status, cudaStream_t st) {
    const int64_t nb = q.rows * q.cols / (32 * V);
    QuantBins bins{};
    const ThreshPairs tp = make_pairs(cb);
    const bool use_bins = make_quant_bins(tp, &bins);
    const bool exact_half = make_exact_halves(tp, &bins);
    auto kern = exact_half ? k_nf4_quantize_blk<V, true> : k_nf4_quantize_blk<V, false>;
    prof_begin(kProfQuant, st);
    kern<<<(unsigned)((nb + 255) / 256), kQbThreads, 0, st>>>(W, nb, tp, bins, use_bins, zero_idx,
                                                              q.double_quant, q.packed, q.absmax,
                                                              q.absmax_code, q.dq_step, q.dq_mean, d_status);
    prof_end(kProfQuant, st);
}

}  // namespace

int launch_nf4_quantize(const float *W, const nf4_weight_t &q, const Codebook &cb, int zero_idx,
                        uint32_t *d_status, cudaStream_t st) {
    const ThreshPairs tp = make_pairs(cb);
    if (q.block != 64) {
        if (q.rows * q.cols == 0) return QLORA_OK;
        QuantBins bins32;
        if (q.block == 32 && make_quant_bins(tp, &bins32)) {   // two blocks per warp, as at 64
            const int64_t nb = q.rows * q.cols / 32;
            auto kern = make_exact_halves(tp, &bins32) ? k_nf4_quantize_fast<true, 2>
                                                       : k_nf4_quantize_fast<false, 2>;
            prof_begin(kProfQuant, st);
            kern<<<(unsigned)((nb + 255) / 256), kQfThreads, kQfSmem, st>>>(
                W, nb, tp, bins32, zero_idx, q.double_quant, q.packed, q.absmax, q.absmax_code,
                q.dq_step, q.dq_mean, d_status);
            prof_end(kProfQuant, st);
        } else if (q.block == 32) launch_quantize_blk<1>(W, q, cb, zero_idx, d_status, st);
        else if (q.block == 128) launch_quantize_blk<4>(W, q, cb, zero_idx, d_status, st);
        else if (q.block == 256) launch_quantize_blk<8>(W, q, cb, zero_idx, d_status, st);
        else return QLORA_EUNSUPPORTED;
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    const int64_t nb = q.rows * q.cols / 64;
    if (nb == 0) return QLORA_OK;
    QuantBins bins;
    if ((reinterpret_cast<uintptr_t>(W) & 15u) == 0 && make_quant_bins(tp, &bins)) {
        const bool exact_half = make_exact_halves(tp, &bins);
        auto kern = exact_half ? k_nf4_quantize_fast<true, 4> : k_nf4_quantize_fast<false, 4>;
        if (set_max_smem(reinterpret_cast<const void *>(kern), kQfSmem) != cudaSuccess) return QLORA_ECUDA;
        prof_begin(kProfQuant, st);
        kern<<<(unsigned)((nb + 255) / 256), kQfThreads, kQfSmem, st>>>(
            W, nb, tp, bins, zero_idx, q.double_quant, q.packed, q.absmax, q.absmax_code, q.dq_step,
            q.dq_mean, d_status);
        prof_end(kProfQuant, st);
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    const int64_t grid = (nb + kQuantThreads - 1) / kQuantThreads;
    // the weight viewed as [nb rows][64 fp32], loaded 32 columns x 256 rows at a time
    CUtensorMap tW;
    if (!tc::make_map(&tW, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 64, (uint64_t)nb, 256, 32, 256,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return QLORA_EUNSUPPORTED;
    if (set_max_smem(reinterpret_cast<const void *>(k_nf4_quantize), kQuantSmem) != cudaSuccess) return QLORA_ECUDA;
    prof_begin(kProfQuant, st);
    k_nf4_quantize<<<(unsigned)grid, kQuantThreads, kQuantSmem, st>>>(
        tW, nb, tp, zero_idx, q.double_quant, q.packed, q.absmax, q.absmax_code, q.dq_step,
        q.dq_mean, d_status);
    prof_end(kProfQuant, st);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_nf4_dequantize(const nf4_weight_t &q, const Codebook &cb, uint16_t *out,
                          cudaStream_t st) {
    if (q.block != 64) {
        const int64_t n16 = q.rows * q.cols / 16;
        if (n16 == 0) return QLORA_OK;
        int lg = 0;
        while ((16 << lg) < q.block) ++lg;
        if ((16 << lg) != q.block) return QLORA_EUNSUPPORTED;
        const ScaleSrc sc = scale_src(q);
        const int64_t need = (n16 + 255) / 256, cap = (int64_t)device_sms() * 8;
        k_nf4_dequantize_blk<<<(unsigned)(need < cap ? need : cap), 256, 0, st>>>(q.packed, sc, n16, lg,
                                                                               cb, out);
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    const int64_t nb = q.rows * q.cols / 64;
    if (nb == 0) return QLORA_OK;
    const ScaleSrc sc = scale_src(q);
    const int64_t threads = nb * 4;
    const int64_t grid = (threads + 255) / 256;
    k_nf4_dequantize<<<(unsigned)grid, 256, 0, st>>>(q.packed, sc, nb, cb, out);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_nf4_dequantize_dtype(const nf4_weight_t &q, const Codebook &cb, int dtype, void *out,
                                cudaStream_t st) {
    const int64_t n = q.rows * q.cols;
    if (n == 0) return QLORA_OK;
    int lg = 0;                                   // block = 8 << lg
    while ((8 << lg) < q.block) ++lg;
    if ((8 << lg) != q.block) return QLORA_EUNSUPPORTED;
    const ScaleSrc sc = scale_src(q);
    const int64_t cap = (int64_t)device_sms() * 8;
    if (dtype == QLORA_DTYPE_FP16) {
        const int64_t n16 = n / 16, need = (n16 + 255) / 256;
        k_nf4_dequantize_f16<<<(unsigned)(need < cap ? need : cap), 256, 0, st>>>(
            q.packed, sc, n16, lg - 1, cb, static_cast<uint16_t *>(out));
    } else if (dtype == QLORA_DTYPE_FP32) {
        const int64_t n8 = n / 8, need = (n8 + 255) / 256;
        k_nf4_dequantize_f32<<<(unsigned)(need < cap ? need : cap), 256, 0, st>>>(
            q.packed, sc, n8, lg, cb, static_cast<float *>(out));
    } else {
        return QLORA_EINVAL;
    }
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
