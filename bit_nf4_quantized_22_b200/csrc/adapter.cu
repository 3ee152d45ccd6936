// adapter.cu -- the rank-r adapter products and their helpers.
//
//   T  = u . A        u = x, or pool(x) = mean over runs of 64 inputs
//   G  = dY . B^T
//   dA = s u^T G      dB = s T^T dY
//
// (LoRA/QLoRA/QA-LoRA blog sections 2-5; bitsandbytes article (CSDN) 12.2.)
// The four products themselves run on the tcgen05 skinny GEMM (umma_skinny.cu);
// this file holds the helpers around them: adapter padding, pooling, the
// hi/lo split of fp32 operands and the deterministic split-K reduce.  fp32
// operands (T, G, pool(x)) are carried as two bf16 terms hi + lo,
// hi = RN_bf16(v), lo = RN_bf16(v - hi), which keeps ~16 mantissa bits; the
// GEMM multiplies both terms and the reduce kernel adds the two halves in fp32.
#include "common.cuh"

namespace qlora {
namespace {

// dst[i][j] = j < r ? src[(i / rep)][j] * mul : 0     (dst: [rows][rp]; 16-bit
// values in the compute dtype, bf16 or fp16 when f16)
__global__ void k_pad_rows(const uint16_t *__restrict__ src, int64_t rows, int r, int rp, int rep,
                           float mul, uint16_t *__restrict__ dst, bool f16) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * rp) return;
    const int64_t row = i / rp;
    const int j = (int)(i % rp);
    dst[i] = j < r ? enc16(dec16(src[(row / rep) * r + j], f16) * mul, f16) : (uint16_t)0;
}

// pool(x)[m][k'] = (1/g) sum_i x[m][k' g + i], emitted as hi/lo terms of the
// compute dtype into [M][ld] buffers (columns k' >= Din/g are zero).
__global__ void k_pool_split(const uint16_t *__restrict__ X, int64_t M, int64_t Din, int g,
                             int64_t ld, uint16_t *__restrict__ hi, uint16_t *__restrict__ lo, bool f16) {
    const int64_t Da = Din / g;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * ld) return;
    const int64_t m = i / ld, k = i % ld;
    if (k >= Da) {
        hi[i] = 0;
        lo[i] = 0;
        return;
    }
    const uint16_t *p = X + m * Din + k * g;
    float sum = 0.f;
    for (int e = 0; e < g; ++e) sum += dec16(p[e], f16);
    const float v = sum / (float)g;
    const uint16_t h = enc16(v, f16);
    hi[i] = h;
    lo[i] = enc16(v - dec16(h, f16), f16);
}

// fp32 [rows][r] -> compute dtype [rows][2 rp] = [hi | lo] with zero padding
__global__ void k_split_f32(const float *__restrict__ src, int64_t rows, int r, int rp,
                            uint16_t *__restrict__ dst, bool f16) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * rp) return;
    const int64_t row = i / rp;
    const int j = (int)(i % rp);
    uint16_t h = 0, l = 0;
    if (j < r) {
        const float v = src[row * r + j];
        h = enc16(v, f16);
        l = enc16(v - dec16(h, f16), f16);
    }
    dst[row * 2 * rp + j] = h;
    dst[row * 2 * rp + rp + j] = l;
}

// Deterministic split-K reduce (fixed summation order) with the adapter
// epilogues.  v(p,q) = sum_z partial[z][p][q] (+ partial[z][p][q+H] when H>0),
// for q < Qv:
//   out_f32[p*fsp + q*fsq]  = f32_scale * v
//   out_bf16[p*bsp + q]     = RN_bf16(bf_scale * v)          (row stride bsp)
//   out_split[p*2*sp + q], [p*2*sp + sp + q] = hi/lo of v    (row stride 2 sp)
struct ReduceArgs {
    const float *partial;
    int splits;
    int64_t P, Qp;        // partial layout [splits][P][Qp]
    int H;                // 0, or the offset of the second half to add
    int Qv;               // valid output columns
    float f32_scale; float *out_f32; int64_t fsp, fsq;
    float bf_scale; uint16_t *out_bf16; int64_t bsp;
    uint16_t *out_split; int64_t sp;
    bool f16;             // 16-bit outputs in fp16 (else bf16)
};

// General layout (any Qp): one thread per output element.
__global__ void k_reduce_scalar(ReduceArgs a) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.P * a.Qv) return;
    const int64_t p = i / a.Qv;
    const int q = (int)(i % a.Qv);
    float v = 0.f;
    for (int z = 0; z < a.splits; ++z) {
        const float *base = a.partial + ((int64_t)z * a.P + p) * a.Qp;
        v += base[q];
        if (a.H) v += base[q + a.H];
    }
    if (a.out_f32) a.out_f32[p * a.fsp + q * a.fsq] = a.f32_scale * v;
    if (a.out_bf16) a.out_bf16[p * a.bsp + q] = enc16(a.bf_scale * v, a.f16);
    if (a.out_split) {
        const uint16_t h = enc16(v, a.f16);
        a.out_split[p * 2 * a.sp + q] = h;
        a.out_split[p * 2 * a.sp + a.sp + q] = enc16(v - dec16(h, a.f16), a.f16);
    }
}

// block (32, 8): thread (x, y) handles the 4 columns [4x + 128 bx, +4) of row
// p = 8 by + y with 16-byte loads (Qp and H are multiples of 4), splits
// unrolled 4 at a time; the sum order over z is fixed.
__global__ void __launch_bounds__(256) k_reduce(ReduceArgs a) {
    const int64_t p = (int64_t)blockIdx.y * 8 + threadIdx.y;
    const int q0 = 4 * (blockIdx.x * 32 + threadIdx.x);
    if (p >= a.P || q0 >= a.Qv) return;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *base = a.partial + p * a.Qp + q0;
    const int64_t zs = a.P * a.Qp;
#pragma unroll 4
    for (int z = 0; z < a.splits; ++z) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(base + z * zs));
        v.x += x.x, v.y += x.y, v.z += x.z, v.w += x.w;
        if (a.H) {
            const float4 y = __ldg(reinterpret_cast<const float4 *>(base + z * zs + a.H));
            v.x += y.x, v.y += y.y, v.z += y.z, v.w += y.w;
        }
    }
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int q = q0 + e;
        if (q >= a.Qv) break;
        if (a.out_f32) a.out_f32[p * a.fsp + q * a.fsq] = a.f32_scale * vv[e];
        if (a.out_bf16) a.out_bf16[p * a.bsp + q] = enc16(a.bf_scale * vv[e], a.f16);
        if (a.out_split) {
            const uint16_t h = enc16(vv[e], a.f16);
            a.out_split[p * 2 * a.sp + q] = h;
            a.out_split[p * 2 * a.sp + a.sp + q] = enc16(vv[e] - dec16(h, a.f16), a.f16);
        }
    }
}

inline unsigned blocks_for(int64_t n, int t = 256) { return (unsigned)((n + t - 1) / t); }

}  // namespace

int launch_pad_rows(const uint16_t *src, int64_t rows, int r, int rp, int rep, float mul,
                    uint16_t *dst, cudaStream_t st, bool f16) {
    const int64_t n = rows * rp;
    if (n == 0) return QLORA_OK;
    k_pad_rows<<<blocks_for(n), 256, 0, st>>>(src, rows, r, rp, rep, mul, dst, f16);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_pool_split(const uint16_t *X, int64_t M, int64_t Din, int g, int64_t ld, uint16_t *hi,
                      uint16_t *lo, cudaStream_t st, bool f16) {
    const int64_t n = M * ld;
    if (n == 0) return QLORA_OK;
    k_pool_split<<<blocks_for(n), 256, 0, st>>>(X, M, Din, g, ld, hi, lo, f16);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_split_f32(const float *src, int64_t rows, int r, int rp, uint16_t *dst, cudaStream_t st,
                     bool f16) {
    const int64_t n = rows * rp;
    if (n == 0) return QLORA_OK;
    k_split_f32<<<blocks_for(n), 256, 0, st>>>(src, rows, r, rp, dst, f16);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_reduce(const float *partial, int splits, int64_t P, int64_t Qp, int H, int Qv,
                  float f32_scale, float *out_f32, int64_t fsp, int64_t fsq, float bf_scale,
                  uint16_t *out_bf16, int64_t bsp, uint16_t *out_split, int64_t sp,
                  cudaStream_t st, bool f16) {
    ReduceArgs a{partial, splits, P, Qp, H, Qv, f32_scale, out_f32, fsp, fsq,
                 bf_scale, out_bf16, bsp, out_split, sp, f16};
    if (P * Qv == 0) return QLORA_OK;
    if (Qp % 4 != 0 || H % 4 != 0 || (reinterpret_cast<uintptr_t>(partial) & 15u) != 0) {
        k_reduce_scalar<<<blocks_for(P * Qv), 256, 0, st>>>(a);
    } else {
        dim3 grid((unsigned)((Qv + 127) / 128), (unsigned)((P + 7) / 8));
        k_reduce<<<grid, dim3(32, 8), 0, st>>>(a);
    }
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
