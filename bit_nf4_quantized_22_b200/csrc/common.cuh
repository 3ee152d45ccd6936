// common.cuh -- device helpers shared by the QLoRA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora.h"

namespace qlora {

// The 16-level codebook, passed to kernels by value.
struct Codebook {
    float c[16];
};

// Decoded first-level scale of block b: the fp32 absmax (dq == 0), or with
// double quantization RN32(code * step) (dq == 1: unsigned code, step max/255;
// dq == 2: signed INT8 code, step max/127; one rounding of an exact product),
// or RN32(mean + RN32(code * step)) with a signed code (dq == 3: the code of
// the scale minus its group's mean).  One step and one mean per 256 blocks.
struct ScaleSrc {
    const float *absmax;      // when !dq
    const uint8_t *code;      // when dq
    const float *step;        // when dq
    int dq;
    const float *mean;        // when dq == 3
};

// The value of an E4M3 code with the sign bit clear (QLORA_DQ_F8): exponent
// field e, mantissa m; e = 0 holds the subnormals m * 2^-9.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : __fmul_rn((float)m, 0x1p-9f);
}

__device__ __forceinline__ float dq_decode(uint32_t code, float step, float mean, int dq) {
    if (dq == 3) return __fadd_rn(mean, __fmul_rn((float)(int8_t)(uint8_t)code, step));
    if (dq == 4) return __fmul_rn(e4m3_value(code), step);
    return __fmul_rn((float)code, step);
}

__device__ __forceinline__ float load_scale(const ScaleSrc &s, int64_t b) {
    if (!s.dq) return __ldg(s.absmax + b);
    const float f = __ldg(s.step + (b >> 8));
    const float mu = s.dq == 3 ? __ldg(s.mean + (b >> 8)) : 0.f;
    return dq_decode(__ldg(s.code + b), f, mu, s.dq);
}

__host__ __forceinline__ ScaleSrc scale_src(const nf4_weight_t &q) {
    return ScaleSrc{q.absmax, q.absmax_code, q.dq_step, q.double_quant, q.dq_mean};
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// The layer's 16-bit compute dtype (bitsandbytes article (CSDN) 8.3):
// bf16 (f16 == false) or IEEE binary16 (f16 == true).  Conversions round to
// nearest even; fp16 keeps subnormals and overflows to infinity.
__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool f16) {
    if (!f16) return bf16x2_bits(lo, hi);
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float lo16(uint32_t v, bool f16) {
    return f16 ? __half2float(__ushort_as_half((unsigned short)(v & 0xffffu))) : bf16_lo(v);
}
__device__ __forceinline__ float hi16(uint32_t v, bool f16) {
    return f16 ? __half2float(__ushort_as_half((unsigned short)(v >> 16))) : bf16_hi(v);
}
__device__ __forceinline__ float dec16(uint16_t v, bool f16) {
    return f16 ? __half2float(__ushort_as_half(v)) : __bfloat162float(__ushort_as_bfloat16(v));
}
__device__ __forceinline__ uint16_t enc16(float v, bool f16) {
    return f16 ? __half_as_ushort(__float2half_rn(v)) : __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// ---------------------------------------------------------------------------
// NF4 decode through a per-block product table.
//
// For one block with decoded scale a_hat, entry j of the table is the bf16
// weight RN_bf16(RN32(a_hat * c_j)).  The 16 entries are held as two byte
// planes (low and high byte of each bf16) of four registers each, so a
// lookup of four 4-bit indices is two byte-permutes per plane plus a select
// on the index's top bit: no shared memory, no local memory.
// ---------------------------------------------------------------------------
// (r0, r1) = (RN32(a b0), RN32(a b1)) as one packed fp32x2 multiply.
__device__ __forceinline__ void mul2_rn(float a, float b0, float b1, float &r0, float &r1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %2};\n\t"
        "mov.b64 rb, {%3, %4};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r0), "=f"(r1) : "f"(a), "f"(b0), "f"(b1));
}

// (r0, r1) = (fma(a, b0, c0), fma(a, b1, c1)), each correctly rounded, as one packed fp32x2 fma.
__device__ __forceinline__ void fma2_rn(float a, float b0, float b1, float c0, float c1, float &r0, float &r1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %2};\n\t"
        "mov.b64 rb, {%3, %4};\n\t"
        "mov.b64 rc, {%5, %6};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r0), "=f"(r1) : "f"(a), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

struct ProdTable {
    uint32_t lo[4];   // lo[i] byte k = low byte of entry 4i+k
    uint32_t hi[4];   // hi[i] byte k = high byte of entry 4i+k
};

// The products RN32(a_hat c_j) come two at a time from the packed fp32x2
// multiply (each lane rounded as a scalar multiply would be).
__device__ __forceinline__ void build_table(float ah, const Codebook &cb, ProdTable &t, bool f16 = false) {
    uint32_t p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float lo, hi;
        mul2_rn(ah, cb.c[2 * i], cb.c[2 * i + 1], lo, hi);
        p[i] = pack2(lo, hi, f16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        t.lo[i] = __byte_perm(p[2 * i], p[2 * i + 1], 0x6420);
        t.hi[i] = __byte_perm(p[2 * i], p[2 * i + 1], 0x7531);
    }
}

// Decode the 8 indices of one packed 32-bit word (bytes b0..b3 in memory
// order; byte i holds element 2i in its high nibble and 2i+1 in its low
// nibble) into four bf16x2 registers: out[k] = (element 2k, element 2k+1).
__device__ __forceinline__ void decode8(uint32_t w, const ProdTable &t, uint32_t out[4]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t v = (h == 0) ? w : (w >> 16);
        // selector nibbles, output byte n <- nibble n of v: [e1, e0, e3, e2]
        const uint32_t sel = v & 0x7777u;
        const uint32_t m = __byte_perm(0u, 0xffffffffu, (v >> 1) & 0x4444u);
        const uint32_t l0 = __byte_perm(t.lo[0], t.lo[1], sel);
        const uint32_t l1 = __byte_perm(t.lo[2], t.lo[3], sel);
        const uint32_t h0 = __byte_perm(t.hi[0], t.hi[1], sel);
        const uint32_t h1 = __byte_perm(t.hi[2], t.hi[3], sel);
        const uint32_t L = (l0 & ~m) | (l1 & m);
        const uint32_t H = (h0 & ~m) | (h1 & m);
        out[2 * h + 0] = __byte_perm(L, H, 0x4051);   // (e0, e1)
        out[2 * h + 1] = __byte_perm(L, H, 0x6273);   // (e2, e3)
    }
}

// ---------------------------------------------------------------------------
// Legacy warp-level tensor-core helpers (m16n8k16, bf16 in, fp32 accumulate).
// Used where the tensor unit is not the bottleneck (HBM-bound GEMV, skinny
// adapter products).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], const uint32_t b[2]) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], const uint32_t b[2]) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// m16n8k16 in the compute dtype (both operands of one type, fp32 accumulate)
template <bool F16>
__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], const uint32_t b[2]) {
    if (F16)
        mma_f16_16816(d, a, b);
    else
        mma_bf16_16816(d, a, b);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t r[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool pred) {
    const int n = pred ? 16 : 0;   // src-size 0 zero-fills the 16 bytes
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
                 "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace qlora

namespace qlora {
// Launch accounting and optional per-kernel event timing (profile.cu).
enum ProfKind { kProfUmma = 0, kProfGemv = 1, kProfQuant = 2, kProfAdapter = 3, kProfMerge = 4, kProfKinds = 5 };
void count_launch();
void prof_begin(int kind, cudaStream_t st);
void prof_end(int kind, cudaStream_t st);
// Streaming multiprocessors of the current device (cached per device; 148
// if the query fails), for grids sized to whole waves.
int device_sms();
// cudaFuncSetAttribute(fn, MaxDynamicSharedMemorySize, bytes), made once per
// (device, kernel) and remembered.
cudaError_t set_max_smem(const void *fn, int bytes);
}  // namespace qlora

// Host-side launch check used after every kernel launch.
#define QLORA_LAUNCH_CHECK()                                              \
    do {                                                                  \
        ::qlora::count_launch();                                          \
        if (cudaPeekAtLastError() != cudaSuccess) return QLORA_ECUDA;     \
    } while (0)
