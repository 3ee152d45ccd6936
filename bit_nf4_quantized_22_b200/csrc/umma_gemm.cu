// umma_gemm.cu -- large-M forward and input-gradient GEMMs on the 5th-gen
// tensor cores (tcgen05 / TMEM), with the NF4 weight dequantized in shared
// memory and the rank-r adapter product accumulated into the same TMEM
// accumulator before the epilogue.
//
//   forward : y [M, Dout] = x  [M, Din ] . W^T  + (s T)  . B      (T = u A)
//   backward: dX[M, Din ] = dY [M, Dout] . W    + (s G)  . A^T    (G = dY B^T)
//
// (LoRA/QLoRA blog section 2: W_eff = dequant(W4) + (alpha/r) A B; the
// bitsandbytes article (CSDN) 8.6: packed weights are read per tile,
// restored on chip and used at once, never materialised in full.)
//
// One CTA computes a 256 x 256 output tile as two 128 x 256 UMMA
// accumulators (512 TMEM columns).  Warp roles:
//   warp 0      TMA producer: activation tile (256 x 64 bf16, 128B swizzle)
//               and packed weight tile (8 KB) per 64-deep k-tile;
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma and commits;
//   warps 2..5  dequantize the packed tile into the bf16 UMMA B operand
//               (K-major for the forward, MN-major for the backward), then
//               run the epilogue TMEM -> registers -> bf16 -> global.
// After the K loop, ceil(r/64) extension k-tiles multiply the scaled
// adapter activations (s T or s G, bf16, zero-padded to 64 columns) by the
// adapter matrix (B, or A^T), both brought in by TMA.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace qlora {
namespace {

constexpr int kBM = 256, kBN = 256, kBK = 64, kStages = 3;
constexpr int kABytes = kBM * kBK * 2;                  // 32 KB
constexpr int kPBytes = 8192;                           // packed tile
constexpr int kBBytes = kBN * kBK * 2;                  // 32 KB
constexpr int kStageBytes = kABytes + kPBytes + kBBytes;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;

struct UmmaParams {
    int mode;            // 0 forward, 1 backward
    int64_t M, N;        // output extent
    int64_t Din, Dout;   // weight shape (Wt: [Dout, Din])
    int nk, ne;          // main and extension k-tiles
    int r;
    ScaleSrc sc;
    Codebook cb;
    uint16_t *Y;
    uint32_t *status;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on an mbarrier phase.  Gives up (returns false) after
// kWaitLimit polls, or early when another role has already given up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start,
// leading and stride byte offsets in 16-byte units, version 1).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor for kind::f16: bf16 x bf16 -> fp32, M = 128, N = 256.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t m, uint32_t n, uint32_t b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major << 16) | ((n >> 3) << 17) |
           ((m >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d));
}

// Raw scale words, fetched ahead of use and decoded when the tile arrives.
struct ScaleRaw {
    float absmax_or_step;
    uint32_t code;
    bool valid;
};
__device__ __forceinline__ ScaleRaw fetch_scale(const ScaleSrc &s, int64_t b, bool valid) {
    ScaleRaw r{0.f, 0u, valid};
    if (valid) {
        if (s.dq) {
            r.code = __ldg(s.code + b);
            r.absmax_or_step = __ldg(s.step + (b >> 8));
        } else {
            r.absmax_or_step = __ldg(s.absmax + b);
        }
    }
    return r;
}
__device__ __forceinline__ float decode_scale(const ScaleRaw &r, int dq) {
    if (!r.valid) return 0.f;
    return dq ? __fmul_rn((float)r.code, r.absmax_or_step) : r.absmax_or_step;
}

// Decode one 64-weight block (32 packed bytes in two 16-byte chunks) and
// store it as one 128-byte swizzled row at `row_addr` (1024-aligned atom
// base + 128 * (row & 7)); `sw` = row & 7.
__device__ __forceinline__ void decode_row(uint4 c0, uint4 c1, float ah, const Codebook &cb,
                                           uint32_t row_addr, uint32_t sw) {
    ProdTable tab;
    build_table(ah, cb, tab);
    uint32_t o[16];
    decode8(c0.x, tab, o + 0);
    decode8(c0.y, tab, o + 4);
    decode8(c0.z, tab, o + 8);
    decode8(c0.w, tab, o + 12);
#pragma unroll
    for (int c = 0; c < 4; ++c) sts128(row_addr + ((c ^ sw) << 4), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
    decode8(c1.x, tab, o + 0);
    decode8(c1.y, tab, o + 4);
    decode8(c1.z, tab, o + 8);
    decode8(c1.w, tab, o + 12);
#pragma unroll
    for (int c = 0; c < 4; ++c)
        sts128(row_addr + (((c + 4) ^ sw) << 4), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

__global__ void __launch_bounds__(kThreads, 1)
k_umma_qgemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
             const __grid_constant__ CUtensorMap tmAe, const __grid_constant__ CUtensorMap tmBe,
             const UmmaParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *gen_base = smem_raw + (base - raw_addr);
    const uint32_t bar0 = base + kStages * kStageBytes;       // 3*kStages + 1 barriers
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto bready_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto empty_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
    const uint32_t acc_bar = bar0 + 8u * (3 * kStages);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gen_base + kStages * kStageBytes + 128);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gen_base + kStages * kStageBytes + 160);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.y * kBM, n0 = (int64_t)blockIdx.x * kBN;
    const int total = p.nk + p.ne;
    const bool fwd = p.mode == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(bready_bar(s), 4);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        fence_proxy_async();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(tmem_holder)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            for (int it = 0; it < total && ok; ++it) {
                const int s = it % kStages;
                if (it >= kStages) ok = mbar_wait(empty_bar(s), ((it / kStages) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const uint32_t sa = base + s * kStageBytes;
                if (it < p.nk) {
                    mbar_expect_tx(full_bar(s), kABytes + kPBytes);
                    tma_load_2d(sa, &tmA, it * kBK, (int)m0, full_bar(s));
                    if (fwd)
                        tma_load_2d(sa + kABytes, &tmP, it * (kBK / 2), (int)n0, full_bar(s));
                    else
                        tma_load_2d(sa + kABytes, &tmP, (int)(n0 / 2), it * kBK, full_bar(s));
                } else {
                    const int e = it - p.nk;
                    mbar_expect_tx(full_bar(s), kABytes + kBBytes);
                    tma_load_2d(sa, &tmAe, e * 64, (int)m0, full_bar(s));
                    const uint32_t sb = sa + kABytes + kPBytes;
                    if (fwd) {
#pragma unroll
                        for (int a = 0; a < 4; ++a)
                            tma_load_2d(sb + a * 8192, &tmBe, (int)(n0 + 64 * a), e * 64, full_bar(s));
                    } else {
                        tma_load_2d(sb, &tmBe, e * 64, (int)n0, full_bar(s));
                    }
                }
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_k = idesc_bf16(128, 256, 0);
            const uint32_t id_mn = idesc_bf16(128, 256, 1);
            for (int it = 0; it < total && ok; ++it) {
                const int s = it % kStages;
                const uint32_t par = (it / kStages) & 1;
                const bool main = it < p.nk;
                ok = mbar_wait(full_bar(s), par, abort_flag);
                if (ok && main) ok = mbar_wait(bready_bar(s), par, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sa = base + s * kStageBytes;
                const uint32_t sb = sa + kABytes + kPBytes;
                int nsteps = 4;
                if (!main) {
                    const int rem = p.r - (it - p.nk) * 64;
                    nsteps = rem >= 64 ? 4 : (rem + 15) / 16;
                }
                // B operand: forward main and backward extension are K-major
                // (rows of 64 k, 128 B, 8-row groups 1 KB apart); backward main
                // and forward extension are MN-major ([4 atoms of 64 columns]
                // x [64 k rows of 128 B]: atoms 8 KB apart, 8-row k groups 1 KB
                // apart).
                const bool b_kmajor = (fwd == main);
                const uint32_t idesc = b_kmajor ? id_k : id_mn;
                for (int kk = 0; kk < nsteps; ++kk) {
                    const uint64_t bd = b_kmajor ? sdesc(sb + kk * 32, 16, 1024)
                                                 : sdesc(sb + kk * 2048, 8192, 1024);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t ad = sdesc(sa + h * 16384 + kk * 32, 16, 1024);
                        umma_bf16(tmem + h * 256, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(empty_bar(s));
            }
            if (ok) umma_commit(acc_bar);
            else *abort_flag = 1;
        }
    } else {
        // ---------------------------------------------------------- dequant
        const int d = threadIdx.x - 64;   // 0..127
        const int64_t nbr = p.Din / 64;   // blocks per weight row
        auto scale_index = [&](int kt, int j, bool &valid) -> int64_t {
            if (fwd) {
                const int64_t n = n0 + d + 128 * j;
                valid = n < p.Dout;
                return n * nbr + kt;
            }
            const int pidx = d + 128 * j;
            const int64_t row = (int64_t)kt * 64 + (pidx & 63);
            const int64_t col = n0 + 64 * (pidx >> 6);
            valid = row < p.Dout && col < p.Din;
            return row * nbr + col / 64;
        };
        // scales are fetched one k-tile ahead, before waiting for the tile
        ScaleRaw pf[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            bool v = false;
            const int64_t b = scale_index(0, j, v);
            pf[j] = fetch_scale(p.sc, b, v);
        }
        for (int it = 0; it < p.nk && ok; ++it) {
            const int s = it % kStages;
            const ScaleRaw cur[2] = {pf[0], pf[1]};
            if (it + 1 < p.nk) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    bool v = false;
                    const int64_t b = scale_index(it + 1, j, v);
                    pf[j] = fetch_scale(p.sc, b, v);
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait(full_bar(s), (it / kStages) & 1, abort_flag));
            if (!ok) break;
            const uint32_t sp = base + s * kStageBytes + kABytes;
            const uint32_t sb = sp + kPBytes;
            float ah[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) ah[j] = decode_scale(cur[j], p.sc.dq);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (fwd) {
                    // packed tile [256 rows][32 B], 32-byte swizzle
                    const uint32_t nl = d + 128 * j;
                    const uint32_t psw = (nl >> 2) & 1;
                    const uint4 c0 = lds128(sp + nl * 32 + ((0 ^ psw) << 4));
                    const uint4 c1 = lds128(sp + nl * 32 + ((1 ^ psw) << 4));
                    decode_row(c0, c1, ah[j], p.cb, sb + (nl >> 3) * 1024 + (nl & 7) * 128, nl & 7);
                } else {
                    // packed tile [64 rows][128 B], 128-byte swizzle
                    const uint32_t pidx = d + 128 * j;
                    const uint32_t nl = pidx & 63, a = pidx >> 6;
                    const uint32_t rsw = nl & 7;
                    const uint4 c0 = lds128(sp + nl * 128 + (((2 * a) ^ rsw) << 4));
                    const uint4 c1 = lds128(sp + nl * 128 + (((2 * a + 1) ^ rsw) << 4));
                    decode_row(c0, c1, ah[j], p.cb, sb + a * 8192 + nl * 128, rsw);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(bready_bar(s));
        }
        if (!ok) *abort_flag = 1;

        // ---------------------------------------------------------- epilogue
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_bar, 0, abort_flag));
        if (ok) {
            tc_fence_after();
            const int q = warp & 3;
            for (int h = 0; h < 2; ++h) {
                const int64_t m = m0 + h * 128 + 32 * q + lane;
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + h * 256 + c * 32, v);
                    if (m < p.M) {
                        uint16_t *dst = p.Y + m * p.N + n0 + c * 32;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (n0 + c * 32 + 8 * i < p.N) {
                                uint4 o;
                                o.x = bf16x2_bits(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
                                o.y = bf16x2_bits(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
                                o.z = bf16x2_bits(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
                                o.w = bf16x2_bits(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
                                *reinterpret_cast<uint4 *>(dst + 8 * i) = o;
                            }
                        }
                    }
                }
            }
        } else {
            *abort_flag = 1;
        }
    }

    if (!ok && p.status) atomicOr(p.status, QLORA_STATUS_TIMEOUT);
    __syncwarp();   // reconverge single-lane roles before the block barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // Let copies already issued land before the CTA's shared memory is
        // released: wait (bounded) for every stage's last armed phase.
        for (int s = 0; s < kStages && s < total; ++s) {
            const int last = ((total - 1 - s) / kStages) * kStages + s;
            for (uint32_t i = 0; i < kWaitLimit; ++i)
                if (mbar_try_wait(full_bar(s), (last / kStages) & 1)) break;
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int esize, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    (void)esize;
    return fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// mode 0: Y[M, Dout] = X[M, Din] W^T + sAct[M, rp64] . Bl[r, Dout]
// mode 1: Y[M, Din]  = X[M, Dout] W  + sAct[M, rp64] . Apad[Din, rp64]^T
int launch_umma_qgemm(int mode, const uint16_t *X, int64_t M, const nf4_weight_t &q,
                       const Codebook &cb, const uint16_t *sAct, int r, const uint16_t *adapter,
                       uint16_t *Y, uint32_t *d_status, cudaStream_t st) {
    const int64_t Din = q.cols, Dout = q.rows;
    const int rp64 = (r + 63) / 64 * 64;
    CUtensorMap tA, tP, tAe, tBe;
    const uint64_t Kmain = mode == 0 ? Din : Dout;
    const uint64_t N = mode == 0 ? Dout : Din;
    bool ok = make_map(&tA, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Kmain, M, Kmain * 2, 64, 256,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (mode == 0)
        ok = ok && make_map(&tP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                            32, 256, CU_TENSOR_MAP_SWIZZLE_32B);
    else
        ok = ok && make_map(&tP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                            128, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tAe, sAct, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rp64, M, (uint64_t)rp64 * 2,
                        64, 256, CU_TENSOR_MAP_SWIZZLE_128B);
    if (mode == 0)
        ok = ok && make_map(&tBe, adapter, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dout, r, Dout * 2,
                            64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ok = ok && make_map(&tBe, adapter, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rp64, Din,
                            (uint64_t)rp64 * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return QLORA_EUNSUPPORTED;

    UmmaParams p;
    p.mode = mode;
    p.M = M;
    p.N = (int64_t)N;
    p.Din = Din;
    p.Dout = Dout;
    p.nk = (int)((Kmain + kBK - 1) / kBK);
    p.ne = rp64 / 64;
    p.r = r;
    p.sc = ScaleSrc{q.absmax, q.absmax_code, q.dq_step, q.double_quant};
    p.cb = cb;
    p.Y = Y;
    p.status = d_status;
    cudaFuncSetAttribute(k_umma_qgemm, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    dim3 grid((unsigned)((N + kBN - 1) / kBN), (unsigned)((M + kBM - 1) / kBM));
    prof_begin(kProfUmma, st);
    k_umma_qgemm<<<grid, kThreads, kSmemBytes, st>>>(tA, tP, tAe, tBe, p);
    prof_end(kProfUmma, st);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
