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
// A cluster of two CTAs (one per SM) computes a 512 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256): CTA r holds rows
// [128r, 128r+128) of both 256-row MMA halves and columns [128r, 128r+128)
// of the weight tile, so each weight element is dequantized once per 512
// activation rows -- half the dequant work per tensor-core cycle of a
// single-CTA 256 x 256 tile.  Accumulators: 2 x 256 TMEM columns per CTA.
// Warp roles (both CTAs):
//   warp 0      TMA producer: activation slabs (completion counted on CTA
//               0's barrier) and this CTA's packed weight tile (local);
//   warp 1      TMEM allocation; in CTA 0 lane 0 issues the pair MMAs and
//               commits them to both CTAs' barriers;
//   warps 2..9  dequantize half a 64-weight block per thread per k-tile into
//               the UMMA B operand in the compute dtype, bf16 or fp16 (K-major for the forward, MN-major
//               for the backward) and arrive on a local barrier, which
//               CTA 1's warp 1 forwards to CTA 0 once per stage; then the epilogue
//               TMEM -> registers -> compute dtype -> global.
// After the K loop, ceil(r/64) extension k-tiles multiply the scaled
// adapter activations (s T or s G, bf16, zero-padded to 64 columns) by the
// adapter matrix (B, or A^T), both brought in by TMA.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace qlora {
namespace {
using namespace tc;

constexpr int kBK = 64, kStages = 4;
constexpr int kSlabBytes = 128 * kBK * 2;               // 16 KB: 128 rows x 64 bf16
constexpr int kABytes = 2 * kSlabBytes;                 // two slabs per CTA
constexpr int kPBytes = 4096;                           // this CTA's packed tile
constexpr int kBBytes = 128 * kBK * 2;                  // 16 KB: this CTA's half of B
constexpr int kStageBytes = kABytes + kPBytes + kBBytes;
constexpr int kDqWarps = 8;                             // dequant + epilogue warps
constexpr int kDqThreads = kDqWarps * 32;
constexpr int kThreads = 64 + kDqThreads;
static_assert(kDqThreads == 256, "one half 64-block per dequant thread");
static_assert(kStageBytes % 1024 == 0, "stages keep 1 KB swizzle alignment");
static_assert(kStages * kStageBytes >= 2 * 65536, "the epilogue stages a 256 x 256 bf16 tile in the ring");
constexpr uint32_t kTmemCols = 512;
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
    int f16;             // the compute dtype: fp16 operands and output (else bf16)
};

// Raw scale words, fetched ahead of use and decoded when the tile arrives.
struct ScaleRaw {
    float absmax_or_step;
    float mu;            // group mean (mean-offset double quantization)
    uint32_t code;
    bool valid;
};
__device__ __forceinline__ ScaleRaw fetch_scale(const ScaleSrc &s, int64_t b, bool valid) {
    ScaleRaw r{0.f, 0.f, 0u, valid};
    if (valid) {
        if (s.dq) {
            r.code = __ldg(s.code + b);
            r.absmax_or_step = __ldg(s.step + (b >> 8));
            if (s.dq == QLORA_DQ_MEAN) r.mu = __ldg(s.mean + (b >> 8));
        } else {
            r.absmax_or_step = __ldg(s.absmax + b);
        }
    }
    return r;
}
__device__ __forceinline__ float decode_scale(const ScaleRaw &r, int dq) {
    if (!r.valid) return 0.f;
    return dq ? dq_decode(r.code, r.absmax_or_step, r.mu, dq) : r.absmax_or_step;
}

// Decode 32 weights (one 16-byte packed chunk) with block scale `ah` and
// store them as 16-byte chunks [4h, 4h+4) of a 128-byte swizzled row at
// `row_addr` (1 KB-aligned atom base + 128 * (row & 7)); `sw` = row & 7.
__device__ __forceinline__ void decode_half(uint4 c, float ah, const Codebook &cb,
                                            uint32_t row_addr, uint32_t sw, uint32_t h, bool f16) {
    ProdTable tab;
    build_table(ah, cb, tab, f16);
    uint32_t o[16];
    decode8(c.x, tab, o + 0);
    decode8(c.y, tab, o + 4);
    decode8(c.z, tab, o + 8);
    decode8(c.w, tab, o + 12);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        sts128(row_addr + (((4 * h + k) ^ sw) << 4), o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_umma_qgemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
             const __grid_constant__ CUtensorMap tmAe, const __grid_constant__ CUtensorMap tmBe,
             const __grid_constant__ CUtensorMap tmY, const UmmaParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *gen_base = smem_raw + (base - raw_addr);
    const uint32_t bar0 = base + kStages * kStageBytes;
    // CTA 0's full_a(s): the stage is ready for the MMA -- both CTAs' A (and
    // extension) bytes landed, CTA 0's 8 dequant warps wrote its B half, and
    // CTA 1's forwarder reported CTA 1's half (1 + 8 + 1 arrivals).  One wait
    // per k-tile keeps the single MMA-issuing thread's loop short: it is on
    // the critical path of every k-tile.
    auto full_a = [&](int s) { return bar0 + 8u * s; };
    auto full_p = [&](int s) { return bar0 + 8u * (kStages + s); };      // local packed tile
    auto bready = [&](int s) { return bar0 + 8u * (2 * kStages + s); };  // CTA 1: its B half written
    auto empty = [&](int s) { return bar0 + 8u * (3 * kStages + s); };   // stage free (both)
    const uint32_t acc_bar = bar0 + 8u * (5 * kStages);
    // 5 * kStages + 1 barrier slots (168 B; slots 4 kStages .. 5 kStages - 1 unused), then the
    // TMEM address and the abort flag
    static_assert(8 * (5 * kStages + 1) <= 200, "barrier block overlaps the flags");
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gen_base + kStages * kStageBytes + 208);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gen_base + kStages * kStageBytes + 240);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int64_t m0 = (int64_t)blockIdx.y * 512;
    const int64_t n0 = (int64_t)(blockIdx.x >> 1) * 256;
    const int64_t nc = n0 + 128 * rank;            // this CTA's 128 weight-tile columns
    const int total = p.nk + p.ne;
    const bool fwd = p.mode == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_a(s), 2 + kDqWarps);
            mbar_init(full_p(s), 1);
            mbar_init(bready(s), kDqWarps);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        fence_proxy_async();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(tmem_holder)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers initialised before any cross-CTA use
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            for (int it = 0; it < total && ok; ++it) {
                const int s = it % kStages;
                if (it >= kStages) ok = mbar_wait(empty(s), ((it / kStages) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const uint32_t sa = base + s * kStageBytes;
                const uint32_t sp = sa + kABytes, sb = sp + kPBytes;
                const uint32_t fa0 = mapa_shared(full_a(s), 0);
                const int y0 = (int)(m0 + 128 * rank), y1 = (int)(m0 + 256 + 128 * rank);
                if (it < p.nk) {
                    if (rank == 0) mbar_expect_tx(full_a(s), 2 * kABytes);
                    tma_load_2d_pair(sa, &tmA, it * kBK, y0, fa0);
                    tma_load_2d_pair(sa + kSlabBytes, &tmA, it * kBK, y1, fa0);
                    mbar_expect_tx(full_p(s), kPBytes);
                    if (fwd)
                        tma_load_2d(sp, &tmP, it * (kBK / 2), (int)nc, full_p(s));
                    else
                        tma_load_2d(sp, &tmP, (int)(nc / 2), it * kBK, full_p(s));
                } else {
                    const int e = it - p.nk;
                    if (rank == 0) {   // no dequantized half: arrive for the warps and the forwarder
                        mbar_expect_tx(full_a(s), 2 * (kABytes + kBBytes));
                        mbar_arrive_n(full_a(s), 1 + kDqWarps);
                    }
                    tma_load_2d_pair(sa, &tmAe, e * 64, y0, fa0);
                    tma_load_2d_pair(sa + kSlabBytes, &tmAe, e * 64, y1, fa0);
                    if (fwd) {
                        tma_load_2d_pair(sb, &tmBe, (int)nc, e * 64, fa0);
                        tma_load_2d_pair(sb + 8192, &tmBe, (int)(nc + 64), e * 64, fa0);
                    } else {
                        tma_load_2d_pair(sb, &tmBe, e * 64, (int)nc, fa0);
                    }
                }
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- CTA 1: forwarder
        // One cluster-scope arrive per stage tells CTA 0 that this CTA's B
        // half is written (the dequant warps only arrive locally).
        if (lane == 0 && rank == 1) {
            const uint32_t ready0 = mapa_shared(full_a(0), 0);
            for (int it = 0; it < p.nk && ok; ++it) {
                const int s = it % kStages;
                ok = mbar_wait(bready(s), (it / kStages) & 1, abort_flag);
                if (ok) mbar_arrive_cluster(ready0 + 8u * s);
            }
            if (!ok) *abort_flag = 1;
        }
        // ---------------------------------------------------------- MMA issuer (CTA 0)
        if (lane == 0 && rank == 0) {
            const uint32_t id_k = p.f16 ? idesc_as_fp16(idesc_bf16(256, 256, 0)) : idesc_bf16(256, 256, 0);
            const uint32_t id_mn = p.f16 ? idesc_as_fp16(idesc_bf16(256, 256, 1)) : idesc_bf16(256, 256, 1);
            // Descriptors of stage 0's operands; a shared-memory offset o (a
            // multiple of 16 B, the address staying below 256 KB) adds o >> 4
            // to the start-address field.  B operand: forward main and
            // backward extension are K-major (rows of 64 k, 128 B, 8-row groups
            // 1 KB apart, +32 B per 16 k); backward main and forward extension
            // are MN-major (2 atoms of 64 columns 8 KB apart, x 64 k rows of
            // 128 B, +2 KB per 16 k).
            const uint64_t dA = sdesc(base, 16, 1024);
            const uint64_t dBk = sdesc(base + kABytes + kPBytes, 16, 1024);
            const uint64_t dBm = sdesc(base + kABytes + kPBytes, 8192, 1024);
            constexpr uint32_t kStageD = kStageBytes >> 4, kSlabD = kSlabBytes >> 4;
            // main k-tiles, unrolled over the stages (constant stage addresses)
            {
                const uint64_t db0 = fwd ? dBk : dBm;
                const uint32_t idesc = fwd ? id_k : id_mn;
                const uint32_t bstep = fwd ? 2u : 128u;
                for (int it0 = 0; it0 < p.nk && ok; it0 += kStages) {
                    const uint32_t par = (it0 / kStages) & 1;
#pragma unroll
                    for (int j = 0; j < kStages; ++j) {
                        const int it = it0 + j;
                        if (it >= p.nk || !ok) break;
                        ok = mbar_wait_cluster(full_a(j), par, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t so = (uint64_t)(j * kStageD);
                        uint64_t a0[4], a1[4], bd[4];
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            a0[kk] = dA + so + kk * 2;
                            a1[kk] = dA + so + kSlabD + kk * 2;
                            bd[kk] = db0 + so + kk * bstep;
                        }
                        umma_ktile_pair(tmem, tmem + 256, a0, a1, bd, idesc, it > 0 ? 1u : 0u);
                        umma_commit_pair(empty(j), 0x3);
                    }
                }
            }
            // extension k-tiles (the adapter product)
            for (int it = p.nk; it < total && ok; ++it) {
                const uint32_t s = it & (kStages - 1);
                ok = mbar_wait_cluster(full_a(s), (it / kStages) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint64_t so = (uint64_t)(s * kStageD);
                const uint32_t acc0 = it > 0 ? 1u : 0u;
                const int rem = p.r - (it - p.nk) * 64;
                const int nsteps = rem >= 64 ? 4 : (rem + 15) / 16;
                const uint64_t db = (fwd ? dBm : dBk) + so;
                const uint32_t idesc = fwd ? id_mn : id_k;
                const uint32_t bstep = fwd ? 128u : 2u;
                for (int kk = 0; kk < nsteps; ++kk)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        umma_bf16_pair(tmem + h * 256, dA + so + h * kSlabD + kk * 2, db + kk * bstep, idesc,
                                       kk > 0 ? 1u : acc0);
                umma_commit_pair(empty(s), 0x3);
            }
            if (ok) umma_commit_pair(acc_bar, 0x3);
            else *abort_flag = 1;
        }
    } else {
        // ---------------------------------------------------------- dequant
        const int d = threadIdx.x - 64;          // 0 .. 255
        const uint32_t pr = d & 127, h = d >> 7;  // B row/pair, half of its 64-block
        const int64_t nbr = p.Din / 64;          // blocks per weight row
        auto scale_index = [&](int kt, bool &valid) -> int64_t {
            if (fwd) {
                const int64_t n = nc + pr;
                valid = n < p.Dout;
                return n * nbr + kt;
            }
            const int64_t row = (int64_t)kt * 64 + (pr & 63);
            const int64_t col = nc + 64 * (pr >> 6);
            valid = row < p.Dout && col < p.Din;
            return row * nbr + col / 64;
        };
        auto fetch = [&](int kt) -> ScaleRaw {
            bool v = false;
            const int64_t b = kt < p.nk ? scale_index(kt, v) : 0;
            return fetch_scale(p.sc, b, v && kt < p.nk);
        };
        // one k-tile of dequantization, given its (already fetched) scale
        auto body = [&](int it, const ScaleRaw &cur) -> bool {
            const int s = it % kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(full_p(s), (it / kStages) & 1, abort_flag)))
                return false;
            const uint32_t sp = base + s * kStageBytes + kABytes;
            const uint32_t sb = sp + kPBytes;
            const float ah = decode_scale(cur, p.sc.dq);
            if (fwd) {
                // packed tile [128 rows][32 B], 32-byte swizzle
                const uint4 c = lds128(sp + pr * 32 + ((h ^ ((pr >> 2) & 1)) << 4));
                decode_half(c, ah, p.cb, sb + (pr >> 3) * 1024 + (pr & 7) * 128, pr & 7, h, p.f16);
            } else {
                // packed tile [64 rows][64 B], 64-byte swizzle
                const uint32_t nl = pr & 63, a = pr >> 6;
                const uint4 c = lds128(sp + nl * 64 + (((2 * a + h) ^ ((nl >> 1) & 3)) << 4));
                decode_half(c, ah, p.cb, sb + a * 8192 + nl * 128, nl & 7, h, p.f16);
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(rank == 0 ? full_a(s) : bready(s));   // CTA 1: via the forwarder
            return true;
        };
        // scales are fetched three k-tiles ahead of use
        ScaleRaw r0 = fetch(0), r1 = fetch(1), r2 = fetch(2);
        for (int it = 0; it < p.nk && ok; it += 3) {
            ScaleRaw cur = r0;
            r0 = fetch(it + 3);
            ok = body(it, cur);
            if (!ok || it + 1 >= p.nk) break;
            cur = r1;
            r1 = fetch(it + 4);
            ok = body(it + 1, cur);
            if (!ok || it + 2 >= p.nk) break;
            cur = r2;
            r2 = fetch(it + 5);
            ok = body(it + 2, cur);
        }
        if (!ok) *abort_flag = 1;

        // ---------------------------------------------------------- epilogue
        // TMEM -> registers -> bf16 -> the idle stage ring, as 128-byte-swizzled
        // [128 rows][64 columns] boxes (half hh at hh * 64 KB, box j at + 16 KB j),
        // then TMA stores of whole boxes: coalesced, and clipped at M and N.  A
        // box is stored as soon as the four warps of its half have written it,
        // so the stores overlap the remaining TMEM reads.
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(acc_bar, 0, abort_flag));
        if (ok) tc_fence_after();
        else *abort_flag = 1;
        {
            const int q = warp & 3;                       // TMEM lane quarter of this warp
            const int hh = (warp - 2) >> 2;               // accumulator (MMA half) of this warp
            const uint32_t L = 32 * q + lane;             // tile row = TMEM lane
            const uint32_t stile = base + hh * 65536 + L * 128;
            const bool storer = q == 0 && lane == 0;      // one thread per half issues its boxes
            const int64_t y = m0 + 256 * hh + 128 * rank;
            for (int c = 0; c < 8; ++c) {
                if (ok) {
                    uint32_t v[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + hh * 256 + c * 32, v);
                    const uint32_t box = stile + (c >> 1) * 16384;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t chunk = 4 * (c & 1) + i;
                        const bool f16 = p.f16;
                        sts128(box + ((chunk ^ (L & 7)) << 4),
                               pack2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]), f16),
                               pack2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]), f16),
                               pack2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]), f16),
                               pack2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]), f16));
                    }
                }
                if (c & 1) {
                    // box c / 2 of this half is complete once its four warps are here
                    fence_proxy_async();
                    asm volatile("bar.sync %0, 128;\n" ::"r"(2 + hh) : "memory");
                    const int64_t x = n0 + 64 * (c >> 1);
                    if (ok && storer && y < p.M && x < p.N)
                        tma_store_2d(&tmY, base + hh * 65536 + (c >> 1) * 16384, (int)x, (int)y);
                }
            }
            if (storer) {
                bulk_commit();
                bulk_wait_read();
            }
        }
    }

    if (!ok && p.status) atomicOr(p.status, QLORA_STATUS_TIMEOUT);
    __syncwarp();   // reconverge single-lane roles before the barriers
    tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // Let this CTA's packed-tile copies land before its shared memory is
        // released: wait (bounded) for every stage's last armed phase.
        for (int s = 0; s < kStages && s < p.nk; ++s) {
            const int last = ((p.nk - 1 - s) / kStages) * kStages + s;
            for (uint32_t i = 0; i < kWaitLimit; ++i)
                if (mbar_try_wait(full_p(s), (last / kStages) & 1)) break;
        }
    }
    __syncwarp();
    cluster_sync();   // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(kTmemCols));
    }
}

}  // namespace

// mode 0: Y[M, Dout] = X[M, Din] W^T + sAct[M, rp64] . Bl[r, Dout]
// mode 1: Y[M, Din]  = X[M, Dout] W  + sAct[M, rp64] . Apad[Din, rp64]^T
int launch_umma_qgemm(int mode, const uint16_t *X, int64_t M, const nf4_weight_t &q,
                       const Codebook &cb, const uint16_t *sAct, int r, const uint16_t *adapter,
                       uint16_t *Y, uint32_t *d_status, cudaStream_t st, bool f16) {
    const int64_t Din = q.cols, Dout = q.rows;
    const int rp64 = (r + 63) / 64 * 64;
    CUtensorMap tA, tP, tAe, tBe;
    const uint64_t Kmain = mode == 0 ? Din : Dout;
    const uint64_t N = mode == 0 ? Dout : Din;
    // activation slabs 128 x 64 (128 B swizzle); packed tiles: forward
    // [128 rows][32 B] (32 B swizzle), backward [64 rows][64 B] (64 B swizzle)
    bool ok = make_map(&tA, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Kmain, M, Kmain * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    // output boxes [128 rows][64 columns], 128-byte swizzle (the epilogue's staging layout)
    CUtensorMap tY;
    ok = ok && make_map(&tY, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, N * 2, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (mode == 0)
        ok = ok && make_map(&tP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                            32, 128, CU_TENSOR_MAP_SWIZZLE_32B);
    else
        ok = ok && make_map(&tP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                            64, 64, CU_TENSOR_MAP_SWIZZLE_64B);
    ok = ok && make_map(&tAe, sAct, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rp64, M, (uint64_t)rp64 * 2,
                        64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (mode == 0)
        ok = ok && make_map(&tBe, adapter, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dout, r, Dout * 2,
                            64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ok = ok && make_map(&tBe, adapter, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rp64, Din,
                            (uint64_t)rp64 * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
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
    p.sc = scale_src(q);
    p.cb = cb;
    p.Y = Y;
    p.status = d_status;
    p.f16 = f16 ? 1 : 0;
    if (set_max_smem(reinterpret_cast<const void *>(k_umma_qgemm), kSmemBytes) != cudaSuccess) return QLORA_ECUDA;
    // clusters of two CTAs along x: pair index = N tile of 256, rank = half
    dim3 grid((unsigned)(2 * ((N + 255) / 256)), (unsigned)((M + 511) / 512));
    prof_begin(kProfUmma, st);
    k_umma_qgemm<<<grid, kThreads, kSmemBytes, st>>>(tA, tP, tAe, tBe, tY, p);
    prof_end(kProfUmma, st);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
