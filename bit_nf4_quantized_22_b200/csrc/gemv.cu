// gemv.cu -- small-M (M <= 16) forward and input-gradient kernels.
//
// At decode-like M the layer is bound by reading the 4-bit weight from HBM
// (~0.52 B/weight with double quantization).  Each lane streams packed
// nibbles with wide loads, decodes them in registers through a per-block
// bf16 product table (exact RN_bf16(RN32(a_hat * c_q)) weights), and feeds
// the warp-level tensor core (m16n8k16) with the 16 tokens as the M side;
// the tensor unit is far from busy here, it only replaces 16 FMAs per weight.
// Partial sums over the reduction are written per split and reduced by a
// finalize kernel that also adds the rank-r adapter term.
#include "common.cuh"
#include "tcgen05.cuh"

namespace qlora {
namespace {

// Scale words fetched ahead of use (code + step, or the fp32 absmax).
struct ScaleRawG {
    float f;
    uint32_t code;
};
__device__ __forceinline__ ScaleRawG fetch_scale_g(const ScaleSrc &s, int64_t b, bool valid) {
    ScaleRawG r{0.f, 0u};
    if (valid) {
        if (s.dq) {
            r.code = __ldg(s.code + b);
            r.f = __ldg(s.step + (b >> 8));
        } else {
            r.f = __ldg(s.absmax + b);
        }
    }
    return r;
}
__device__ __forceinline__ float decode_scale_g(const ScaleRawG &r, int dq) {
    return dq ? __fmul_rn((float)r.code, r.f) : r.f;
}

constexpr int kGemvWarps = 8;
constexpr int kFwdKS = 1024;         // input slice per CTA (16 blocks of 64)
constexpr int kBwdRowsPerWarp = 64;  // 4 groups of 16 rows

// ------------------------------------------------------------------ forward
// grid (ceil(Dout/128), nsplit); block 256.  A CTA owns 128 weight rows and a
// 1024-deep slice of the inputs.  Warp w owns rows [128*bx + 16w, +16); lane
// (g, t) -- g = lane/4, t = lane%4 -- holds rows g and g+8 and, of every
// 64-weight block, the 16 inputs [16t, 16t+16) (8 packed bytes per row).
// The weight is the M side of the warp MMA (m16n8k16) and the tokens its N
// side (one n8 tile for M <= 8, two for M <= 16).
//
// Decode: every packed byte (two 4-bit indices) is looked up in a 256-entry
// table of bf16 codebook pairs held in shared memory, one copy per lane so
// the 32 lanes never share a bank; the looked-up word is directly an MMA
// fragment register.  The block scale multiplies the fp32 MMA result of the
// block once (acc += a_hat * partial), so no per-block table is built.  The
// k index inside a block is relabelled identically for weight and x.
// Loads run kFwdAhead blocks ahead of the MMAs.
constexpr int kFwdRows = 128;
constexpr int kFwdBlocks = kFwdKS / 64;   // 64-blocks per CTA slice
constexpr int kFwdAhead = 4;

struct FwdBlockData {
    uint2 w[2];          // 8 packed bytes of rows g and g+8
    ScaleRawG s[2];
};

template <int NT>
__global__ void __launch_bounds__(kGemvWarps * 32, 2)
k_gemv_fwd(const uint16_t *__restrict__ X, int M, int64_t Din, int64_t Dout,
           const uint8_t *__restrict__ packed, ScaleSrc sc, Codebook cb,
           float *__restrict__ partial) {    // [nsplit][M][Dout]
    extern __shared__ __align__(16) uint8_t fsm[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(fsm);                    // [256][32]
    uint16_t(*sx)[kFwdKS + 8] = reinterpret_cast<uint16_t(*)[kFwdKS + 8]>(fsm + 256 * 32 * 4);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t k0 = (int64_t)blockIdx.y * kFwdKS;
    const int64_t nbr = Din / 64;
    const int64_t kb0 = k0 / 64;
    const int nblk = (int)((Din - k0) / 64 < kFwdBlocks ? (Din - k0) / 64 : kFwdBlocks);
    const int64_t r0 = (int64_t)blockIdx.x * kFwdRows + warp * 16 + g;
    const bool ok0 = r0 < Dout, ok1 = r0 + 8 < Dout;
    const uint8_t *p0 = packed + r0 * (Din / 2) + k0 / 2 + 8 * t;
    const uint8_t *p1 = p0 + 8 * (Din / 2);

    auto fetch = [&](int b) {
        FwdBlockData d;
        const bool in = b < nblk;
        d.w[0] = (in && ok0) ? __ldg(reinterpret_cast<const uint2 *>(p0 + 32 * b)) : make_uint2(0u, 0u);
        d.w[1] = (in && ok1) ? __ldg(reinterpret_cast<const uint2 *>(p1 + 32 * b)) : make_uint2(0u, 0u);
        d.s[0] = fetch_scale_g(sc, r0 * nbr + kb0 + b, in && ok0);
        d.s[1] = fetch_scale_g(sc, (r0 + 8) * nbr + kb0 + b, in && ok1);
        return d;
    };
    FwdBlockData ring[kFwdAhead];
#pragma unroll
    for (int b = 0; b < kFwdAhead; ++b) ring[b] = fetch(b);

    // lane-replicated pair table: word [e][lane] = (c[e >> 4], c[e & 15]) in bf16.
    // Thread e computes entry e once and writes its 32 copies as eight
    // 16-byte stores, rotated by lane so a warp's stores spread over banks.
    {
        const int e = threadIdx.x;
        const uint32_t v = bf16x2_bits(cb.c[e >> 4], cb.c[e & 15]);
        uint4 *row = reinterpret_cast<uint4 *>(lut + e * 32);
        const uint4 vv = make_uint4(v, v, v, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) row[(i + lane) & 7] = vv;
    }
    // x[:M, k0:k0+KS] (inputs past Din are zero; only M token rows are read)
    for (int i = threadIdx.x; i < M * (kFwdKS / 8); i += blockDim.x) {
        const int m = i / (kFwdKS / 8), kc = (i % (kFwdKS / 8)) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k0 + kc < Din) v = __ldg(reinterpret_cast<const uint4 *>(X + (int64_t)m * Din + k0 + kc));
        *reinterpret_cast<uint4 *>(&sx[m][kc]) = v;
    }
    for (int i = threadIdx.x; i < (8 * NT - M) * (kFwdKS / 8); i += blockDim.x)
        if (M < 8 * NT) {
            const int m = M + i / (kFwdKS / 8), kc = (i % (kFwdKS / 8)) * 8;
            *reinterpret_cast<uint4 *>(&sx[m][kc]) = make_uint4(0, 0, 0, 0);
        }
    __syncthreads();

    const uint32_t *lut_lane = lut + lane;
    auto lookup = [&](uint32_t word, int i) -> uint32_t {
        return lut_lane[__byte_perm(word, 0u, 0x4440u + i) << 5];
    };

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;

#pragma unroll
    for (int b = 0; b < kFwdBlocks; ++b) {
        const FwdBlockData cur = ring[b % kFwdAhead];
        if (b + kFwdAhead < kFwdBlocks) ring[b % kFwdAhead] = fetch(b + kFwdAhead);
        if (b >= nblk) continue;
        float tmp[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) tmp[n][e] = 0.f;
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            const uint32_t w0 = st < 2 ? cur.w[0].x : cur.w[0].y;
            const uint32_t w1 = st < 2 ? cur.w[1].x : cur.w[1].y;
            const int i0 = (2 * st) & 3;
            const uint32_t a[4] = {lookup(w0, i0), lookup(w1, i0), lookup(w0, i0 + 1),
                                   lookup(w1, i0 + 1)};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const uint2 xv = *reinterpret_cast<const uint2 *>(&sx[g + 8 * n][64 * b + 16 * t + 4 * st]);
                const uint32_t bb[2] = {xv.x, xv.y};
                mma_bf16_16816(tmp[n], a, bb);
            }
        }
        const float a0 = decode_scale_g(cur.s[0], sc.dq), a1 = decode_scale_g(cur.s[1], sc.dq);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            acc[n][0] = fmaf(a0, tmp[n][0], acc[n][0]);
            acc[n][1] = fmaf(a0, tmp[n][1], acc[n][1]);
            acc[n][2] = fmaf(a1, tmp[n][2], acc[n][2]);
            acc[n][3] = fmaf(a1, tmp[n][3], acc[n][3]);
        }
    }

    // acc[n]: (row g, tokens 8n + 2t, +1) and (row g + 8, same tokens)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = 8 * n + 2 * t + (e & 1);
            const int64_t row = r0 + 8 * (e >> 1);
            if (m < M && row < Dout)
                partial[((int64_t)blockIdx.y * M + m) * Dout + row] = acc[n][e];
        }
}

// ------------------------------------------------------------------ forward, streamed
// Persistent variant: one CTA per SM walks a contiguous range of
// (input-slice, 128-row) tiles, slices of 1024 inputs.  A producer warp
// streams each tile as two half-tiles (128 rows x 256 packed bytes, two
// 128-byte-swizzled TMA boxes, plus the rows' scale codes) through a
// three-stage shared-memory ring, so loads run ahead independently of
// registers.
//
// Sixteen compute warps: warps w and w + 8 own the same 16 rows and take
// the even and the odd 64-blocks of each half-tile, four blocks each; the
// two warps' sums meet in shared memory once per tile (even + odd).
//
// Decode: the byte -> bf16-pair table has one 256-byte row per byte value,
// lane l's copy at +4l, so the shared address of a lookup is exactly
// (byte << 8) | 4l: one byte permute builds it from the packed word and a
// per-lane constant.  The x slice rows are 2056 bytes apart (= 8 mod 128),
// which puts the 32 lanes' 8-byte fragment loads on distinct bank pairs.
//
// With an adapter (Aad), ceil(r/16) tiles of slice z, spread over its row
// tiles, also compute the adapter-down partials of one rank tile each,
// Tpart[z][b][m][j] = sum over the 64 inputs k of block b of x[m][k] A[k][j],
// warp w taking block w, as MMAs with the 16 ranks on the M side (A^T
// gathered from the row-major A) and the tokens on the N side.  Needs the scale rows to be TMA-tileable: Din/64 a
// multiple of 16 (codes) or of 4 (fp32 absmax).
constexpr int kStRows = 128, kStBlocks = 16;              // tile: 128 rows x 1024 inputs
constexpr int kStHalf = kStRows * 8 * 32;                 // half-tile packed bytes: 32 KB
constexpr int kStStage = kStHalf + 4096;                  // + scales (codes 2 KB / fp32 4 KB)
constexpr int kStStages = 3;
constexpr int kStCompute = 16;                            // compute warps
static_assert(kStCompute == kStBlocks, "the adapter-down work gives each warp one block");
constexpr int kStThreads = (kStCompute + 1) * 32;
constexpr int kStLut = 256 * 256;                         // 64 KB, must start the buffer
constexpr int kStXPitch = kFwdKS + 4;                     // bf16 elements per x row
constexpr int kStX = (16 * kStXPitch * 2 + 1023) / 1024 * 1024;
constexpr int kStRed = 2 * 8 * 32 * 8 * 4;                // two buffers of the odd warps' sums
constexpr int kStSmem = kStLut + kStX + kStStages * kStStage + kStRed + 1024 + 256;

template <int NT>
__global__ void __launch_bounds__(kStThreads, 1)
k_gemv_fwd_stream(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmC,
                  const uint16_t *__restrict__ X, int M, int64_t Din, int64_t Dout, ScaleSrc sc,
                  Codebook cb, int ntr, int ntiles, float *__restrict__ partial,
                  const uint16_t *__restrict__ Aad, int r, float *__restrict__ Tpart,
                  uint32_t *__restrict__ status) {
    extern __shared__ __align__(1024) uint8_t ssm[];
    const uint32_t raw = smem_u32(ssm);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = ssm + (base - raw);
    const uint8_t *lutb = gbase;                                  // [256][256 B]
    uint16_t(*sx)[kStXPitch] = reinterpret_cast<uint16_t(*)[kStXPitch]>(gbase + kStLut);
    const uint32_t ring = base + kStLut + kStX;                   // 1 KB aligned
    uint8_t *gring = gbase + kStLut + kStX;
    float *red = reinterpret_cast<float *>(gring + kStStages * kStStage);   // [2][8][32][8]
    const uint32_t bar0 = ring + kStStages * kStStage + kStRed;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kStStages + s); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + (bar0 - base) + 64);
    // the codebook goes through shared memory: indexing the parameter array
    // by a thread-dependent value would copy it to the stack
    float *cbs = reinterpret_cast<float *>(gbase + (bar0 - base) + 128);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int G = gridDim.x;
    const int t0 = (int)((int64_t)blockIdx.x * ntiles / G);
    const int t1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / G);
    const int64_t nbr = Din / 64;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) cbs[j] = cb.c[j];
        for (int s = 0; s < kStStages; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), kStCompute);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        tc::fence_proxy_async();
    }
    __syncthreads();
    if (threadIdx.x < 256) {   // table row e: 32 copies of (c[e >> 4], c[e & 15]) in bf16
        const int e = threadIdx.x;
        const uint32_t v = bf16x2_bits(cbs[e >> 4], cbs[e & 15]);
        uint4 *row = reinterpret_cast<uint4 *>(gbase + e * 256);
        const uint4 vv = make_uint4(v, v, v, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) row[(i + lane) & 7] = vv;
    }
    for (int i = threadIdx.x; i < (16 - M) * (kFwdKS / 4); i += blockDim.x) {
        const int m = M + i / (kFwdKS / 4), kc = (i % (kFwdKS / 4)) * 4;
        *reinterpret_cast<uint2 *>(&sx[m][kc]) = make_uint2(0u, 0u);
    }
    __syncthreads();
    bool ok = true;
    auto halves = [&](int z) {   // half-tiles holding data in slice z
        const int64_t nb = (Din - (int64_t)z * kFwdKS) / 64;
        return nb > 8 ? 2 : 1;
    };

    if (warp == kStCompute) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint32_t cbytes = sc.dq ? kStRows * 16 : kStRows * 8 * 4;
            int hi = 0;
            for (int tt = t0; tt < t1 && ok; ++tt) {
                const int z = tt / ntr, rt = tt % ntr;
                const int nh = halves(z);
                for (int h = 0; h < nh && ok; ++h, ++hi) {
                    const int s = hi % kStStages;
                    if (hi >= kStStages) ok = tc::mbar_wait(empty(s), ((hi / kStStages) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    const uint32_t st = ring + s * kStStage;
                    tc::mbar_expect_tx(full(s), kStHalf + cbytes);
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        tc::tma_load_2d(st + q * (kStRows * 128), &tmP,
                                        z * (kFwdKS / 2) + h * 256 + 128 * q, rt * kStRows, full(s));
                    if (sc.dq)   // the whole slice's 16 codes per row, read by both halves
                        tc::tma_load_2d(st + kStHalf, &tmC, z * kStBlocks, rt * kStRows, full(s));
                    else
                        tc::tma_load_2d(st + kStHalf, &tmC, z * kStBlocks + 8 * h, rt * kStRows, full(s));
                }
            }
            if (!ok) *abort_flag = 1;
        }
    } else {
        // ---------------------------------------------------------- compute warps
        // lookup address = (byte << 8) | 4 * lane, from one permute
        const uint32_t lanebits = 4u * lane;
        auto lookup = [&](uint32_t word, int k) -> uint32_t {
            const uint32_t off = __byte_perm(word, lanebits, 0x5504u | ((uint32_t)k << 4));
            return *reinterpret_cast<const uint32_t *>(lutb + off);
        };
        const int rl = (warp & 7) * 16 + g;            // rows rl and rl + 8 of the tile
        const int bpar = warp >> 3;                    // this warp's blocks: b = bpar mod 2
        // Every compute warp walks the same tiles and meets the same named
        // barriers; after a failed wait a warp keeps walking (skipping the
        // work) so that no other warp is left at a barrier.
        int prev_z = -1, hi = 0, rpar = 0;
        for (int tt = t0; tt < t1; ++tt, rpar ^= 1) {
            const int z = tt / ntr, rt = tt % ntr;
            const int64_t k0 = (int64_t)z * kFwdKS;
            const int64_t row0 = (int64_t)rt * kStRows + rl;
            const bool ok0 = row0 < Dout, ok1 = row0 + 8 < Dout;
            // with double quantization a row's 16 blocks of this slice start at a
            // multiple of 16 and so lie inside one group of 256 blocks
            float step0 = 0.f, step1 = 0.f;
            if (sc.dq) {
                if (ok0) step0 = __ldg(sc.step + ((row0 * nbr + z * kStBlocks) >> 8));
                if (ok1) step1 = __ldg(sc.step + (((row0 + 8) * nbr + z * kStBlocks) >> 8));
            }
            if (z != prev_z) {                         // stage x[:M, k0 : k0 + 1024]
                asm volatile("bar.sync 1, %0;\n" ::"n"(kStCompute * 32));
                for (int j = threadIdx.x; j < M * (kFwdKS / 4); j += kStCompute * 32) {
                    const int m = j / (kFwdKS / 4), kc = (j % (kFwdKS / 4)) * 4;
                    uint2 v = make_uint2(0u, 0u);
                    if (k0 + kc < Din) v = __ldg(reinterpret_cast<const uint2 *>(X + (int64_t)m * Din + k0 + kc));
                    *reinterpret_cast<uint2 *>(&sx[m][kc]) = v;
                }
                asm volatile("bar.sync 1, %0;\n" ::"n"(kStCompute * 32));
                prev_z = z;
            }
            const int nblk = (int)((Din - k0) / 64 < kStBlocks ? (Din - k0) / 64 : kStBlocks);
            const int nh = halves(z);
            float acc[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
            for (int h = 0; h < nh; ++h, ++hi) {
                const int s = hi % kStStages;
                if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait(full(s), (hi / kStStages) & 1, abort_flag));
                if (!ok) {
                    *abort_flag = 1;
                    continue;
                }
                const uint8_t *stg = gring + s * kStStage;
                const int hb = nblk - 8 * h < 8 ? nblk - 8 * h : 8;   // blocks in this half
                auto block = [&](int bh) {
                    // packed: box bh/4 holds rows x 128 B; this lane's 8 bytes of
                    // block bh are 16-byte chunk 2(bh%4) + t/2 (swizzled by row), half t%2
                    const int chunk = 2 * (bh & 3) + (t >> 1);
                    const uint8_t *pb = stg + (bh >> 2) * (kStRows * 128) + ((chunk ^ (rl & 7)) << 4) + 8 * (t & 1);
                    const uint2 w0 = *reinterpret_cast<const uint2 *>(pb + rl * 128);
                    const uint2 w1 = *reinterpret_cast<const uint2 *>(pb + (rl + 8) * 128);
                    float a0, a1;
                    if (sc.dq) {
                        const uint8_t *cs = stg + kStHalf;
                        a0 = __fmul_rn((float)cs[rl * 16 + 8 * h + bh], step0);
                        a1 = __fmul_rn((float)cs[(rl + 8) * 16 + 8 * h + bh], step1);
                    } else {
                        const float *as = reinterpret_cast<const float *>(stg + kStHalf);
                        a0 = as[rl * 8 + bh];
                        a1 = as[(rl + 8) * 8 + bh];
                    }
                    float tmp[NT][4];
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) tmp[n][e] = 0.f;
                    const int kx = 64 * (8 * h + bh) + 16 * t;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t x0 = q < 2 ? w0.x : w0.y;
                        const uint32_t x1 = q < 2 ? w1.x : w1.y;
                        const int i0 = (2 * q) & 3;
                        const uint32_t a[4] = {lookup(x0, i0), lookup(x1, i0), lookup(x0, i0 + 1),
                                               lookup(x1, i0 + 1)};
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            // token rows past M are zero: skip their shared loads
                            const uint2 xv = g + 8 * n < M
                                                 ? *reinterpret_cast<const uint2 *>(&sx[g + 8 * n][kx + 4 * q])
                                                 : make_uint2(0u, 0u);
                            const uint32_t bb[2] = {xv.x, xv.y};
                            mma_bf16_16816(tmp[n], a, bb);
                        }
                    }
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        acc[n][0] = fmaf(a0, tmp[n][0], acc[n][0]);
                        acc[n][1] = fmaf(a0, tmp[n][1], acc[n][1]);
                        acc[n][2] = fmaf(a1, tmp[n][2], acc[n][2]);
                        acc[n][3] = fmaf(a1, tmp[n][3], acc[n][3]);
                    }
                };
                // this warp's blocks of the half: bh = bpar, bpar + 2, ...
                if (hb == 8) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) block(2 * i + bpar);
                } else {
                    for (int bh = bpar; bh < hb; bh += 2) block(bh);
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(empty(s));
            }
            if (Aad && ok) {
                // adapter down of slice z: rank tile j16 goes to tile rt = j16 * step
                // (spread over the slice's row tiles, so over different CTAs), or
                // with fewer row tiles than rank tiles to rt = j16 mod ntr; warp w
                // takes block w (the 16 warps cover the slice's 16 blocks; blocks
                // past a ragged end write zeros)
                const int ntj = (r + 15) / 16;
                const int step = ntr >= ntj ? ntr / ntj : 1;
                for (int j16 = rt / step; rt % step == 0 && j16 < ntj; j16 += ntr) {
                    const int b = warp;
                    const int ja = 16 * j16 + g, jb = ja + 8;
                    float ta[NT][4];
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) ta[n][e] = 0.f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (b >= nblk) break;
                        const int kk = 64 * b + 16 * t + 4 * q;    // the x fragment's inputs kk..kk+3
                        const uint16_t *ak = Aad + (k0 + kk) * r;
                        uint32_t v[4][2];   // [input kk + i][rank ja / jb]
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            v[i][0] = ja < r ? __ldg(ak + i * r + ja) : 0u;
                            v[i][1] = jb < r ? __ldg(ak + i * r + jb) : 0u;
                        }
                        const uint32_t a[4] = {v[0][0] | (v[1][0] << 16), v[0][1] | (v[1][1] << 16),
                                               v[2][0] | (v[3][0] << 16), v[2][1] | (v[3][1] << 16)};
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const uint2 xv = *reinterpret_cast<const uint2 *>(&sx[g + 8 * n][kk]);
                            const uint32_t bb[2] = {xv.x, xv.y};
                            mma_bf16_16816(ta[n], a, bb);
                        }
                    }
                    // ta[n]: (rank ja, tokens 8n + 2t, +1) and (rank jb, same tokens)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int m = 8 * n + 2 * t + (e & 1);
                            const int j = e < 2 ? ja : jb;
                            if (m < M && j < r)
                                Tpart[(((int64_t)z * kStBlocks + b) * M + m) * r + j] = ta[n][e];
                        }
                }
            }
            // odd-block warps hand their sums to the even-block warps (buffer
            // rpar; the barrier of the next tile orders its reuse)
            float *rb = red + ((rpar * 8 + (warp & 7)) * 32 + lane) * 8;
            if (bpar) {
#pragma unroll
                for (int n = 0; n < NT; ++n)
                    *reinterpret_cast<float4 *>(rb + 4 * n) = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
            }
            asm volatile("bar.sync 2, %0;\n" ::"n"(kStCompute * 32));
            if (!ok || bpar) continue;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float4 o = *reinterpret_cast<const float4 *>(rb + 4 * n);
                acc[n][0] += o.x, acc[n][1] += o.y, acc[n][2] += o.z, acc[n][3] += o.w;
            }
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 8 * n + 2 * t + (e & 1);
                    const int64_t row = row0 + 8 * (e >> 1);
                    if (m < M && row < Dout) partial[((int64_t)z * M + m) * Dout + row] = acc[n][e];
                }
        }
    }
    if (!ok && status) atomicOr(status, QLORA_STATUS_TIMEOUT);
    __syncwarp();
    __syncthreads();
}

// Forward finalize with the adapter-down partials of the streamed kernel:
// T[m, j] = sum over (slice, block) of Tpart, once per CTA in a fixed order
// (and written out by the CTAs of the first column block), then
// y[m, n] = sum_split partial + s * sum_j T[m, j] B[j, n].  grid (ceil(Dout/256), M).
__global__ void __launch_bounds__(256)
k_gemv_fwd_finalize_fused(const float *__restrict__ partial, int nsplit, int M, int64_t Dout,
                          const float *__restrict__ Tpart, int r, const uint16_t *__restrict__ Bl,
                          float s, uint16_t *__restrict__ Y, float *__restrict__ T_out) {
    __shared__ float Ts[QLORA_MAX_RANK];
    __shared__ float Tg[256];
    const int m = blockIdx.y;
    // thread i sums the partials p = i / r, i / r + G, ... of rank i % r
    // (G = 256 / r groups, independent loads); the G group sums are then
    // added in group order
    const int P = kStBlocks * nsplit;
    const int G = r <= 256 ? 256 / r : 1;
    const int jr = threadIdx.x % r, grp = threadIdx.x / r;
    if (grp < G) {
        float v = 0.f;
#pragma unroll 8
        for (int p = grp; p < P; p += G) v += Tpart[((int64_t)p * M + m) * r + jr];
        Tg[threadIdx.x] = v;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < r; j += blockDim.x) {
        float v = 0.f;
        for (int q = 0; q < G; ++q) v += Tg[q * r + j];
        Ts[j] = v;
        if (blockIdx.x == 0 && T_out) T_out[(int64_t)m * r + j] = v;
    }
    __syncthreads();
    const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= Dout) return;
    float v = 0.f;
    for (int z = 0; z < nsplit; ++z) v += partial[((int64_t)z * M + m) * Dout + n];
    float ad = 0.f;
    for (int j = 0; j < r; ++j)
        ad = fmaf(Ts[j], __bfloat162float(__ushort_as_bfloat16(Bl[(int64_t)j * Dout + n])), ad);
    Y[(int64_t)m * Dout + n] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(s, ad, v)));
}

// y[m, n] = sum_split partial + s * sum_j T[m, j] B[j, n]
__global__ void k_gemv_fwd_finalize(const float *__restrict__ partial, int nsplit, int M,
                                    int64_t Dout, const float *__restrict__ T,
                                    const uint16_t *__restrict__ Bl, int r, float s,
                                    uint16_t *__restrict__ Y) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)M * Dout) return;
    const int m = (int)(i / Dout);
    const int64_t nn = i % Dout;
    float v = 0.f;
    for (int z = 0; z < nsplit; ++z) v += partial[(int64_t)z * M * Dout + i];
    float ad = 0.f;
    for (int j = 0; j < r; ++j)
        ad = fmaf(T[m * r + j], __bfloat162float(__ushort_as_bfloat16(Bl[(int64_t)j * Dout + nn])), ad);
    Y[i] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(s, ad, v)));
}

// ------------------------------------------------------------------ backward dX
// grid (Din/64, nsplit); block 256.  All warps of a CTA share one 64-wide
// column block [k0, k0+64) and split the CTA's rows: warp w owns rows
// [nc0 + 64w, nc0 + 64w + 64) in groups of 16.  In a group, lane (g, t)
// owns rows 4t..4t+3 and the 8 columns [k0 + 8g, k0 + 8g + 8).  MMA i
// (0..7) covers columns k0 + 8g' + i for g' = 0..7: the A operand is dY with
// the 16 tokens as M and the 16 rows as the reduction, the B operand the 16
// rows x 8 columns of weights.
__global__ void __launch_bounds__(kGemvWarps * 32)
k_gemv_bwd(const uint16_t *__restrict__ dY, int M, int64_t Din, int64_t Dout,
           const uint8_t *__restrict__ packed, ScaleSrc sc, Codebook cb,
           float *__restrict__ partial,      // [nsplit][M][Din] or null
           const float *__restrict__ G, const uint16_t *__restrict__ Al, int r, int pool,
           float s, uint16_t *__restrict__ dX) {
    constexpr int NS = kGemvWarps * kBwdRowsPerWarp;   // rows per CTA (512)
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint16_t(*sdy)[NS + 8] = reinterpret_cast<uint16_t(*)[NS + 8]>(smem_raw);
    float(*red)[16][64] = reinterpret_cast<float(*)[16][64]>(smem_raw + 16 * (NS + 8) * 2);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t k0 = (int64_t)blockIdx.x * 64;
    const int64_t nc0 = (int64_t)blockIdx.y * NS;
    const int64_t kb = k0 / 64;
    const int64_t nblk_row = Din / 64;

    // weight loads for the warp's 4 groups x 4 rows (one 32-bit word each)
    uint32_t wv[4][4];
    float ah[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t n = nc0 + warp * kBwdRowsPerWarp + 16 * q + 4 * t + j;
            const bool ok = n < Dout;
            wv[q][j] = ok ? __ldg(reinterpret_cast<const uint32_t *>(packed + (n * Din + k0) / 2) + g) : 0u;
            ah[q][j] = ok ? load_scale(sc, n * nblk_row + kb) : 0.f;
        }
    // stage dY[:, nc0:nc0+NS]
    for (int i = threadIdx.x; i < 16 * (NS / 8); i += blockDim.x) {
        const int m = i / (NS / 8), nc = (i % (NS / 8)) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M && nc0 + nc < Dout)
            v = __ldg(reinterpret_cast<const uint4 *>(dY + (int64_t)m * Dout + nc0 + nc));
        *reinterpret_cast<uint4 *>(&sdy[m][nc]) = v;
    }
    __syncthreads();

    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;

#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t R[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            ProdTable tab;
            build_table(ah[q][j], cb, tab);
            decode8(wv[q][j], tab, R[j]);
        }
        const int nl = warp * kBwdRowsPerWarp + 16 * q + 4 * t;
        const uint32_t a[4] = {
            *reinterpret_cast<const uint32_t *>(&sdy[g][nl]),
            *reinterpret_cast<const uint32_t *>(&sdy[g + 8][nl]),
            *reinterpret_cast<const uint32_t *>(&sdy[g][nl + 2]),
            *reinterpret_cast<const uint32_t *>(&sdy[g + 8][nl + 2])};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
            const uint32_t b[2] = {__byte_perm(R[0][i >> 1], R[1][i >> 1], sel),
                                   __byte_perm(R[2][i >> 1], R[3][i >> 1], sel)};
            mma_bf16_16816(acc[i], a, b);
        }
    }

    // acc[i]: (m = g, col slot 2t -> k = 16t + i, slot 2t+1 -> k = 16t + 8 + i), (m = g+8, ...)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        red[warp][g][16 * t + i] = acc[i][0];
        red[warp][g][16 * t + 8 + i] = acc[i][1];
        red[warp][g + 8][16 * t + i] = acc[i][2];
        red[warp][g + 8][16 * t + 8 + i] = acc[i][3];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < 16 * 64; o += blockDim.x) {
        const int m = o >> 6, kk = o & 63;
        if (m >= M) continue;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) v += red[w][m][kk];
        const int64_t k = k0 + kk;
        if (partial) {
            partial[((int64_t)blockIdx.y * M + m) * Din + k] = v;
        } else {
            float ad = 0.f;
            const int64_t ka = k / pool;
            for (int j = 0; j < r; ++j)
                ad = fmaf(G[m * r + j], __bfloat162float(__ushort_as_bfloat16(Al[ka * r + j])), ad);
            dX[(int64_t)m * Din + k] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(s / pool, ad, v)));
        }
    }
}

// ------------------------------------------------------------------ backward dX, streamed
// grid (Din / 512 slices kz, nsplit): CTA (kz, sp) reduces over its range of
// 128-row tiles of the weight, dX[m][k] for the slice's 512 inputs k.  A
// producer warp streams each tile -- the packed rows (two 128-byte-swizzled
// boxes of 128 rows x 128 bytes), the rows' scale codes and dY[:, rows] (two
// 64-column swizzled boxes of min(M, 16) token rows; the rows past M hold
// whatever the buffer held, which only reaches output rows that are never
// stored) -- through a three-stage ring.
//
// Sixteen compute warps: warp w owns the 64-block kb = w % 8 of the slice
// and the 16-row groups q = w / 8, w / 8 + 2, ... of every tile, and keeps
// its 16 tokens x 64 inputs accumulator in registers across the whole range
// (warps w and w + 8 are added once at the end).  MMA m16n8k16: the tokens
// are M, 8 inputs {8g' + i} are N (MMA i = 0..7), and the group's 16 rows are
// K, relabelled so that lane t's K slots 2t, 2t+1, 2t+8, 2t+9 are its rows
// 4t..4t+3.  Lane (g, t) reads one packed word (inputs 8g..8g+7) of each of
// its four rows, decodes it with four lookups of the byte -> bf16-pair table
// (the same table as the forward), and pairs rows with byte permutes.  The
// weights there are the bare codebook values, so the per-row block scale is
// moved onto dY: dY[m][n] * a_hat[n][kb], exactly, as a hi + lo pair of bf16
// (two MMAs), so that only the codebook's own bf16 rounding remains.
constexpr int kBsRows = 128, kBsCols = 512;
constexpr int kBsPacked = kBsRows * kBsCols / 2;           // 32 KB
constexpr int kBsScale = kBsRows * 8 * 4;                   // 4 KB (codes use 2 KB)
constexpr int kBsDy = 2 * 16 * 128;                         // two [16][64] bf16 boxes
constexpr int kBsStage = kBsPacked + kBsScale + kBsDy;      // 40 KB
constexpr int kBsStages = 3;
constexpr int kBsThreads = 17 * 32;
constexpr int kBsRed = 8 * 32 * 32 * 4;                    // odd-parity warps' sums
constexpr int kBsSmem = kStLut + kBsStages * kBsStage + kBsRed + 1024 + 256;
static_assert(kBsStage % 1024 == 0, "stages keep 1 KB swizzle alignment");

__global__ void __launch_bounds__(kBsThreads, 1)
k_gemv_bwd_stream(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmC,
                  const __grid_constant__ CUtensorMap tmD, int M, int Mb, int64_t Din, int64_t Dout,
                  ScaleSrc sc, Codebook cb, int ntn, int nsplit, float *__restrict__ partial,
                  uint32_t *__restrict__ status) {
    extern __shared__ __align__(1024) uint8_t ssm[];
    const uint32_t raw = smem_u32(ssm);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = ssm + (base - raw);
    const uint8_t *lutb = gbase;                                  // [256][256 B]
    const uint32_t ring = base + kStLut;
    uint8_t *gring = gbase + kStLut;
    float *red = reinterpret_cast<float *>(gring + kBsStages * kBsStage);   // [8][32][32]
    const uint32_t bar0 = ring + kBsStages * kBsStage + kBsRed;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kBsStages + s); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + (bar0 - base) + 64);
    float *cbs = reinterpret_cast<float *>(gbase + (bar0 - base) + 128);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int kz = blockIdx.x, sp = blockIdx.y;
    const int t0 = (int)((int64_t)sp * ntn / nsplit), t1 = (int)((int64_t)(sp + 1) * ntn / nsplit);
    const int64_t nbr = Din / 64;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) cbs[j] = cb.c[j];
        for (int s = 0; s < kBsStages; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), 16);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        tc::fence_proxy_async();
    }
    __syncthreads();
    if (threadIdx.x < 256) {   // table row e: 32 copies of (c[e >> 4], c[e & 15]) in bf16
        const int e = threadIdx.x;
        const uint32_t v = bf16x2_bits(cbs[e >> 4], cbs[e & 15]);
        uint4 *row = reinterpret_cast<uint4 *>(gbase + e * 256);
        const uint4 vv = make_uint4(v, v, v, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) row[(i + lane) & 7] = vv;
    }
    __syncthreads();
    bool ok = true;

    if (warp == 16) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint32_t cbytes = sc.dq ? kBsRows * 16 : kBsRows * 8 * 4;
            for (int i = 0, tt = t0; tt < t1 && ok; ++i, ++tt) {
                const int s = i % kBsStages;
                if (i >= kBsStages) ok = tc::mbar_wait(empty(s), ((i / kBsStages) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const uint32_t st = ring + s * kBsStage;
                const int n0 = tt * kBsRows;
                tc::mbar_expect_tx(full(s), kBsPacked + cbytes + 2 * Mb * 128);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    tc::tma_load_2d(st + q * (kBsRows * 128), &tmP, kz * (kBsCols / 2) + 128 * q, n0, full(s));
                if (sc.dq)   // 16 codes per row from the 16-aligned start; this slice's 8 at 8 * (kz % 2)
                    tc::tma_load_2d(st + kBsPacked, &tmC, 16 * (kz >> 1), n0, full(s));
                else
                    tc::tma_load_2d(st + kBsPacked, &tmC, 8 * kz, n0, full(s));
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    tc::tma_load_2d(st + kBsPacked + kBsScale + q * 2048, &tmD, n0 + 64 * q, 0, full(s));
            }
            if (!ok) *abort_flag = 1;
        }
    } else {
        // ---------------------------------------------------------- compute warps
        const uint32_t lanebits = 4u * lane;
        auto lookup = [&](uint32_t word, int k) -> uint32_t {
            const uint32_t off = __byte_perm(word, lanebits, 0x5504u | ((uint32_t)k << 4));
            return *reinterpret_cast<const uint32_t *>(lutb + off);
        };
        const int kb = warp & 7, qpar = warp >> 3;
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
        for (int i = 0, tt = t0; tt < t1; ++i, ++tt) {
            const int s = i % kBsStages;
            if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait(full(s), (i / kBsStages) & 1, abort_flag));
            if (!ok) {
                *abort_flag = 1;
                break;   // no CTA-wide barrier inside this loop
            }
            const uint8_t *stg = gring + s * kBsStage;
            const int64_t n0 = (int64_t)tt * kBsRows;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int q = 2 * qq + qpar;                 // 16-row group of the tile
                float ah[4];
                uint32_t R[4][4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int rl = 16 * q + 4 * t + j;       // tile row
                    const int64_t n = n0 + rl;
                    // packed word: bytes 32 kb + 4 g .. + 3 of the tile row (box kb / 4)
                    const int chunk = 2 * (kb & 3) + (g >> 2);
                    const uint32_t word = *reinterpret_cast<const uint32_t *>(
                        stg + (kb >> 2) * (kBsRows * 128) + rl * 128 + ((chunk ^ (rl & 7)) << 4) + 4 * (g & 3));
                    float a = 0.f;
                    if (n < Dout) {
                        if (sc.dq) {
                            const uint8_t code = stg[kBsPacked + rl * 16 + 8 * (kz & 1) + kb];
                            // the slice's blocks of row n lie in one double-quant group
                            const float step = __ldg(sc.step + (((uint32_t)n * (uint32_t)nbr +
                                                                 16u * (uint32_t)(kz >> 1)) >> 8));
                            a = __fmul_rn((float)code, step);
                        } else {
                            a = reinterpret_cast<const float *>(stg + kBsPacked)[rl * 8 + kb];
                        }
                    }
                    ah[j] = a;
#pragma unroll
                    for (int p = 0; p < 4; ++p) R[j][p] = lookup(word, p);
                }
                // A fragments: dY[token][row] * a_hat[row] as hi + lo bf16; rows 4t..4t+3
                // of the group are K slots 2t, 2t+1 (reg 0/1) and 2t+8, 2t+9 (reg 2/3)
                uint32_t ahi[4], alo[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {            // token g (h = 0) or g + 8
                    const int m = g + 8 * h;
                    const int nn = 16 * q + 4 * t;          // tile row of j = 0 (column of dY)
                    const uint8_t *dyb = stg + kBsPacked + kBsScale + (nn >> 6) * 2048 + m * 128;
                    const int cch = (nn & 63) >> 3;         // 16-byte chunk, 4 rows = 8 bytes
                    const uint2 dv = *reinterpret_cast<const uint2 *>(dyb + ((cch ^ (m & 7)) << 4) + 2 * (nn & 7));
                    const float d0 = bf16_lo(dv.x) * ah[0], d1 = bf16_hi(dv.x) * ah[1];
                    const float d2 = bf16_lo(dv.y) * ah[2], d3 = bf16_hi(dv.y) * ah[3];
                    const uint32_t h01 = bf16x2_bits(d0, d1), h23 = bf16x2_bits(d2, d3);
                    ahi[h] = h01;
                    ahi[2 + h] = h23;
                    alo[h] = bf16x2_bits(d0 - bf16_lo(h01), d1 - bf16_hi(h01));
                    alo[2 + h] = bf16x2_bits(d2 - bf16_lo(h23), d3 - bf16_hi(h23));
                }
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    const uint32_t sel = (ii & 1) ? 0x7632u : 0x5410u;
                    const uint32_t b[2] = {__byte_perm(R[0][ii >> 1], R[1][ii >> 1], sel),
                                           __byte_perm(R[2][ii >> 1], R[3][ii >> 1], sel)};
                    mma_bf16_16816(acc[ii], ahi, b);
                    mma_bf16_16816(acc[ii], alo, b);
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(empty(s));
        }
        // warps w + 8 hand their sums to warps w; columns: acc[ii] holds (token g,
        // input 16t + ii), (g, 16t + 8 + ii), (g + 8, 16t + ii), (g + 8, 16t + 8 + ii)
        float *rb = red + (kb * 32 + lane) * 32;
        if (qpar) {
#pragma unroll
            for (int ii = 0; ii < 8; ++ii)
                *reinterpret_cast<float4 *>(rb + 4 * ii) = make_float4(acc[ii][0], acc[ii][1], acc[ii][2], acc[ii][3]);
        }
        asm volatile("bar.sync 1, %0;\n" ::"n"(16 * 32));
        if (!qpar && ok) {
#pragma unroll
            for (int ii = 0; ii < 8; ++ii) {
                const float4 o = *reinterpret_cast<const float4 *>(rb + 4 * ii);
                const float v[4] = {acc[ii][0] + o.x, acc[ii][1] + o.y, acc[ii][2] + o.z, acc[ii][3] + o.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = g + 8 * (e >> 1);
                    const int64_t k = (int64_t)kz * kBsCols + 64 * kb + 16 * t + 8 * (e & 1) + ii;
                    if (m < M && k < Din) partial[((int64_t)sp * M + m) * Din + k] = v[e];
                }
            }
        }
    }
    if (!ok && status) atomicOr(status, QLORA_STATUS_TIMEOUT);
    __syncwarp();
    __syncthreads();
}

__global__ void k_gemv_bwd_finalize(const float *__restrict__ partial, int nsplit, int M,
                                    int64_t Din, const float *__restrict__ G,
                                    const uint16_t *__restrict__ Al, int r, int pool, float s,
                                    uint16_t *__restrict__ dX) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)M * Din) return;
    const int m = (int)(i / Din);
    const int64_t k = i % Din;
    float v = 0.f;
    for (int z = 0; z < nsplit; ++z) v += partial[(int64_t)z * M * Din + i];
    float ad = 0.f;
    const int64_t ka = k / pool;
    for (int j = 0; j < r; ++j)
        ad = fmaf(G[m * r + j], __bfloat162float(__ushort_as_bfloat16(Al[ka * r + j])), ad);
    dX[i] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(s / pool, ad, v)));
}

}  // namespace

size_t gemv_fwd_partial_bytes(int M, int64_t Din, int64_t Dout) {
    const int64_t nsplit = (Din + kFwdKS - 1) / kFwdKS;
    return (size_t)nsplit * M * Dout * sizeof(float);
}

// splits of the streamed backward: at most one CTA per SM over the slices
// (one CTA fits on an SM; a second wave would double the time)
static int bwd_stream_splits(int64_t Din, int64_t Dout) {
    const int64_t nkz = (Din + kBsCols - 1) / kBsCols, ntn = (Dout + kBsRows - 1) / kBsRows;
    int64_t ns = device_sms() / nkz;
    if (ns > ntn) ns = ntn;
    return (int)(ns < 1 ? 1 : ns);
}

size_t gemv_bwd_partial_bytes(int M, int64_t Din, int64_t Dout) {
    const int64_t NS = kGemvWarps * kBwdRowsPerWarp;
    int64_t nsplit = (Dout + NS - 1) / NS;
    const int64_t ns2 = bwd_stream_splits(Din, Dout);   // the streamed kernel always writes partials
    if (ns2 > nsplit) nsplit = ns2;
    return (size_t)nsplit * M * Din * sizeof(float);
}

size_t gemv_fwd_tpart_floats(int M, int64_t Din, int r) {
    const int64_t nsplit = (Din + kFwdKS - 1) / kFwdKS;
    return (size_t)nsplit * kStBlocks * M * r;
}

// With Aad set, the streamed kernel also computes the adapter-down partials
// (Tpart) and the fused finalize reduces them; if the streamed kernel cannot
// run for this weight, QLORA_EUNSUPPORTED is returned before anything is
// enqueued.  Without Aad, T is the finished adapter-down product.
int launch_gemv_fwd(const uint16_t *X, int M, const nf4_weight_t &q, const Codebook &cb,
                    const float *T, const uint16_t *Bl, int r, float s, uint16_t *Y,
                    float *partial, uint32_t *d_status, cudaStream_t st, const uint16_t *Aad,
                    float *Tpart, float *T_out) {
    const int64_t Din = q.cols, Dout = q.rows;
    ScaleSrc sc{q.absmax, q.absmax_code, q.dq_step, q.double_quant};
    const int64_t nsplit = (Din + kFwdKS - 1) / kFwdKS;
    const int64_t nbr = Din / 64;
    // streamed kernel: scale rows must be TMA-tileable (row pitch a multiple
    // of 16 bytes) and the weight at least one slice wide; else the register kernel
    bool stream = Din >= kFwdKS && (q.double_quant ? (nbr % 16 == 0) : (nbr % 4 == 0));
    CUtensorMap tmP, tmC;
    if (stream) {
        stream = tc::make_map(&tmP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                              128, kStRows, CU_TENSOR_MAP_SWIZZLE_128B);
        if (q.double_quant)
            stream = stream && tc::make_map(&tmC, q.absmax_code, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, nbr,
                                            Dout, nbr, 16, kStRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        else
            stream = stream && tc::make_map(&tmC, q.absmax, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, nbr,
                                            Dout, nbr * 4, 8, kStRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (Aad && !stream) return QLORA_EUNSUPPORTED;
    prof_begin(kProfGemv, st);
    if (stream) {
        const int ntr = (int)((Dout + kStRows - 1) / kStRows);
        const int ntiles = (int)(ntr * nsplit);
        const int grid = ntiles < device_sms() ? ntiles : device_sms();
        if (M <= 8) {
            cudaFuncSetAttribute(k_gemv_fwd_stream<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStSmem);
            k_gemv_fwd_stream<1><<<grid, kStThreads, kStSmem, st>>>(
                tmP, tmC, X, M, Din, Dout, sc, cb, ntr, ntiles, partial, Aad, r, Tpart, d_status);
        } else {
            cudaFuncSetAttribute(k_gemv_fwd_stream<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStSmem);
            k_gemv_fwd_stream<2><<<grid, kStThreads, kStSmem, st>>>(
                tmP, tmC, X, M, Din, Dout, sc, cb, ntr, ntiles, partial, Aad, r, Tpart, d_status);
        }
    } else {
        const size_t smem = 256 * 32 * 4 + 16 * (kFwdKS + 8) * 2;   // pair table + x slice
        dim3 grid((unsigned)((Dout + kFwdRows - 1) / kFwdRows), (unsigned)nsplit);
        if (M <= 8) {
            cudaFuncSetAttribute(k_gemv_fwd<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            k_gemv_fwd<1><<<grid, kGemvWarps * 32, smem, st>>>(X, M, Din, Dout, q.packed, sc, cb, partial);
        } else {
            cudaFuncSetAttribute(k_gemv_fwd<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            k_gemv_fwd<2><<<grid, kGemvWarps * 32, smem, st>>>(X, M, Din, Dout, q.packed, sc, cb, partial);
        }
    }
    prof_end(kProfGemv, st);
    QLORA_LAUNCH_CHECK();
    if (Aad) {
        dim3 fg((unsigned)((Dout + 255) / 256), (unsigned)M);
        k_gemv_fwd_finalize_fused<<<fg, 256, 0, st>>>(partial, (int)nsplit, M, Dout, Tpart, r, Bl, s, Y,
                                                     T_out);
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    const int64_t n = (int64_t)M * Dout;
    k_gemv_fwd_finalize<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, (int)nsplit, M, Dout,
                                                                     T, Bl, r, s, Y);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_gemv_bwd(const uint16_t *dY, int M, const nf4_weight_t &q, const Codebook &cb,
                    const float *G, const uint16_t *Al, int r, int pool, float s, uint16_t *dX,
                    float *partial, cudaStream_t st) {
    const int64_t Din = q.cols, Dout = q.rows;
    ScaleSrc sc{q.absmax, q.absmax_code, q.dq_step, q.double_quant};
    // streamed kernel: scale rows TMA-tileable, at least one 512-input slice and one 128-row tile
    const int64_t nbr = Din / 64;
    bool stream = Din >= kBsCols && Dout >= kBsRows && Dout * nbr < (int64_t(1) << 32) &&
                  (q.double_quant ? (nbr % 16 == 0) : (nbr % 4 == 0));
    CUtensorMap tmP, tmC, tmD;
    const int Mb = M < 16 ? M : 16;
    if (stream) {
        stream = tc::make_map(&tmP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                              128, kBsRows, CU_TENSOR_MAP_SWIZZLE_128B);
        if (q.double_quant)
            stream = stream && tc::make_map(&tmC, q.absmax_code, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, nbr,
                                            Dout, nbr, 16, kBsRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        else
            stream = stream && tc::make_map(&tmC, q.absmax, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, nbr,
                                            Dout, nbr * 4, 8, kBsRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        stream = stream && tc::make_map(&tmD, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dout, M, Dout * 2,
                                        64, Mb, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (stream) {
        const int nkz = (int)((Din + kBsCols - 1) / kBsCols), ntn = (int)((Dout + kBsRows - 1) / kBsRows);
        const int nsplit = bwd_stream_splits(Din, Dout);
        cudaFuncSetAttribute(k_gemv_bwd_stream, cudaFuncAttributeMaxDynamicSharedMemorySize, kBsSmem);
        prof_begin(kProfGemv, st);
        k_gemv_bwd_stream<<<dim3((unsigned)nkz, (unsigned)nsplit), kBsThreads, kBsSmem, st>>>(
            tmP, tmC, tmD, M, Mb, Din, Dout, sc, cb, ntn, nsplit, partial, nullptr);
        prof_end(kProfGemv, st);
        QLORA_LAUNCH_CHECK();
        const int64_t n = (int64_t)M * Din;
        k_gemv_bwd_finalize<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, nsplit, M, Din, G,
                                                                         Al, r, pool, s, dX);
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    constexpr int NS = kGemvWarps * kBwdRowsPerWarp;
    const int64_t nsplit = (Dout + NS - 1) / NS;
    const size_t smem = 16 * (NS + 8) * 2 + kGemvWarps * 16 * 64 * 4;
    cudaFuncSetAttribute(k_gemv_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((unsigned)(Din / 64), (unsigned)nsplit);
    prof_begin(kProfGemv, st);
    k_gemv_bwd<<<grid, kGemvWarps * 32, smem, st>>>(dY, M, Din, Dout, q.packed, sc, cb,
                                                    nsplit > 1 ? partial : nullptr, G, Al, r,
                                                    pool, s, dX);
    prof_end(kProfGemv, st);
    QLORA_LAUNCH_CHECK();
    if (nsplit > 1) {
        const int64_t n = (int64_t)M * Din;
        k_gemv_bwd_finalize<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, (int)nsplit, M,
                                                                         Din, G, Al, r, pool, s, dX);
        QLORA_LAUNCH_CHECK();
    }
    return QLORA_OK;
}

}  // namespace qlora
