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

// Scale words fetched ahead of use (code + step (+ group mean), or the fp32 absmax).
struct ScaleRawG {
    float f;
    float mu;
    uint32_t code;
};
__device__ __forceinline__ ScaleRawG fetch_scale_g(const ScaleSrc &s, int64_t b, bool valid) {
    ScaleRawG r{0.f, 0.f, 0u};
    if (valid) {
        if (s.dq) {
            r.code = __ldg(s.code + b);
            r.f = __ldg(s.step + (b >> 8));
            if (s.dq == QLORA_DQ_MEAN) r.mu = __ldg(s.mean + (b >> 8));
        } else {
            r.f = __ldg(s.absmax + b);
        }
    }
    return r;
}
__device__ __forceinline__ float decode_scale_g(const ScaleRawG &r, int dq) {
    return dq ? dq_decode(r.code, r.f, r.mu, dq) : r.f;
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

template <int NT, bool F16>
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
        const uint32_t v = pack2(cb.c[e >> 4], cb.c[e & 15], F16);
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
                mma16816<F16>(tmp[n], a, bb);
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
// Persistent: one CTA per SM walks a contiguous range of units (slice z of
// 1024 inputs, tile of 128 rows), numbered slice-major so that a CTA
// restages its x slice rarely.  A producer warp streams each unit as two
// half-tiles (128 rows x 256 packed bytes, two 128-byte-swizzled TMA boxes)
// through a three-stage shared-memory ring.  Its 32 lanes also decode the
// half-tile's block scales a_hat (lane l: rows l, l + 32, l + 64, l + 96, eight
// blocks each, from scale words loaded one half-tile ahead) into the stage,
// stored [block parity][row][4] so that a compute lane reads the four scales
// it needs of one row with a single 16-byte load.
//
// Sixteen compute warps: warps w and w + 8 own the same 16 rows and take the
// even and the odd 64-blocks of each half-tile, four blocks each.  The four
// blocks' MMA chains are independent (one accumulator set per block, scaled
// by its a_hat and summed afterwards).  The two warps' sums meet in shared
// memory once per unit, ordered by a barrier of those two warps alone.
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
// gathered from the row-major A) and the tokens on the N side.
constexpr int kStRows = 128, kStBlocks = 16;              // tile: 128 rows x 1024 inputs
constexpr int kStHalf = kStRows * 8 * 32;                 // half-tile packed bytes: 32 KB
constexpr int kStStage = kStHalf + 4096;                  // + a_hat [2][128][4] fp32
constexpr int kStStages = 3;
constexpr int kStCompute = 16;                            // compute warps
static_assert(kStCompute == kStBlocks, "the adapter-down work gives each warp one block");
constexpr int kStThreads = (kStCompute + 1) * 32;
constexpr int kStLut = 256 * 256;                         // 64 KB, must start the buffer
constexpr int kStXPitch = kFwdKS + 4;                     // bf16 elements per x row
constexpr int kStX = (16 * kStXPitch * 2 + 1023) / 1024 * 1024;
constexpr int kStRed = 2 * 8 * 32 * 8 * 4;                // two buffers of the odd warps' sums
constexpr int kStSmem = kStLut + kStX + kStStages * kStStage + kStRed + 1024 + 256;

template <bool DQ, int NT, bool F16>
__global__ void __launch_bounds__(kStThreads, 1)
k_gemv_fwd_stream(const __grid_constant__ CUtensorMap tmP, const uint16_t *__restrict__ X, int M,
                  int64_t Din, int64_t Dout, ScaleSrc sc, Codebook cb, int ntr, int ntiles,
                  float *__restrict__ partial, const uint16_t *__restrict__ Aad, int r,
                  float *__restrict__ Tpart, uint32_t *__restrict__ status) {
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
            tc::mbar_init(full(s), 32);
            tc::mbar_init(empty(s), kStCompute);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        tc::fence_proxy_async();
    }
    __syncthreads();
    if (threadIdx.x < 256) {   // table row e: 32 copies of (c[e >> 4], c[e & 15]) in bf16
        const int e = threadIdx.x;
        const uint32_t v = pack2(cbs[e >> 4], cbs[e & 15], F16);
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
        uint2 cw[4];        // DQ: the half's 8 codes of rows lane + 32 j
        float sf[4], smu[4];   // DQ: their second-level step (and group mean)
        float4 am[4][2];    // fp32 absmax of the same rows
        auto fetch = [&](int tt, int h) {
            const int z = tt / ntr, rt = tt % ntr;
            const int64_t kb0 = (int64_t)z * kStBlocks + 8 * h;      // first block of the half
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t n = (int64_t)rt * kStRows + lane + 32 * j;
                const bool okr = n < Dout;
                const int64_t b0 = n * nbr + kb0;
                if (DQ) {
                    // 8 | nbr: the half's 8 blocks start 8-aligned, inside one group of 256
                    cw[j] = okr ? __ldg(reinterpret_cast<const uint2 *>(sc.code + b0)) : make_uint2(0u, 0u);
                    sf[j] = okr ? __ldg(sc.step + (b0 >> 8)) : 0.f;
                    smu[j] = okr && sc.dq == QLORA_DQ_MEAN ? __ldg(sc.mean + (b0 >> 8)) : 0.f;
                } else {
                    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 *p = reinterpret_cast<const float4 *>(sc.absmax + b0);
                    am[j][0] = okr ? __ldg(p) : z4;
                    am[j][1] = (okr && kb0 + 4 < nbr) ? __ldg(p + 1) : z4;
                }
            }
        };
        int hi = 0;
        if (t0 < t1) fetch(t0, 0);
        for (int tt = t0; tt < t1 && ok; ++tt) {
            const int z = tt / ntr, rt = tt % ntr;
            const int nh = halves(z);
            for (int h = 0; h < nh; ++h, ++hi) {
                const int s = hi % kStStages;
                if (hi >= kStStages)
                    ok = __all_sync(0xffffffffu, tc::mbar_wait(empty(s), ((hi / kStStages) & 1) ^ 1, abort_flag));
                if (!ok) break;
                const uint32_t st = ring + s * kStStage;
                if (lane == 0) {
                    tc::mbar_expect_tx_only(full(s), kStHalf);
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        tc::tma_load_2d(st + q * (kStRows * 128), &tmP,
                                        z * (kFwdKS / 2) + h * 256 + 128 * q, rt * kStRows, full(s));
                }
                float4 *ah = reinterpret_cast<float4 *>(gring + s * kStStage + kStHalf);   // [2][128]
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float4 ev, od;   // blocks 0, 2, 4, 6 and 1, 3, 5, 7 of the half
                    if (DQ) {
                        const uint32_t x = cw[j].x, y = cw[j].y;
                        const float f = sf[j], mu = smu[j];
                        const int k = sc.dq;
                        // rows of scale-less padding (past Dout) decode to 0 or mu * 0: harmless
                        ev = make_float4(dq_decode(x & 0xffu, f, mu, k), dq_decode((x >> 16) & 0xffu, f, mu, k),
                                         dq_decode(y & 0xffu, f, mu, k), dq_decode((y >> 16) & 0xffu, f, mu, k));
                        od = make_float4(dq_decode((x >> 8) & 0xffu, f, mu, k), dq_decode(x >> 24, f, mu, k),
                                         dq_decode((y >> 8) & 0xffu, f, mu, k), dq_decode(y >> 24, f, mu, k));
                    } else {
                        const float4 a0 = am[j][0], a1 = am[j][1];
                        ev = make_float4(a0.x, a0.z, a1.x, a1.z);
                        od = make_float4(a0.y, a0.w, a1.y, a1.w);
                    }
                    ah[lane + 32 * j] = ev;
                    ah[kStRows + lane + 32 * j] = od;
                }
                tc::mbar_arrive(full(s));
                if (h + 1 < nh) fetch(tt, h + 1);
                else if (tt + 1 < t1) fetch(tt + 1, 0);
            }
        }
        if (!ok && lane == 0) *abort_flag = 1;
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
        const uint32_t pair_bar = 8u + (uint32_t)(warp & 7);   // named barrier of warps w, w + 8
        // packed bytes of block bh = 2i + bpar of row rl: box bh / 4 holds rows x 128 B;
        // this lane's 8 bytes are 16-byte chunk 2 (bh % 4) + t / 2 (swizzled by row), half t % 2
        int pko[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int bh = 2 * i + bpar;
            const int chunk = 2 * (bh & 3) + (t >> 1);
            pko[i] = (bh >> 2) * (kStRows * 128) + rl * 128 + ((chunk ^ (rl & 7)) << 4) + 8 * (t & 1);
        }
        const int aho = kStHalf + (bpar * kStRows + rl) * 16;
        // Every compute warp walks the same tiles and meets the same named
        // barriers; after a failed wait a warp keeps walking (skipping the
        // work) so that no other warp is left at a barrier.
        int prev_z = -1, hi = 0, rpar = 0;
        for (int tt = t0; tt < t1; ++tt, rpar ^= 1) {
            const int z = tt / ntr, rt = tt % ntr;
            const int64_t k0 = (int64_t)z * kFwdKS;
            const int64_t row0 = (int64_t)rt * kStRows + rl;
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
                    if (lane == 0) *abort_flag = 1;
                    continue;
                }
                const uint8_t *stg = gring + s * kStStage;
                // blocks past a ragged end hold zero-filled packed bytes, a zero
                // scale and zero x: they add nothing
                const float4 s0 = *reinterpret_cast<const float4 *>(stg + aho);
                const float4 s1 = *reinterpret_cast<const float4 *>(stg + aho + 8 * 16);
                uint2 w0[4], w1[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    w0[i] = *reinterpret_cast<const uint2 *>(stg + pko[i]);
                    w1[i] = *reinterpret_cast<const uint2 *>(stg + pko[i] + 8 * 128);
                }
                float tmp[4][NT][4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) tmp[i][n][e] = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t x0 = q < 2 ? w0[i].x : w0[i].y;
                        const uint32_t x1 = q < 2 ? w1[i].x : w1[i].y;
                        const int i0 = (2 * q) & 3;
                        const uint32_t a[4] = {lookup(x0, i0), lookup(x1, i0), lookup(x0, i0 + 1),
                                               lookup(x1, i0 + 1)};
                        const int kx = 64 * (8 * h + 2 * i + bpar) + 16 * t + 4 * q;
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            // token rows past M are zero: skip their shared loads
                            const uint2 xv = g + 8 * n < M
                                                 ? *reinterpret_cast<const uint2 *>(&sx[g + 8 * n][kx])
                                                 : make_uint2(0u, 0u);
                            const uint32_t bb[2] = {xv.x, xv.y};
                            mma16816<F16>(tmp[i][n], a, bb);
                        }
                    }
                }
                const float c0[4] = {s0.x, s0.y, s0.z, s0.w}, c1[4] = {s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        acc[n][0] = fmaf(c0[i], tmp[i][n][0], acc[n][0]);
                        acc[n][1] = fmaf(c0[i], tmp[i][n][1], acc[n][1]);
                        acc[n][2] = fmaf(c1[i], tmp[i][n][2], acc[n][2]);
                        acc[n][3] = fmaf(c1[i], tmp[i][n][3], acc[n][3]);
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
                            mma16816<F16>(ta[n], a, bb);
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
            // rpar; the pair's barrier of the next unit orders its reuse)
            float *rb = red + ((rpar * 8 + (warp & 7)) * 32 + lane) * 8;
            if (bpar) {
#pragma unroll
                for (int n = 0; n < NT; ++n)
                    *reinterpret_cast<float4 *>(rb + 4 * n) = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
            }
            asm volatile("bar.sync %0, 64;\n" ::"r"(pair_bar) : "memory");
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
                          float s, uint16_t *__restrict__ Y, float *__restrict__ T_out, bool f16) {
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
        ad = fmaf(Ts[j], dec16(Bl[(int64_t)j * Dout + n], f16), ad);
    Y[(int64_t)m * Dout + n] = enc16(fmaf(s, ad, v), f16);
}

// y[m, n] = sum_split partial + s * sum_j T[m, j] B[j, n]
__global__ void k_gemv_fwd_finalize(const float *__restrict__ partial, int nsplit, int M,
                                    int64_t Dout, const float *__restrict__ T,
                                    const uint16_t *__restrict__ Bl, int r, float s,
                                    uint16_t *__restrict__ Y, bool f16) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)M * Dout) return;
    const int m = (int)(i / Dout);
    const int64_t nn = i % Dout;
    float v = 0.f;
    for (int z = 0; z < nsplit; ++z) v += partial[(int64_t)z * M * Dout + i];
    float ad = 0.f;
    for (int j = 0; j < r; ++j)
        ad = fmaf(T[m * r + j], dec16(Bl[(int64_t)j * Dout + nn], f16), ad);
    Y[i] = enc16(fmaf(s, ad, v), f16);
}

// ------------------------------------------------------------------ backward dX
// grid (Din/64, nsplit); block 256.  All warps of a CTA share one 64-wide
// column block [k0, k0+64) and split the CTA's rows: warp w owns rows
// [nc0 + 64w, nc0 + 64w + 64) in groups of 16.  In a group, lane (g, t)
// owns rows 4t..4t+3 and the 8 columns [k0 + 8g, k0 + 8g + 8).  MMA i
// (0..7) covers columns k0 + 8g' + i for g' = 0..7: the A operand is dY with
// the 16 tokens as M and the 16 rows as the reduction, the B operand the 16
// rows x 8 columns of weights.
template <bool F16>
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
            build_table(ah[q][j], cb, tab, F16);
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
            mma16816<F16>(acc[i], a, b);
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
                ad = fmaf(G[m * r + j], dec16(Al[ka * r + j], F16), ad);
            dX[(int64_t)m * Din + k] = enc16(fmaf(s / pool, ad, v), F16);
        }
    }
}

// ------------------------------------------------------------------ backward dX, streamed
// Work units are (slice kz of 512 inputs, tile of 128 weight rows), numbered
// slice-major: u = kz * ntn + tile.  CTA c of G takes the contiguous units
// [c T / G, (c + 1) T / G) of the T = nkz * ntn, so every SM gets the same
// share of the weight whatever its shape.  Inside one slice a CTA's warps
// keep dX[:, slice] in registers over its tiles and flush it to a partial
// slot when the slice changes or the range ends; the slot of CTA c for slice
// kz is c - owner(kz * ntn), owner(u) being the CTA whose range holds unit u.
//
// Producer warp, per unit: lane 0 starts the TMA copies of the packed rows
// (two 128-byte-swizzled boxes of 128 rows x 128 bytes) and of dY[:, rows]
// (two 64-column boxes of min(M, 16) token rows; the rows past M hold
// whatever the buffer held and only reach output rows that are never
// stored).  All 32 lanes decode the block scales a_hat of their four rows
// 4l..4l+3 for the slice's eight blocks, from scale words loaded one unit
// ahead, store them [block][row] into the stage and arrive.
//
// Sixteen compute warps: warp w owns the 64-input block kb = w % 8 of the
// slice and the 16-row groups q = w / 8, w / 8 + 2, ... of every tile.  MMA
// m16n8k16: the tokens are M, 8 inputs {8g' + i} are N (MMA i = 0..7), the
// group's 16 rows are K, relabelled so that lane t's K slots 2t, 2t+1, 2t+8,
// 2t+9 are its rows 4t..4t+3.  The A operand is d = dY[m][n] a_hat[n][kb]
// as an unevaluated pair of bf16 terms hi + lo (about 16 significant bits):
// the row's block scale rides on dY.  With M <= 8 the lo terms fill the
// MMA's empty token rows 8..15 and are added to rows 0..7 at the flush; with
// more tokens a second MMA takes them.  For B, lane (g, t) reads
// one packed word (inputs 8g..8g+7) of each of its four rows; interleaving
// the nibbles of rows 4t and 4t+1 (and of 4t+2 and 4t+3) gives bytes holding
// one input of both rows, and one lookup of the byte -> bf16-pair table (the
// forward's) turns each such byte into the B register (row 4t, row 4t+1) of
// that input.
constexpr int kBsRows = 128, kBsCols = 512;
constexpr int kBsPacked = kBsRows * kBsCols / 2;           // 32 KB
constexpr int kBsDy = 2 * 16 * 128;                         // two [16][64] bf16 boxes
constexpr int kBsScale = 8 * kBsRows * 4;                   // a_hat [8 blocks][128 rows] fp32
constexpr int kBsStage = kBsPacked + kBsDy + kBsScale;      // 40 KB
constexpr int kBsStages = 3;
constexpr int kBsThreads = 17 * 32;
constexpr int kBsRed = 8 * 32 * 32 * 4;                    // odd-parity warps' sums
constexpr int kBsSmem = kStLut + kBsStages * kBsStage + kBsRed + 1024 + 256;
static_assert(kBsStage % 1024 == 0, "stages keep 1 KB swizzle alignment");

// (r0, r1) = (a0 op b0, a1 op b1) as one packed fp32x2 operation, each lane rounded as
// the scalar operation would be.
__device__ __forceinline__ void mul2_pair(float a0, float a1, float b0, float b1, float &r0, float &r1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void sub2_pair(float a0, float a1, float b0, float b1, float &r0, float &r1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// dY pair v (two 16-bit values of the compute dtype) times two scales, as
// hi + lo pairs of that dtype: hi = RN(d), lo = RN(d - hi), d = RN32(dY * a_hat).
// The two products and the two differences each take one packed operation.
template <bool F16>
__device__ __forceinline__ void split_scaled(uint32_t v, float s0, float s1, uint32_t &hi, uint32_t &lo) {
    float d0, d1, e0, e1;
    mul2_pair(lo16(v, F16), hi16(v, F16), s0, s1, d0, d1);
    hi = pack2(d0, d1, F16);
    sub2_pair(d0, d1, lo16(hi, F16), hi16(hi, F16), e0, e1);
    lo = pack2(e0, e1, F16);
}

// The CTA (of G, over T units) whose contiguous range holds unit u.
__host__ __device__ __forceinline__ int64_t unit_owner(int64_t u, int64_t G, int64_t T) {
    return ((u + 1) * G - 1) / T;
}

template <bool DQ, int MT, bool F16>
__global__ void __launch_bounds__(kBsThreads, 1)
k_gemv_bwd_stream(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmD,
                  int M, int Mb, int64_t Din, int64_t Dout, ScaleSrc sc, Codebook cb, int ntn,
                  int nkz, int nslot, float *__restrict__ partial, uint32_t *__restrict__ status) {
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
    const int64_t T = (int64_t)nkz * ntn, G = gridDim.x, c = blockIdx.x;
    const int64_t u0 = c * T / G, u1 = (c + 1) * T / G;
    const int64_t nbr = Din / 64;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) cbs[j] = cb.c[j];
        for (int s = 0; s < kBsStages; ++s) {
            tc::mbar_init(full(s), 32);
            tc::mbar_init(empty(s), 16);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        tc::fence_proxy_async();
    }
    __syncthreads();
    if (threadIdx.x < 256) {   // table row e: 32 copies of (c[e >> 4], c[e & 15]) in bf16
        const int e = threadIdx.x;
        const uint32_t v = pack2(cbs[e >> 4], cbs[e & 15], F16);
        uint4 *row = reinterpret_cast<uint4 *>(gbase + e * 256);
        const uint4 vv = make_uint4(v, v, v, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) row[(i + lane) & 7] = vv;
    }
    __syncthreads();
    bool ok = true;

    if (warp == 16) {
        // ---------------------------------------------------------- producer
        uint2 cw[4];        // DQ: the 8 codes of rows 4l + j in this slice
        float sf[4], smu[4];   // DQ: their second-level step (and group mean)
        float4 am[4][2];    // fp32 absmax of rows 4l + j
        auto fetch = [&](int64_t u) {
            const int64_t kz = u / ntn, n0 = (u % ntn) * kBsRows;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t n = n0 + 4 * lane + j;
                const bool okr = n < Dout;
                const int64_t b0 = n * nbr + 8 * kz;
                if (DQ) {
                    // 8 | nbr: the slice's 8 blocks start 8-aligned, inside one group of 256
                    cw[j] = okr ? __ldg(reinterpret_cast<const uint2 *>(sc.code + b0)) : make_uint2(0u, 0u);
                    sf[j] = okr ? __ldg(sc.step + (b0 >> 8)) : 0.f;
                    smu[j] = okr && sc.dq == QLORA_DQ_MEAN ? __ldg(sc.mean + (b0 >> 8)) : 0.f;
                } else {
                    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 *p = reinterpret_cast<const float4 *>(sc.absmax + b0);
                    am[j][0] = okr ? __ldg(p) : z4;
                    am[j][1] = (okr && 8 * kz + 4 < nbr) ? __ldg(p + 1) : z4;
                }
            }
        };
        int64_t i = 0;
        if (u0 < u1) fetch(u0);
        for (int64_t u = u0; u < u1; ++u, ++i) {
            const int s = (int)(i % kBsStages);
            if (i >= kBsStages)
                ok = __all_sync(0xffffffffu, tc::mbar_wait(empty(s), (int)((i / kBsStages) & 1) ^ 1, abort_flag));
            if (!ok) break;
            const int kz = (int)(u / ntn), n0 = (int)(u % ntn) * kBsRows;
            const uint32_t st = ring + s * kBsStage;
            if (lane == 0) {
                tc::mbar_expect_tx_only(full(s), kBsPacked + 2 * Mb * 128);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    tc::tma_load_2d(st + q * (kBsRows * 128), &tmP, kz * (kBsCols / 2) + 128 * q, n0, full(s));
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    tc::tma_load_2d(st + kBsPacked + q * 2048, &tmD, n0 + 64 * q, 0, full(s));
            }
            uint8_t *ah = gring + s * kBsStage + kBsPacked + kBsDy;
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) {
                float v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (DQ) {
                        const uint32_t word = kb < 4 ? cw[j].x : cw[j].y;
                        v[j] = dq_decode((word >> (8 * (kb & 3))) & 0xffu, sf[j], smu[j], sc.dq);
                    } else {
                        const float4 a = am[j][kb >> 2];
                        v[j] = (kb & 3) == 0 ? a.x : (kb & 3) == 1 ? a.y : (kb & 3) == 2 ? a.z : a.w;
                    }
                }
                *reinterpret_cast<float4 *>(ah + kb * (kBsRows * 4) + 16 * lane) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
            tc::mbar_arrive(full(s));
            if (u + 1 < u1) fetch(u + 1);
        }
        if (!ok && lane == 0) *abort_flag = 1;
    } else {
        // ---------------------------------------------------------- compute warps
        const uint32_t lanebits = 4u * lane;
        auto lookup = [&](uint32_t word, int k) -> uint32_t {
            const uint32_t off = __byte_perm(word, lanebits, 0x5504u | ((uint32_t)k << 4));
            return *reinterpret_cast<const uint32_t *>(lutb + off);
        };
        const int kb = warp & 7, qpar = warp >> 3;
        // stage offsets of this lane's data; group q = 2 qq + qpar adds qq * 4096
        // (packed), qq * 128 (a_hat) and, for dY, box qq / 2 and chunk 4 (qq % 2)
        int pko[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int chunk = 2 * (kb & 3) + (g >> 2);
            pko[j] = (kb >> 2) * (kBsRows * 128) + (16 * qpar + 4 * t + j) * 128 +
                     ((chunk ^ ((4 * t + j) & 7)) << 4) + 4 * (g & 3);
        }
        const int aho = kBsPacked + kBsDy + (kb * kBsRows + 16 * qpar + 4 * t) * 4;
        int dyo[2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
            dyo[h] = kBsPacked + g * 128 + (((4 * h + 2 * qpar + (t >> 1)) ^ g) << 4) + 8 * (t & 1);
        const bool tok0 = g < M, tok1 = g + 8 < M;

        float acc[8][4];
        auto flush = [&](int64_t kz) {
            if (MT == 1) {   // rows g + 8 hold the lo terms of tokens g
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    acc[ii][0] += acc[ii][2];
                    acc[ii][1] += acc[ii][3];
                    acc[ii][2] = acc[ii][3] = 0.f;
                }
            }
            // warps w + 8 hand their sums to warps w, which write the slot; acc[ii]
            // holds (token g, input 16t + ii), (g, 16t + 8 + ii), (g + 8, 16t + ii),
            // (g + 8, 16t + 8 + ii) of block kb
            float *rb = red + (kb * 32 + lane) * 32;
            asm volatile("bar.sync 1, %0;\n" ::"n"(16 * 32));   // red free
            if (qpar) {
#pragma unroll
                for (int ii = 0; ii < 8; ++ii)
                    *reinterpret_cast<float4 *>(rb + 4 * ii) =
                        make_float4(acc[ii][0], acc[ii][1], acc[ii][2], acc[ii][3]);
            }
            asm volatile("bar.sync 1, %0;\n" ::"n"(16 * 32));
            if (!qpar && ok) {
                const int64_t slot = c - unit_owner(kz * ntn, G, T);
                float *pp = partial + (kz * nslot + slot) * (int64_t)M * kBsCols;
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    const float4 o = *reinterpret_cast<const float4 *>(rb + 4 * ii);
                    const float v[4] = {acc[ii][0] + o.x, acc[ii][1] + o.y, acc[ii][2] + o.z,
                                        acc[ii][3] + o.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int m = g + 8 * (e >> 1);
                        const int kk = 64 * kb + 16 * t + 8 * (e & 1) + ii;
                        if (m < M && kz * kBsCols + kk < Din) pp[(int64_t)m * kBsCols + kk] = v[e];
                    }
                }
            }
        };

        int64_t cur = -1;
        int64_t i = 0;
        for (int64_t u = u0; u < u1; ++u, ++i) {
            const int64_t kz = u / ntn;
            if (kz != cur) {
                if (cur >= 0) flush(cur);
#pragma unroll
                for (int ii = 0; ii < 8; ++ii)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[ii][e] = 0.f;
                cur = kz;
            }
            const int s = (int)(i % kBsStages);
            if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait(full(s), (int)((i / kBsStages) & 1), abort_flag));
            if (!ok) {
                // keep walking, without work, so that every warp meets the flush barriers
                if (lane == 0) *abort_flag = 1;
                continue;
            }
            const uint8_t *stg = gring + s * kBsStage;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const float4 ah = *reinterpret_cast<const float4 *>(stg + aho + qq * 128);
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const uint32_t *>(stg + pko[j] + qq * 4096);
                // A: d = dY[token][rows 4t..4t+3] * a_hat as hi + lo bf16 pairs
                // (hi = RN_bf16(d), lo = RN_bf16(d - hi)); rows 4t, 4t+1 in reg 0/1,
                // 4t+2, 4t+3 in reg 2/3.  With M <= 8 the lo terms take the empty
                // token rows g + 8 of the same MMA; else a second MMA carries them.
                uint32_t a[4], alo[4];
                {
                    const uint8_t *d0 = stg + dyo[qq & 1] + (qq >> 1) * 2048;
                    const uint2 v0 = tok0 ? *reinterpret_cast<const uint2 *>(d0) : make_uint2(0u, 0u);
                    split_scaled<F16>(v0.x, ah.x, ah.y, a[0], alo[0]);
                    split_scaled<F16>(v0.y, ah.z, ah.w, a[2], alo[2]);
                    if (MT == 2) {
                        const uint2 v1 = tok1 ? *reinterpret_cast<const uint2 *>(d0 + 1024) : make_uint2(0u, 0u);
                        split_scaled<F16>(v1.x, ah.x, ah.y, a[1], alo[1]);
                        split_scaled<F16>(v1.y, ah.z, ah.w, a[3], alo[3]);
                    } else {
                        a[1] = alo[0];
                        a[3] = alo[2];
                    }
                }
                // B: byte p of e01 holds input 8g + 2p of rows 4t (high nibble) and
                // 4t + 1 (low nibble); o01 the same for input 8g + 2p + 1
                const uint32_t e01 = (w[0] & 0xF0F0F0F0u) | ((w[1] >> 4) & 0x0F0F0F0Fu);
                const uint32_t o01 = ((w[0] << 4) & 0xF0F0F0F0u) | (w[1] & 0x0F0F0F0Fu);
                const uint32_t e23 = (w[2] & 0xF0F0F0F0u) | ((w[3] >> 4) & 0x0F0F0F0Fu);
                const uint32_t o23 = ((w[2] << 4) & 0xF0F0F0F0u) | (w[3] & 0x0F0F0F0Fu);
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    const uint32_t b[2] = {lookup((ii & 1) ? o01 : e01, ii >> 1),
                                           lookup((ii & 1) ? o23 : e23, ii >> 1)};
                    mma16816<F16>(acc[ii], a, b);
                    if (MT == 2) mma16816<F16>(acc[ii], alo, b);
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(empty(s));
        }
        if (cur >= 0) flush(cur);
    }
    if (!ok && status) atomicOr(status, QLORA_STATUS_TIMEOUT);
    __syncwarp();
    __syncthreads();
}

// dX[m, k] = sum over the slots of slice k / 512 of partial + (s / g) G[m, :] A[k / g, :]^T
__global__ void k_gemv_bwd_finalize(const float *__restrict__ partial, int ntn, int nkz, int Gc,
                                    int nslot, int M, int64_t Din, const float *__restrict__ G,
                                    const uint16_t *__restrict__ Al, int r, int pool, float s,
                                    uint16_t *__restrict__ dX, bool f16) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)M * Din) return;
    const int m = (int)(i / Din);
    const int64_t k = i % Din;
    const int64_t kz = k / kBsCols, kk = k % kBsCols;
    const int64_t T = (int64_t)nkz * ntn;
    const int64_t c0 = unit_owner(kz * ntn, Gc, T), c1 = unit_owner(kz * ntn + ntn - 1, Gc, T);
    float v = 0.f;
    for (int64_t sl = 0; sl <= c1 - c0; ++sl) v += partial[((kz * nslot + sl) * M + m) * kBsCols + kk];
    float ad = 0.f;
    const int64_t ka = k / pool;
    for (int j = 0; j < r; ++j)
        ad = fmaf(G[m * r + j], dec16(Al[ka * r + j], f16), ad);
    dX[i] = enc16(fmaf(s / pool, ad, v), f16);
}

// dX[m, k] = sum over nsplit partials [nsplit][M][Din] + the adapter term (register kernel)
__global__ void k_gemv_bwd_finalize_split(const float *__restrict__ partial, int nsplit, int M,
                                          int64_t Din, const float *__restrict__ G,
                                          const uint16_t *__restrict__ Al, int r, int pool, float s,
                                          uint16_t *__restrict__ dX, bool f16) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)M * Din) return;
    const int m = (int)(i / Din);
    const int64_t k = i % Din;
    float v = 0.f;
    for (int z = 0; z < nsplit; ++z) v += partial[(int64_t)z * M * Din + i];
    float ad = 0.f;
    const int64_t ka = k / pool;
    for (int j = 0; j < r; ++j)
        ad = fmaf(G[m * r + j], dec16(Al[ka * r + j], f16), ad);
    dX[i] = enc16(fmaf(s / pool, ad, v), f16);
}

}  // namespace

size_t gemv_fwd_partial_bytes(int M, int64_t Din, int64_t Dout) {
    const int64_t nsplit = (Din + kFwdKS - 1) / kFwdKS;
    return (size_t)nsplit * M * Dout * sizeof(float);
}

// Grid of the streamed backward: one CTA per SM (one fits) over the
// T = nkz * ntn units, and the most CTAs that share one slice (its slots).
struct BwdPlan {
    int nkz, ntn, G, nslot;
};
static BwdPlan bwd_plan(int64_t Din, int64_t Dout) {
    BwdPlan p;
    p.nkz = (int)((Din + kBsCols - 1) / kBsCols);
    p.ntn = (int)((Dout + kBsRows - 1) / kBsRows);
    const int64_t T = (int64_t)p.nkz * p.ntn;
    p.G = (int)(T < device_sms() ? T : device_sms());
    int64_t mx = 1;
    for (int64_t kz = 0; kz < p.nkz; ++kz) {
        const int64_t d = unit_owner(kz * p.ntn + p.ntn - 1, p.G, T) - unit_owner(kz * p.ntn, p.G, T) + 1;
        if (d > mx) mx = d;
    }
    p.nslot = (int)mx;
    return p;
}

size_t gemv_bwd_partial_bytes(int M, int64_t Din, int64_t Dout) {
    const int64_t NS = kGemvWarps * kBwdRowsPerWarp;
    const size_t split = (size_t)((Dout + NS - 1) / NS) * M * Din * sizeof(float);
    const BwdPlan p = bwd_plan(Din, Dout);
    const size_t slots = (size_t)p.nkz * p.nslot * M * kBsCols * sizeof(float);
    return split > slots ? split : slots;
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
                    float *partial, uint32_t *d_status, cudaStream_t st, bool f16, const uint16_t *Aad,
                    float *Tpart, float *T_out) {
    const int64_t Din = q.cols, Dout = q.rows;
    const ScaleSrc sc = scale_src(q);
    const int64_t nsplit = (Din + kFwdKS - 1) / kFwdKS;
    const int64_t nbr = Din / 64;
    // streamed kernel: the weight at least one slice wide; the producer reads a
    // row's 8 scale codes of a half-tile as one aligned 8-byte word (8 | Din/64),
    // or its fp32 absmax as 16-byte words (4 | Din/64); else the register kernel
    bool stream = Din >= kFwdKS &&
                  (q.double_quant ? (nbr % 8 == 0 && (reinterpret_cast<uintptr_t>(q.absmax_code) & 7) == 0)
                                  : (nbr % 4 == 0 && (reinterpret_cast<uintptr_t>(q.absmax) & 15) == 0));
    CUtensorMap tmP;
    if (stream)
        stream = tc::make_map(&tmP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                              128, kStRows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (Aad && !stream) return QLORA_EUNSUPPORTED;
    if (stream) {
        const int ntr = (int)((Dout + kStRows - 1) / kStRows);
        const int ntiles = (int)(ntr * nsplit);
        const int grid = ntiles < device_sms() ? ntiles : device_sms();
        auto kern = f16 ? (q.double_quant ? (M > 8 ? k_gemv_fwd_stream<true, 2, true> : k_gemv_fwd_stream<true, 1, true>)
                                          : (M > 8 ? k_gemv_fwd_stream<false, 2, true> : k_gemv_fwd_stream<false, 1, true>))
                        : (q.double_quant ? (M > 8 ? k_gemv_fwd_stream<true, 2, false> : k_gemv_fwd_stream<true, 1, false>)
                                          : (M > 8 ? k_gemv_fwd_stream<false, 2, false> : k_gemv_fwd_stream<false, 1, false>));
        if (set_max_smem(reinterpret_cast<const void *>(kern), kStSmem) != cudaSuccess) return QLORA_ECUDA;
        prof_begin(kProfGemv, st);
        kern<<<grid, kStThreads, kStSmem, st>>>(tmP, X, M, Din, Dout, sc, cb, ntr, ntiles, partial, Aad, r,
                                                Tpart, d_status);
    } else {
        const int smem = 256 * 32 * 4 + 16 * (kFwdKS + 8) * 2;   // pair table + x slice
        dim3 grid((unsigned)((Dout + kFwdRows - 1) / kFwdRows), (unsigned)nsplit);
        auto kern = f16 ? (M <= 8 ? k_gemv_fwd<1, true> : k_gemv_fwd<2, true>)
                        : (M <= 8 ? k_gemv_fwd<1, false> : k_gemv_fwd<2, false>);
        if (set_max_smem(reinterpret_cast<const void *>(kern), smem) != cudaSuccess) return QLORA_ECUDA;
        prof_begin(kProfGemv, st);
        kern<<<grid, kGemvWarps * 32, smem, st>>>(X, M, Din, Dout, q.packed, sc, cb, partial);
    }
    prof_end(kProfGemv, st);
    QLORA_LAUNCH_CHECK();
    if (Aad) {
        dim3 fg((unsigned)((Dout + 255) / 256), (unsigned)M);
        k_gemv_fwd_finalize_fused<<<fg, 256, 0, st>>>(partial, (int)nsplit, M, Dout, Tpart, r, Bl, s, Y,
                                                     T_out, f16);
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    const int64_t n = (int64_t)M * Dout;
    k_gemv_fwd_finalize<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, (int)nsplit, M, Dout,
                                                                     T, Bl, r, s, Y, f16);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

int launch_gemv_bwd(const uint16_t *dY, int M, const nf4_weight_t &q, const Codebook &cb,
                    const float *G, const uint16_t *Al, int r, int pool, float s, uint16_t *dX,
                    float *partial, cudaStream_t st, bool f16) {
    const int64_t Din = q.cols, Dout = q.rows;
    const ScaleSrc sc = scale_src(q);
    // streamed kernel: at least one 512-input slice and one 128-row tile; the
    // producer reads a row's 8 scale codes of a slice as one aligned 8-byte
    // word (8 | Din/64), or its fp32 absmax as 16-byte words (4 | Din/64)
    const int64_t nbr = Din / 64;
    bool stream = Din >= kBsCols && Dout >= kBsRows &&
                  (q.double_quant ? (nbr % 8 == 0 && (reinterpret_cast<uintptr_t>(q.absmax_code) & 7) == 0)
                                  : (nbr % 4 == 0 && (reinterpret_cast<uintptr_t>(q.absmax) & 15) == 0));
    CUtensorMap tmP, tmD;
    const int Mb = M < 16 ? M : 16;
    if (stream) {
        stream = tc::make_map(&tmP, q.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Din / 2, Dout, Din / 2,
                              128, kBsRows, CU_TENSOR_MAP_SWIZZLE_128B);
        stream = stream && tc::make_map(&tmD, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dout, M, Dout * 2,
                                        64, Mb, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (stream) {
        const BwdPlan p = bwd_plan(Din, Dout);
        auto kern = f16 ? (q.double_quant ? (M > 8 ? k_gemv_bwd_stream<true, 2, true> : k_gemv_bwd_stream<true, 1, true>)
                                          : (M > 8 ? k_gemv_bwd_stream<false, 2, true> : k_gemv_bwd_stream<false, 1, true>))
                        : (q.double_quant ? (M > 8 ? k_gemv_bwd_stream<true, 2, false> : k_gemv_bwd_stream<true, 1, false>)
                                          : (M > 8 ? k_gemv_bwd_stream<false, 2, false> : k_gemv_bwd_stream<false, 1, false>));
        if (set_max_smem(reinterpret_cast<const void *>(kern), kBsSmem) != cudaSuccess) return QLORA_ECUDA;
        prof_begin(kProfGemv, st);
        kern<<<(unsigned)p.G, kBsThreads, kBsSmem, st>>>(tmP, tmD, M, Mb, Din, Dout, sc, cb, p.ntn, p.nkz,
                                                         p.nslot, partial, nullptr);
        prof_end(kProfGemv, st);
        QLORA_LAUNCH_CHECK();
        const int64_t n = (int64_t)M * Din;
        k_gemv_bwd_finalize<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            partial, p.ntn, p.nkz, p.G, p.nslot, M, Din, G, Al, r, pool, s, dX, f16);
        QLORA_LAUNCH_CHECK();
        return QLORA_OK;
    }
    constexpr int NS = kGemvWarps * kBwdRowsPerWarp;
    const int64_t nsplit = (Dout + NS - 1) / NS;
    const int smem = 16 * (NS + 8) * 2 + kGemvWarps * 16 * 64 * 4;
    auto kbr = f16 ? k_gemv_bwd<true> : k_gemv_bwd<false>;
    if (set_max_smem(reinterpret_cast<const void *>(kbr), smem) != cudaSuccess) return QLORA_ECUDA;
    dim3 grid((unsigned)(Din / 64), (unsigned)nsplit);
    prof_begin(kProfGemv, st);
    kbr<<<grid, kGemvWarps * 32, smem, st>>>(dY, M, Din, Dout, q.packed, sc, cb,
                                                    nsplit > 1 ? partial : nullptr, G, Al, r,
                                                    pool, s, dX);
    prof_end(kProfGemv, st);
    QLORA_LAUNCH_CHECK();
    if (nsplit > 1) {
        const int64_t n = (int64_t)M * Din;
        k_gemv_bwd_finalize_split<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, (int)nsplit, M,
                                                                               Din, G, Al, r, pool, s, dX, f16);
        QLORA_LAUNCH_CHECK();
    }
    return QLORA_OK;
}

}  // namespace qlora
