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

size_t gemv_bwd_partial_bytes(int M, int64_t Din, int64_t Dout) {
    const int64_t NS = kGemvWarps * kBwdRowsPerWarp;
    const int64_t nsplit = (Dout + NS - 1) / NS;
    return nsplit > 1 ? (size_t)nsplit * M * Din * sizeof(float) : 0;
}

int launch_gemv_fwd(const uint16_t *X, int M, const nf4_weight_t &q, const Codebook &cb,
                    const float *T, const uint16_t *Bl, int r, float s, uint16_t *Y,
                    float *partial, cudaStream_t st) {
    const int64_t Din = q.cols, Dout = q.rows;
    ScaleSrc sc{q.absmax, q.absmax_code, q.dq_step, q.double_quant};
    const int64_t nsplit = (Din + kFwdKS - 1) / kFwdKS;
    const size_t smem = 256 * 32 * 4 + 16 * (kFwdKS + 8) * 2;   // pair table + x slice
    dim3 grid((unsigned)((Dout + kFwdRows - 1) / kFwdRows), (unsigned)nsplit);
    prof_begin(kProfGemv, st);
    if (M <= 8) {
        cudaFuncSetAttribute(k_gemv_fwd<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_gemv_fwd<1><<<grid, kGemvWarps * 32, smem, st>>>(X, M, Din, Dout, q.packed, sc, cb, partial);
    } else {
        cudaFuncSetAttribute(k_gemv_fwd<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_gemv_fwd<2><<<grid, kGemvWarps * 32, smem, st>>>(X, M, Din, Dout, q.packed, sc, cb, partial);
    }
    prof_end(kProfGemv, st);
    QLORA_LAUNCH_CHECK();
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
