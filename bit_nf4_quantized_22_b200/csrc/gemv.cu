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

constexpr int kGemvWarps = 8;
constexpr int kFwdKS = 512;          // k-slice per CTA (4 chunks of 128)
constexpr int kBwdRowsPerWarp = 64;  // 4 groups of 16 rows

// ------------------------------------------------------------------ forward
// grid (ceil(Dout/64), nsplit); block 256.  Warp w owns weight rows
// n0 = blockIdx.x*64 + 8w + g (g = lane/4); lane t = lane%4 owns the 32
// consecutive inputs [kc + 32t, kc + 32t + 32) of each 128-wide chunk.
// MMA step s uses the lane's inputs 4s..4s+3: the reduction index of the
// fragment is relabelled, identically for x and for W.
__global__ void __launch_bounds__(kGemvWarps * 32)
k_gemv_fwd(const uint16_t *__restrict__ X, int M, int64_t Din, int64_t Dout,
           const uint8_t *__restrict__ packed, ScaleSrc sc, Codebook cb,
           float *__restrict__ partial,            // [nsplit][M][Dout] or null
           const float *__restrict__ T, const uint16_t *__restrict__ Bl, int r, float s,
           uint16_t *__restrict__ Y) {
    __shared__ __align__(16) uint16_t sx[16][kFwdKS + 8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t k0 = (int64_t)blockIdx.y * kFwdKS;
    const int64_t kend = k0 + kFwdKS < Din ? k0 + kFwdKS : Din;
    const int64_t n = (int64_t)blockIdx.x * 64 + warp * 8 + g;
    const bool nvalid = n < Dout;

    // issue the weight loads first (4 chunks, 16 bytes each)
    uint4 wv[4];
    float ah[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int64_t kk = k0 + 128 * c + 32 * t;
        const bool ok = nvalid && kk < kend;
        wv[c] = ok ? __ldg(reinterpret_cast<const uint4 *>(packed + (n * Din + kk) / 2))
                   : make_uint4(0, 0, 0, 0);
        ah[c] = ok ? load_scale(sc, (n * Din + kk) / 64) : 0.f;
    }
    // stage x[:, k0:kend] (rows >= M and columns >= kend are zero)
    for (int i = threadIdx.x; i < 16 * (kFwdKS / 8); i += blockDim.x) {
        const int m = i / (kFwdKS / 8), kc = (i % (kFwdKS / 8)) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M && k0 + kc < kend)
            v = __ldg(reinterpret_cast<const uint4 *>(X + (int64_t)m * Din + k0 + kc));
        *reinterpret_cast<uint4 *>(&sx[m][kc]) = v;
    }
    __syncthreads();

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        ProdTable tab;
        build_table(ah[c], cb, tab);
        uint32_t wd[16];
        decode8(wv[c].x, tab, wd + 0);
        decode8(wv[c].y, tab, wd + 4);
        decode8(wv[c].z, tab, wd + 8);
        decode8(wv[c].w, tab, wd + 12);
        const int col = 128 * c + 32 * t;
#pragma unroll
        for (int st = 0; st < 8; ++st) {
            const uint2 xa = *reinterpret_cast<const uint2 *>(&sx[g][col + 4 * st]);
            const uint2 xb = *reinterpret_cast<const uint2 *>(&sx[g + 8][col + 4 * st]);
            const uint32_t a[4] = {xa.x, xb.x, xa.y, xb.y};
            const uint32_t b[2] = {wd[2 * st], wd[2 * st + 1]};
            mma_bf16_16816(acc, a, b);
        }
    }

    // acc: (m = g, cols 2t, 2t+1) and (m = g+8, same); col j <-> row n0 + j
    const int64_t nbase = (int64_t)blockIdx.x * 64 + warp * 8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int m = g + 8 * h;
        if (m >= M) continue;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int64_t nn = nbase + 2 * t + e;
            if (nn >= Dout) continue;
            const float v = acc[2 * h + e];
            if (partial) {
                partial[((int64_t)blockIdx.y * M + m) * Dout + nn] = v;
            } else {
                float ad = 0.f;
                for (int j = 0; j < r; ++j)
                    ad = fmaf(T[m * r + j], __bfloat162float(__ushort_as_bfloat16(Bl[(int64_t)j * Dout + nn])), ad);
                Y[(int64_t)m * Dout + nn] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(s, ad, v)));
            }
        }
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
    return nsplit > 1 ? (size_t)nsplit * M * Dout * sizeof(float) : 0;
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
    dim3 grid((unsigned)((Dout + 63) / 64), (unsigned)nsplit);
    prof_begin(kProfGemv, st);
    k_gemv_fwd<<<grid, kGemvWarps * 32, 0, st>>>(X, M, Din, Dout, q.packed, sc, cb,
                                                 nsplit > 1 ? partial : nullptr, T, Bl, r, s, Y);
    prof_end(kProfGemv, st);
    QLORA_LAUNCH_CHECK();
    if (nsplit > 1) {
        const int64_t n = (int64_t)M * Dout;
        k_gemv_fwd_finalize<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, (int)nsplit, M,
                                                                         Dout, T, Bl, r, s, Y);
        QLORA_LAUNCH_CHECK();
    }
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
