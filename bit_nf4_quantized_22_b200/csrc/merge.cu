// merge.cu -- adapter merge for deployment: the bf16 weight with the LoRA
// update folded in, W_eff = dequant(W4) + (alpha/r) A B, stored [Dout, Din]
// ("从 LoRA 到 QLoRA、QA-LoRA" section 2, W_eff; bitsandbytes article (CSDN)
// 12.10, merging the adapter before deployment; pooled adapter: every input
// of a group shares (A_p B)/g, same blog section 5).
//
//   W_out[n][k] = RN_bf16( w_hat[n][k] + (s/g) sum_j A[k/g][j] B[j][n] )
//
// w_hat = RN_bf16(RN32(a_hat c_q)) is the dequantized weight; the rank-r sum
// is an fp32 MMA.  HBM-bound: 0.52 bytes in and 2 bytes out per weight.
//
// grid (ceil(Dout/256), ceil(Din/256)), 16 warps.  Warp w owns rows
// [256 bx + 16 w, +16) and walks the CTA's 256 columns one 64-block at a
// time.  256 x 256 tiles keep the staged operands small next to the
// output (B^T once per CTA, A once per block of 64 columns).  MMA m16n8k16
// with the 16 rows as M, 8 columns as N and 16 ranks as K: the A operand is
// B^T, staged transposed in shared memory once per CTA; the B operand is the
// adapter A, whose 64 rows for the current block are staged (one row when
// pooled: the block shares it) with cp.async into one of two buffers while
// the previous block computes.  Row pitches of ceil64(r) + 8 elements
// (= 16 mod 128 bytes) keep the 32-bit fragment loads on distinct banks.  The accumulator fragment of lane
// (g, t) holds columns 8nt + 2t, +1 of rows g and g+8: byte 4nt + t of each
// row's 32 packed bytes, i.e. byte t of word nt, decoded in place.
#include "common.cuh"

namespace qlora {
namespace {

constexpr int kMgRows = 256, kMgCols = 256, kMgThreads = 512;

__device__ __forceinline__ int mg_pitch(int r) { return (r + 63) / 64 * 64 + 8; }

__global__ void __launch_bounds__(kMgThreads, 1)
k_merge(const uint8_t *__restrict__ packed, ScaleSrc sc, Codebook cb,
        const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, int r, int gp, float sg,
        int64_t Dout, int64_t Din, uint16_t *__restrict__ W_out) {
    extern __shared__ __align__(16) uint16_t msm[];
    const int pitch = mg_pitch(r);
    uint16_t *sBt = msm;                         // [64 rows][pitch]: B^T
    uint16_t *sA2 = msm + kMgRows * pitch;       // [2][64 inputs][pitch]: A rows of a block
    __shared__ float cbs[16];
    const int rp = (r + 15) / 16 * 16;
    const int64_t nb0 = (int64_t)blockIdx.x * kMgRows;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) cbs[j] = cb.c[j];
    }
    for (int i = threadIdx.x; i < rp * kMgRows; i += blockDim.x) {
        const int j = i / kMgRows, n = i % kMgRows;     // consecutive threads: consecutive n
        uint16_t v = 0;
        if (j < r && nb0 + n < Dout) v = B[(int64_t)j * Dout + nb0 + n];
        sBt[n * pitch + j] = v;
    }

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t ra = nb0 + 16 * warp + g, rb = ra + 8;   // this lane's two rows
    const bool vec = (r & 7) == 0 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0;
    // ranks r .. rp-1 of the staged A rows stay zero (the copies never reach them)
    for (int row = warp; row < 2 * 64; row += 16)
        for (int j = r + lane; j < rp; j += 32) sA2[row * pitch + j] = 0;
    const int64_t nbr = Din / 64;
    const uint16_t *bt0 = sBt + (16 * warp + g) * pitch + 2 * t;
    const uint16_t *bt1 = bt0 + 8 * pitch;
    const int arows = gp == 1 ? 64 : 1;              // staged A rows per block
    const int astep = gp == 1 ? 8 * pitch : 0;       // next n tile: 8 inputs on
    // A rows of block c into buffer c % 2: cp.async 16-byte pieces (r % 8 == 0,
    // A 16-byte aligned), else plain loads
    auto stage = [&](int c) {
        const int64_t kc = (int64_t)blockIdx.y * kMgCols + 64 * c;
        uint16_t *sA = sA2 + (c & 1) * 64 * pitch;
        const int64_t arow0 = kc / gp;
        if (vec) {
            const int nv = r / 8;
            for (int i = threadIdx.x; i < arows * nv; i += kMgThreads) {
                const int row = i / nv, v = i % nv;
                cp_async16(sA + row * pitch + 8 * v, A + (arow0 + row) * r + 8 * v, true);
            }
            cp_async_commit();
        } else {
            for (int row = warp; row < arows; row += 16)
                for (int j = lane; j < r; j += 32) sA[row * pitch + j] = A[(arow0 + row) * r + j];
        }
    };
    stage(0);

    for (int c = 0; c < kMgCols / 64; ++c) {
        const int64_t kc = (int64_t)blockIdx.y * kMgCols + 64 * c;   // this 64-block's first input
        if (kc >= Din) break;
        const bool next = c + 1 < kMgCols / 64 && kc + 64 < Din;
        if (c) __syncthreads();                      // block c-1's reads of buffer (c+1) % 2 done
        if (next) stage(c + 1);
        const uint16_t *sa = sA2 + (c & 1) * 64 * pitch + (gp == 1 ? g : 0) * pitch + 2 * t;
        // this lane's packed words: rows ra, rb, 32 bytes each
        uint32_t pw[2][8];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int64_t row = hr ? rb : ra;
            uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
            if (row < Dout) {
                const uint4 *src = reinterpret_cast<const uint4 *>(packed + row * (Din / 2) + kc / 2);
                lo = __ldg(src);
                hi = __ldg(src + 1);
            }
            pw[hr][0] = lo.x, pw[hr][1] = lo.y, pw[hr][2] = lo.z, pw[hr][3] = lo.w;
            pw[hr][4] = hi.x, pw[hr][5] = hi.y, pw[hr][6] = hi.z, pw[hr][7] = hi.w;
        }
        const float aha = ra < Dout ? load_scale(sc, ra * nbr + kc / 64) : 0.f;
        const float ahb = rb < Dout ? load_scale(sc, rb * nbr + kc / 64) : 0.f;
        if (vec) {
            if (next) cp_async_wait<1>();            // block c's copies landed, c+1's may fly
            else cp_async_wait<0>();
        }
        __syncthreads();                             // sA of block c (and, first time, sBt) ready
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        for (int ks = 0; ks < rp; ks += 16) {
            const uint32_t a[4] = {*reinterpret_cast<const uint32_t *>(bt0 + ks),
                                   *reinterpret_cast<const uint32_t *>(bt1 + ks),
                                   *reinterpret_cast<const uint32_t *>(bt0 + ks + 8),
                                   *reinterpret_cast<const uint32_t *>(bt1 + ks + 8)};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                // B operand: ranks ks + 2t, +1 (and +8, +9) of input kc + 8nt + g
                const uint16_t *ar = sa + nt * astep + ks;
                const uint32_t bb[2] = {*reinterpret_cast<const uint32_t *>(ar),
                                        *reinterpret_cast<const uint32_t *>(ar + 8)};
                mma_bf16_16816(acc[nt], a, bb);
            }
        }
        // epilogue: rows ra / rb, inputs kc + 8nt + 2t and +1 (byte t of word nt)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int64_t col = kc + 8 * nt + 2 * t;
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int64_t row = hr ? rb : ra;
                if (row >= Dout) continue;
                const float ah = hr ? ahb : aha;
                const uint32_t byte = (pw[hr][nt] >> (8 * t)) & 0xffu;
                const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(ah, cbs[byte >> 4])));
                const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(ah, cbs[byte & 15])));
                const float v0 = fmaf(sg, acc[nt][2 * hr], w0);
                const float v1 = fmaf(sg, acc[nt][2 * hr + 1], w1);
                *reinterpret_cast<uint32_t *>(W_out + row * Din + col) = bf16x2_bits(v0, v1);
            }
        }
    }
}

}  // namespace

size_t merge_smem_bytes(int r) { return (size_t)(kMgRows + 2 * 64) * ((r + 63) / 64 * 64 + 8) * 2; }

int launch_merge(const nf4_weight_t &q, const Codebook &cb, const uint16_t *A, const uint16_t *B,
                 int r, int gp, float s, uint16_t *W_out, cudaStream_t st) {
    const int64_t Dout = q.rows, Din = q.cols;
    if (Dout * Din == 0) return QLORA_OK;
    ScaleSrc sc{q.absmax, q.absmax_code, q.dq_step, q.double_quant};
    const size_t smem = merge_smem_bytes(r);
    cudaFuncSetAttribute(k_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((unsigned)((Dout + kMgRows - 1) / kMgRows), (unsigned)((Din + kMgCols - 1) / kMgCols));
    prof_begin(kProfMerge, st);
    k_merge<<<grid, kMgThreads, smem, st>>>(q.packed, sc, cb, A, B, r, gp, s / (float)gp, Dout, Din, W_out);
    prof_end(kProfMerge, st);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
