// mma_gemm.cuh -- tiled bf16 GEMM on the warp-level tensor-core path
// (mma.sync m16n8k16, fp32 accumulate) with cp.async staging.
//
//   C[p, q] = sum over segments s, t < R_s of  A_s(p, t) * B_s(t, q)
//
// Each operand is a bf16 matrix in global memory, either "t-contiguous"
// (A: element (p,t) at ptr[p*ld + t];  B: element (t,q) at ptr[q*ld + t]) or
// "index-contiguous" (A: ptr[t*ld + p];  B: ptr[t*ld + q]).  Tiles are staged
// in shared memory in their global orientation and turned into fragments by
// ldmatrix (.trans where the reduction index is the slow one).
//
// Requirements: base pointers 16-byte aligned; ld a multiple of 8; along the
// contiguous index the extent is a multiple of 8 (out-of-range chunks of 8
// are zero-filled; rows beyond the other extent are zero-filled too).
#pragma once
#include "common.cuh"

namespace qlora {

struct MmaOperand {
    const uint16_t *ptr;
    int64_t ld;
    int tcontig;
};

struct MmaSeg {
    MmaOperand a, b;
    int64_t R;          // reduction length of this segment
};

struct MmaGemmArgs {
    MmaSeg seg[2];
    int nseg;
    int64_t P, Q;       // output extent; columns q >= Q are never stored
    // direct epilogue (splits == 1 and partial == nullptr)
    float out_scale;
    float *out_f32;  int64_t f32_sp, f32_sq;          // optional fp32 output
    uint16_t *out_bf16; int64_t bf_sp, bf_sq;         // optional bf16 output
    // partial epilogue: raw fp32 sums into partial[split][P][Q]
    float *partial;
    int splits;
};

constexpr int kMmaBK = 32;
constexpr int kMmaStages = 3;
constexpr int kMmaThreads = 256;

template <int BM, int BN>
struct MmaSmem {
    // one stage holds A and B in either orientation; sized for the larger
    static constexpr int A_T = BM * (kMmaBK + 8);        // [BM][BK+8]
    static constexpr int A_N = kMmaBK * (BM + 8);        // [BK][BM+8]
    static constexpr int B_T = BN * (kMmaBK + 8);
    static constexpr int B_N = kMmaBK * (BN + 8);
    static constexpr int A_ELEMS = A_T > A_N ? A_T : A_N;
    static constexpr int B_ELEMS = B_T > B_N ? B_T : B_N;
    static constexpr int STAGE = A_ELEMS + B_ELEMS;
    static constexpr size_t BYTES = (size_t)STAGE * kMmaStages * 2;
};

template <int BM, int BN>
__device__ __forceinline__ void mma_load_tile(uint16_t *sA, uint16_t *sB, const MmaSeg &sg,
                                              int64_t p0, int64_t q0, int64_t t0, int64_t P,
                                              int64_t Q, int tid) {
    // A
    if (sg.a.tcontig) {
        constexpr int CH = BM * (kMmaBK / 8);
        for (int c = tid; c < CH; c += kMmaThreads) {
            const int row = c / (kMmaBK / 8), kc = (c % (kMmaBK / 8)) * 8;
            const int64_t p = p0 + row, t = t0 + kc;
            const bool ok = p < P && t < sg.R;
            const uint16_t *g = ok ? sg.a.ptr + p * sg.a.ld + t : sg.a.ptr;
            cp_async16(sA + row * (kMmaBK + 8) + kc, g, ok);
        }
    } else {
        constexpr int CH = kMmaBK * (BM / 8);
        for (int c = tid; c < CH; c += kMmaThreads) {
            const int row = c / (BM / 8), pc = (c % (BM / 8)) * 8;
            const int64_t t = t0 + row, p = p0 + pc;
            const bool ok = t < sg.R && p < P;
            const uint16_t *g = ok ? sg.a.ptr + t * sg.a.ld + p : sg.a.ptr;
            cp_async16(sA + row * (BM + 8) + pc, g, ok);
        }
    }
    // B
    if (sg.b.tcontig) {
        constexpr int CH = BN * (kMmaBK / 8);
        for (int c = tid; c < CH; c += kMmaThreads) {
            const int row = c / (kMmaBK / 8), kc = (c % (kMmaBK / 8)) * 8;
            const int64_t q = q0 + row, t = t0 + kc;
            const bool ok = q < Q && t < sg.R;
            const uint16_t *g = ok ? sg.b.ptr + q * sg.b.ld + t : sg.b.ptr;
            cp_async16(sB + row * (kMmaBK + 8) + kc, g, ok);
        }
    } else {
        constexpr int CH = kMmaBK * (BN / 8);
        for (int c = tid; c < CH; c += kMmaThreads) {
            const int row = c / (BN / 8), qc = (c % (BN / 8)) * 8;
            const int64_t t = t0 + row, q = q0 + qc;
            const bool ok = t < sg.R && q < Q;
            const uint16_t *g = ok ? sg.b.ptr + t * sg.b.ld + q : sg.b.ptr;
            cp_async16(sB + row * (BN + 8) + qc, g, ok);
        }
    }
}

// grid: (ceil(Q/BN), ceil(P/BM), splits).  Split z covers k-tiles
// [z*per, (z+1)*per) of the concatenated segment k-tile sequence.
template <int BM, int BN>
__global__ void __launch_bounds__(kMmaThreads)
k_mma_gemm(MmaGemmArgs args) {
    extern __shared__ __align__(16) uint16_t smem[];
    using S = MmaSmem<BM, BN>;
    constexpr int WM = BM / 4, WN = BN / 2;        // 4 x 2 warps
    constexpr int MI = WM / 16, NI = WN / 8;
    static_assert(NI % 2 == 0, "B fragments are loaded two n8 tiles at a time");

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp & 3, wn = warp >> 2;
    const int64_t p0 = (int64_t)blockIdx.y * BM, q0 = (int64_t)blockIdx.x * BN;

    // k-tile schedule over both segments
    const int64_t nk0 = (args.seg[0].R + kMmaBK - 1) / kMmaBK;
    const int64_t nk1 = args.nseg > 1 ? (args.seg[1].R + kMmaBK - 1) / kMmaBK : 0;
    const int64_t nkt = nk0 + nk1;
    const int64_t per = (nkt + args.splits - 1) / args.splits;
    const int64_t kbeg = (int64_t)blockIdx.z * per;
    const int64_t kend = kbeg + per < nkt ? kbeg + per : nkt;
    const int n_local = kend > kbeg ? (int)(kend - kbeg) : 0;

    float acc[MI][NI][4];
#pragma unroll
    for (int i = 0; i < MI; ++i)
#pragma unroll
        for (int j = 0; j < NI; ++j)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i][j][k] = 0.f;

    auto stageA = [&](int s) { return smem + s * S::STAGE; };
    auto stageB = [&](int s) { return smem + s * S::STAGE + S::A_ELEMS; };
    auto issue = [&](int i) {
        if (i < n_local) {
            const int64_t kt = kbeg + i;
            const int sidx = kt < nk0 ? 0 : 1;
            const int64_t t0 = (sidx == 0 ? kt : kt - nk0) * kMmaBK;
            mma_load_tile<BM, BN>(stageA(i % kMmaStages), stageB(i % kMmaStages),
                                  args.seg[sidx], p0, q0, t0, args.P, args.Q, tid);
        }
        cp_async_commit();
    };

#pragma unroll
    for (int s = 0; s < kMmaStages - 1; ++s) issue(s);

    for (int i = 0; i < n_local; ++i) {
        cp_async_wait<kMmaStages - 2>();
        __syncthreads();
        issue(i + kMmaStages - 1);
        const int64_t kt = kbeg + i;
        const MmaSeg &sg = args.seg[kt < nk0 ? 0 : 1];
        const uint16_t *sA = stageA(i % kMmaStages);
        const uint16_t *sB = stageB(i % kMmaStages);
#pragma unroll
        for (int kk = 0; kk < kMmaBK; kk += 16) {
            uint32_t af[MI][4], bfr[NI][2];
#pragma unroll
            for (int mi = 0; mi < MI; ++mi) {
                const int pm = wm * WM + mi * 16;
                if (sg.a.tcontig) {
                    const int row = pm + (lane & 15), col = kk + (lane >> 4) * 8;
                    ldmatrix_x4(af[mi], sA + row * (kMmaBK + 8) + col);
                } else {
                    const int row = kk + (lane & 7) + ((lane >> 4) << 3);
                    const int col = pm + ((lane >> 3) & 1) * 8;
                    ldmatrix_x4_trans(af[mi], sA + row * (BM + 8) + col);
                }
            }
#pragma unroll
            for (int nj = 0; nj < NI; nj += 2) {
                const int qn = wn * WN + nj * 8;
                uint32_t r[4];
                if (sg.b.tcontig) {
                    const int row = qn + (lane & 7) + ((lane >> 4) << 3);
                    const int col = kk + ((lane >> 3) & 1) * 8;
                    ldmatrix_x4(r, sB + row * (kMmaBK + 8) + col);
                } else {
                    const int row = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int col = qn + (lane >> 4) * 8;
                    ldmatrix_x4_trans(r, sB + row * (BN + 8) + col);
                }
                bfr[nj][0] = r[0]; bfr[nj][1] = r[1];
                bfr[nj + 1][0] = r[2]; bfr[nj + 1][1] = r[3];
            }
#pragma unroll
            for (int mi = 0; mi < MI; ++mi)
#pragma unroll
                for (int nj = 0; nj < NI; ++nj) mma_bf16_16816(acc[mi][nj], af[mi], bfr[nj]);
        }
    }
    cp_async_wait<0>();

    // epilogue: fragment (row g / g+8, cols 2t, 2t+1)
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int nj = 0; nj < NI; ++nj)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t p = p0 + wm * WM + mi * 16 + g + 8 * h;
                if (p >= args.P) continue;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int64_t q = q0 + wn * WN + nj * 8 + 2 * t4 + e;
                    if (q >= args.Q) continue;
                    const float v = acc[mi][nj][2 * h + e];
                    if (args.partial) {
                        args.partial[((int64_t)blockIdx.z * args.P + p) * args.Q + q] = v;
                    } else {
                        const float o = v * args.out_scale;
                        if (args.out_f32) args.out_f32[p * args.f32_sp + q * args.f32_sq] = o;
                        if (args.out_bf16)
                            args.out_bf16[p * args.bf_sp + q * args.bf_sq] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(o));
                    }
                }
            }
}

}  // namespace qlora
