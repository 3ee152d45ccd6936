// merge.cu -- adapter merge for deployment: the weight with the LoRA update
// folded in, W_eff = dequant(W4) + (alpha/r) A B, stored [Dout, Din] in the
// compute dtype (bf16, or fp16)
// ("从 LoRA 到 QLoRA、QA-LoRA" section 2, W_eff; bitsandbytes article (CSDN)
// 12.10, merging the adapter before deployment; pooled adapter: every input
// of a group shares (A_p B)/g, same blog section 5).
//
//   W_out[n][k] = RN_dt( w_hat[n][k] + (s/g) sum_j A[k/g][j] B[j][n] )
//
// w_hat = RN_dt(RN32(a_hat c_q)) is the dequantized weight in the compute
// dtype dt; the rank-r sum
// is an fp32 MMA.  HBM-bound: 0.52 bytes in and 2 bytes out per weight.
//
// Persistent: one CTA of 16 warps per SM walks a contiguous range of units,
// a unit being 256 output rows x one 64-input block, row tile by row tile.
// Warp w owns rows [256 rt + 16 w, +16) of row tile rt.  MMA m16n8k16 with
// the 16 rows as M, 8 inputs as N and 16 ranks as K.
//  - The A operand is B^T: the tile's B rows (ranks x 256 outputs) are staged
//    as they lie in memory, once per row tile, and read with ldmatrix.trans.
//  - The B operand is the adapter A: the 64 rows of each unit (one row when
//    pooled: the block shares it) go by cp.async into a ring of three buffers
//    (two when the rank is too large for three), two units ahead of use, so
//    one barrier per unit both publishes a buffer and frees the oldest.
//  - The inputs of a block are permuted among the 8 MMA tiles so that lane
//    (g, t) of tile nt holds inputs 16t + 2nt and +1: each lane owns 16
//    consecutive inputs of its two rows, i.e. 8 consecutive packed bytes (one
//    8-byte load per row) and 32 consecutive output bytes (two 16-byte
//    stores).  Staged row 8nt + n holds adapter row 16(n/2) + 2nt + n%2, so
//    each tile's 8 rows are adjacent for ldmatrix.
//  - The next unit's packed bytes and scales are loaded one unit ahead.
// Row pitches of (ranks + 8) and (256 + 8) elements are odd multiples of 16
// bytes, which keeps ldmatrix's eight 16-byte rows on distinct banks.
#include "common.cuh"

namespace qlora {
namespace {

constexpr size_t kMgSmemMax = 227 * 1024 - 1024;    // opt-in limit less the static part
constexpr int kMgRows = 256, kMgThreads = 512, kMgBPitch = kMgRows + 8;

__host__ __device__ __forceinline__ int mg_rp(int r) { return (r + 15) / 16 * 16; }
__host__ __device__ __forceinline__ size_t mg_smem(int r, int nbuf) {
    return ((size_t)mg_rp(r) * kMgBPitch + (size_t)nbuf * 64 * (mg_rp(r) + 8)) * 2;
}

// Adapter row k of a block -> its staged row (tile (k/2) % 8, column 2(k/16) + k%2).
__device__ __forceinline__ int mg_slot(int k) { return 8 * ((k >> 1) & 7) + 2 * (k >> 4) + (k & 1); }

// Packed bytes and raw scale of one row of one unit: a_hat = RN32(code * f)
// (code = 1, f = absmax without double quantization; both exact as before).
struct MgRow {
    uint2 p;
    uint32_t code;
    float f;
    float mu;      // group mean (mean-offset double quantization)
};

__device__ __forceinline__ MgRow mg_load(const uint8_t *__restrict__ packed, const ScaleSrc &sc,
                                         int64_t row, int64_t Dout, int64_t Din, int64_t kc, int t) {
    MgRow m{make_uint2(0u, 0u), 0u, 0.f, 0.f};
    if (row < Dout) {
        m.p = __ldg(reinterpret_cast<const uint2 *>(packed + row * (Din / 2) + kc / 2) + t);
        const int64_t b = row * (Din / 64) + kc / 64;
        if (sc.dq) {
            m.code = __ldg(sc.code + b);
            m.f = __ldg(sc.step + (b >> 8));
            if (sc.dq == QLORA_DQ_MEAN) m.mu = __ldg(sc.mean + (b >> 8));
        } else {
            m.code = 1u;
            m.f = __ldg(sc.absmax + b);
        }
    }
    return m;
}

// B rows 0 .. rp-1 of row tile rt into sB (zeros past r and past Dout).
__device__ __forceinline__ void mg_stage_b(uint16_t *sB, const uint16_t *__restrict__ B, int rt, int r,
                                           int rp, int64_t Dout, bool bvec, int tid) {
    const int64_t n0 = (int64_t)rt * kMgRows;
    if (bvec) {   // Dout % 8 == 0 and B 16-byte aligned: whole 16-byte pieces are in or out
        for (int i = tid; i < rp * (kMgRows / 8); i += kMgThreads) {
            const int j = i / (kMgRows / 8), v = i % (kMgRows / 8);
            const bool ok = j < r && n0 + 8 * v < Dout;
            cp_async16(sB + j * kMgBPitch + 8 * v, ok ? B + (int64_t)j * Dout + n0 + 8 * v : B, ok);
        }
    } else {
        for (int i = tid; i < rp * kMgRows; i += kMgThreads) {
            const int j = i / kMgRows, n = i % kMgRows;
            sB[j * kMgBPitch + n] = (j < r && n0 + n < Dout) ? B[(int64_t)j * Dout + n0 + n] : 0;
        }
    }
    cp_async_commit();
}

// Adapter rows of 64-input block blk into buffer buf, in staged-row order.
// One group is committed even when there is no unit to stage, which keeps
// the group count.  With one 16-byte piece per thread at most (the common
// case, r <= 64), every thread moves the same piece of every unit, located
// once at the start (dst, src: element offsets; dst < 0: no piece).
struct MgCopy {
    int dst, src;
};

__device__ __forceinline__ void mg_stage_a(uint16_t *sA, const uint16_t *__restrict__ A, bool valid, int blk,
                                           int buf, int r, int gp, int pitch, bool avec, bool one,
                                           MgCopy cp, int tid) {
    if (valid) {
        const int arows = gp == 1 ? 64 : 1;
        const uint16_t *src = A + (int64_t)blk * 64 / gp * r;
        uint16_t *dst = sA + buf * 64 * pitch;
        if (one) {
            if (cp.dst >= 0) cp_async16(dst + cp.dst, src + cp.src, true);
        } else if (avec) {   // r % 8 == 0 and A 16-byte aligned
            const int nv = r / 8;
            for (int i = tid; i < arows * nv; i += kMgThreads) {
                const int k = i / nv, v = i - k * nv;
                cp_async16(dst + (gp == 1 ? mg_slot(k) : 0) * pitch + 8 * v, src + k * r + 8 * v, true);
            }
        } else {
            for (int i = tid; i < arows * r; i += kMgThreads) {
                const int k = i / r, j = i - k * r;
                dst[(gp == 1 ? mg_slot(k) : 0) * pitch + j] = src[k * r + j];
            }
        }
    }
    cp_async_commit();
}

template <bool F16>
__global__ void __launch_bounds__(kMgThreads, 1)
k_merge(const uint8_t *__restrict__ packed, ScaleSrc sc, Codebook cb,
        const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, int r, int gp, float sg,
        int64_t Dout, int64_t Din, int nbuf, uint16_t *__restrict__ W_out) {
    extern __shared__ __align__(16) uint16_t msm[];
    __shared__ float cbs[16];
    const int rp = mg_rp(r), pitch = rp + 8;
    uint16_t *sB = msm;                              // [rp ranks][kMgBPitch]: B of the row tile
    uint16_t *sA = msm + rp * kMgBPitch;             // [nbuf][64][pitch]: adapter rows of a unit
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    if (tid == 0) {   // constant indices: a dynamic index into the parameter would copy it to the stack
#pragma unroll
        for (int j = 0; j < 16; ++j) cbs[j] = cb.c[j];
    }

    const int nblk = (int)(Din / 64);
    const int64_t units = (Dout + kMgRows - 1) / kMgRows * nblk;
    const int u0 = (int)(units * blockIdx.x / gridDim.x), u1 = (int)(units * (blockIdx.x + 1) / gridDim.x);
    if (u0 >= u1) return;

    const bool bvec = (Dout & 7) == 0 && (reinterpret_cast<uintptr_t>(B) & 15u) == 0;
    const bool avec = (r & 7) == 0 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0;

    // ranks r .. rp-1 of every adapter buffer stay zero (no copy reaches them)
    for (int i = tid; i < nbuf * 64 * (rp - r); i += kMgThreads) {
        const int row = i / (rp - r), j = r + i % (rp - r);
        sA[row * pitch + j] = 0;
    }
    const int ahead = nbuf - 1;                      // units staged ahead of use
    int cur_rt = u0 / nblk;
    const int arows = gp == 1 ? 64 : 1;
    const bool one = avec && arows * (r / 8) <= kMgThreads;
    MgCopy cp{-1, 0};
    if (one && tid < arows * (r / 8)) {
        const int k = tid / (r / 8), v = tid - k * (r / 8);
        cp = MgCopy{(gp == 1 ? mg_slot(k) : 0) * pitch + 8 * v, k * r + 8 * v};
    }
    mg_stage_b(sB, B, cur_rt, r, rp, Dout, bvec, tid);
    int sblk = u0 - cur_rt * nblk;                   // block of the next unit to stage
    for (int d = 0; d < ahead; ++d) {
        mg_stage_a(sA, A, u0 + d < u1, sblk, d, r, gp, pitch, avec, one, cp, tid);
        if (++sblk == nblk) sblk = 0;
    }

    // ldmatrix row addresses of this lane (element offsets; ks and the tile pair added later)
    const int lda = (((lane >> 4) << 3) + (lane & 7)) * kMgBPitch + 16 * warp + 8 * ((lane >> 3) & 1);
    const int ldb = (gp == 1 ? (8 * (lane >> 4) + (lane & 7)) * pitch : 0) + 8 * ((lane >> 3) & 1);
    const int ldb_np = gp == 1 ? 16 * pitch : 0;

    int rt = cur_rt, cblk = u0 - cur_rt * nblk;
    MgRow nxt0, nxt1;
    {
        const int64_t ra = (int64_t)rt * kMgRows + 16 * warp + g;
        nxt0 = mg_load(packed, sc, ra, Dout, Din, 64 * (int64_t)cblk, t);
        nxt1 = mg_load(packed, sc, ra + 8, Dout, Din, 64 * (int64_t)cblk, t);
    }
    int buf = 0;
    for (int u = u0; u < u1; ++u) {
        const int64_t kc = 64 * (int64_t)cblk;
        const int64_t ra = (int64_t)rt * kMgRows + 16 * warp + g;
        const MgRow cur0 = nxt0, cur1 = nxt1;
        int nrt = rt, ncb = cblk + 1;                // the next unit
        if (ncb == nblk) ncb = 0, ++nrt;
        if (u + 1 < u1) {
            const int64_t na = (int64_t)nrt * kMgRows + 16 * warp + g;
            nxt0 = mg_load(packed, sc, na, Dout, Din, 64 * (int64_t)ncb, t);
            nxt1 = mg_load(packed, sc, na + 8, Dout, Din, 64 * (int64_t)ncb, t);
        }
        if (rt != cur_rt) {                          // new row tile: restage B
            __syncthreads();                         // every warp is past its last read of sB
            mg_stage_b(sB, B, rt, r, rp, Dout, bvec, tid);
            cp_async_wait<0>();
            cur_rt = rt;
        }
        if (ahead == 2) cp_async_wait<1>();          // this unit's rows landed; the next may fly
        else cp_async_wait<0>();
        __syncthreads();                             // ... for every thread; buffer (buf-1) is free
        mg_stage_a(sA, A, u + ahead < u1, sblk, buf == 0 ? nbuf - 1 : buf - 1, r, gp, pitch, avec, one, cp,
                   tid);
        if (++sblk == nblk) sblk = 0;

        const uint16_t *sAc = sA + buf * 64 * pitch;
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        for (int ks = 0; ks < rp; ks += 16) {
            uint32_t a[4];
            ldmatrix_x4_trans(a, sB + lda + ks * kMgBPitch);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b4[4];
                ldmatrix_x4(b4, sAc + ldb + np * ldb_np + ks);
                const uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
                mma16816<F16>(acc[2 * np], a, b0);
                mma16816<F16>(acc[2 * np + 1], a, b1);
            }
        }
        // epilogue: row ra (hr 0) / ra + 8 (hr 1), inputs kc + 16t + 2nt, +1 = byte 8t + nt
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int64_t row = ra + 8 * hr;
            if (row >= Dout) continue;
            const MgRow m = hr ? cur1 : cur0;
            const float ah = sc.dq ? dq_decode(m.code, m.f, m.mu, sc.dq) : m.f;
            uint32_t o[8];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const uint32_t byte = ((nt < 4 ? m.p.x : m.p.y) >> (8 * (nt & 3))) & 0xffu;
                // both weights rounded to the compute dtype by one paired conversion; the
                // products and the adapter fmas as packed fp32x2 pairs
                float p0, p1, y0, y1;
                mul2_rn(ah, cbs[byte >> 4], cbs[byte & 15], p0, p1);
                const uint32_t w = pack2(p0, p1, F16);
                fma2_rn(sg, acc[nt][2 * hr], acc[nt][2 * hr + 1], lo16(w, F16), hi16(w, F16), y0, y1);
                o[nt] = pack2(y0, y1, F16);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(W_out + row * Din + kc + 16 * t);
            __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
            __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
        }
        rt = nrt, cblk = ncb;
        buf = buf + 1 == nbuf ? 0 : buf + 1;
    }
    cp_async_wait<0>();                              // no copy outlives the CTA
}

}  // namespace

size_t merge_smem_bytes(int r) {
    const size_t three = mg_smem(r, 3);
    return three <= kMgSmemMax ? three : mg_smem(r, 2);
}

int launch_merge(const nf4_weight_t &q, const Codebook &cb, const uint16_t *A, const uint16_t *B,
                 int r, int gp, float s, uint16_t *W_out, cudaStream_t st, bool f16) {
    const int64_t Dout = q.rows, Din = q.cols;
    if (Dout * Din == 0) return QLORA_OK;
    const ScaleSrc sc = scale_src(q);
    const size_t smem = merge_smem_bytes(r);
    const int nbuf = smem == mg_smem(r, 3) ? 3 : 2;
    auto kern = f16 ? k_merge<true> : k_merge<false>;
    if (set_max_smem(reinterpret_cast<const void *>(kern), (int)smem) != cudaSuccess) return QLORA_ECUDA;
    const int64_t units = (Dout + kMgRows - 1) / kMgRows * (Din / 64);
    const unsigned grid = (unsigned)(units < device_sms() ? units : device_sms());
    prof_begin(kProfMerge, st);
    kern<<<grid, kMgThreads, smem, st>>>(q.packed, sc, cb, A, B, r, gp, s / (float)gp, Dout, Din,
                                            nbuf, W_out);
    prof_end(kProfMerge, st);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
