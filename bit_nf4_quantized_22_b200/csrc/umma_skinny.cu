// umma_skinny.cu -- the rank-r adapter products on the tcgen05 tensor cores:
//
//   C[P, Q] = sum over segments s, t < R_s of  A_s(p, t) * B_s(t, q)
//
// with Q small (the adapter rank, or twice it when an fp32 operand is carried
// as bf16 hi/lo halves) and P, R large.  Used for T = u.A, G = dY.B^T,
// dA^T-free dA = u^T.G and dB^T = dY^T.T.  Each operand is loaded by TMA
// either K-major (reduction index contiguous) or MN-major (row/column index
// contiguous), so x and dY are read once, in place, in whichever orientation
// the product needs: no transpose copies.  Output is fp32 split-K partials
// [split][P][Qp] summed by the deterministic reduce kernel.
//
// CTA: 128 rows of P x N columns (N = 64/128/192/256, one UMMA of
// 128 x N x 16 per 16-deep step, accumulator in TMEM); warp 0 = TMA,
// warp 1 = MMA issuer, warps 2..5 = epilogue.  4-stage mbarrier ring.
#include "common.cuh"
#include "tcgen05.cuh"

namespace qlora {

struct SkinnySeg {
    const uint16_t *a;   // bf16
    int64_t lda;         // elements
    int a_kmajor;        // 1: A(p,t) at a[p*lda + t]; 0: at a[t*lda + p]
    const uint16_t *b;
    int64_t ldb;
    int b_kmajor;        // 1: B(t,q) at b[q*ldb + t]; 0: at b[t*ldb + q]
    int64_t qext;        // extent of B along q (rows if K-major, columns if MN-major)
    int64_t R;           // reduction length
};

namespace {
using namespace tc;

constexpr int kSBM = 128, kSBK = 64, kSThreads = 192, kSMaxStages = 8;
constexpr int kSABytes = kSBM * kSBK * 2;          // 16 KB
constexpr int kSRingBudget = 98304;                // ring bytes: two CTAs fit on an SM
// Stage = A tile + B tile (N x 64 bf16); as many stages as the budget holds.
inline int skinny_stage_bytes(int N) { return kSABytes + N * kSBK * 2; }
inline int skinny_stages(int N) {
    const int s = kSRingBudget / skinny_stage_bytes(N);
    return s < kSMaxStages ? s : kSMaxStages;
}
inline int skinny_smem_bytes(int N) { return skinny_stages(N) * skinny_stage_bytes(N) + 1024 + 256; }

struct SkinnyParams {
    int64_t P;
    int N;                 // UMMA N = columns per CTA tile
    int a_kmajor, b_kmajor;  // bit s: segment s's operand is K-major
    int nk0, nk1, per;     // k-tiles per segment, k-tiles per split
    int stages, stage_bytes;
    float *partial;        // [splits][P][Qp]
    int64_t Qp;
    uint32_t *status;
    int f16;               // operands in fp16 (else bf16)
};

__global__ void __launch_bounds__(kSThreads, 2)
k_umma_skinny(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
              const __grid_constant__ CUtensorMap tB0, const __grid_constant__ CUtensorMap tB1,
              const SkinnyParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *gen_base = smem_raw + (base - raw_addr);
    const int kSStages = p.stages, kSStageBytes = p.stage_bytes;
    const uint32_t bar0 = base + kSStages * kSStageBytes;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kSMaxStages + s); };
    const uint32_t acc_bar = bar0 + 8u * (2 * kSMaxStages);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gen_base + kSStages * kSStageBytes + 160);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gen_base + kSStages * kSStageBytes + 192);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t p0 = (int64_t)blockIdx.x * kSBM;
    const int q0 = blockIdx.y * p.N;
    const int nk = p.nk0 + p.nk1;
    const int kbeg = blockIdx.z * p.per;
    const int kend = kbeg + p.per < nk ? kbeg + p.per : nk;
    const int nloc = kend - kbeg;                      // >= 1 by construction
    const uint32_t tmem_cols = p.N <= 64 ? 64u : (p.N <= 128 ? 128u : 256u);
    const uint32_t bbytes = (uint32_t)p.N * kSBK * 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(full_bar(s), 1);
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
                     "r"(tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            for (int i = 0; i < nloc && ok; ++i) {
                const int s = i % kSStages;
                if (i >= kSStages) ok = mbar_wait(empty_bar(s), ((i / kSStages) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const int kt = kbeg + i;
                const int sg = kt < p.nk0 ? 0 : 1;
                const int t0 = (sg == 0 ? kt : kt - p.nk0) * kSBK;
                const CUtensorMap *ta = sg == 0 ? &tA0 : &tA1;
                const CUtensorMap *tb = sg == 0 ? &tB0 : &tB1;
                const uint32_t sa = base + s * kSStageBytes, sb = sa + kSABytes;
                mbar_expect_tx(full_bar(s), kSABytes + bbytes);
                if ((p.a_kmajor >> sg) & 1) {
                    tma_load_2d(sa, ta, t0, (int)p0, full_bar(s));
                } else {
                    tma_load_2d(sa, ta, (int)p0, t0, full_bar(s));
                    tma_load_2d(sa + 8192, ta, (int)p0 + 64, t0, full_bar(s));
                }
                if ((p.b_kmajor >> sg) & 1) {
                    tma_load_2d(sb, tb, t0, q0, full_bar(s));
                } else {
                    for (int a = 0; a < p.N / 64; ++a)
                        tma_load_2d(sb + a * 8192, tb, q0 + 64 * a, t0, full_bar(s));
                }
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int i = 0; i < nloc && ok; ++i) {
                const int s = i % kSStages;
                ok = mbar_wait(full_bar(s), (i / kSStages) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const int sg = (kbeg + i) < p.nk0 ? 0 : 1;
                const uint32_t sa = base + s * kSStageBytes, sb = sa + kSABytes;
                // K-major: rows of 64 k (128 B), 8-row groups 1 KB apart, a
                // 16-deep step advances 32 B.  MN-major: 64-wide atoms 8 KB
                // apart, 8 k-rows per 1 KB group, a step advances 2 KB.
                const bool akm = (p.a_kmajor >> sg) & 1, bkm = (p.b_kmajor >> sg) & 1;
                uint32_t idesc = idesc_bf16(128, (uint32_t)p.N, bkm ? 0u : 1u) | (akm ? 0u : (1u << 15));
                if (p.f16) idesc = idesc_as_fp16(idesc);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = akm ? sdesc(sa + kk * 32, 16, 1024)
                                            : sdesc(sa + kk * 2048, 8192, 1024);
                    const uint64_t bd = bkm ? sdesc(sb + kk * 32, 16, 1024)
                                            : sdesc(sb + kk * 2048, 8192, 1024);
                    umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(empty_bar(s));
            }
            if (ok) umma_commit(acc_bar);
            else *abort_flag = 1;
        }
    } else {
        ok = __all_sync(0xffffffffu, mbar_wait(acc_bar, 0, abort_flag));
        if (ok) {
            tc_fence_after();
            const int q = warp & 3;
            const int64_t prow = p0 + 32 * q + lane;
            float *dst = p.partial + ((int64_t)blockIdx.z * p.P + prow) * p.Qp;
            for (int c = 0; c < p.N / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + c * 32, v);
                if (prow < p.P) {
                    const int64_t col0 = q0 + c * 32;
                    if (col0 + 32 <= p.Qp) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            *reinterpret_cast<float4 *>(dst + col0 + 4 * i) =
                                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                    } else {
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < p.Qp) dst[col0 + i] = __uint_as_float(v[i]);
                    }
                }
            }
        } else {
            *abort_flag = 1;
        }
    }

    if (!ok && p.status) atomicOr(p.status, QLORA_STATUS_TIMEOUT);
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        for (int s = 0; s < kSStages && s < nloc; ++s) {
            const int last = ((nloc - 1 - s) / kSStages) * kSStages + s;
            for (uint32_t i = 0; i < kWaitLimit; ++i)
                if (mbar_try_wait(full_bar(s), (last / kSStages) & 1)) break;
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(tmem_cols));
    }
}

bool make_operand_map(CUtensorMap *m, const uint16_t *ptr, int64_t ld, int kmajor,
                      int64_t idx_extent, int64_t R, uint32_t idx_box) {
    if (kmajor)   // [idx][t]: inner t
        return make_map(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)R,
                        (uint64_t)idx_extent, (uint64_t)ld * 2, 64, idx_box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    return make_map(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)idx_extent, (uint64_t)R,
                    (uint64_t)ld * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

int skinny_n(int64_t Q) { return Q <= 64 ? 64 : (Q <= 128 ? 128 : (Q <= 192 ? 192 : 256)); }

// Split count and k-tiles per split for a (P, Q, total k-tiles) problem:
// about one CTA per SM, at least 4 k-tiles per split, no empty split.
void skinny_splits(int64_t P, int64_t Q, int nk, int *splits, int *per) {
    const int64_t tiles = ((P + kSBM - 1) / kSBM) * ((Q + 255) / 256);
    // two resident CTAs per SM; round down so that the grid is one wave
    // (a few CTAs over the slots would cost a whole second round)
    int64_t s = 2 * device_sms() / tiles;
    const int64_t cap = nk / 4 > 1 ? nk / 4 : 1;
    if (s > cap) s = cap;
    if (s < 1) s = 1;
    int pr = (int)((nk + s - 1) / s);
    *per = pr;
    *splits = (nk + pr - 1) / pr;
}

int skinny_k_tiles(const SkinnySeg *segs, int nseg) {
    int nk = 0;
    for (int i = 0; i < nseg; ++i) nk += (int)((segs[i].R + kSBK - 1) / kSBK);
    return nk;
}

// C[P, Q] partial sums into partial[splits][P][Qp] (Qp >= Q, multiple of 4).
int launch_umma_skinny(const SkinnySeg *segs, int nseg, int64_t P, int64_t Q, int64_t Qp,
                       float *partial, uint32_t *d_status, cudaStream_t st, bool f16) {
    if (P <= 0 || Q <= 0) return QLORA_OK;
    const int N = skinny_n(Q < 256 ? Q : 256);
    CUtensorMap tA[2], tB[2];
    SkinnyParams prm{};
    for (int i = 0; i < 2; ++i) {
        const SkinnySeg &s = segs[i < nseg ? i : 0];
        bool ok = make_operand_map(&tA[i], s.a, s.lda, s.a_kmajor, P, s.R, kSBM);
        ok = ok && make_operand_map(&tB[i], s.b, s.ldb, s.b_kmajor, s.qext, s.R, (uint32_t)N);
        if (!ok) return QLORA_EUNSUPPORTED;
        prm.a_kmajor |= (s.a_kmajor ? 1 : 0) << i;
        prm.b_kmajor |= (s.b_kmajor ? 1 : 0) << i;
    }
    prm.nk0 = (int)((segs[0].R + kSBK - 1) / kSBK);
    prm.nk1 = nseg > 1 ? (int)((segs[1].R + kSBK - 1) / kSBK) : 0;
    int splits = 1, per = 1;
    skinny_splits(P, Q, prm.nk0 + prm.nk1, &splits, &per);
    prm.P = P;
    prm.N = N;
    prm.stages = skinny_stages(N);
    prm.stage_bytes = skinny_stage_bytes(N);
    const int smem = skinny_smem_bytes(N);
    prm.per = per;
    prm.partial = partial;
    prm.Qp = Qp;
    prm.status = d_status;
    prm.f16 = f16 ? 1 : 0;
    if (set_max_smem(reinterpret_cast<const void *>(k_umma_skinny), (int)smem) != cudaSuccess) return QLORA_ECUDA;
    dim3 grid((unsigned)((P + kSBM - 1) / kSBM), (unsigned)((Q + N - 1) / N), (unsigned)splits);
    k_umma_skinny<<<grid, kSThreads, smem, st>>>(tA[0], tA[1], tB[0], tB[1], prm);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}

}  // namespace qlora
