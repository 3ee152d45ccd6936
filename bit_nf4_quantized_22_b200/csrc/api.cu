// api.cu -- the extern "C" entry points declared in include/qlora.h:
// argument validation, workspace layout and kernel dispatch.
#include <cmath>
#include <mutex>
#include <unordered_map>

#include "common.cuh"

namespace qlora {
// quantize.cu
int launch_nf4_quantize(const float *W, const nf4_weight_t &q, const Codebook &cb, int zero_idx,
                        uint32_t *d_status, cudaStream_t st);
int launch_nf4_dequantize(const nf4_weight_t &q, const Codebook &cb, uint16_t *out, cudaStream_t st);
int launch_nf4_dequantize_dtype(const nf4_weight_t &q, const Codebook &cb, int dtype, void *out,
                                cudaStream_t st);
// merge.cu
int launch_merge(const nf4_weight_t &q, const Codebook &cb, const uint16_t *A, const uint16_t *B,
                 int r, int gp, float s, uint16_t *W_out, cudaStream_t st, bool f16);
// gemv.cu
size_t gemv_fwd_partial_bytes(int M, int64_t Din, int64_t Dout);
size_t gemv_bwd_partial_bytes(int M, int64_t Din, int64_t Dout);
size_t gemv_fwd_tpart_floats(int M, int64_t Din, int r);
int launch_gemv_fwd(const uint16_t *X, int M, const nf4_weight_t &q, const Codebook &cb,
                    const float *T, const uint16_t *Bl, int r, float s, uint16_t *Y,
                    float *partial, uint32_t *d_status, cudaStream_t st, bool f16,
                    const uint16_t *Aad = nullptr, float *Tpart = nullptr, float *T_out = nullptr);
int launch_gemv_bwd(const uint16_t *dY, int M, const nf4_weight_t &q, const Codebook &cb,
                    const float *G, const uint16_t *Al, int r, int pool, float s, uint16_t *dX,
                    float *partial, cudaStream_t st, bool f16);
// adapter.cu
int launch_pad_rows(const uint16_t *src, int64_t rows, int r, int rp, int rep, float mul,
                    uint16_t *dst, cudaStream_t st, bool f16);
int launch_pool_split(const uint16_t *X, int64_t M, int64_t Din, int g, int64_t ld, uint16_t *hi,
                      uint16_t *lo, cudaStream_t st, bool f16);
int launch_split_f32(const float *src, int64_t rows, int r, int rp, uint16_t *dst, cudaStream_t st,
                     bool f16);
int launch_reduce(const float *partial, int splits, int64_t P, int64_t Qp, int H, int Qv,
                  float f32_scale, float *out_f32, int64_t fsp, int64_t fsq, float bf_scale,
                  uint16_t *out_bf16, int64_t bsp, uint16_t *out_split, int64_t sp, cudaStream_t st,
                  bool f16);
// umma_skinny.cu
struct SkinnySeg {
    const uint16_t *a;
    int64_t lda;
    int a_kmajor;
    const uint16_t *b;
    int64_t ldb;
    int b_kmajor;
    int64_t qext;
    int64_t R;
};
int skinny_k_tiles(const SkinnySeg *segs, int nseg);
void skinny_splits(int64_t P, int64_t Q, int nk, int *splits, int *per);
int launch_umma_skinny(const SkinnySeg *segs, int nseg, int64_t P, int64_t Q, int64_t Qp,
                       float *partial, uint32_t *d_status, cudaStream_t st, bool f16);
// umma_gemm.cu
int launch_umma_qgemm(int mode, const uint16_t *X, int64_t M, const nf4_weight_t &q,
                      const Codebook &cb, const uint16_t *sAct, int r, const uint16_t *adapter,
                      uint16_t *Y, uint32_t *d_status, cudaStream_t st, bool f16);

namespace {

constexpr int kGemvMaxM = 16;

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 16 finite levels in [-1, 1], strictly increasing except that the zero
// level may appear twice in a row (the FP4 table's -0 and +0); zero_idx is
// the first zero, the level an all-zero block maps to.
int check_codebook(const float *cb, int *zero_idx) {
    if (!cb) return QLORA_EINVAL;
    int zi = -1;
    for (int j = 0; j < 16; ++j) {
        if (!std::isfinite(cb[j]) || cb[j] < -1.f || cb[j] > 1.f) return QLORA_EINVAL;
        if (j > 0 && !(cb[j] > cb[j - 1]) && !(cb[j] == 0.f && cb[j - 1] == 0.f)) return QLORA_EINVAL;
        if (j > 1 && cb[j] == 0.f && cb[j - 2] == 0.f) return QLORA_EINVAL;   // at most two zeros
        if (cb[j] == 0.f && zi < 0) zi = j;
    }
    if (zi < 0) return QLORA_EINVAL;
    if (zero_idx) *zero_idx = zi;
    return QLORA_OK;
}

// codec: nf4_quantize / nf4_dequantize, which also take blocks of 32, 128
// and 256 weights (cols a multiple of the block); every other call needs 64.
int check_weight(const nf4_weight_t *q, bool need_rows, bool codec = false) {
    if (!q) return QLORA_EINVAL;
    if (q->rows < 0 || q->cols < 0) return QLORA_EINVAL;
    if (need_rows && q->rows < 1) return QLORA_EINVAL;
    if (codec) {
        if (q->block != 32 && q->block != 64 && q->block != 128 && q->block != 256)
            return QLORA_EUNSUPPORTED;
        if (q->cols % q->block != 0) return QLORA_EINVAL;
    } else {
        if (q->cols % 64 != 0) return QLORA_EINVAL;
        if (q->block != 64) return QLORA_EUNSUPPORTED;
    }
    if (q->double_quant < QLORA_DQ_NONE || q->double_quant > QLORA_DQ_F8) return QLORA_EINVAL;
    if (q->compute_dtype != QLORA_DTYPE_BF16 && q->compute_dtype != QLORA_DTYPE_FP16) return QLORA_EINVAL;
    if (q->rows * q->cols == 0) return QLORA_OK;
    if (!q->packed || !aligned16(q->packed)) return QLORA_EINVAL;
    if (q->double_quant) {
        if (q->dq_group != 256) return QLORA_EUNSUPPORTED;
        if (!q->absmax_code || !q->dq_step) return QLORA_EINVAL;
        if (q->double_quant == QLORA_DQ_MEAN && !q->dq_mean) return QLORA_EINVAL;
    } else {
        if (!q->absmax) return QLORA_EINVAL;
    }
    return QLORA_OK;
}

// Bump allocator over the caller's workspace (256-byte aligned pieces).
struct Bump {
    uintptr_t base;
    size_t off = 0;
    explicit Bump(void *b) : base(reinterpret_cast<uintptr_t>(b)) {}
    template <class T>
    T *take(size_t count) {
        off = (off + 255) & ~size_t(255);
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += count * sizeof(T);
        return p;
    }
};

struct Dims {
    int64_t M, Din, Dout;
    int r, rp, rp64, g;
    int64_t Da, Dap;
    bool small;
    bool f16;   // the compute dtype is fp16 (else bf16)
};

Dims make_dims(int64_t M, const nf4_weight_t *q, int r, int g) {
    Dims d;
    d.M = M;
    d.Din = q->cols;
    d.Dout = q->rows;
    d.r = r;
    d.rp = (int)round_up(r, 16);
    d.rp64 = (int)round_up(r, 64);
    d.g = g;
    d.Da = d.Din / g;
    d.Dap = round_up(d.Da, 8);
    d.small = M <= kGemvMaxM;
    d.f16 = q->compute_dtype == QLORA_DTYPE_FP16;
    return d;
}

// ---------------------------------------------------------------- adapter products
// C[P, Q] = sum over segments of A(p,t) B(t,q), as fp32 split-K partials
// [splits][P][Qp], on the tcgen05 skinny-GEMM engine.
struct Prod {
    SkinnySeg seg[2];
    int nseg;
    int64_t P, Q;
};
struct ProdPlan {
    int splits;
    int64_t Qp;
};

ProdPlan plan_prod(const Prod &pr) {
    ProdPlan pl;
    int per = 1;
    skinny_splits(pr.P, pr.Q, skinny_k_tiles(pr.seg, pr.nseg), &pl.splits, &per);
    pl.Qp = round_up(pr.Q, 4);
    return pl;
}

size_t prod_partial_floats(const Prod &pr) {
    const ProdPlan pl = plan_prod(pr);
    return (size_t)pl.splits * pr.P * pl.Qp;
}

int run_prod(const Prod &pr, float *partial, uint32_t *status, cudaStream_t st, ProdPlan *plan,
             bool f16) {
    *plan = plan_prod(pr);
    return launch_umma_skinny(pr.seg, pr.nseg, pr.P, pr.Q, plan->Qp, partial, status, st, f16);
}

// T = u . A    (u = x [M, Din], or pooled hi/lo [M, Dap]; A padded [Da, rp])
Prod prod_T(const Dims &d, const uint16_t *X, const uint16_t *Apad, const uint16_t *ph,
            const uint16_t *pl) {
    Prod pr{};
    if (d.g == 1) {
        pr.seg[0] = SkinnySeg{X, d.Din, 1, Apad, d.rp, 0, d.rp, d.Din};
        pr.nseg = 1;
    } else {
        pr.seg[0] = SkinnySeg{ph, d.Dap, 1, Apad, d.rp, 0, d.rp, d.Da};
        pr.seg[1] = SkinnySeg{pl, d.Dap, 1, Apad, d.rp, 0, d.rp, d.Da};
        pr.nseg = 2;
    }
    pr.P = d.M;
    pr.Q = d.r;
    return pr;
}
// G = dY . B^T   (B [r, Dout] is K-major for this product)
Prod prod_G(const Dims &d, const uint16_t *dY, const uint16_t *B) {
    Prod pr{};
    pr.seg[0] = SkinnySeg{dY, d.Dout, 1, B, d.Dout, 1, d.r, d.Dout};
    pr.nseg = 1;
    pr.P = d.M;
    pr.Q = d.r;
    return pr;
}
// dA-sum = u^T . [G_hi | G_lo]   (reduction over tokens; both MN-major)
Prod prod_dA(const Dims &d, const uint16_t *X, const uint16_t *ph, const uint16_t *pl,
             const uint16_t *Gsplit) {
    Prod pr{};
    if (d.g == 1) {
        pr.seg[0] = SkinnySeg{X, d.Din, 0, Gsplit, 2 * d.rp, 0, 2 * d.rp, d.M};
        pr.nseg = 1;
    } else {
        pr.seg[0] = SkinnySeg{ph, d.Dap, 0, Gsplit, 2 * d.rp, 0, 2 * d.rp, d.M};
        pr.seg[1] = SkinnySeg{pl, d.Dap, 0, Gsplit, 2 * d.rp, 0, 2 * d.rp, d.M};
        pr.nseg = 2;
    }
    pr.P = d.Da;
    pr.Q = 2 * d.rp;
    return pr;
}
// dB^T-sum = dY^T . [T_hi | T_lo]
Prod prod_dB(const Dims &d, const uint16_t *dY, const uint16_t *Tsplit) {
    Prod pr{};
    pr.seg[0] = SkinnySeg{dY, d.Dout, 0, Tsplit, 2 * d.rp, 0, 2 * d.rp, d.M};
    pr.nseg = 1;
    pr.P = d.Dout;
    pr.Q = 2 * d.rp;
    return pr;
}

// Workspace pieces.  The same function sizes (base == nullptr) and carves.
struct FwdWs {
    uint16_t *Apad, *ph, *pl, *sT;
    float *T32, *Tpart, *gemv_part, *gemv_tpart;
};
struct BwdWs {
    uint16_t *Apad, *ph, *pl, *sG, *Gsplit, *Tsplit, *Aext;
    float *G32, *Gpart, *T32, *Tpart, *dApart, *dBpart, *gemv_part;
};

size_t layout_fwd(const Dims &d, bool have_tsave, void *base, FwdWs *w) {
    Bump b(base);
    FwdWs x{};
    x.Apad = b.take<uint16_t>(d.Da * d.rp);
    if (d.g > 1) {
        x.ph = b.take<uint16_t>(d.M * d.Dap);
        x.pl = b.take<uint16_t>(d.M * d.Dap);
    }
    if (!have_tsave) x.T32 = b.take<float>(d.M * d.r);
    x.Tpart = b.take<float>(prod_partial_floats(prod_T(d, 0, 0, 0, 0)));
    if (d.small) {
        x.gemv_part = b.take<float>(gemv_fwd_partial_bytes((int)d.M, d.Din, d.Dout) / 4 + 1);
        if (d.g == 1) x.gemv_tpart = b.take<float>(gemv_fwd_tpart_floats((int)d.M, d.Din, d.r));
    } else {
        x.sT = b.take<uint16_t>(d.M * d.rp64);
    }
    if (w) *w = x;
    return b.off;
}

size_t layout_bwd(const Dims &d, bool have_tsaved, bool want_dx, bool want_da, bool want_db,
                  void *base, BwdWs *w) {
    Bump b(base);
    BwdWs x{};
    x.G32 = b.take<float>(d.M * d.r);
    x.Gpart = b.take<float>(prod_partial_floats(prod_G(d, 0, 0)));
    if (want_da) x.Gsplit = b.take<uint16_t>(d.M * 2 * d.rp);
    if (d.g > 1 && (want_da || (want_db && !have_tsaved))) {
        x.ph = b.take<uint16_t>(d.M * d.Dap);
        x.pl = b.take<uint16_t>(d.M * d.Dap);
    }
    if (want_db) {
        if (!have_tsaved) {
            x.Apad = b.take<uint16_t>(d.Da * d.rp);
            x.T32 = b.take<float>(d.M * d.r);
            x.Tpart = b.take<float>(prod_partial_floats(prod_T(d, 0, 0, 0, 0)));
        }
        x.Tsplit = b.take<uint16_t>(d.M * 2 * d.rp);
        x.dBpart = b.take<float>(prod_partial_floats(prod_dB(d, 0, 0)));
    }
    if (want_da) x.dApart = b.take<float>(prod_partial_floats(prod_dA(d, 0, 0, 0, 0)));
    if (want_dx) {
        if (d.small) {
            x.gemv_part = b.take<float>(gemv_bwd_partial_bytes((int)d.M, d.Din, d.Dout) / 4 + 1);
        } else {
            x.sG = b.take<uint16_t>(d.M * d.rp64);
            x.Aext = b.take<uint16_t>(d.Din * d.rp64);
        }
    }
    if (w) *w = x;
    return b.off;
}

int check_layer_args(int64_t M, const nf4_weight_t *q, const float *cb, int r, float alpha, int g,
                     int *zero_idx) {
    if (M < 0 || M > (int64_t)0x7fffffff) return QLORA_EINVAL;
    int rc = check_weight(q, true);
    if (rc) return rc;
    if (q->rows % 8 != 0) return QLORA_EUNSUPPORTED;
    rc = check_codebook(cb, zero_idx);
    if (rc) return rc;
    if (r < 1 || r > QLORA_MAX_RANK) return QLORA_EINVAL;
    if (!std::isfinite(alpha)) return QLORA_EINVAL;
    if (g != 1 && g != 64) return QLORA_EINVAL;
    return QLORA_OK;
}

Codebook to_cb(const float *c) {
    Codebook cb;
    for (int j = 0; j < 16; ++j) cb.c[j] = c[j];
    return cb;
}

#define RC(x)                    \
    do {                         \
        int _rc = (x);           \
        if (_rc) return _rc;     \
    } while (0)

// T = u . A  ->  T32 [M, r] (and s*T as bf16 into sT [M, rp64] if sT)
int run_adapter_down(const Dims &d, const uint16_t *X, const uint16_t *A, uint16_t *Apad,
                     const uint16_t *ph, const uint16_t *pl, float *Tpart, float *T32, float s,
                     uint16_t *sT, uint32_t *status, cudaStream_t st) {
    // A already has the padded row length (r a multiple of 16): use it in place
    const uint16_t *Ause = A;
    if (d.r != d.rp || !aligned16(A)) {
        RC(launch_pad_rows(A, d.Da, d.r, d.rp, 1, 1.f, Apad, st, d.f16));
        Ause = Apad;
    }
    ProdPlan plan;
    RC(run_prod(prod_T(d, X, Ause, ph, pl), Tpart, status, st, &plan, d.f16));
    if (sT && cudaMemsetAsync(sT, 0, d.M * d.rp64 * sizeof(uint16_t), st) != cudaSuccess)
        return QLORA_ECUDA;
    return launch_reduce(Tpart, plan.splits, d.M, plan.Qp, 0, d.r, 1.f, T32, d.r, 1, s, sT, d.rp64,
                         nullptr, 0, st, d.f16);
}

int run_pool(const Dims &d, const uint16_t *X, uint16_t *ph, uint16_t *pl, cudaStream_t st) {
    return launch_pool_split(X, d.M, d.Din, d.g, d.Dap, ph, pl, st, d.f16);
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

const char *qlora_strerror(int code) {
    switch (code) {
        case QLORA_OK: return "ok";
        case QLORA_EINVAL: return "invalid argument";
        case QLORA_EUNSUPPORTED: return "unsupported configuration";
        case QLORA_ECUDA: return "CUDA launch failure";
        case QLORA_EWORKSPACE: return "workspace too small";
        default: return "unknown error";
    }
}

int qlora_version(void) { return 200; }

int qlora_check_codebook(const float codebook[16]) { return check_codebook(codebook, nullptr); }

int nf4_quantize(const float *W, const nf4_weight_t *q, const float codebook[16],
                 uint32_t *d_status, void *stream) {
    int zi = 0;
    RC(check_weight(q, false, true));
    RC(check_codebook(codebook, &zi));
    if (q->rows * q->cols == 0) return QLORA_OK;
    if (!W || !aligned16(W)) return QLORA_EINVAL;
    return launch_nf4_quantize(W, *q, to_cb(codebook), zi, d_status, (cudaStream_t)stream);
}

int nf4_dequantize_dtype(const nf4_weight_t *q, const float codebook[16], int32_t dtype,
                         void *W_out, void *stream) {
    if (dtype != QLORA_DTYPE_BF16 && dtype != QLORA_DTYPE_FP16 && dtype != QLORA_DTYPE_FP32)
        return QLORA_EINVAL;
    RC(check_weight(q, false, true));
    RC(check_codebook(codebook, nullptr));
    if (q->rows * q->cols == 0) return QLORA_OK;
    if (!W_out || !aligned16(W_out)) return QLORA_EINVAL;
    if (dtype == QLORA_DTYPE_BF16)
        return launch_nf4_dequantize(*q, to_cb(codebook), static_cast<uint16_t *>(W_out),
                                     (cudaStream_t)stream);
    return launch_nf4_dequantize_dtype(*q, to_cb(codebook), dtype, W_out, (cudaStream_t)stream);
}

int nf4_dequantize(const nf4_weight_t *q, const float codebook[16], uint16_t *W_out, void *stream) {
    RC(check_weight(q, false, true));
    RC(check_codebook(codebook, nullptr));
    if (q->rows * q->cols == 0) return QLORA_OK;
    if (!W_out || !aligned16(W_out)) return QLORA_EINVAL;
    return launch_nf4_dequantize(*q, to_cb(codebook), W_out, (cudaStream_t)stream);
}

int qlora_merge(const nf4_weight_t *q, const float codebook[16], const uint16_t *A,
                const uint16_t *B, int32_t r, float alpha, int32_t pool_group, uint16_t *W_out,
                void *stream) {
    RC(check_weight(q, false));
    RC(check_codebook(codebook, nullptr));
    if (r < 1 || r > QLORA_MAX_RANK || !std::isfinite(alpha)) return QLORA_EINVAL;
    if (pool_group != 1 && pool_group != 64) return QLORA_EINVAL;
    if (q->rows * q->cols == 0) return QLORA_OK;
    if (!A || !B || !W_out || !aligned16(W_out)) return QLORA_EINVAL;
    return launch_merge(*q, to_cb(codebook), A, B, r, pool_group, alpha / (float)r, W_out,
                        (cudaStream_t)stream, q->compute_dtype == QLORA_DTYPE_FP16);
}

size_t qlora_workspace_size(int64_t M, const nf4_weight_t *q, int32_t r, int32_t pool_group,
                            int32_t which) {
    static const float kCb[16] = {-1, -.875f, -.75f, -.625f, -.5f, -.375f, -.25f, 0,
                                  .125f, .25f, .375f, .5f, .625f, .75f, .875f, 1};
    if (check_layer_args(M, q, kCb, r, 0.f, pool_group, nullptr)) return 0;
    if (M == 0) return 0;
    const Dims d = make_dims(M, q, r, pool_group);
    if (which == 0) return layout_fwd(d, false, nullptr, nullptr);
    return layout_bwd(d, false, true, true, true, nullptr, nullptr);
}

int qlora_forward(const uint16_t *X, int64_t M, const nf4_weight_t *q, const float codebook[16],
                  const uint16_t *A, const uint16_t *B, int32_t r, float alpha, int32_t pool_group,
                  uint16_t *Y, float *T_save, void *workspace, size_t ws_bytes, uint32_t *d_status,
                  void *stream) {
    RC(check_layer_args(M, q, codebook, r, alpha, pool_group, nullptr));
    if (M == 0) return QLORA_OK;
    if (!X || !A || !B || !Y) return QLORA_EINVAL;
    if (!aligned16(X) || !aligned16(B) || !aligned16(Y)) return QLORA_EINVAL;
    const Dims d = make_dims(M, q, r, pool_group);
    const size_t need = layout_fwd(d, T_save != nullptr, nullptr, nullptr);
    if (need > ws_bytes || (need > 0 && !workspace)) return QLORA_EWORKSPACE;
    FwdWs w;
    layout_fwd(d, T_save != nullptr, workspace, &w);
    cudaStream_t st = (cudaStream_t)stream;
    const Codebook cb = to_cb(codebook);
    const float s = alpha / (float)r;
    float *T32 = T_save ? T_save : w.T32;

    if (d.small && d.g == 1) {
        // one streamed kernel computes the base product and the adapter-down
        // partials, one finalize reduces both; else the general sequence
        const int rc = launch_gemv_fwd(X, (int)M, *q, cb, nullptr, B, r, s, Y, w.gemv_part, d_status,
                                       st, d.f16, A, w.gemv_tpart, T32);
        if (rc != QLORA_EUNSUPPORTED) return rc;
    }
    if (d.g > 1) RC(run_pool(d, X, w.ph, w.pl, st));
    RC(run_adapter_down(d, X, A, w.Apad, w.ph, w.pl, w.Tpart, T32, s, d.small ? nullptr : w.sT,
                        d_status, st));
    if (d.small)
        return launch_gemv_fwd(X, (int)M, *q, cb, T32, B, r, s, Y, w.gemv_part, d_status, st, d.f16);
    return launch_umma_qgemm(0, X, M, *q, cb, w.sT, r, B, Y, d_status, st, d.f16);
}

// A second stream per device for the backward's adapter-gradient products,
// which run beside the dX tensor-core GEMM and fill the SMs its last wave
// leaves idle.  Shared by all calls on the device; each call orders its work
// on it with its own events.
static cudaStream_t side_stream() {
    static std::mutex mu;
    static std::unordered_map<int, cudaStream_t> streams;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    auto it = streams.find(dev);
    if (it != streams.end()) return it->second;
    cudaStream_t s = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    streams[dev] = s;
    return s;
}

int qlora_backward(const uint16_t *X, const uint16_t *dY, int64_t M, const nf4_weight_t *q,
                   const float codebook[16], const uint16_t *A, const uint16_t *B, int32_t r,
                   float alpha, int32_t pool_group, const float *T_saved, uint16_t *dX, float *dA,
                   float *dB, void *workspace, size_t ws_bytes, uint32_t *d_status, void *stream) {
    RC(check_layer_args(M, q, codebook, r, alpha, pool_group, nullptr));
    if (M == 0) return QLORA_OK;
    if (!dY || !A || !B) return QLORA_EINVAL;
    const bool want_dx = dX != nullptr, want_da = dA != nullptr, want_db = dB != nullptr;
    if ((want_da || (want_db && !T_saved)) && !X) return QLORA_EINVAL;
    if (!aligned16(dY) || !aligned16(B) || (X && !aligned16(X)) || (dX && !aligned16(dX)))
        return QLORA_EINVAL;
    const Dims d = make_dims(M, q, r, pool_group);
    const size_t need = layout_bwd(d, T_saved != nullptr, want_dx, want_da, want_db, nullptr, nullptr);
    if (need > ws_bytes || (need > 0 && !workspace)) return QLORA_EWORKSPACE;
    BwdWs w;
    layout_bwd(d, T_saved != nullptr, want_dx, want_da, want_db, workspace, &w);
    cudaStream_t st = (cudaStream_t)stream;
    const Codebook cb = to_cb(codebook);
    const float s = alpha / (float)r;

    // G = dY . B^T  (fp32), s*G (compute dtype, large M), hi/lo split (for dA)
    {
        ProdPlan pl;
        RC(run_prod(prod_G(d, dY, B), w.Gpart, d_status, st, &pl, d.f16));
        uint16_t *sG = (want_dx && !d.small) ? w.sG : nullptr;
        if (sG && cudaMemsetAsync(sG, 0, M * d.rp64 * 2, st) != cudaSuccess) return QLORA_ECUDA;
        if (w.Gsplit && cudaMemsetAsync(w.Gsplit, 0, M * 2 * d.rp * 2, st) != cudaSuccess)
            return QLORA_ECUDA;
        RC(launch_reduce(w.Gpart, pl.splits, M, pl.Qp, 0, r, 1.f, w.G32, r, 1, s, sG, d.rp64,
                         w.Gsplit, d.rp, st, d.f16));
    }
    if (d.g > 1 && w.ph) RC(run_pool(d, X, w.ph, w.pl, st));

    // With the tensor-core dX GEMM, dA and dB go to the side stream (after
    // G): the GEMM is enqueued first, so its CTAs are placed first and the
    // adapter products take the SMs its last wave leaves free.
    cudaStream_t side = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    if (want_dx && !d.small && (want_da || want_db)) {
        side = side_stream();
        if (side && (cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess ||
                     cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess ||
                     cudaEventRecord(ev_fork, st) != cudaSuccess))
            side = nullptr;
    }
    const cudaStream_t ast = side ? side : st;   // stream of the dA and dB work

    if (want_dx) {
        if (d.small) {
            RC(launch_gemv_bwd(dY, (int)M, *q, cb, w.G32, A, r, d.g, s, dX, w.gemv_part, st, d.f16));
        } else {
            // the extension operand is A itself when no padding, pooling or scaling applies
            const bool direct = d.g == 1 && r == d.rp64 && aligned16(A);
            int rcx = direct ? QLORA_OK
                             : launch_pad_rows(A, d.Din, r, d.rp64, d.g, 1.f / d.g, w.Aext, st, d.f16);
            if (rcx == QLORA_OK)
                rcx = launch_umma_qgemm(1, dY, M, *q, cb, w.sG, r, direct ? A : w.Aext, dX, d_status, st,
                                        d.f16);
            if (rcx != QLORA_OK) {
                if (ev_fork) cudaEventDestroy(ev_fork);
                if (ev_join) cudaEventDestroy(ev_join);
                return rcx;
            }
        }
    }
    int rc = QLORA_OK;
    if (side && cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess) rc = QLORA_ECUDA;
    if (rc == QLORA_OK && want_da) {
        ProdPlan pl;
        rc = run_prod(prod_dA(d, X, w.ph, w.pl, w.Gsplit), w.dApart, d_status, ast, &pl, d.f16);
        if (rc == QLORA_OK)
            rc = launch_reduce(w.dApart, pl.splits, d.Da, pl.Qp, d.rp, r, s, dA, r, 1, 0.f, nullptr,
                               0, nullptr, 0, ast, d.f16);
    }
    if (rc == QLORA_OK && want_db) {
        const float *T32 = T_saved;
        if (!T32) {
            rc = run_adapter_down(d, X, A, w.Apad, w.ph, w.pl, w.Tpart, w.T32, s, nullptr, d_status,
                                  ast);
            T32 = w.T32;
        }
        if (rc == QLORA_OK) rc = launch_split_f32(T32, M, r, d.rp, w.Tsplit, ast, d.f16);
        ProdPlan pl;
        if (rc == QLORA_OK)
            rc = run_prod(prod_dB(d, dY, w.Tsplit), w.dBpart, d_status, ast, &pl, d.f16);
        if (rc == QLORA_OK)
            rc = launch_reduce(w.dBpart, pl.splits, d.Dout, pl.Qp, d.rp, r, s, dB, 1, d.Dout, 0.f,
                               nullptr, 0, nullptr, 0, ast, d.f16);
    }
    if (side) {
        // join: the caller's stream sees all of the backward (also on errors,
        // so that nothing is left running unordered)
        if (cudaEventRecord(ev_join, side) != cudaSuccess || cudaStreamWaitEvent(st, ev_join, 0) != cudaSuccess)
            rc = rc == QLORA_OK ? QLORA_ECUDA : rc;
    }
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (ev_join) cudaEventDestroy(ev_join);
    return rc;
}

}  // extern "C"
