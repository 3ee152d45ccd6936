/*
 * qlora.h -- C ABI of the QLoRA linear-layer library (libqlora.so, sm_100a).
 *
 * The layer, in row-vector convention with x:[M,Din], A:[Din,r], B:[r,Dout]:
 *
 *     y  = x . dequant(W4) + s (x . A) . B,          s = alpha / r
 *     dX = dY . dequant(W4)^T + s (dY . B^T) . A^T   (no gradient for W4)
 *     dA = s x^T (dY . B^T),   dB = s (x . A)^T dY
 *
 * Sources: "从 LoRA 到 QLoRA、QA-LoRA：低秩更新如何进入量化模型" (ludovicoyin.github.io),
 * section 2 (y = x dequant(W4) + xAB; W_eff = dequant(W4) + (alpha/r) AB) and
 * sections 3-5 (pooled adapter input); "大模型量化从0到1（十）：bitsandbytes"
 * (aicoding.csdn.net), section 5.2 (block absmax, nearest codebook level,
 * two indices per byte), 7.2 (double quantization: 8-bit first-level scales,
 * one fp32 constant per 256), 8.6 (dequantize fused into the matmul),
 * 12.2/12.4 (s = lora_alpha / r; the gradient passes through the frozen
 * base, which receives none).
 *
 * Conventions shared by every entry point
 *   - All array pointers are DEVICE pointers owned by the caller, except the
 *     16-entry codebook, which is a HOST array read during the call.  The
 *     library allocates nothing: scratch memory is the caller's `workspace`
 *     buffer, sized by qlora_workspace_size().
 *   - 16-bit arrays are passed as uint16_t bit patterns: for the layer calls
 *     and qlora_merge in the weight's compute dtype (q->compute_dtype: bf16,
 *     or IEEE fp16), for nf4_dequantize in bf16.  Every 2-D array is
 *     row-major and densely packed.
 *   - The frozen weight is stored transposed, Wt:[Dout, Din] (the
 *     nn.Linear layout).  Flattened row-major it is cut into blocks of 64
 *     consecutive weights, each inside one row; Din must be a multiple of 64.
 *     nf4_quantize and nf4_dequantize also take blocks of 32, 128 or 256
 *     (q->block; Din a multiple of it; the article's section 5.1 weighs
 *     smaller blocks' finer scales against their metadata); the layer calls
 *     and qlora_merge read one scale per 64 inputs and return
 *     QLORA_EUNSUPPORTED for any other block.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; no call synchronizes the host.
 *   - Return value: QLORA_OK, or an error code.  Arguments are validated on
 *     the host before anything is enqueued; a failed validation enqueues
 *     nothing.  QLORA_ECUDA reports a launch failure (the CUDA error is left
 *     for the caller to query).
 *   - `d_status` (optional, may be NULL): a device uint32_t into which
 *     kernels OR the QLORA_STATUS_* bits they detect.  The library never
 *     clears it.  Device-side conditions never trap or abort the context.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QLORA_OK 0
#define QLORA_EINVAL 1          /* bad pointer, size, rank, alpha or codebook   */
#define QLORA_EUNSUPPORTED 2    /* valid request outside what this build does  */
#define QLORA_ECUDA 3           /* a kernel launch failed                       */
#define QLORA_EWORKSPACE 4      /* workspace missing or smaller than required  */

#define QLORA_STATUS_NONFINITE 1u /* nf4_quantize met a NaN or Inf weight      */
#define QLORA_STATUS_TIMEOUT 2u   /* a pipeline wait in a kernel gave up       */

#define QLORA_BLOCK 64
#define QLORA_DQ_GROUP 256
#define QLORA_MAX_RANK 256

/* Double-quantization codes of the first-level scales (nf4_weight_t's
 * double_quant).  bitsandbytes article (CSDN) 7.2 gives the structure -- an
 * 8-bit code per block scale, one fp32 constant per 256 scales -- but not the
 * code; three are provided, each step one stated rounding:
 *   QLORA_DQ_U8    unsigned: step f = RN32(group max / 255),
 *                  code = round-half-even(a / f) in 0..255
 *   QLORA_DQ_S8    the signed INT8 absmax code of section 4.1 applied to the
 *                  scales: f = RN32(group max / 127), code in 0..127 (scales
 *                  are >= 0)
 *   QLORA_DQ_MEAN  the group mean taken out first: mu = RN32(S / n), S the
 *                  fp64 sum of the group's scales in block order; d = RN32(a - mu);
 *                  f = RN32(max |d| / 127); code = round-half-even(d / f) in
 *                  -127..127 stored as int8; one mu per group in dq_mean
 *   QLORA_DQ_F8    an 8-bit float code: the E4M3 layout (1 sign, 4 exponent
 *                  bits biased by 7, 3 mantissa bits; no infinity, largest
 *                  finite value 448, subnormals m * 2^-9); f = RN32(group max /
 *                  448), code = the E4M3 value nearest to RN32(a / f), ties to
 *                  the even code, 448 for quotients above it; codes 0..0x7E
 * Decoded scale: RN32(code * f), RN32(mu + RN32(code * f)) for QLORA_DQ_MEAN,
 * RN32(E4M3(code) * f) for QLORA_DQ_F8.
 * The weights themselves are encoded with the exact block absmax. */
/* Compute dtypes (bitsandbytes article (CSDN) 8.3: the dequantized weight
 * and the arithmetic are FP32, BF16 or FP16; 8.5 on FP16's narrower range).
 * The layer calls take BF16 or FP16 (nf4_weight_t's compute_dtype);
 * nf4_dequantize_dtype also writes FP32. */
#define QLORA_DTYPE_BF16 0
#define QLORA_DTYPE_FP16 1
#define QLORA_DTYPE_FP32 2

#define QLORA_DQ_NONE 0
#define QLORA_DQ_U8 1
#define QLORA_DQ_S8 2
#define QLORA_DQ_MEAN 3
#define QLORA_DQ_F8 4

/* One quantized weight Wt:[rows = Dout, cols = Din]; nb = rows*cols/block.
 *   packed      [rows*cols/2] uint8   two 4-bit codebook indices per byte;
 *                                     element 2i in the HIGH nibble of byte i
 *   absmax      [nb] fp32             block absmax (double_quant == 0)
 *   absmax_code [nb] uint8 / int8     8-bit scale codes (double_quant != 0)
 *   dq_step     [ceil(nb/256)] fp32   one second-level step per 256 blocks
 *   dq_mean     [ceil(nb/256)] fp32   group means (double_quant == QLORA_DQ_MEAN)
 * Unused arrays may be NULL. */
typedef struct {
    int64_t rows;
    int64_t cols;
    int32_t block;          /* 64; the codec calls also take 32, 128, 256 */
    int32_t double_quant;   /* QLORA_DQ_NONE, _U8, _S8, _MEAN or _F8 */
    int32_t dq_group;       /* must be 256 when double_quant != 0 */
    int32_t compute_dtype;  /* QLORA_DTYPE_BF16 or _FP16: the layer calls' 16-bit arrays */
    uint8_t *packed;
    float *absmax;
    uint8_t *absmax_code;
    float *dq_step;
    float *dq_mean;
} nf4_weight_t;

/* Human-readable name of a return code (static storage). */
const char *qlora_strerror(int code);

/* Library ABI version (major*100 + minor). */
int qlora_version(void);

/* nf4_codebook -- the 16 NF4 levels, built on the host (no device work).
 * "QLoRA：用4比特行李箱装下整个大模型" chapter 3: the levels are standard-normal
 * quantiles of equal-probability pieces of the CDF; bitsandbytes article (CSDN)
 * section 6.2: one fixed table, normalised to [-1, 1], built asymmetrically
 * around an exact 0.  With Phi^-1 the standard normal quantile:
 *   out[0..6]  = -Phi^-1(delta + (1/2 - delta) i / 7) / Phi^-1(delta), i = 0..6
 *   out[7]     = 0
 *   out[15-i]  =  Phi^-1(delta + (1/2 - delta) i / 8) / Phi^-1(delta), i = 0..7
 * each rounded once to fp32, so out[0] = -1, out[15] = +1 and the table is
 * strictly increasing.  QLORA_NF4_DELTA, 1 - (1/32 + 1/30)/2, is the mean of
 * the outermost interval-midpoint probabilities for 16 and for 15 pieces.
 *   delta   in (1/2, 1)
 *   out     host fp32[16] (output, caller-owned)
 * Errors: EINVAL for a NULL out or delta outside (1/2, 1). */
#define QLORA_NF4_DELTA 0.96770833333333333333
int nf4_codebook(double delta, float out[16]);

/* fp4_codebook -- the FP4 table, built on the host (no device work).
 * bitsandbytes article (CSDN) sections 6.4-6.5 and 9.3 name a "4-bit
 * float-style" table (the library's default type) and print no values; the
 * layout used is FP4 E2M1 (OCP Microscaling formats: sign bit, two exponent
 * bits with bias 1, one mantissa bit, exponent field 0 subnormal), divided by
 * its largest magnitude 6:
 *   out = [-1, -2/3, -1/2, -1/3, -1/4, -1/6, -1/12, -0,
 *          +0, 1/12, 1/6, 1/4, 1/3, 1/2, 2/3, 1]   (each rounded to fp32).
 * Zero appears twice (-0, +0).  Quantization takes the first nearest level,
 * so every weight in zero's basin gets -0 and the +0 code is never written.
 *   out     host fp32[16] (output, caller-owned)
 * Errors: EINVAL for a NULL out. */
int fp4_codebook(float out[16]);

/* Host-side check of a codebook (no device work): 16 finite fp32 values
 * inside [-1, 1], strictly increasing except that the zero level may appear
 * twice in a row (-0 then +0, as in the FP4 table), with at least one zero.
 * Returns QLORA_OK or QLORA_EINVAL. */
int qlora_check_codebook(const float codebook[16]);

/* nf4_quantize -- blockwise 4-bit quantization of W (bitsandbytes article
 * (CSDN) section 5.2, with section 7.2 double quantization).
 *   W          device fp32 [q->rows, q->cols], the frozen weight Wt.
 *   q          host struct naming the output buffers (device); the fields
 *              selected by q->double_quant are written.
 *   codebook   host fp32[16] (see qlora_check_codebook).
 * Per block: a = max|w|; index = argmin_j |w - c_j a| in exact arithmetic,
 * ties to the lower index; an all-zero block maps to the exact-zero level.
 * A NaN/Inf weight sets QLORA_STATUS_NONFINITE; that block's outputs are
 * unspecified.  Reads 4 bytes and writes 0.5 + 1/block (+ 4/(256 block)
 * with double quantization) bytes per weight: ~0.52 at block 64.
 * Errors: EINVAL for a NULL or unaligned W or buffer, cols not a multiple of
 * the block, a bad codebook; EUNSUPPORTED for a block outside {32, 64, 128,
 * 256} or dq_group != 256. */
int nf4_quantize(const float *W, const nf4_weight_t *q, const float codebook[16],
                 uint32_t *d_status, void *stream);

/* nf4_dequantize -- W_out[rows, cols] (bf16) = RN_bf16(RN32(a_hat * c_q))
 * (section 5.2, w_hat = a c_q, in the bf16 compute dtype of section 8.3);
 * element e takes the scale of block e / q->block.  W_out 16-byte aligned.
 * Errors as nf4_quantize. */
int nf4_dequantize(const nf4_weight_t *q, const float codebook[16], uint16_t *W_out,
                   void *stream);

/* nf4_dequantize_dtype -- as nf4_dequantize, into the compute dtype `dtype`
 * (bitsandbytes article (CSDN) section 8.3: the dequantized weights and the
 * arithmetic are FP32, BF16 or FP16; 8.5 on FP16's narrower range):
 *   W_out[e] = RN_dtype(RN32(a_hat * c_q)), one rounding of the fp32
 *   product; fp16 follows IEEE binary16 (subnormals kept, magnitudes past
 *   65504 after rounding become infinite); fp32 is the product itself.
 *   W_out   device [rows, cols] of 16-bit patterns (bf16, fp16) or fp32,
 *           16-byte aligned.
 * Errors as nf4_dequantize, plus EINVAL for an unknown dtype. */
int nf4_dequantize_dtype(const nf4_weight_t *q, const float codebook[16], int32_t dtype,
                         void *W_out, void *stream);

/* qlora_merge -- the weight with the adapter folded in, for deployment
 * ("从 LoRA 到 QLoRA、QA-LoRA" section 2, W_eff = dequant(W4) + (alpha/r) A B;
 * bitsandbytes article (CSDN) 12.10, merging before deployment):
 *   W_out[n][k] = RN_dt( w_hat[n][k] + (s/g) sum_j A[k/g][j] B[j][n] ),
 * s = alpha/r, g = pool_group, dt = q->compute_dtype, w_hat the dequantized
 * weight RN_dt(RN32(a_hat c_q)), as
 * nf4_dequantize writes it; the rank-r sum is accumulated in fp32.  With
 * g = 64 every input of a group shares (A_p B)/g (the same blog, section 5),
 * so that x . W_out^T is the pooled layer's forward.
 *   A       device dt [Din/pool_group, r];  B  device dt [r, Dout]
 *   W_out   device dt [Dout, Din], 16-byte aligned (output)
 * No workspace.  Errors as nf4_dequantize, plus EINVAL for r outside
 * [1, QLORA_MAX_RANK], a non-finite alpha or pool_group not 1 or 64. */
int qlora_merge(const nf4_weight_t *q, const float codebook[16], const uint16_t *A,
                const uint16_t *B, int32_t r, float alpha, int32_t pool_group, uint16_t *W_out,
                void *stream);

/* Scratch bytes qlora_forward (which = 0) or qlora_backward (which = 1)
 * needs for this problem.  Returns 0 when the arguments are invalid. */
size_t qlora_workspace_size(int64_t M, const nf4_weight_t *q, int32_t r, int32_t pool_group,
                            int32_t which);

/* qlora_forward -- y = x . dequant(W4) + (alpha/r) T . B with
 * T = u . A, u = x (pool_group == 1) or the mean of each run of 64 input
 * features (pool_group == 64, the pooled adapter of QA-LoRA sections 3-4).
 *   X       device [M, Din] in the compute dtype dt = q->compute_dtype
 *           (bf16 or fp16; bitsandbytes article (CSDN) 8.3)
 *   A       device dt [Din/pool_group, r];  B  device dt [r, Dout]
 *   r       1..256;  alpha finite;  pool_group 1 or 64
 *   Y       device dt [M, Dout] (output)
 *   T_save  device fp32 [M, r] receiving T, or NULL
 *   workspace/ws_bytes  caller scratch of at least qlora_workspace_size(.., 0)
 * Accumulation is fp32; y is rounded once to dt.  With fp16, the fp32
 * adapter intermediates (T, G, pooled inputs) are carried as fp16 hi + lo
 * pairs, so they keep about 22 significant bits inside fp16's range (8.5). */
int qlora_forward(const uint16_t *X, int64_t M, const nf4_weight_t *q, const float codebook[16],
                  const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                  int32_t pool_group, uint16_t *Y, float *T_save, void *workspace,
                  size_t ws_bytes, uint32_t *d_status, void *stream);

/* qlora_backward -- gradients of the layer for the upstream gradient dY:
 *   G  = dY . B^T                               (fp32 [M, r], internal)
 *   dX = dY . dequant(W4)^T + (s/g) G . A^T     (dt [M, Din]; with pooling
 *                                                each input feature of a
 *                                                group receives 1/g of it)
 *   dA = s u^T G                                (fp32 [Din/g, r])
 *   dB = s T^T dY                               (fp32 [r, Dout])
 * T_saved is the forward's T (fp32 [M, r]) or NULL to recompute it.  Any of
 * dX, dA, dB may be NULL to skip it.  No gradient is produced for W4. */
int qlora_backward(const uint16_t *X, const uint16_t *dY, int64_t M, const nf4_weight_t *q,
                   const float codebook[16], const uint16_t *A, const uint16_t *B, int32_t r,
                   float alpha, int32_t pool_group, const float *T_saved, uint16_t *dX,
                   float *dA, float *dB, void *workspace, size_t ws_bytes,
                   uint32_t *d_status, void *stream);

/* ---- Forward without caller-provided scratch -------------------------------
 * No counterpart on the pages: this entry point exists for callers that cannot
 * allocate device memory -- code that runs where cudaMalloc is not allowed or
 * not wanted (inside another allocator's arena, in a process that must not
 * grow its device footprint after start-up, or a host that simply has no
 * workspace to hand over).  It computes exactly what qlora_forward computes,
 * with the same kernels and the same arguments minus the workspace; its
 * scratch is a fixed array of QLORA_NOALLOC_SCRATCH_BYTES bytes inside the
 * library, which every GPU that loads the library holds until the process
 * exits.
 *   - Requests needing more scratch than that return QLORA_EWORKSPACE before
 *     anything is enqueued; qlora_workspace_size(M, q, r, pool_group, 0)
 *     tells the need.  Decode shapes that fit: M <= 16 at 4096 x 4096
 *     (r <= 64), and M = 1 on the 8192 <-> 28672 projections (r = 64); M = 16
 *     there does not (its split partials alone take 14.7 MB).  On the
 *     tensor-core path (M > 16) the need also depends on the GPU's SM count.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it for the
 *     life of the process; make that first call before any stream capture.
 *     cudaDeviceReset after the first call on a device is not supported:
 *     the module may come back at another address, and later calls would
 *     still use the old one.
 *   - Every call shares the one array and leaves its contents behind; each
 *     call clears what it needs zeroed.  Calls that overlap on the GPU (two
 *     streams, or two host threads) race on the array: serialize them. */
#define QLORA_NOALLOC_SCRATCH_BYTES (8u << 20)
int qlora_forward_noalloc(const uint16_t *X, int64_t M, const nf4_weight_t *q,
                          const float codebook[16], const uint16_t *A, const uint16_t *B,
                          int32_t r, float alpha, int32_t pool_group, uint16_t *Y, float *T_save,
                          uint32_t *d_status, void *stream);

/* qlora_selftest_wait_timeout -- failure-path check (not part of the layer's
 * computation): launches one warp that waits, with the library's bounded
 * mbarrier wait, on a barrier nothing arrives on.  The wait gives up after
 * its poll limit (at most about two seconds) and ORs QLORA_STATUS_TIMEOUT into
 * *d_status (device uint32, required); nothing traps, and the stream stays
 * usable.  Returns EINVAL for a null status pointer. */
int qlora_selftest_wait_timeout(uint32_t *d_status, void *stream);

/* ---- Benchmark support (not part of the layer's computation) ----------
 * Kernel launches made by the library since the last qlora_profile_reset(). */
int64_t qlora_launch_count(void);

/* When enabled, each launch of the library's main kernels is bracketed by a
 * CUDA event pair recorded on its launch stream.  Kinds: 0 tensor-core GEMM
 * (tcgen05), 1 small-M GEMV kernels, 2 quantize kernel, 3 adapter products,
 * 4 merge kernel. */
void qlora_profile_enable(int on);

/* Which kinds are timed while profiling is enabled: bit k for kind k (all by
 * default).  Each timed launch adds an event pair to the stream, and inside a
 * CUDA graph each event record is a node of its own, so a benchmark times
 * only the kinds it reads. */
void qlora_profile_kinds(uint32_t mask);

/* Forget recorded events and zero the launch count (host only). */
void qlora_profile_reset(void);

/* Number of timed launches of `kind` since the reset and their summed
 * duration in milliseconds; waits for the recorded events to complete. */
int qlora_profile_read(int32_t kind, int64_t *launches, double *total_ms);

/* The durations (ms) of the first min(cap, launches) timed launches of `kind`
 * since the reset, in launch order, into ms_each (caller-owned host array of
 * cap doubles); *launches receives the count of timed launches.  Waits for
 * the events like qlora_profile_read.  EINVAL for an unknown kind, cap < 0, a
 * null count, or a null array with cap > 0. */
int qlora_profile_read_each(int32_t kind, int64_t cap, double *ms_each, int64_t *launches);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_H */
