// noalloc.cu -- qlora_forward_noalloc: the forward pass for callers that
// cannot allocate device memory (no cudaMalloc, no allocator of their own,
// no workspace to hand over).  Its scratch is one fixed device array that
// lives in this library's module: every GPU that loads the library holds it
// until the process exits.
#include <mutex>

#include "common.cuh"

// The scratch.  In host code this name is only a host-side stand-in for the
// device symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached for the life of the process.
// A cudaDeviceReset after that would leave the cached address stale; the
// header states that resets are not supported once this entry point ran.
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ECUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QLORA_ECUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return QLORA_OK;
}
}  // namespace

extern "C" int qlora_forward_noalloc(const uint16_t *X, int64_t M, const nf4_weight_t *q,
                                     const float codebook[16], const uint16_t *A,
                                     const uint16_t *B, int32_t r, float alpha,
                                     int32_t pool_group, uint16_t *Y, float *T_save,
                                     uint32_t *d_status, void *stream) {
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != QLORA_OK) return rc;
    // Same kernels as qlora_forward, with the fixed array as the workspace;
    // a request that needs more than the array holds is rejected before
    // anything is enqueued (QLORA_EWORKSPACE).
    return qlora_forward(X, M, q, codebook, A, B, r, alpha, pool_group, Y, T_save, scratch,
                         (size_t)QLORA_NOALLOC_SCRATCH_BYTES, d_status, stream);
}
