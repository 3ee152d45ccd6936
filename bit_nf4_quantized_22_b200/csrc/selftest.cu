// selftest.cu -- a check of the library's failure path on a GPU: the
// pipeline kernels wait on mbarriers with a bounded number of polls and, when
// a wait gives up, report QLORA_STATUS_TIMEOUT instead of hanging or
// trapping.  This kernel makes one such wait run out on purpose (an
// mbarrier nothing arrives on) so that a test can see the status word set
// and the context still usable afterwards.
#include "common.cuh"
#include "tcgen05.cuh"

namespace qlora {
namespace {

__global__ void __launch_bounds__(32) k_selftest_wait(uint32_t *status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(smem_u32(&bar), 1);   // expects one arrival; none comes
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(smem_u32(&bar), 0, &abort_flag));
    if (!ok && threadIdx.x == 0 && status) atomicOr(status, QLORA_STATUS_TIMEOUT);
}

}  // namespace
}  // namespace qlora

extern "C" int qlora_selftest_wait_timeout(uint32_t *d_status, void *stream) {
    if (!d_status) return QLORA_EINVAL;
    qlora::k_selftest_wait<<<1, 32, 0, (cudaStream_t)stream>>>(d_status);
    QLORA_LAUNCH_CHECK();
    return QLORA_OK;
}
