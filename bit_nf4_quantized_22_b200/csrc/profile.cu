// profile.cu -- launch counting and opt-in CUDA-event timing of the
// library's main kernels, for benchmarks.  When enabled, an event pair is
// recorded on the launch stream around each timed kernel; reading the totals
// synchronizes on those events.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace qlora {
namespace {
std::atomic<int64_t> g_launches{0};
std::atomic<int> g_on{0};
std::atomic<uint32_t> g_kinds{0xffffffffu};   // kinds that are timed while enabled
std::mutex g_mu;
struct Pairs {
    std::vector<cudaEvent_t> start, stop;
    size_t used = 0;
};
Pairs g_pairs[kProfKinds];
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int device_sms() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
    std::atomic<int> &slot = cache[dev < 64 ? dev : 63];
    int n = slot.load(std::memory_order_relaxed);
    if (n <= 0 || dev >= 64) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        if (dev < 64) slot.store(n, std::memory_order_relaxed);
    }
    return n;
}

cudaError_t set_max_smem(const void *fn, int bytes) {
    static std::mutex mu;
    static std::vector<std::pair<std::pair<int, const void *>, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    std::lock_guard<std::mutex> lk(mu);
    for (const auto &d : done)
        if (d.first.first == dev && d.first.second == fn && d.second >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.push_back({{dev, fn}, bytes});
    return e;
}

// Inside a stream capture a plain event record becomes a dependency inside the
// graph, not a timestamp: record as an external event node, which each replay
// of the graph records like cudaEventRecord would.
static void record_timing_event(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, st);
}

static bool timed(int kind) {
    return g_on.load(std::memory_order_relaxed) && ((g_kinds.load(std::memory_order_relaxed) >> kind) & 1u);
}

void prof_begin(int kind, cudaStream_t st) {
    if (!timed(kind)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    Pairs &p = g_pairs[kind];
    if (p.used == p.start.size()) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return;
        if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return; }
        p.start.push_back(a);
        p.stop.push_back(b);
    }
    record_timing_event(p.start[p.used], st);
}

void prof_end(int kind, cudaStream_t st) {
    if (!timed(kind)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    Pairs &p = g_pairs[kind];
    if (p.used < p.start.size()) {
        record_timing_event(p.stop[p.used], st);
        ++p.used;
    }
}

}  // namespace qlora

extern "C" {

void qlora_profile_enable(int on) { qlora::g_on.store(on ? 1 : 0); }

void qlora_profile_kinds(uint32_t mask) { qlora::g_kinds.store(mask); }

void qlora_profile_reset(void) {
    std::lock_guard<std::mutex> lk(qlora::g_mu);
    for (auto &p : qlora::g_pairs) p.used = 0;
    qlora::g_launches.store(0);
}

int64_t qlora_launch_count(void) { return qlora::g_launches.load(); }

int qlora_profile_read(int32_t kind, int64_t *launches, double *total_ms) {
    if (kind < 0 || kind >= qlora::kProfKinds || !launches || !total_ms) return QLORA_EINVAL;
    std::lock_guard<std::mutex> lk(qlora::g_mu);
    auto &p = qlora::g_pairs[kind];
    double t = 0.0;
    for (size_t i = 0; i < p.used; ++i) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.stop[i]) != cudaSuccess ||
            cudaEventElapsedTime(&ms, p.start[i], p.stop[i]) != cudaSuccess) {
            (void)cudaGetLastError();   // a failed readout must not fail the next launch check
            return QLORA_ECUDA;
        }
        t += ms;
    }
    *launches = (int64_t)p.used;
    *total_ms = t;
    return QLORA_OK;
}

int qlora_profile_read_each(int32_t kind, int64_t cap, double *ms_each, int64_t *launches) {
    if (kind < 0 || kind >= qlora::kProfKinds || cap < 0 || !launches || (cap > 0 && !ms_each))
        return QLORA_EINVAL;
    std::lock_guard<std::mutex> lk(qlora::g_mu);
    auto &p = qlora::g_pairs[kind];
    const size_t n = p.used < (size_t)cap ? p.used : (size_t)cap;
    for (size_t i = 0; i < n; ++i) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.stop[i]) != cudaSuccess ||
            cudaEventElapsedTime(&ms, p.start[i], p.stop[i]) != cudaSuccess) {
            (void)cudaGetLastError();
            return QLORA_ECUDA;
        }
        ms_each[i] = ms;
    }
    *launches = (int64_t)p.used;
    return QLORA_OK;
}

}  // extern "C"
