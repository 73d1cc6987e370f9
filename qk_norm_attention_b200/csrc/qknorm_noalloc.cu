// qknorm_noalloc.cu -- the split path in one call, for callers that cannot
// allocate device memory.
//
// qknorm_partial_sumsq + qknorm_apply need a [T, P] fp32 statistics array
// between the two kernels. Some callers cannot provide one: their device
// memory is owned by a framework's pool with no out-of-band allocations, or
// they run in a latency-critical loop where cudaMalloc's implicit device
// synchronisation is not acceptable. qknorm_split_noalloc keeps that array in
// this file's static device buffer instead; it calls no cudaMalloc, cudaFree
// or other allocating routine.
//
// The buffer is shared by every call on a device and keeps the last call's
// contents. Nothing needs clearing: the statistics pass writes every entry
// the apply pass reads. Calls that overlap on the GPU (on different streams,
// say) use the same buffer and race.
#include <mutex>

#include "../../include/qknorm.h"

// The statistics of one call: T * P floats at most (4 MiB on every device
// that loads the library, held until the process exits).
constexpr long long kNoallocMaxStats = 1ll << 20;
static __device__ __align__(256) float g_noalloc_stats[kNoallocMaxStats];

namespace {

constexpr int kMaxDevices = 64;
float *g_stats_ptr[kMaxDevices];
std::mutex g_setup_mu;

// The device address of g_noalloc_stats on the current device (its host-side
// name is only a stand-in). Looked up once per device, on that device's first
// call, with that device current.
int stats_address(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QKNORM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_stats_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_stats) != cudaSuccess || p == nullptr)
            return QKNORM_ERR_CUDA;
        g_stats_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_stats_ptr[dev];
    return QKNORM_OK;
}

}  // namespace

extern "C" {

QKNORM_API int64_t qknorm_split_noalloc_max_stats(void) { return kNoallocMaxStats; }

QKNORM_API int qknorm_split_noalloc(const void *x, const float *gamma, void *out, int64_t T,
                                    int32_t D, int32_t P, float eps, int32_t dtype, void *stream) {
    if (T < 0 || P <= 0) return QKNORM_ERR_INVALID_ARG;
    if (T == 0) return QKNORM_OK;
    if (T > kNoallocMaxStats / P) return QKNORM_ERR_UNSUPPORTED;  // T * P beyond the buffer
    float *stats = nullptr;
    int st = stats_address(&stats);
    if (st != QKNORM_OK) return st;
    st = qknorm_partial_sumsq(x, stats, T, D, P, dtype, stream);
    if (st != QKNORM_OK) return st;
    return qknorm_apply(x, gamma, stats, out, T, D, P, eps, dtype, stream);
}

}  // extern "C"
