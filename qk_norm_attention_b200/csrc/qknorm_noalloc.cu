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
#include <cuda.h>  // CUcontext / CUresult types only; the driver is reached through the runtime
#include <mutex>

#include "../../include/qknorm.h"

// The statistics of one call: T * P floats at most (4 MiB on every device
// that loads the library, held until the process exits).
constexpr long long kNoallocMaxStats = 1ll << 20;
static __device__ __align__(256) float g_noalloc_stats[kNoallocMaxStats];

namespace {

// The buffer's device address is looked up once per (device, CUDA context):
// on a device's first call, and again on the first call after the device's
// context was destroyed and re-created (cudaDeviceReset), when the module is
// loaded anew and the buffer may sit at another address. Contexts are told
// apart by the driver's process-unique context ID.
struct Setup {
    int dev;
    unsigned long long ctx_id;
    float *ptr;
};
constexpr int kMaxDevices = 64;
Setup g_setup[kMaxDevices];
std::mutex g_setup_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
bool g_entry_points_resolved = false;

// The ID of the context current on this thread; 0 if there is none yet (the
// runtime creates the primary context on its first call that needs one) or
// the driver lacks the query. Called with g_setup_mu held.
unsigned long long current_ctx_id() {
    if (!g_entry_points_resolved) {
        g_entry_points_resolved = true;
        cudaDriverEntryPointQueryResult q1, q2;
        void *f1 = nullptr, *f2 = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1) ==
                cudaSuccess && q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) ==
                cudaSuccess && q2 == cudaDriverEntryPointSuccess) {
            g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f1);
            g_ctx_id = reinterpret_cast<CtxGetIdFn>(f2);
        }
        cudaGetLastError();  // a failed query must not leak into the caller's error state
    }
    if (!g_ctx_current || !g_ctx_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// The device address of g_noalloc_stats in the current device's context (its
// host-side name is only a stand-in).
int stats_address(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QKNORM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    Setup &s = g_setup[dev];
    const unsigned long long id = current_ctx_id();
    if (s.ptr == nullptr || id == 0 || id != s.ctx_id) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_stats) != cudaSuccess || p == nullptr)
            return QKNORM_ERR_CUDA;
        s.dev = dev;
        s.ptr = static_cast<float *>(p);
        s.ctx_id = current_ctx_id();  // the lookup made the primary context current if it was not
    }
    *out = s.ptr;
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
