// copy_floor.cpp -- yardstick for small launches: the device time per launch
// of a plain streaming copy and a plain streaming read of B bytes, launched
// back to back on one stream the way the library's kernels are (256 threads,
// 8 blocks per SM, grid-stride, four 16-byte loads in flight per thread,
// programmatic dependent launch on). Eight buffer sets rotate, so every
// launch reads HBM. A kernel that moves B bytes in one launch can be judged
// against these times: the copy's fixed cost per launch and its steady rate
// bound what any one-launch kernel of that size reaches on the box.
//
// Compiled as CUDA by build_lib.py (nvcc -x cu); not part of libqknorm.so.
// Usage: copy_floor [MB ...]   (default 21 42 84 100 168 336; for the copy,
//        MB counts the bytes read plus the bytes written)
// Prints one JSON object: {"copy": {MB: us}, "read": {MB: us}, "sms": N}.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ void dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__global__ void __launch_bounds__(256) copy_k(const uint4 *__restrict__ x, uint4 *__restrict__ y, int64_t n) {
    dep_wait();
    dep_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const uint4 a = __ldcs(x + i), b = __ldcs(x + i + stride);
        const uint4 c = __ldcs(x + i + 2 * stride), d = __ldcs(x + i + 3 * stride);
        __stcs(y + i, a);
        __stcs(y + i + stride, b);
        __stcs(y + i + 2 * stride, c);
        __stcs(y + i + 3 * stride, d);
    }
    for (; i < n; i += stride) __stcs(y + i, __ldcs(x + i));
}

// Reads n vectors; the xor of the words is stored only if it equals a fixed
// pattern, so the loads stay live and (almost) nothing is written.
__global__ void __launch_bounds__(256) read_k(const uint4 *__restrict__ x, unsigned *__restrict__ out, int64_t n) {
    dep_wait();
    dep_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    unsigned acc = 0;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const uint4 a = __ldcs(x + i), b = __ldcs(x + i + stride);
        const uint4 c = __ldcs(x + i + 2 * stride), d = __ldcs(x + i + 3 * stride);
        acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
    }
    for (; i < n; i += stride) {
        const uint4 a = __ldcs(x + i);
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
    if (acc == 0x9e3779b9u) out[blockIdx.x] = acc;
}

int fail(cudaError_t e, const char *what) {
    std::fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
    return 1;
}

}  // namespace

int main(int argc, char **argv) {
    std::vector<double> mbs;
    for (int i = 1; i < argc; ++i) mbs.push_back(std::atof(argv[i]));
    if (mbs.empty()) mbs = {21, 42, 84, 100, 168, 336};
    double maxmb = 0;
    for (double m : mbs) {
        if (!(m > 0) || m > 4096) {
            std::fprintf(stderr, "sizes must be in (0, 4096] MB\n");
            return 2;
        }
        if (m > maxmb) maxmb = m;
    }
    cudaError_t e;
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0)) != cudaSuccess) return fail(e, "sms");
    constexpr int kSets = 8, kLaunches = 200, kWarm = 20, kPerSm = 8;
    // A set holds the largest read (maxmb) in x and the largest copy's half in y.
    const size_t xbytes = ((size_t)(maxmb * 1e6) + 15) / 16 * 16;
    std::vector<uint4 *> xs(kSets, nullptr), ys(kSets, nullptr);
    for (int s = 0; s < kSets; ++s) {
        if ((e = cudaMalloc(&xs[s], xbytes)) != cudaSuccess) return fail(e, "malloc");
        if ((e = cudaMalloc(&ys[s], xbytes / 2 + 16)) != cudaSuccess) return fail(e, "malloc");
        if ((e = cudaMemset(xs[s], 0x3c + s, xbytes)) != cudaSuccess) return fail(e, "memset");
    }
    unsigned *out = nullptr;
    if ((e = cudaMalloc(&out, sizeof(unsigned) * sms * kPerSm)) != cudaSuccess) return fail(e, "malloc");
    cudaStream_t st;
    if ((e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking)) != cudaSuccess) return fail(e, "stream");
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    std::printf("{\"sms\": %d, \"blocks_per_sm\": %d, \"launches\": %d", sms, kPerSm, kLaunches);
    for (int kind = 0; kind < 2; ++kind) {
        std::printf(", \"%s\": {", kind == 0 ? "copy" : "read");
        for (size_t j = 0; j < mbs.size(); ++j) {
            // copy: mbs[j] = read + write, so n vectors of each; read: n vectors
            const int64_t n = kind == 0 ? (int64_t)(mbs[j] * 1e6 / 32) : (int64_t)(mbs[j] * 1e6 / 16);
            auto go = [&](int s) -> cudaError_t {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3((unsigned)(sms * kPerSm));
                cfg.blockDim = dim3(256);
                cfg.stream = st;
                cudaLaunchAttribute at[1];
                at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                at[0].val.programmaticStreamSerializationAllowed = 1;
                cfg.attrs = at;
                cfg.numAttrs = 1;
                if (kind == 0) return cudaLaunchKernelEx(&cfg, copy_k, (const uint4 *)xs[s], ys[s], n);
                return cudaLaunchKernelEx(&cfg, read_k, (const uint4 *)xs[s], out, n);
            };
            for (int i = 0; i < kWarm; ++i)
                if ((e = go(i % kSets)) != cudaSuccess) return fail(e, "launch");
            if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return fail(e, "sync");
            cudaEventRecord(e0, st);
            for (int i = 0; i < kLaunches; ++i)
                if ((e = go(i % kSets)) != cudaSuccess) return fail(e, "launch");
            cudaEventRecord(e1, st);
            if ((e = cudaEventSynchronize(e1)) != cudaSuccess) return fail(e, "sync");
            float ms = 0;
            cudaEventElapsedTime(&ms, e0, e1);
            std::printf("%s\"%g\": %.3f", j ? ", " : "", mbs[j], ms * 1000.0 / kLaunches);
        }
        std::printf("}");
    }
    std::printf("}\n");
    return 0;
}
