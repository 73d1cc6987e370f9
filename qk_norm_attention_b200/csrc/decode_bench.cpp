// decode_bench.cpp -- time qknorm_fwd at decode sizes from C++, through the
// C ABI (no Python): calls issued back to back on one stream, CUDA events
// around them (launch cost included), and the host time per call.
//
// Usage: decode_bench [D P calls]   (defaults: 4096 4, 2000 calls)
// Prints one JSON object: for each T in {1, 8, 32, 64}, the device time per
// call (us) and the host enqueue time per call (us).
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/qknorm.h"

static int check(cudaError_t e, const char *what) {
    if (e != cudaSuccess) {
        std::fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
        return 1;
    }
    return 0;
}

int main(int argc, char **argv) {
    const int D = argc > 1 ? std::atoi(argv[1]) : 4096;
    const int P = argc > 2 ? std::atoi(argv[2]) : 4;
    const int calls = argc > 3 ? std::atoi(argv[3]) : 2000;
    const int Ts[] = {1, 8, 32, 64};
    const size_t row = (size_t)D * 2;  // bf16
    void *q, *k, *oq, *ok;
    float *g;
    if (check(cudaMalloc(&q, 64 * row), "malloc") || check(cudaMalloc(&k, 64 * row), "malloc") ||
        check(cudaMalloc(&oq, 64 * row), "malloc") || check(cudaMalloc(&ok, 64 * row), "malloc") ||
        check(cudaMalloc(&g, (size_t)D * 4), "malloc"))
        return 1;
    // bf16 1.0 (0x3f80) everywhere, gamma 1.0f.
    std::vector<unsigned short> ones(64 * (size_t)D, 0x3f80);
    std::vector<float> gh((size_t)D, 1.0f);
    if (check(cudaMemcpy(q, ones.data(), 64 * row, cudaMemcpyHostToDevice), "copy") ||
        check(cudaMemcpy(k, ones.data(), 64 * row, cudaMemcpyHostToDevice), "copy") ||
        check(cudaMemcpy(g, gh.data(), (size_t)D * 4, cudaMemcpyHostToDevice), "copy"))
        return 1;
    cudaStream_t s;
    cudaEvent_t e0, e1;
    if (check(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking), "stream") ||
        check(cudaEventCreate(&e0), "event") || check(cudaEventCreate(&e1), "event"))
        return 1;
    std::printf("{\"D\": %d, \"P\": %d, \"calls\": %d, \"dtype\": \"bf16\"", D, P, calls);
    for (int T : Ts) {
        for (int i = 0; i < 100; ++i)
            if (qknorm_fwd(q, k, g, g, oq, ok, T, D, D, P, 1e-6f, QKNORM_BF16, s) != QKNORM_OK) {
                std::fprintf(stderr, "qknorm_fwd failed: %s\n", qknorm_last_error());
                return 1;
            }
        if (check(cudaStreamSynchronize(s), "sync")) return 1;
        cudaEventRecord(e0, s);
        const auto h0 = std::chrono::steady_clock::now();
        for (int i = 0; i < calls; ++i) qknorm_fwd(q, k, g, g, oq, ok, T, D, D, P, 1e-6f, QKNORM_BF16, s);
        const auto h1 = std::chrono::steady_clock::now();
        cudaEventRecord(e1, s);
        if (check(cudaEventSynchronize(e1), "sync")) return 1;
        float ms = 0.f;
        cudaEventElapsedTime(&ms, e0, e1);
        const double host_us = std::chrono::duration<double, std::micro>(h1 - h0).count() / calls;
        std::printf(", \"%d\": {\"device_us\": %.3f, \"host_us\": %.3f}", T, 1000.0 * ms / calls, host_us);
    }
    std::printf("}\n");
    cudaFree(q);
    cudaFree(k);
    cudaFree(oq);
    cudaFree(ok);
    cudaFree(g);
    return 0;
}
