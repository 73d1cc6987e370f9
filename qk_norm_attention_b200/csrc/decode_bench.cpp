// decode_bench.cpp -- time qknorm_fwd at decode sizes from C++, through the
// C ABI (no Python): calls issued back to back on one stream, CUDA events
// around them (launch cost included), the host time per call, and the same
// calls replayed from a CUDA graph.
//
// Usage: decode_bench [Dq P calls] [--dk Dk] [--variant V] [--gamma-regs G]
//                     [--dtype bf16|f32|e4m3]
//   (defaults: Dq = Dk = 4096, P = 4, 2000 calls, the selector's variant,
//   automatic gamma placement, bf16). --variant takes a qknorm_variant value
//   (-1 automatic); --gamma-regs is passed to qknorm_set_tuning.
// Prints one JSON object: for each T in {1, 8, 32, 64}, the device time per
// call (us), the host enqueue time per call (us), the device time per call
// replayed from a graph of 100 calls (us), and the kernel the plan chose.
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
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
    int Dq = 4096, Dk = -1, P = 4, calls = 2000, variant = QKNORM_VARIANT_AUTO, gregs = -1;
    int dtype = QKNORM_BF16;
    int pos = 0;
    for (int i = 1; i < argc; ++i) {
        if (!std::strcmp(argv[i], "--dk") && i + 1 < argc) Dk = std::atoi(argv[++i]);
        else if (!std::strcmp(argv[i], "--variant") && i + 1 < argc) variant = std::atoi(argv[++i]);
        else if (!std::strcmp(argv[i], "--gamma-regs") && i + 1 < argc) gregs = std::atoi(argv[++i]);
        else if (!std::strcmp(argv[i], "--dtype") && i + 1 < argc) {
            ++i;
            dtype = !std::strcmp(argv[i], "f32") ? QKNORM_F32
                  : !std::strcmp(argv[i], "e4m3") ? QKNORM_E4M3 : QKNORM_BF16;
        } else if (pos == 0) { Dq = std::atoi(argv[i]); ++pos; }
        else if (pos == 1) { P = std::atoi(argv[i]); ++pos; }
        else if (pos == 2) { calls = std::atoi(argv[i]); ++pos; }
    }
    if (Dk < 0) Dk = Dq;
    const int Ts[] = {1, 8, 32, 64};
    const size_t es = dtype == QKNORM_BF16 ? 2 : (dtype == QKNORM_E4M3 ? 1 : 4);
    const size_t rq = (size_t)Dq * es, rk = (size_t)Dk * es;
    void *q, *k, *oq, *ok;
    float *gq, *gk;
    if (check(cudaMalloc(&q, 64 * rq), "malloc") || check(cudaMalloc(&k, 64 * rk), "malloc") ||
        check(cudaMalloc(&oq, 64 * rq), "malloc") || check(cudaMalloc(&ok, 64 * rk), "malloc") ||
        check(cudaMalloc(&gq, (size_t)Dq * 4), "malloc") || check(cudaMalloc(&gk, (size_t)Dk * 4), "malloc"))
        return 1;
    // Every value 1.0 in its storage type, gamma 1.0f.
    std::vector<unsigned char> ones(64 * (rq > rk ? rq : rk));
    for (size_t i = 0; i < ones.size(); i += es) {
        if (dtype == QKNORM_BF16) { ones[i] = 0x80; ones[i + 1] = 0x3f; }
        else if (dtype == QKNORM_E4M3) ones[i] = 0x38;
        else { const float one = 1.0f; std::memcpy(&ones[i], &one, 4); }
    }
    std::vector<float> gh((size_t)(Dq > Dk ? Dq : Dk), 1.0f);
    if (check(cudaMemcpy(q, ones.data(), 64 * rq, cudaMemcpyHostToDevice), "copy") ||
        check(cudaMemcpy(k, ones.data(), 64 * rk, cudaMemcpyHostToDevice), "copy") ||
        check(cudaMemcpy(gq, gh.data(), (size_t)Dq * 4, cudaMemcpyHostToDevice), "copy") ||
        check(cudaMemcpy(gk, gh.data(), (size_t)Dk * 4, cudaMemcpyHostToDevice), "copy"))
        return 1;
    if (qknorm_force_variant(variant, 0) != QKNORM_OK || qknorm_set_tuning(0, 0, gregs, 0) != QKNORM_OK) {
        std::fprintf(stderr, "bad --variant or --gamma-regs\n");
        return 1;
    }
    cudaStream_t s;
    cudaEvent_t e0, e1;
    if (check(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking), "stream") ||
        check(cudaEventCreate(&e0), "event") || check(cudaEventCreate(&e1), "event"))
        return 1;
    std::printf("{\"Dq\": %d, \"Dk\": %d, \"P\": %d, \"calls\": %d, \"dtype\": \"%s\", \"variant\": %d, "
                "\"gamma_regs\": %d", Dq, Dk, P, calls,
                dtype == QKNORM_BF16 ? "bf16" : (dtype == QKNORM_E4M3 ? "e4m3" : "f32"), variant, gregs);
    auto fwd = [&](int T) {
        return qknorm_fwd(q, k, gq, gk, oq, ok, T, Dq, Dk, P, 1e-6f, dtype, s);
    };
    constexpr int kGraphCalls = 100, kGraphReps = 20;
    for (int T : Ts) {
        for (int i = 0; i < 100; ++i)
            if (fwd(T) != QKNORM_OK) {
                std::fprintf(stderr, "qknorm_fwd failed: %s\n", qknorm_last_error());
                return 1;
            }
        if (check(cudaStreamSynchronize(s), "sync")) return 1;
        qknorm_plan pl;
        qknorm_launch_plan(T, Dq, Dk, P, dtype, &pl);
        cudaEventRecord(e0, s);
        const auto h0 = std::chrono::steady_clock::now();
        for (int i = 0; i < calls; ++i) fwd(T);
        const auto h1 = std::chrono::steady_clock::now();
        cudaEventRecord(e1, s);
        if (check(cudaEventSynchronize(e1), "sync")) return 1;
        float ms = 0.f;
        cudaEventElapsedTime(&ms, e0, e1);
        const double host_us = std::chrono::duration<double, std::micro>(h1 - h0).count() / calls;
        // The same calls replayed from a CUDA graph: the device-side cost per call.
        cudaGraph_t g;
        cudaGraphExec_t ge;
        if (check(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal), "capture")) return 1;
        for (int i = 0; i < kGraphCalls; ++i) fwd(T);
        if (check(cudaStreamEndCapture(s, &g), "capture") ||
            check(cudaGraphInstantiate(&ge, g, 0), "instantiate"))
            return 1;
        cudaGraphLaunch(ge, s);
        if (check(cudaStreamSynchronize(s), "sync")) return 1;
        float gms = 0.f;
        cudaEventRecord(e0, s);
        for (int r = 0; r < kGraphReps; ++r) cudaGraphLaunch(ge, s);
        cudaEventRecord(e1, s);
        if (check(cudaEventSynchronize(e1), "sync")) return 1;
        cudaEventElapsedTime(&gms, e0, e1);
        cudaGraphExecDestroy(ge);
        cudaGraphDestroy(g);
        std::printf(", \"%d\": {\"device_us\": %.3f, \"host_us\": %.3f, \"graph_us\": %.3f, "
                    "\"plan\": {\"variant\": %d, \"block\": %d, \"grid\": %lld, \"gamma_regs\": %d}}",
                    T, 1000.0 * ms / calls, host_us, 1000.0 * gms / (kGraphCalls * kGraphReps),
                    pl.variant, pl.block, (long long)pl.grid, pl.gamma_regs);
    }
    std::printf("}\n");
    cudaFree(q);
    cudaFree(k);
    cudaFree(oq);
    cudaFree(ok);
    cudaFree(gq);
    cudaFree(gk);
    return 0;
}
