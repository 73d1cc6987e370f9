// qknorm_deferred.cu -- the two steps on either side of the path, on their own.
//
// xgamma: u = x * gamma, element-wise, no reduction. A deferred normalisation
//   stores this when a later RMSNorm cancels the per-token factor (pull
//   request "perf(dsv4 decode swa): deferred attention RMSNorm and dep
//   cleanup", attn_norm_xgamma); it is also Algorithm 1's Phase B compute
//   path by itself (SwiftQK technical review, Section 3).
// inv_rms: r[t] = rsqrt(S[t] / D + eps) alone, the one dynamic scalar per
//   token that RMSNorm factors into (abstract "QK-Normed MLA: QK
//   normalization without full key caching"). One warp per row walks the P
//   shards in the library's reduction order, so r equals the factor the
//   fused kernels apply, bit for bit.
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

template <class Tag>
__global__ void __launch_bounds__(256) xgamma_k(const void *x, const float *g, void *y, int64_t T,
                                                int32_t D) {
    constexpr int VEC = Tag::kVec;
    constexpr int UNR = 4;
    pdl_wait();
    pdl_trigger();
    const int64_t rowvec = D / VEC;
    const int nthr = blockDim.x;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x) + t * rowvec;
        uint4 *dst = reinterpret_cast<uint4 *>(y) + t * rowvec;
        for (int64_t v0 = threadIdx.x; v0 < rowvec; v0 += (int64_t)nthr * UNR) {
            uint4 xv[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int64_t v = v0 + (int64_t)u * nthr;
                if (v < rowvec) xv[u] = ld_stream(src + v);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int64_t v = v0 + (int64_t)u * nthr;
                if (v < rowvec) st_stream(dst + v, vxgamma(Tag{}, xv[u], g + v * VEC));
            }
        }
    }
}

template <class Tag>
__global__ void __launch_bounds__(256) inv_rms_k(const void *x, float *r, int64_t T, int32_t D,
                                                 int32_t P, int32_t nv, int32_t K, float eps) {
    constexpr int VEC = Tag::kVec;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t rowvec = D / VEC;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int stride = kLanes * K;
    const float Df = (float)D;
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nwarps) {
        const uint4 *row = reinterpret_cast<const uint4 *>(x) + t * rowvec;
        float S = 0.f;
        if (K == 1) {
            // Four shards at a time, their chains advancing together (the
            // order inside each shard is unchanged).
            const int cnt = slot_count(lane, nv, kLanes);
            for (int p0 = 0; p0 < P; p0 += 4) {
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                const uint4 *sh = row + (int64_t)p0 * nv + lane;
                // Two slots' loads are issued before either is reduced.
#pragma unroll 2
                for (int i = 0; i < cnt; ++i) {
                    uint4 v[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (p0 + b < P) v[b] = ld_stream(sh + (int64_t)b * nv + i * kLanes);
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (p0 + b < P) c[b] = __fadd_rn(c[b], vsumsq(Tag{}, v[b]));
                }
#pragma unroll
                for (int b = 0; b < 4; ++b) c[b] = butterfly(c[b]);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if (p0 + b < P) S = __fadd_rn(S, c[b]);
            }
        } else {
            for (int p = 0; p < P; ++p) {
                const uint4 *sh = row + (int64_t)p * nv;
                float Sp = 0.f;
                for (int kg = 0; kg < K; ++kg) {
                    float c = 0.f;
#pragma unroll 4
                    for (int v = kg * kLanes + lane; v < nv; v += stride)
                        c = __fadd_rn(c, vsumsq(Tag{}, ld_stream(sh + v)));
                    Sp = __fadd_rn(Sp, butterfly(c));
                }
                S = __fadd_rn(S, Sp);
            }
        }
        if (lane == 0) r[t] = factor(S, Df, eps);
    }
}

const void *xgamma_kernel(int dtype) {
    if (dtype == 0) return reinterpret_cast<const void *>(&xgamma_k<F32Tag>);
    if (dtype == 1) return reinterpret_cast<const void *>(&xgamma_k<BF16Tag>);
    if (dtype == 2) return reinterpret_cast<const void *>(&xgamma_k<E4M3Tag>);
    return nullptr;
}

const void *inv_rms_kernel(int dtype) {
    if (dtype == 0) return reinterpret_cast<const void *>(&inv_rms_k<F32Tag>);
    if (dtype == 1) return reinterpret_cast<const void *>(&inv_rms_k<BF16Tag>);
    if (dtype == 2) return reinterpret_cast<const void *>(&inv_rms_k<E4M3Tag>);
    return nullptr;
}

cudaError_t launch_xgamma(int dtype, const void *x, const float *g, void *y, int64_t T, int32_t D,
                          int block, int64_t grid, cudaStream_t s) {
    const void *fn = xgamma_kernel(dtype);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {const_cast<void **>(&x), const_cast<float **>(&g), &y, &T, &D};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

cudaError_t launch_inv_rms(int dtype, const void *x, float *r, int64_t T, const TensorShape &sh,
                           int32_t P, float eps, int block, int64_t grid, cudaStream_t s) {
    const void *fn = inv_rms_kernel(dtype);
    if (!fn) return cudaErrorInvalidValue;
    int32_t D = sh.D, nv = sh.nv, K = sh.K;
    void *args[] = {const_cast<void **>(&x), &r, &T, &D, &P, &nv, &K, &eps};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

}  // namespace qkn
