// qknorm_fused_warp.cu -- warp-per-token fused QK-Norm, the rows held in
// registers.
//
// SwiftQK technical review, Section 3, Algorithm 1 (Phases A-C per token),
// with one warp owning a whole token: its Q row and its K row. Lane l holds,
// for every shard p of each tensor, the vectors l, l + 32, l + 64, ... of that
// shard (the single lane group of the reduction order stated in
// include/qknorm.h: shards of at most 256 vectors), so the warp walks the
// shards itself: P independent lane chains per tensor, P butterflies, the
// shard sums added in order of p in registers, the factor, then the weight
// multiply and the scale straight from the registers. No shared memory and no
// CTA barrier; every element is read once and written once.
//
// The shard count and the vectors per lane per shard are template
// parameters, so that the chains and the register slots unroll completely.
// A warp holds P * (VQ + VK) 16-byte vectors per lane (at most 32: 128
// registers), which fits the decode shapes (D = 4096 in 4 shards of bf16: 4 +
// 4 vectors per shard; Dq = 5120, Dk = 1024 in 8 shards: 3 + 1).
//
// The same arithmetic as every other kernel of the library, in the same
// order, so the outputs are bit-identical to theirs.
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

constexpr int kWarpMaxThreads = 128;  // up to 4 warps (tokens) per CTA

template <class Tag, int P, int VQ, int VK>
__global__ void __launch_bounds__(kWarpMaxThreads) fused_warp(const FusedArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int64_t W = (int64_t)gridDim.x * wpb;
    const int nvq = a.nv[0], nvk = a.nv[1];
    // Slots this lane fills in every shard (the same for all shards of a tensor).
    const int cq = slot_count(lane, nvq, kLanes);
    const int ck = slot_count(lane, nvk, kLanes);
    const uint4 *xq0 = reinterpret_cast<const uint4 *>(a.x[0]) + lane;
    const uint4 *xk0 = reinterpret_cast<const uint4 *>(a.x[1]) + lane;
    uint4 *yq0 = reinterpret_cast<uint4 *>(a.y[0]) + lane;
    uint4 *yk0 = reinterpret_cast<uint4 *>(a.y[1]) + lane;
    const float *gq0 = a.g[0] + (int64_t)lane * Tag::kVec;
    const float *gk0 = a.g[1] + (int64_t)lane * Tag::kVec;

    for (int64_t t = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); t < a.T; t += W) {
        const uint4 *xq = xq0 + t * a.ldx[0];
        const uint4 *xk = xk0 + t * a.ldx[1];
        uint4 rq[P][VQ], rk[P][VK];
        // Phase A loads: every slot of both rows in flight at once.
#pragma unroll
        for (int p = 0; p < P; ++p) {
#pragma unroll
            for (int i = 0; i < VQ; ++i)
                if (i < cq) rq[p][i] = ld_stream(xq + p * nvq + i * kLanes);
#pragma unroll
            for (int i = 0; i < VK; ++i)
                if (i < ck) rk[p][i] = ld_stream(xk + p * nvk + i * kLanes);
        }
        // Phase A: the lane chain of every shard, then the shards' butterflies.
        float sq[P], sk[P];
#pragma unroll
        for (int p = 0; p < P; ++p) {
            float c = 0.f;
#pragma unroll
            for (int i = 0; i < VQ; ++i)
                if (i < cq) c = __fadd_rn(c, vsumsq(Tag{}, rq[p][i]));
            sq[p] = c;
            c = 0.f;
#pragma unroll
            for (int i = 0; i < VK; ++i)
                if (i < ck) c = __fadd_rn(c, vsumsq(Tag{}, rk[p][i]));
            sk[p] = c;
        }
#pragma unroll
        for (int p = 0; p < P; ++p) {
            sq[p] = butterfly(sq[p]);
            sk[p] = butterfly(sk[p]);
        }
        // Phase B: the shard sums in order of p (one group per shard: each
        // shard sum is 0 + its group sum, exact), and the factors.
        float Sq = 0.f, Sk = 0.f;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            Sq = __fadd_rn(Sq, sq[p]);
            Sk = __fadd_rn(Sk, sk[p]);
        }
        const float fq = factor(Sq, a.Df[0], a.eps);
        const float fk = factor(Sk, a.Df[1], a.eps);
        // Phase B weight multiply and Phase C, from the registers.
        uint4 *yq = yq0 + t * a.ldy[0];
        uint4 *yk = yk0 + t * a.ldy[1];
#pragma unroll
        for (int p = 0; p < P; ++p) {
#pragma unroll
            for (int i = 0; i < VQ; ++i)
                if (i < cq) {
                    const int v = p * nvq + i * kLanes;
                    st_stream(yq + v, vapply(Tag{}, rq[p][i], gq0 + (int64_t)v * Tag::kVec, fq));
                }
#pragma unroll
            for (int i = 0; i < VK; ++i)
                if (i < ck) {
                    const int v = p * nvk + i * kLanes;
                    st_stream(yk + v, vapply(Tag{}, rk[p][i], gk0 + (int64_t)v * Tag::kVec, fk));
                }
        }
    }
}

// ---------------------------------------------------------------- instances

// (P, VQ, VK) with P in {2, 4, 8}, 1 <= VK <= VQ <= 4 and P * (VQ + VK) <= 32
// registers' worth of vectors per lane.
constexpr bool warp_exists(int P, int vq, int vk) {
    return (P == 2 || P == 4 || P == 8) && vk >= 1 && vq >= vk && vq <= 4 && P * (vq + vk) <= 32;
}

template <class Tag, int P, int VQ, int VK>
const void *warp_fn() {
    if constexpr (warp_exists(P, VQ, VK))
        return reinterpret_cast<const void *>(&fused_warp<Tag, P, VQ, VK>);
    else
        return nullptr;
}

template <class Tag, int P, int VQ>
const void *warp_vk(int vk) {
    switch (vk) {
    case 1: return warp_fn<Tag, P, VQ, 1>();
    case 2: return warp_fn<Tag, P, VQ, 2>();
    case 3: return warp_fn<Tag, P, VQ, 3>();
    case 4: return warp_fn<Tag, P, VQ, 4>();
    default: return nullptr;
    }
}

template <class Tag, int P>
const void *warp_vq(int vq, int vk) {
    switch (vq) {
    case 1: return warp_vk<Tag, P, 1>(vk);
    case 2: return warp_vk<Tag, P, 2>(vk);
    case 3: return warp_vk<Tag, P, 3>(vk);
    case 4: return warp_vk<Tag, P, 4>(vk);
    default: return nullptr;
    }
}

template <class Tag>
const void *warp_p(int P, int vq, int vk) {
    switch (P) {
    case 2: return warp_vq<Tag, 2>(vq, vk);
    case 4: return warp_vq<Tag, 4>(vq, vk);
    case 8: return warp_vq<Tag, 8>(vq, vk);
    default: return nullptr;
    }
}

const void *fused_warp_kernel(int dtype, int P, int vq, int vk) {
    if (!warp_exists(P, vq, vk)) return nullptr;
    if (dtype == 0) return warp_p<F32Tag>(P, vq, vk);
    if (dtype == 1) return warp_p<BF16Tag>(P, vq, vk);
    if (dtype == 2) return warp_p<E4M3Tag>(P, vq, vk);
    return nullptr;
}

int fused_warp_max_threads() { return kWarpMaxThreads; }

cudaError_t launch_fused_warp(int dtype, int P, int vq, int vk, const FusedArgs &a, int block,
                              int64_t grid, cudaStream_t s) {
    const void *fn = fused_warp_kernel(dtype, P, vq, vk);
    if (!fn || block < kLanes || block > kWarpMaxThreads || block % kLanes) return cudaErrorInvalidValue;
    void *args[] = {const_cast<FusedArgs *>(&a)};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

}  // namespace qkn
