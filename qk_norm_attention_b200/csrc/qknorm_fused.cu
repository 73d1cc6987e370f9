// qknorm_fused.cu -- single-pass fused QK-Norm kernels for sm_100a.
//
// SwiftQK technical review, Section 3, Algorithm 1: per token, Phase A sums
// the squares of each shard, Phase B adds the shard scalars and forms the
// factor while x * gamma is formed independently, Phase C writes the
// weighted row times the factor. Here the shards are slices of one row in
// this GPU's memory, so the "exchange" of Phase B is a read of a few floats
// from shared memory; one HBM read and one HBM write per element remain.
//
// fused_cta: one CTA per token (Q row and K row), one warp per (tensor,
//   shard, group) task. Each lane keeps its <= VMAX vectors of the row in
//   registers between the reduction and the apply, so every element is read
//   once. The grid is persistent (a stride loop over tokens, Algorithm 1's
//   "persistent block-level stride loop", sized by the occupancy calculator
//   as B_res x N_SM); with PREFETCH a CTA issues the loads of its next token
//   before reducing the current one, so HBM reads stay in flight across the
//   CTA barrier.
// fused_generic: any shape. A CTA per token whose warps loop over the tasks;
//   the apply pass re-reads the row (an L1/L2 hit). With one warp per CTA it
//   is the warp-per-token variant.
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

// Task decode shared by both kernels: task j of a token -> (tensor z, shard p,
// group kg). Tasks 0 .. P*K0-1 belong to Q, the rest to K.
struct Task {
    int z, p, kg, K, nv;
};

// Select element z (0 or 1) of a two-entry kernel-argument array without
// indexing it at run time (which would copy the arguments to local memory).
template <class T>
__device__ __forceinline__ T sel(const T (&arr)[2], int z) {
    return z ? arr[1] : arr[0];
}

__device__ __forceinline__ Task decode_task(const FusedArgs &a, int j) {
    Task t;
    const int nt0 = a.P * a.K[0];
    t.z = j < nt0 ? 0 : 1;
    const int jj = t.z ? j - nt0 : j;
    t.K = sel(a.K, t.z);
    t.p = jj / t.K;
    t.kg = jj - t.p * t.K;
    t.nv = sel(a.nv, t.z);
    return t;
}

template <class Tag, int VMAX, bool PREFETCH, bool FULL, int MAXT, bool GREG>
__global__ void __launch_bounds__(MAXT, 1) fused_cta(const FusedArgs a) {
    constexpr int VEC = Tag::kVec;
    __shared__ float red[2][32];
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Task tk = decode_task(a, warp);
    const int stride = kLanes * tk.K;            // vector stride between a lane's slots
    const int first = tk.kg * kLanes + lane;     // slot 0, as a vector index in the shard
    // FULL: every lane of every task holds exactly VMAX vectors (no guards).
    const int cnt = FULL ? VMAX : slot_count(first, tk.nv, stride);
    const int64_t ldx = sel(a.ldx, tk.z);             // row strides, in vectors
    const int64_t ldy = sel(a.ldy, tk.z);
    const int64_t col0 = (int64_t)tk.p * tk.nv + first;
    const uint4 *xs = reinterpret_cast<const uint4 *>(sel(a.x, tk.z)) + col0;
    uint4 *ys = reinterpret_cast<uint4 *>(sel(a.y, tk.z)) + col0;
    const float *gs = sel(a.g, tk.z) + col0 * VEC;
    const float Df = sel(a.Df, tk.z);
    const float eps = a.eps;
    const int red_base = tk.z ? a.P * a.K[0] : 0;

    int64_t t = blockIdx.x;
    const int64_t T = a.T;
    const int64_t G = gridDim.x;

    uint4 cur[VMAX];
    if (t < T) {
        const uint4 *src = xs + t * ldx;
#pragma unroll
        for (int i = 0; i < VMAX; ++i)
            if (FULL || i < cnt) cur[i] = ld_stream(src + (int64_t)i * stride);
    }
    // GREG: the lane's gamma in registers, its loads in flight together with
    // the row's (otherwise they are issued after the CTA barrier, one more
    // dependent round trip per token).
    float gr[GREG ? VMAX : 1][GREG ? VEC : 1];
    if constexpr (GREG) {
#pragma unroll
        for (int i = 0; i < VMAX; ++i)
            if (FULL || i < cnt) {
#pragma unroll
                for (int j = 0; j < VEC; j += 4) {
                    const float4 g4 = __ldg(reinterpret_cast<const float4 *>(gs + (int64_t)i * stride * VEC + j));
                    gr[i][j] = g4.x;
                    gr[i][j + 1] = g4.y;
                    gr[i][j + 2] = g4.z;
                    gr[i][j + 3] = g4.w;
                }
            }
    }
    int buf = 0;
    for (; t < T; t += G) {
        const int64_t tn = t + G;
        uint4 nxt[VMAX];
        if (PREFETCH && tn < T) {
            const uint4 *src = xs + tn * ldx;
#pragma unroll
            for (int i = 0; i < VMAX; ++i)
                if (FULL || i < cnt) nxt[i] = ld_stream(src + (int64_t)i * stride);
        }
        // Phase A: this lane's chain, then the butterfly -> group sum.
        float c = 0.f;
#pragma unroll
        for (int i = 0; i < VMAX; ++i)
            if (FULL || i < cnt) c = __fadd_rn(c, vsumsq(Tag{}, cur[i]));
        c = butterfly(c);
        if (lane == 0) red[buf][warp] = c;
        __syncthreads();
        // Phase B: shard sums in order, the factor.
        const float r = factor(combine_fast(&red[buf][red_base], a.P, tk.K), Df, eps);
        // Phase B weight multiply and Phase C, straight from registers.
        uint4 *dst = ys + t * ldy;
#pragma unroll
        for (int i = 0; i < VMAX; ++i)
            if (FULL || i < cnt) {
                if constexpr (GREG)
                    st_stream(dst + (int64_t)i * stride, vapply_regs(Tag{}, cur[i], gr[i], r));
                else
                    st_stream(dst + (int64_t)i * stride,
                              vapply(Tag{}, cur[i], gs + (int64_t)i * stride * VEC, r));
            }
        if (PREFETCH) {
#pragma unroll
            for (int i = 0; i < VMAX; ++i) cur[i] = nxt[i];
        } else if (tn < T) {
            const uint4 *src = xs + tn * ldx;
#pragma unroll
            for (int i = 0; i < VMAX; ++i)
                if (FULL || i < cnt) cur[i] = ld_stream(src + (int64_t)i * stride);
        }
        buf ^= 1;
    }
}

template <class Tag>
__global__ void __launch_bounds__(256, 1) fused_generic(const FusedArgs a) {
    constexpr int VEC = Tag::kVec;
    extern __shared__ float red[];  // one float per task
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int nt0 = a.P * a.K[0];
    const int ntask = nt0 + a.P * a.K[1];
    for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        for (int j = warp; j < ntask; j += nw) {
            const Task tk = decode_task(a, j);
            const int stride = kLanes * tk.K;
            const uint4 *src = reinterpret_cast<const uint4 *>(sel(a.x, tk.z)) +
                               t * sel(a.ldx, tk.z) + (int64_t)tk.p * tk.nv;
            float c = 0.f;
#pragma unroll 4
            for (int v = tk.kg * kLanes + lane; v < tk.nv; v += stride)
                c = __fadd_rn(c, vsumsq(Tag{}, src[v]));
            c = butterfly(c);
            if (lane == 0) red[j] = c;
        }
        __syncthreads();
        const float r0 = factor(combine(red, a.P, a.K[0]), a.Df[0], a.eps);
        const float r1 = factor(combine(red + nt0, a.P, a.K[1]), a.Df[1], a.eps);
        for (int j = warp; j < ntask; j += nw) {
            const Task tk = decode_task(a, j);
            const int stride = kLanes * tk.K;
            const int64_t col = (int64_t)tk.p * tk.nv;
            const uint4 *src = reinterpret_cast<const uint4 *>(sel(a.x, tk.z)) + t * sel(a.ldx, tk.z) + col;
            uint4 *dst = reinterpret_cast<uint4 *>(sel(a.y, tk.z)) + t * sel(a.ldy, tk.z) + col;
            const float *g = sel(a.g, tk.z) + (int64_t)tk.p * tk.nv * VEC;
            const float r = tk.z ? r1 : r0;
#pragma unroll 4
            for (int v = tk.kg * kLanes + lane; v < tk.nv; v += stride)
                st_stream(dst + v, vapply(Tag{}, src[v], g + (int64_t)v * VEC, r));
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- instance tables

// 1024-thread instances only while a lane holds <= 16 values (64 registers).
constexpr int cta_max_threads(int vmax, int vec) { return (vmax <= 2 && vmax * vec <= 16) ? 1024 : 512; }
// Register-resident instances exist up to 8 vectors per lane (4 for FP8,
// whose 16 values per vector take twice the registers of bf16 once widened).
constexpr bool cta_exists(int vmax, int vec) { return vmax >= 1 && vmax <= (vec == 16 ? 4 : kVcap); }

// Gamma in registers while a lane's gamma is at most 32 floats, and only for
// one token per CTA (no prefetch: the decode sizes).
constexpr bool cta_greg_exists(int vmax, int vec) { return vmax * vec <= 32; }

template <class Tag, int VMAX, bool PF, bool FULL, bool GREG>
const void *cta_fn() {
    if constexpr (cta_exists(VMAX, Tag::kVec) && (!GREG || (!PF && cta_greg_exists(VMAX, Tag::kVec))))
        return reinterpret_cast<const void *>(
            &fused_cta<Tag, VMAX, PF, FULL, cta_max_threads(VMAX, Tag::kVec), GREG>);
    else
        return nullptr;
}

template <class Tag, bool PF, bool FULL, bool GREG>
const void *cta_table(int vmax) {
    switch (vmax) {
    case 1: return cta_fn<Tag, 1, PF, FULL, GREG>();
    case 2: return cta_fn<Tag, 2, PF, FULL, GREG>();
    case 3: return cta_fn<Tag, 3, PF, FULL, GREG>();
    case 4: return cta_fn<Tag, 4, PF, FULL, GREG>();
    case 5: return cta_fn<Tag, 5, PF, FULL, GREG>();
    case 6: return cta_fn<Tag, 6, PF, FULL, GREG>();
    case 7: return cta_fn<Tag, 7, PF, FULL, GREG>();
    case 8: return cta_fn<Tag, 8, PF, FULL, GREG>();
    default: return nullptr;
    }
}

template <class Tag>
const void *cta_pick(int vmax, bool prefetch, bool full, bool greg) {
    if (greg) {
        if (prefetch) return nullptr;
        return full ? cta_table<Tag, false, true, true>(vmax) : cta_table<Tag, false, false, true>(vmax);
    }
    if (prefetch)
        return full ? cta_table<Tag, true, true, false>(vmax) : cta_table<Tag, true, false, false>(vmax);
    return full ? cta_table<Tag, false, true, false>(vmax) : cta_table<Tag, false, false, false>(vmax);
}

const void *fused_cta_kernel(int dtype, int vmax, bool prefetch, bool full, bool greg, int *max_threads) {
    const int vec = dtype == 1 ? 8 : (dtype == 2 ? 16 : 4);
    if (!cta_exists(vmax, vec)) return nullptr;
    if (greg && (prefetch || !cta_greg_exists(vmax, vec))) return nullptr;
    if (max_threads) *max_threads = cta_max_threads(vmax, vec);
    if (dtype == 0) return cta_pick<F32Tag>(vmax, prefetch, full, greg);
    if (dtype == 1) return cta_pick<BF16Tag>(vmax, prefetch, full, greg);
    if (dtype == 2) return cta_pick<E4M3Tag>(vmax, prefetch, full, greg);
    return nullptr;
}

const void *fused_generic_kernel(int dtype) {
    if (dtype == 0) return reinterpret_cast<const void *>(&fused_generic<F32Tag>);
    if (dtype == 1) return reinterpret_cast<const void *>(&fused_generic<BF16Tag>);
    if (dtype == 2) return reinterpret_cast<const void *>(&fused_generic<E4M3Tag>);
    return nullptr;
}

cudaError_t launch_fused_cta(int dtype, int vmax, bool prefetch, bool full, bool greg,
                             const FusedArgs &a, int block, int64_t grid, cudaStream_t s) {
    const void *fn = fused_cta_kernel(dtype, vmax, prefetch, full, greg, nullptr);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {const_cast<FusedArgs *>(&a)};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

cudaError_t launch_fused_generic(int dtype, const FusedArgs &a, int block, int64_t grid,
                                 size_t smem, cudaStream_t s) {
    const void *fn = fused_generic_kernel(dtype);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {const_cast<FusedArgs *>(&a)};
    return launch(fn, dim3((unsigned)grid), dim3(block), smem, s, args);
}

}  // namespace qkn
