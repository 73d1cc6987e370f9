// qknorm_split.cu -- the split path: statistics, then apply.
//
// SwiftQK technical review, Section 3, Algorithm 1, and Section 4's
// "MiniMax(eager)" ladder rung (scalar statistics first, normalisation
// afterwards, not fused): qknorm_partial_sumsq is Phase A alone and writes
// each shard's sum of squares to stats[T, P] (the scalar a rank would
// publish to its IPC slot); qknorm_apply is Phases B and C given stats.
//
// stats: one warp per (token, shard) task, the same reduction order as the
//   fused kernels (groups of 32 lane chains, butterfly, groups in order), so
//   S[t,p] equals the fused kernel's shard sum bit for bit. No barriers; the
//   grid is a stride loop over tasks, R tasks per warp turn with all their
//   loads issued first.
// apply: one CTA per row (stride loop over rows). Every thread adds the P
//   shard sums of its row in order and forms the factor, then streams its
//   vectors of the row through (x * gamma) * r. The row's first loads are
//   issued before the factor so the statistic's latency overlaps them.
//
// Both kernels take one or two tensors ("sides") per launch: blocks below
// split take side 0, the others side 1, each block with its own side's
// pointers and widths and its share of the grid as its stride. Q and K of
// one layer (e.g. one rank's slices) then cost one launch per step.
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

// The gathered shard sums of row t, n = Pb * nb of them in blocks of Pb at
// stride sg (block b, shard p at st[b * sg + t * Pb + p]), loaded by the 32
// lanes of a warp at once: lane l takes global shard index c0 + l (0 past
// the end). stat_fold then adds the m lanes' values in lane order, which is
// the order of the global shard index; every lane ends with the same S.
__device__ __forceinline__ float stat_load(const float *st, int64_t t, int Pb, int n, int64_t sg,
                                           int c0, int lane) {
    const int j = c0 + lane;
    if (j >= n) return 0.f;
    const int b = j / Pb;
    return __ldg(st + b * sg + t * Pb + (j - b * Pb));
}

__device__ __forceinline__ float stat_fold(float S, float v, int m) {
    for (int u = 0; u < m; ++u) S = __fadd_rn(S, __shfl_sync(kFull, v, u));
    return S;
}

// S of row t from its gathered shard sums, in order of the global shard
// index. FOLD = false: block by block, each block's Pb sums loaded by every
// thread (one round trip per block). FOLD = true: the warp's lanes load 32
// sums at a time and stat_fold adds them (one round trip per 32 sums, at the
// cost of registers: 62 against 48 for the narrow two-tensor apply, one
// resident block per SM fewer). Measured on one tensor-parallel rank's apply
// at the 13B shape: 8 ranks (8 blocks of 1) 12.8 -> 11.2 us with the fold;
// 2 and 4 ranks (2 x 4, 4 x 2) 29.5 and 17.7 us with the blocks against
// 31.1 and 18.7 us with the fold.
template <bool FOLD>
__device__ __forceinline__ float stat_sum(const float *st, int64_t t, int Pb, int nb, int64_t sg, int lane) {
    float S = 0.f;
    if constexpr (FOLD) {
        const int n = Pb * nb;
        for (int c0 = 0; c0 < n; c0 += 32)
            S = stat_fold(S, stat_load(st, t, Pb, n, sg, c0, lane), n - c0 < 32 ? n - c0 : 32);
    } else {
        st += t * Pb;
        for (int b = 0; b < nb; ++b, st += sg) {
#pragma unroll 8
            for (int p = 0; p < Pb; ++p) S = __fadd_rn(S, __ldg(st + p));
        }
    }
    return S;
}

// TWO: the launch may carry two sides (one-side launches compile without
// the selection, which costs registers). KEEP: rows read with the default L2
// policy instead of evict-first, so that an apply launch soon after finds
// them in L2 (taken for launches that read at most kStatsKeepBytes).
template <class Tag, int VMAX, int R, bool TWO, bool KEEP>
__device__ __forceinline__ void stats_body(const StatsArgs &a) {
    constexpr int VEC = Tag::kVec;
    pdl_wait();
    pdl_trigger();
    const int z = TWO && (int)blockIdx.x >= a.split ? 1 : 0;
    const int bz = z ? (int)blockIdx.x - a.split : (int)blockIdx.x;   // block within its side
    const int gz = z ? (int)gridDim.x - a.split : a.split;            // the side's blocks
    // Each field selected on its own (indexing the parameter array by z
    // would copy it to the stack).
    const void *x = z ? a.side[1].x : a.side[0].x;
    float *stats = z ? a.side[1].stats : a.side[0].stats;
    const int64_t T = a.T;
    const int32_t P = a.P;
    const int32_t nv = z ? a.side[1].nv : a.side[0].nv;
    const int32_t K = z ? a.side[1].K : a.side[0].K;
    const int lane = threadIdx.x & 31;
    const int64_t rowvec = (z ? a.side[1].D : a.side[0].D) / VEC;
    const int64_t ntask = T * (int64_t)P;
    const int64_t nwarps = (int64_t)gz * (blockDim.x >> 5);
    const int stride = kLanes * K;
    const int64_t w0 = (int64_t)bz * (blockDim.x >> 5) + (threadIdx.x >> 5);
    // Task = t * P + p. The (t, p) of a warp's tasks advance by a fixed step
    // (nwarps tasks), so they are carried along instead of divided out.
    const int64_t dt = nwarps / P;
    const int dp = (int)(nwarps - dt * P);
    int64_t tb = w0 / P;
    int pb = (int)(w0 - tb * P);
    // A warp takes R tasks per turn (tasks w0 + (n*R + j)*nwarps) and issues
    // all their loads before reducing any, to keep more bytes in flight.
    for (int64_t base = w0; base < ntask; base += (int64_t)R * nwarps) {
        float S[R];
        int64_t tj[R];
        int pj[R];
#pragma unroll
        for (int j = 0; j < R; ++j) {
            tj[j] = tb;
            pj[j] = pb;
            tb += dt;
            pb += dp;
            if (pb >= P) {
                pb -= P;
                ++tb;
            }
        }
        for (int kg = 0; kg < K; ++kg) {
            const int first = kg * kLanes + lane;
            const int cnt = slot_count(first, nv, stride);
            uint4 v[R][VMAX];
#pragma unroll
            for (int j = 0; j < R; ++j) {
                const int64_t task = base + (int64_t)j * nwarps;
                const int64_t t = tj[j];
                const int p = pj[j];
                const uint4 *src = reinterpret_cast<const uint4 *>(x) + t * rowvec + (int64_t)p * nv;
#pragma unroll
                for (int i = 0; i < VMAX; ++i)
                    if (task < ntask && i < cnt)
                        v[j][i] = KEEP ? __ldg(src + first + (int64_t)i * stride)
                                       : ld_stream(src + first + (int64_t)i * stride);
            }
#pragma unroll
            for (int j = 0; j < R; ++j) {
                float c = 0.f;
#pragma unroll
                for (int i = 0; i < VMAX; ++i)
                    if (base + (int64_t)j * nwarps < ntask && i < cnt) c = __fadd_rn(c, vsumsq(Tag{}, v[j][i]));
                const float b = butterfly(c);
                S[j] = kg == 0 ? b : __fadd_rn(S[j], b);
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < R; ++j) {
                const int64_t task = base + (int64_t)j * nwarps;
                if (task < ntask) stats[task] = S[j];
            }
        }
    }
}

template <class Tag, int VMAX, int R, bool TWO, bool KEEP>
__global__ void __launch_bounds__(256) stats_k(const StatsArgs a) {
    stats_body<Tag, VMAX, R, TWO, KEEP>(a);
}

// The same kernel with registers for 4 resident blocks per SM, for the
// instances whose lane holds at most 7 vectors per turn (no spills; measured
// on one tensor-parallel rank's slices at 2 ranks, 2 x 2560 columns: 66.6 ->
// 74.3 % of the HBM peak for the statistics launch). The others keep the
// bound above: stating a minimum of one block makes the compiler take more
// registers (80 -> 102 at 2 vectors x 4 tasks, 95 -> 114 us on T = 65536,
// D = 4096, P = 8).
constexpr bool stats_four_blocks(int vmax, int r) { return vmax * r <= 7; }

template <class Tag, int VMAX, int R, bool TWO, bool KEEP>
__global__ void __launch_bounds__(256, 4) stats_k4(const StatsArgs a) {
    stats_body<Tag, VMAX, R, TWO, KEEP>(a);
}

// The statistics of token t are nb blocks of Pb shard sums, block b at
// stats[b * sg + t * Pb + 0 .. Pb-1]: one block [T, P] for the split path
// (nb = 1, Pb = P), or one block per rank of a tensor-parallel group as an
// all-gather lays them out ([ranks, T, P_local]). They are added block by
// block, each in order, which is the order of the global shard index.
// The divisor Df is the full width (the local row width D, or the width
// summed over the group).
//
// MULTI = false: one row per block (tpr == blockDim.x), the row index uniform
// over the block. MULTI = true: tpr threads per row and blockDim.x / tpr rows
// per block, so narrow rows (e.g. one rank's slice) still give every thread
// UNR vectors; the row index then varies within the block, which costs
// registers (60 against 34), so wide rows keep the uniform form.
//
// apply_rows: the rows of one tensor that block bz of the tensor's gz blocks
// takes. apply_k runs it for a one-tensor launch, apply2_k for a launch over
// two tensors.
template <class Tag, bool MULTI, bool FOLD>
__device__ __forceinline__ void apply_rows(const void *x, const float *g, const float *stats, void *y,
                                           int64_t T, int32_t D, int32_t Pb, int32_t nb, int64_t sg,
                                           float Df, float eps, int32_t tpr, int64_t bz, int64_t gz) {
    constexpr int VEC = Tag::kVec;
    constexpr int UNR = 4;
    const int64_t rowvec = D / VEC;
    // tpr threads per row; rows beyond rpb * tpr threads of a block idle.
    const int nthr = MULTI ? tpr : (int)blockDim.x;
    const int rpb = MULTI ? (int)blockDim.x / tpr : 1;
    const int lt = MULTI ? (int)threadIdx.x % tpr : (int)threadIdx.x;
    const int64_t t0 = MULTI ? bz * rpb + threadIdx.x / tpr : bz;
    if (MULTI && (int)threadIdx.x >= rpb * tpr) return;
    for (int64_t t = t0; t < T; t += gz * rpb) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x) + t * rowvec;
        uint4 *dst = reinterpret_cast<uint4 *>(y) + t * rowvec;
        float r = 0.f;
        for (int64_t v0 = 0; v0 < rowvec; v0 += (int64_t)nthr * UNR) {
            uint4 xv[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int64_t v = v0 + lt + (int64_t)u * nthr;
                if (v < rowvec) xv[u] = ld_stream(src + v);
            }
            if (v0 == 0) {
                // Phase B: S = sum of the shard sums in order of the global
                // shard index (tpr is a multiple of 32, so the lanes of a warp
                // share the row, as the fold needs).
                r = factor(stat_sum<FOLD>(stats, t, Pb, nb, sg, threadIdx.x & 31), Df, eps);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int64_t v = v0 + lt + (int64_t)u * nthr;
                if (v < rowvec) st_stream(dst + v, vapply(Tag{}, xv[u], g + v * VEC, r));
            }
        }
    }
}

// One tensor per launch.
template <class Tag, bool MULTI, bool FOLD>
__global__ void __launch_bounds__(256) apply_k(const void *x, const float *g, const float *stats,
                                               void *y, int64_t T, int32_t D, int32_t Pb, int32_t nb,
                                               int64_t sg, float Df, float eps, int32_t tpr) {
    pdl_wait();
    pdl_trigger();
    apply_rows<Tag, MULTI, FOLD>(x, g, stats, y, T, D, Pb, nb, sg, Df, eps, tpr, blockIdx.x, gridDim.x);
}

// Two tensors per launch: blocks below a.split take side 0, the rest side 1.
template <class Tag, bool MULTI, bool FOLD>
__global__ void __launch_bounds__(256) apply2_k(const ApplyArgs a) {
    pdl_wait();
    pdl_trigger();
    const int z = (int)blockIdx.x >= a.split ? 1 : 0;
    // Each field selected on its own (indexing the parameter array by z
    // would copy it to the stack).
    apply_rows<Tag, MULTI, FOLD>(z ? a.side[1].x : a.side[0].x, z ? a.side[1].g : a.side[0].g,
                           z ? a.side[1].stats : a.side[0].stats, z ? a.side[1].y : a.side[0].y, a.T,
                           z ? a.side[1].D : a.side[0].D, a.Pb, a.nb, a.sg,
                           z ? a.side[1].Df : a.side[0].Df, a.eps, z ? a.side[1].tpr : a.side[0].tpr,
                           z ? (int64_t)blockIdx.x - a.split : (int64_t)blockIdx.x,
                           z ? (int64_t)gridDim.x - a.split : (int64_t)a.split);
}

// Narrow rows of at most 32 * V vectors (one rank's slice of a
// tensor-parallel group, e.g. 640 bf16 columns at 8 ranks): one warp per row
// over the flat row space of the launch (rows 0 .. T-1 of side 0, then
// T .. 2T-1 of side 1, so the warps share the two tensors' rows evenly),
// lane l taking vectors l, l + 32, ...; the row's loads are issued before
// its shard sums are read. Registers are bounded so that 6-8 blocks are
// resident per SM: a narrow row gives a thread few vectors, so what an SM
// keeps in flight comes from its thread count (the several-rows-per-block
// apply above holds 4 blocks at 58 registers). Measured on one rank's step
// at the 13B shape, same box: 8 ranks (80 vectors per row) 61.0 -> 64.3 %
// eager, 63.2 -> 66.0 % in a graph; 4 ranks (160) 68.1 -> 69.2 % eager,
// 72.7 -> 77.3 % in a graph.
// CRV, CPB, CNB: the row's vectors, the sums per block and the blocks fixed
// at compile time for the shapes that have their own instance (0: read from
// the arguments); fixed, the guards, the block index of each sum and the
// fold's length are constants, the arithmetic and its order the same.
constexpr int apply_w_blocks(int v) { return v <= 2 ? 8 : (v <= 4 ? 6 : 5); }

template <class Tag, int V, bool TWO, bool FOLD, int CRV = 0, int CPB = 0, int CNB = 0>
__global__ void __launch_bounds__(256, apply_w_blocks(V)) apply_w(const ApplyArgs a) {
    constexpr int VEC = Tag::kVec;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t T = a.T;
    const int64_t nrows = TWO ? 2 * T : T;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < nrows; w += nw) {
        const int z = TWO && w >= T ? 1 : 0;
        const int64_t t = z ? w - T : w;
        const int rowvec = CRV ? CRV : (z ? a.side[1].D : a.side[0].D) / VEC;
        const uint4 *src = reinterpret_cast<const uint4 *>(z ? a.side[1].x : a.side[0].x) + t * rowvec;
        uint4 xv[V];
#pragma unroll
        for (int i = 0; i < V; ++i)
            if (lane + 32 * i < rowvec) xv[i] = ld_stream(src + lane + 32 * i);
        // Phase B: the shard sums in order of the global shard index.
        const float r = factor(stat_sum<FOLD>(z ? a.side[1].stats : a.side[0].stats, t, CPB ? CPB : a.Pb,
                                              CNB ? CNB : a.nb, a.sg, lane),
                               z ? a.side[1].Df : a.side[0].Df, a.eps);
        uint4 *dst = reinterpret_cast<uint4 *>(z ? a.side[1].y : a.side[0].y) + t * rowvec;
        const float *g = z ? a.side[1].g : a.side[0].g;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int v = lane + 32 * i;
            if (v < rowvec) st_stream(dst + v, vapply(Tag{}, xv[i], g + (int64_t)v * VEC, r));
        }
    }
}

// ---------------------------------------------------------------- instance tables

// Tasks per warp turn: as many as keep R x VMAX <= 8 vectors per lane.
constexpr int stats_r(int vmax) { return vmax <= 2 ? 4 : (vmax <= 4 ? 2 : 1); }

template <class Tag, int V, bool KEEP>
const void *stats_fn(bool two) {
    if constexpr (stats_four_blocks(V, stats_r(V)))
        return two ? reinterpret_cast<const void *>(&stats_k4<Tag, V, stats_r(V), true, KEEP>)
                   : reinterpret_cast<const void *>(&stats_k4<Tag, V, stats_r(V), false, KEEP>);
    else
        return two ? reinterpret_cast<const void *>(&stats_k<Tag, V, stats_r(V), true, KEEP>)
                   : reinterpret_cast<const void *>(&stats_k<Tag, V, stats_r(V), false, KEEP>);
}

template <class Tag, bool KEEP>
const void *stats_table(int vmax, bool two) {
    switch (vmax) {
    case 1: return stats_fn<Tag, 1, KEEP>(two);
    case 2: return stats_fn<Tag, 2, KEEP>(two);
    case 3: return stats_fn<Tag, 3, KEEP>(two);
    case 4: return stats_fn<Tag, 4, KEEP>(two);
    case 5: return stats_fn<Tag, 5, KEEP>(two);
    case 6: return stats_fn<Tag, 6, KEEP>(two);
    case 7: return stats_fn<Tag, 7, KEEP>(two);
    case 8: return stats_fn<Tag, 8, KEEP>(two);
    default: return nullptr;
    }
}

const void *stats_kernel(int dtype, int vmax, bool two, bool keep) {
    if (dtype == 0) return keep ? stats_table<F32Tag, true>(vmax, two) : stats_table<F32Tag, false>(vmax, two);
    if (dtype == 1) return keep ? stats_table<BF16Tag, true>(vmax, two) : stats_table<BF16Tag, false>(vmax, two);
    if (dtype == 2) return keep ? stats_table<E4M3Tag, true>(vmax, two) : stats_table<E4M3Tag, false>(vmax, two);
    return nullptr;
}

template <class Tag, bool MULTI, bool FOLD>
const void *apply_fn(bool two) {
    return two ? reinterpret_cast<const void *>(&apply2_k<Tag, MULTI, FOLD>)
               : reinterpret_cast<const void *>(&apply_k<Tag, MULTI, FOLD>);
}

template <class Tag>
const void *apply_table(bool multi, bool two, bool fold) {
    if (multi) return fold ? apply_fn<Tag, true, true>(two) : apply_fn<Tag, true, false>(two);
    return fold ? apply_fn<Tag, false, true>(two) : apply_fn<Tag, false, false>(two);
}

const void *apply_kernel(int dtype, bool multi, bool two, bool fold) {
    if (dtype == 0) return apply_table<F32Tag>(multi, two, fold);
    if (dtype == 1) return apply_table<BF16Tag>(multi, two, fold);
    if (dtype == 2) return apply_table<E4M3Tag>(multi, two, fold);
    return nullptr;
}

bool apply_fold(int32_t nb) { return nb > 4; }

template <class Tag, bool TWO, bool FOLD>
const void *apply_w_fn(int v) {
    switch (v) {
    case 1: return reinterpret_cast<const void *>(&apply_w<Tag, 1, TWO, FOLD>);
    case 2: return reinterpret_cast<const void *>(&apply_w<Tag, 2, TWO, FOLD>);
    case 3: return reinterpret_cast<const void *>(&apply_w<Tag, 3, TWO, FOLD>);
    case 4: return reinterpret_cast<const void *>(&apply_w<Tag, 4, TWO, FOLD>);
    case 5: return reinterpret_cast<const void *>(&apply_w<Tag, 5, TWO, FOLD>);
    default: return nullptr;
    }
}

template <class Tag>
const void *apply_w_table(int v, bool two, bool fold) {
    if (two) return fold ? apply_w_fn<Tag, true, true>(v) : apply_w_fn<Tag, true, false>(v);
    return fold ? apply_w_fn<Tag, false, true>(v) : apply_w_fn<Tag, false, false>(v);
}

const void *apply_narrow_kernel(int dtype, int v, bool two, bool fold) {
    if (dtype == 0) return apply_w_table<F32Tag>(v, two, fold);
    if (dtype == 1) return apply_w_table<BF16Tag>(v, two, fold);
    if (dtype == 2) return apply_w_table<E4M3Tag>(v, two, fold);
    return nullptr;
}

// The instance for these shapes where one exists (two sides, bf16), else
// the general one. A tensor-parallel rank of the 13B shape (Dq = Dk = 5120,
// P = 8): at 8 ranks, 8 blocks of 1 sum (the row's width, 80 vectors, stays
// a run-time value: fixing it as well made ptxas spill under the register
// bound of 6 blocks per SM, 61.7 %), measured 64.1 -> 65.8 % eager and
// 66.0 -> 67.8 % in a graph for the rank's step; at 4 ranks, rows of 160
// vectors and 4 blocks of 2 sums, 69.0 -> 72.1 % and 77.3 -> 79.1 % (same box).
const void *apply_narrow_kernel_for(int dtype, int v, bool two, int rv0, int rv1, int Pb, int nb) {
    const bool fold = apply_fold(nb);
    if (dtype == 1 && two) {
        if (v == 3 && fold && Pb == 1 && nb == 8)
            return reinterpret_cast<const void *>(&apply_w<BF16Tag, 3, true, true, 0, 1, 8>);
        if (v == 5 && !fold && rv0 == 160 && rv1 == 160 && Pb == 2 && nb == 4)
            return reinterpret_cast<const void *>(&apply_w<BF16Tag, 5, true, false, 160, 2, 4>);
    }
    return apply_narrow_kernel(dtype, v, two, fold);
}

cudaError_t launch_apply_narrow(int dtype, int v, const ApplyArgs &a, bool two, int64_t grid, cudaStream_t s) {
    const int vec = dtype == 1 ? 8 : (dtype == 2 ? 16 : 4);
    const void *fn = apply_narrow_kernel_for(dtype, v, two, a.side[0].D / vec, a.side[1].D / vec, a.Pb, a.nb);
    if (!fn || grid < 1 || a.side[0].D / vec > 32 * v || (two && a.side[1].D / vec > 32 * v))
        return cudaErrorInvalidValue;
    void *args[] = {const_cast<ApplyArgs *>(&a)};
    return launch(fn, dim3((unsigned)grid), dim3(256), 0, s, args);
}

cudaError_t launch_stats(int dtype, int vmax, bool keep, const StatsArgs &a, int block, int64_t grid,
                         cudaStream_t s) {
    const void *fn = stats_kernel(dtype, vmax, a.split < grid, keep);
    if (!fn || a.split < 1 || a.split > grid) return cudaErrorInvalidValue;
    void *args[] = {const_cast<StatsArgs *>(&a)};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

// Threads per row of apply_k; a 256-thread block takes 256 / tpr rows at a
// time. Rows of up to 384 vectors (e.g. one rank's slice of a tensor-parallel
// group) get enough threads for UNR = 4 vectors each, so each thread keeps
// four loads in flight (measured: a 640-wide bf16 slice 27 -> 31 %, 2560-wide
// 61 -> 69.5 % of the HBM peak for a rank's step); wider rows a thread per
// vector up to 256 (measured best at 4096 wide: 97 % against 92.6 % with four
// vectors per thread).
int apply_threads_per_row(int32_t D, int dtype) {
    const int vec = dtype == 1 ? 8 : (dtype == 2 ? 16 : 4);
    const int64_t rowvec = D / vec;
    int64_t t = rowvec <= 384 ? (rowvec + 3) / 4 : rowvec;
    t = (t + 31) / 32 * 32;
    return (int)(t < 256 ? t : 256);
}

cudaError_t launch_apply(int dtype, bool multi, const ApplyArgs &a, int block, int64_t grid,
                         cudaStream_t s) {
    const void *fn = apply_kernel(dtype, multi, a.split < grid, apply_fold(a.nb));
    if (!fn || a.split < 1 || a.split > grid) return cudaErrorInvalidValue;
    for (int z = 0; z < (a.split < grid ? 2 : 1); ++z) {
        const int tpr = a.side[z].tpr;
        if (tpr < 1 || tpr > block || (!multi && tpr != block)) return cudaErrorInvalidValue;
    }
    if (a.split < grid) {
        void *args[] = {const_cast<ApplyArgs *>(&a)};
        return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
    }
    const ApplySide &d = a.side[0];
    int64_t T = a.T, sg = a.sg;
    int32_t D = d.D, Pb = a.Pb, nb = a.nb, tpr = d.tpr;
    float Df = d.Df, eps = a.eps;
    void *args[] = {const_cast<void **>(&d.x), const_cast<float **>(&d.g), const_cast<float **>(&d.stats),
                    const_cast<void **>(&d.y), &T, &D, &Pb, &nb, &sg, &Df, &eps, &tpr};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

}  // namespace qkn
