// qknorm_internal.h -- host-side interfaces between the C ABI (qknorm_api.cu)
// and the kernel launchers (qknorm_fused.cu, qknorm_split.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qkn {

// Shape of one tensor (Q or K) as the kernels see it.
struct TensorShape {
    int32_t D;    // width
    int32_t nv;   // 16-byte vectors per shard
    int32_t K;    // groups per shard: ceil(nv / (32 * kVcap))
    int32_t vmax; // vectors per lane per group: ceil(nv / (32 * K))
};

// Arguments of the fused kernels; index 0 is Q, index 1 is K.
struct FusedArgs {
    const void *x[2];
    const float *g[2];
    void *y[2];
    int64_t T;
    int32_t D[2];
    int32_t nv[2];
    int32_t K[2];
    int32_t P;
    float Df[2];
    float eps;
    int64_t ldx[2];  // row strides of the inputs, in 16-byte vectors
    int64_t ldy[2];  // row strides of the outputs, in 16-byte vectors
};

TensorShape make_shape(int32_t D, int32_t P, int vec);

// Kernel handles for occupancy queries and launches. Each returns nullptr if
// the combination does not exist.
// full: every lane holds exactly vmax vectors in every task (guard-free instance).
// greg: gamma in registers, loaded with the row (no prefetch; vmax * vec <= 32).
const void *fused_cta_kernel(int dtype, int vmax, bool prefetch, bool full, bool greg,
                             int *max_threads);
const void *fused_generic_kernel(int dtype);
// two: the instance for launches over two tensors; keep: rows read with the
// default L2 policy (for launches of at most kStatsKeepBytes, whose rows an
// apply launch soon after then finds in L2), else evict-first.
const void *stats_kernel(int dtype, int vmax, bool two, bool keep);
// Measured on one tensor-parallel rank's step at the 13B shape: 8 ranks
// (21 MB read) 58.5 -> 60.9 % eager with the rows kept; 2 ranks (84 MB)
// 81.7 -> 81.0 %, and the large split shape's statistics launch 96 -> 98 us.
constexpr int64_t kStatsKeepBytes = 32ll << 20;
// multi: the several-rows-per-block instance of apply_k (block != tpr);
// fold: the row's shard sums loaded by a warp's lanes at once (apply_fold).
const void *apply_kernel(int dtype, bool multi, bool two, bool fold);
// Whether an apply over nb blocks of gathered sums takes the lane-parallel form.
bool apply_fold(int32_t nb);

// Launchers: enqueue one kernel; return the cudaError_t of the launch.
cudaError_t launch_fused_cta(int dtype, int vmax, bool prefetch, bool full, bool greg,
                             const FusedArgs &a, int block, int64_t grid, cudaStream_t s);
// Warp per token, rows in registers (qknorm_fused_warp.cu): P shards of one
// group each, vq / vk vectors per lane per Q / K shard; block = 32 x tokens per CTA.
const void *fused_warp_kernel(int dtype, int P, int vq, int vk);
int fused_warp_max_threads();
cudaError_t launch_fused_warp(int dtype, int P, int vq, int vk, const FusedArgs &a, int block,
                              int64_t grid, cudaStream_t s);
cudaError_t launch_fused_generic(int dtype, const FusedArgs &a, int block, int64_t grid,
                                 size_t smem, cudaStream_t s);
// The split path's kernels take one or two tensors ("sides") per launch:
// blocks [0, split) work on side 0 and blocks [split, grid) on side 1, each
// side with its share of the grid. split == grid: one tensor.
struct StatsSide {
    const void *x;
    float *stats;     // [T, P]
    int32_t D, nv, K; // row width; vectors per shard; lane groups per shard
};
struct StatsArgs {
    StatsSide side[2];
    int64_t T;
    int32_t P;
    int32_t split;
};
cudaError_t launch_stats(int dtype, int vmax, bool keep, const StatsArgs &a, int block, int64_t grid,
                         cudaStream_t s);
// stats of token t: nb blocks of Pb sums, block b at stats + b * sg + t * Pb;
// Df the divisor (full width); tpr threads per row (apply_threads_per_row).
struct ApplySide {
    const void *x;
    const float *g;
    const float *stats;
    void *y;
    int32_t D, tpr;
    float Df;
};
struct ApplyArgs {
    ApplySide side[2];
    int64_t T, sg;
    int32_t Pb, nb;
    float eps;
    int32_t split;
};
int apply_threads_per_row(int32_t D, int dtype);
// multi: the several-rows-per-block instance (needed unless every side's tpr
// equals block).
cudaError_t launch_apply(int dtype, bool multi, const ApplyArgs &a, int block, int64_t grid,
                         cudaStream_t s);
// Rows of at most 32 * v vectors (v = 1..kApplyNarrowMaxV): one warp per row
// over the flat row space of one or two tensors (apply_w), 256 threads.
constexpr int kApplyNarrowMaxV = 5;
const void *apply_narrow_kernel(int dtype, int v, bool two, bool fold);
// The same, or the instance compiled for this shape (rows of rv0 and rv1
// vectors, nb blocks of Pb sums) where one exists: what launch_apply_narrow
// launches.
const void *apply_narrow_kernel_for(int dtype, int v, bool two, int rv0, int rv1, int Pb, int nb);
cudaError_t launch_apply_narrow(int dtype, int v, const ApplyArgs &a, bool two, int64_t grid, cudaStream_t s);

// The bulk-copy fed fused kernel (qknorm_fused_bulk.cu).
// tb = tokens per ring stage (1 or 2); mode: 0 any shape, 1 every lane holds
// vmax whole vectors, 2 (FP8) vmax - 1 whole vectors and half a vector of the
// last slot (see the kernel); nullptr if the combination has no instance.
const void *fused_bulk_kernel(int dtype, int vmax, bool gamma_regs, int tb, int mode,
                              int *max_threads);
uint32_t bulk_stage_stride(int64_t qbytes, int64_t kbytes, int tb);
size_t bulk_smem_bytes(int stages, uint32_t stage_stride);
int bulk_max_stages();
cudaError_t launch_fused_bulk(int dtype, int vmax, bool gamma_regs, int tb, int mode,
                              const FusedArgs &a, int stages, int block, int64_t grid,
                              uint64_t timeout_ns, cudaStream_t s);
// The shard-pair token ring (qknorm_fused_bulk.cu): P even, P <= 16, one group
// per shard, P warps per CTA; Q shards of <= 32 * vq vectors, in pairs. K
// shards of <= 16 vectors on lane halves (kw false, GQA-like shapes), or of
// <= 32 * vq vectors in pairs like Q's (kw true).
const void *fused_pair_kernel(int dtype, int vq, bool gamma_regs, bool kw);
// The same, or the instance compiled for this exact shape where one exists:
// what launch_fused_pair launches.
const void *fused_pair_kernel_for(int dtype, int vq, bool gamma_regs, bool kw, int P, int nvq, int nvk);
cudaError_t launch_fused_pair(int dtype, int vq, bool gamma_regs, bool kw, const FusedArgs &a,
                              int stages, int64_t grid, uint64_t timeout_ns, cudaStream_t s);
// The shard-pair ring with gamma staged in shared memory (qknorm_gpair.cuh):
// each warp takes two shards of one tensor (P warps per token) or, mixed, two
// shards of Q and the same two of K (P / 2 warps); nw whole slots per lane
// per shard and, for FP8, h = the last slot (<= 16 vectors) split in halves.
const void *fused_gpair_kernel(int dtype, int nwq, bool hq, int nwk, bool hk, bool mix);
// The same, or the instance compiled for this exact shape (P shards of nvq
// and nvk vectors) where one exists: what launch_fused_gpair launches.
const void *fused_gpair_kernel_for(int dtype, int nwq, bool hq, int nwk, bool hk, bool mix, int P, int nvq,
                                   int nvk);
void gpair_slots(int nv, int dtype, int *nw, bool *h);
size_t gpair_smem_bytes(int dtype, int P, int nwq, bool hq, int nwk, bool hk, int nvq, int nvk, int stages,
                        int64_t qbytes, int64_t kbytes, uint32_t *stage_base, uint32_t *gq4,
                        uint32_t *gk4, uint32_t *stride);
int gpair_max_threads();
cudaError_t launch_fused_gpair(int dtype, int nwq, bool hq, int nwk, bool hk, bool mix,
                               const FusedArgs &a, int stages, int64_t grid, uint64_t timeout_ns,
                               cudaStream_t s);
// The warp-per-row bulk-copy fed fused kernel (qknorm_fused_bulk.cu).
// wq warps take Q rows and wk warps take K rows in each CTA.
struct RowsLayout {
    uint32_t qstage, kstage, gq_off, gk_off, qring_off, kring_off;
    size_t smem_bytes;
};
const void *fused_rows_kernel(int dtype);
RowsLayout rows_layout(int64_t Dq, int64_t Dk, int es, int wq, int wk, int stages, bool gamma_smem);
cudaError_t launch_fused_rows(int dtype, const FusedArgs &a, int wq, int wk, int stages,
                              bool gamma_smem, int64_t grid, uint64_t timeout_ns, cudaStream_t s);
cudaError_t launch_bounded_wait_probe(uint64_t timeout_ns, cudaStream_t s);
cudaError_t read_device_errors(unsigned *out, bool clear);

// Arguments of the headwise kernel; index 0 is Q, index 1 is K.
struct HeadArgs {
    const void *x[2];
    const float *g[2];  // head_dim entries each, shared by the heads
    void *y[2];
    int64_t T;
    int32_t H[2];       // heads
    int32_t nv;         // 16-byte vectors per head
    float Df;           // head_dim
    float inv_df;       // 1 / head_dim when head_dim is a power of two (exact), else 0
    float eps;
    int64_t ldx[2];     // row strides, in 16-byte vectors
    int64_t ldy[2];
};
const void *headwise_kernel(int dtype, int nv);
// Work groups of the headwise kernel for nv (one warp each): T * (ceil(Q units / R) +
// ceil(K units / R)).
int64_t headwise_groups(int64_t T, int32_t Hq, int32_t Hk, int32_t nv);
cudaError_t launch_headwise(int dtype, const HeadArgs &a, int block, int64_t grid, cudaStream_t s);

// The deferred-normalisation steps (qknorm_deferred.cu).
const void *xgamma_kernel(int dtype);
const void *inv_rms_kernel(int dtype);
cudaError_t launch_xgamma(int dtype, const void *x, const float *g, void *y, int64_t T, int32_t D,
                          int block, int64_t grid, cudaStream_t s);
cudaError_t launch_inv_rms(int dtype, const void *x, float *r, int64_t T, const TensorShape &sh,
                           int32_t P, float eps, int block, int64_t grid, cudaStream_t s);

// Launch with programmatic dependent launch when enabled (qknorm_set_pdl).
bool pdl_enabled();
inline cudaError_t launch(const void *fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          void **args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// Largest dynamic shared memory the generic kernel is given (bytes).
constexpr int kGenericMaxSmem = 200 * 1024;

}  // namespace qkn
