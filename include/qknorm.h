/*
 * qknorm.h -- C ABI of libqknorm.so: layerwise Query-Key RMSNorm (QK-Norm)
 * on one NVIDIA B200 (sm_100a).
 *
 * The operation (SwiftQK technical review, "SwiftQK: When Normalization
 * Becomes the Bottleneck of Tensor Parallelism", "Prerequisites", Eq. (1) and
 * the layerwise QK-Norm paragraph): for every token t and each of the two
 * tensors X in {Q, K}, with width D and learned weight gamma,
 *
 *     y[t,j] = x[t,j] * gamma[j] / sqrt( (1/D) * sum_j x[t,j]^2 + eps ).
 *
 * The mean of squares is formed the way Section 3, Algorithm 1 decomposes
 * it: the width is cut into P equal logical shards, each shard's sum of
 * squares S[t,p] is the only statistic (Phase A), the P scalars are added
 * (Phase B), and x * gamma is formed independently of that sum (Phase B,
 * compute path) before the factor is applied (Phase C). All accumulation is
 * fp32 (Section 4, numerical precision). Here the P shards are slices of one
 * row in one GPU's memory; nothing is exchanged between GPUs.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers on the current CUDA device unless stated.
 *   The caller owns every buffer. The library allocates nothing and keeps
 *   no state besides per-device caches of launch parameters.
 * - Tensors are dense row-major: x[T, D] (row t starts at x + t*D), gamma[D]
 *   fp32, stats[T, P] fp32 (row t holds S[t,0..P-1]).
 * - dtype selects the storage type of x and y: QKNORM_F32, QKNORM_BF16 or
 *   QKNORM_E4M3 (the FP8 activations of the review's Section 4 precision
 *   study). Accumulation and the factor are always fp32. y is rounded to
 *   nearest even from fp32, once.
 * - stream is a cudaStream_t (0 = legacy default stream). Calls only
 *   enqueue work; none synchronises the host.
 * - Every pointer must be 16-byte aligned, and the shard width D/P must be a
 *   multiple of 16 (E4M3), 8 (bf16) or 4 (fp32) elements, so that every row
 *   and shard starts on a 16-byte vector.
 * - An output may be the same buffer as its own input (exact in-place); any
 *   other overlap between an output and any other buffer is rejected.
 * - T == 0 returns QKNORM_OK and launches nothing.
 * - Arguments are checked before anything is launched; a failed check
 *   launches nothing and returns one of the codes below. A CUDA error at
 *   launch returns QKNORM_ERR_CUDA; qknorm_last_error() gives its text.
 *
 * Reduction order (identical in every kernel of this library, so the fused
 * path and the split path give bit-identical outputs): a shard of nv
 * 16-byte vectors (16 E4M3, 8 bf16 or 4 fp32 values) is covered by K = ceil(nv/256)
 * groups; group k, lane l (0..31) sums, in increasing i, the per-vector sums
 * of squares of vectors v = 32k + l + 32Ki; the 32 lane sums are combined by
 * an xor butterfly (16, 8, 4, 2, 1); the K group sums are added in order of
 * k, giving S[t,p]; the P shard sums are added in order of p. A vector's sum
 * of squares is e0*e0 followed by fused multiply-adds of e1..e_last; for FP8
 * (16 values) it is h(e0..e7) + h(e8..e15), where h of 8 values is the sum of
 * two chains formed side by side (as packed f32x2 operations): the even
 * elements' squares (e0*e0, then fused multiply-adds of e2, e4, e6) plus the
 * odd elements' (e1*e1, then e3, e5, e7).
 * Then r = rsqrt(S / D + eps) and y = (x * gamma) * r, each step fp32.
 */
#ifndef QKNORM_H
#define QKNORM_H

#include <stdint.h>

#if defined(__GNUC__)
#define QKNORM_API __attribute__((visibility("default")))
#else
#define QKNORM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QKNORM_F32 = 0,
    QKNORM_BF16 = 1,
    QKNORM_E4M3 = 2   /* FP8 E4M3 (OCP "fn": max 448, no infinities); outputs are
                         rounded to nearest even and saturate to +-448 */
} qknorm_dtype;

typedef enum {
    QKNORM_OK = 0,
    QKNORM_ERR_INVALID_ARG = 1, /* null pointer with T > 0, T < 0, D <= 0, P <= 0,
                                   D % P != 0, eps < 0 or not finite, overlapping
                                   buffers */
    QKNORM_ERR_MISALIGNED = 2,  /* a pointer not 16-byte aligned */
    QKNORM_ERR_UNSUPPORTED = 3, /* unknown dtype, or D/P not a multiple of the
                                   16-byte vector (8 bf16 / 4 fp32 elements) */
    QKNORM_ERR_CUDA = 4         /* the CUDA runtime reported an error */
} qknorm_status;

/*
 * qknorm_fwd -- the single-pass fused QK-Norm of Q and K.
 *
 * Algorithm 1 (Phases A, B and C) for every token of both tensors, in one
 * launch: each element of q and k is read once from HBM and each element of
 * out_q and out_k written once; the per-shard statistics never leave the SM.
 *
 *   q       [T, Dq] input, dtype          out_q [T, Dq] output, dtype
 *   k       [T, Dk] input, dtype          out_k [T, Dk] output, dtype
 *   gamma_q [Dq] fp32, gamma_k [Dk] fp32
 *   T       tokens (rows); Dq, Dk widths; P logical shards of each width
 *           (Dq/P and Dk/P are the shard widths)
 *   eps     added to the mean of squares inside the root (Eq. (1))
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_fwd(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
               void *out_q, void *out_k, int64_t T, int32_t Dq, int32_t Dk, int32_t P,
               float eps, int32_t dtype, void *stream);

/*
 * qknorm_fwd_strided -- qknorm_fwd on rows that are not dense: row t of q
 * starts at q + t*ldq elements (likewise k, out_q, out_k with ldk, ldoq,
 * ldok). The common use is Q and K as column slices of one fused QKV
 * projection buffer (q = qkv, k = qkv + Dq, ldq = ldk = Dq + 2*Dk), normalised
 * in place (out_q = q, out_k = k, same strides) or into dense outputs.
 * Strides are in elements, >= the width, and multiples of the 16-byte vector
 * (8 bf16 / 4 fp32). Tensors with the same stride may interleave (the slices
 * of one buffer) as long as their rows do not touch; an output may be its
 * own input with the same stride. qknorm_fwd is this call with ld = D.
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_fwd_strided(const void *q, const void *k, const float *gamma_q,
                                  const float *gamma_k, void *out_q, void *out_k, int64_t T,
                                  int32_t Dq, int32_t Dk, int32_t P, float eps, int32_t dtype,
                                  int64_t ldq, int64_t ldk, int64_t ldoq, int64_t ldok,
                                  void *stream);

/*
 * qknorm_headwise_fwd -- headwise QK-Norm of Q and K: one factor per head.
 *
 * SwiftQK technical review, "Prerequisites" (layerwise vs. headwise) and
 * Section 4c: the reduction of Eq. (1) spans one head's head_dim elements;
 * gamma has head_dim entries shared by all heads of its tensor. For head h
 * of row t: S = sum of squares of the head in the reduction order above
 * (the head as the only shard), r = rsqrt(S / head_dim + eps),
 * y = (x * gamma) * r.
 *   q [T, Hq*head_dim] with row stride ldq, k [T, Hk*head_dim] stride ldk;
 *   gamma_q, gamma_k [head_dim] fp32; out_q, out_k strides ldoq, ldok.
 * head_dim must be a multiple of the 16-byte vector and at most 256 vectors;
 * strides as in qknorm_fwd_strided (pass ld = H*head_dim for dense rows).
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_headwise_fwd(const void *q, const void *k, const float *gamma_q,
                                   const float *gamma_k, void *out_q, void *out_k, int64_t T,
                                   int32_t Hq, int32_t Hk, int32_t head_dim, float eps,
                                   int32_t dtype, int64_t ldq, int64_t ldk, int64_t ldoq,
                                   int64_t ldok, void *stream);

/*
 * qknorm_partial_sumsq -- the statistics half of the split path.
 *
 * Algorithm 1, Phase A for one tensor: stats[t*P + p] = fp32 sum of
 * squares of shard p of row t (the scalar each rank publishes to its IPC
 * slot in the review's multi-GPU form), in the reduction order above.
 *   x [T, D] input, dtype (16-byte aligned); stats [T, P] fp32 output
 *   (4-byte alignment suffices: it is written one value at a time).
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_partial_sumsq(const void *x, float *stats, int64_t T, int32_t D, int32_t P,
                         int32_t dtype, void *stream);

/*
 * qknorm_apply -- the apply half of the split path.
 *
 * Algorithm 1, Phases B and C for one tensor, given the statistics:
 * S = stats[t,0] + ... + stats[t,P-1] (in order of p), r = rsqrt(S/D + eps),
 * out[t,j] = (x[t,j] * gamma[j]) * r. A caller that already holds combined
 * per-token sums passes them as stats [T, 1] with P = 1.
 *   x [T, D] input, dtype; gamma [D] fp32; stats [T, P] fp32 (4-byte
 *   alignment suffices: it is read one value at a time); out [T, D].
 * With stats from qknorm_partial_sumsq, out equals qknorm_fwd's bit for bit.
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_apply(const void *x, const float *gamma, const float *stats, void *out,
                 int64_t T, int32_t D, int32_t P, float eps, int32_t dtype, void *stream);

/*
 * qknorm_apply_tp -- the apply step of one rank of a tensor-parallel group.
 *
 * SwiftQK technical review, Section 3, Algorithm 1 in its tensor-parallel
 * form: the hidden dimension is split across `ranks` GPUs; each rank holds
 * the D_local-wide slice of every row (its P_local shards), forms its shard
 * sums (Phase A, qknorm_partial_sumsq on its slice), the group exchanges
 * them, and each rank finishes its own slice (Phases B and C) with the full
 * width H_total = ranks * D_local as the divisor. This call is that last
 * step, given the exchanged sums as an all-gather of every rank's [T, P_local]
 * leaves them:
 *   stats: ranks blocks of [T, P_local] fp32, block g (rank g's shard sums)
 *   at stats + g * stats_block_stride floats (0 means T * P_local, the dense
 *   [ranks, T, P_local]; a larger stride serves a gather of several tensors'
 *   sums at once, e.g. [ranks, 2, T, P_local] for Q and K with stride
 *   2 * T * P_local and stats offset by T * P_local for K; stats need only
 *   4-byte alignment here and in qknorm_apply);
 *   S = the ranks * P_local sums in order of the global shard index
 *       (g * P_local + p), r = rsqrt(S / (ranks * D_local) + eps),
 *   out[t,j] = (x[t,j] * gamma[j]) * r for the local slice.
 *   x [T, D_local] input, dtype; gamma [D_local] fp32 (the rank's slice of
 *   gamma); out [T, D_local] output, dtype.
 * With rank g's stats from qknorm_partial_sumsq(x_g, ..., D_local, P_local),
 * out on rank g equals columns [g * D_local, (g + 1) * D_local) of qknorm_fwd
 * on the whole rows with P = ranks * P_local, bit for bit. ranks = 1 is
 * qknorm_apply. Errors as qknorm_apply; also QKNORM_ERR_INVALID_ARG for
 * ranks < 1 or a stride below T * P_local (overlapping blocks).
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_apply_tp(const void *x, const float *gamma, const float *stats,
                               int64_t stats_block_stride, void *out, int64_t T, int32_t D_local,
                               int32_t P_local, int32_t ranks, float eps, int32_t dtype, void *stream);

/*
 * qknorm_partial_sumsq_qk -- qknorm_partial_sumsq of Q and of K in one launch.
 *
 * Algorithm 1, Phase A for both tensors of a layer (e.g. one rank's Q and K
 * slices in the tensor-parallel form): stats_q [T, P] from q [T, Dq] and
 * stats_k [T, P] from k [T, Dk], each exactly as qknorm_partial_sumsq
 * writes it (bit for bit). The launch's blocks are shared between the two in
 * proportion to their widths, so the pair costs one launch's fixed start and
 * drain instead of two. Same requirements as qknorm_partial_sumsq for each
 * tensor; QKNORM_ERR_INVALID_ARG also when a statistics array overlaps the
 * other statistics array or the other tensor.
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_partial_sumsq_qk(const void *q, const void *k, float *stats_q, float *stats_k,
                                       int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                                       void *stream);

/*
 * qknorm_apply_tp_qk -- qknorm_apply_tp of Q and of K in one launch.
 *
 * Phases B and C of Algorithm 1's tensor-parallel form for both tensors of
 * one rank: out_q from q [T, Dq_local], gamma_q and stats_q, and out_k from
 * k [T, Dk_local], gamma_k and stats_k, each exactly as qknorm_apply_tp
 * computes it (bit for bit), with one stats_block_stride for both (an
 * all-gather of [2, T, P_local] per rank gives [ranks, 2, T, P_local]:
 * stats_q = its base, stats_k = base + T * P_local, stride 2 * T * P_local).
 * ranks = 1 with stride 0 is qknorm_apply of both tensors. Same requirements
 * as qknorm_apply_tp for each tensor; QKNORM_ERR_INVALID_ARG also when an
 * output overlaps the other output or any input of the other tensor.
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_apply_tp_qk(const void *q, const void *k, const float *gamma_q,
                                  const float *gamma_k, const float *stats_q, const float *stats_k,
                                  int64_t stats_block_stride, void *out_q, void *out_k, int64_t T,
                                  int32_t Dq_local, int32_t Dk_local, int32_t P_local, int32_t ranks,
                                  float eps, int32_t dtype, void *stream);

/*
 * qknorm_fwd_host -- qknorm_fwd on rows in HOST memory, end to end: the rows
 * go to the device, are normalised there and come back (no counterpart in
 * the paper; it is the path a caller with host-resident activations takes).
 *
 * The T tokens are processed in chunks of chunk_tokens (0 = 1024). Each chunk
 * is copied host-to-device into one of three workspace sets, normalised in
 * place by qknorm_fwd on `stream`, and copied back, with the copies on two
 * streams of the library's own, so the host-to-device copy of one chunk, the
 * kernel of the next and the device-to-host copy of a third overlap (the two
 * copy directions use separate copy engines). Results equal qknorm_fwd's bit
 * for bit.
 *   q, k [T, Dq], [T, Dk] host input, dtype; out_q, out_k host outputs of
 *   the same shapes (each may be its own input; no other overlap); gamma_q,
 *   gamma_k fp32 on the DEVICE; workspace: device memory of at least
 *   qknorm_fwd_host_workspace(chunk_tokens, Dq, Dk, dtype) bytes, 16-byte
 *   aligned, owned by the caller and not used by anything else until the
 *   call's work has completed.
 * Ordering: all work is ordered after the work already on `stream`, and work
 * enqueued on `stream` afterwards waits until the outputs are in host memory
 * (synchronise `stream` before reading them). Host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister); pageable memory works but its copies do
 * not overlap. Enqueueing is serialised across host threads.
 * Returns a qknorm_status (QKNORM_ERR_INVALID_ARG also for a workspace that
 * is too small or a negative chunk_tokens).
 */
QKNORM_API int qknorm_fwd_host(const void *q, const void *k, const float *gamma_q,
                               const float *gamma_k, void *out_q, void *out_k, int64_t T,
                               int32_t Dq, int32_t Dk, int32_t P, float eps, int32_t dtype,
                               void *workspace, int64_t workspace_bytes, int64_t chunk_tokens,
                               void *stream);

/* Workspace bytes qknorm_fwd_host needs for chunk_tokens (0 = the default),
 * or -1 for invalid widths or dtype. */
QKNORM_API int64_t qknorm_fwd_host_workspace(int64_t chunk_tokens, int32_t Dq, int32_t Dk,
                                             int32_t dtype);

/*
 * qknorm_xgamma -- the weight multiply alone: out[t,j] = x[t,j] * gamma[j],
 * rounded once to dtype, no normalisation.
 *
 * Algorithm 1's Phase B compute path on its own. It is also what a deferred
 * normalisation stores when a later RMSNorm cancels the per-token factor
 * (pull request "perf(dsv4 decode swa): deferred attention RMSNorm and dep
 * cleanup", attn_norm_xgamma): since RMSNorm(s * z) = RMSNorm(z) for a
 * per-token s > 0, the factor of an earlier norm need not be applied.
 *   x [T, D] input, dtype; gamma [D] fp32; out [T, D] output, dtype.
 * D must be a multiple of the 16-byte vector (8 bf16 / 4 fp32 elements).
 * out may be x (exact in-place). Returns a qknorm_status.
 */
QKNORM_API int qknorm_xgamma(const void *x, const float *gamma, void *out, int64_t T, int32_t D,
                             int32_t dtype, void *stream);

/*
 * qknorm_inv_rms -- the per-token factor alone: inv_rms[t] = rsqrt(S[t]/D + eps),
 * S[t] formed from P shard sums in the reduction order above, fp32.
 *
 * The one dynamic scalar per token that RMSNorm factors into besides the
 * static weight (abstract "QK-Normed MLA: QK normalization without full key
 * caching"); bit-identical to the factor qknorm_fwd applies to that row, so
 * out = xgamma(x) * inv_rms reproduces Eq. (1) up to the rounding of xgamma.
 *   x [T, D] input, dtype; inv_rms [T] fp32 output.
 * Returns a qknorm_status.
 */
QKNORM_API int qknorm_inv_rms(const void *x, float *inv_rms, int64_t T, int32_t D, int32_t P,
                              float eps, int32_t dtype, void *stream);

/*
 * qknorm_split_noalloc -- qknorm_partial_sumsq followed by qknorm_apply in one
 * call, with the [T, P] statistics kept in a buffer inside the library, so
 * that the caller allocates nothing (no counterpart in the paper; it is a
 * convenience for callers who cannot allocate device memory, e.g. because all
 * device memory belongs to a framework's pool, or because cudaMalloc's
 * implicit synchronisation is unacceptable in their loop).
 *
 * Arguments, layouts, checks and results are those of the two calls it
 * makes; out equals qknorm_fwd's output for that tensor bit for bit.
 * The library holds one buffer of qknorm_split_noalloc_max_stats() floats
 * (2^20, 4 MiB) on each device that loads it, until exit; T * P beyond that
 * returns QKNORM_ERR_UNSUPPORTED without launching anything. The call itself
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 * The first call on a device looks up the buffer's device address (with that
 * device current); make that first call before any stream capture. The first
 * call after the device's context is destroyed and re-created (e.g. by
 * cudaDeviceReset) looks the address up again, since the buffer may then sit
 * elsewhere. All calls share the buffer: calls that overlap on the GPU race.
 * Nothing in it needs clearing between calls.
 */
QKNORM_API int qknorm_split_noalloc(const void *x, const float *gamma, void *out, int64_t T,
                                    int32_t D, int32_t P, float eps, int32_t dtype, void *stream);

/* The buffer size of qknorm_split_noalloc, in floats (the largest T * P). */
QKNORM_API int64_t qknorm_split_noalloc_max_stats(void);

/* Static text for a qknorm_status value ("unknown status" otherwise). */
QKNORM_API const char *qknorm_status_string(int status);

/* Text of the last CUDA error seen by this thread ("" if none). */
QKNORM_API const char *qknorm_last_error(void);

/* Kernel variants of qknorm_fwd, for qknorm_plan_fwd and qknorm_force_variant. */
typedef enum {
    QKNORM_VARIANT_AUTO = -1,
    QKNORM_VARIANT_CTA = 0,     /* CTA per token: one warp per (shard, group), row
                                   held in registers, persistent grid, next token
                                   prefetched when a CTA has more than one */
    QKNORM_VARIANT_WARP = 1,    /* warp per token: one warp walks all shards of a
                                   token's Q and K rows, holding them in registers
                                   (shards of one lane group, at most 32 vectors per
                                   lane); other shapes loop and re-read the row */
    QKNORM_VARIANT_GENERIC = 2, /* CTA per token, any shape: warps loop over the
                                   shard groups, re-read the row to apply */
    QKNORM_VARIANT_BULK = 3,    /* as CTA, but rows arrive by bulk asynchronous
                                   copies (TMA engine) into a ring of token stages
                                   in shared memory, completed on mbarriers */
    QKNORM_VARIANT_ROWS = 4,    /* warp per row: a CTA has a pool of warps for
                                   Q rows and one for K rows; each warp has its
                                   own ring of bulk-copied row stages, walks all
                                   P shards of the row itself and applies from
                                   shared memory; no CTA barrier per row */
    QKNORM_VARIANT_PAIR = 5,    /* as BULK with P warps per token instead of 2P
                                   (GQA-like shapes: P even, K shards of <= 16
                                   vectors): a warp takes two Q shards, or two
                                   K shards on its lane halves */
    QKNORM_VARIANT_GPAIR = 6    /* as PAIR with gamma staged once per CTA in shared
                                   memory (no gamma registers): a warp takes two
                                   shards of one tensor, or (mixed, when Q and K
                                   shards differ) the same two shards of Q and of
                                   K; FP8 splits a last slot of <= 16 vectors in
                                   halves over the lanes */
} qknorm_variant;

/* A launch plan chosen by the selector (host-side description). */
typedef struct {
    int32_t variant;     /* qknorm_variant */
    int32_t block;       /* threads per CTA */
    int64_t grid;        /* CTAs */
    int32_t vmax;        /* 16-byte vectors per lane per (shard, group); 0 if looped */
    int32_t prefetch;    /* 1 if a CTA prefetches its next token */
    int32_t groups_q;    /* K for a Q shard */
    int32_t groups_k;    /* K for a K shard */
    int32_t stages;      /* ring stages per CTA (bulk) or per warp (rows), else 0 */
    int32_t tokens_per_stage; /* tokens a bulk stage holds (1 or 2), else 0 */
    int32_t gamma_regs;  /* 1 if each lane keeps its gamma in registers (bulk, pair; CTA:
                            loaded together with the row) */
    int32_t full_lanes;  /* 1 if every lane holds exactly vmax vectors per task; 2 (FP8,
                            bulk) if every lane holds vmax - 1 and the last slot's
                            <= 16 vectors are split in halves over the 32 lanes */
    int64_t smem_bytes;  /* dynamic shared memory per CTA */
    int32_t q_warps;     /* rows: warps per CTA that take Q rows (the rest take K rows) */
    int32_t gamma_smem;  /* rows: 1 if gamma is staged in shared memory, 0 if read via L1 */
    int32_t k_pairs;     /* pair: 1 if each K warp takes two K shards like a Q warp, 0 if
                            two K shards of <= 16 vectors share a warp's lane halves */
    int32_t vmax_k;      /* warp: 16-byte vectors per lane per K shard (vmax is Q's);
                            0 when the warp variant loops over the row instead;
                            gpair: whole slots per lane per K shard (vmax: Q's) */
    int32_t half_slots;  /* gpair: bit 0 Q's, bit 1 K's last slot split in lane halves */
    int32_t mixed;       /* gpair: 1 if every warp takes Q and K shards */
} qknorm_plan;

/*
 * qknorm_plan_fwd -- the selector, as a pure host function (no CUDA call).
 *
 * Chooses the kernel variant, block and grid for qknorm_fwd given the shape
 * and the device's SM count and resident-CTA count for the chosen kernel
 * (num_sms, blocks_per_sm; pass <= 0 for blocks_per_sm to let the plan use
 * its block-size-only estimate). Honours qknorm_force_variant. Returns
 * QKNORM_OK and fills *plan, or an argument error code.
 */
QKNORM_API int qknorm_plan_fwd(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                    int32_t num_sms, int32_t blocks_per_sm, qknorm_plan *plan);

/*
 * qknorm_force_variant -- process-wide override of the selector for tests and
 * benchmarks: variant (QKNORM_VARIANT_AUTO restores automatic choice) and,
 * if grid > 0, the CTA count of a persistent launch. A forced variant that
 * cannot run a shape makes qknorm_fwd return QKNORM_ERR_UNSUPPORTED.
 * Not thread-safe with concurrent qknorm_fwd calls. Returns a qknorm_status.
 */
QKNORM_API int qknorm_force_variant(int32_t variant, int64_t grid);

/*
 * qknorm_launch_plan -- the plan qknorm_fwd would use on the current device
 * (queries the SM count and occupancy; no kernel runs). Returns a status.
 */
QKNORM_API int qknorm_launch_plan(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                       qknorm_plan *plan);

/*
 * qknorm_set_tuning -- process-wide tuning of the bulk variant for tests and
 * benchmarks: ring stages per CTA (0 = automatic), tokens per stage (0 =
 * automatic, else 1 or 2), gamma in registers (-1 = automatic, 0 = no,
 * 1 = yes; also the CTA variant's gamma registers, where an instance has
 * them), the bound of every wait in milliseconds (0 = the default of
 * 2000 ms). A combination without a kernel instance makes qknorm_fwd return
 * QKNORM_ERR_UNSUPPORTED. Not thread-safe with concurrent calls.
 */
QKNORM_API int qknorm_set_tuning(int32_t stages, int32_t tokens_per_stage, int32_t gamma_regs,
                                 int32_t wait_limit_ms);

/*
 * qknorm_set_rows_tuning -- process-wide tuning of the warp-per-row variant:
 * warps per CTA of the Q pool and of the K pool (both 0 = automatic: the
 * split in proportion to Dq : Dk with the most resident warps per SM; else
 * each >= 1 and their sum <= 16), row stages per warp (0 = automatic) and
 * gamma staging (-1 = automatic, 0 = read through L1, 1 = staged in shared
 * memory once per CTA). Not thread-safe with concurrent calls.
 */
QKNORM_API int qknorm_set_rows_tuning(int32_t q_warps, int32_t k_warps, int32_t stages,
                                      int32_t gamma_smem);

/*
 * qknorm_set_pdl -- programmatic dependent launch on (1, the default) or off
 * (0), process-wide. When on, every kernel is launched with the programmatic
 * stream serialization attribute: it may start while the previous kernel in
 * the stream finishes, does only shared-memory set-up until that kernel has
 * completed and its memory is visible (griddepcontrol.wait), and lets the
 * next such kernel start early. Results are the same either way.
 */
QKNORM_API int qknorm_set_pdl(int32_t enable);

/*
 * qknorm_device_errors -- read (and with clear != 0, reset) the library's
 * device error word. Bit 1: a bounded wait of the bulk variant ran out of
 * time (that launch's outputs are incomplete); bit 2: copies were still in
 * flight when such a CTA left. Synchronises with the device (blocking copy).
 */
QKNORM_API int qknorm_device_errors(uint32_t *flags, int32_t clear);

/*
 * qknorm_selftest_bounded_wait -- launch one CTA that waits on an mbarrier
 * nobody arrives on, with the bulk variant's bounded wait and the given limit
 * (nanoseconds). It must time out and set bit 1 of the device error word.
 * No copy is in flight, so nothing is left pending. Asynchronous on stream.
 */
QKNORM_API int qknorm_selftest_bounded_wait(uint64_t limit_ns, void *stream);

/* ABI version of this header (major * 100 + minor). */
QKNORM_API int qknorm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKNORM_H */
