// qknorm_fused_bulk.cu -- the fused QK-Norm kernel fed by bulk copies.
//
// Same computation and reduction order as fused_cta (SwiftQK technical
// review, Section 3, Algorithm 1, Phases A-C; one warp per (tensor, shard,
// group) task; persistent stride loop over tokens), but the rows reach the SM
// through the TMA engine: one elected thread issues cp.async.bulk copies of
// whole Q and K rows into a ring of S stages in shared memory, each stage
// completed on its own mbarrier. Bytes in flight per SM are then set by
// shared memory, not by registers.
//
// A stage holds TB tokens (those the CTA meets in TB consecutive turns of its
// stride loop). One pass of the loop reduces all TB tokens with independent
// chains and butterflies, crosses ONE CTA barrier for all of them, and streams
// their outputs, so the serial per-token work (shared-memory reads, FMA chain,
// butterfly, barrier, combine, divide, rsqrt) overlaps across TB tokens and
// each lane's gamma registers serve TB tokens.
//
// Per pass: wait for the stage (bounded), copy this lane's vectors of the TB
// tokens from shared memory to registers, chains, butterflies, group sums to
// shared memory; one barrier; thread 0 refills the stage with the tokens S
// passes ahead; every lane forms the TB factors and writes (x*gamma)*r.
#include "qknorm_bulk.cuh"
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

__device__ unsigned int g_device_errors;

struct BulkArgs {
    uint32_t stages;       // S
    uint32_t qbytes;       // bytes of one Q row
    uint32_t kbytes;       // bytes of one K row
    uint32_t stage_stride; // bytes between stages (multiple of 128)
    uint64_t timeout_ns;   // bound of every wait
};

// Shared memory: [S mbarriers | pad][red: 2 x TBMAX x 32 floats][S stages].
constexpr uint32_t kBarBytes = 128;
constexpr int kMaxTB = 4;
constexpr uint32_t kRedBytes = 2 * kMaxTB * 32 * sizeof(float);
constexpr uint32_t kStageBase = kBarBytes + kRedBytes;
constexpr uint32_t kMaxStages = 16;

}  // namespace qkn

// Gamma staged in shared memory in a lane-permuted layout, and the shard-pair
// ring built on it (they share this file's device error word).
#include "qknorm_gpair.cuh"

namespace qkn {

// MODE (how lanes hold vectors): 0 any shape (guards); 1 every lane of every
// task holds exactly VMAX vectors (no guards); 2 (FP8) every lane holds
// VMAX - 1 whole vectors and the last slot's r <= 16 vectors are split in
// halves over the 32 lanes (lane l and l + 16 take the low and high 8 bytes
// of vector l), so the last slot costs half a slot instead of running with
// half the lanes idle. The vector sum of squares is defined as the sum of its
// two halves' sums, so the split changes no bits.
template <class Tag, int VMAX, bool GREG, int TB, int MODE, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) fused_bulk(const FusedArgs a, const BulkArgs b) {
    constexpr int VEC = Tag::kVec;
    constexpr bool FULL = MODE == 1;
    constexpr bool HALF = MODE == 2;
    constexpr int NW = HALF ? VMAX - 1 : VMAX;     // whole-vector slots
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    float(*red)[kMaxTB][32] = reinterpret_cast<float(*)[kMaxTB][32]>(smem + kBarBytes);
    unsigned char *stages = smem + kStageBase;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int nt0 = a.P * a.K[0];
    const int z = warp < nt0 ? 0 : 1;
    const int jj = z ? warp - nt0 : warp;
    const int K = z ? a.K[1] : a.K[0];
    const int p = jj / K;
    const int kg = jj - p * K;
    const int nv = z ? a.nv[1] : a.nv[0];
    const int stride = kLanes * K;
    const int first = kg * kLanes + lane;
    const int cnt = (FULL || HALF) ? NW : slot_count(first, nv, stride);
    // HALF: this lane's half of the last slot: vector hv of the slot, bytes
    // 8*hh .. 8*hh + 7 of it; hok if that vector exists.
    const int hv = lane & 15, hh = lane >> 4;
    const bool hok = HALF && hv < nv - kLanes * NW;
    const int64_t hcol = (int64_t)p * nv + kLanes * NW + hv;   // its vector index in the row
    const int64_t ldy = z ? a.ldy[1] : a.ldy[0];     // output row stride, in vectors
    const int64_t col0 = (int64_t)p * nv + first;
    uint4 *ys = reinterpret_cast<uint4 *>(z ? a.y[1] : a.y[0]) + col0;
    const float *gs = (z ? a.g[1] : a.g[0]) + col0 * VEC;
    const float Df = z ? a.Df[1] : a.Df[0];
    const float eps = a.eps;
    const int red_base = z ? nt0 : 0;
    const uint32_t tok_bytes = b.qbytes + b.kbytes;
    // This lane's first vector inside a token of a stage (Q row, then K row).
    const uint32_t lane_off = (z ? b.qbytes : 0u) + (uint32_t)col0 * 16u;
    const uint32_t half_off = (z ? b.qbytes : 0u) + (uint32_t)hcol * 16u + 8u * hh;

    const int64_t T = a.T;
    const int64_t G = gridDim.x;
    const int S = (int)b.stages;
    const char *qsrc = static_cast<const char *>(a.x[0]);
    const char *ksrc = static_cast<const char *>(a.x[1]);
    const int64_t ldq_b = a.ldx[0] * 16, ldk_b = a.ldx[1] * 16;   // input row strides, bytes

    // Tokens of pass n: blockIdx.x + (n*TB + j)*G, j < TB (those below T).
    auto issue = [&](int s, int64_t n) {
        unsigned char *st = stages + (size_t)s * b.stage_stride;
        const int64_t t0 = blockIdx.x + n * TB * G;
        int ntok = 0;
#pragma unroll
        for (int j = 0; j < TB; ++j) ntok += (t0 + j * G < T) ? 1 : 0;
        mbar_arrive_expect_tx(&full[s], (uint32_t)ntok * tok_bytes);
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const int64_t tt = t0 + j * G;
            if (tt < T) {
                bulk_copy_g2s(st + j * tok_bytes, qsrc + tt * ldq_b, b.qbytes, &full[s]);
                bulk_copy_g2s(st + j * tok_bytes + b.qbytes, ksrc + tt * ldk_b, b.kbytes, &full[s]);
            }
        }
    };

    const int64_t npass = (T - blockIdx.x + TB * G - 1) / (TB * G);  // >= 1 since blockIdx.x < T
    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Shared memory only so far; global reads start after the previous grid.
    pdl_wait();
    pdl_trigger();
    if (tid == 0) {
        for (int s = 0; s < S && s < npass; ++s) issue(s, s);
    }

    float gam[GREG ? VMAX * VEC : 1];
    if (GREG) {
#pragma unroll
        for (int i = 0; i < NW; ++i)
            if (FULL || HALF || i < cnt) {
#pragma unroll
                for (int e = 0; e < VEC; e += 4) {
                    const float4 g4 = __ldg(reinterpret_cast<const float4 *>(
                        gs + (int64_t)i * stride * VEC + e));
                    gam[i * VEC + e] = g4.x;
                    gam[i * VEC + e + 1] = g4.y;
                    gam[i * VEC + e + 2] = g4.z;
                    gam[i * VEC + e + 3] = g4.w;
                }
            }
        if (HALF && hok) {
#pragma unroll
            for (int e = 0; e < VEC / 2; e += 4) {
                const float4 g4 = __ldg(reinterpret_cast<const float4 *>(
                    (z ? a.g[1] : a.g[0]) + hcol * VEC + 8 * hh + e));
                gam[NW * VEC + e] = g4.x;
                gam[NW * VEC + e + 1] = g4.y;
                gam[NW * VEC + e + 2] = g4.z;
                gam[NW * VEC + e + 3] = g4.w;
            }
        }
    }

    int s = 0;
    uint32_t phase = 0;
    int buf = 0;
    for (int64_t n = 0; n < npass; ++n) {
        const int64_t t0 = blockIdx.x + n * TB * G;
        const bool ok = mbar_wait_bounded(&full[s], phase, b.timeout_ns);
        const unsigned char *st = stages + (size_t)s * b.stage_stride + lane_off;
        uint4 cur[TB][NW > 0 ? NW : 1];
        uint2 hlf[TB];
        const unsigned char *sth = stages + (size_t)s * b.stage_stride + half_off;
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const uint4 *src = reinterpret_cast<const uint4 *>(st + j * tok_bytes);
#pragma unroll
            for (int i = 0; i < NW; ++i)
                cur[j][i] = ((FULL || HALF || i < cnt) && (j == 0 || t0 + j * G < T)) ? src[i * stride]
                                                                                      : make_uint4(0, 0, 0, 0);
            if constexpr (HALF)
                hlf[j] = (hok && (j == 0 || t0 + j * G < T))
                             ? *reinterpret_cast<const uint2 *>(sth + j * tok_bytes)
                             : make_uint2(0, 0);
        }
        // Phase A for TB tokens: independent chains and butterflies. A lane's
        // missing vectors are its last slots and read as zeros, whose sum of
        // squares (+0) leaves the chain unchanged, so the chains need no branch.
        float c[TB];
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            c[j] = 0.f;
#pragma unroll
            for (int i = 0; i < NW; ++i) c[j] = __fadd_rn(c[j], vsumsq(Tag{}, cur[j][i]));
            if constexpr (HALF) {
                // The last slot: this lane's half sum; lane l < 16 adds the
                // high half's sum from lane l + 16 to its own low half (the
                // vector's sum, by its definition), then to its chain.
                const float h = e4m3x8_sumsq(hlf[j].x, hlf[j].y);
                const float hi = __shfl_down_sync(kFull, h, 16);
                if (lane < 16) c[j] = __fadd_rn(c[j], __fadd_rn(h, hi));
            }
        }
#pragma unroll
        for (int j = 0; j < TB; ++j) c[j] = butterfly(c[j]);
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < TB; ++j) red[buf][j][warp] = c[j];
        }
        if (__syncthreads_or(!ok)) {
            // A stage never arrived: record it, let copies in flight land, leave.
            if (tid == 0) {
                atomicOr(&g_device_errors, kErrWaitTimeout);
                int ds = s;
                uint32_t dp = phase;
                for (int64_t m = n; m < npass && m < n + S; ++m) {
                    if (!mbar_wait_bounded(&full[ds], dp, b.timeout_ns))
                        atomicOr(&g_device_errors, kErrDrainTimeout);
                    if (++ds == S) {
                        ds = 0;
                        dp ^= 1u;
                    }
                }
            }
            return;
        }
        // Every lane holds its vectors in registers now: refill this stage.
        if (tid == 0 && n + S < npass) {
            fence_proxy_async_smem();
            issue(s, n + S);
        }
        // Phase B: shard sums in order and the factor; weight multiply, Phase C.
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const int64_t t = t0 + j * G;
            if (j == 0 || t < T) {
                const float r = factor(combine_fast(&red[buf][j][red_base], a.P, K), Df, eps);
                uint4 *dst = ys + t * ldy;
#pragma unroll
                for (int i = 0; i < NW; ++i)
                    if (FULL || HALF || i < cnt) {
                        uint4 y;
                        if (GREG)
                            y = vapply_regs(Tag{}, cur[j][i], &gam[i * VEC], r);
                        else
                            y = vapply(Tag{}, cur[j][i], gs + (int64_t)i * stride * VEC, r);
                        st_stream(dst + (int64_t)i * stride, y);
                    }
                if constexpr (HALF) {
                  if (hok) {
                    float gh[VEC / 2];
#pragma unroll
                    for (int e = 0; e < VEC / 2; ++e)
                        gh[e] = GREG ? gam[NW * VEC + e]
                                     : __ldg((z ? a.g[1] : a.g[0]) + hcol * VEC + 8 * hh + e);
                    const uint2 y = vapply_half(Tag{}, hlf[j], gh, r);
                    unsigned char *yb = reinterpret_cast<unsigned char *>(z ? a.y[1] : a.y[0]);
                    __stcs(reinterpret_cast<uint2 *>(yb + (t * ldy + hcol) * 16 + 8 * hh), y);
                  }
                }
            }
        }
        buf ^= 1;
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
    }
}

// ---------------------------------------------------------------- warp per row

// Warp-per-row kernel. A CTA holds two pools of warps: WQ warps that take Q
// rows and W - WQ warps that take K rows, so that each pool's ring stages have
// the size of its own rows and the pools can be sized in proportion to the
// bytes of Q and K. Each warp owns a ring of S row stages in shared memory and
// processes whole rows on its own: lane 0 issues the bulk copies of the
// warp's next rows, the warp walks the row's P shards in the order of the
// reduction (per group: lane chains, butterfly; groups in order; shards in
// order), forms the factor, and applies (x*gamma)*r re-reading the row from
// shared memory, with gamma read from shared memory (staged once per CTA) or
// through the L1 cache. No CTA-wide barrier is crossed per row, so warps never
// wait for one another and the per-row bookkeeping is amortised over the row.
struct RowsArgs {
    uint32_t stages;       // S, per warp
    uint32_t wq;           // warps of the Q pool (the others take K rows)
    uint32_t qstage;       // bytes of one Q row stage (multiple of 128)
    uint32_t kstage;       // bytes of one K row stage (multiple of 128)
    uint32_t gq_off;       // shared-memory offset of gamma_q (when staged)
    uint32_t gk_off;       // shared-memory offset of gamma_k (when staged)
    uint32_t qring_off;    // shared-memory offset of the Q pool's rings
    uint32_t kring_off;    // shared-memory offset of the K pool's rings
    uint32_t gamma_smem;   // 1: gamma staged in shared memory, 0: read through L1
    uint64_t timeout_ns;
};

template <class Tag>
__global__ void __launch_bounds__(512, 1) fused_rows(const FusedArgs a, const RowsArgs b) {
    constexpr int VEC = Tag::kVec;
    extern __shared__ __align__(128) unsigned char smem[];
    const int W = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = (int)b.stages;
    const int WQ = (int)b.wq;
    const int z = warp < WQ ? 0 : 1;                          // 0: Q pool, 1: K pool
    const int wz = z ? warp - WQ : warp;                      // index in the pool
    const int Wz = z ? W - WQ : WQ;                           // pool size
    const bool gsm = b.gamma_smem != 0;
    uint64_t *gbar = reinterpret_cast<uint64_t *>(smem);      // gamma barrier
    uint64_t *full = gbar + 1 + warp * S;                     // this warp's stage barriers
    const uint32_t stage_bytes = z ? b.kstage : b.qstage;
    unsigned char *ring = smem + (z ? b.kring_off : b.qring_off) + (size_t)wz * S * stage_bytes;
    const float *g = gsm ? reinterpret_cast<const float *>(smem + (z ? b.gk_off : b.gq_off)) : (z ? a.g[1] : a.g[0]);

    const int64_t T = a.T;
    const int64_t NW = (int64_t)gridDim.x * Wz;               // warps of this pool in the grid
    const int64_t gw = (int64_t)blockIdx.x * Wz + wz;
    const uint32_t nb = (uint32_t)(z ? a.D[1] : a.D[0]) * (uint32_t)Tag::kBytes;
    const char *xsrc = static_cast<const char *>((z ? a.x[1] : a.x[0]));
    const int64_t ldx_b = (z ? a.ldx[1] : a.ldx[0]) * 16;

    auto issue = [&](int s, int64_t t) {
        mbar_arrive_expect_tx(&full[s], nb);
        bulk_copy_g2s(ring + (size_t)s * stage_bytes, xsrc + t * ldx_b, nb, &full[s]);
    };

    if (threadIdx.x == 0) {
        mbar_init(gbar, 1);
        for (int i = 0; i < W * S; ++i) mbar_init(gbar + 1 + i, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Shared memory only so far; global reads start after the previous grid.
    pdl_wait();
    pdl_trigger();
    if (gsm && threadIdx.x == 0) {
        const uint32_t gqb = (uint32_t)a.D[0] * 4u, gkb = (uint32_t)a.D[1] * 4u;
        mbar_arrive_expect_tx(gbar, gqb + gkb);
        bulk_copy_g2s(smem + b.gq_off, a.g[0], gqb, gbar);
        bulk_copy_g2s(smem + b.gk_off, a.g[1], gkb, gbar);
    }
    if (lane == 0) {
        for (int s = 0; s < S; ++s) {
            const int64_t t = gw + (int64_t)s * NW;
            if (t < T) issue(s, t);
        }
    }
    // Leave after recording an error, once this warp's copies in flight have
    // landed (each wait bounded).
    auto fail = [&](int64_t n_first, int s0, uint32_t ph0) {
        if (lane == 0) {
            atomicOr(&g_device_errors, kErrWaitTimeout);
            int ds = s0;
            uint32_t dp = ph0;
            for (int64_t n = n_first; n < n_first + S && gw + n * NW < T; ++n) {
                if (!mbar_wait_bounded(&full[ds], dp, b.timeout_ns))
                    atomicOr(&g_device_errors, kErrDrainTimeout);
                if (++ds == S) {
                    ds = 0;
                    dp ^= 1u;
                }
            }
            if (gsm && warp == 0 && !mbar_wait_bounded(gbar, 0, b.timeout_ns))
                atomicOr(&g_device_errors, kErrDrainTimeout);
        }
    };
    if (gsm && !__all_sync(kFull, mbar_wait_bounded(gbar, 0, b.timeout_ns))) {
        fail(0, 0, 0);
        return;
    }

    const int P = a.P;
    const int K = (z ? a.K[1] : a.K[0]);
    const int nv = (z ? a.nv[1] : a.nv[0]);
    const int stride = kLanes * K;
    const float Df = (z ? a.Df[1] : a.Df[0]);
    const int rowvec = (z ? a.D[1] : a.D[0]) / VEC;
    const int64_t ldy = (z ? a.ldy[1] : a.ldy[0]);
    uint4 *ybase = reinterpret_cast<uint4 *>((z ? a.y[1] : a.y[0]));
    int s = 0;
    uint32_t phase = 0;
    for (int64_t n = 0;; ++n) {
        const int64_t t = gw + n * NW;
        if (t >= T) break;
        if (!__all_sync(kFull, mbar_wait_bounded(&full[s], phase, b.timeout_ns))) {
            fail(n, s, phase);
            return;
        }
        const uint4 *row = reinterpret_cast<const uint4 *>(ring + (size_t)s * stage_bytes);
        // Phase A and the ordered sums of Phase B.
        float Ssum = 0.f;
        if (K == 1) {
            // One group per shard. Four shards at a time: their lane chains
            // advance together (slot-major), then four independent
            // butterflies, then the ordered adds. Each shard's own order is
            // unchanged (0 + x is exact), so the bits equal the general order.
            const int cnt = slot_count(lane, nv, kLanes);
            for (int p0 = 0; p0 < P; p0 += 4) {
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                const uint4 *sh = row + (int64_t)p0 * nv + lane;
                for (int i = 0; i < cnt; ++i) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (p0 + q < P)
                            c[q] = __fadd_rn(c[q], vsumsq(Tag{}, sh[(int64_t)q * nv + i * kLanes]));
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) c[q] = butterfly(c[q]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (p0 + q < P) Ssum = __fadd_rn(Ssum, c[q]);
            }
        } else {
            for (int p = 0; p < P; ++p) {
                const uint4 *sh = row + (int64_t)p * nv;
                float Sp = 0.f;
                for (int kg = 0; kg < K; ++kg) {
                    float c = 0.f;
#pragma unroll 4
                    for (int v = kg * kLanes + lane; v < nv; v += stride)
                        c = __fadd_rn(c, vsumsq(Tag{}, sh[v]));
                    Sp = __fadd_rn(Sp, butterfly(c));
                }
                Ssum = __fadd_rn(Ssum, Sp);
            }
        }
        const float rr = factor(Ssum, Df, a.eps);
        // Phase B weight multiply and Phase C, element-wise over the row.
        uint4 *dst = ybase + t * ldy;
        if (gsm) {
#pragma unroll 4
            for (int v = lane; v < rowvec; v += kLanes)
                st_stream(dst + v, vapply_ptr(Tag{}, row[v], g + (int64_t)v * VEC, rr));
        } else {
#pragma unroll 4
            for (int v = lane; v < rowvec; v += kLanes)
                st_stream(dst + v, vapply(Tag{}, row[v], g + (int64_t)v * VEC, rr));
        }
        __syncwarp();
        // Every lane is done with this stage: refill it with the warp's row S ahead.
        if (lane == 0) {
            const int64_t tn = gw + (n + S) * NW;
            if (tn < T) {
                fence_proxy_async_smem();
                issue(s, tn);
            }
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
    }
}

// ---------------------------------------------------------------- shard pairs

// The token ring for GQA-like shapes (P even, K shards of at most 16 vectors):
// a CTA of P warps per token instead of 2P. Warp w < P/2 takes Q shards 2w and
// 2w + 1 (two independent lane chains and butterflies, each shard's order
// unchanged); warp P/2 + w takes K shards 2w and 2w + 1 on its lane halves
// (lanes 0-15 and 16-31, one vector per lane) and reduces each half with a
// 16-lane butterfly. That equals the 32-lane butterfly bit for bit: the xor-16
// step it skips adds the exact zeros of the lanes past a shard's 16 vectors.
// With half the warps per token, two CTAs fit an SM and each warp carries
// twice the work per token barrier. One token per stage.
//
// KW: K shards as wide as Q's (more than 16 vectors) are taken like Q's,
// warp P/2 + w holding K shards 2w and 2w + 1 with its own two chains and
// butterflies. This halves the warps per token of the ring for equal-width
// tensors, which pays where a warp's fixed work per token (wait, butterfly,
// barrier, factor) weighs most: one or two vectors per lane, FP8.
// CP, CNQ, CNK: shard count and vectors per Q / K shard fixed at compile
// time for the shape that has its own instance (0: from the arguments);
// every slot count, offset and the combine then fold to constants, and a
// power-of-two width forms the factor by a multiply (same bits).
template <class Tag, int VQ, bool GREG, bool KW, int CP = 0, int CNQ = 0, int CNK = 0>
__global__ void __launch_bounds__(512, 1) fused_pair(const FusedArgs a, const BulkArgs b) {
    constexpr int VEC = Tag::kVec;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    float(*red)[64] = reinterpret_cast<float(*)[64]>(smem + kBarBytes);   // [buf][Q: 0..31, K: 32..63]
    unsigned char *stages = smem + kStageBase;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int P = CP ? CP : a.P;
    const int half = P >> 1;
    const int z = warp < half ? 0 : 1;
    const int w = z ? warp - half : warp;
    const int pa = 2 * w;                                // first shard of the pair
    const int nvq = CNQ ? CNQ : a.nv[0], nvk = CNK ? CNK : a.nv[1];
    // Shard pairs (Q warps; K warps too with KW): this lane's vectors of
    // shards pa, pa + 1 of tensor z: lane + 32 i, i < cnt.
    const bool pairs = KW || z == 0;
    const int nvz = z ? nvk : nvq;
    const int cnt = pairs ? slot_count(lane, nvz, kLanes) : 0;
    // K: lane half h takes shard pa + h, vector kv of it.
    const int hk = lane >> 4, kv = lane & 15;
    const bool kok = !pairs && kv < nvk;
    const int kshard = pa + hk;
    const float Df = z ? a.Df[1] : a.Df[0];
    const float eps = a.eps;
    const uint32_t tok_bytes = b.qbytes + b.kbytes;
    // Offsets inside a stage (bytes): Q vector (p, v) at (p*nvq + v)*16; K at
    // qbytes + (p*nvk + v)*16.
    const uint32_t qoff = (z ? b.qbytes : 0u) + (uint32_t)((pa * nvz + lane) * 16);
    const float *gz = z ? a.g[1] : a.g[0];
    const uint32_t koff = b.qbytes + (uint32_t)((kshard * nvk + kv) * 16);

    const int64_t T = a.T;
    const int64_t G = gridDim.x;
    const int S = (int)b.stages;
    const char *qsrc = static_cast<const char *>(a.x[0]);
    const char *ksrc = static_cast<const char *>(a.x[1]);
    const int64_t ldq_b = a.ldx[0] * 16, ldk_b = a.ldx[1] * 16;

    auto issue = [&](int s, int64_t n) {
        unsigned char *st = stages + (size_t)s * b.stage_stride;
        const int64_t tt = blockIdx.x + n * G;
        mbar_arrive_expect_tx(&full[s], tok_bytes);
        bulk_copy_g2s(st, qsrc + tt * ldq_b, b.qbytes, &full[s]);
        bulk_copy_g2s(st + b.qbytes, ksrc + tt * ldk_b, b.kbytes, &full[s]);
    };

    const int64_t npass = (T - blockIdx.x + G - 1) / G;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    if (tid == 0) {
        for (int s = 0; s < S && s < npass; ++s) issue(s, s);
    }

    // Gamma in registers: shard-pair lanes 2 x VQ vectors, K half lanes one vector.
    float gam[GREG ? 2 * VQ * VEC : 1];
    if (GREG) {
        if (pairs) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < VQ; ++i)
                    if (i < cnt)
#pragma unroll
                        for (int e = 0; e < VEC; e += 4) {
                            const float4 g4 = __ldg(reinterpret_cast<const float4 *>(
                                gz + ((int64_t)(pa + h) * nvz + lane + 32 * i) * VEC + e));
                            float *d = &gam[(h * VQ + i) * VEC + e];
                            d[0] = g4.x;
                            d[1] = g4.y;
                            d[2] = g4.z;
                            d[3] = g4.w;
                        }
        } else if (kok) {
#pragma unroll
            for (int e = 0; e < VEC; e += 4) {
                const float4 g4 = __ldg(reinterpret_cast<const float4 *>(
                    a.g[1] + ((int64_t)kshard * nvk + kv) * VEC + e));
                gam[e] = g4.x;
                gam[e + 1] = g4.y;
                gam[e + 2] = g4.z;
                gam[e + 3] = g4.w;
            }
        }
    }

    int s = 0;
    uint32_t phase = 0;
    int buf = 0;
    for (int64_t n = 0; n < npass; ++n) {
        const int64_t t = blockIdx.x + n * G;
        const bool ok = mbar_wait_bounded(&full[s], phase, b.timeout_ns);
        const unsigned char *st = stages + (size_t)s * b.stage_stride;
        uint4 cur[2][VQ];
        float c0 = 0.f, c1 = 0.f;
        if (pairs) {
            const uint4 *src0 = reinterpret_cast<const uint4 *>(st + qoff);
            const uint4 *src1 = src0 + nvz;
#pragma unroll
            for (int i = 0; i < VQ; ++i) {
                cur[0][i] = i < cnt ? src0[32 * i] : make_uint4(0, 0, 0, 0);
                cur[1][i] = i < cnt ? src1[32 * i] : make_uint4(0, 0, 0, 0);
            }
            // Missing vectors are a lane's last slots and add +0 (no change).
#pragma unroll
            for (int i = 0; i < VQ; ++i) {
                c0 = __fadd_rn(c0, vsumsq(Tag{}, cur[0][i]));
                c1 = __fadd_rn(c1, vsumsq(Tag{}, cur[1][i]));
            }
            c0 = butterfly(c0);
            c1 = butterfly(c1);
            if (lane == 0) {
                red[buf][32 * z + pa] = c0;
                red[buf][32 * z + pa + 1] = c1;
            }
        } else {
            cur[0][0] = kok ? *reinterpret_cast<const uint4 *>(st + koff) : make_uint4(0, 0, 0, 0);
            // One vector per lane: the lane chain is its vector's sum (0 + s).
            c0 = vsumsq(Tag{}, cur[0][0]);
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) c0 = __fadd_rn(c0, __shfl_xor_sync(kFull, c0, off));
            if (kv == 0) red[buf][32 + kshard] = c0;
        }
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_device_errors, kErrWaitTimeout);
                int ds = s;
                uint32_t dp = phase;
                for (int64_t m = n; m < npass && m < n + S; ++m) {
                    if (!mbar_wait_bounded(&full[ds], dp, b.timeout_ns))
                        atomicOr(&g_device_errors, kErrDrainTimeout);
                    if (++ds == S) {
                        ds = 0;
                        dp ^= 1u;
                    }
                }
            }
            return;
        }
        if (tid == 0 && n + S < npass) {
            fence_proxy_async_smem();
            issue(s, n + S);
        }
        const float Sz = combine_fast(&red[buf][z ? 32 : 0], P, 1);
        const float r = z ? factor_w<CP * CNK * VEC>(Sz, Df, eps) : factor_w<CP * CNQ * VEC>(Sz, Df, eps);
        if (pairs) {
            uint4 *dst = reinterpret_cast<uint4 *>(z ? a.y[1] : a.y[0]) + t * (z ? a.ldy[1] : a.ldy[0]) +
                         (int64_t)pa * nvz + lane;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < VQ; ++i)
                    if (i < cnt) {
                        const int64_t col = (int64_t)h * nvz + 32 * i;
                        uint4 y;
                        if (GREG)
                            y = vapply_regs(Tag{}, cur[h][i], &gam[(h * VQ + i) * VEC], r);
                        else
                            y = vapply(Tag{}, cur[h][i], gz + ((int64_t)pa * nvz + lane + col) * VEC, r);
                        st_stream(dst + col, y);
                    }
        } else if (kok) {
            uint4 *dst = reinterpret_cast<uint4 *>(a.y[1]) + t * a.ldy[1] + (int64_t)kshard * nvk + kv;
            uint4 y;
            if (GREG)
                y = vapply_regs(Tag{}, cur[0][0], gam, r);
            else
                y = vapply(Tag{}, cur[0][0], a.g[1] + ((int64_t)kshard * nvk + kv) * VEC, r);
            st_stream(dst, y);
        }
        buf ^= 1;
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
    }
}

// A kernel that waits on an mbarrier nobody arrives on, with the same bounded
// wait as fused_bulk: it must time out, record kErrWaitTimeout and return.
__global__ void bounded_wait_probe(uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait_bounded(&bar, 0, timeout_ns);
    if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicOr(&g_device_errors, kErrWaitTimeout);
}

// ---------------------------------------------------------------- instances and launch

// Combinations that exist: TB (1 or 2) tokens x VMAX vectors per lane <= 12;
// for FP8 (16 values per vector) TB x VMAX <= 4, two tokens only with gamma
// read per use, gamma in registers only up to 3 vectors, so that no instance
// spills.
constexpr bool bulk_exists(int vmax, int tb, int vec, bool greg) {
    return vmax >= 1 && vmax <= kVcap && (tb == 1 || tb == 2) && vmax * tb <= 12 &&
           (vec != 16 || (vmax * tb <= 4 && (tb == 1 || !greg) && (!greg || vmax <= 3)));
}
// The half-slot mode exists for FP8 with one token per stage.
constexpr bool bulk_mode_exists(int vmax, int tb, int vec, bool greg, int mode) {
    return bulk_exists(vmax, tb, vec, greg) && mode >= 0 && mode <= 2 &&
           (mode != 2 || (vec == 16 && tb == 1));
}
constexpr int bulk_max_threads(int vmax, int tb, int vec) {
    return (vmax * tb <= 2 && vmax * tb * vec <= 16) ? 1024 : 512;
}

template <class Tag, bool GREG, int V, int TB, int MODE>
const void *bulk_fn() {
    if constexpr (bulk_mode_exists(V, TB, Tag::kVec, GREG, MODE))
        return reinterpret_cast<const void *>(
            &fused_bulk<Tag, V, GREG, TB, MODE, bulk_max_threads(V, TB, Tag::kVec)>);
    else
        return nullptr;
}

template <class Tag, bool GREG, int TB, int MODE>
const void *bulk_table_tb(int vmax) {
    switch (vmax) {
    case 1: return bulk_fn<Tag, GREG, 1, TB, MODE>();
    case 2: return bulk_fn<Tag, GREG, 2, TB, MODE>();
    case 3: return bulk_fn<Tag, GREG, 3, TB, MODE>();
    case 4: return bulk_fn<Tag, GREG, 4, TB, MODE>();
    case 5: return bulk_fn<Tag, GREG, 5, TB, MODE>();
    case 6: return bulk_fn<Tag, GREG, 6, TB, MODE>();
    case 7: return bulk_fn<Tag, GREG, 7, TB, MODE>();
    case 8: return bulk_fn<Tag, GREG, 8, TB, MODE>();
    default: return nullptr;
    }
}

template <class Tag, bool GREG, int TB>
const void *bulk_table_mode(int vmax, int mode) {
    switch (mode) {
    case 0: return bulk_table_tb<Tag, GREG, TB, 0>(vmax);
    case 1: return bulk_table_tb<Tag, GREG, TB, 1>(vmax);
    case 2: return bulk_table_tb<Tag, GREG, TB, 2>(vmax);
    default: return nullptr;
    }
}

template <class Tag, bool GREG>
const void *bulk_table(int vmax, int tb, int mode) {
    if (tb == 1) return bulk_table_mode<Tag, GREG, 1>(vmax, mode);
    if (tb == 2) return bulk_table_mode<Tag, GREG, 2>(vmax, mode);
    return nullptr;
}

const void *fused_bulk_kernel(int dtype, int vmax, bool gamma_regs, int tb, int mode,
                              int *max_threads) {
    const int vec = dtype == 1 ? 8 : (dtype == 2 ? 16 : 4);
    if (!bulk_exists(vmax, tb, vec, gamma_regs) || mode < 0 || mode > 2 ||
        (mode == 2 && (vec != 16 || tb != 1)))
        return nullptr;
    if (max_threads) *max_threads = bulk_max_threads(vmax, tb, vec);
    if (dtype == 0)
        return gamma_regs ? bulk_table<F32Tag, true>(vmax, tb, mode) : bulk_table<F32Tag, false>(vmax, tb, mode);
    if (dtype == 1)
        return gamma_regs ? bulk_table<BF16Tag, true>(vmax, tb, mode) : bulk_table<BF16Tag, false>(vmax, tb, mode);
    if (dtype == 2)
        return gamma_regs ? bulk_table<E4M3Tag, true>(vmax, tb, mode) : bulk_table<E4M3Tag, false>(vmax, tb, mode);
    return nullptr;
}

uint32_t bulk_stage_stride(int64_t qbytes, int64_t kbytes, int tb) {
    return (uint32_t)((tb * (qbytes + kbytes) + 127) / 128 * 128);
}

size_t bulk_smem_bytes(int stages, uint32_t stage_stride) {
    return (size_t)kStageBase + (size_t)stages * stage_stride;
}

int bulk_max_stages() { return (int)kMaxStages; }

cudaError_t launch_fused_bulk(int dtype, int vmax, bool gamma_regs, int tb, int mode,
                              const FusedArgs &a, int stages, int block, int64_t grid,
                              uint64_t timeout_ns, cudaStream_t s) {
    const void *fn = fused_bulk_kernel(dtype, vmax, gamma_regs, tb, mode, nullptr);
    if (!fn || stages < 1 || stages > (int)kMaxStages) return cudaErrorInvalidValue;
    const int64_t es = dtype == 1 ? 2 : (dtype == 2 ? 1 : 4);
    BulkArgs b;
    b.stages = (uint32_t)stages;
    b.qbytes = (uint32_t)(a.D[0] * es);
    b.kbytes = (uint32_t)(a.D[1] * es);
    b.stage_stride = bulk_stage_stride(b.qbytes, b.kbytes, tb);
    b.timeout_ns = timeout_ns;
    const size_t smem = bulk_smem_bytes(stages, b.stage_stride);
    void *args[] = {const_cast<FusedArgs *>(&a), &b};
    return launch(fn, dim3((unsigned)grid), dim3(block), smem, s, args);
}

const void *fused_rows_kernel(int dtype) {
    if (dtype == 0) return reinterpret_cast<const void *>(&fused_rows<F32Tag>);
    if (dtype == 1) return reinterpret_cast<const void *>(&fused_rows<BF16Tag>);
    if (dtype == 2) return reinterpret_cast<const void *>(&fused_rows<E4M3Tag>);
    return nullptr;
}

// Shared-memory layout of fused_rows: [gamma barrier + W*S stage barriers,
// padded to 128][gamma_q][gamma_k (both only when staged)][WQ Q rings of S
// stages][WK K rings of S stages].
RowsLayout rows_layout(int64_t Dq, int64_t Dk, int es, int wq, int wk, int stages, bool gamma_smem) {
    RowsLayout L;
    auto up = [](int64_t x) { return (x + 127) / 128 * 128; };
    L.qstage = (uint32_t)up(Dq * es);
    L.kstage = (uint32_t)up(Dk * es);
    L.gq_off = (uint32_t)up(8 * (1 + (int64_t)(wq + wk) * stages));
    L.gk_off = L.gq_off + (gamma_smem ? (uint32_t)up(Dq * 4) : 0u);
    L.qring_off = L.gk_off + (gamma_smem ? (uint32_t)up(Dk * 4) : 0u);
    L.kring_off = L.qring_off + (uint32_t)((int64_t)wq * stages * L.qstage);
    L.smem_bytes = (size_t)L.kring_off + (size_t)wk * stages * L.kstage;
    return L;
}

cudaError_t launch_fused_rows(int dtype, const FusedArgs &a, int wq, int wk, int stages,
                              bool gamma_smem, int64_t grid, uint64_t timeout_ns, cudaStream_t s) {
    const void *fn = fused_rows_kernel(dtype);
    if (!fn || wq < 1 || wk < 1 || wq + wk > 16 || stages < 1) return cudaErrorInvalidValue;
    const RowsLayout L = rows_layout(a.D[0], a.D[1], dtype == 1 ? 2 : (dtype == 2 ? 1 : 4), wq, wk,
                                     stages, gamma_smem);
    RowsArgs b;
    b.stages = (uint32_t)stages;
    b.wq = (uint32_t)wq;
    b.qstage = L.qstage;
    b.kstage = L.kstage;
    b.gq_off = L.gq_off;
    b.gk_off = L.gk_off;
    b.qring_off = L.qring_off;
    b.kring_off = L.kring_off;
    b.gamma_smem = gamma_smem ? 1u : 0u;
    b.timeout_ns = timeout_ns;
    void *args[] = {const_cast<FusedArgs *>(&a), &b};
    return launch(fn, dim3((unsigned)grid), dim3(32 * (wq + wk)), L.smem_bytes, s, args);
}

// fused_pair instances: VQ 1..3 vectors per lane per shard, gamma in
// registers or not, K shards on lane halves or in pairs (kw).
template <class Tag, bool KW>
const void *pair_fn(int vq, bool greg) {
    switch (vq) {
    case 1: return greg ? reinterpret_cast<const void *>(&fused_pair<Tag, 1, true, KW>)
                        : reinterpret_cast<const void *>(&fused_pair<Tag, 1, false, KW>);
    case 2: return greg ? reinterpret_cast<const void *>(&fused_pair<Tag, 2, true, KW>)
                        : reinterpret_cast<const void *>(&fused_pair<Tag, 2, false, KW>);
    case 3: return greg ? reinterpret_cast<const void *>(&fused_pair<Tag, 3, true, KW>)
                        : reinterpret_cast<const void *>(&fused_pair<Tag, 3, false, KW>);
    default: return nullptr;
    }
}

template <class Tag>
const void *pair_table(int vq, bool greg, bool kw) {
    return kw ? pair_fn<Tag, true>(vq, greg) : pair_fn<Tag, false>(vq, greg);
}

const void *fused_pair_kernel(int dtype, int vq, bool gamma_regs, bool kw) {
    if (dtype == 0) return pair_table<F32Tag>(vq, gamma_regs, kw);
    if (dtype == 1) return pair_table<BF16Tag>(vq, gamma_regs, kw);
    // FP8 with gamma in registers for 3 vectors per lane (2 with K in pairs too)
    // would spill: no instance.
    if (dtype == 2)
        return (gamma_regs && vq >= (kw ? 2 : 3)) ? nullptr : pair_table<E4M3Tag>(vq, gamma_regs, kw);
    return nullptr;
}

// The instance compiled for this exact shape where one exists (FP8, one
// vector per lane, K in pairs, 8 shards of 32 vectors: e.g. D = 4096, P = 8),
// else the general one.
const void *fused_pair_kernel_for(int dtype, int vq, bool gamma_regs, bool kw, int P, int nvq, int nvk) {
    const void *gen = fused_pair_kernel(dtype, vq, gamma_regs, kw);
    if (gen && dtype == 2 && vq == 1 && gamma_regs && kw && P == 8 && nvq == 32 && nvk == 32)
        return reinterpret_cast<const void *>(&fused_pair<E4M3Tag, 1, true, true, 8, 32, 32>);
    return gen;
}

cudaError_t launch_fused_pair(int dtype, int vq, bool gamma_regs, bool kw, const FusedArgs &a,
                              int stages, int64_t grid, uint64_t timeout_ns, cudaStream_t s) {
    const void *fn = fused_pair_kernel_for(dtype, vq, gamma_regs, kw, a.P, a.nv[0], a.nv[1]);
    if (!fn || stages < 1 || stages > (int)kMaxStages || (a.P & 1) || a.P > 16) return cudaErrorInvalidValue;
    // Each lane's slots must cover its shards: lane halves take at most 16 K vectors.
    if (a.K[0] != 1 || a.K[1] != 1 || a.nv[0] > kLanes * vq || a.nv[1] > (kw ? kLanes * vq : kLanes / 2))
        return cudaErrorInvalidValue;
    const int64_t es = dtype == 1 ? 2 : (dtype == 2 ? 1 : 4);
    BulkArgs b;
    b.stages = (uint32_t)stages;
    b.qbytes = (uint32_t)(a.D[0] * es);
    b.kbytes = (uint32_t)(a.D[1] * es);
    b.stage_stride = bulk_stage_stride(b.qbytes, b.kbytes, 1);
    b.timeout_ns = timeout_ns;
    const size_t smem = bulk_smem_bytes(stages, b.stage_stride);
    void *args[] = {const_cast<FusedArgs *>(&a), &b};
    return launch(fn, dim3((unsigned)grid), dim3(32 * a.P), smem, s, args);
}

cudaError_t launch_bounded_wait_probe(uint64_t timeout_ns, cudaStream_t s) {
    void *args[] = {&timeout_ns};
    return cudaLaunchKernel(reinterpret_cast<const void *>(&bounded_wait_probe), dim3(1), dim3(64),
                            args, 0, s);
}

cudaError_t read_device_errors(unsigned *out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_errors, sizeof(unsigned));
    if (e != cudaSuccess || !clear) return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(g_device_errors, &zero, sizeof(unsigned));
}

}  // namespace qkn
