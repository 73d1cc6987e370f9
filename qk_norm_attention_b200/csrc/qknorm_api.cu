// qknorm_api.cu -- the C ABI of libqknorm.so (declared in include/qknorm.h):
// argument checks, the launch selector and the launches.
//
// The selector follows the SwiftQK review's launch rule for its persistent
// kernel (Section 3, "Why deadlock-safety needs its own argument", and
// Section 5b): the grid is at most B_res x N_SM CTAs, B_res from the CUDA
// occupancy calculator, with a stride loop over tokens. On one GPU nothing
// waits on another CTA, so the bound is kept for its performance effect
// (every CTA resident, tokens spread evenly) rather than for deadlock safety.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/qknorm.h"
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

bool g_pdl = true;  // programmatic dependent launch (qknorm_set_pdl)
bool pdl_enabled() { return g_pdl; }

TensorShape make_shape(int32_t D, int32_t P, int vec) {
    TensorShape s;
    s.D = D;
    s.nv = (D / P) / vec;
    const int per_group = kLanes * kVcap;
    s.K = (s.nv + per_group - 1) / per_group;
    if (s.K < 1) s.K = 1;
    const int lanes_total = kLanes * s.K;
    s.vmax = (s.nv + lanes_total - 1) / lanes_total;
    return s;
}

namespace {

thread_local char g_last_error[256] = "";

int32_t g_forced_variant = QKNORM_VARIANT_AUTO;
int64_t g_forced_grid = 0;

void set_error(cudaError_t e) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
}

int vec_of(int32_t dtype) { return dtype == QKNORM_BF16 ? 8 : (dtype == QKNORM_E4M3 ? 16 : 4); }
int64_t elem_of(int32_t dtype) { return dtype == QKNORM_BF16 ? 2 : (dtype == QKNORM_E4M3 ? 1 : 4); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};
Range rng(const void *p, int64_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + (uintptr_t)bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }
// An output may coincide exactly with its own input; any other overlap is an error.
bool bad_alias(Range out, Range in, bool may_alias) {
    if (!overlap(out, in)) return false;
    return !(may_alias && out.lo == in.lo && out.hi == in.hi);
}

// A strided tensor: T rows of `row` bytes whose starts are `ld` bytes apart.
struct Strided {
    uintptr_t base;
    int64_t row, ld, T;
};
Strided strided(const void *p, int64_t row, int64_t ld, int64_t T) {
    return Strided{reinterpret_cast<uintptr_t>(p), row, ld, T};
}
// True if any byte of a may be a byte of b. Tensors with the same row period
// interleave without touching when their row segments are disjoint modulo
// the period (e.g. the Q, K and V slices of one fused QKV buffer); otherwise
// the test falls back to the spans.
bool strided_overlap(const Strided &a, const Strided &b) {
    if (a.T <= 0 || b.T <= 0) return false;
    const Range ra{a.base, a.base + (uintptr_t)((a.T - 1) * a.ld + a.row)};
    const Range rb{b.base, b.base + (uintptr_t)((b.T - 1) * b.ld + b.row)};
    if (!overlap(ra, rb)) return false;
    if (a.ld == b.ld && a.ld > 0) {
        const int64_t d = (int64_t)(b.base - a.base);
        const int64_t r = ((d % a.ld) + a.ld) % a.ld;  // b's row start within a's period
        if (r >= a.row && r + b.row <= a.ld) return false;
    }
    return true;
}
// An output may be exactly its own input (same base, row and stride).
bool strided_bad_alias(const Strided &out, const Strided &in, bool may_alias) {
    if (may_alias && out.base == in.base && out.row == in.row && out.ld == in.ld) return false;
    return strided_overlap(out, in);
}

// Checks common to every entry point for one [T, D] tensor with P shards.
int check_shape(int64_t T, int32_t D, int32_t P, int32_t dtype) {
    if (T < 0 || D <= 0 || P <= 0) return QKNORM_ERR_INVALID_ARG;
    if (D % P != 0) return QKNORM_ERR_INVALID_ARG;
    if (dtype != QKNORM_F32 && dtype != QKNORM_BF16 && dtype != QKNORM_E4M3) return QKNORM_ERR_UNSUPPORTED;
    if ((D / P) % vec_of(dtype) != 0) return QKNORM_ERR_UNSUPPORTED;
    if (T > 0 && T > INT64_MAX / ((int64_t)D * elem_of(dtype))) return QKNORM_ERR_INVALID_ARG;
    return QKNORM_OK;
}

int check_eps(float eps) {
    return (std::isfinite(eps) && eps >= 0.f) ? QKNORM_OK : QKNORM_ERR_INVALID_ARG;
}

// ---------------------------------------------------------------- device caches

constexpr int kMaxDevices = 64;
int g_num_sms[kMaxDevices];

struct OccEntry {
    int device;
    const void *fn;
    int block;
    size_t smem;
    int blocks;
};
constexpr int kOccSlots = 256;
OccEntry g_occ[kOccSlots];
int g_occ_n = 0;
std::mutex g_occ_mu;

cudaError_t device_sms(int *dev, int *sms) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (*dev < 0 || *dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (g_num_sms[*dev] == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, *dev);
        if (e != cudaSuccess) return e;
        g_num_sms[*dev] = n;
    }
    *sms = g_num_sms[*dev];
    return cudaSuccess;
}

cudaError_t resident_blocks(int dev, const void *fn, int block, size_t smem, int *out) {
    std::lock_guard<std::mutex> lock(g_occ_mu);
    for (int i = 0; i < g_occ_n; ++i) {
        const OccEntry &o = g_occ[i];
        if (o.device == dev && o.fn == fn && o.block == block && o.smem == smem) {
            *out = o.blocks;
            return cudaSuccess;
        }
    }
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, block, smem);
    if (e != cudaSuccess) return e;
    if (n < 1) n = 1;
    if (g_occ_n < kOccSlots) g_occ[g_occ_n++] = OccEntry{dev, fn, block, smem, n};
    *out = n;
    return cudaSuccess;
}

// ---------------------------------------------------------------- the selector

int32_t g_tune_stages = 0;           // bulk stages per CTA; 0 = automatic
int32_t g_tune_tb = 0;               // tokens per bulk stage; 0 = automatic
int32_t g_tune_gamma_regs = -1;      // -1 = automatic
uint64_t g_wait_limit_ns = 2000000000ull;
int32_t g_rows_wq = 0;               // Q-pool warps per CTA of the rows variant; 0 = automatic
int32_t g_rows_wk = 0;               // K-pool warps per CTA; 0 = automatic
int32_t g_rows_stages = 0;           // row stages per warp; 0 = automatic
int32_t g_rows_gsm = -1;             // gamma staged in shared memory: -1 automatic, 0, 1
constexpr int kRowsStagesAuto = 2;
constexpr int kRowsMaxWarps = 16;

constexpr int kSmemPerSm = 228 * 1024;      // shared memory of one SM
constexpr int kSmemPerCta = 227 * 1024;     // largest opt-in dynamic shared memory of a CTA
constexpr int kSmemReservedPerCta = 1024;   // the runtime's per-CTA reservation
constexpr int kRegsPerSm = 65536;
constexpr int kThreadsPerSm = 2048;
constexpr int kMaxStagesAuto = 2;   // measured best on B200 (2 CTAs x 2 stages per SM)
constexpr int kRegsHint = 64;               // register estimate when no device is queried

struct Shapes {
    TensorShape q, k;
    int64_t ntask;
    int vmax;
};

Shapes shapes_of(int32_t Dq, int32_t Dk, int32_t P, int32_t dtype) {
    Shapes s;
    s.q = make_shape(Dq, P, vec_of(dtype));
    s.k = make_shape(Dk, P, vec_of(dtype));
    s.ntask = (int64_t)P * (s.q.K + s.k.K);
    s.vmax = s.q.vmax > s.k.vmax ? s.q.vmax : s.k.vmax;
    return s;
}

// True when every lane of every (shard, group) task of both tensors holds
// exactly vmax vectors, so the kernels need no per-lane guards.
bool full_lanes(const Shapes &sh) {
    auto full = [&](const TensorShape &t) {
        return t.nv % (kLanes * t.K) == 0 && t.nv / (kLanes * t.K) == sh.vmax;
    };
    return full(sh.q) && full(sh.k);
}

// How the bulk kernel's lanes hold vectors: 1 full (as above); 2 when the
// dtype is FP8 and each tensor's shards are one group whose last slot holds
// at most 16 vectors (split in halves over the 32 lanes); else 0.
int lane_mode(const Shapes &sh, int32_t dtype) {
    if (full_lanes(sh)) return 1;
    auto half = [&](const TensorShape &t) {
        const int r = t.nv - kLanes * (sh.vmax - 1);
        return t.K == 1 && r > 0 && r <= kLanes / 2;
    };
    return (dtype == QKNORM_E4M3 && half(sh.q) && half(sh.k)) ? 2 : 0;
}

// Gamma in registers pays off while a lane holds few vectors (measured on
// B200: +5 % at 2 vectors per lane, -7 % at 5, where the registers cost
// occupancy and gamma hits L1 anyway).
bool gamma_regs_for(int32_t dtype, int vmax) {
    if (g_tune_gamma_regs >= 0) return g_tune_gamma_regs != 0;
    // FP8 pays four 16-byte gamma loads per vector otherwise (measured: +80 %
    // at 2 vectors per lane), so it keeps gamma in registers while it can.
    if (dtype == QKNORM_E4M3) return vmax <= 3;
    return vmax * vec_of(dtype) <= 24;
}

// Tokens per bulk stage: one (two tokens per stage measured within noise of
// one and less steady across boxes).
int tokens_per_stage_for(int vmax) {
    (void)vmax;
    return g_tune_tb > 0 ? g_tune_tb : 1;
}

// Stage count of the bulk kernel: the most stages (up to kMaxStagesAuto) that
// fit when as many CTAs share an SM as threads and registers allow; fewer
// CTAs per SM if that leaves less than two stages each.
void bulk_stages(uint32_t stride, int block, int regs, qknorm_plan *pl) {
    int ctas = kThreadsPerSm / block;
    const int by_regs = kRegsPerSm / (regs * block);
    if (by_regs < ctas) ctas = by_regs;
    if (ctas < 1) ctas = 1;
    int S = 0;
    for (; ctas >= 1; --ctas) {
        const int per_cta = kSmemPerSm / ctas - kSmemReservedPerCta;
        const int cap = per_cta < kSmemPerCta ? per_cta : kSmemPerCta;
        S = 0;
        while (S < kMaxStagesAuto && (int64_t)bulk_smem_bytes(S + 1, stride) <= cap) ++S;
        if (S >= 2) break;
    }
    if (g_tune_stages > 0) S = g_tune_stages;
    pl->stages = S;
    pl->smem_bytes = (int64_t)bulk_smem_bytes(S, stride);
}

// Warps of the rows variant. A Q warp moves Dq/wq of a CTA's row bytes per
// round and a K warp Dk/wk; the CTA moves (Dq + Dk) per round in the time of
// the busier pool, so it works like (Dq + Dk) / max(Dq/wq, Dk/wk) fully busy
// warps. Among the CTA shapes (wq + wk <= kRowsMaxWarps, wq, wk >= 1) and
// CTAs per SM (1 to 8) that threads, registers and shared memory allow, take
// the most such warps per SM; ties go to fewer warps per CTA.
struct RowsChoice {
    int wq = 0, wk = 0;
    bool gsm = false;
};

bool rows_fits(int32_t Dq, int32_t Dk, int32_t dtype, int wq, int wk, int S, bool gsm, int ctas) {
    const size_t sm = rows_layout(Dq, Dk, (int)elem_of(dtype), wq, wk, S, gsm).smem_bytes;
    return sm <= (size_t)kSmemPerCta && (int64_t)ctas * (sm + kSmemReservedPerCta) <= kSmemPerSm;
}

RowsChoice rows_auto(int32_t Dq, int32_t Dk, int32_t dtype, int S, int gsm_pref, int regs) {
    RowsChoice best;
    double best_score = 0.0;
    const int warp_regs = (regs + 7) / 8 * 8 * kLanes;   // registers are granted 8 per thread at a time
    for (int g = 0; g <= 1; ++g) {
        if (gsm_pref >= 0 && g != gsm_pref) continue;
        for (int W = 2; W <= kRowsMaxWarps; ++W) {
            for (int wq = 1; wq < W; ++wq) {
                const int wk = W - wq;
                const double busy = (double)(Dq + Dk) /
                                    ((double)Dq / wq > (double)Dk / wk ? (double)Dq / wq : (double)Dk / wk);
                for (int ctas = 8; ctas >= 1; --ctas) {
                    if (ctas * W * kLanes > kThreadsPerSm || ctas * W * warp_regs > kRegsPerSm) continue;
                    if (!rows_fits(Dq, Dk, dtype, wq, wk, S, g != 0, ctas)) continue;
                    if (ctas * busy > best_score + 1e-9) {
                        best_score = ctas * busy;
                        best.wq = wq;
                        best.wk = wk;
                        best.gsm = g != 0;
                    }
                    break;
                }
            }
        }
    }
    return best;
}

bool rows_fit(int32_t Dq, int32_t Dk, int32_t dtype) {
    return rows_fits(Dq, Dk, dtype, 1, 1, 1, false, 1);
}

// The shard-pair ring's conditions: P even and at most 16 (P warps), one
// group per shard, shards of at most 3 vectors per lane, and an instance for
// the gamma placement. K shards of at most 16 vectors share a warp's lane
// halves; wider K shards go in pairs like Q's (pair_kw).
bool pair_kw(const Shapes &sh) { return sh.k.nv > kLanes / 2; }

int pair_vq(const Shapes &sh) { return pair_kw(sh) ? sh.vmax : sh.q.vmax; }

bool pair_greg(const Shapes &sh, int32_t dtype) {
    if (g_tune_gamma_regs >= 0) return g_tune_gamma_regs != 0;
    return !(dtype == QKNORM_E4M3 && pair_vq(sh) >= (pair_kw(sh) ? 2 : 3));
}

bool pair_fits(const Shapes &sh, int32_t P, int32_t dtype) {
    return !(P & 1) && P <= 16 && sh.q.K == 1 && sh.k.K == 1 && pair_vq(sh) <= 3 &&
           fused_pair_kernel(dtype, pair_vq(sh), pair_greg(sh, dtype), pair_kw(sh)) != nullptr;
}

// The CTA kernel keeps a lane's gamma in registers, loaded together with the
// row, while it is at most 32 floats (one token per CTA: no prefetch).
bool cta_greg(const Shapes &sh, int32_t dtype, bool full) {
    if (g_tune_gamma_regs == 0) return false;
    return fused_cta_kernel(dtype, sh.vmax, false, full, true, nullptr) != nullptr;
}

// The register-resident warp-per-token kernel: one lane group per shard and
// an instance for (P, Q vectors per lane, K vectors per lane).
bool warp_regs_fit(const Shapes &sh, int32_t P, int32_t dtype) {
    return sh.q.K == 1 && sh.k.K == 1 &&
           fused_warp_kernel(dtype, P, sh.q.vmax, sh.k.vmax) != nullptr;
}

// The shard-pair ring with staged gamma: P even, one lane group per shard;
// Q and K of the same slot geometry take separate warps, others share them
// (mixed); an instance must exist.
struct GPairShape {
    int nwq, nwk;
    bool hq, hk, mix;
};

bool gpair_fits(const Shapes &sh, int32_t P, int32_t dtype, GPairShape *g) {
    if ((P & 1) || P > 32 || sh.q.K != 1 || sh.k.K != 1) return false;
    gpair_slots(sh.q.nv, dtype, &g->nwq, &g->hq);
    gpair_slots(sh.k.nv, dtype, &g->nwk, &g->hk);
    g->mix = sh.q.nv != sh.k.nv;
    if ((g->mix ? P / 2 : P) * kLanes > gpair_max_threads()) return false;
    return fused_gpair_kernel(dtype, g->nwq, g->hq, g->nwk, g->hk, g->mix) != nullptr;
}

// Stages of the staged-gamma ring: two per CTA, so that as many CTAs as the
// SM's shared memory, registers and threads allow are resident (measured at
// the 13B shape in FP8: 3 CTAs x 2 stages 80.8 %, 3 x 3 78.6 %; D = 4096,
// P = 4: 88.8 % vs 84.0 %; groups of warps sharing one staged gamma in a
// larger CTA were slower at every setting); three if two do not fit.
void gpair_stages(int32_t Dq, int32_t Dk, int32_t P, int32_t dtype, const GPairShape &g, qknorm_plan *pl) {
    const int64_t qb = (int64_t)Dq * elem_of(dtype), kb = (int64_t)Dk * elem_of(dtype);
    int S = g_tune_stages > 0 ? g_tune_stages : 2;
    pl->block = (g.mix ? P / 2 : P) * kLanes;
    pl->tokens_per_stage = 1;
    pl->stages = S;
    pl->smem_bytes = (int64_t)gpair_smem_bytes(dtype, P, g.nwq, g.hq, g.nwk, g.hk, Dq / P / vec_of(dtype),
                                               Dk / P / vec_of(dtype), S, qb, kb, nullptr, nullptr, nullptr,
                                               nullptr);
}

// Static part of the plan: which kernel, block size, template width, stages.
int plan_static(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype, int32_t variant,
                int num_sms, int regs, qknorm_plan *pl) {
    const Shapes sh = shapes_of(Dq, Dk, P, dtype);
    std::memset(pl, 0, sizeof *pl);
    pl->groups_q = sh.q.K;
    pl->groups_k = sh.k.K;
    int cta_max = 0;
    fused_cta_kernel(dtype, sh.vmax, false, false, false, &cta_max);
    pl->full_lanes = lane_mode(sh, dtype);
    const bool cta_ok = sh.ntask * kLanes <= cta_max;
    const int tb = tokens_per_stage_for(sh.vmax);
    if (pl->full_lanes == 2 && tb != 1) pl->full_lanes = 0;   // the half-slot mode has one token per stage
    const bool greg = gamma_regs_for(dtype, sh.vmax);
    int bulk_max = 0;
    const bool bulk_inst = fused_bulk_kernel(dtype, sh.vmax, greg, tb, 0, &bulk_max) != nullptr;
    const uint32_t stride = bulk_stage_stride((int64_t)Dq * elem_of(dtype),
                                              (int64_t)Dk * elem_of(dtype), tb);
    const bool bulk_ok = bulk_inst && sh.ntask * kLanes <= bulk_max &&
                         (int64_t)bulk_smem_bytes(2, stride) <= kSmemPerCta;
    const bool rows_ok = rows_fit(Dq, Dk, dtype);
    if (variant == QKNORM_VARIANT_AUTO) {
        // Measured on B200: a CTA per token with registers wins while a CTA
        // sees one token (decode). With several tokens per CTA the token ring
        // wins when every lane holds the same number of vectors; with ragged
        // lanes (e.g. GQA widths) its CTA carries idle lanes and unequal Q/K
        // warps, and the warp-per-row kernel wins. Shapes whose tasks do not
        // fit one CTA go to the rows kernel too.
        // FP8 is instruction-bound, and the token ring with gamma in registers
        // wins for it even on ragged lanes (measured 63 % vs 46 % for rows).
        // GQA-like shapes (Q shards wider than a warp, K shards of at most 16
        // vectors) take the shard-pair ring: P warps per token instead of 2P,
        // two CTAs per SM (measured at T = 4096, 5120/1024, P = 8: 84.8 % vs
        // 66.4 % for rows and 59.8 % for the ring with 2P warps).
        // K shards as wide as Q's go in pairs too (P warps per token) where a
        // warp's fixed work per token weighs most: FP8 at one vector per lane
        // (measured 60.4 -> 82.3 % at T = 65536, D = 4096, P = 8; 58.9 ->
        // 76.4 % at D = 2048, P = 4) and ragged bf16/fp32 lanes (5120/4096,
        // P = 8: 83.4 % vs 76.1 % for rows). Not on full bf16 lanes (99.1 %
        // for the ring with 2P warps vs 89.9 %), nor for FP8 at two or more
        // vectors per lane, whose gamma no longer fits registers (77.7 % vs
        // 44.9 %).
        const bool ragged = !pl->full_lanes && dtype != QKNORM_E4M3;
        const bool kpairs = pair_fits(sh, P, dtype) && pair_kw(sh) && pair_greg(sh, dtype) &&
                            (dtype == QKNORM_E4M3 ? pair_vq(sh) == 1 : ragged);
        // FP8 takes the shard-pair ring with gamma staged in shared memory
        // (two shards per warp, no gamma registers, so 3 CTAs fit an SM) where
        // a lane holds more than one vector per shard or Q and K shards differ
        // (mixed warps). Measured: 13B shape 80.8 % vs 73.9 % for the bulk
        // ring; D = 4096, P = 4, T = 16384: 88.8 % vs 78.1 %; GQA widths, P = 8:
        // 45.8 % vs 37 %. At one vector per lane (D = 4096, P = 8) the
        // shard-pair ring with gamma in registers stays (82.5 % vs 76 %).
        // The instances compiled for an exact shape take it in bf16 as well
        // below 48 tokens per SM (GQA widths, P = 8, one box: T = 4096 93.7 %
        // vs 83.5 % for the shard-pair ring with gamma in registers; 6144:
        // 93.8 vs 88.2 %; 8192: 85.4 vs 91.4 %; 16384: 83.2 vs 98.7 %: the
        // staged-gamma ring's steady rate stays near 85 %, so the register
        // ring takes the large batches).
        GPairShape gp;
        if (T <= 2 * (int64_t)num_sms)
            variant = cta_ok ? QKNORM_VARIANT_CTA : QKNORM_VARIANT_GENERIC;
        else if (dtype == QKNORM_E4M3 && gpair_fits(sh, P, dtype, &gp) && (gp.mix || gp.hq || gp.nwq >= 2))
            variant = QKNORM_VARIANT_GPAIR;
        else if (dtype == QKNORM_BF16 && T < 48 * (int64_t)num_sms && gpair_fits(sh, P, dtype, &gp) &&
                 fused_gpair_kernel_for(dtype, gp.nwq, gp.hq, gp.nwk, gp.hk, gp.mix, P, sh.q.nv, sh.k.nv) !=
                     fused_gpair_kernel(dtype, gp.nwq, gp.hq, gp.nwk, gp.hk, gp.mix))
            variant = QKNORM_VARIANT_GPAIR;
        else if (pair_fits(sh, P, dtype) && !pair_kw(sh) && sh.q.nv > kLanes)
            variant = QKNORM_VARIANT_PAIR;
        else if (kpairs)
            variant = QKNORM_VARIANT_PAIR;
        else if (bulk_ok && !(ragged && rows_ok))
            variant = QKNORM_VARIANT_BULK;
        else if (rows_ok)
            variant = QKNORM_VARIANT_ROWS;
        else
            variant = cta_ok ? QKNORM_VARIANT_CTA : QKNORM_VARIANT_GENERIC;
    }
    if (variant == QKNORM_VARIANT_CTA || variant == QKNORM_VARIANT_BULK) {
        if (variant == QKNORM_VARIANT_CTA ? !cta_ok : !bulk_ok) return QKNORM_ERR_UNSUPPORTED;
        pl->variant = variant;
        pl->block = (int32_t)(sh.ntask * kLanes);
        pl->vmax = sh.vmax;
        if (variant == QKNORM_VARIANT_CTA)
            pl->gamma_regs = cta_greg(sh, dtype, pl->full_lanes == 1) ? 1 : 0;
        if (variant == QKNORM_VARIANT_BULK) {
            pl->gamma_regs = greg ? 1 : 0;
            pl->tokens_per_stage = tb;
            bulk_stages(stride, pl->block, regs > 0 ? regs : kRegsHint, pl);
            if (pl->stages < 1 || pl->stages > bulk_max_stages() ||
                pl->smem_bytes > kSmemPerCta)
                return QKNORM_ERR_UNSUPPORTED;
        }
        return QKNORM_OK;
    }
    if (variant == QKNORM_VARIANT_PAIR) {
        // P warps: Q shards in pairs; K shards in pairs, on lane halves if <= 16 vectors.
        if (!pair_fits(sh, P, dtype)) return QKNORM_ERR_UNSUPPORTED;
        const bool greg_p = pair_greg(sh, dtype);
        pl->variant = QKNORM_VARIANT_PAIR;
        pl->block = P * kLanes;
        pl->vmax = pair_vq(sh);
        pl->k_pairs = pair_kw(sh) ? 1 : 0;
        pl->gamma_regs = greg_p ? 1 : 0;
        pl->tokens_per_stage = 1;
        const uint32_t stride1 = bulk_stage_stride((int64_t)Dq * elem_of(dtype),
                                                   (int64_t)Dk * elem_of(dtype), 1);
        bulk_stages(stride1, pl->block, regs > 0 ? regs : kRegsHint, pl);
        // A third stage pays once a CTA meets about 20 tokens or more (measured:
        // T = 8192, 86.1 -> 89.5 %; T = 16384, 90.9 -> 95.6 %; T = 4096, 84.8 -> 83.7 %).
        if (g_tune_stages == 0 && pl->stages == 2 && T >= 40 * (int64_t)num_sms &&
            2 * ((int64_t)bulk_smem_bytes(3, stride1) + kSmemReservedPerCta) <= kSmemPerSm) {
            pl->stages = 3;
            pl->smem_bytes = (int64_t)bulk_smem_bytes(3, stride1);
        }
        if (pl->stages < 1 || pl->stages > bulk_max_stages() || pl->smem_bytes > kSmemPerCta)
            return QKNORM_ERR_UNSUPPORTED;
        return QKNORM_OK;
    }
    if (variant == QKNORM_VARIANT_GPAIR) {
        GPairShape g;
        if (!gpair_fits(sh, P, dtype, &g)) return QKNORM_ERR_UNSUPPORTED;
        pl->variant = QKNORM_VARIANT_GPAIR;
        pl->vmax = g.nwq;
        pl->vmax_k = g.nwk;
        pl->half_slots = (g.hq ? 1 : 0) | (g.hk ? 2 : 0);
        pl->mixed = g.mix ? 1 : 0;
        gpair_stages(Dq, Dk, P, dtype, g, pl);
        if (pl->stages < 1 || pl->stages > bulk_max_stages() || pl->smem_bytes > kSmemPerCta ||
            pl->block > gpair_max_threads())
            return QKNORM_ERR_UNSUPPORTED;
        return QKNORM_OK;
    }
    if (variant == QKNORM_VARIANT_ROWS) {
        const int S = g_rows_stages > 0 ? g_rows_stages : kRowsStagesAuto;
        RowsChoice c = rows_auto(Dq, Dk, dtype, S, g_rows_gsm, regs > 0 ? regs : kRegsHint);
        if (g_rows_wq > 0) {
            c.wq = g_rows_wq;
            c.wk = g_rows_wk;
            if (g_rows_gsm >= 0) c.gsm = g_rows_gsm != 0;
        }
        if (c.wq < 1 || c.wk < 1 || c.wq + c.wk > kRowsMaxWarps) return QKNORM_ERR_UNSUPPORTED;
        const RowsLayout L = rows_layout(Dq, Dk, (int)elem_of(dtype), c.wq, c.wk, S, c.gsm);
        if (L.smem_bytes > (size_t)kSmemPerCta) return QKNORM_ERR_UNSUPPORTED;
        pl->variant = QKNORM_VARIANT_ROWS;
        pl->block = (c.wq + c.wk) * kLanes;
        pl->stages = S;
        pl->q_warps = c.wq;
        pl->gamma_smem = c.gsm ? 1 : 0;
        pl->smem_bytes = (int64_t)L.smem_bytes;
        return QKNORM_OK;
    }
    if (variant == QKNORM_VARIANT_WARP && warp_regs_fit(sh, P, dtype)) {
        pl->variant = QKNORM_VARIANT_WARP;
        pl->block = kLanes;              // one token per CTA: the tokens spread over the SMs
        pl->vmax = sh.q.vmax;
        pl->vmax_k = sh.k.vmax;
        return QKNORM_OK;
    }
    if ((size_t)sh.ntask * sizeof(float) > (size_t)kGenericMaxSmem) return QKNORM_ERR_UNSUPPORTED;
    pl->smem_bytes = (int64_t)(sh.ntask * sizeof(float));
    if (variant == QKNORM_VARIANT_WARP) {
        pl->variant = QKNORM_VARIANT_WARP;
        pl->block = kLanes;
        return QKNORM_OK;
    }
    if (variant == QKNORM_VARIANT_GENERIC) {
        pl->variant = QKNORM_VARIANT_GENERIC;
        const int64_t b = sh.ntask * kLanes;
        pl->block = (int32_t)(b < 256 ? b : 256);
        return QKNORM_OK;
    }
    return QKNORM_ERR_INVALID_ARG;
}

// Units of work a CTA can take: tokens, or for the rows variant the CTAs
// that give every warp of the smaller pool a row (T Q rows over q_warps
// warps per CTA, T K rows over the others).
int64_t plan_units(int64_t T, const qknorm_plan &pl) {
    if (pl.variant == QKNORM_VARIANT_WARP && pl.vmax > 0) {
        const int64_t w = pl.block / kLanes;             // tokens per CTA
        return (T + w - 1) / w;
    }
    if (pl.variant != QKNORM_VARIANT_ROWS) return T;
    const int64_t wq = pl.q_warps, wk = pl.block / kLanes - pl.q_warps;
    const int64_t w = wq < wk ? wq : wk;
    return (T + w - 1) / w;
}

// Grid: T CTAs up to B_res x N_SM (or the forced grid); the register variant
// prefetches when a CTA gets more than one token.
void plan_grid(int64_t T, int num_sms, int blocks_per_sm, qknorm_plan *pl) {
    int64_t cap = (int64_t)num_sms * blocks_per_sm;
    if (g_forced_grid > 0) cap = g_forced_grid;
    if (cap < 1) cap = 1;
    pl->grid = T < cap ? T : cap;
    if (pl->grid < 1) pl->grid = 1;
    pl->prefetch = (pl->variant == QKNORM_VARIANT_CTA && T > pl->grid) ? 1 : 0;
    if (pl->prefetch) pl->gamma_regs = 0;   // the gamma-register instances take one token per CTA
}

// The kernel a plan launches (for the occupancy query: the register variant
// with prefetch, whose footprint is the larger).
const void *plan_kernel(const qknorm_plan &pl, int32_t dtype, int32_t P, int32_t Dq, int32_t Dk,
                        bool for_occupancy) {
    switch (pl.variant) {
    case QKNORM_VARIANT_CTA:
        if (pl.gamma_regs && !for_occupancy)
            return fused_cta_kernel(dtype, pl.vmax, false, pl.full_lanes == 1, true, nullptr);
        return fused_cta_kernel(dtype, pl.vmax, for_occupancy || pl.prefetch != 0,
                                pl.full_lanes == 1, false, nullptr);
    case QKNORM_VARIANT_WARP:
        if (pl.vmax > 0) return fused_warp_kernel(dtype, P, pl.vmax, pl.vmax_k);
        return fused_generic_kernel(dtype);
    case QKNORM_VARIANT_BULK:
        return fused_bulk_kernel(dtype, pl.vmax, pl.gamma_regs != 0, pl.tokens_per_stage,
                                 pl.full_lanes, nullptr);
    case QKNORM_VARIANT_ROWS:
        return fused_rows_kernel(dtype);
    case QKNORM_VARIANT_PAIR:
        return fused_pair_kernel_for(dtype, pl.vmax, pl.gamma_regs != 0, pl.k_pairs != 0, P,
                                     Dq / P / vec_of(dtype), Dk / P / vec_of(dtype));
    case QKNORM_VARIANT_GPAIR:
        return fused_gpair_kernel_for(dtype, pl.vmax, (pl.half_slots & 1) != 0, pl.vmax_k,
                                      (pl.half_slots & 2) != 0, pl.mixed != 0, P, Dq / P / vec_of(dtype),
                                      Dk / P / vec_of(dtype));
    default:
        return fused_generic_kernel(dtype);
    }
}

// Per-device, per-kernel one-time set-up: the dynamic shared memory opt-in.
struct Prepared {
    int device;
    const void *fn;
};
constexpr int kPreparedSlots = 512;
Prepared g_prepared[kPreparedSlots];
int g_prepared_n = 0;
std::mutex g_prepared_mu;

cudaError_t prepare_kernel(int dev, const void *fn, int max_dynamic_smem) {
    std::lock_guard<std::mutex> lock(g_prepared_mu);
    for (int i = 0; i < g_prepared_n; ++i)
        if (g_prepared[i].device == dev && g_prepared[i].fn == fn) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dynamic_smem);
    if (e != cudaSuccess) return e;
    if (g_prepared_n < kPreparedSlots) g_prepared[g_prepared_n++] = Prepared{dev, fn};
    return cudaSuccess;
}

struct RegEntry {
    const void *fn;
    int regs;
};
RegEntry g_regs[kPreparedSlots];
int g_regs_n = 0;

cudaError_t kernel_regs(const void *fn, int *regs) {
    std::lock_guard<std::mutex> lock(g_prepared_mu);
    for (int i = 0; i < g_regs_n; ++i)
        if (g_regs[i].fn == fn) {
            *regs = g_regs[i].regs;
            return cudaSuccess;
        }
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, fn);
    if (e != cudaSuccess) return e;
    *regs = attr.numRegs > 0 ? attr.numRegs : kRegsHint;
    if (g_regs_n < kPreparedSlots) g_regs[g_regs_n++] = RegEntry{fn, *regs};
    return cudaSuccess;
}

// Full device plan: the kernel's registers and the device's SM count, then
// occupancy with the plan's shared memory gives B_res.
cudaError_t plan_device(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                        qknorm_plan *pl, int *status) {
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return e;
    *status = plan_static(T, Dq, Dk, P, dtype, g_forced_variant, sms, kRegsHint, pl);
    if (*status != QKNORM_OK) return cudaSuccess;
    if (pl->variant == QKNORM_VARIANT_BULK || pl->variant == QKNORM_VARIANT_ROWS ||
        pl->variant == QKNORM_VARIANT_PAIR || pl->variant == QKNORM_VARIANT_GPAIR) {
        int regs = kRegsHint;
        e = kernel_regs(plan_kernel(*pl, dtype, P, Dq, Dk, true), &regs);
        if (e != cudaSuccess) return e;
        *status = plan_static(T, Dq, Dk, P, dtype, g_forced_variant, sms, regs, pl);
        if (*status != QKNORM_OK) return cudaSuccess;
    }
    const void *fn = plan_kernel(*pl, dtype, P, Dq, Dk, true);
    if (pl->smem_bytes > 48 * 1024 || pl->variant == QKNORM_VARIANT_GENERIC ||
        (pl->variant == QKNORM_VARIANT_WARP && pl->vmax == 0)) {
        e = prepare_kernel(dev, fn, (pl->variant == QKNORM_VARIANT_BULK ||
                                     pl->variant == QKNORM_VARIANT_ROWS ||
                                     pl->variant == QKNORM_VARIANT_PAIR ||
                                     pl->variant == QKNORM_VARIANT_GPAIR) ? kSmemPerCta : kGenericMaxSmem);
        if (e != cudaSuccess) return e;
    }
    int bres = 1;
    e = resident_blocks(dev, fn, pl->block, (size_t)pl->smem_bytes, &bres);
    if (e != cudaSuccess) return e;
    plan_grid(plan_units(T, *pl), sms, bres, pl);
    return cudaSuccess;
}

int finish(cudaError_t e) {
    if (e != cudaSuccess) {
        set_error(e);
        return QKNORM_ERR_CUDA;
    }
    return QKNORM_OK;
}

// ---------------------------------------------------------------- host buffers

// qknorm_fwd_host's pipeline: per device, a stream for host-to-device copies,
// one for device-to-host copies (both non-blocking) and kHostSets workspace
// sets with three events each, created once. The caller's stream runs the
// kernels. Calls are serialised by a mutex while they enqueue.
constexpr int kHostSets = 3;
// Tokens per chunk. Every copy has a fixed cost and the pipeline's fill and
// drain grow with the chunk: at the 13B shape (336 MB per call) 256-token
// chunks took 4.61 ms, 512 4.06-4.14, 1024 3.98-4.03, 2048 4.18-4.26 (one
// box each); chunks tapered to a quarter and a half at both ends measured
// slower than uniform ones (4.09 vs 4.03 ms at 1024).
constexpr int64_t kHostChunkDefault = 1024;
constexpr int kHostMaxDevices = 64;

struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t in_done[kHostSets] = {}, k_done[kHostSets] = {}, out_done[kHostSets] = {};
};
HostPipe g_host_pipes[kHostMaxDevices];
std::mutex g_host_mu;

cudaError_t host_pipe(HostPipe **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kHostMaxDevices) return cudaErrorInvalidDevice;
    HostPipe &hp = g_host_pipes[dev];
    if (!hp.ready) {
        if ((e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming)) != cudaSuccess) return e;
        for (int i = 0; i < kHostSets; ++i) {
            if ((e = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming)) != cudaSuccess) return e;
            if ((e = cudaEventCreateWithFlags(&hp.k_done[i], cudaEventDisableTiming)) != cudaSuccess) return e;
            if ((e = cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming)) != cudaSuccess) return e;
        }
        hp.ready = true;
    }
    *out = &hp;
    return cudaSuccess;
}

int64_t host_chunk(int64_t chunk_tokens) { return chunk_tokens > 0 ? chunk_tokens : kHostChunkDefault; }

}  // namespace
}  // namespace qkn

using namespace qkn;

// Grid shares of a launch over n (1 or 2) tensors: at most cap blocks in
// all, side z at most need[z] (its work) and at least 1, the rest in
// proportion to the sides' bytes. Returns side 0's share; *total the grid.
static int64_t split_grid(int n, const int64_t *need, const int64_t *bytes, int64_t cap,
                          int64_t *total) {
    if (n == 1) {
        *total = need[0] < cap ? need[0] : cap;
        return *total;
    }
    int64_t all = need[0] + need[1];
    if (all > cap) all = cap;
    if (all < 2) all = 2;
    int64_t g0 = (int64_t)((double)all * (double)bytes[0] / (double)(bytes[0] + bytes[1]) + 0.5);
    if (g0 > need[0]) g0 = need[0];
    if (g0 > all - 1) g0 = all - 1;
    if (g0 < 1) g0 = 1;
    int64_t g1 = all - g0;
    if (g1 > need[1]) g1 = need[1];
    *total = g0 + g1;
    return g0;
}

// Argument checks of the statistics pass for one tensor.
static int check_stats_side(const void *x, const float *stats, int64_t T, int32_t D, int32_t P,
                            int32_t dtype) {
    int st = check_shape(T, D, P, dtype);
    if (st != QKNORM_OK || T == 0) return st;
    if (!x || !stats) return QKNORM_ERR_INVALID_ARG;
    // The sums are written one fp32 at a time: 4-byte alignment suffices (the
    // K half of a [2, T, P] array starts T * P floats in).
    if (!aligned16(x) || reinterpret_cast<uintptr_t>(stats) % 4 != 0) return QKNORM_ERR_MISALIGNED;
    if (T > INT64_MAX / 4 / P) return QKNORM_ERR_INVALID_ARG;
    if (overlap(rng(stats, T * P * 4), rng(x, T * D * elem_of(dtype)))) return QKNORM_ERR_INVALID_ARG;
    return QKNORM_OK;
}

// The statistics pass over n (1 or 2) checked tensors of T > 0 rows: one launch.
static int stats_launch(int n, const void *const *x, float *const *stats, const int32_t *D,
                        int64_t T, int32_t P, int32_t dtype, void *stream) {
    TensorShape sh[2];
    int vmax = 0;
    for (int z = 0; z < n; ++z) {
        sh[z] = make_shape(D[z], P, vec_of(dtype));
        if (sh[z].vmax > vmax) vmax = sh[z].vmax;
    }
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    const int block = 256;
    int64_t in_bytes = 0;
    for (int z = 0; z < n; ++z) in_bytes += T * D[z] * elem_of(dtype);
    const bool keep = in_bytes <= kStatsKeepBytes;
    int bres = 1;
    e = resident_blocks(dev, stats_kernel(dtype, vmax, n == 2, keep), block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    // A block takes (block / 32) warps x R tasks per turn.
    const int64_t per_block = (block / kLanes) * (vmax <= 2 ? 4 : (vmax <= 4 ? 2 : 1));
    int64_t need[2], bytes[2], grid = 0;
    for (int z = 0; z < n; ++z) {
        need[z] = (T * P + per_block - 1) / per_block;
        bytes[z] = (int64_t)D[z];
    }
    StatsArgs a;
    for (int z = 0; z < 2; ++z) {
        const int w = z < n ? z : 0;
        a.side[z] = StatsSide{x[w], stats[w], D[w], sh[w].nv, sh[w].K};
    }
    a.T = T;
    a.P = P;
    a.split = (int32_t)split_grid(n, need, bytes, (int64_t)sms * bres, &grid);
    return finish(launch_stats(dtype, vmax, keep, a, block, grid, reinterpret_cast<cudaStream_t>(stream)));
}

// Argument checks of the apply step for one tensor, stats laid out as nb
// blocks [nb, T, Pb] (nb = 1: the split path's [T, P]; nb = ranks: an
// all-gather of each rank's [T, P_local] in a tensor-parallel group, whose
// rows are the D-wide local slices of nb * D-wide rows). *sg is set to the
// block stride in use.
static int check_apply_side(const void *x, const float *gamma, const float *stats, int64_t *sg,
                            const void *out, int64_t T, int32_t D, int32_t Pb, int32_t nb, float eps,
                            int32_t dtype) {
    int st = check_shape(T, D, Pb, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    if (nb < 1 || (int64_t)D * nb > INT32_MAX) return QKNORM_ERR_INVALID_ARG;
    if (T == 0) return QKNORM_OK;
    if (!x || !gamma || !stats || !out) return QKNORM_ERR_INVALID_ARG;
    // The statistics are read one fp32 at a time: 4-byte alignment suffices
    // (a gather of Q's and K's sums puts K's blocks T * P floats further on).
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(out) ||
        reinterpret_cast<uintptr_t>(stats) % 4 != 0)
        return QKNORM_ERR_MISALIGNED;
    if (T > INT64_MAX / 4 / Pb / nb) return QKNORM_ERR_INVALID_ARG;
    if (*sg == 0) *sg = T * Pb;
    if (*sg < T * Pb || *sg > INT64_MAX / 4 / nb) return QKNORM_ERR_INVALID_ARG;   // blocks may not overlap
    const int64_t es = elem_of(dtype);
    const Range ro = rng(out, T * D * es);
    if (bad_alias(ro, rng(x, T * D * es), true) || bad_alias(ro, rng(gamma, (int64_t)D * 4), false) ||
        bad_alias(ro, rng(stats, ((int64_t)(nb - 1) * *sg + T * Pb) * 4), false))
        return QKNORM_ERR_INVALID_ARG;
    return QKNORM_OK;
}

// The apply step over n (1 or 2) checked tensors of T > 0 rows: one launch.
// The divisor of side z is nb * D[z].
static int apply_launch(int n, const void *const *x, const float *const *gamma,
                        const float *const *stats, void *const *out, const int32_t *D, int64_t sg,
                        int64_t T, int32_t Pb, int32_t nb, float eps, int32_t dtype, void *stream) {
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    // Rows of at most 32 x kApplyNarrowMaxV vectors: a warp per row (apply_w).
    int64_t rowvec = 0;
    for (int z = 0; z < n; ++z)
        if (D[z] / vec_of(dtype) > rowvec) rowvec = D[z] / vec_of(dtype);
    if (rowvec <= 32 * kApplyNarrowMaxV) {
        const int v = (int)((rowvec + 31) / 32);
        int bres = 1;
        const int vec = vec_of(dtype);
        e = resident_blocks(dev,
                            apply_narrow_kernel_for(dtype, v, n == 2, D[0] / vec, D[n == 2 ? 1 : 0] / vec, Pb, nb),
                            256, 0, &bres);
        if (e != cudaSuccess) return finish(e);
        ApplyArgs a;
        for (int z = 0; z < 2; ++z) {
            const int w = z < n ? z : 0;
            a.side[z] = ApplySide{x[w], gamma[w], stats[w], out[w], D[w], kLanes, (float)((int64_t)D[w] * nb)};
        }
        a.T = T;
        a.sg = sg;
        a.Pb = Pb;
        a.nb = nb;
        a.eps = eps;
        a.split = 0;
        const int64_t need = (T * n + 7) / 8, cap = (int64_t)sms * (bres > 0 ? bres : 1);
        return finish(launch_apply_narrow(dtype, v, a, n == 2, need < cap ? need : cap,
                                          reinterpret_cast<cudaStream_t>(stream)));
    }
    // apply_threads_per_row(D) threads per row. One tensor: as many rows per
    // 256-thread block as fit. Two: a block size both sides' row groups
    // divide (192 for 96-thread rows, else 256; a side's spare threads idle).
    int tpr[2] = {0, 0};
    bool multi = false, has96 = false, wide = false;
    for (int z = 0; z < n; ++z) {
        tpr[z] = apply_threads_per_row(D[z], dtype);
        multi = multi || tpr[z] != 256;
        has96 = has96 || tpr[z] == 96;
        wide = wide || tpr[z] == 256;
    }
    const int block = n == 1 ? tpr[0] * (256 / tpr[0]) : (has96 && !wide ? 192 : 256);
    int bres = 1;
    e = resident_blocks(dev, apply_kernel(dtype, multi, n == 2, apply_fold(nb)), block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    int64_t need[2], bytes[2], grid = 0;
    ApplyArgs a;
    for (int z = 0; z < 2; ++z) {
        const int w = z < n ? z : 0;
        const int rpb = block / tpr[w];
        need[z] = (T + rpb - 1) / rpb;
        bytes[z] = (int64_t)D[w];
        a.side[z] = ApplySide{x[w], gamma[w], stats[w], out[w], D[w], tpr[w],
                              (float)((int64_t)D[w] * nb)};
    }
    a.T = T;
    a.sg = sg;
    a.Pb = Pb;
    a.nb = nb;
    a.eps = eps;
    a.split = (int32_t)split_grid(n, need, bytes, (int64_t)sms * bres, &grid);
    return finish(launch_apply(dtype, multi, a, block, grid, reinterpret_cast<cudaStream_t>(stream)));
}

static int apply_blocks(const void *x, const float *gamma, const float *stats, int64_t sg, void *out,
                        int64_t T, int32_t D, int32_t Pb, int32_t nb, float eps, int32_t dtype,
                        void *stream) {
    int st = check_apply_side(x, gamma, stats, &sg, out, T, D, Pb, nb, eps, dtype);
    if (st != QKNORM_OK || T == 0) return st;
    return apply_launch(1, &x, &gamma, &stats, &out, &D, sg, T, Pb, nb, eps, dtype, stream);
}

extern "C" {

int qknorm_version(void) { return 125; }

const char *qknorm_status_string(int status) {
    switch (status) {
    case QKNORM_OK: return "ok";
    case QKNORM_ERR_INVALID_ARG: return "invalid argument";
    case QKNORM_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case QKNORM_ERR_UNSUPPORTED: return "unsupported dtype or shard width";
    case QKNORM_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
    }
}

const char *qknorm_last_error(void) { return g_last_error; }

int qknorm_force_variant(int32_t variant, int64_t grid) {
    if (variant < QKNORM_VARIANT_AUTO || variant > QKNORM_VARIANT_GPAIR || grid < 0)
        return QKNORM_ERR_INVALID_ARG;
    g_forced_variant = variant;
    g_forced_grid = grid;
    return QKNORM_OK;
}

int qknorm_plan_fwd(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                    int32_t num_sms, int32_t blocks_per_sm, qknorm_plan *plan) {
    if (plan == nullptr || num_sms <= 0) return QKNORM_ERR_INVALID_ARG;
    int st = check_shape(T, Dq, P, dtype);
    if (st == QKNORM_OK) st = check_shape(T, Dk, P, dtype);
    if (st != QKNORM_OK) return st;
    st = plan_static(T, Dq, Dk, P, dtype, g_forced_variant, num_sms, kRegsHint, plan);
    if (st != QKNORM_OK) return st;
    if (blocks_per_sm <= 0) {
        blocks_per_sm = kThreadsPerSm / plan->block;
        if (plan->smem_bytes > 0) {
            const int by_smem = kSmemPerSm / (int)(plan->smem_bytes + kSmemReservedPerCta);
            if (by_smem < blocks_per_sm) blocks_per_sm = by_smem;
        }
        if (blocks_per_sm > 32) blocks_per_sm = 32;
        if (blocks_per_sm < 1) blocks_per_sm = 1;
    }
    plan_grid(plan_units(T, *plan), num_sms, blocks_per_sm, plan);
    return QKNORM_OK;
}

int qknorm_launch_plan(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                       qknorm_plan *plan) {
    if (plan == nullptr) return QKNORM_ERR_INVALID_ARG;
    int st = check_shape(T, Dq, P, dtype);
    if (st == QKNORM_OK) st = check_shape(T, Dk, P, dtype);
    if (st != QKNORM_OK) return st;
    cudaError_t e = plan_device(T > 0 ? T : 1, Dq, Dk, P, dtype, plan, &st);
    if (e != cudaSuccess) return finish(e);
    return st;
}

int qknorm_fwd_strided(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
                       void *out_q, void *out_k, int64_t T, int32_t Dq, int32_t Dk, int32_t P,
                       float eps, int32_t dtype, int64_t ldq, int64_t ldk, int64_t ldoq,
                       int64_t ldok, void *stream) {
    int st = check_shape(T, Dq, P, dtype);
    if (st == QKNORM_OK) st = check_shape(T, Dk, P, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    if (ldq < Dq || ldk < Dk || ldoq < Dq || ldok < Dk) return QKNORM_ERR_INVALID_ARG;
    const int vec = vec_of(dtype);
    if (ldq % vec || ldk % vec || ldoq % vec || ldok % vec) return QKNORM_ERR_MISALIGNED;
    const int64_t es = elem_of(dtype);
    const int64_t ldmax = ldq > ldk ? (ldq > ldoq ? (ldq > ldok ? ldq : ldok) : (ldoq > ldok ? ldoq : ldok))
                                    : (ldk > ldoq ? (ldk > ldok ? ldk : ldok) : (ldoq > ldok ? ldoq : ldok));
    if (T > 0 && T > INT64_MAX / (ldmax * es)) return QKNORM_ERR_INVALID_ARG;
    if (T == 0) return QKNORM_OK;
    if (!q || !k || !gamma_q || !gamma_k || !out_q || !out_k) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(gamma_q) || !aligned16(gamma_k) ||
        !aligned16(out_q) || !aligned16(out_k))
        return QKNORM_ERR_MISALIGNED;
    const Strided mq = strided(q, Dq * es, ldq * es, T), mk = strided(k, Dk * es, ldk * es, T);
    const Strided mgq = strided(gamma_q, (int64_t)Dq * 4, (int64_t)Dq * 4, 1);
    const Strided mgk = strided(gamma_k, (int64_t)Dk * 4, (int64_t)Dk * 4, 1);
    const Strided moq = strided(out_q, Dq * es, ldoq * es, T), mok = strided(out_k, Dk * es, ldok * es, T);
    if (strided_bad_alias(moq, mq, true) || strided_bad_alias(moq, mk, false) ||
        strided_bad_alias(moq, mgq, false) || strided_bad_alias(moq, mgk, false) ||
        strided_bad_alias(moq, mok, false) || strided_bad_alias(mok, mk, true) ||
        strided_bad_alias(mok, mq, false) || strided_bad_alias(mok, mgq, false) ||
        strided_bad_alias(mok, mgk, false))
        return QKNORM_ERR_INVALID_ARG;

    qknorm_plan pl;
    cudaError_t e = plan_device(T, Dq, Dk, P, dtype, &pl, &st);
    if (e != cudaSuccess) return finish(e);
    if (st != QKNORM_OK) return st;

    const TensorShape sq = make_shape(Dq, P, vec_of(dtype));
    const TensorShape sk = make_shape(Dk, P, vec_of(dtype));
    FusedArgs a;
    a.x[0] = q;
    a.x[1] = k;
    a.g[0] = gamma_q;
    a.g[1] = gamma_k;
    a.y[0] = out_q;
    a.y[1] = out_k;
    a.T = T;
    a.D[0] = Dq;
    a.D[1] = Dk;
    a.nv[0] = sq.nv;
    a.nv[1] = sk.nv;
    a.K[0] = sq.K;
    a.K[1] = sk.K;
    a.P = P;
    a.Df[0] = (float)Dq;
    a.Df[1] = (float)Dk;
    a.eps = eps;
    a.ldx[0] = ldq / vec;
    a.ldx[1] = ldk / vec;
    a.ldy[0] = ldoq / vec;
    a.ldy[1] = ldok / vec;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (pl.variant == QKNORM_VARIANT_CTA) {
        e = launch_fused_cta(dtype, pl.vmax, pl.prefetch != 0, pl.full_lanes == 1,
                             pl.gamma_regs != 0, a, pl.block, pl.grid, s);
    } else if (pl.variant == QKNORM_VARIANT_WARP && pl.vmax > 0) {
        e = launch_fused_warp(dtype, P, pl.vmax, pl.vmax_k, a, pl.block, pl.grid, s);
    } else if (pl.variant == QKNORM_VARIANT_ROWS) {
        e = launch_fused_rows(dtype, a, pl.q_warps, pl.block / kLanes - pl.q_warps, pl.stages,
                              pl.gamma_smem != 0, pl.grid, g_wait_limit_ns, s);
    } else if (pl.variant == QKNORM_VARIANT_GPAIR) {
        e = launch_fused_gpair(dtype, pl.vmax, (pl.half_slots & 1) != 0, pl.vmax_k,
                               (pl.half_slots & 2) != 0, pl.mixed != 0, a, pl.stages, pl.grid,
                               g_wait_limit_ns, s);
    } else if (pl.variant == QKNORM_VARIANT_PAIR) {
        e = launch_fused_pair(dtype, pl.vmax, pl.gamma_regs != 0, pl.k_pairs != 0, a, pl.stages,
                              pl.grid, g_wait_limit_ns, s);
    } else if (pl.variant == QKNORM_VARIANT_BULK) {
        e = launch_fused_bulk(dtype, pl.vmax, pl.gamma_regs != 0, pl.tokens_per_stage,
                              pl.full_lanes, a, pl.stages, pl.block, pl.grid,
                              g_wait_limit_ns, s);
    } else {
        e = launch_fused_generic(dtype, a, pl.block, pl.grid, (size_t)pl.smem_bytes, s);
    }
    return finish(e);
}

int qknorm_fwd(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
               void *out_q, void *out_k, int64_t T, int32_t Dq, int32_t Dk, int32_t P,
               float eps, int32_t dtype, void *stream) {
    return qknorm_fwd_strided(q, k, gamma_q, gamma_k, out_q, out_k, T, Dq, Dk, P, eps, dtype, Dq, Dk,
                              Dq, Dk, stream);
}

int qknorm_headwise_fwd(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
                        void *out_q, void *out_k, int64_t T, int32_t Hq, int32_t Hk,
                        int32_t head_dim, float eps, int32_t dtype, int64_t ldq, int64_t ldk,
                        int64_t ldoq, int64_t ldok, void *stream) {
    if (T < 0 || Hq <= 0 || Hk <= 0 || head_dim <= 0) return QKNORM_ERR_INVALID_ARG;
    if (Hq > INT32_MAX / head_dim || Hk > INT32_MAX / head_dim) return QKNORM_ERR_INVALID_ARG;
    const int32_t Dq = Hq * head_dim, Dk = Hk * head_dim;
    int st = check_shape(T, Dq, Hq, dtype);
    if (st == QKNORM_OK) st = check_shape(T, Dk, Hk, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    const int vec = vec_of(dtype);
    const int nv = head_dim / vec;
    if (nv > 256) return QKNORM_ERR_UNSUPPORTED;
    if (ldq < Dq || ldk < Dk || ldoq < Dq || ldok < Dk) return QKNORM_ERR_INVALID_ARG;
    if (ldq % vec || ldk % vec || ldoq % vec || ldok % vec) return QKNORM_ERR_MISALIGNED;
    const int64_t es = elem_of(dtype);
    int64_t ldmax = ldq;
    if (ldk > ldmax) ldmax = ldk;
    if (ldoq > ldmax) ldmax = ldoq;
    if (ldok > ldmax) ldmax = ldok;
    if (T > 0 && T > INT64_MAX / (ldmax * es)) return QKNORM_ERR_INVALID_ARG;
    if (T == 0) return QKNORM_OK;
    if (!q || !k || !gamma_q || !gamma_k || !out_q || !out_k) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(gamma_q) || !aligned16(gamma_k) ||
        !aligned16(out_q) || !aligned16(out_k))
        return QKNORM_ERR_MISALIGNED;
    const Strided mq = strided(q, Dq * es, ldq * es, T), mk = strided(k, Dk * es, ldk * es, T);
    const Strided mgq = strided(gamma_q, (int64_t)head_dim * 4, (int64_t)head_dim * 4, 1);
    const Strided mgk = strided(gamma_k, (int64_t)head_dim * 4, (int64_t)head_dim * 4, 1);
    const Strided moq = strided(out_q, Dq * es, ldoq * es, T), mok = strided(out_k, Dk * es, ldok * es, T);
    if (strided_bad_alias(moq, mq, true) || strided_bad_alias(moq, mk, false) ||
        strided_bad_alias(moq, mgq, false) || strided_bad_alias(moq, mgk, false) ||
        strided_bad_alias(moq, mok, false) || strided_bad_alias(mok, mk, true) ||
        strided_bad_alias(mok, mq, false) || strided_bad_alias(mok, mgq, false) ||
        strided_bad_alias(mok, mgk, false))
        return QKNORM_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    const void *fn = headwise_kernel(dtype, nv);
    if (!fn) return QKNORM_ERR_UNSUPPORTED;
    const int block = 256;
    int bres = 1;
    e = resident_blocks(dev, fn, block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    // One warp per work group, up to a resident grid.
    int64_t grid = (headwise_groups(T, Hq, Hk, nv) + block / kLanes - 1) / (block / kLanes);
    if (grid > (int64_t)sms * bres) grid = (int64_t)sms * bres;
    HeadArgs a;
    a.x[0] = q;
    a.x[1] = k;
    a.g[0] = gamma_q;
    a.g[1] = gamma_k;
    a.y[0] = out_q;
    a.y[1] = out_k;
    a.T = T;
    a.H[0] = Hq;
    a.H[1] = Hk;
    a.nv = nv;
    a.Df = (float)head_dim;
    a.inv_df = (head_dim & (head_dim - 1)) == 0 ? 1.0f / (float)head_dim : 0.f;
    a.eps = eps;
    a.ldx[0] = ldq / vec;
    a.ldx[1] = ldk / vec;
    a.ldy[0] = ldoq / vec;
    a.ldy[1] = ldok / vec;
    return finish(launch_headwise(dtype, a, block, grid, reinterpret_cast<cudaStream_t>(stream)));
}

int qknorm_xgamma(const void *x, const float *gamma, void *out, int64_t T, int32_t D,
                  int32_t dtype, void *stream) {
    int st = check_shape(T, D, 1, dtype);
    if (st != QKNORM_OK) return st;
    if (T == 0) return QKNORM_OK;
    if (!x || !gamma || !out) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(out)) return QKNORM_ERR_MISALIGNED;
    const int64_t es = elem_of(dtype);
    const Range ro = rng(out, T * D * es);
    if (bad_alias(ro, rng(x, T * D * es), true) || bad_alias(ro, rng(gamma, (int64_t)D * 4), false))
        return QKNORM_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    const int64_t rowvec = D / vec_of(dtype);
    int block = (int)((rowvec + kLanes - 1) / kLanes * kLanes);
    if (block > 256) block = 256;
    int bres = 1;
    e = resident_blocks(dev, xgamma_kernel(dtype), block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    int64_t grid = (int64_t)sms * bres;
    if (grid > T) grid = T;
    return finish(launch_xgamma(dtype, x, gamma, out, T, D, block, grid,
                                reinterpret_cast<cudaStream_t>(stream)));
}

int qknorm_inv_rms(const void *x, float *inv_rms, int64_t T, int32_t D, int32_t P, float eps,
                   int32_t dtype, void *stream) {
    int st = check_shape(T, D, P, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    if (T == 0) return QKNORM_OK;
    if (!x || !inv_rms) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(inv_rms)) return QKNORM_ERR_MISALIGNED;
    if (overlap(rng(inv_rms, T * 4), rng(x, T * D * elem_of(dtype)))) return QKNORM_ERR_INVALID_ARG;
    const TensorShape sh = make_shape(D, P, vec_of(dtype));
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    const int block = 256;
    int bres = 1;
    e = resident_blocks(dev, inv_rms_kernel(dtype), block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    int64_t grid = (T + block / kLanes - 1) / (block / kLanes);
    if (grid > (int64_t)sms * bres) grid = (int64_t)sms * bres;
    return finish(launch_inv_rms(dtype, x, inv_rms, T, sh, P, eps, block, grid,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

int qknorm_set_tuning(int32_t stages, int32_t tokens_per_stage, int32_t gamma_regs,
                      int32_t wait_limit_ms) {
    if (stages < 0 || stages > bulk_max_stages() || gamma_regs < -1 || gamma_regs > 1 ||
        wait_limit_ms < 0 || !(tokens_per_stage == 0 || tokens_per_stage == 1 ||
                               tokens_per_stage == 2))
        return QKNORM_ERR_INVALID_ARG;
    g_tune_stages = stages;
    g_tune_tb = tokens_per_stage;
    g_tune_gamma_regs = gamma_regs;
    g_wait_limit_ns = wait_limit_ms > 0 ? (uint64_t)wait_limit_ms * 1000000ull : 2000000000ull;
    return QKNORM_OK;
}

int qknorm_set_rows_tuning(int32_t q_warps, int32_t k_warps, int32_t stages, int32_t gamma_smem) {
    const bool autow = q_warps == 0 && k_warps == 0;
    if (!autow && (q_warps < 1 || k_warps < 1 || q_warps + k_warps > kRowsMaxWarps))
        return QKNORM_ERR_INVALID_ARG;
    if (stages < 0 || stages > bulk_max_stages() || gamma_smem < -1 || gamma_smem > 1)
        return QKNORM_ERR_INVALID_ARG;
    g_rows_wq = q_warps;
    g_rows_wk = k_warps;
    g_rows_stages = stages;
    g_rows_gsm = gamma_smem;
    return QKNORM_OK;
}

int qknorm_set_pdl(int32_t enable) {
    if (enable != 0 && enable != 1) return QKNORM_ERR_INVALID_ARG;
    g_pdl = enable != 0;
    return QKNORM_OK;
}

int qknorm_device_errors(uint32_t *flags, int32_t clear) {
    if (flags == nullptr) return QKNORM_ERR_INVALID_ARG;
    unsigned v = 0;
    cudaError_t e = read_device_errors(&v, clear != 0);
    if (e != cudaSuccess) return finish(e);
    *flags = v;
    return QKNORM_OK;
}

int qknorm_selftest_bounded_wait(uint64_t limit_ns, void *stream) {
    if (limit_ns == 0 || limit_ns > 10000000000ull) return QKNORM_ERR_INVALID_ARG;
    return finish(launch_bounded_wait_probe(limit_ns, reinterpret_cast<cudaStream_t>(stream)));
}

int qknorm_partial_sumsq(const void *x, float *stats, int64_t T, int32_t D, int32_t P,
                         int32_t dtype, void *stream) {
    const int st = check_stats_side(x, stats, T, D, P, dtype);
    if (st != QKNORM_OK || T == 0) return st;
    return stats_launch(1, &x, &stats, &D, T, P, dtype, stream);
}

int qknorm_partial_sumsq_qk(const void *q, const void *k, float *stats_q, float *stats_k, int64_t T,
                            int32_t Dq, int32_t Dk, int32_t P, int32_t dtype, void *stream) {
    int st = check_stats_side(q, stats_q, T, Dq, P, dtype);
    if (st == QKNORM_OK) st = check_stats_side(k, stats_k, T, Dk, P, dtype);
    if (st != QKNORM_OK || T == 0) return st;
    const Range sq = rng(stats_q, T * P * 4), sk = rng(stats_k, T * P * 4);
    if (overlap(sq, sk) || overlap(sq, rng(k, T * Dk * elem_of(dtype))) ||
        overlap(sk, rng(q, T * Dq * elem_of(dtype))))
        return QKNORM_ERR_INVALID_ARG;
    const void *x[2] = {q, k};
    float *stats[2] = {stats_q, stats_k};
    const int32_t D[2] = {Dq, Dk};
    return stats_launch(2, x, stats, D, T, P, dtype, stream);
}

int qknorm_apply(const void *x, const float *gamma, const float *stats, void *out, int64_t T,
                 int32_t D, int32_t P, float eps, int32_t dtype, void *stream) {
    return apply_blocks(x, gamma, stats, 0, out, T, D, P, 1, eps, dtype, stream);
}

int qknorm_apply_tp(const void *x, const float *gamma, const float *stats, int64_t stats_block_stride,
                    void *out, int64_t T, int32_t D_local, int32_t P_local, int32_t ranks, float eps,
                    int32_t dtype, void *stream) {
    if (stats_block_stride < 0) return QKNORM_ERR_INVALID_ARG;
    return apply_blocks(x, gamma, stats, stats_block_stride, out, T, D_local, P_local, ranks, eps,
                        dtype, stream);
}

int qknorm_apply_tp_qk(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
                       const float *stats_q, const float *stats_k, int64_t stats_block_stride,
                       void *out_q, void *out_k, int64_t T, int32_t Dq_local, int32_t Dk_local,
                       int32_t P_local, int32_t ranks, float eps, int32_t dtype, void *stream) {
    if (stats_block_stride < 0) return QKNORM_ERR_INVALID_ARG;
    int64_t sgq = stats_block_stride, sgk = stats_block_stride;
    int st = check_apply_side(q, gamma_q, stats_q, &sgq, out_q, T, Dq_local, P_local, ranks, eps, dtype);
    if (st == QKNORM_OK)
        st = check_apply_side(k, gamma_k, stats_k, &sgk, out_k, T, Dk_local, P_local, ranks, eps, dtype);
    if (st != QKNORM_OK || T == 0) return st;
    // Across the two tensors nothing an output overlaps may be read or written.
    const int64_t es = elem_of(dtype);
    const int64_t sbytes = ((int64_t)(ranks - 1) * sgq + T * P_local) * 4;
    const Range oq = rng(out_q, T * Dq_local * es), ok = rng(out_k, T * Dk_local * es);
    if (overlap(oq, ok) || overlap(oq, rng(k, T * Dk_local * es)) ||
        overlap(oq, rng(gamma_k, (int64_t)Dk_local * 4)) || overlap(oq, rng(stats_k, sbytes)) ||
        overlap(ok, rng(q, T * Dq_local * es)) || overlap(ok, rng(gamma_q, (int64_t)Dq_local * 4)) ||
        overlap(ok, rng(stats_q, sbytes)))
        return QKNORM_ERR_INVALID_ARG;
    const void *x[2] = {q, k};
    const float *g[2] = {gamma_q, gamma_k};
    const float *stats[2] = {stats_q, stats_k};
    void *out[2] = {out_q, out_k};
    const int32_t D[2] = {Dq_local, Dk_local};
    return apply_launch(2, x, g, stats, out, D, sgq, T, P_local, ranks, eps, dtype, stream);
}

int64_t qknorm_fwd_host_workspace(int64_t chunk_tokens, int32_t Dq, int32_t Dk, int32_t dtype) {
    if (Dq <= 0 || Dk <= 0 || (dtype != QKNORM_F32 && dtype != QKNORM_BF16 && dtype != QKNORM_E4M3))
        return -1;
    const int64_t C = host_chunk(chunk_tokens);
    const int64_t row = ((int64_t)Dq + Dk) * elem_of(dtype);
    if (C > INT64_MAX / kHostSets / row) return -1;
    return kHostSets * C * row;
}

int qknorm_fwd_host(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
                    void *out_q, void *out_k, int64_t T, int32_t Dq, int32_t Dk, int32_t P, float eps,
                    int32_t dtype, void *workspace, int64_t workspace_bytes, int64_t chunk_tokens,
                    void *stream) {
    int st = check_shape(T, Dq, P, dtype);
    if (st == QKNORM_OK) st = check_shape(T, Dk, P, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    if (chunk_tokens < 0) return QKNORM_ERR_INVALID_ARG;
    if (T == 0) return QKNORM_OK;
    if (!q || !k || !gamma_q || !gamma_k || !out_q || !out_k || !workspace) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return QKNORM_ERR_MISALIGNED;
    int64_t C = host_chunk(chunk_tokens);
    if (C > T) C = T;
    const int64_t es = elem_of(dtype);
    const int64_t qrow = (int64_t)Dq * es, krow = (int64_t)Dk * es;
    if (T > INT64_MAX / (qrow + krow)) return QKNORM_ERR_INVALID_ARG;
    const int64_t need = qknorm_fwd_host_workspace(C, Dq, Dk, dtype);
    if (need < 0 || workspace_bytes < need) return QKNORM_ERR_INVALID_ARG;
    // Host ranges must not overlap the outputs (inputs and outputs are
    // distinct host buffers; an output may be its own input).
    const Range roq = rng(out_q, T * qrow), rok = rng(out_k, T * krow);
    if (bad_alias(roq, rng(q, T * qrow), true) || bad_alias(roq, rng(k, T * krow), false) ||
        bad_alias(rok, rng(k, T * krow), true) || bad_alias(rok, rng(q, T * qrow), false) ||
        overlap(roq, rok))
        return QKNORM_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_host_mu);
    HostPipe *hp = nullptr;
    cudaError_t e = host_pipe(&hp);
    if (e != cudaSuccess) return finish(e);
    // Everything is ordered after the work already on the caller's stream.
    if ((e = cudaEventRecord(hp->start, s)) != cudaSuccess) return finish(e);
    if ((e = cudaStreamWaitEvent(hp->h2d, hp->start, 0)) != cudaSuccess) return finish(e);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const unsigned char *qh = static_cast<const unsigned char *>(q);
    const unsigned char *kh = static_cast<const unsigned char *>(k);
    unsigned char *oqh = static_cast<unsigned char *>(out_q);
    unsigned char *okh = static_cast<unsigned char *>(out_k);
    int64_t c = 0;
    for (int64_t t0 = 0; t0 < T; t0 += C, ++c) {
        const int64_t n = (T - t0) < C ? (T - t0) : C;
        const int i = (int)(c % kHostSets);
        unsigned char *dq = ws + (int64_t)i * C * (qrow + krow);
        unsigned char *dk = dq + C * qrow;
        // Set i is free once its previous contents have left for the host.
        if ((e = cudaStreamWaitEvent(hp->h2d, hp->out_done[i], 0)) != cudaSuccess) return finish(e);
        if ((e = cudaMemcpyAsync(dq, qh + t0 * qrow, n * qrow, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess ||
            (e = cudaMemcpyAsync(dk, kh + t0 * krow, n * krow, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess ||
            (e = cudaEventRecord(hp->in_done[i], hp->h2d)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(s, hp->in_done[i], 0)) != cudaSuccess)
            return finish(e);
        // The chunk is normalised in place in the workspace.
        st = qknorm_fwd(dq, dk, gamma_q, gamma_k, dq, dk, n, Dq, Dk, P, eps, dtype, stream);
        if (st != QKNORM_OK) return st;
        if ((e = cudaEventRecord(hp->k_done[i], s)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(hp->d2h, hp->k_done[i], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(oqh + t0 * qrow, dq, n * qrow, cudaMemcpyDeviceToHost, hp->d2h)) != cudaSuccess ||
            (e = cudaMemcpyAsync(okh + t0 * krow, dk, n * krow, cudaMemcpyDeviceToHost, hp->d2h)) != cudaSuccess ||
            (e = cudaEventRecord(hp->out_done[i], hp->d2h)) != cudaSuccess)
            return finish(e);
    }
    // Later work on the caller's stream waits for the outputs to reach the host.
    for (int i = 0; i < kHostSets && i < c; ++i)
        if ((e = cudaStreamWaitEvent(s, hp->out_done[i], 0)) != cudaSuccess) return finish(e);
    return QKNORM_OK;
}

}  // extern "C"
