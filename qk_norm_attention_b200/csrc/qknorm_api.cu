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

int vec_of(int32_t dtype) { return dtype == QKNORM_BF16 ? 8 : 4; }
int64_t elem_of(int32_t dtype) { return dtype == QKNORM_BF16 ? 2 : 4; }

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

// Checks common to every entry point for one [T, D] tensor with P shards.
int check_shape(int64_t T, int32_t D, int32_t P, int32_t dtype) {
    if (T < 0 || D <= 0 || P <= 0) return QKNORM_ERR_INVALID_ARG;
    if (D % P != 0) return QKNORM_ERR_INVALID_ARG;
    if (dtype != QKNORM_F32 && dtype != QKNORM_BF16) return QKNORM_ERR_UNSUPPORTED;
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

// Static part of the plan: which kernel, block size and template width.
int plan_static(int32_t Dq, int32_t Dk, int32_t P, int32_t dtype, int32_t variant,
                qknorm_plan *pl) {
    const TensorShape sq = make_shape(Dq, P, vec_of(dtype));
    const TensorShape sk = make_shape(Dk, P, vec_of(dtype));
    const int64_t ntask = (int64_t)P * (sq.K + sk.K);
    const int vmax = sq.vmax > sk.vmax ? sq.vmax : sk.vmax;
    std::memset(pl, 0, sizeof *pl);
    pl->groups_q = sq.K;
    pl->groups_k = sk.K;
    int cta_max = 0;
    fused_cta_kernel(dtype, vmax, false, &cta_max);
    const bool cta_ok = ntask * kLanes <= cta_max;
    if (variant == QKNORM_VARIANT_AUTO) variant = cta_ok ? QKNORM_VARIANT_CTA : QKNORM_VARIANT_GENERIC;
    if (variant == QKNORM_VARIANT_CTA) {
        if (!cta_ok) return QKNORM_ERR_UNSUPPORTED;
        pl->variant = QKNORM_VARIANT_CTA;
        pl->block = (int32_t)(ntask * kLanes);
        pl->vmax = vmax;
        return QKNORM_OK;
    }
    if ((size_t)ntask * sizeof(float) > (size_t)kGenericMaxSmem) return QKNORM_ERR_UNSUPPORTED;
    if (variant == QKNORM_VARIANT_WARP) {
        pl->variant = QKNORM_VARIANT_WARP;
        pl->block = kLanes;
        return QKNORM_OK;
    }
    if (variant == QKNORM_VARIANT_GENERIC) {
        pl->variant = QKNORM_VARIANT_GENERIC;
        const int64_t b = ntask * kLanes;
        pl->block = (int32_t)(b < 256 ? b : 256);
        return QKNORM_OK;
    }
    return QKNORM_ERR_INVALID_ARG;
}

// Grid: T CTAs up to B_res x N_SM (or the forced grid), prefetch when a CTA
// gets more than one token.
void plan_grid(int64_t T, int num_sms, int blocks_per_sm, qknorm_plan *pl) {
    int64_t cap = (int64_t)num_sms * blocks_per_sm;
    if (g_forced_grid > 0) cap = g_forced_grid;
    if (cap < 1) cap = 1;
    pl->grid = T < cap ? T : cap;
    if (pl->grid < 1) pl->grid = 1;
    pl->prefetch = (pl->variant == QKNORM_VARIANT_CTA && T > pl->grid) ? 1 : 0;
}

const void *plan_kernel(const qknorm_plan &pl, int32_t dtype) {
    if (pl.variant == QKNORM_VARIANT_CTA) return fused_cta_kernel(dtype, pl.vmax, pl.prefetch != 0, nullptr);
    return fused_generic_kernel(dtype);
}

size_t plan_smem(const qknorm_plan &pl, int32_t P) {
    if (pl.variant == QKNORM_VARIANT_CTA) return 0;
    return (size_t)P * (pl.groups_q + pl.groups_k) * sizeof(float);
}

bool generic_smem_ready[kMaxDevices][2];

cudaError_t prepare_generic(int dtype) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!generic_smem_ready[dev][dtype]) {
        e = cudaFuncSetAttribute(fused_generic_kernel(dtype),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kGenericMaxSmem);
        if (e != cudaSuccess) return e;
        generic_smem_ready[dev][dtype] = true;
    }
    return cudaSuccess;
}

// Full device plan: occupancy for the chosen kernel (with prefetch, which has
// the larger register footprint, for the persistent case).
cudaError_t plan_device(int64_t T, int32_t Dq, int32_t Dk, int32_t P, int32_t dtype,
                        qknorm_plan *pl, int *status) {
    *status = plan_static(Dq, Dk, P, dtype, g_forced_variant, pl);
    if (*status != QKNORM_OK) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return e;
    if (pl->variant != QKNORM_VARIANT_CTA) {
        e = prepare_generic(dtype);
        if (e != cudaSuccess) return e;
    }
    qknorm_plan probe = *pl;
    probe.prefetch = 1;
    const void *fn = plan_kernel(probe, dtype);
    int bres = 1;
    e = resident_blocks(dev, fn, pl->block, plan_smem(probe, P), &bres);
    if (e != cudaSuccess) return e;
    plan_grid(T, sms, bres, pl);
    return cudaSuccess;
}

int finish(cudaError_t e) {
    if (e != cudaSuccess) {
        set_error(e);
        return QKNORM_ERR_CUDA;
    }
    return QKNORM_OK;
}

}  // namespace
}  // namespace qkn

using namespace qkn;

extern "C" {

int qknorm_version(void) { return 100; }

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
    if (variant < QKNORM_VARIANT_AUTO || variant > QKNORM_VARIANT_GENERIC || grid < 0)
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
    st = plan_static(Dq, Dk, P, dtype, g_forced_variant, plan);
    if (st != QKNORM_OK) return st;
    if (blocks_per_sm <= 0) {
        blocks_per_sm = 2048 / plan->block;
        if (blocks_per_sm > 32) blocks_per_sm = 32;
        if (blocks_per_sm < 1) blocks_per_sm = 1;
    }
    plan_grid(T, num_sms, blocks_per_sm, plan);
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

int qknorm_fwd(const void *q, const void *k, const float *gamma_q, const float *gamma_k,
               void *out_q, void *out_k, int64_t T, int32_t Dq, int32_t Dk, int32_t P,
               float eps, int32_t dtype, void *stream) {
    int st = check_shape(T, Dq, P, dtype);
    if (st == QKNORM_OK) st = check_shape(T, Dk, P, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    if (T == 0) return QKNORM_OK;
    if (!q || !k || !gamma_q || !gamma_k || !out_q || !out_k) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(gamma_q) || !aligned16(gamma_k) ||
        !aligned16(out_q) || !aligned16(out_k))
        return QKNORM_ERR_MISALIGNED;
    const int64_t es = elem_of(dtype);
    const Range rq = rng(q, T * Dq * es), rk = rng(k, T * Dk * es);
    const Range rgq = rng(gamma_q, (int64_t)Dq * 4), rgk = rng(gamma_k, (int64_t)Dk * 4);
    const Range roq = rng(out_q, T * Dq * es), rok = rng(out_k, T * Dk * es);
    if (bad_alias(roq, rq, true) || bad_alias(roq, rk, false) || bad_alias(roq, rgq, false) ||
        bad_alias(roq, rgk, false) || bad_alias(roq, rok, false) || bad_alias(rok, rk, true) ||
        bad_alias(rok, rq, false) || bad_alias(rok, rgq, false) || bad_alias(rok, rgk, false))
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
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (pl.variant == QKNORM_VARIANT_CTA) {
        e = launch_fused_cta(dtype, pl.vmax, pl.prefetch != 0, a, pl.block, pl.grid, s);
    } else {
        e = launch_fused_generic(dtype, a, pl.block, pl.grid, plan_smem(pl, P), s);
    }
    return finish(e);
}

int qknorm_partial_sumsq(const void *x, float *stats, int64_t T, int32_t D, int32_t P,
                         int32_t dtype, void *stream) {
    int st = check_shape(T, D, P, dtype);
    if (st != QKNORM_OK) return st;
    if (T == 0) return QKNORM_OK;
    if (!x || !stats) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(stats)) return QKNORM_ERR_MISALIGNED;
    if (T > INT64_MAX / 4 / P) return QKNORM_ERR_INVALID_ARG;
    if (overlap(rng(stats, T * P * 4), rng(x, T * D * elem_of(dtype)))) return QKNORM_ERR_INVALID_ARG;
    const TensorShape sh = make_shape(D, P, vec_of(dtype));
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    const int block = 256;
    int bres = 1;
    e = resident_blocks(dev, stats_kernel(dtype, sh.vmax), block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    const int64_t ntask = T * P;
    int64_t grid = (ntask + block / kLanes - 1) / (block / kLanes);
    const int64_t cap = (int64_t)sms * bres;
    if (grid > cap) grid = cap;
    return finish(launch_stats(dtype, sh.vmax, x, stats, T, sh, P, block, grid,
                               reinterpret_cast<cudaStream_t>(stream)));
}

int qknorm_apply(const void *x, const float *gamma, const float *stats, void *out, int64_t T,
                 int32_t D, int32_t P, float eps, int32_t dtype, void *stream) {
    int st = check_shape(T, D, P, dtype);
    if (st == QKNORM_OK) st = check_eps(eps);
    if (st != QKNORM_OK) return st;
    if (T == 0) return QKNORM_OK;
    if (!x || !gamma || !stats || !out) return QKNORM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(stats) || !aligned16(out))
        return QKNORM_ERR_MISALIGNED;
    if (T > INT64_MAX / 4 / P) return QKNORM_ERR_INVALID_ARG;
    const int64_t es = elem_of(dtype);
    const Range ro = rng(out, T * D * es);
    if (bad_alias(ro, rng(x, T * D * es), true) || bad_alias(ro, rng(gamma, (int64_t)D * 4), false) ||
        bad_alias(ro, rng(stats, T * P * 4), false))
        return QKNORM_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    cudaError_t e = device_sms(&dev, &sms);
    if (e != cudaSuccess) return finish(e);
    const int64_t rowvec = D / vec_of(dtype);
    int block = (int)((rowvec + kLanes - 1) / kLanes * kLanes);
    if (block > 256) block = 256;
    int bres = 1;
    e = resident_blocks(dev, apply_kernel(dtype), block, 0, &bres);
    if (e != cudaSuccess) return finish(e);
    int64_t grid = (int64_t)sms * bres;
    if (grid > T) grid = T;
    return finish(launch_apply(dtype, x, gamma, stats, out, T, D, P, eps, block, grid,
                               reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
