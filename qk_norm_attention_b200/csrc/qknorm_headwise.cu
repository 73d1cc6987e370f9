// qknorm_headwise.cu -- headwise QK-Norm: one factor per attention head.
//
// SwiftQK technical review, "Prerequisites" (layerwise vs. headwise QK-Norm)
// and Section 4c's comparison table: headwise QK-Norm normalises each head
// on its own, the reduction of Eq. (1) spanning one head's head_dim elements;
// the weight gamma has head_dim entries shared by the heads.
//
// Per head: S = sum of squares in the library's reduction order with the
// head as the only shard (lane chains over vectors lane + 32 i, butterfly),
// r = rsqrt(S / head_dim + eps), y = (x * gamma) * r.
//
// One warp per token walks that token's Q heads, then its K heads, in units:
// with head_dim <= 32 vectors a unit packs 32 / SEG heads into the warp, SEG
// lanes per head (SEG the smallest power of two >= the head's vectors), and
// the butterfly runs over each SEG-lane segment. That equals the 32-lane
// butterfly bit for bit: the xor steps it skips would only add the exact
// zeros of lanes past the head's last vector. Larger heads take a whole warp,
// each lane holding VMAX vectors. R units' loads are issued before any is
// reduced.
//
// Work is dealt in groups of up to R consecutive units of one tensor of one
// token, not in whole tokens: at T = 8192 a resident grid of ~4700 warps would otherwise hold one
// or two tokens each, and the second half of the launch would run with the
// one-token warps already gone. Groups are ~5x finer, so every warp ends
// within one group of the others.
#include "qknorm_device.cuh"
#include "qknorm_internal.h"

namespace qkn {

template <int SEG>
__device__ __forceinline__ float seg_butterfly(float c) {
#pragma unroll
    for (int off = SEG / 2; off >= 1; off /= 2) c = __fadd_rn(c, __shfl_xor_sync(kFull, c, off));
    return c;
}

// CTAs per SM the register budget is sized for. bf16/fp32 heads of up to 32
// vectors: four (64 registers; a 16-byte spill, measured faster than three
// CTAs at 80 registers: 86.3 against 85.4 % at 32 + 8 heads of 128); up to 4
// vectors per lane: two. FP8 keeps 2 x 16 gamma values per lane in registers
// and needs more.
constexpr int headwise_min_blocks(int vec, int vmax) {
    return vec <= 8 && vmax <= 4 ? (vmax == 1 ? 4 : 2) : 1;
}

// One group: units u0 .. u0 + R - 1 of tensor Z (< Uz) of token t. The
// tensor is a template argument, so its row pointers are formed once per
// group and its gamma registers are used without a select.
// CNV: vectors per head fixed at compile time (the instance for heads of 128
// values), 0 read from the arguments; the slot guards and head offsets then
// fold to constants (the arithmetic and its order are the same).
template <class Tag, int SEG, int VMAX, int R, int Z, int CNV>
__device__ __forceinline__ void headwise_group(const HeadArgs &a, int64_t t, int u0, int Uz, int slot,
                                               int hsub, const float *gz) {
    constexpr int VEC = Tag::kVec;
    constexpr int HPW = 32 / SEG;
    const int nv = CNV ? CNV : a.nv;
    const uint4 *xrow = reinterpret_cast<const uint4 *>(a.x[Z]) + t * a.ldx[Z];
    uint4 *yrow = reinterpret_cast<uint4 *>(a.y[Z]) + t * a.ldy[Z];
    uint4 v[R][VMAX];
    bool ok[R];
    int col[R];
#pragma unroll
    for (int j = 0; j < R; ++j) {
        const int head = (u0 + j) * HPW + hsub;
        ok[j] = u0 + j < Uz && head < a.H[Z];
        col[j] = head * nv;
#pragma unroll
        for (int i = 0; i < VMAX; ++i) {
            const int vv = slot + 32 * i;
            if (ok[j] && vv < nv) v[j][i] = ld_stream(xrow + col[j] + vv);
        }
    }
#pragma unroll
    for (int j = 0; j < R; ++j) {
        float c = 0.f;
#pragma unroll
        for (int i = 0; i < VMAX; ++i)
            if (ok[j] && slot + 32 * i < nv) c = __fadd_rn(c, vsumsq(Tag{}, v[j][i]));
        // rsqrt(S / head_dim + eps) as factor() forms it. For a power-of-two
        // head_dim, S * (1 / head_dim) is the same correctly rounded number
        // as the division (the quotient is S scaled by a power of two), so
        // the multiply replaces it bit for bit.
        const float S = seg_butterfly<SEG>(c);
        const float r = a.inv_df != 0.f ? rsqrtf(__fadd_rn(__fmul_rn(S, a.inv_df), a.eps))
                                        : factor(S, a.Df, a.eps);
#pragma unroll
        for (int i = 0; i < VMAX; ++i) {
            const int vv = slot + 32 * i;
            if (ok[j] && vv < nv) {
                const uint4 y = VMAX == 1 ? vapply_regs(Tag{}, v[j][i], gz, r)
                                          : vapply(Tag{}, v[j][i], a.g[Z] + (int64_t)vv * VEC, r);
                st_stream(yrow + col[j] + vv, y);
            }
        }
    }
}

template <class Tag, int SEG, int VMAX, int R, int CNV = 0>
__global__ void __launch_bounds__(256, headwise_min_blocks(Tag::kVec, VMAX)) headwise_k(const HeadArgs a) {
    constexpr int VEC = Tag::kVec;
    constexpr int HPW = 32 / SEG;  // heads per unit
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int slot = lane & (SEG - 1);
    const int hsub = lane / SEG;
    const int nv = CNV ? CNV : a.nv;
    const int64_t NW = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int Uq = (a.H[0] + HPW - 1) / HPW;
    const int Uk = (a.H[1] + HPW - 1) / HPW;
    // Small heads: this lane's gamma for both tensors stays in registers.
    float gr[2][VMAX == 1 ? VEC : 1];
    if (VMAX == 1 && slot < nv) {
#pragma unroll
        for (int z = 0; z < 2; ++z)
#pragma unroll
            for (int e = 0; e < VEC; e += 4) {
                const float4 g4 = __ldg(reinterpret_cast<const float4 *>(a.g[z] + slot * VEC + e));
                gr[z][e] = g4.x;
                gr[z][e + 1] = g4.y;
                gr[z][e + 2] = g4.z;
                gr[z][e + 3] = g4.w;
            }
    }
    // A token's groups: Gq of Q units, then Gk of K units (no group spans both).
    const int Gq = (Uq + R - 1) / R;
    const int G = Gq + (Uk + R - 1) / R;
    // Group gi = t * G + gsub; a warp's groups advance by NW, so (t, gsub) are
    // carried along instead of divided out.
    const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t dt = NW / G;
    const int dg = (int)(NW - dt * G);
    int64_t t = w0 / G;
    int gsub = (int)(w0 - t * G);
    while (t < a.T) {
        if (gsub < Gq)
            headwise_group<Tag, SEG, VMAX, R, 0, CNV>(a, t, gsub * R, Uq, slot, hsub, gr[0]);
        else
            headwise_group<Tag, SEG, VMAX, R, 1, CNV>(a, t, (gsub - Gq) * R, Uk, slot, hsub, gr[1]);
        t += dt;
        gsub += dg;
        if (gsub >= G) {
            gsub -= G;
            ++t;
        }
    }
}

// Lanes per head for a head of nv vectors (nv <= 32), else 32.
static int seg_of(int nv) {
    int s = 1;
    while (s < nv && s < 32) s *= 2;
    return s;
}

// Units per group (R) for heads of up to 32 * VMAX vectors: as many as keep
// R x VMAX <= 8 vectors per lane.
constexpr int units_per_group(int vmax) { return vmax <= 2 ? 4 : (vmax <= 4 ? 2 : 1); }

template <class Tag, int SEG, int VMAX>
const void *headwise_fn() {
    return reinterpret_cast<const void *>(&headwise_k<Tag, SEG, VMAX, units_per_group(VMAX)>);
}

template <class Tag>
const void *headwise_table(int nv) {
    if (nv <= 32) {
        switch (seg_of(nv)) {
        case 1: return headwise_fn<Tag, 1, 1>();
        case 2: return headwise_fn<Tag, 2, 1>();
        case 4: return headwise_fn<Tag, 4, 1>();
        case 8: return headwise_fn<Tag, 8, 1>();
        case 16: return headwise_fn<Tag, 16, 1>();
        default: return headwise_fn<Tag, 32, 1>();
        }
    }
    switch ((nv + 31) / 32) {
    case 2: return headwise_fn<Tag, 32, 2>();
    case 3: return headwise_fn<Tag, 32, 3>();
    case 4: return headwise_fn<Tag, 32, 4>();
    case 5: return headwise_fn<Tag, 32, 5>();
    case 6: return headwise_fn<Tag, 32, 6>();
    case 7: return headwise_fn<Tag, 32, 7>();
    case 8: return headwise_fn<Tag, 32, 8>();
    default: return nullptr;
    }
}

int64_t headwise_groups(int64_t T, int32_t Hq, int32_t Hk, int32_t nv) {
    const int hpw = nv <= kLanes ? kLanes / seg_of(nv) : 1;
    const int64_t uq = (Hq + hpw - 1) / hpw, uk = (Hk + hpw - 1) / hpw;
    const int r = units_per_group((nv + kLanes - 1) / kLanes);
    return T * ((uq + r - 1) / r + (uk + r - 1) / r);
}

// Heads of 128 values (the common head_dim) have an instance with the vectors
// per head compiled in: 32 fp32, 16 bf16, 8 FP8 vectors.
const void *headwise_kernel(int dtype, int nv) {
    if (nv < 1 || nv > 256) return nullptr;
    if (dtype == 0 && nv == 32) return reinterpret_cast<const void *>(&headwise_k<F32Tag, 32, 1, 4, 32>);
    if (dtype == 1 && nv == 16) return reinterpret_cast<const void *>(&headwise_k<BF16Tag, 16, 1, 4, 16>);
    if (dtype == 2 && nv == 8) return reinterpret_cast<const void *>(&headwise_k<E4M3Tag, 8, 1, 4, 8>);
    if (dtype == 0) return headwise_table<F32Tag>(nv);
    if (dtype == 1) return headwise_table<BF16Tag>(nv);
    if (dtype == 2) return headwise_table<E4M3Tag>(nv);
    return nullptr;
}

cudaError_t launch_headwise(int dtype, const HeadArgs &a, int block, int64_t grid, cudaStream_t s) {
    const void *fn = headwise_kernel(dtype, a.nv);
    if (!fn) return cudaErrorInvalidValue;
    void *args[] = {const_cast<HeadArgs *>(&a)};
    return launch(fn, dim3((unsigned)grid), dim3(block), 0, s, args);
}

}  // namespace qkn
