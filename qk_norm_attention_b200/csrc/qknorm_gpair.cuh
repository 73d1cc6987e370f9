// qknorm_gpair.cuh -- the shard-pair token ring with gamma staged in shared
// memory. Included by qknorm_fused_bulk.cu (it shares that file's device
// error word and bulk-copy ring conventions).
//
// SwiftQK technical review, Section 3, Algorithm 1 (Phases A-C per token),
// as a token ring like fused_bulk, but with each warp taking a PAIR of
// shards, so that a warp's fixed work per token (the stage wait, the
// butterflies, the CTA barrier, the factor) is paid once per two shards:
//
//   separate (MIX = false): P warps per token; warp w < P/2 takes Q shards
//     2w and 2w + 1, warp P/2 + w takes K shards 2w and 2w + 1 (Q and K of
//     the same geometry);
//   mixed (MIX = true): P/2 warps per token; warp w takes Q shards 2w, 2w + 1
//     AND K shards 2w, 2w + 1 (GQA-like shapes, whose narrow K shards would
//     leave a K-only warp mostly idle).
//
// Lane l holds, of each of its shards, the vectors l + 32 i (i < NW: the
// single lane group of the library's reduction order), plus, in the HALF
// mode (FP8, a last slot of at most 16 vectors), half of vector 32 NW +
// (l & 15): lane l < 16 the low 8 bytes, lane l + 16 the high 8 bytes. A
// vector's FP8 sum of squares is the sum of its halves' sums, so lane l
// adds lane l + 16's half to its own and the chain has the bits it has in
// every other kernel.
//
// The butterflies of a warp's 2 (or 4) shard chains are one transposed
// butterfly: at the xor-16 step the lane halves trade the chains they do not
// keep (and, with 4, the xor-8 step again), so each shard's sum is completed
// by 16 (or 8) lanes; every addition has the same two operands as in the
// 32-lane butterfly of that shard, so the sums are bit-identical to it.
//
// Gamma is staged once per CTA in shared memory, permuted so that the float4
// a lane needs for (shard, slot, chunk) sits at 32 * index + lane: a warp's
// gamma reads are conflict-free and no gamma lives in registers.
#pragma once

#include <type_traits>

namespace qkn {

struct GPairArgs {
    uint32_t stages;       // S
    uint32_t qbytes;       // bytes of one Q row
    uint32_t kbytes;       // bytes of one K row
    uint32_t stage_stride; // bytes between stages (multiple of 128)
    uint32_t gq4;          // float4 slots of Q's staged gamma
    uint32_t gk4;          // float4 slots of K's staged gamma
    uint32_t stage_base;   // byte offset of the first stage
    uint64_t timeout_ns;   // bound of every wait
};

constexpr uint32_t kGPairRedBytes = 2 * 64 * sizeof(float);   // [buf][Q: 0..31, K: 32..63]
constexpr uint32_t kGPairGammaOff = kBarBytes + kGPairRedBytes;

// Staged-gamma geometry of one tensor: NW whole slots per lane per shard, a
// half slot (H), C = VEC / 4 float4 chunks per vector. Whole slot i, chunk c
// of shard p is read by lane l at float4 index
//   NV = 0 (shard width known at run time): ((p * NW + i) * C + c) * 32 + l,
//     every slot 32 lanes wide (a ragged last slot padded with zeros);
//   compact (compiled for NV vectors per shard, no half slot): p * NV * C
//     + 32 * i * C + c * L_i + l, with L_i = min(32, NV - 32 i) lanes in
//     slot i, so the shard's block is exactly its NV * C float4 (no padding;
//     with a half slot the whole slots are full and both forms agree).
// Either way the lanes of a slot read consecutive float4: conflict-free.
// The half slot (FP8, the last R <= 16 vectors of a shard, lanes l and l + 16
// on the two halves of vector 32 NW + (l & 15)) is read at
//   ((p * CH + c) * 32 + l) padded, or, compiled for NV vectors,
//   p * CH * 2R + c * 2R + (l >> 4) * R + (l & 15): only its 2R lanes.
template <class Tag, int NW, bool H, int NV = 0>
struct GSlots {
    static constexpr int C = Tag::kVec / 4;
    static constexpr int CH = C / 2;
    static constexpr bool kCompact = NV > 0 && !H;
    static constexpr bool kCompactH = NV > 0 && H;
    static constexpr int R = H && NV > 0 ? NV - 32 * NW : 16;   // vectors in the half slot
    __host__ __device__ static int64_t whole(int P) {
        return kCompact ? (int64_t)P * NV * C : (int64_t)P * NW * C * 32;
    }
    __host__ __device__ static int64_t total(int P) {
        return whole(P) + (H ? (int64_t)P * CH * 2 * R : 0);
    }
    __device__ __forceinline__ static int hidx(int p, int c, int lane) {
        if constexpr (kCompactH) return p * CH * 2 * R + c * 2 * R + (lane >> 4) * R + (lane & 15);
        else return (p * CH + c) * 32 + lane;
    }
    __device__ __forceinline__ static int idx(int p, int i, int c, int lane) {
        if constexpr (kCompact) {
            const int L = NV - 32 * i < 32 ? NV - 32 * i : 32;
            return p * NV * C + 32 * i * C + c * L + lane;
        } else {
            return ((p * NW + i) * C + c) * 32 + lane;
        }
    }
    // Where chunk c of vector v of shard p sits: a whole slot's lane v & 31,
    // or a half slot's (half c / CH on lanes r and r + 16).
    __device__ __forceinline__ static int at(int P, int p, int v, int c) {
        if (!H || v < 32 * NW) return idx(p, v >> 5, c, v & 31);
        const int r = v - 32 * NW, hh = c / CH;
        return (int)whole(P) + hidx(p, c - hh * CH, r + 16 * hh);
    }
};

// One tensor's gamma slots of shard p that lane `lane` copies into the
// permuted shared-memory layout: vector l + 32 i, chunk c of each whole slot,
// and the lane's half-slot chunks; zero for vectors the shard does not have.
template <class Tag, int NW, bool H, int NV = 0>
struct GStage {
    using G = GSlots<Tag, NW, H, NV>;
    static constexpr int NL = NW * G::C + (H ? G::CH : 0);   // float4 slots per lane per shard

    __device__ __forceinline__ static void load(float4 (&val)[NL > 0 ? NL : 1], const float *g, int p, int nv,
                                                int lane) {
        constexpr int VEC = Tag::kVec;
        const float4 *gp = reinterpret_cast<const float4 *>(g + (int64_t)p * nv * VEC);
#pragma unroll
        for (int i = 0; i < NW; ++i)
#pragma unroll
            for (int c = 0; c < G::C; ++c) {
                const int v = lane + 32 * i;
                val[i * G::C + c] = v < nv ? __ldg(gp + v * G::C + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        if constexpr (H) {
            const int hv = 32 * NW + (lane & 15);
#pragma unroll
            for (int c = 0; c < G::CH; ++c)
                val[NW * G::C + c] = hv < nv ? __ldg(gp + hv * G::C + (lane >> 4) * G::CH + c)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }

    __device__ __forceinline__ static void store(float4 *dst, const float4 (&val)[NL > 0 ? NL : 1], int P, int p,
                                                 int lane) {
        const int64_t whole = G::whole(P);
#pragma unroll
        for (int i = 0; i < NW; ++i)
            if (!G::kCompact || lane + 32 * i < NV) {
#pragma unroll
                for (int c = 0; c < G::C; ++c) dst[G::idx(p, i, c, lane)] = val[i * G::C + c];
            }
        if constexpr (H) {
            if (!G::kCompactH || (lane & 15) < G::R) {
#pragma unroll
                for (int c = 0; c < G::CH; ++c) dst[whole + G::hidx(p, c, lane)] = val[NW * G::C + c];
            }
        }
    }
};

// Copy both tensors' gamma into their permuted shared-memory layouts. Warp w
// takes shards w, w + nwarps, ...; lane l copies its own slots of a shard of
// Q and of K, all of those loads issued before any store (one L2 round trip
// per shard, not one per slot), with the slot indices fixed at compile time
// so that only the shard offset is computed at run time.
template <class Tag, int NWQ, bool HQ, int NWK, bool HK, int CNQ = 0, int CNK = 0>
__device__ __forceinline__ void gpair_stage_gamma(float4 *gq, float4 *gk, const float *gammaq, const float *gammak,
                                                  int P, int nvq, int nvk, int warp, int nwarps, int lane) {
    using SQ = GStage<Tag, NWQ, HQ, CNQ>;
    using SK = GStage<Tag, NWK, HK, CNK>;
    for (int p = warp; p < P; p += nwarps) {
        float4 vq[SQ::NL > 0 ? SQ::NL : 1], vk[SK::NL > 0 ? SK::NL : 1];
        SQ::load(vq, gammaq, p, nvq, lane);
        SK::load(vk, gammak, p, nvk, lane);
        SQ::store(gq, vq, P, p, lane);
        SK::store(gk, vk, P, p, lane);
    }
}

// Staging for the instances compiled for their shape (CP shards of CNQ and
// CNK vectors): a warp reads each of its shards' gamma in memory order, 32
// consecutive float4 per load (4 cache lines, where the lane-slot order above
// touches 16 with its 64-byte lane stride and so costs the L1 four times the
// cycles), all of its loads before any store, and each store puts a float4
// where the slot layout wants it. Warp w takes shards w, w + nwarps, ... (two
// in the mixed form, one in the separate). With COMB, Q's vectors after its
// whole slots and all of K's go to the combined half slots (see GComb).
// `mid` runs between the loads and the stores.
template <class Tag, int NWQ, bool HQ, int NWK, bool HK, bool MIX, int CP, int CNQ, int CNK, bool COMB, class Mid>
__device__ __forceinline__ void gpair_stage_rows(float4 *gq, float4 *gk, float4 *gcomb, const float *gammaq,
                                                 const float *gammak, int warp, int nwarps, int lane, Mid &&mid) {
    constexpr int C = Tag::kVec / 4;
    constexpr int NQ4 = CNQ * C, NK4 = CNK * C;              // float4 of one shard
    constexpr int LQ = (NQ4 + 31) / 32, LK = (NK4 + 31) / 32;  // per lane
    constexpr int HPW = MIX ? 2 : 1;                         // shards per warp
    using GQ = GSlots<Tag, NWQ, COMB ? false : HQ, COMB ? 0 : CNQ>;
    using GK = GSlots<Tag, NWK, HK, CNK>;
    float4 vq[HPW][LQ], vk[HPW][LK];
#pragma unroll
    for (int h = 0; h < HPW; ++h) {
        const int p = warp + h * nwarps;
        if (p < CP) {
            const float4 *sq = reinterpret_cast<const float4 *>(gammaq) + p * NQ4;
            const float4 *sk = reinterpret_cast<const float4 *>(gammak) + p * NK4;
#pragma unroll
            for (int m = 0; m < LQ; ++m)
                if (lane + 32 * m < NQ4) vq[h][m] = __ldg(sq + lane + 32 * m);
#pragma unroll
            for (int m = 0; m < LK; ++m)
                if (lane + 32 * m < NK4) vk[h][m] = __ldg(sk + lane + 32 * m);
        }
    }
    mid();
#pragma unroll
    for (int h = 0; h < HPW; ++h) {
        const int p = warp + h * nwarps;
        if (p < CP) {
#pragma unroll
            for (int m = 0; m < LQ; ++m) {
                const int g = lane + 32 * m, v = g / C, c = g % C;
                if (g >= NQ4) continue;
                if (COMB && v >= 32 * NWQ)   // combined slot: lane (v - 32 NWQ) + 8 x half, chunk c & 1
                    gcomb[(p * 2 + (c & 1)) * 32 + (v - 32 * NWQ) + 8 * (c >> 1)] = vq[h][m];
                else
                    gq[GQ::at(CP, p, v, c)] = vq[h][m];
            }
#pragma unroll
            for (int m = 0; m < LK; ++m) {
                const int g = lane + 32 * m, v = g / C, c = g % C;
                if (g >= NK4) continue;
                if (COMB)
                    gcomb[(p * 2 + (c & 1)) * 32 + 16 + v + 8 * (c >> 1)] = vk[h][m];
                else
                    gk[GK::at(CP, p, v, c)] = vk[h][m];
            }
        }
    }
}

// The lane's vectors of shards pa, pa + 1 of one tensor (row = the tensor's
// row in a ring stage, nv vectors per shard) and their two lane chains.
template <class Tag, int NW, bool H>
__device__ __forceinline__ void gpair_chains(const unsigned char *row, int nv, int pa, int lane,
                                             uint4 (&x)[2][NW > 0 ? NW : 1], uint2 (&hx)[2],
                                             float (&c)[2]) {
    static_assert(!H || Tag::kVec == 16, "half slots are defined for FP8 vectors only");
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 *sh = reinterpret_cast<const uint4 *>(row) + (pa + h) * nv;
        float ch = 0.f;
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            const int v = lane + 32 * i;
            x[h][i] = v < nv ? sh[v] : make_uint4(0, 0, 0, 0);
            ch = __fadd_rn(ch, vsumsq(Tag{}, x[h][i]));   // a missing vector adds +0
        }
        if constexpr (H) {
            const int hv = 32 * NW + (lane & 15);
            hx[h] = hv < nv ? *reinterpret_cast<const uint2 *>(reinterpret_cast<const unsigned char *>(sh + hv) +
                                                               8 * (lane >> 4))
                            : make_uint2(0, 0);
            const float hs = e4m3x8_sumsq(hx[h].x, hx[h].y);
            const float hi = __shfl_down_sync(kFull, hs, 16);
            if (lane < 16) ch = __fadd_rn(ch, __fadd_rn(hs, hi));
        }
        c[h] = ch;
    }
}

// (x * gamma) * r for the lane's vectors of shards pa, pa + 1 of one tensor,
// gamma from its staged layout g (P shards), written to the output row dst.
template <class Tag, int NW, bool H, int NV = 0>
__device__ __forceinline__ void gpair_apply(const uint4 (&x)[2][NW > 0 ? NW : 1], const uint2 (&hx)[2],
                                            const float4 *g, int P, uint4 *dst, int nv, int pa, int lane,
                                            float r) {
    using G = GSlots<Tag, NW, H, NV>;
    constexpr int VEC = Tag::kVec;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = pa + h;
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            const int v = lane + 32 * i;
            if (v < nv) {
                float gg[VEC];
#pragma unroll
                for (int c = 0; c < G::C; ++c) {
                    const float4 t = g[G::idx(p, i, c, lane)];
                    gg[4 * c] = t.x;
                    gg[4 * c + 1] = t.y;
                    gg[4 * c + 2] = t.z;
                    gg[4 * c + 3] = t.w;
                }
                st_stream(dst + p * nv + v, vapply_regs(Tag{}, x[h][i], gg, r));
            }
        }
        if constexpr (H) {
            const int hv = 32 * NW + (lane & 15);
            if (hv < nv) {
                float gh[VEC / 2];
                const float4 *gb = g + G::whole(P);
#pragma unroll
                for (int c = 0; c < G::CH; ++c) {
                    const float4 t = gb[G::hidx(p, c, lane)];
                    gh[4 * c] = t.x;
                    gh[4 * c + 1] = t.y;
                    gh[4 * c + 2] = t.z;
                    gh[4 * c + 3] = t.w;
                }
                const uint2 y = vapply_half(Tag{}, hx[h], gh, r);
                __stcs(reinterpret_cast<uint2 *>(reinterpret_cast<unsigned char *>(dst + p * nv + hv) +
                                                 8 * (lane >> 4)),
                       y);
            }
        }
    }
}

// Combined half slot (FP8, mixed, shapes compiled with a Q remainder of
// RQ <= 8 vectors after NWQ whole slots and K shards of RK <= 8 vectors):
// the last Q vectors and the K vectors of a shard share one 32-lane slot
// instead of a half-empty slot each. Lane l takes tensor l >> 4 (Q, K),
// half (l >> 3) & 1 of vector vv = l & 7 (Q: vector 32 NWQ + vv of the
// shard, K: vector vv); lanes l and l + 8 hold the two halves of a vector.
// The vector's sum is its halves' sums added (the FP8 vector sum's
// definition), formed in lane l; a K vector's sum then moves to lane vv,
// the lane that owns it in the shard's butterfly. Every addition has the
// operands it has in the half-slot form, so the bits are the same.
template <int NWQ, int CNQ, int CNK>
struct GComb {
    static constexpr int RQ = CNQ - 32 * NWQ, RK = CNK;
    __device__ __forceinline__ static bool valid(int lane) {
        return (lane >> 4) ? (lane & 7) < RK : (lane & 7) < RQ;
    }
    // Byte offset of the lane's half inside a row, shard p.
    __device__ __forceinline__ static int off(int p, int lane) {
        const int vv = lane & 7, hh = (lane >> 3) & 1;
        return (lane >> 4) ? (p * CNK + vv) * 16 + 8 * hh : (p * CNQ + 32 * NWQ + vv) * 16 + 8 * hh;
    }
};

// Gamma of the combined slots: per shard p, 2 float4 per lane at
// (p * 2 + c) * 32 + lane (all 32 lanes; zeros where a lane has no vector).
// When the warps take two shards each (P = 2 x warps), both shards' loads
// are issued before either's stores: one L2 round trip instead of two
// (measured at T = 4096: 12.53 -> 12.15 us per launch).
template <int NWQ, int CNQ, int CNK>
__device__ __forceinline__ void gpair_stage_comb(float4 *gq, float4 *gcomb, const float *gammaq, const float *gammak,
                                                 int P, int warp, int nwarps, int lane) {
    using CB = GComb<NWQ, CNQ, CNK>;
    using SQ = GStage<E4M3Tag, NWQ, false>;
    if (2 * nwarps == P) {
        const bool ok = CB::valid(lane);
        float4 vq[2][SQ::NL > 0 ? SQ::NL : 1];
        float4 c0[2], c1[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int p = warp + h * nwarps;
            SQ::load(vq[h], gammaq, p, CNQ, lane);
            const float *src = ((lane >> 4) ? gammak : gammaq) + CB::off(p, lane);   // 16 floats per vector
            c0[h] = ok ? __ldg(reinterpret_cast<const float4 *>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
            c1[h] = ok ? __ldg(reinterpret_cast<const float4 *>(src) + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int p = warp + h * nwarps;
            SQ::store(gq, vq[h], P, p, lane);
            gcomb[(p * 2 + 0) * 32 + lane] = c0[h];
            gcomb[(p * 2 + 1) * 32 + lane] = c1[h];
        }
        return;
    }
    for (int p = warp; p < P; p += nwarps) {
        float4 vq[SQ::NL > 0 ? SQ::NL : 1];
        SQ::load(vq, gammaq, p, CNQ, lane);
        const bool ok = CB::valid(lane);
        const float *src = ((lane >> 4) ? gammak : gammaq) + CB::off(p, lane);   // floats: 16 per vector = bytes
        const float4 c0 = ok ? __ldg(reinterpret_cast<const float4 *>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 c1 = ok ? __ldg(reinterpret_cast<const float4 *>(src) + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        SQ::store(gq, vq, P, p, lane);
        gcomb[(p * 2 + 0) * 32 + lane] = c0;
        gcomb[(p * 2 + 1) * 32 + lane] = c1;
    }
}

// The lane's vectors of Q shards pa, pa + 1 (whole slots) and its combined
// half of each shard; the Q and K lane chains of both shards.
template <int NWQ, int CNQ, int CNK>
__device__ __forceinline__ void gpair_chains_comb(const unsigned char *rowq, const unsigned char *rowk, int pa,
                                                  int lane, uint4 (&xq)[2][NWQ > 0 ? NWQ : 1], uint2 (&hx)[2],
                                                  float (&cq)[2], float (&ck)[2]) {
    using CB = GComb<NWQ, CNQ, CNK>;
    const bool ok = CB::valid(lane);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = pa + h;
        const uint4 *sh = reinterpret_cast<const uint4 *>(rowq) + p * CNQ;
        float ch = 0.f;
#pragma unroll
        for (int i = 0; i < NWQ; ++i) {
            xq[h][i] = sh[lane + 32 * i];
            ch = __fadd_rn(ch, vsumsq(E4M3Tag{}, xq[h][i]));
        }
        hx[h] = ok ? *reinterpret_cast<const uint2 *>(((lane >> 4) ? rowk : rowq) + CB::off(p, lane))
                   : make_uint2(0, 0);
        const float hf = e4m3x8_sumsq(hx[h].x, hx[h].y);
        const float vs = __fadd_rn(hf, __shfl_down_sync(kFull, hf, 8));   // half 0 + half 1 in lanes l & 8 == 0
        if (lane < CB::RQ) ch = __fadd_rn(ch, vs);
        const float kv = __shfl_sync(kFull, vs, (lane & 7) + 16);
        cq[h] = ch;
        ck[h] = lane < CB::RK ? kv : 0.f;
    }
}

// (x * gamma) * r for the combined halves of shards pa, pa + 1.
template <int NWQ, int CNQ, int CNK>
__device__ __forceinline__ void gpair_apply_comb(const uint2 (&hx)[2], const float4 *gcomb, unsigned char *yq,
                                                 unsigned char *yk, int pa, int lane, float rq, float rk) {
    using CB = GComb<NWQ, CNQ, CNK>;
    if (!CB::valid(lane)) return;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = pa + h;
        const float4 t0 = gcomb[(p * 2 + 0) * 32 + lane], t1 = gcomb[(p * 2 + 1) * 32 + lane];
        const float gh[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
        const uint2 y = vapply_half(E4M3Tag{}, hx[h], gh, (lane >> 4) ? rk : rq);
        __stcs(reinterpret_cast<uint2 *>(((lane >> 4) ? yk : yq) + CB::off(p, lane)), y);
    }
}

// The factor with the width fixed at compile time (W > 0): for a power of
// two, S * (1 / W) is the same correctly rounded number as S / W (the
// quotient is S scaled by a power of two), so the multiply replaces the
// division bit for bit; otherwise, or with W unknown, factor() as everywhere.
template <int W>
__device__ __forceinline__ float factor_w(float S, float Df, float eps) {
    if constexpr (W > 0 && (W & (W - 1)) == 0) return rsqrtf(__fadd_rn(__fmul_rn(S, 1.0f / W), eps));
    else return factor(S, Df, eps);
}

// Transposed butterflies (see the top comment). Two chains: lanes 0-15 end
// with shard 0's sum, lanes 16-31 with shard 1's.
__device__ __forceinline__ float butterfly_pair(float c0, float c1, int lane) {
    const bool lo = lane < 16;
    float v = __fadd_rn(lo ? c0 : c1, __shfl_xor_sync(kFull, lo ? c1 : c0, 16));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 8));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 4));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 2));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 1));
    return v;
}

// Four chains (a, b, c, d): lanes 0-7 end with a's sum, 8-15 b's, 16-23 c's,
// 24-31 d's.
__device__ __forceinline__ float butterfly_quad(float a, float b, float c, float d, int lane) {
    const bool lo = lane < 16;
    const float u0 = __fadd_rn(lo ? a : c, __shfl_xor_sync(kFull, lo ? c : a, 16));
    const float u1 = __fadd_rn(lo ? b : d, __shfl_xor_sync(kFull, lo ? d : b, 16));
    const bool l8 = (lane & 8) == 0;
    float v = __fadd_rn(l8 ? u0 : u1, __shfl_xor_sync(kFull, l8 ? u1 : u0, 8));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 4));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 2));
    v = __fadd_rn(v, __shfl_xor_sync(kFull, v, 1));
    return v;
}

// Separate form: NW whole slots (+ half slot H) per lane per shard for both
// tensors (their shards have the same vector count).
// Mixed form: Q with (NWQ, HQ), K with (NWK, HK), both in every warp.
constexpr int kGPairMaxThreads = 256;

// CP, CNQ, CNK: the shard count and the vectors per Q / K shard fixed at
// compile time for the shapes that have their own instance (0: read from the
// arguments). Fixed, every slot index, output offset and guard of a token
// folds to a constant; the arithmetic and its order are the same.
template <class Tag, int NWQ, bool HQ, int NWK, bool HK, bool MIX, int CP = 0, int CNQ = 0, int CNK = 0>
__global__ void __launch_bounds__(kGPairMaxThreads, 1) fused_gpair(const FusedArgs a, const GPairArgs b) {
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    float(*red)[64] = reinterpret_cast<float(*)[64]>(smem + kBarBytes);
    float4 *gq = reinterpret_cast<float4 *>(smem + kGPairGammaOff);
    float4 *gk = gq + b.gq4;
    unsigned char *stages = smem + b.stage_base;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int P = CP ? CP : a.P;
    const int halfP = P >> 1;
    const int z = MIX ? 0 : (warp < halfP ? 0 : 1);        // separate form: this warp's tensor
    const int pa = 2 * (MIX ? warp : (z ? warp - halfP : warp));
    const int nvq = CNQ ? CNQ : a.nv[0], nvk = CNK ? CNK : a.nv[1];
    const uint32_t tok_bytes = b.qbytes + b.kbytes;
    // The combined half slot (see GComb) for the FP8 GQA-shaped instance; its
    // gamma follows Q's whole slots, in the space of Q's and K's half slots.
    constexpr bool COMB = std::is_same<Tag, E4M3Tag>::value && MIX && HQ && HK && NWK == 0 && CNQ > 0 &&
                          CNK > 0 && CNQ - 32 * NWQ <= 8 && CNK <= 8;
    float4 *gcomb = gq + (int64_t)(CP > 0 ? CP : 1) * NWQ * (Tag::kVec / 4) * 32;

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

    const int64_t npass = (T - blockIdx.x + G - 1) / G;   // >= 1 since blockIdx.x < T
    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Shared memory only so far; global reads start after the previous grid.
    pdl_wait();
    pdl_trigger();
    auto first_issue = [&]() {
        if (tid == 0) {
            for (int s = 0; s < S && s < npass; ++s) issue(s, s);
        }
    };
    // Gamma of both tensors into shared memory (visible after the first
    // barrier). The compiled shapes issue their gamma loads before the first
    // stages' bulk copies: those are L2 hits, and behind the grid's burst of
    // row copies (every CTA's first stages at once) they waited about 2.8 us.
    if constexpr (CP > 0 && CNQ > 0 && CNK > 0) {
        gpair_stage_rows<Tag, NWQ, HQ, NWK, HK, MIX, CP, CNQ, CNK, COMB>(gq, gk, gcomb, a.g[0], a.g[1], warp,
                                                                       blockDim.x >> 5, lane, first_issue);
    } else {
        first_issue();
        if constexpr (COMB)
            gpair_stage_comb<NWQ, CNQ, CNK>(gq, gcomb, a.g[0], a.g[1], P, warp, blockDim.x >> 5, lane);
        else
            gpair_stage_gamma<Tag, NWQ, HQ, NWK, HK, CNQ, CNK>(gq, gk, a.g[0], a.g[1], P, nvq, nvk, warp,
                                                              blockDim.x >> 5, lane);
    }

    constexpr int AQ = NWQ > 0 ? NWQ : 1, AK = NWK > 0 ? NWK : 1;
    int s = 0;
    uint32_t phase = 0;
    int buf = 0;
    for (int64_t n = 0; n < npass; ++n) {
        const int64_t t = blockIdx.x + n * G;
        const bool ok = mbar_wait_bounded(&full[s], phase, b.timeout_ns);
        const unsigned char *st = stages + (size_t)s * b.stage_stride;
        uint4 xq[2][AQ], xk[2][AK];
        uint2 hq[2], hk[2];
        float cq[2], ck[2];
        if constexpr (COMB) {
            gpair_chains_comb<NWQ, CNQ, CNK>(st, st + b.qbytes, pa, lane, xq, hq, cq, ck);
            const float v = butterfly_quad(cq[0], cq[1], ck[0], ck[1], lane);
            if ((lane & 7) == 0) red[buf][32 * (lane >> 4) + pa + ((lane >> 3) & 1)] = v;
        } else if constexpr (MIX) {
            gpair_chains<Tag, NWQ, HQ>(st, nvq, pa, lane, xq, hq, cq);
            gpair_chains<Tag, NWK, HK>(st + b.qbytes, nvk, pa, lane, xk, hk, ck);
            const float v = butterfly_quad(cq[0], cq[1], ck[0], ck[1], lane);
            if ((lane & 7) == 0) red[buf][32 * (lane >> 4) + pa + ((lane >> 3) & 1)] = v;
        } else {
            gpair_chains<Tag, NWQ, HQ>(st + (z ? b.qbytes : 0u), z ? nvk : nvq, pa, lane, xq, hq, cq);
            const float v = butterfly_pair(cq[0], cq[1], lane);
            if ((lane & 15) == 0) red[buf][32 * z + pa + (lane >> 4)] = v;
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
        // Phase B: shard sums in order of p, the factor; weight multiply and Phase C.
        if constexpr (COMB) {
            const float rq = factor_w<CP * CNQ * Tag::kVec>(combine_fast(&red[buf][0], P, 1), a.Df[0], a.eps);
            const float rk = factor_w<CP * CNK * Tag::kVec>(combine_fast(&red[buf][32], P, 1), a.Df[1], a.eps);
            uint2 hdummy[2] = {make_uint2(0, 0), make_uint2(0, 0)};
            gpair_apply<Tag, NWQ, false>(xq, hdummy, gq, P, reinterpret_cast<uint4 *>(a.y[0]) + t * a.ldy[0], nvq,
                                         pa, lane, rq);
            gpair_apply_comb<NWQ, CNQ, CNK>(hq, gcomb, reinterpret_cast<unsigned char *>(a.y[0]) + t * a.ldy[0] * 16,
                                            reinterpret_cast<unsigned char *>(a.y[1]) + t * a.ldy[1] * 16, pa, lane,
                                            rq, rk);
        } else if constexpr (MIX) {
            const float rq = factor_w<CP * CNQ * Tag::kVec>(combine_fast(&red[buf][0], P, 1), a.Df[0], a.eps);
            const float rk = factor_w<CP * CNK * Tag::kVec>(combine_fast(&red[buf][32], P, 1), a.Df[1], a.eps);
            gpair_apply<Tag, NWQ, HQ, CNQ>(xq, hq, gq, P, reinterpret_cast<uint4 *>(a.y[0]) + t * a.ldy[0], nvq,
                                           pa, lane, rq);
            gpair_apply<Tag, NWK, HK, CNK>(xk, hk, gk, P, reinterpret_cast<uint4 *>(a.y[1]) + t * a.ldy[1], nvk,
                                           pa, lane, rk);
        } else {
            const float r = factor(combine_fast(&red[buf][32 * z], P, 1), z ? a.Df[1] : a.Df[0], a.eps);
            gpair_apply<Tag, NWQ, HQ, CNQ>(xq, hq, z ? gk : gq, P,
                                      reinterpret_cast<uint4 *>(z ? a.y[1] : a.y[0]) + t * (z ? a.ldy[1] : a.ldy[0]),
                                      z ? nvk : nvq, pa, lane, r);
        }
        buf ^= 1;
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }
    }
}

// ---------------------------------------------------------------- instances and launch

// (NWQ, HQ, NWK, HK, MIX) of the instances that exist, per dtype:
//   FP8 separate: (2, half) -- e.g. D = 5120 in 4 shards; (1) -- D = 4096 in 8;
//                 (2) -- D = 4096 in 4;
//   FP8 mixed:    Q (1, half), K (0, half) -- e.g. Dq = 5120, Dk = 1024 in 8;
//   bf16 mixed:   Q (3), K (1) -- the same GQA widths in bf16.
template <class Tag, int NWQ, bool HQ, int NWK, bool HK, bool MIX, int CP = 0, int CNQ = 0, int CNK = 0>
const void *gpair_fn() {
    return reinterpret_cast<const void *>(&fused_gpair<Tag, NWQ, HQ, NWK, HK, MIX, CP, CNQ, CNK>);
}

const void *fused_gpair_kernel(int dtype, int nwq, bool hq, int nwk, bool hk, bool mix) {
    if (dtype == 2) {
        if (!mix && nwq == nwk && hq == hk) {
            if (nwq == 2 && hq) return gpair_fn<E4M3Tag, 2, true, 2, true, false>();
            if (nwq == 1 && !hq) return gpair_fn<E4M3Tag, 1, false, 1, false, false>();
            if (nwq == 2 && !hq) return gpair_fn<E4M3Tag, 2, false, 2, false, false>();
        }
        if (mix && nwq == 1 && hq && nwk == 0 && hk) return gpair_fn<E4M3Tag, 1, true, 0, true, true>();
    }
    if (dtype == 1) {
        if (mix && nwq == 3 && !hq && nwk == 1 && !hk) return gpair_fn<BF16Tag, 3, false, 1, false, true>();
    }
    return nullptr;
}

// The instance for this exact shape where one exists (P shards of nvq and
// nvk vectors, compiled with them as constants), else the general one:
//   FP8 13B-shaped, D = 5120 in 4 shards (80 vectors each);
//   FP8 GQA-shaped, Dq = 5120, Dk = 1024 in 8 shards (40 and 8 vectors);
//   bf16 GQA-shaped, the same widths (80 and 16 vectors).
const void *fused_gpair_kernel_for(int dtype, int nwq, bool hq, int nwk, bool hk, bool mix, int P, int nvq,
                                   int nvk) {
    const void *gen = fused_gpair_kernel(dtype, nwq, hq, nwk, hk, mix);
    if (!gen) return nullptr;
    if (dtype == 2 && !mix && nwq == 2 && hq && P == 4 && nvq == 80 && nvk == 80)
        return gpair_fn<E4M3Tag, 2, true, 2, true, false, 4, 80, 80>();
    if (dtype == 2 && mix && nwq == 1 && hq && nwk == 0 && hk && P == 8 && nvq == 40 && nvk == 8)
        return gpair_fn<E4M3Tag, 1, true, 0, true, true, 8, 40, 8>();
    if (dtype == 1 && mix && nwq == 3 && !hq && nwk == 1 && !hk && P == 8 && nvq == 80 && nvk == 16)
        return gpair_fn<BF16Tag, 3, false, 1, false, true, 8, 80, 16>();
    return gen;
}

// Slots per lane of one tensor: whole slots, and whether the last (at most
// 16 vectors) is split in halves (FP8 only); a ragged last slot of more than
// 16 vectors is a guarded whole slot.
void gpair_slots(int nv, int dtype, int *nw, bool *h) {
    *nw = nv / 32;
    const int rem = nv - 32 * *nw;
    *h = false;
    if (rem == 0) return;
    if (dtype == 2 && rem <= 16) {
        *h = true;
        return;
    }
    *nw += 1;
}

// Float4 slots of one tensor's staged gamma (GSlots::total): compact (nv
// vectors per shard exactly) for an instance compiled for the shape without
// a half slot, else 32 lanes per slot.
int64_t gpair_gamma_slots(int dtype, int P, int nw, bool h, int nv, bool compiled) {
    const int C = (dtype == 1 ? 8 : (dtype == 2 ? 16 : 4)) / 4;
    const int64_t whole = compiled && !h ? (int64_t)P * nv * C : (int64_t)P * nw * C * 32;
    const int64_t R = compiled && h ? nv - 32 * nw : 16;   // vectors in the half slot
    return whole + (h ? (int64_t)P * (C / 2) * 2 * R : 0);
}

size_t gpair_smem_bytes(int dtype, int P, int nwq, bool hq, int nwk, bool hk, int nvq, int nvk, int stages,
                        int64_t qbytes, int64_t kbytes, uint32_t *stage_base, uint32_t *gq4,
                        uint32_t *gk4, uint32_t *stride) {
    const bool mix = nvq != nvk;
    const bool compiled = fused_gpair_kernel_for(dtype, nwq, hq, nwk, hk, mix, P, nvq, nvk) !=
                          fused_gpair_kernel(dtype, nwq, hq, nwk, hk, mix);
    const int64_t q4 = gpair_gamma_slots(dtype, P, nwq, hq, nvq, compiled),
                  k4 = gpair_gamma_slots(dtype, P, nwk, hk, nvk, compiled);
    const int64_t base = ((int64_t)kGPairGammaOff + 16 * (q4 + k4) + 127) / 128 * 128;
    const uint32_t st = bulk_stage_stride(qbytes, kbytes, 1);
    if (stage_base) *stage_base = (uint32_t)base;
    if (gq4) *gq4 = (uint32_t)q4;
    if (gk4) *gk4 = (uint32_t)k4;
    if (stride) *stride = st;
    return (size_t)base + (size_t)stages * st;
}

int gpair_max_threads() { return kGPairMaxThreads; }

cudaError_t launch_fused_gpair(int dtype, int nwq, bool hq, int nwk, bool hk, bool mix,
                               const FusedArgs &a, int stages, int64_t grid, uint64_t timeout_ns,
                               cudaStream_t s) {
    const void *fn = fused_gpair_kernel_for(dtype, nwq, hq, nwk, hk, mix, a.P, a.nv[0], a.nv[1]);
    if (!fn || stages < 1 || stages > (int)kMaxStages || (a.P & 1) || a.P > 32 || a.K[0] != 1 ||
        a.K[1] != 1)
        return cudaErrorInvalidValue;
    // The slots must cover every shard exactly as planned.
    int w;
    bool h;
    gpair_slots(a.nv[0], dtype, &w, &h);
    if (w != nwq || h != hq) return cudaErrorInvalidValue;
    gpair_slots(a.nv[1], dtype, &w, &h);
    if (w != nwk || h != hk) return cudaErrorInvalidValue;
    const int block = 32 * (mix ? a.P / 2 : a.P);
    if (block > kGPairMaxThreads) return cudaErrorInvalidValue;
    const int64_t es = dtype == 1 ? 2 : (dtype == 2 ? 1 : 4);
    GPairArgs b;
    b.stages = (uint32_t)stages;
    b.qbytes = (uint32_t)(a.D[0] * es);
    b.kbytes = (uint32_t)(a.D[1] * es);
    b.timeout_ns = timeout_ns;
    const size_t smem = gpair_smem_bytes(dtype, a.P, nwq, hq, nwk, hk, a.nv[0], a.nv[1], stages, b.qbytes,
                                         b.kbytes, &b.stage_base, &b.gq4, &b.gk4, &b.stage_stride);
    void *args[] = {const_cast<FusedArgs *>(&a), &b};
    return launch(fn, dim3((unsigned)grid), dim3(block), smem, s, args);
}

}  // namespace qkn
