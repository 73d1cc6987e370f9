// qknorm_device.cuh -- device building blocks shared by every kernel of
// libqknorm: 16-byte vector loads and stores, the per-vector sum of squares,
// the lane butterfly, the shard combine, the factor and the apply step.
//
// Every kernel builds its sums from these functions in the same order (the
// order stated in include/qknorm.h), which is why qknorm_fwd and the split
// path (qknorm_partial_sumsq + qknorm_apply) give bit-identical outputs.
// All floating-point steps use explicitly rounded intrinsics so that the
// compiler cannot contract or reorder them differently in different kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qkn {

constexpr int kLanes = 32;
constexpr int kVcap = 8;  // 16-byte vectors per lane per group; fixes K = ceil(nv / 256)
constexpr unsigned kFull = 0xffffffffu;

struct F32Tag {
    static constexpr int kVec = 4;  // fp32 values per 16-byte vector
    static constexpr int kBytes = 4;
};
struct BF16Tag {
    static constexpr int kVec = 8;  // bf16 values per 16-byte vector
    static constexpr int kBytes = 2;
};
struct E4M3Tag {
    static constexpr int kVec = 16;  // FP8 E4M3 values per 16-byte vector
    static constexpr int kBytes = 1;
};

// ---------------------------------------------------------------- widening

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two FP8 E4M3 values (the low byte first) widened exactly to fp32.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// The 16 values of a 16-byte FP8 vector as 8 float pairs, element 0 first.
__device__ __forceinline__ void e4m3x16_to_float(const uint4 &v, float (&f)[16]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = e4m3x2_to_float2(w[i]);
        const float2 b = e4m3x2_to_float2(w[i] >> 16);
        f[4 * i] = a.x;
        f[4 * i + 1] = a.y;
        f[4 * i + 2] = b.x;
        f[4 * i + 3] = b.y;
    }
}

// Two fp32 values to FP8 E4M3 (round to nearest even, saturating to +-448),
// the first in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

// Two fp32 products rounded to nearest even, as one packed sm_100 f32x2
// multiply (each lane is exactly __fmul_rn of its operands).
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b) { return __fmul2_rn(a, b); }

// ---------------------------------------------------------------- Phase A: x^2

// Sum of squares of one vector: e0*e0, then e_i*e_i + q fused, i = 1..3.
__device__ __forceinline__ float vsumsq(F32Tag, const uint4 &v) {
    const float e0 = __uint_as_float(v.x), e1 = __uint_as_float(v.y);
    const float e2 = __uint_as_float(v.z), e3 = __uint_as_float(v.w);
    float q = __fmul_rn(e0, e0);
    q = __fmaf_rn(e1, e1, q);
    q = __fmaf_rn(e2, e2, q);
    q = __fmaf_rn(e3, e3, q);
    return q;
}

// Same for 8 bf16 values; element 0 is the low half of v.x.
// (A bf16 square is exact in fp32, so each fma rounds only the running sum.)
__device__ __forceinline__ float vsumsq(BF16Tag, const uint4 &v) {
    float q = __fmul_rn(bf_lo(v.x), bf_lo(v.x));
    q = __fmaf_rn(bf_hi(v.x), bf_hi(v.x), q);
    q = __fmaf_rn(bf_lo(v.y), bf_lo(v.y), q);
    q = __fmaf_rn(bf_hi(v.y), bf_hi(v.y), q);
    q = __fmaf_rn(bf_lo(v.z), bf_lo(v.z), q);
    q = __fmaf_rn(bf_hi(v.z), bf_hi(v.z), q);
    q = __fmaf_rn(bf_lo(v.w), bf_lo(v.w), q);
    q = __fmaf_rn(bf_hi(v.w), bf_hi(v.w), q);
    return q;
}

// The 8 FP8 values of half a vector (w0, w1; element 0 in the low byte of
// w0), as two interleaved chains over its element pairs (e0,e1), (e2,e3),
// (e4,e5), (e6,e7): the even elements' squares summed in order in one fp32
// chain and the odd elements' in the other (e0*e0, then e2*e2 + q fused, ...;
// e1*e1, then e3*e3 + q fused, ...), each step of the two chains one packed
// f32x2 fused multiply-add; then even sum + odd sum. An E4M3 square is exact
// in fp32, so each step rounds only the running sums.
__device__ __forceinline__ float e4m3x8_sumsq(uint32_t w0, uint32_t w1) {
    const float2 a = e4m3x2_to_float2(w0), b = e4m3x2_to_float2(w0 >> 16);
    const float2 c = e4m3x2_to_float2(w1), d = e4m3x2_to_float2(w1 >> 16);
    float2 q = __fmul2_rn(a, a);
    q = __ffma2_rn(b, b, q);
    q = __ffma2_rn(c, c, q);
    q = __ffma2_rn(d, d, q);
    return __fadd_rn(q.x, q.y);
}

// Same for 16 FP8 values: the sums of the two halves (elements 0-7, 8-15),
// each as above, then added. A half vector is a unit the bulk kernel can hand
// to another lane.
__device__ __forceinline__ float vsumsq(E4M3Tag, const uint4 &v) {
    return __fadd_rn(e4m3x8_sumsq(v.x, v.y), e4m3x8_sumsq(v.z, v.w));
}

// xor butterfly over the 32 lanes; every lane ends with the same bits
// (fp32 addition is commutative, so both partners of a pair agree).
__device__ __forceinline__ float butterfly(float c) {
    c = __fadd_rn(c, __shfl_xor_sync(kFull, c, 16));
    c = __fadd_rn(c, __shfl_xor_sync(kFull, c, 8));
    c = __fadd_rn(c, __shfl_xor_sync(kFull, c, 4));
    c = __fadd_rn(c, __shfl_xor_sync(kFull, c, 2));
    c = __fadd_rn(c, __shfl_xor_sync(kFull, c, 1));
    return c;
}

// ---------------------------------------------------------------- Phase B: combine, factor

// S = sum over p (in order) of S_p, S_p = sum over k (in order) of B[p*K + k].
__device__ __forceinline__ float combine(const float *B, int P, int K) {
    float S = 0.f;
    for (int p = 0; p < P; ++p) {
        float Sp = 0.f;
        for (int k = 0; k < K; ++k) Sp = __fadd_rn(Sp, B[p * K + k]);
        S = __fadd_rn(S, Sp);
    }
    return S;
}

// combine() with the common single-group shards (K = 1) as one short loop:
// the same additions in the same order (0 + B[p] is exact), fewer branches.
__device__ __forceinline__ float combine_fast(const float *B, int P, int K) {
    if (K != 1) return combine(B, P, K);
    float S = 0.f;
#pragma unroll 4
    for (int p = 0; p < P; ++p) S = __fadd_rn(S, B[p]);
    return S;
}

// r = rsqrt(S / D + eps): the global RMS factor with the full width D.
__device__ __forceinline__ float factor(float S, float Df, float eps) {
    return rsqrtf(__fadd_rn(__fdiv_rn(S, Df), eps));
}

// ---------------------------------------------------------------- Phase B weight, Phase C

__device__ __forceinline__ float wmul(float x, float g, float r) {
    return __fmul_rn(__fmul_rn(x, g), r);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// (x * gamma) * r for two values at once: two packed f32x2 multiplies, each
// lane rounded exactly as wmul's two __fmul_rn (so the bits are wmul's).
__device__ __forceinline__ float2 wmul2(float2 x, float2 g, float2 rr) {
    return fmul2_rn(fmul2_rn(x, g), rr);
}

__device__ __forceinline__ uint4 vapply_regs(F32Tag, const uint4 &v, const float *g, float r);
__device__ __forceinline__ uint4 vapply_regs(BF16Tag, const uint4 &v, const float *g, float r);

// y = (x * gamma) * r for one vector; g points at the vector's gamma (fp32).
__device__ __forceinline__ uint4 vapply(F32Tag, const uint4 &v, const float *g, float r) {
    const float4 g4 = __ldg(reinterpret_cast<const float4 *>(g));
    const float gg[4] = {g4.x, g4.y, g4.z, g4.w};
    return vapply_regs(F32Tag{}, v, gg, r);
}

__device__ __forceinline__ uint4 vapply(BF16Tag, const uint4 &v, const float *g, float r) {
    const float4 ga = __ldg(reinterpret_cast<const float4 *>(g));
    const float4 gb = __ldg(reinterpret_cast<const float4 *>(g) + 1);
    const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    return vapply_regs(BF16Tag{}, v, gg, r);
}

__device__ __forceinline__ uint4 vapply_regs(E4M3Tag, const uint4 &v, const float *g, float r);

__device__ __forceinline__ uint4 vapply(E4M3Tag, const uint4 &v, const float *g, float r) {
    float gg[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 g4 = __ldg(reinterpret_cast<const float4 *>(g) + i);
        gg[4 * i] = g4.x;
        gg[4 * i + 1] = g4.y;
        gg[4 * i + 2] = g4.z;
        gg[4 * i + 3] = g4.w;
    }
    return vapply_regs(E4M3Tag{}, v, gg, r);
}

// Same as vapply with gamma already in registers (g[0..vec-1], indexed with
// compile-time constants after unrolling).
__device__ __forceinline__ uint4 vapply_regs(F32Tag, const uint4 &v, const float *g, float r) {
    const float2 rr = make_float2(r, r);
    const float2 a = wmul2(make_float2(__uint_as_float(v.x), __uint_as_float(v.y)), make_float2(g[0], g[1]), rr);
    const float2 b = wmul2(make_float2(__uint_as_float(v.z), __uint_as_float(v.w)), make_float2(g[2], g[3]), rr);
    return make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
}

// FP8, half a vector (8 values, gamma g[0..7]): the two multiplies of each
// pair of values as packed f32x2 multiplies (the same roundings as wmul),
// which halves their issue slots.
__device__ __forceinline__ uint2 vapply_half_regs(E4M3Tag, uint32_t w0, uint32_t w1, const float *g,
                                                  float r) {
    const uint32_t w[2] = {w0, w1};
    const float2 rr = make_float2(r, r);
    uint32_t o[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float2 x01 = e4m3x2_to_float2(w[i]);
        const float2 x23 = e4m3x2_to_float2(w[i] >> 16);
        const float2 y01 = wmul2(x01, make_float2(g[4 * i], g[4 * i + 1]), rr);
        const float2 y23 = wmul2(x23, make_float2(g[4 * i + 2], g[4 * i + 3]), rr);
        o[i] = pack_e4m3x2(y01.x, y01.y) | (pack_e4m3x2(y23.x, y23.y) << 16);
    }
    return make_uint2(o[0], o[1]);
}

__device__ __forceinline__ uint2 vapply_half(E4M3Tag, const uint2 &h, const float *g, float r) {
    return vapply_half_regs(E4M3Tag{}, h.x, h.y, g, r);
}

__device__ __forceinline__ uint4 vapply_regs(E4M3Tag, const uint4 &v, const float *g, float r) {
    const uint2 lo = vapply_half_regs(E4M3Tag{}, v.x, v.y, g, r);
    const uint2 hi = vapply_half_regs(E4M3Tag{}, v.z, v.w, g + 8, r);
    return make_uint4(lo.x, lo.y, hi.x, hi.y);
}

__device__ __forceinline__ uint4 vapply_regs(BF16Tag, const uint4 &v, const float *g, float r) {
    const float2 rr = make_float2(r, r);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 y = wmul2(make_float2(bf_lo(w[i]), bf_hi(w[i])), make_float2(g[2 * i], g[2 * i + 1]), rr);
        o[i] = pack_bf16x2(y.x, y.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// u = x * gamma for one vector, rounded to the storage type (no factor);
// packed f32x2 multiplies, each lane exactly __fmul_rn.
__device__ __forceinline__ uint4 vxgamma(F32Tag, const uint4 &v, const float *g) {
    const float4 g4 = __ldg(reinterpret_cast<const float4 *>(g));
    const float2 a = fmul2_rn(make_float2(__uint_as_float(v.x), __uint_as_float(v.y)), make_float2(g4.x, g4.y));
    const float2 b = fmul2_rn(make_float2(__uint_as_float(v.z), __uint_as_float(v.w)), make_float2(g4.z, g4.w));
    return make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
}

__device__ __forceinline__ uint4 vxgamma(BF16Tag, const uint4 &v, const float *g) {
    const float4 ga = __ldg(reinterpret_cast<const float4 *>(g));
    const float4 gb = __ldg(reinterpret_cast<const float4 *>(g) + 1);
    const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 y = fmul2_rn(make_float2(bf_lo(w[i]), bf_hi(w[i])), make_float2(gg[2 * i], gg[2 * i + 1]));
        o[i] = pack_bf16x2(y.x, y.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 vxgamma(E4M3Tag, const uint4 &v, const float *g) {
    float f[16], gg[16];
    e4m3x16_to_float(v, f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 g4 = __ldg(reinterpret_cast<const float4 *>(g) + i);
        gg[4 * i] = g4.x;
        gg[4 * i + 1] = g4.y;
        gg[4 * i + 2] = g4.z;
        gg[4 * i + 3] = g4.w;
    }
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = pack_e4m3x2(__fmul_rn(f[4 * i], gg[4 * i]), __fmul_rn(f[4 * i + 1], gg[4 * i + 1])) |
               (pack_e4m3x2(__fmul_rn(f[4 * i + 2], gg[4 * i + 2]), __fmul_rn(f[4 * i + 3], gg[4 * i + 3])) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Same as vapply with gamma read through an arbitrary pointer (used with
// gamma staged in shared memory); same arithmetic, bit for bit.
__device__ __forceinline__ uint4 vapply_ptr(F32Tag, const uint4 &v, const float *g, float r) {
    const float4 g4 = *reinterpret_cast<const float4 *>(g);
    const float gg[4] = {g4.x, g4.y, g4.z, g4.w};
    return vapply_regs(F32Tag{}, v, gg, r);
}

__device__ __forceinline__ uint4 vapply_ptr(BF16Tag, const uint4 &v, const float *g, float r) {
    const float4 ga = *reinterpret_cast<const float4 *>(g);
    const float4 gb = *(reinterpret_cast<const float4 *>(g) + 1);
    const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    return vapply_regs(BF16Tag{}, v, gg, r);
}

// ---------------------------------------------------------------- launch order

// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialization attribute may start while the previous kernel in the
// stream is still running. pdl_wait() blocks until that kernel has completed
// and its memory is visible; every kernel here calls it before its first
// global-memory access (and it returns at once when there is nothing to wait
// for). pdl_trigger() lets the next such kernel in the stream launch now; its
// own pdl_wait() still orders its memory accesses after this kernel's.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::); }

__device__ __forceinline__ uint4 vapply_ptr(E4M3Tag, const uint4 &v, const float *g, float r) {
    float gg[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 g4 = *(reinterpret_cast<const float4 *>(g) + i);
        gg[4 * i] = g4.x;
        gg[4 * i + 1] = g4.y;
        gg[4 * i + 2] = g4.z;
        gg[4 * i + 3] = g4.w;
    }
    return vapply_regs(E4M3Tag{}, v, gg, r);
}

// ---------------------------------------------------------------- memory

// Streaming (read-once / write-once) 16-byte accesses: evict-first in L1/L2.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(uint4 *p, const uint4 &v) { __stcs(p, v); }

// Number of vectors lane `first` of a group holds: v = first + stride*i < nv.
__device__ __forceinline__ int slot_count(int first, int nv, int stride) {
    return first < nv ? (nv - first + stride - 1) / stride : 0;
}

}  // namespace qkn
