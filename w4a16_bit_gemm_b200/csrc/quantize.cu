// quantize.cu -- group-wise RTN quantize+pack and dequantize kernels (sm_100a).
//
// Quantize ("Affine Quantization", "Symmetric and Asymmetric", "Per-group"
// sections of "LLM Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)"):
// per group of g consecutive input-channel weights, x_min' = min(0, min x),
// x_max' = max(0, max x) (asymmetric) or amax = max|x| (symmetric);
// s = fp16_rn((x_max' - x_min') / 15) or fp16_rn(amax / 7);
// z = clamp(rint(-x_min'/s), 0, 15); q = clamp(rint(x/s) + z, q_min, q_max).
//
// Data layout: the weights are a flat row-major array, so group gi covers the
// elements [gi*g, (gi+1)*g) and its scale/zero live at index gi; packed word w
// holds elements [8w, 8w+8).  A "segment" is 8 consecutive weights = one
// 16-byte load and one packed output word.  For g <= 256 one group spans
// L = g/8 lanes of a warp; the min/max is a butterfly shuffle over those
// lanes.  For larger g one warp owns a group and loops over it twice.
// All loads/stores are 128-bit (input) and 32-bit (packed output), fully
// coalesced: consecutive lanes touch consecutive addresses.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

constexpr uint32_t kFlagNonfinite = 0x1u;
constexpr uint32_t kFlagRange = 0x2u;

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float f[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

struct ScaleZero {
    uint16_t s16;
    int z;
    bool range;
};

// Scale and zero point from the (already reduced) statistics.
__device__ __forceinline__ ScaleZero scale_zero(float lo, float hi, bool symmetric) {
    // lo <= 0 <= hi (range widened to contain zero)
    float s32;
    if (symmetric) {
        float amax = fmaxf(-lo, hi);
        s32 = __fdiv_rn(amax, 7.0f);
    } else {
        s32 = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
    }
    ScaleZero r;
    r.s16 = __half_as_ushort(__float2half_rn(s32));
    r.range = false;
    r.z = 0;
    if (r.s16 == 0x7c00u) {  // fp16 overflow: saturate
        r.s16 = 0x7bffu;
        r.range = true;
    }
    if (r.s16 == 0u) {  // all-zero or underflowing group
        r.s16 = 0x3c00u;
    } else if (!symmetric) {
        float s = __half2float(__ushort_as_half(r.s16));
        float zf = rintf(__fsub_rn(0.0f, __fdiv_rn(lo, s)));
        zf = fminf(fmaxf(zf, 0.0f), 15.0f);
        r.z = (int)zf;
    }
    return r;
}

// rcp.approx.f32: at most 1 ulp from 1/s.
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

// rint(fl32(-lo / s)) with the IEEE division (rare: near a half-integer).
__device__ __noinline__ float exact_neg_quotient_rint(float lo, float s) {
    return rintf(__fsub_rn(0.0f, __fdiv_rn(lo, s)));
}

// scale_zero without fp32 divisions on the common path.
//  - fl32(r / 15) (or / 7) equals fl32(fl64(r) * fl64(1/15)): r has 24
//    significant bits, so a quotient that is not exact lies at least 2^-29
//    (relative) away from every fp32 rounding midpoint, while the fp64
//    product is within 2^-52 of the quotient (correct rounding of the
//    quotient is preserved).
//  - z = rint(fl32(-lo / s)) through f = -lo * rcp(s) with the quotient
//    guard of rint_quotient (the exact division decides near a half-integer).
// Also returns rcp(s) for the code path.
__device__ __forceinline__ ScaleZero scale_zero_fast(float lo, float hi, bool symmetric, float& rcp_out) {
    float s32;
    if (symmetric)
        s32 = __double2float_rn((double)fmaxf(-lo, hi) * (1.0 / 7.0));
    else
        s32 = __double2float_rn((double)__fsub_rn(hi, lo) * (1.0 / 15.0));
    ScaleZero r;
    r.s16 = __half_as_ushort(__float2half_rn(s32));
    r.range = false;
    r.z = 0;
    if (r.s16 == 0x7c00u) {  // fp16 overflow: saturate
        r.s16 = 0x7bffu;
        r.range = true;
    }
    if (r.s16 == 0u) r.s16 = 0x3c00u;  // all-zero or underflowing group
    const float s = __half2float(__ushort_as_half(r.s16));
    const float rcp = rcp_approx(s);
    rcp_out = rcp;
    if (!symmetric && lo != 0.0f) {
        const float f = __fmul_rn(-lo, rcp);
        float t = rintf(f);
        if (fabsf(f) < 32.0f && fabsf(__fsub_rn(f, t)) > 0.5f - 0x1p-17f) t = exact_neg_quotient_rint(lo, s);
        r.z = (int)fminf(fmaxf(t, 0.0f), 15.0f);
    }
    return r;
}

// rint(x / s) for the IEEE-rounded quotient, without a division on the fast
// path.  f = x * rcp_rn(s) differs from x/s by at most (2^-23 + 2^-48)|x/s|
// and the rounded quotient fl(x/s) by at most 2^-24|x/s|, so for |f| < 32
// the two lie within 3 * 2^-24 * 32 < 2^-17 of each other: when f is more
// than 2^-17 away from the nearest half-integer both round to the same
// integer.  Otherwise the exact IEEE division decides.  For |f| >= 32 the
// code is clamped to the same end of the range either way (|q - z| <= 15).
__device__ __forceinline__ float rint_quotient(float x, float s, float rcp) {
    const float f = __fmul_rn(x, rcp);
    float t = rintf(f);
    if (fabsf(f) < 32.0f && fabsf(__fsub_rn(f, t)) > 0.5f - 0x1p-17f) t = rintf(__fdiv_rn(x, s));
    return t;
}

// Codes of 8 weights packed into one word (low nibble first).
__device__ __noinline__ uint32_t encode8_slow(const uint4 raw, const ScaleZero sz, bool symmetric);

__device__ __forceinline__ uint32_t encode8(const float v[8], const ScaleZero& sz, bool symmetric) {
    const float s = __half2float(__ushort_as_half(sz.s16));
    const float rcp = __frcp_rn(s);
    const float qmin = symmetric ? -8.0f : 0.0f;
    const float qmax = symmetric ? 7.0f : 15.0f;
    const float zf = (float)sz.z;
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int q;
        if (isnan(v[i])) {
            q = sz.z;
        } else {
            const float t = rint_quotient(v[i], s, rcp);
            const float c = fminf(fmaxf(__fadd_rn(t, zf), qmin), qmax);
            q = (int)c;
        }
        word |= ((uint32_t)q & 0xfu) << (4 * i);
    }
    return word;
}

constexpr int kQuantThreads = 256;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// Statistics of 32 values skipping NaN (rare: only threads that hold a NaN).
__device__ __noinline__ float2 nan_skipping_min_max(const uint4 r0, const uint4 r1, const uint4 r2, const uint4 r3) {
    const uint4 rr[4] = {r0, r1, r2, r3};
    float lo = 0.0f, hi = 0.0f;
    for (int v = 0; v < 4; ++v) {
        float f[8];
        unpack_bf16x8(rr[v], f);
        for (int i = 0; i < 8; ++i) {
            lo = fminf(lo, f[i]);
            hi = fmaxf(hi, f[i]);
        }
    }
    return make_float2(lo, hi);
}

// Offset codes (q + z, or q + 8 when symmetric) of 16 packed bf16 pairs through
// f = x * rcp and the rounding constant; dmax collects |f - rint(f)|.
template <bool CLAMP>
__device__ __forceinline__ void fast_codes(const uint32_t (&w)[16], float rcp, uint32_t coff, bool sym,
                                           uint32_t (&word)[4], float& dmax) {
    const float2 rcp2 = make_float2(rcp, rcp);
    const float2 mag2 = make_float2(kRoundMagic, kRoundMagic);
    const float2 nmag2 = make_float2(-kRoundMagic, -kRoundMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    float dm0 = 0.0f, dm1 = 0.0f;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t wv = w[4 * h + i];
            const float2 x2 = make_float2(__uint_as_float(wv << 16), __uint_as_float(wv & 0xffff0000u));
            const float2 f2 = __fmul2_rn(x2, rcp2);
            const float2 t2 = __fadd2_rn(f2, mag2);
            const float2 r2 = __fadd2_rn(t2, nmag2);    // rint(f), exact
            const float2 d2 = __ffma2_rn(r2, neg1, f2);  // f - rint(f), exact
            dm0 = fmaxf(dm0, fabsf(d2.x));
            dm1 = fmaxf(dm1, fabsf(d2.y));
            int c0 = (int)(__float_as_uint(t2.x) + coff), c1 = (int)(__float_as_uint(t2.y) + coff);
            if (CLAMP) {  // offset codes: [0, 15] for both encodings
                c0 = min(max(c0, 0), 15);
                c1 = min(max(c1, 0), 15);
            }
            // elements 2i and 2i + 1 of the word: nibbles 2i and 2i + 1 (low first)
            acc |= (uint32_t)c0 << (8 * i);
            acc |= (uint32_t)c1 << (8 * i + 4);
        }
        word[h] = sym ? acc ^ 0x88888888u : acc;  // q + 8 -> two's-complement nibble
    }
    dmax = fmaxf(dm0, dm1);
}

__device__ __noinline__ uint32_t encode8_slow(const uint4 raw, const ScaleZero sz, bool symmetric) {
    float v[8];
    unpack_bf16x8(raw, v);
    return encode8(v, sz, symmetric);
}

// g <= 256: each thread takes four consecutive segments (32 weights, four
// 16-byte loads), so the per-group work is shared by 32 weights per thread;
// L = g/32 lanes per group, 32/L groups per warp.
//
// Fast path (finite group, scale not saturated -- then |x/s| <= 15.01):
//  - statistics with packed bf16x2 max/min that propagate NaN, so one test
//    per thread tells whether its values are all non-NaN;
//  - scale and zero without fp32 divisions (scale_zero_fast);
//  - f = x * rcp(s) in packed fp32x2; t = f + 1.5*2^23 puts rint(f) (round
//    half to even) in the low mantissa bits, so the code is bits(t) + const;
//  - the quotient guard of rint_quotient: if some |f - rint(f)| is within
//    2^-17 of 1/2, the thread redoes its codes with the IEEE division;
//  - fl(x/s) and rint are monotone, so the codes of the group's extremes
//    bound all its codes: when both are inside the code range (and neither
//    is near a tie) no code needs clamping.
// Anything else (NaN or Inf in the warp's groups, a saturated scale) takes
// the general per-value path of encode8.
constexpr int kUnitsPerThread = 2;  // 32-weight units in flight per thread

// Fast code of x (offset form: q + z, or q + 8 when symmetric) and |f - rint(f)|.
__device__ __forceinline__ int fast_code(float x, float rcp, uint32_t coff, float& dist) {
    const float f = __fmul_rn(x, rcp);
    const float t = __fadd_rn(f, kRoundMagic);
    dist = fabsf(__fsub_rn(f, __fsub_rn(t, kRoundMagic)));
    return (int)(__float_as_uint(t) + coff);
}

template <int L>
__global__ void __launch_bounds__(kQuantThreads) quantize_small_group_kernel(
    const uint4* __restrict__ W, int64_t nunit, int symmetric, uint32_t* __restrict__ qweight,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const bool sym = symmetric != 0;
    bool nonfinite = false, range = false;
    const int64_t stride = (int64_t)gridDim.x * (kQuantThreads * kUnitsPerThread);
    for (int64_t base = (int64_t)blockIdx.x * (kQuantThreads * kUnitsPerThread) + threadIdx.x;
         base - threadIdx.x < nunit; base += stride) {
        uint4 raw[kUnitsPerThread][4];
#pragma unroll
        for (int u = 0; u < kUnitsPerThread; ++u) {
            const int64_t un = base + (int64_t)u * kQuantThreads;
#pragma unroll
            for (int v = 0; v < 4; ++v) raw[u][v] = un < nunit ? ld_nc_v4(W + 4 * un + v) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnitsPerThread; ++u) {
            const int64_t un = base + (int64_t)u * kQuantThreads;
            uint32_t w[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                w[4 * v] = raw[u][v].x;
                w[4 * v + 1] = raw[u][v].y;
                w[4 * v + 2] = raw[u][v].z;
                w[4 * v + 3] = raw[u][v].w;
            }
            // ---- statistics of the thread's 32 values (NaN propagates) ----
            __nv_bfloat162 mx = __hmax2_nan(bits_bf2(w[0]), bits_bf2(w[1]));
            __nv_bfloat162 mn = __hmin2_nan(bits_bf2(w[0]), bits_bf2(w[1]));
#pragma unroll
            for (int i = 2; i < 16; ++i) {
                mx = __hmax2_nan(mx, bits_bf2(w[i]));
                mn = __hmin2_nan(mn, bits_bf2(w[i]));
            }
            const uint32_t mxb = bf2_bits(mx), mnb = bf2_bits(mn);
            const float mx0 = __uint_as_float(mxb << 16), mx1 = __uint_as_float(mxb & 0xffff0000u);
            const bool has_nan = isnan(mx0) || isnan(mx1);
            float hi = fmaxf(fmaxf(mx0, mx1), 0.0f);
            float lo = fminf(fminf(__uint_as_float(mnb << 16), __uint_as_float(mnb & 0xffff0000u)), 0.0f);
            if (__any_sync(0xffffffffu, has_nan) && has_nan) {  // NaN inputs are skipped by the statistics
                const float2 m = nan_skipping_min_max(raw[u][0], raw[u][1], raw[u][2], raw[u][3]);
                lo = m.x;
                hi = m.y;
            }
#pragma unroll
            for (int o = 1; o < L; o <<= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            }
            const bool inf = isinf(lo) || isinf(hi);
            nonfinite |= has_nan || inf;
            float rcp;
            const ScaleZero sz = scale_zero_fast(lo, hi, sym, rcp);
            if (un < nunit) range |= sz.range;
            uint32_t word[4];
            const bool general = __any_sync(0xffffffffu, has_nan || inf || sz.range);
            bool slow = general;
            if (!general) {
                const uint32_t coff = (uint32_t)(sym ? 8 : sz.z) - kRoundMagicBits;
                float dlo, dhi;
                const int clo = fast_code(lo, rcp, coff, dlo), chi = fast_code(hi, rcp, coff, dhi);
                const float tie = 0.5f - 0x1p-17f;
                const bool clamp = __any_sync(0xffffffffu, clo < 0 || chi > 15 || dlo > tie || dhi > tie);
                float dmax;
                if (clamp)
                    fast_codes<true>(w, rcp, coff, sym, word, dmax);
                else
                    fast_codes<false>(w, rcp, coff, sym, word, dmax);
                slow = dmax > tie;
            }
            if (slow)
                for (int h = 0; h < 4; ++h) word[h] = encode8_slow(raw[u][h], sz, sym);
            if (un < nunit) {
                reinterpret_cast<uint4*>(qweight)[un] = make_uint4(word[0], word[1], word[2], word[3]);
                if ((lane & (L - 1)) == 0) {
                    const int64_t gi = un / L;
                    scales[gi] = sz.s16;
                    if (!sym) zeros[gi] = __half_as_ushort(__int2half_rn(sz.z));
                }
            }
        }
    }
    const unsigned bad_nf = __ballot_sync(0xffffffffu, nonfinite);
    const unsigned bad_rg = __ballot_sync(0xffffffffu, range);
    if (lane == 0 && (bad_nf | bad_rg))
        raise_flag(status, (bad_nf ? kFlagNonfinite : 0u) | (bad_rg ? kFlagRange : 0u));
}

// g a multiple of 256: one warp per group, two passes over the group.
__global__ void __launch_bounds__(kQuantThreads) quantize_large_group_kernel(
    const uint4* __restrict__ W, int64_t ngroups, int g, int symmetric, uint32_t* __restrict__ qweight,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t gi = (int64_t)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    if (gi >= ngroups) return;  // whole warp leaves together
    const int segs = g / 8;
    const uint4* Wg = W + gi * segs;
    bool nonfinite = false;
    float lo = 0.0f, hi = 0.0f;
    for (int s = lane; s < segs; s += 32) {
        float v[8];
        unpack_bf16x8(ld_nc_v4(Wg + s), v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            nonfinite |= !isfinite(v[i]);
            lo = fminf(lo, v[i]);
            hi = fmaxf(hi, v[i]);
        }
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    ScaleZero sz = scale_zero(lo, hi, symmetric != 0);
    for (int s = lane; s < segs; s += 32) {
        float v[8];
        unpack_bf16x8(ld_nc_v4(Wg + s), v);
        qweight[gi * segs + s] = encode8(v, sz, symmetric != 0);
    }
    if (lane == 0) {
        scales[gi] = sz.s16;
        if (!symmetric) zeros[gi] = __half_as_ushort(__int2half_rn(sz.z));
    }
    const unsigned bad_nf = __ballot_sync(0xffffffffu, nonfinite);
    if (lane == 0 && (bad_nf || sz.range))
        raise_flag(status, (bad_nf ? kFlagNonfinite : 0u) | (sz.range ? kFlagRange : 0u));
}

// Dequantize: each thread expands 4 packed words (32 weights of one group)
// into 64 bytes of bf16, using the exact bf16x2 dequantization shared with the
// linear-layer kernels.  Grid-stride with two quads in flight per thread.
constexpr int kDeqThreads = 256;
constexpr int kDeqPerThread = 2;  // 2-word units in flight per thread

// One thread per unit of 2 packed words (16 weights, always inside one group
// because g is a multiple of 32): an 8-byte load and two 16-byte stores, so a
// warp reads 256 contiguous bytes and writes 1 KB contiguous.
__global__ void __launch_bounds__(kDeqThreads) dequantize_kernel(
    const uint2* __restrict__ qweight, const uint16_t* __restrict__ scales,
    const uint16_t* __restrict__ zeros, int64_t npair, int g, int symmetric, uint4* __restrict__ W_hat) {
    const int64_t stride = (int64_t)gridDim.x * (kDeqThreads * kDeqPerThread);
    for (int64_t base = (int64_t)blockIdx.x * (kDeqThreads * kDeqPerThread) + threadIdx.x; base < npair;
         base += stride) {
        uint2 q[kDeqPerThread];
        uint16_t s16[kDeqPerThread], z16[kDeqPerThread];
#pragma unroll
        for (int u = 0; u < kDeqPerThread; ++u) {
            const int64_t t = base + (int64_t)u * kDeqThreads;
            if (t < npair) {
                q[u] = __ldg(qweight + t);
                const int64_t gi = (t * 16) / g;
                s16[u] = scales[gi];
                z16[u] = symmetric ? (uint16_t)0 : zeros[gi];
            }
        }
#pragma unroll
        for (int u = 0; u < kDeqPerThread; ++u) {
            const int64_t t = base + (int64_t)u * kDeqThreads;
            if (t >= npair) continue;
            const int z = symmetric ? 0 : (int)__half2float(__ushort_as_half(z16[u]));
            const GroupConsts c = make_group_consts(s16[u], z, symmetric != 0);
            uint32_t o[4], o2[4];
            dequant_word_natural(q[u].x, c, o);
            dequant_word_natural(q[u].y, c, o2);
            W_hat[t * 2] = make_uint4(o[0], o[1], o[2], o[3]);
            W_hat[t * 2 + 1] = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        }
    }
}

// ------------------------------------------------------------------------
// MSE-optimal clipping per group ("LLM Quantization: GPTQ, AWQ, SmoothQuant,
// FP8, KV Cache (7/10)", Clipping Trade-off; "Quantization Algorithms" notes,
// calibration 4, MSE-optimal argmin ||x - x_dq||^2 per group).
// Candidate i shrinks the group's RTN range by alpha_i = fl32((20 - i) / 20),
// i = 0..10; scale, zero and codes follow the RTN formulas on that range (the
// exact scale_zero / encode path).  The candidate's error is
// sum_k (x_k - x_hat_k)^2 over finite x_k, x_hat_k the bf16 dequant, in fp64
// (difference, then the square rounded once, then the add; no fused
// multiply-add), summed sequentially over each lane's 8 consecutive weights
// and then by an xor butterfly over the group's L = g/8 lanes, i.e. a
// pairwise tree over the 8-weight runs in index order -- the same operations
// in the same order as the oracle, so the choice is identical.  The smallest error
// wins; ties keep the smaller i.  alpha_0 = 1 reproduces RTN.
// ------------------------------------------------------------------------
constexpr int kClipCandidates = 11;

// Exact codes (offset by nothing: q in [q_min, q_max]) of 8 values.
__device__ __forceinline__ void codes8(const float v[8], const ScaleZero& sz, bool symmetric, int q[8]) {
    const float s = __half2float(__ushort_as_half(sz.s16));
    const float rcp = __frcp_rn(s);
    const float qmin = symmetric ? -8.0f : 0.0f;
    const float qmax = symmetric ? 7.0f : 15.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (isnan(v[i])) {
            q[i] = sz.z;
        } else {
            const float t = rint_quotient(v[i], s, rcp);
            q[i] = (int)fminf(fmaxf(__fadd_rn(t, (float)sz.z), qmin), qmax);
        }
    }
}

template <int L>
__global__ void __launch_bounds__(kQuantThreads) quantize_clip_kernel(
    const uint4* __restrict__ W, int64_t nseg, int symmetric, uint32_t* __restrict__ qweight,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const bool sym = symmetric != 0;
    bool nonfinite = false, range = false;
    const int64_t stride = (int64_t)gridDim.x * kQuantThreads;
    for (int64_t base = (int64_t)blockIdx.x * kQuantThreads + threadIdx.x; base - threadIdx.x < nseg;
         base += stride) {
        const int64_t seg = base;
        const uint4 raw = seg < nseg ? ld_nc_v4(W + seg) : make_uint4(0, 0, 0, 0);
        float v[8];
        unpack_bf16x8(raw, v);
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            nonfinite |= !isfinite(v[i]);
            lo = fminf(lo, v[i]);  // NaN is skipped (minNum / maxNum)
            hi = fmaxf(hi, v[i]);
        }
#pragma unroll
        for (int o = 1; o < L; o <<= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        double best_err = 0.0;
        uint32_t best_word = 0;
        ScaleZero best_sz = {0x3c00u, 0, false};
        for (int i = 0; i < kClipCandidates; ++i) {
            const float alpha = __fdiv_rn((float)(20 - i), 20.0f);
            const ScaleZero sz = scale_zero(__fmul_rn(alpha, lo), __fmul_rn(alpha, hi), sym);
            int q[8];
            codes8(v, sz, sym, q);
            const float s = __half2float(__ushort_as_half(sz.s16));
            double err = 0.0;
            uint32_t word = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                word |= ((uint32_t)q[k] & 0xfu) << (4 * k);
                const float xh = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s, (float)(q[k] - sz.z))));
                const double e = __dsub_rn((double)v[k], (double)xh);
                if (isfinite(v[k])) err = __dadd_rn(err, __dmul_rn(e, e));  // no fused multiply-add
            }
#pragma unroll
            for (int o = 1; o < L; o <<= 1) err = __dadd_rn(err, __shfl_xor_sync(0xffffffffu, err, o));
            if (i == 0 || err < best_err) {
                best_err = err;
                best_word = word;
                best_sz = sz;
            }
        }
        if (seg < nseg) {
            range |= best_sz.range;
            qweight[seg] = best_word;
            if ((lane & (L - 1)) == 0) {
                const int64_t gi = seg / L;
                scales[gi] = best_sz.s16;
                if (!sym) zeros[gi] = __half_as_ushort(__int2half_rn(best_sz.z));
            }
        }
    }
    const unsigned bad_nf = __ballot_sync(0xffffffffu, nonfinite);
    const unsigned bad_rg = __ballot_sync(0xffffffffu, range);
    if (lane == 0 && (bad_nf | bad_rg))
        raise_flag(status, (bad_nf ? kFlagNonfinite : 0u) | (bad_rg ? kFlagRange : 0u));
}

}  // namespace

cudaError_t launch_quantize(const void* W, int64_t d_out, int64_t d_in, int g, int symmetric,
                            uint32_t* qweight, uint16_t* scales, uint16_t* zeros, uint32_t* status, int num_sms,
                            cudaStream_t stream) {
    const int64_t P = d_out * d_in;
    const uint4* W4 = static_cast<const uint4*>(W);
    if (g <= 256) {
        const int64_t nunit = P / 32;
        const int64_t per_block = (int64_t)kQuantThreads * kUnitsPerThread;
        int64_t blocks = (nunit + per_block - 1) / per_block;
        if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
        switch (g) {
            case 32:
                quantize_small_group_kernel<1><<<blocks, kQuantThreads, 0, stream>>>(W4, nunit, symmetric, qweight,
                                                                                       scales, zeros, status);
                break;
            case 64:
                quantize_small_group_kernel<2><<<blocks, kQuantThreads, 0, stream>>>(W4, nunit, symmetric, qweight,
                                                                                       scales, zeros, status);
                break;
            case 128:
                quantize_small_group_kernel<4><<<blocks, kQuantThreads, 0, stream>>>(W4, nunit, symmetric, qweight,
                                                                                       scales, zeros, status);
                break;
            case 256:
                quantize_small_group_kernel<8><<<blocks, kQuantThreads, 0, stream>>>(W4, nunit, symmetric, qweight,
                                                                                        scales, zeros, status);
                break;
            default:
                return cudaErrorInvalidValue;
        }
    } else {
        const int64_t ngroups = P / g;
        const int64_t warps_per_block = kQuantThreads / 32;
        const int64_t blocks = (ngroups + warps_per_block - 1) / warps_per_block;
        quantize_large_group_kernel<<<blocks, kQuantThreads, 0, stream>>>(W4, ngroups, g, symmetric, qweight, scales,
                                                                           zeros, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_clip(const void* W, int64_t d_out, int64_t d_in, int g, int symmetric,
                                 uint32_t* qweight, uint16_t* scales, uint16_t* zeros, uint32_t* status,
                                 int num_sms, cudaStream_t stream) {
    const int64_t nseg = d_out * d_in / 8;
    int64_t blocks = (nseg + kQuantThreads - 1) / kQuantThreads;
    if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
    const uint4* W4 = static_cast<const uint4*>(W);
    switch (g) {
        case 32:
            quantize_clip_kernel<4><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight, scales,
                                                                           zeros, status);
            break;
        case 64:
            quantize_clip_kernel<8><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight, scales,
                                                                           zeros, status);
            break;
        case 128:
            quantize_clip_kernel<16><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight, scales,
                                                                            zeros, status);
            break;
        case 256:
            quantize_clip_kernel<32><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight, scales,
                                                                            zeros, status);
            break;
        default:
            return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                              int64_t d_out, int64_t d_in, int g, int symmetric, void* W_hat, int num_sms,
                              cudaStream_t stream) {
    const int64_t npair = d_out * d_in / 16;
    int64_t blocks = (npair + kDeqThreads * kDeqPerThread - 1) / (kDeqThreads * kDeqPerThread);
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    dequantize_kernel<<<blocks, kDeqThreads, 0, stream>>>(reinterpret_cast<const uint2*>(qweight), scales, zeros,
                                                          npair, g, symmetric, static_cast<uint4*>(W_hat));
    return cudaGetLastError();
}

}  // namespace wq
