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
// holds elements [8w, 8w+8).  For g <= 256 (quantize_stream_kernel) a copy
// warp streams 32-weight units into shared memory with TMA, one consumer
// thread quantizes one unit, and a group spans L = g/32 lanes (butterfly
// shuffles for its min/max).  For larger g (quantize_large_group_kernel) one
// warp owns a group and loops over it twice.  Outputs are written with
// coalesced stores: consecutive lanes touch consecutive addresses.
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

__device__ __noinline__ uint32_t encode8_slow(const uint4 raw, const ScaleZero sz, bool symmetric) {
    float v[8];
    unpack_bf16x8(raw, v);
    return encode8(v, sz, symmetric);
}

// ------------------------------------------------------------------------
// Streaming quantize for g <= 256 (the common group sizes).
//
// The weights are read as rows of one 32-weight unit (64 bytes): a copy warp
// keeps a ring of kQsStages stages of 256 units (16 KB) in flight with 2D TMA
// loads (SWIZZLE_64B, so the 64-byte rows read by consecutive threads fall on
// different banks); each of the 256 consumer threads quantizes one unit per
// stage.  Two CTAs per SM; the units are split evenly over the grid in whole
// quanta of 8 units (whole groups for every g <= 256).
//
// Codes without a division and without a per-value test: with rcp = rn(1/s),
// q0 = rn(x rcp), the residual r = fma(-q0, s, x) and q1 = fma(r, rcp, q0)
// (Markstein's correction step for a correctly rounded reciprocal), q1 is the
// IEEE quotient fl(x/s) wherever the quotient is not subnormal, and rint(q1)
// equals rint(fl(x/s)) for every bf16 x and every finite fp16 s with
// |x/s| <= 40 (checked exhaustively on the CPU over all such pairs).  Then
// t = q1 + 1.5*2^23 puts rint(q1) (round half to even) in the low mantissa
// bits and t + off adds the zero point (or 8) exactly.  fl(x/s) and rint are
// monotone, so the codes of the group's extremes bound all its codes: when
// both lie in [0, 15], no code needs clamping.
// ------------------------------------------------------------------------
constexpr int kQsWarps = 8;                         // consumer warps
constexpr int kQsConsumers = kQsWarps * 32;         // one unit per thread per stage
constexpr int kQsThreads = kQsConsumers + 32;       // + the copy warp
constexpr int kQsStageBytes = kQsConsumers * 64;    // 16 KB
constexpr int kQsStages = 4;
constexpr int kQsCtasPerSm = 2;
constexpr int kQsSmem = kQsStages * kQsStageBytes + 1024;  // + base alignment slack
constexpr int64_t kQsMaxUnits = int64_t(1) << 30;   // units per launch (TMA coordinates are 32-bit)

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

// fl(x/s) for two values through the corrected product (see above).
__device__ __forceinline__ float2 quotient2(float2 x2, float2 rcp2, float2 ns2) {
    const float2 q0 = __fmul2_rn(x2, rcp2);
    const float2 r = __ffma2_rn(q0, ns2, x2);
    return __ffma2_rn(r, rcp2, q0);
}

// Scale and zero exactly as scale_zero, with the zero point through the
// corrected product; also returns rn(1/s).
__device__ __forceinline__ ScaleZero scale_zero_rcp(float lo, float hi, bool symmetric, float& rcp) {
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
    rcp = __frcp_rn(s);
    if (!symmetric && lo != 0.0f) {
        if (isinf(lo)) {
            r.z = 15;  // rint(-lo/s) = +inf, clamped
        } else {
            // -lo/s >= 0; a quotient far above 15 stays far above it
            const float y = __fsub_rn(0.0f, lo);
            const float q0 = __fmul_rn(y, rcp);
            const float q1 = __fmaf_rn(__fmaf_rn(q0, -s, y), rcp, q0);
            r.z = (int)fminf(rintf(q1), 15.0f);
        }
    }
    return r;
}

// Offset codes (q + z, or q + 8 when symmetric, as nibbles low first) of 16
// packed bf16 pairs.
template <bool CLAMP>
__device__ __forceinline__ void exact_codes(const uint32_t (&w)[16], float rcp, float s, float off, bool sym,
                                            uint32_t (&word)[4]) {
    const float2 rcp2 = make_float2(rcp, rcp), ns2 = make_float2(-s, -s);
    const float2 m2 = make_float2(kRoundMagic, kRoundMagic), off2 = make_float2(off, off);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint32_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t wv = w[4 * h + i];
            const float2 x2 = make_float2(__uint_as_float(wv << 16), __uint_as_float(wv & 0xffff0000u));
            const float2 t = __fadd2_rn(__fadd2_rn(quotient2(x2, rcp2, ns2), m2), off2);
            const uint32_t l0 = __float_as_uint(t.x), l1 = __float_as_uint(t.y);
            if (CLAMP) {
                const int c0 = min(max((int)(l0 - kRoundMagicBits), 0), 15);
                const int c1 = min(max((int)(l1 - kRoundMagicBits), 0), 15);
                b[i] = (uint32_t)c0 | ((uint32_t)c1 << 4);
            } else {
                b[i] = l1 * 16u + l0;  // low byte: (code1 << 4) | code0, both in [0, 15]
            }
        }
        const uint32_t lo2 = __byte_perm(b[0], b[1], 0x0040), hi2 = __byte_perm(b[2], b[3], 0x0040);
        const uint32_t acc = __byte_perm(lo2, hi2, 0x5410);
        word[h] = sym ? acc ^ 0x88888888u : acc;  // q + 8 -> two's-complement nibble
    }
}

template <int L>
__global__ void __launch_bounds__(kQsThreads, kQsCtasPerSm) quantize_stream_kernel(
    const __grid_constant__ CUtensorMap tmap, int64_t nunit, int symmetric, uint32_t* __restrict__ qweight,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, uint32_t* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ uint64_t full[kQsStages], empty[kQsStages];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // the CTA's units [u0, u1): quanta of 8 units split evenly over the grid
    const int64_t nq = (nunit + 7) / 8;
    const int64_t per = nq / gridDim.x, extra = nq - per * gridDim.x;
    const int64_t u0 = 8 * ((int64_t)blockIdx.x * per + min((int64_t)blockIdx.x, extra));
    const int64_t u1 = min(u0 + 8 * (per + ((int64_t)blockIdx.x < extra ? 1 : 0)), nunit);
    const int nst = u1 > u0 ? (int)((u1 - u0 + kQsConsumers - 1) / kQsConsumers) : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQsStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kQsWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kQsWarps) {
        // ---------------- copy warp ----------------
        if (lane == 0) {
            prefetch_tmap(&tmap);
            for (int k = 0; k < nst; ++k) {
                const int slot = k % kQsStages;
                if (k >= kQsStages && !mbar_wait(&empty[slot], (uint32_t)((k / kQsStages) - 1) & 1u, status)) break;
                mbar_arrive_expect_tx(&full[slot], kQsStageBytes);
                tma_load_2d(stages + slot * kQsStageBytes, &tmap, &full[slot], 0,
                            (int32_t)(u0 + (int64_t)k * kQsConsumers));
            }
        }
        return;
    }

    // ---------------- consumers: one unit per thread per stage ----------------
    const bool sym = symmetric != 0;
    bool nonfinite = false, range = false;
    // row threadIdx.x of a stage; its 16-byte chunk c sits at c ^ ((row >> 1) & 3)
    const uint32_t row_addr = smem_u32(stages) + threadIdx.x * 64;
    const uint32_t swz = (threadIdx.x >> 1) & 3;
    for (int k = 0; k < nst; ++k) {
        const int slot = k % kQsStages;
        const bool ok = mbar_wait(&full[slot], (uint32_t)(k / kQsStages) & 1u, status);
        if (!__all_sync(0xffffffffu, ok)) break;
        uint4 raw[4];
        const uint32_t a = row_addr + slot * kQsStageBytes;
#pragma unroll
        for (int v = 0; v < 4; ++v) raw[v] = ld_shared_u4(a + (((uint32_t)v ^ swz) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);

        const int64_t un = u0 + (int64_t)k * kQsConsumers + threadIdx.x;
        const bool valid = un < u1;
        uint32_t w[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            w[4 * v] = raw[v].x;
            w[4 * v + 1] = raw[v].y;
            w[4 * v + 2] = raw[v].z;
            w[4 * v + 3] = raw[v].w;
        }
        // ---- statistics of the thread's 32 values (NaN propagates), as a tree ----
        __nv_bfloat162 mx[8], mn[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mx[i] = __hmax2_nan(bits_bf2(w[2 * i]), bits_bf2(w[2 * i + 1]));
            mn[i] = __hmin2_nan(bits_bf2(w[2 * i]), bits_bf2(w[2 * i + 1]));
        }
#pragma unroll
        for (int n = 4; n >= 1; n >>= 1) {
#pragma unroll
            for (int i = 0; i < n; ++i) {
                mx[i] = __hmax2_nan(mx[i], mx[i + n]);
                mn[i] = __hmin2_nan(mn[i], mn[i + n]);
            }
        }
        const uint32_t mxb = bf2_bits(mx[0]), mnb = bf2_bits(mn[0]);
        const float mx0 = __uint_as_float(mxb << 16), mx1 = __uint_as_float(mxb & 0xffff0000u);
        const bool has_nan = isnan(mx0) || isnan(mx1);
        float hi = fmaxf(fmaxf(mx0, mx1), 0.0f);
        float lo = fminf(fminf(__uint_as_float(mnb << 16), __uint_as_float(mnb & 0xffff0000u)), 0.0f);
        if (__any_sync(0xffffffffu, has_nan) && has_nan) {  // NaN inputs are skipped by the statistics
            const float2 m = nan_skipping_min_max(raw[0], raw[1], raw[2], raw[3]);
            lo = m.x;
            hi = m.y;
        }
#pragma unroll
        for (int o = 1; o < L; o <<= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const bool inf = isinf(lo) || isinf(hi);
        float rcp;
        const ScaleZero sz = scale_zero_rcp(lo, hi, sym, rcp);
        if (valid) {
            nonfinite |= has_nan || inf;
            range |= sz.range;
        }
        uint32_t word[4];
        const bool slow = __any_sync(0xffffffffu, has_nan || inf || sz.range);
        if (!slow) {
            const float s = __half2float(__ushort_as_half(sz.s16));
            const float off = sym ? 8.0f : (float)sz.z;
            // codes of the extremes (exact), as one pair
            const float2 e = __fadd2_rn(
                __fadd2_rn(quotient2(make_float2(lo, hi), make_float2(rcp, rcp), make_float2(-s, -s)),
                           make_float2(kRoundMagic, kRoundMagic)),
                make_float2(off, off));
            const int clo = (int)(__float_as_uint(e.x) - kRoundMagicBits);
            const int chi = (int)(__float_as_uint(e.y) - kRoundMagicBits);
            if (__any_sync(0xffffffffu, clo < 0 || chi > 15))
                exact_codes<true>(w, rcp, s, off, sym, word);
            else
                exact_codes<false>(w, rcp, s, off, sym, word);
        }
        if (slow)
            for (int h = 0; h < 4; ++h) word[h] = encode8_slow(raw[h], sz, sym);
        if (valid) {
            reinterpret_cast<uint4*>(qweight)[un] = make_uint4(word[0], word[1], word[2], word[3]);
            if ((lane & (L - 1)) == 0) {
                const int64_t gi = un / L;
                scales[gi] = sz.s16;
                if (!sym) zeros[gi] = __half_as_ushort(__int2half_rn(sz.z));
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

// Dequantize: each thread expands 2-word units (16 weights of one group) into
// 32 bytes of bf16, using the exact bf16x2 dequantization shared with the
// linear-layer kernels.  Small blocks with one unit per thread and a grid that
// covers the whole matrix (no grid-stride cap) measured fastest on B200: at
// 4096 x 4096 g128, 10.4 us against 11.7 us for 256 threads x 2 units on a
// grid capped at 8 blocks per SM, and 22.8 against 28.2 us at 11008 x 4096;
// more units per thread (4, 8) were slower still.
constexpr int kDeqThreads = 128;
constexpr int kDeqPerThread = 1;  // 2-word units per thread per grid-stride step

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

template <int L>
cudaError_t launch_quantize_stream(const uint16_t* W, int64_t nunit, int symmetric, uint32_t* qweight,
                                   uint16_t* scales, uint16_t* zeros, uint32_t* status, int num_sms,
                                   cudaStream_t stream) {
    CUtensorMap tmap;
    if (encode_tensor_map_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, W, 32, (uint64_t)nunit, 64, 32, kQsConsumers,
                             CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = quantize_stream_kernel<L>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQsSmem);
    if (e != cudaSuccess) return e;
    // the whole unified L1/shared array as shared memory, so that kQsCtasPerSm CTAs fit
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    const int64_t nq = (nunit + 7) / 8;
    const int64_t resident = (int64_t)kQsCtasPerSm * num_sms;
    const int grid = (int)(nq < resident ? nq : resident);
    kern<<<grid, kQsThreads, kQsSmem, stream>>>(tmap, nunit, symmetric, qweight, scales, zeros, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* W, int64_t d_out, int64_t d_in, int g, int symmetric,
                            uint32_t* qweight, uint16_t* scales, uint16_t* zeros, uint32_t* status, int num_sms,
                            cudaStream_t stream) {
    const int64_t P = d_out * d_in;
    if (g <= 256) {
        const int64_t nunit = P / 32;
        const uint16_t* W16 = static_cast<const uint16_t*>(W);
        for (int64_t c0 = 0; c0 < nunit; c0 += kQsMaxUnits) {
            const int64_t n = nunit - c0 < kQsMaxUnits ? nunit - c0 : kQsMaxUnits;
            const int64_t gi0 = c0 * 32 / g;
            cudaError_t e;
            uint16_t* zc = zeros ? zeros + gi0 : nullptr;
            switch (g) {
                case 32:
                    e = launch_quantize_stream<1>(W16 + c0 * 32, n, symmetric, qweight + c0 * 4, scales + gi0, zc,
                                                  status, num_sms, stream);
                    break;
                case 64:
                    e = launch_quantize_stream<2>(W16 + c0 * 32, n, symmetric, qweight + c0 * 4, scales + gi0, zc,
                                                  status, num_sms, stream);
                    break;
                case 128:
                    e = launch_quantize_stream<4>(W16 + c0 * 32, n, symmetric, qweight + c0 * 4, scales + gi0, zc,
                                                  status, num_sms, stream);
                    break;
                case 256:
                    e = launch_quantize_stream<8>(W16 + c0 * 32, n, symmetric, qweight + c0 * 4, scales + gi0, zc,
                                                  status, num_sms, stream);
                    break;
                default:
                    return cudaErrorInvalidValue;
            }
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    const int64_t ngroups = P / g;
    const int64_t warps_per_block = kQuantThreads / 32;
    const int64_t blocks = (ngroups + warps_per_block - 1) / warps_per_block;
    quantize_large_group_kernel<<<blocks, kQuantThreads, 0, stream>>>(static_cast<const uint4*>(W), ngroups, g,
                                                                       symmetric, qweight, scales, zeros, status);
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
    if (blocks > (int64_t)num_sms * 4096) blocks = (int64_t)num_sms * 4096;
    dequantize_kernel<<<blocks, kDeqThreads, 0, stream>>>(reinterpret_cast<const uint2*>(qweight), scales, zeros,
                                                          npair, g, symmetric, static_cast<uint4*>(W_hat));
    return cudaGetLastError();
}

}  // namespace wq
