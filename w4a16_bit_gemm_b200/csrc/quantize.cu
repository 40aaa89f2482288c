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

// g <= 256: L = g/8 lanes per group, 32/L groups per warp.  Grid-stride:
// each thread handles kSegPerThread segments spaced one block-width apart per
// iteration, all loads issued before any arithmetic.
constexpr int kQuantThreads = 256;
constexpr int kSegPerThread = 2;

template <int L>
__global__ void __launch_bounds__(kQuantThreads) quantize_small_group_kernel(
    const uint4* __restrict__ W, int64_t nseg, int symmetric, uint32_t* __restrict__ qweight,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    bool nonfinite = false, range = false;
    const int64_t stride = (int64_t)gridDim.x * (kQuantThreads * kSegPerThread);
    for (int64_t base = (int64_t)blockIdx.x * (kQuantThreads * kSegPerThread) + threadIdx.x; base - threadIdx.x < nseg;
         base += stride) {
        uint4 raw[kSegPerThread];
#pragma unroll
        for (int u = 0; u < kSegPerThread; ++u) {
            const int64_t seg = base + (int64_t)u * kQuantThreads;
            raw[u] = seg < nseg ? ld_nc_v4(W + seg) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kSegPerThread; ++u) {
            const int64_t seg = base + (int64_t)u * kQuantThreads;
            float v[8];
            unpack_bf16x8(raw[u], v);
            float lo = 0.0f, hi = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                nonfinite |= !isfinite(v[i]);
                lo = fminf(lo, v[i]);
                hi = fmaxf(hi, v[i]);
            }
#pragma unroll
            for (int o = 1; o < L; o <<= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            }
            ScaleZero sz = scale_zero(lo, hi, symmetric != 0);
            if (seg < nseg) {
                range |= sz.range;
                qweight[seg] = encode8(v, sz, symmetric != 0);
                if ((lane & (L - 1)) == 0) {
                    const int64_t gi = seg / L;
                    scales[gi] = sz.s16;
                    if (!symmetric) zeros[gi] = __half_as_ushort(__int2half_rn(sz.z));
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
constexpr int kDeqPerThread = 2;

__global__ void __launch_bounds__(kDeqThreads) dequantize_kernel(
    const uint4* __restrict__ qweight, const uint16_t* __restrict__ scales,
    const uint16_t* __restrict__ zeros, int64_t nquad, int g, int symmetric, uint4* __restrict__ W_hat) {
    const int64_t stride = (int64_t)gridDim.x * (kDeqThreads * kDeqPerThread);
    for (int64_t base = (int64_t)blockIdx.x * (kDeqThreads * kDeqPerThread) + threadIdx.x; base < nquad;
         base += stride) {
        uint4 q[kDeqPerThread];
        uint16_t s16[kDeqPerThread], z16[kDeqPerThread];
#pragma unroll
        for (int u = 0; u < kDeqPerThread; ++u) {
            const int64_t t = base + (int64_t)u * kDeqThreads;
            if (t < nquad) {
                q[u] = ld_nc_v4(qweight + t);
                const int64_t gi = (t * 32) / g;
                s16[u] = scales[gi];
                z16[u] = symmetric ? (uint16_t)0 : zeros[gi];
            }
        }
#pragma unroll
        for (int u = 0; u < kDeqPerThread; ++u) {
            const int64_t t = base + (int64_t)u * kDeqThreads;
            if (t >= nquad) continue;
            const int z = symmetric ? 0 : (int)__half2float(__ushort_as_half(z16[u]));
            const GroupConsts c = make_group_consts(s16[u], z, symmetric != 0);
            const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t o[4];
                dequant_word_natural(w[j], c, o);
                W_hat[t * 4 + j] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_quantize(const void* W, int64_t d_out, int64_t d_in, int g, int symmetric,
                            uint32_t* qweight, uint16_t* scales, uint16_t* zeros, uint32_t* status, int num_sms,
                            cudaStream_t stream) {
    const int64_t P = d_out * d_in;
    const uint4* W4 = static_cast<const uint4*>(W);
    if (g <= 256) {
        const int64_t nseg = P / 8;
        const int64_t per_block = (int64_t)kQuantThreads * kSegPerThread;
        int64_t blocks = (nseg + per_block - 1) / per_block;
        if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
        switch (g) {
            case 32:
                quantize_small_group_kernel<4><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight,
                                                                                       scales, zeros, status);
                break;
            case 64:
                quantize_small_group_kernel<8><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight,
                                                                                       scales, zeros, status);
                break;
            case 128:
                quantize_small_group_kernel<16><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight,
                                                                                        scales, zeros, status);
                break;
            case 256:
                quantize_small_group_kernel<32><<<blocks, kQuantThreads, 0, stream>>>(W4, nseg, symmetric, qweight,
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

cudaError_t launch_dequantize(const uint32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                              int64_t d_out, int64_t d_in, int g, int symmetric, void* W_hat, int num_sms,
                              cudaStream_t stream) {
    const int64_t nquad = d_out * d_in / 32;
    int64_t blocks = (nquad + kDeqThreads * kDeqPerThread - 1) / (kDeqThreads * kDeqPerThread);
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    dequantize_kernel<<<blocks, kDeqThreads, 0, stream>>>(reinterpret_cast<const uint4*>(qweight), scales, zeros,
                                                          nquad, g, symmetric, static_cast<uint4*>(W_hat));
    return cudaGetLastError();
}

}  // namespace wq
