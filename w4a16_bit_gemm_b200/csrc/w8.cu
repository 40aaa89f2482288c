// w8.cu -- W8A16: symmetric INT8 weights, bf16 activations (sm_100a).
//
// "LLM Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)", "Which
// tensor is quantized" (weight-only INT4 / INT8, 16-bit activations: W4A16,
// W8A16) and Granularity (per-channel: one scale per output channel, i.e. one
// group spanning d_in); "Quantization Algorithms" study notes 1.8 (symmetric
// INT8 uses [-127, 127], leaving -128 out so the range stays symmetric).
//
//   s = fp16_rn(fl32(amax / 127)) per group (0 -> 1, overflow -> 65504 and
//       WQ_DEVFLAG_RANGE), q = clamp(rint(fl32(x / s)), -127, 127) (NaN -> 0,
//       non-finite inputs raise WQ_DEVFLAG_NONFINITE);
//   x_hat = bf16_rn(s q): s has 11 significant bits and |q| <= 127 has 7, so
//       the fp32 product is exact and the only rounding is the one to bf16;
//   packing: 4 codes per uint32, byte j of word c = column 4c + j, two's
//       complement, low byte first; scales fp16 [d_out][d_in / g].
//
// The linear layer for M <= 16 is a split-K GEMV on mma.sync m16n8k16: a CTA
// owns 16 output rows, its 16 warps split d_in, lane (r, t) dequantizes 16
// consecutive codes of rows r and r + 8 straight into bf16x2 A fragments and
// reads the matching activation pairs as B fragments (the sum over k is order
// free, so each lane group t may own its own column chunks); partial sums
// meet in shared memory in a fixed warp order.  M > 16 runs the tcgen05 GEMM
// (gemm.cu) with 8-bit weight tiles.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/wq.h"
#include "w8_device.cuh"
#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

// 16 codes (one uint4) times the scale -> 8 bf16x2 pairs (exact bf16_rn(s q)).
__device__ __forceinline__ void dequant16_w8(const uint4 w, float s, uint32_t out[8]) {
    dequant_word_w8(w.x, s, out[0], out[1]);
    dequant_word_w8(w.y, s, out[2], out[3]);
    dequant_word_w8(w.z, s, out[4], out[5]);
    dequant_word_w8(w.w, s, out[6], out[7]);
}

__device__ __forceinline__ void mma_bf16_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Quantize: one warp per (row, group); two passes over the group (amax, codes).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_w8_kernel(const uint16_t* __restrict__ W, int64_t N, int64_t K,
                                                          int g, uint32_t* __restrict__ qweight,
                                                          uint16_t* __restrict__ scales, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t G = K / g;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < N * G; u += warps) {
        const int64_t n = u / G, gi = u - n * G;
        const uint16_t* x = W + n * K + gi * g;
        float amax = 0.0f;
        bool nonfinite = false;
        for (int c = lane; c < g / 4; c += 32) {
            const uint2 v = *reinterpret_cast<const uint2*>(x + 4 * c);
            const uint32_t h[4] = {v.x << 16, v.x & 0xffff0000u, v.y << 16, v.y & 0xffff0000u};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float f = __uint_as_float(h[j]);
                if (!isfinite(f)) nonfinite = true;
                if (!isnan(f)) amax = fmaxf(amax, fabsf(f));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        nonfinite = __any_sync(0xffffffffu, nonfinite);
        uint16_t s16 = __half_as_ushort(__float2half_rn(__fdiv_rn(amax, 127.0f)));
        bool range = false;
        if (s16 == 0x7c00u) {
            s16 = 0x7bffu;
            range = true;
        }
        if (s16 == 0) s16 = 0x3c00u;
        const float s = __half2float(__ushort_as_half(s16));
        for (int c = lane; c < g / 4; c += 32) {
            const uint2 v = *reinterpret_cast<const uint2*>(x + 4 * c);
            const uint32_t h[4] = {v.x << 16, v.x & 0xffff0000u, v.y << 16, v.y & 0xffff0000u};
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float f = __uint_as_float(h[j]);
                int q = 0;
                if (!isnan(f)) q = (int)fminf(fmaxf(rintf(__fdiv_rn(f, s)), -127.0f), 127.0f);
                word |= ((uint32_t)q & 0xffu) << (8 * j);
            }
            qweight[(n * K + gi * g) / 4 + c] = word;
        }
        if (lane == 0) {
            scales[n * G + gi] = s16;
            if (nonfinite) raise_flag(status, WQ_DEVFLAG_NONFINITE);
            if (range) raise_flag(status, WQ_DEVFLAG_RANGE);
        }
    }
}

// x_hat = bf16_rn(s q), 4 weights per thread-iteration.
__global__ void __launch_bounds__(256) dequantize_w8_kernel(const uint32_t* __restrict__ qweight,
                                                            const uint16_t* __restrict__ scales, int64_t N, int64_t K,
                                                            int g, uint16_t* __restrict__ out) {
    const int64_t words = N * (K / 4), G = K / g;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < words; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = u / (K / 4), c = (u - n * (K / 4)) * 4;
        const float s = __half2float(__ushort_as_half(scales[n * G + c / g]));
        const uint32_t w = qweight[u] ^ 0x80808080u;
        float f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            f[j] = __fmul_rn(__fadd_rn(__uint_as_float(__byte_perm(w, 0x4Bu, 0x4550u + j)), -kW8Magic), s);
        *reinterpret_cast<uint2*>(out + n * K + c) =
            make_uint2(bf2_bits(__floats2bfloat162_rn(f[0], f[1])), bf2_bits(__floats2bfloat162_rn(f[2], f[3])));
    }
}

// ---------------------------------------------------------------------------
// GEMV, M <= 16 (NT = 1: M <= 8, NT = 2: M <= 16).
// ---------------------------------------------------------------------------
constexpr int kGemvWarps = 16;

template <int NT>
__global__ void __launch_bounds__(kGemvWarps * 32, 2) gemv_w8a16_kernel(const W8Args a) {
    __shared__ float red[kGemvWarps][16][16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, t = lane & 3;
    const int64_t n0 = (int64_t)blockIdx.x * 16;
    const int64_t rowA = n0 + r, rowB = n0 + r + 8;
    const bool vA = rowA < a.N, vB = rowB < a.N;
    const int64_t KC = a.K / 16;  // 16-column chunks per row
    const int64_t c_begin = KC * warp / kGemvWarps, c_end = KC * (warp + 1) / kGemvWarps;
    const int64_t iters = (c_end - c_begin + 3) / 4;  // same trip count on every lane
    const uint4* qA = reinterpret_cast<const uint4*>(a.qweight) + (vA ? rowA : 0) * KC;
    const uint4* qB = reinterpret_cast<const uint4*>(a.qweight) + (vB ? rowB : 0) * KC;
    const uint16_t* sA = a.scales + (vA ? rowA : 0) * a.G;
    const uint16_t* sB = a.scales + (vB ? rowB : 0) * a.G;
    const uint16_t* X = static_cast<const uint16_t*>(a.X);
    float d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.0f;
    // the weight loads of kPre chunks are issued before any is used
    constexpr int kPre = NT == 1 ? 2 : 1;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i0 = 0; i0 < iters; i0 += kPre) {
        uint4 wa[kPre], wb[kPre];
        float s_a[kPre], s_b[kPre];
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
            const int64_t c = c_begin + t + 4 * (i0 + u);
            const bool live = (i0 + u) < iters && c < c_end;
            wa[u] = (live && vA) ? ld_nc_v4(qA + c) : zero;
            wb[u] = (live && vB) ? ld_nc_v4(qB + c) : zero;
            const int64_t gi = live ? (c * 16) / a.g : 0;
            s_a[u] = (live && vA) ? __half2float(__ushort_as_half(sA[gi])) : 0.0f;
            s_b[u] = (live && vB) ? __half2float(__ushort_as_half(sB[gi])) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
            const int64_t c = c_begin + t + 4 * (i0 + u);
            const bool live = (i0 + u) < iters && c < c_end;
            uint32_t fa[8], fb[8];
            dequant16_w8(wa[u], s_a[u], fa);
            dequant16_w8(wb[u], s_b[u], fb);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m = r + 8 * nt;
                uint4 x0 = zero, x1 = zero;
                if (live && m < a.M) {
                    const uint4* xp = reinterpret_cast<const uint4*>(X + (int64_t)m * a.K + c * 16);
                    x0 = __ldg(xp);
                    x1 = __ldg(xp + 1);
                }
                const uint32_t xb[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16_16816(d[nt], fa[2 * j], fb[2 * j], fa[2 * j + 1], fb[2 * j + 1], xb[2 * j],
                                   xb[2 * j + 1]);
            }
        }
    }
    // d[nt]: (row r, token 8nt + 2t), (r, 8nt + 2t + 1), (r + 8, 8nt + 2t), (r + 8, 8nt + 2t + 1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        red[warp][r][8 * nt + 2 * t] = d[nt][0];
        red[warp][r][8 * nt + 2 * t + 1] = d[nt][1];
        red[warp][r + 8][8 * nt + 2 * t] = d[nt][2];
        red[warp][r + 8][8 * nt + 2 * t + 1] = d[nt][3];
    }
    __syncthreads();
    // 16 rows x 16 tokens: the first 256 threads finish one output each
    const int rr = threadIdx.x >> 4, m = threadIdx.x & 15;
    const int64_t n = n0 + rr;
    if (threadIdx.x < 256 && m < a.M && m < 8 * NT && n < a.N) {
        float y = 0.0f;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) y += red[w][rr][m];
        if (a.y_fp32)
            static_cast<float*>(a.Y)[(int64_t)m * a.N + n] = y;
        else
            static_cast<__nv_bfloat16*>(a.Y)[(int64_t)m * a.N + n] = __float2bfloat16_rn(y);
    }
}

}  // namespace

cudaError_t launch_quantize_w8(const void* W, int64_t N, int64_t K, int g, uint32_t* qweight, uint16_t* scales,
                               uint32_t* status, int num_sms, cudaStream_t stream) {
    const int64_t units = N * (K / g);
    int64_t blocks = (units + 7) / 8;
    if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
    quantize_w8_kernel<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(W), N, K, g, qweight,
                                                             scales, status);
    return cudaGetLastError();
}

cudaError_t launch_dequantize_w8(const uint32_t* qweight, const uint16_t* scales, int64_t N, int64_t K, int g,
                                 void* out, int num_sms, cudaStream_t stream) {
    int64_t blocks = (N * (K / 4) + 255) / 256;
    if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
    dequantize_w8_kernel<<<(unsigned)blocks, 256, 0, stream>>>(qweight, scales, N, K, g,
                                                               static_cast<uint16_t*>(out));
    return cudaGetLastError();
}

cudaError_t launch_gemv_w8a16(const W8Args& a, cudaStream_t stream) {
    const unsigned blocks = (unsigned)((a.N + 15) / 16);
    if (a.M <= 8)
        gemv_w8a16_kernel<1><<<blocks, kGemvWarps * 32, 0, stream>>>(a);
    else
        gemv_w8a16_kernel<2><<<blocks, kGemvWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace wq
