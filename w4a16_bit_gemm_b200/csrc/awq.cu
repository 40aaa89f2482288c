// awq.cu -- kernels of the AWQ per-input-channel scaling search (sm_100a).
//
// "Quantization Algorithms" study notes, AWQ procedure: per-channel mean |x|
// over a calibration batch; for alpha in {0, 0.1, ..., 1.0}: s = mean|x|^alpha
// / geomean, W' = W diag(s), loss = ||W X - Q(W') (X / s)||; keep the argmin.
// The search itself is orchestrated on the host side of the library; these
// kernels compute the statistics, the scales, W' and X', and the losses:
//  - m_j = (sum_t |X[t,j]|) / T in fp64 (an exact sum of bf16 values, so the
//    summation order does not matter), floored at 2^-30, kept as ln m_j;
//  - s_j = bf16_rn(fl32(exp(alpha (ln m_j - mean_j ln m_j)))), with ln and exp
//    evaluated by one fixed sequence of IEEE fp64 operations (below) and the
//    mean summed in channel order, so the scales are reproducible bit for bit;
//  - W'[n,j] = bf16_rn(fl32(W[n,j] s_j)), X'[t,j] = bf16_rn(fl32(X[t,j] / s_j));
//  - loss = sum (Y_ref - Y')^2 in fp64 over fp32 outputs, reduced in a fixed
//    order (deterministic).
#include <cuda_bf16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

constexpr int kAwqThreads = 256;
constexpr int kAwqReduceThreads = 1024;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// ln and exp as fixed sequences of IEEE binary64 operations: every product,
// sum and quotient rounded on its own through the _rn intrinsics (no fused
// multiply-add), with the argument reduction of W. J. Cody and W. Waite,
// "Software Manual for the Elementary Functions" (1980): ln 2 as a head with 21
// trailing zero bits (k * head exact for |k| < 2^21) plus a tail.
constexpr double kLn2Hi = 0x1.62e42fee00000p-1;
constexpr double kLn2Lo = 0x1.a39ef35793c76p-33;
constexpr double kInvLn2 = 0x1.71547652b82fep+0;
constexpr double kSqrt2 = 0x1.6a09e667f3bcdp+0;

// ln x, x positive and normal: x = f 2^e with f in [sqrt(2)/2, sqrt(2));
// ln f = 2 atanh(u), u = (f - 1) / (f + 1), as 2 u times the series
// sum_{k=0}^{11} u^(2k) / (2k + 1) in Horner form (|u| <= 0.1716);
// ln x = e ln2_hi + (e ln2_lo + ln f).
__device__ double awq_ln(double x) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(x);
    int e = (int)((b >> 52) & 0x7ffull) - 1023;
    double f = __longlong_as_double((long long)((b & 0x000fffffffffffffull) | 0x3ff0000000000000ull));
    if (f > kSqrt2) {
        f = __dmul_rn(f, 0.5);
        e += 1;
    }
    const double u = __ddiv_rn(__dsub_rn(f, 1.0), __dadd_rn(f, 1.0));
    const double v = __dmul_rn(u, u);
    double p = __ddiv_rn(1.0, 23.0);
    for (int k = 10; k >= 0; --k) p = __dadd_rn(__dmul_rn(p, v), __ddiv_rn(1.0, (double)(2 * k + 1)));
    const double lnf = __dmul_rn(__dadd_rn(u, u), p);
    const double de = (double)e;
    return __dadd_rn(__dmul_rn(de, kLn2Hi), __dadd_rn(__dmul_rn(de, kLn2Lo), lnf));
}

// e^x, |x| < 700: k = rint(x / ln 2) (half to even: add and subtract 1.5 2^52),
// r = (x - k ln2_hi) - k ln2_lo, e^r by its degree-13 Taylor polynomial
// (coefficients 1/i!, Horner form, |r| <= 0.347), times 2^k (exact).
__device__ double awq_exp(double x) {
    const double magic = 0x1.8p52;
    const double kd = __dsub_rn(__dadd_rn(__dmul_rn(x, kInvLn2), magic), magic);
    const double r = __dsub_rn(__dsub_rn(x, __dmul_rn(kd, kLn2Hi)), __dmul_rn(kd, kLn2Lo));
    double fact = 1.0;
    for (int i = 2; i <= 13; ++i) fact = __dmul_rn(fact, (double)i);  // 13!
    double p = __ddiv_rn(1.0, fact);
    for (int i = 12; i >= 0; --i) {
        fact = __ddiv_rn(fact, (double)(i + 1));  // i!, exact
        p = __dadd_rn(__dmul_rn(p, r), __ddiv_rn(1.0, fact));
    }
    const double scale = __longlong_as_double((long long)(((unsigned long long)((long long)kd + 1023)) << 52));
    return __dmul_rn(p, scale);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__global__ void __launch_bounds__(kAwqThreads) awq_colstats_kernel(const uint16_t* __restrict__ X, int64_t T,
                                                                   int64_t K, double* __restrict__ lnm) {
    const int64_t j = (int64_t)blockIdx.x * kAwqThreads + threadIdx.x;
    if (j >= K) return;
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) acc = __dadd_rn(acc, fabs((double)bf16_bits_to_f32(X[t * K + j])));
    double m = __ddiv_rn(acc, (double)T);
    if (m < 0x1p-30) m = 0x1p-30;
    lnm[j] = awq_ln(m);
}

// Mean of v[0..n), summed in index order by one thread (once per search).
__global__ void awq_mean_kernel(const double* __restrict__ v, int64_t n, double* __restrict__ out) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double acc = 0.0;
    for (int64_t i = 0; i < n; ++i) acc = __dadd_rn(acc, v[i]);
    *out = __ddiv_rn(acc, (double)n);
}

// s for alpha = i / 10, with i = *best if best is given, else alpha_idx.
__global__ void __launch_bounds__(kAwqThreads) awq_scales_kernel(const double* __restrict__ lnm,
                                                                 const double* __restrict__ mean_ln, int64_t K,
                                                                 int alpha_idx, const int32_t* __restrict__ best,
                                                                 uint16_t* __restrict__ s) {
    const int64_t j = (int64_t)blockIdx.x * kAwqThreads + threadIdx.x;
    if (j >= K) return;
    const int i = best ? *best : alpha_idx;
    const double alpha = __ddiv_rn((double)i, 10.0);
    s[j] = f32_to_bf16_bits(__double2float_rn(awq_exp(__dmul_rn(alpha, __dsub_rn(lnm[j], *mean_ln)))));
}

// W' = bf16(W s) for n_w rows, X' = bf16(X / s) for n_x rows; 8 weights per thread.
__global__ void __launch_bounds__(kAwqThreads) awq_apply_kernel(const uint4* __restrict__ W, int64_t n_w,
                                                                const uint4* __restrict__ X, int64_t n_x, int64_t K,
                                                                const uint16_t* __restrict__ s, uint4* __restrict__ Wp,
                                                                uint4* __restrict__ Xp) {
    const int64_t per_row = K / 8;
    const int64_t total = (n_w + n_x) * per_row;
    for (int64_t u = (int64_t)blockIdx.x * kAwqThreads + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * kAwqThreads) {
        const bool is_w = u < n_w * per_row;
        const int64_t v = is_w ? u : u - n_w * per_row;
        const int64_t j0 = (v % per_row) * 8;
        const uint4 in = is_w ? W[v] : X[v];
        const uint32_t iw[4] = {in.x, in.y, in.z, in.w};
        uint32_t ow[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(iw[q] << 16), b = __uint_as_float(iw[q] & 0xffff0000u);
            const float sa = bf16_bits_to_f32(s[j0 + 2 * q]), sb = bf16_bits_to_f32(s[j0 + 2 * q + 1]);
            const float ra = is_w ? __fmul_rn(a, sa) : __fdiv_rn(a, sa);
            const float rb = is_w ? __fmul_rn(b, sb) : __fdiv_rn(b, sb);
            ow[q] = (uint32_t)f32_to_bf16_bits(ra) | ((uint32_t)f32_to_bf16_bits(rb) << 16);
        }
        const uint4 out = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        if (is_w)
            Wp[v] = out;
        else
            Xp[v] = out;
    }
}

// Partial sums of (a - b)^2 in fp64: block b writes part[b] (fixed order inside the block).
__global__ void __launch_bounds__(kAwqThreads) awq_sqdiff_kernel(const float* __restrict__ a,
                                                                 const float* __restrict__ b, int64_t n,
                                                                 double* __restrict__ part) {
    __shared__ double sh[kAwqThreads];
    double acc = 0.0;
    for (int64_t i = (int64_t)blockIdx.x * kAwqThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kAwqThreads) {
        const double d = (double)a[i] - (double)b[i];
        acc += d * d;
    }
    sh[threadIdx.x] = acc;
    __syncthreads();
    for (int w = kAwqThreads / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[blockIdx.x] = sh[0];
}

__global__ void __launch_bounds__(kAwqReduceThreads) awq_sum_kernel(const double* __restrict__ part, int n,
                                                                    double* __restrict__ out) {
    __shared__ double sh[kAwqReduceThreads];
    double acc = 0.0;
    for (int i = threadIdx.x; i < n; i += kAwqReduceThreads) acc += part[i];
    sh[threadIdx.x] = acc;
    __syncthreads();
    for (int w = kAwqReduceThreads / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = sh[0];
}

// argmin over the losses; ties keep the smaller index.
__global__ void awq_select_kernel(const double* __restrict__ losses, int n, int32_t* __restrict__ best) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int b = 0;
    for (int i = 1; i < n; ++i)
        if (losses[i] < losses[b]) b = i;
    *best = b;
}

}  // namespace

constexpr int kAwqLossBlocks = 296;

cudaError_t launch_awq_colstats(const uint16_t* X, int64_t T, int64_t K, double* lnm, double* mean_ln,
                                cudaStream_t stream) {
    awq_colstats_kernel<<<(unsigned)((K + kAwqThreads - 1) / kAwqThreads), kAwqThreads, 0, stream>>>(X, T, K, lnm);
    awq_mean_kernel<<<1, 32, 0, stream>>>(lnm, K, mean_ln);
    return cudaGetLastError();
}

cudaError_t launch_awq_scale_apply(const uint16_t* W, int64_t N, const uint16_t* X, int64_t T, int64_t K,
                                   const double* lnm, const double* mean_ln, int alpha_idx, const int32_t* best,
                                   uint16_t* s, uint16_t* Wp, uint16_t* Xp, int num_sms, cudaStream_t stream) {
    awq_scales_kernel<<<(unsigned)((K + kAwqThreads - 1) / kAwqThreads), kAwqThreads, 0, stream>>>(
        lnm, mean_ln, K, alpha_idx, best, s);
    const int64_t units = (N + (Xp ? T : 0)) * (K / 8);
    int64_t blocks = (units + kAwqThreads - 1) / kAwqThreads;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    awq_apply_kernel<<<(unsigned)blocks, kAwqThreads, 0, stream>>>(
        reinterpret_cast<const uint4*>(W), N, reinterpret_cast<const uint4*>(X), Xp ? T : 0, K, s,
        reinterpret_cast<uint4*>(Wp), reinterpret_cast<uint4*>(Xp));
    return cudaGetLastError();
}

cudaError_t launch_awq_divide(const uint16_t* X, int64_t T, int64_t K, const uint16_t* s, uint16_t* Xp, int num_sms,
                              cudaStream_t stream) {
    int64_t blocks = (T * (K / 8) + kAwqThreads - 1) / kAwqThreads;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    awq_apply_kernel<<<(unsigned)blocks, kAwqThreads, 0, stream>>>(nullptr, 0, reinterpret_cast<const uint4*>(X), T,
                                                                    K, s, nullptr, reinterpret_cast<uint4*>(Xp));
    return cudaGetLastError();
}

cudaError_t launch_awq_loss(const float* Yref, const float* Y, int64_t n, double* part, double* out,
                            cudaStream_t stream) {
    awq_sqdiff_kernel<<<kAwqLossBlocks, kAwqThreads, 0, stream>>>(Yref, Y, n, part);
    awq_sum_kernel<<<1, kAwqReduceThreads, 0, stream>>>(part, kAwqLossBlocks, out);
    return cudaGetLastError();
}

cudaError_t launch_awq_select(const double* losses, int n, int32_t* best, cudaStream_t stream) {
    awq_select_kernel<<<1, 32, 0, stream>>>(losses, n, best);
    return cudaGetLastError();
}

int awq_loss_partials() { return kAwqLossBlocks; }

}  // namespace wq
