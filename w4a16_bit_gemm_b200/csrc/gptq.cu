// gptq.cu -- GPTQ error feedback on the GPU (sm_100a), in fp64.
//
// "Quantization Algorithms" study notes, GPTQ chapter: objective
// ||W X - W_hat X||^2; H = 2 X X^T dampened by 1 % of its mean diagonal;
// L = Cholesky(H^-1); columns quantized one at a time in blocks of 128,
// err = (w_j - q_j) / L[j][j] fed into the block's later columns at once and
// into the columns after the block through the block's errors; act-order.
//
// Every step is an fp64 computation whose result is fixed by its operation
// order: each product is rounded before its add or subtract (explicit
// __dmul_rn / __dadd_rn / __dsub_rn, so no contraction into fused
// multiply-adds), every sum runs in ascending index order, divisions and
// square roots are IEEE.  The blocked kernels below keep that per-element
// order:
//  - Cholesky, right-looking in panels of 32 columns: an entry (i, c) is
//    decremented by l[i][k] l[c][k] for k = 0, 1, ... in turn, previous panels
//    first, then the panel's own columns, then divided by l[c][c];
//  - L^-1 by forward substitution in row blocks of 32: the accumulator of
//    entry (i, j) receives l[i][k] Linv[k][j] for k = j, j+1, ... in turn (the
//    terms for k < j are exact zeros and leave it unchanged);
//  - H^-1[i][j] = sum_k Linv[k][i] Linv[k][j] over ascending k (terms with
//    k < max(i, j) are exact zeros);
//  - the sweep's block tail: acc = sum_{j in block} err_j U[j][k] in order,
//    then w_k - acc.
// The Hessian is the one place a fused multiply-add is used: the product of
// two bf16 values is exact in fp64, so fma(a, b, acc) rounds exactly like
// acc + a b.
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/wq.h"
#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

constexpr int kTile = 64;        // output tile edge of the fp64 tiled kernels
constexpr int kTileThreads = 256;  // 16 x 16 threads, 4 x 4 entries each
constexpr int kPanel = 32;       // Cholesky panel width / inverse row block
constexpr int kChunk = 32;       // inner-dimension chunk staged in shared memory
constexpr int kSweepWarps = 32;  // rows per sweep CTA (one warp per row)

__device__ __forceinline__ double bf16_bits_to_f64(uint16_t b) {
    return (double)__uint_as_float((uint32_t)b << 16);
}

// ---------------------------------------------------------------------------
// H[a][b] = 2 sum_t x[t][a] x[t][b] for the tiles on or below the diagonal;
// both (a, b) and (b, a) are written (the sums are the same operations).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kTileThreads) gptq_hessian_kernel(const uint16_t* __restrict__ X, int64_t T,
                                                                    int64_t K, double* __restrict__ H) {
    const int64_t ta = blockIdx.y, tb = blockIdx.x;
    if (tb > ta) return;
    const int64_t a0 = ta * kTile, b0 = tb * kTile;
    __shared__ double xa[kChunk][kTile + 1];
    __shared__ double xb[kChunk][kTile + 1];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int64_t t0 = 0; t0 < T; t0 += kChunk) {
        for (int e = threadIdx.x; e < kChunk * kTile; e += kTileThreads) {
            const int r = e / kTile, c = e % kTile;
            const int64_t t = t0 + r;
            xa[r][c] = (t < T && a0 + c < K) ? bf16_bits_to_f64(X[t * K + a0 + c]) : 0.0;
            xb[r][c] = (t < T && b0 + c < K) ? bf16_bits_to_f64(X[t * K + b0 + c]) : 0.0;
        }
        __syncthreads();
        const int tn = (int)(T - t0 < kChunk ? T - t0 : kChunk);
        for (int r = 0; r < tn; ++r) {
            double va[4], vb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) va[i] = xa[r][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) vb[j] = xb[r][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fma_rn(va[i], vb[j], acc[i][j]);  // exact product
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t a = a0 + ty + 16 * i, b = b0 + tx + 16 * j;
            if (a < K && b < K) {
                const double h = 2.0 * acc[i][j];
                H[a * K + b] = h;
                H[b * K + a] = h;
            }
        }
}

// Dampening: d = 0.01 mean(diag H) (diagonal summed in index order; d = 1 if
// the mean is 0), added to every diagonal entry.  One CTA: the diagonal is
// gathered into shared memory in parallel, then one thread sums it in order.
constexpr int kDampThreads = 1024;
constexpr int kDampChunk = 4096;

__global__ void __launch_bounds__(kDampThreads) gptq_damp_kernel(double* __restrict__ H, int64_t K) {
    __shared__ double diag[kDampChunk];
    __shared__ double total;
    if (threadIdx.x == 0) total = 0.0;
    for (int64_t j0 = 0; j0 < K; j0 += kDampChunk) {
        const int n = (int)(K - j0 < kDampChunk ? K - j0 : kDampChunk);
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kDampThreads) diag[i] = H[(j0 + i) * K + j0 + i];
        __syncthreads();
        if (threadIdx.x == 0) {
            double s = total;
            for (int i = 0; i < n; ++i) s = __dadd_rn(s, diag[i]);
            total = s;
        }
    }
    __syncthreads();
    double d = __dmul_rn(0.01, __ddiv_rn(total, (double)K));
    if (d == 0.0) d = 1.0;
    for (int64_t j = threadIdx.x; j < K; j += kDampThreads) H[j * K + j] = __dadd_rn(H[j * K + j], d);
}

// Processing order: by decreasing diagonal, ties in index order (the rank of
// column j is the number of columns that come before it).  Without act-order,
// or when a diagonal entry is not finite, the identity.
__global__ void gptq_perm_kernel(const double* __restrict__ H, int64_t K, int act_order, int32_t* __restrict__ perm,
                                 int* __restrict__ nonfinite) {
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    if (!act_order || *nonfinite) {
        perm[j] = (int32_t)j;
        return;
    }
    const double dj = H[j * K + j];
    int64_t r = 0;
    for (int64_t i = 0; i < K; ++i) {
        const double di = H[i * K + i];
        r += (di > dj) || (di == dj && i < j);
    }
    perm[r] = (int32_t)j;
}

__global__ void gptq_diag_check_kernel(const double* __restrict__ H, int64_t K, int* __restrict__ nonfinite) {
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j < K && !isfinite(H[j * K + j])) *nonfinite = 1;
}

// Hp[a][b] = H[perm[a]][perm[b]].
__global__ void gptq_gather_kernel(const double* __restrict__ H, const int32_t* __restrict__ perm, int64_t K,
                                   double* __restrict__ Hp) {
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < K * K; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t a = u / K, b = u - a * K;
        Hp[u] = H[(int64_t)perm[a] * K + perm[b]];
    }
}

// ---------------------------------------------------------------------------
// Cholesky, lower, in place (lower triangle of A), panel [p0, p1).
// ---------------------------------------------------------------------------

// The panel's diagonal block: one CTA of kPanel threads, column by column.
constexpr int kDiagThreads = 256;

__global__ void __launch_bounds__(kDiagThreads) gptq_chol_diag_kernel(double* __restrict__ A, int64_t K, int64_t p0,
                                                                      uint32_t* __restrict__ status) {
    // right-looking inside the block: after column j is final, every later
    // entry (i, c) of the block takes its term l[i][j] l[c][j] in turn, so
    // each entry still receives its terms in ascending j
    __shared__ double Ls[kPanel][kPanel + 1];
    const int w = (int)(K - p0 < kPanel ? K - p0 : kPanel);
    for (int e = threadIdx.x; e < kPanel * kPanel; e += kDiagThreads) {
        const int r = e / kPanel, c = e % kPanel;
        if (r < w && c <= r) Ls[r][c] = A[(p0 + r) * K + p0 + c];
    }
    __syncthreads();
    for (int j = 0; j < w; ++j) {
        if (threadIdx.x == 0) {
            double d = Ls[j][j];
            if (!(d > 0.0) || !isfinite(d)) {
                d = 1.0;
                raise_flag(status, WQ_DEVFLAG_RANGE);
            }
            Ls[j][j] = __dsqrt_rn(d);
        }
        __syncthreads();
        for (int i = j + 1 + (int)threadIdx.x; i < w; i += kDiagThreads) Ls[i][j] = __ddiv_rn(Ls[i][j], Ls[j][j]);
        __syncthreads();
        // trailing entries (i, c), j < c <= i < w
        const int m = w - j - 1;
        for (int e = threadIdx.x; e < m * m; e += kDiagThreads) {
            const int i = j + 1 + e / m, c = j + 1 + e % m;
            if (c <= i) Ls[i][c] = __dsub_rn(Ls[i][c], __dmul_rn(Ls[i][j], Ls[c][j]));
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kPanel * kPanel; e += kDiagThreads) {
        const int r = e / kPanel, c = e % kPanel;
        if (r < w && c <= r) A[(p0 + r) * K + p0 + c] = Ls[r][c];
    }
}

// Rows below the diagonal block: one thread per row.
__global__ void __launch_bounds__(128) gptq_chol_panel_kernel(double* __restrict__ A, int64_t K, int64_t p0) {
    __shared__ double Ls[kPanel][kPanel + 1];
    const int w = (int)(K - p0 < kPanel ? K - p0 : kPanel);
    for (int e = threadIdx.x; e < kPanel * kPanel; e += blockDim.x) {
        const int r = e / kPanel, c = e % kPanel;
        Ls[r][c] = (r < w && c <= r) ? A[(p0 + r) * K + p0 + c] : 0.0;
    }
    __syncthreads();
    const int64_t i = p0 + w + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= K) return;
    // the row's panel entries in registers; right-looking: once entry j is
    // final, the later entries take their term row[j] l[c][j] in turn
    double row[kPanel];
#pragma unroll
    for (int j = 0; j < kPanel; ++j) row[j] = j < w ? A[i * K + p0 + j] : 0.0;
#pragma unroll
    for (int j = 0; j < kPanel; ++j) {
        if (j < w) {
            row[j] = __ddiv_rn(row[j], Ls[j][j]);
#pragma unroll
            for (int c = j + 1; c < kPanel; ++c) row[c] = __dsub_rn(row[c], __dmul_rn(row[j], Ls[c][j]));
        }
    }
#pragma unroll
    for (int j = 0; j < kPanel; ++j)
        if (j < w) A[i * K + p0 + j] = row[j];
}

// Trailing update: A[i][c] -= l[i][k] l[c][k], k = p0 .. p1-1 in turn, for
// p1 <= c <= i (tiles on or below the diagonal).
__global__ void __launch_bounds__(kTileThreads) gptq_chol_update_kernel(double* __restrict__ A, int64_t K,
                                                                        int64_t p0) {
    const int64_t p1 = p0 + kPanel;
    const int64_t ti = blockIdx.y, tc = blockIdx.x;
    if (tc > ti) return;
    const int64_t i0 = p1 + ti * kTile, c0 = p1 + tc * kTile;
    __shared__ double Li[kTile][kPanel + 1];
    __shared__ double Lc[kTile][kPanel + 1];
    for (int e = threadIdx.x; e < kTile * kPanel; e += kTileThreads) {
        const int r = e / kPanel, k = e % kPanel;
        Li[r][k] = i0 + r < K ? A[(i0 + r) * K + p0 + k] : 0.0;
        Lc[r][k] = c0 + r < K ? A[(c0 + r) * K + p0 + k] : 0.0;
    }
    __syncthreads();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double v[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + ty + 16 * a, c = c0 + tx + 16 * b;
            v[a][b] = (i < K && c <= i) ? A[i * K + c] : 0.0;
        }
#pragma unroll 4
    for (int k = 0; k < kPanel; ++k) {
        double li[4], lc[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) li[a] = Li[ty + 16 * a][k];
#pragma unroll
        for (int b = 0; b < 4; ++b) lc[b] = Lc[tx + 16 * b][k];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) v[a][b] = __dsub_rn(v[a][b], __dmul_rn(li[a], lc[b]));
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + ty + 16 * a, c = c0 + tx + 16 * b;
            if (i < K && c <= i) A[i * K + c] = v[a][b];
        }
}

// ---------------------------------------------------------------------------
// Linv = L^-1 (lower).  Li holds zeros above the diagonal and, for rows not
// yet finished, the running accumulators.  Row block [r0, r1).
// ---------------------------------------------------------------------------

// Finish the block's rows: one thread per column j < r1.
__global__ void __launch_bounds__(128) gptq_trinv_block_kernel(const double* __restrict__ L, double* __restrict__ Li,
                                                               int64_t K, int64_t r0) {
    __shared__ double Ls[kPanel][kPanel + 1];
    const int w = (int)(K - r0 < kPanel ? K - r0 : kPanel);
    for (int e = threadIdx.x; e < kPanel * kPanel; e += blockDim.x) {
        const int r = e / kPanel, c = e % kPanel;
        Ls[r][c] = (r < w && c <= r) ? L[(r0 + r) * K + r0 + c] : 0.0;
    }
    __syncthreads();
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= r0 + w) return;
    // acc[ii]: the accumulator of entry (r0 + ii, j); right-looking: once
    // Linv[r0 + ii][j] is final, the later rows of the block take their term
    // l[r0 + i2][r0 + ii] Linv[r0 + ii][j] in turn (terms with r0 + ii < j are
    // skipped: the sum of entry (i, j) starts at k = j)
    double acc[kPanel];
#pragma unroll
    for (int ii = 0; ii < kPanel; ++ii) acc[ii] = (ii < w && r0 + ii > j) ? Li[(r0 + ii) * K + j] : 0.0;
#pragma unroll
    for (int ii = 0; ii < kPanel; ++ii) {
        if (ii < w) {
            const int64_t i = r0 + ii;
            if (i >= j) {
                const double out = i == j ? __ddiv_rn(1.0, Ls[ii][ii]) : __ddiv_rn(-acc[ii], Ls[ii][ii]);
                Li[i * K + j] = out;
#pragma unroll
                for (int i2 = ii + 1; i2 < kPanel; ++i2) acc[i2] = __dadd_rn(acc[i2], __dmul_rn(Ls[i2][ii], out));
            }
        }
    }
}

// Accumulators of the rows below the block: Li[i][j] += l[i][k] Linv[k][j],
// k in the block in turn, for i >= r1 and j < r1.
__global__ void __launch_bounds__(kTileThreads) gptq_trinv_update_kernel(const double* __restrict__ L,
                                                                         double* __restrict__ Li, int64_t K,
                                                                         int64_t r0) {
    const int64_t r1 = r0 + kPanel;
    const int64_t i0 = r1 + (int64_t)blockIdx.y * kTile, j0 = (int64_t)blockIdx.x * kTile;
    if (j0 >= r1) return;
    __shared__ double Lb[kTile][kPanel + 1];
    __shared__ double Vb[kPanel][kTile + 1];
    for (int e = threadIdx.x; e < kTile * kPanel; e += kTileThreads) {
        const int r = e / kPanel, k = e % kPanel;
        Lb[r][k] = i0 + r < K ? L[(i0 + r) * K + r0 + k] : 0.0;
        const int kk = e / kTile, c = e % kTile;
        Vb[kk][c] = j0 + c < r1 ? Li[(r0 + kk) * K + j0 + c] : 0.0;
    }
    __syncthreads();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double v[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
            v[a][b] = (i < K && j < r1) ? Li[i * K + j] : 0.0;
        }
#pragma unroll 4
    for (int k = 0; k < kPanel; ++k) {
        double l[4], x[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) l[a] = Lb[ty + 16 * a][k];
#pragma unroll
        for (int b = 0; b < 4; ++b) x[b] = Vb[k][tx + 16 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) v[a][b] = __dadd_rn(v[a][b], __dmul_rn(l[a], x[b]));
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
            if (i < K && j < r1) Li[i * K + j] = v[a][b];
        }
}

// Hinv[i][j] = sum_k Linv[k][i] Linv[k][j] (ascending k) for i >= j.
__global__ void __launch_bounds__(kTileThreads) gptq_gram_kernel(const double* __restrict__ Li, int64_t K,
                                                                 double* __restrict__ Hi) {
    const int64_t ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti) return;
    const int64_t i0 = ti * kTile, j0 = tj * kTile;
    __shared__ double Ai[kChunk][kTile + 1];
    __shared__ double Aj[kChunk][kTile + 1];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    for (int64_t k0 = i0; k0 < K; k0 += kChunk) {
        for (int e = threadIdx.x; e < kChunk * kTile; e += kTileThreads) {
            const int r = e / kTile, c = e % kTile;
            const int64_t k = k0 + r;
            Ai[r][c] = (k < K && i0 + c < K) ? Li[k * K + i0 + c] : 0.0;
            Aj[r][c] = (k < K && j0 + c < K) ? Li[k * K + j0 + c] : 0.0;
        }
        __syncthreads();
        const int kn = (int)(K - k0 < kChunk ? K - k0 : kChunk);
        for (int r = 0; r < kn; ++r) {
            double a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) a[q] = Ai[r][ty + 16 * q];
#pragma unroll
            for (int q = 0; q < 4; ++q) b[q] = Aj[r][tx + 16 * q];
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = __dadd_rn(acc[p][q], __dmul_rn(a[p], b[q]));
        }
        __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t i = i0 + ty + 16 * p, j = j0 + tx + 16 * q;
            if (i < K && j <= i) Hi[i * K + j] = acc[p][q];
        }
}

// U[i][j] = L2[j][i] for j >= i, 0 below the diagonal.
__global__ void gptq_transpose_kernel(const double* __restrict__ L2, int64_t K, double* __restrict__ U) {
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < K * K; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = u / K, j = u - i * K;
        U[u] = j >= i ? L2[j * K + i] : 0.0;
    }
}

// ---------------------------------------------------------------------------
// Sweep
// ---------------------------------------------------------------------------

// Wf[n][p] = W[n][perm[p]] in fp64.
__global__ void gptq_load_rows_kernel(const uint16_t* __restrict__ W, const int32_t* __restrict__ perm, int64_t N,
                                      int64_t K, double* __restrict__ Wf) {
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < N * K; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = u / K, p = u - n * K;
        Wf[u] = bf16_bits_to_f64(W[n * K + perm[p]]);
    }
}

struct SweepArgs {
    const double* U;
    const int32_t* perm;
    const uint16_t* scales;
    const uint16_t* zeros;  // null when symmetric
    double* Wf;
    double* E;       // [N][128] errors of the block
    uint8_t* codes;  // [N][K] original column order, code + 8 when symmetric
    int64_t N, K, b0;
    int bw, g, G, qmin, qmax;
};

// One warp per row, lane l owns the block's columns l, l + 32, l + 64, l + 96.
// U[b0 .. b0+bw)[b0 .. b0+bw) is staged in shared memory.
__global__ void __launch_bounds__(kSweepWarps * 32) gptq_sweep_block_kernel(SweepArgs a) {
    extern __shared__ double Ub[];  // [128][128]
    const int bw = a.bw;
    for (int e = threadIdx.x; e < 128 * 128; e += blockDim.x) {
        const int r = e / 128, c = e % 128;
        Ub[e] = (r < bw && c < bw) ? a.U[(a.b0 + r) * a.K + a.b0 + c] : 0.0;
    }
    __syncthreads();
    const int lane = threadIdx.x % 32;
    const int64_t n = (int64_t)blockIdx.x * kSweepWarps + threadIdx.x / 32;
    if (n >= a.N) return;
    double w[4], s[4];
    int z[4];
    int64_t col[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int jj = lane + 32 * q;
        w[q] = 0.0;
        s[q] = 1.0;
        z[q] = 0;
        col[q] = 0;
        if (jj < bw) {
            col[q] = a.perm[a.b0 + jj];
            w[q] = a.Wf[n * a.K + a.b0 + jj];
            const int64_t gi = col[q] / a.g;
            const uint16_t s16 = a.scales[n * a.G + gi];
            s[q] = (double)__half2float(__ushort_as_half(s16));
            z[q] = a.zeros ? (int)__half2float(__ushort_as_half(a.zeros[n * a.G + gi])) : 0;
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        for (int l = 0; l < 32; ++l) {
            const int j = l + 32 * q;
            if (j >= bw) break;  // uniform across the warp
            double err = 0.0;
            if (lane == l) {
                int code;
                if (isnan(w[q])) {
                    code = z[q];
                } else {
                    double t = __dadd_rn(rint(__ddiv_rn(w[q], s[q])), (double)z[q]);
                    if (t < (double)a.qmin) t = (double)a.qmin;
                    if (t > (double)a.qmax) t = (double)a.qmax;
                    code = (int)t;
                }
                a.codes[n * a.K + col[q]] = (uint8_t)(code - a.qmin);
                // bf16_rn(s (q - z)): the fp32 product is exact
                const float prod = __fmul_rn((float)s[q], (float)(code - z[q]));
                const double wh = (double)__bfloat162float(__float2bfloat16_rn(prod));
                err = __ddiv_rn(__dsub_rn(w[q], wh), Ub[j * 128 + j]);
                a.E[n * 128 + j] = err;
            }
            err = __shfl_sync(0xffffffffu, err, l);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int k = lane + 32 * r;
                if (r >= q && k > j && k < bw) w[r] = __dsub_rn(w[r], __dmul_rn(err, Ub[j * 128 + k]));
            }
        }
    }
}

// Tail: Wf[n][k] -= sum_{j in block} E[n][j] U[b0 + j][k] (ascending j), for
// k >= b0 + bw.  64 x 64 output tiles.
__global__ void __launch_bounds__(kTileThreads) gptq_sweep_tail_kernel(SweepArgs a) {
    const int64_t k1 = a.b0 + a.bw;
    const int64_t n0 = (int64_t)blockIdx.y * kTile, c0 = k1 + (int64_t)blockIdx.x * kTile;
    __shared__ double Es[kTile][kChunk + 1];
    __shared__ double Us[kChunk][kTile + 1];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = 0.0;
    for (int j0 = 0; j0 < a.bw; j0 += kChunk) {
        for (int e = threadIdx.x; e < kTile * kChunk; e += kTileThreads) {
            const int r = e / kChunk, jj = e % kChunk;
            Es[r][jj] = (n0 + r < a.N && j0 + jj < a.bw) ? a.E[(n0 + r) * 128 + j0 + jj] : 0.0;
            const int rr = e / kTile, c = e % kTile;
            Us[rr][c] = (j0 + rr < a.bw && c0 + c < a.K) ? a.U[(a.b0 + j0 + rr) * a.K + c0 + c] : 0.0;
        }
        __syncthreads();
        const int jn = a.bw - j0 < kChunk ? a.bw - j0 : kChunk;
        for (int jj = 0; jj < jn; ++jj) {
            double e4[4], u4[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) e4[p] = Es[ty + 16 * p][jj];
#pragma unroll
            for (int q = 0; q < 4; ++q) u4[q] = Us[jj][tx + 16 * q];
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = __dadd_rn(acc[p][q], __dmul_rn(e4[p], u4[q]));
        }
        __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t n = n0 + ty + 16 * p, k = c0 + tx + 16 * q;
            if (n < a.N && k < a.K) a.Wf[n * a.K + k] = __dsub_rn(a.Wf[n * a.K + k], acc[p][q]);
        }
}

// qweight word c of row n: codes of columns 8c .. 8c+7, low nibble first.
__global__ void gptq_pack_kernel(const uint8_t* __restrict__ codes, int64_t N, int64_t K, int qmin,
                                 uint32_t* __restrict__ qweight) {
    const int64_t words = N * (K / 8);
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < words; u += (int64_t)gridDim.x * blockDim.x) {
        const uint8_t* c = codes + u * 8;
        uint32_t v = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) v |= ((uint32_t)((int)c[j] + qmin) & 0xfu) << (4 * j);
        qweight[u] = v;
    }
}

unsigned tiles(int64_t n) { return (unsigned)((n + kTile - 1) / kTile); }

cudaError_t cholesky_lower(double* A, int64_t K, uint32_t* status, cudaStream_t s) {
    for (int64_t p0 = 0; p0 < K; p0 += kPanel) {
        gptq_chol_diag_kernel<<<1, kDiagThreads, 0, s>>>(A, K, p0, status);
        const int64_t p1 = p0 + kPanel;
        if (p1 >= K) break;
        gptq_chol_panel_kernel<<<(unsigned)((K - p1 + 127) / 128), 128, 0, s>>>(A, K, p0);
        const unsigned t = tiles(K - p1);
        gptq_chol_update_kernel<<<dim3(t, t), kTileThreads, 0, s>>>(A, K, p0);
    }
    return cudaGetLastError();
}

}  // namespace

size_t gptq_workspace_bytes(int64_t N, int64_t K) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return 2 * al((size_t)(K * K) * 8) + al((size_t)(N * K) * 8) + al((size_t)N * 128 * 8) + al((size_t)(N * K)) +
           al((size_t)K * 4) + 256;
}

cudaError_t launch_gptq(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T, int g, int symmetric,
                        int act_order, uint32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                        int32_t* perm_out, void* workspace, uint32_t* status, cudaStream_t s) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    double* B1 = reinterpret_cast<double*>(ws);
    ws += al((size_t)(K * K) * 8);
    double* B2 = reinterpret_cast<double*>(ws);
    ws += al((size_t)(K * K) * 8);
    double* Wf = reinterpret_cast<double*>(ws);
    ws += al((size_t)(N * K) * 8);
    double* E = reinterpret_cast<double*>(ws);
    ws += al((size_t)N * 128 * 8);
    uint8_t* codes = ws;
    ws += al((size_t)(N * K));
    int32_t* perm = reinterpret_cast<int32_t*>(ws);
    ws += al((size_t)K * 4);
    int* nonfinite = reinterpret_cast<int*>(ws);

    cudaError_t e = cudaMemsetAsync(nonfinite, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    // H, dampening, processing order, permuted copy
    const unsigned tk = tiles(K);
    gptq_hessian_kernel<<<dim3(tk, tk), kTileThreads, 0, s>>>(X, T, K, B1);
    gptq_damp_kernel<<<1, kDampThreads, 0, s>>>(B1, K);
    const unsigned kb = (unsigned)((K + 255) / 256);
    gptq_diag_check_kernel<<<kb, 256, 0, s>>>(B1, K, nonfinite);
    gptq_perm_kernel<<<kb, 256, 0, s>>>(B1, K, act_order, perm, nonfinite);
    gptq_gather_kernel<<<1184, 256, 0, s>>>(B1, perm, K, B2);
    // L = chol(Hp) in B2; Linv in B1; H^-1 in B2; chol again; U in B1
    if ((e = cholesky_lower(B2, K, status, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(B1, 0, (size_t)(K * K) * 8, s)) != cudaSuccess) return e;
    for (int64_t r0 = 0; r0 < K; r0 += kPanel) {
        const int64_t r1 = r0 + kPanel < K ? r0 + kPanel : K;
        gptq_trinv_block_kernel<<<(unsigned)((r1 + 127) / 128), 128, 0, s>>>(B2, B1, K, r0);
        if (r1 < K) gptq_trinv_update_kernel<<<dim3(tiles(r1), tiles(K - r1)), kTileThreads, 0, s>>>(B2, B1, K, r0);
    }
    gptq_gram_kernel<<<dim3(tk, tk), kTileThreads, 0, s>>>(B1, K, B2);
    if ((e = cholesky_lower(B2, K, status, s)) != cudaSuccess) return e;
    gptq_transpose_kernel<<<1184, 256, 0, s>>>(B2, K, B1);
    // sweep
    gptq_load_rows_kernel<<<1184, 256, 0, s>>>(W, perm, N, K, Wf);
    SweepArgs a;
    a.U = B1;
    a.perm = perm;
    a.scales = scales;
    a.zeros = symmetric ? nullptr : zeros;
    a.Wf = Wf;
    a.E = E;
    a.codes = codes;
    a.N = N;
    a.K = K;
    a.g = g;
    a.G = (int)(K / g);
    a.qmin = symmetric ? -8 : 0;
    a.qmax = symmetric ? 7 : 15;
    const size_t smem = 128 * 128 * sizeof(double);
    if ((e = cudaFuncSetAttribute(gptq_sweep_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
        return e;
    for (int64_t b0 = 0; b0 < K; b0 += 128) {
        a.b0 = b0;
        a.bw = (int)(K - b0 < 128 ? K - b0 : 128);
        gptq_sweep_block_kernel<<<(unsigned)((N + kSweepWarps - 1) / kSweepWarps), kSweepWarps * 32, smem, s>>>(a);
        if (b0 + a.bw < K)
            gptq_sweep_tail_kernel<<<dim3(tiles(K - b0 - a.bw), tiles(N)), kTileThreads, 0, s>>>(a);
    }
    gptq_pack_kernel<<<1184, 256, 0, s>>>(codes, N, K, a.qmin, qweight);
    if (perm_out) {
        if ((e = cudaMemcpyAsync(perm_out, perm, (size_t)K * 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

}  // namespace wq
