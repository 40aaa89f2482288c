// gemv.cu -- W4A16 decode GEMV (M <= 16) for sm_100a.
//
// y[m, n] = sum_k x_hat[n, k] * x[m, k], x_hat = bf16_rn(s (q - z)), fp32
// accumulation: the "fused load/dequant/matmul" path of "LLM Quantization:
// GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)" (section "Fused low-bit
// kernel"); decode is memory-bound (section "Batch and context"), so the
// kernel is built around streaming the packed weights once at full HBM rate.
//
// Design
// - One CTA per SM.  CTA c owns `rows_per_cta` consecutive output rows and
//   all of K, so no cross-CTA reduction is needed.  Its rows are processed in
//   `npass` passes of BR <= 64 rows.
// - A producer warp streams the packed weights with 2D TMA boxes of
//   [BR rows x 16 words] (128 k per row, 64 bytes) into a ring of shared
//   memory slots; every slot has a "full" mbarrier (TMA transaction bytes) and
//   an "empty" mbarrier (consumer releases).  When the CTA's whole share fits
//   (the common decode case) every load is issued at kernel start.
// - Consumer warp w takes chunks (k blocks) w, w+8, ... of a pass, all BR
//   rows of each; a slot is always read by the same warp, so its phases are
//   awaited in order.  A lane reads one 16-byte run (4 words = 32 k) of rows
//   r and r+8 of a 16-row tile with one LDS.128 each: a quarter-warp reads two
//   consecutive 64-byte rows, i.e. all 32 banks once (conflict-free).
// - Nibbles are dequantized exactly in registers (bf16x2, see wq_device.cuh)
//   straight into mma.sync m16n8k16 A fragments; the k order inside a
//   fragment is permuted to match the nibble pairs (n, n+4) of a word, and the
//   activations (B fragments, read from global/L2) are permuted the same way
//   with byte permutes.  Tokens are the MMA n dimension (8 per n-tile).
// - Partial sums of the consumer warps are reduced in shared memory in a
//   fixed order (deterministic), converted and stored.
// - Programmatic dependent launch: the weight stream does not depend on the
//   previous kernel, so it starts before griddepcontrol.wait; activations are
//   read (and y written) only after it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvThreads = (kGemvConsumerWarps + 1) * 32;
constexpr int kChunkK = 128;  // k per TMA chunk
constexpr int kChunkRowBytes = kChunkK / 2;

__host__ __device__ inline int round_up(int x, int a) { return (x + a - 1) / a * a; }

struct GemvSmemLayout {
    int bar_off, sz_off, red_off, slot_off, total;
};

__host__ __device__ inline GemvSmemLayout gemv_smem_layout(const GemvArgs& a) {
    GemvSmemLayout L;
    const int T = (a.BR + 15) / 16;
    L.bar_off = 0;
    L.sz_off = round_up(16 * a.nslots, 128);
    L.red_off = L.sz_off + round_up(a.BR * a.G * 4, 128);
    L.slot_off = L.red_off + round_up(kGemvConsumerWarps * T * 16 * a.M * 4, 128);
    L.total = L.slot_off + a.nslots * a.slot_bytes;
    return L;
}

__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// B fragments of one 128-wide k block for token n (lane's 32 k values,
// permuted to match dequant_word_pairs).
struct BFrag {
    uint32_t b01[8], b23[8];
};

__device__ __forceinline__ void load_bfrag(BFrag& f, const uint16_t* X, int K, int M, int n, int k0, bool kvalid) {
    if (n < M && kvalid) {
        const uint4* p = reinterpret_cast<const uint4*>(X + (int64_t)n * K + k0);
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = p[i];
        const uint32_t xw[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                 v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int h = 4 * (i / 2) + (i % 2);
            f.b01[i] = __byte_perm(xw[h], xw[h + 2], 0x5410);
            f.b23[i] = __byte_perm(xw[h], xw[h + 2], 0x7632);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f.b01[i] = f.b23[i] = 0u;
    }
}

template <int NT, int TMAX>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_w, const GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const GemvSmemLayout L = gemv_smem_layout(a);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    uint64_t* empty = full + a.nslots;
    uint16_t* sz_s = reinterpret_cast<uint16_t*>(smem + L.sz_off);
    uint16_t* sz_z = sz_s + a.BR * a.G;
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint8_t* slots = smem + L.slot_off;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = (a.BR + 15) / 16;
    const int cta_row0 = blockIdx.x * a.rows_per_cta;
    const int total_chunks = a.npass * a.nkb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.nslots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1u);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kGemvConsumerWarps) {
        // ---------------- producer: TMA weight stream ----------------
        if (lane == 0) {
            prefetch_tmap(&tmap_w);
            const uint32_t box_bytes = (uint32_t)(a.BR * kChunkRowBytes);
            for (int c = 0; c < total_chunks; ++c) {
                const int slot = c % a.nslots;
                if (c >= a.nslots) {
                    const uint32_t parity = (uint32_t)((c / a.nslots) - 1) & 1u;
                    if (!mbar_wait(&empty[slot], parity, a.status)) {
                        atomicExch(&abort_flag, 1);
                        break;
                    }
                }
                const int pass = c / a.nkb, kb = c % a.nkb;
                mbar_arrive_expect_tx(&full[slot], box_bytes);
                tma_load_2d(slots + (size_t)slot * a.slot_bytes, &tmap_w, &full[slot], kb * (kChunkK / 8),
                            cta_row0 + pass * a.BR);
            }
        }
        // let the next kernel in the stream begin its own weight prefetch
        pdl_launch_dependents();
        return;
    }

    // ---------------- consumers ----------------
    const int quad = lane >> 2, tq = lane & 3;
    const int nthreads_c = kGemvConsumerWarps * 32;
    const uint16_t* X = static_cast<const uint16_t*>(a.X);
    const bool sym = a.symmetric != 0;

    pdl_wait_prior();  // activations (and y) may belong to the previous kernel

    for (int pass = 0; pass < a.npass; ++pass) {
        const int row0 = cta_row0 + pass * a.BR;
        // group scales / zeros of this pass's rows
        for (int i = threadIdx.x; i < a.BR * a.G; i += nthreads_c) {
            const int r = i / a.G, j = i - r * a.G;
            const int row = row0 + r;
            uint16_t s = 0x3c00u, z = 0;
            if (row < a.N) {
                s = a.scales[(int64_t)row * a.G + j];
                if (!sym) z = a.zeros[(int64_t)row * a.G + j];
            }
            sz_s[i] = s;
            sz_z[i] = z;
        }
        named_sync(1, nthreads_c);

        float acc[TMAX][NT][4];
#pragma unroll
        for (int t = 0; t < TMAX; ++t)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[t][nt][e] = 0.0f;

        // Chunk c (one 128-wide k block, all BR rows; c counts across passes)
        // belongs to consumer warp c % 8, and a ring's slot count is a multiple
        // of 8, so every
        // use of a slot is consumed by the same warp in order: a warp never
        // waits on a slot phase that is two phases ahead of the barrier.
        const int kb0 = (warp - (pass * a.nkb) % kGemvConsumerWarps + kGemvConsumerWarps) % kGemvConsumerWarps;
        for (int kb = kb0; kb < a.nkb; kb += kGemvConsumerWarps) {
            const int c = pass * a.nkb + kb;
            const int slot = c % a.nslots;
            const int k0 = kb * kChunkK + 32 * tq;
            const bool kvalid = k0 < a.K;
            BFrag bf[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) load_bfrag(bf[nt], X, a.K, a.M, nt * 8 + quad, k0, kvalid);
            const bool landed = mbar_wait(&full[slot], (uint32_t)(c / a.nslots) & 1u, a.status);
            if (!__all_sync(0xffffffffu, landed)) {  // warp-uniform give-up
                if (lane == 0) atomicExch(&abort_flag, 1);
                break;
            }
            const uint8_t* sp = slots + (size_t)slot * a.slot_bytes;
            const int gcol = kvalid ? k0 / a.g : 0;
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t >= T) break;
                const int ra = t * 16 + quad, rb = ra + 8;
                uint32_t pa[4][4], pb[4][4];
                if (kvalid) {
                    uint4 wa = make_uint4(0, 0, 0, 0), wb = make_uint4(0, 0, 0, 0);
                    if (ra < a.BR) wa = *reinterpret_cast<const uint4*>(sp + ra * kChunkRowBytes + tq * 16);
                    if (rb < a.BR) wb = *reinterpret_cast<const uint4*>(sp + rb * kChunkRowBytes + tq * 16);
                    const int ia = min(ra, a.BR - 1) * a.G + gcol, ib = min(rb, a.BR - 1) * a.G + gcol;
                    const GroupConsts ca =
                        make_group_consts(sz_s[ia], sym ? 0 : (int)__half2float(__ushort_as_half(sz_z[ia])), sym);
                    const GroupConsts cb =
                        make_group_consts(sz_s[ib], sym ? 0 : (int)__half2float(__ushort_as_half(sz_z[ib])), sym);
                    const uint32_t wav[4] = {wa.x, wa.y, wa.z, wa.w}, wbv[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        dequant_word_pairs(wav[j], ca, pa[j]);
                        dequant_word_pairs(wbv[j], cb, pb[j]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int p = 0; p < 4; ++p) pa[j][p] = pb[j][p] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int j = i / 2, p = 2 * (i % 2);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816(acc[t][nt], pa[j][p], pb[j][p], pa[j][p + 1], pb[j][p + 1], bf[nt].b01[i],
                                  bf[nt].b23[i]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is the slot's only reader
        }

        // ---- deterministic reduction over consumer warps ----
        const int T16 = T * 16;
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
            if (t < T) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int m0 = nt * 8 + 2 * tq;
                    const int r = t * 16 + quad;
                    float* base = red + (size_t)warp * T16 * a.M;
                    if (m0 < a.M) {
                        base[(r)*a.M + m0] = acc[t][nt][0];
                        base[(r + 8) * a.M + m0] = acc[t][nt][2];
                    }
                    if (m0 + 1 < a.M) {
                        base[(r)*a.M + m0 + 1] = acc[t][nt][1];
                        base[(r + 8) * a.M + m0 + 1] = acc[t][nt][3];
                    }
                }
            }
        }
        named_sync(1, nthreads_c);
        for (int i = threadIdx.x; i < a.BR * a.M; i += nthreads_c) {
            const int m = i / a.BR, r = i - m * a.BR;
            const int row = row0 + r;
            float s = 0.0f;
#pragma unroll 4
            for (int w = 0; w < kGemvConsumerWarps; ++w) s += red[((size_t)w * T16 + r) * a.M + m];
            if (row < a.N && !abort_flag) {
                const int64_t o = (int64_t)m * a.N + row;
                if (a.y_fp32)
                    static_cast<float*>(a.Y)[o] = s;
                else
                    static_cast<__nv_bfloat16*>(a.Y)[o] = __float2bfloat16_rn(s);
            }
        }
        named_sync(1, nthreads_c);  // sz / red reused by the next pass
    }
}

}  // namespace

cudaError_t launch_gemv(const uint32_t* qweight, const GemvArgs& base, int num_sms, const LaunchOptions& opt,
                        cudaStream_t stream) {
    GemvArgs a = base;
    const int NT = a.M <= 8 ? 1 : 2;
    const int br_max = NT == 1 ? 64 : 32;
    const int R = (a.N + num_sms - 1) / num_sms;
    a.npass = (R + br_max - 1) / br_max;
    a.BR = (R + a.npass - 1) / a.npass;
    a.rows_per_cta = a.npass * a.BR;
    a.nkb = (a.K + kChunkK - 1) / kChunkK;
    a.slot_bytes = round_up(a.BR * kChunkRowBytes, 128);
    const int grid = (a.N + a.rows_per_cta - 1) / a.rows_per_cta;

    // shared memory budget: whole share if it fits, else a ring
    const int budget = 100 * 1024;
    a.nslots = 1;
    GemvSmemLayout L = gemv_smem_layout(a);
    const int fixed = L.slot_off;
    const int nslots_fit = (budget - fixed) / a.slot_bytes;
    const int total_chunks = a.npass * a.nkb;
    int nslots;
    if (nslots_fit >= total_chunks && total_chunks <= 64) {
        nslots = total_chunks;  // whole share resident: every slot used once
    } else {
        // ring: every slot is owned by one consumer warp, so the count is a
        // multiple of the warp count
        nslots = nslots_fit < 64 ? nslots_fit : 64;
        nslots = nslots / kGemvConsumerWarps * kGemvConsumerWarps;
        if (nslots < kGemvConsumerWarps) return cudaErrorInvalidConfiguration;
    }
    a.nslots = nslots;
    L = gemv_smem_layout(a);
    if (L.total > 220 * 1024) return cudaErrorInvalidConfiguration;

    CUtensorMap tmap;
    CUresult cr = encode_tensor_map_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)(a.K / 8),
                                       (uint64_t)a.N, (uint64_t)(a.K / 2), kChunkK / 8, (uint32_t)a.BR,
                                       CU_TENSOR_MAP_SWIZZLE_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;

    void (*kern)(const CUtensorMap, const GemvArgs) = NT == 1 ? gemv_w4a16_kernel<1, 4> : gemv_w4a16_kernel<2, 2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = opt.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, a);
}

}  // namespace wq
