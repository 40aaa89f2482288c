// gemm.cu -- W4A16 prefill GEMM on 5th-generation tensor cores (sm_100a).
//
// Y[m, n] = sum_k X[m, k] * x_hat[n, k], x_hat = bf16_rn(s (q - z)), fp32
// accumulation in tensor memory.  This is the large-batch side of the
// W4A16 layer ("large-batch prefill behaves differently": the layer becomes a
// dense contraction), fed from the same packed artifact as the GEMV.
//
// Per CTA: one output tile of (128*MSUB) tokens x 256 output channels.
// Warp roles (10 warps):
//   warp 0      TMA producer: X tile [128*MSUB x 64] (SWIZZLE_128B, K-major)
//               and the packed weight tile [256 rows x 8 words] (SWIZZLE_32B)
//               into ring 1 (S1 stages).
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (kind::f16, bf16 x
//               bf16 -> fp32, M=128, N=256, K=16) and tcgen05.commit.
//   warps 2-9   dequant producers: thread i expands row i of the packed tile
//               (64 weights) with the exact bf16x2 dequantization and writes
//               the bf16 B tile [256 x 64] in the SWIZZLE_128B K-major layout
//               the MMA descriptor expects, into ring 2 (S2 stages); then the
//               same warps run the epilogue (tcgen05.ld -> bf16/fp32 -> global).
// Barriers: full1/empty1 (ring 1: TMA bytes; MMA commit + 8 producer warps),
//           full2/empty2 (ring 2: 8 producer warps; MMA commit), acc (final
//           MMA commit).  Every wait is bounded (WQ_DEVFLAG_TIMEOUT).
// BITS = 16 is the same kernel on unquantized bf16 weights (the reference
// product X W^T of the AWQ search): TMA writes the B tile [256 x 64] straight
// into ring 1 in the SWIZZLE_128B K-major layout the dequant warps produce
// otherwise, and warps 2-9 only run the epilogue.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "w8_device.cuh"
#include "wq_device.cuh"
#include "wq_kernels.h"
#include "wq_tcgen05.cuh"

namespace wq {
namespace {

constexpr int kBN = 256;        // output channels per tile (MMA N)
constexpr int kBK = 64;         // k per stage (one 128-byte swizzle atom of bf16)
constexpr int kS2 = 2;          // dequantized-W ring depth
constexpr int kGemmThreads = 320;
constexpr int kProducerWarp0 = 2;
constexpr int kNumProducerWarps = 8;

template <int MSUB, int BITS>
struct GemmSmem {
    // X / packed-W ring depth: 4, or 3 when 8-bit or bf16 tiles would not fit
    static constexpr int kS1 = ((BITS == 8 || BITS == 16) && MSUB == 2) ? 3 : 4;
    static constexpr int kATile = 128 * MSUB * kBK * 2;  // bytes
    static constexpr int kWqTile = kBN * kBK * BITS / 8; // packed bytes (bf16 B tile when BITS = 16)
    static constexpr int kBTile = BITS == 16 ? 0 : kBN * kBK * 2;
    static constexpr int kStage1 = kATile + kWqTile;
    static constexpr int kOffA = 0;                           // S1 x A tiles
    static constexpr int kOffWq = kOffA + kS1 * kATile;       // S1 x packed tiles
    static constexpr int kOffB = kOffWq + kS1 * kWqTile;      // S2 x B tiles (none for bf16)
    static constexpr int kOffBar = kOffB + kS2 * kBTile;      // barriers
    static constexpr int kBytes = kOffBar + 256;
    static constexpr int kAlloc = kBytes + 1024;              // + alignment slack
};

template <int MSUB, int BITS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_w4a16_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wq,
                              const GemmArgs a) {
    using SL = GemmSmem<MSUB, BITS>;
    constexpr int kS1 = SL::kS1;
    extern __shared__ uint8_t smem_raw[];
    // the dynamic shared-memory base is only guaranteed 16-byte alignment; the
    // 128-byte swizzle atoms need 1024 (the launch adds 1024 bytes of slack)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full1 = reinterpret_cast<uint64_t*>(smem + SL::kOffBar);
    uint64_t* empty1 = full1 + kS1;
    uint64_t* full2 = empty1 + kS1;
    uint64_t* empty2 = full2 + kS2;
    uint64_t* accbar = empty2 + kS2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (a.M + 128 * MSUB - 1) / (128 * MSUB);
    const int m_tile = blockIdx.x % num_m, n_tile = blockIdx.x / num_m;
    const int m0 = m_tile * 128 * MSUB, n0 = n_tile * kBN;
    const int nkb = (a.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kS1; ++s) {
            mbar_init(&full1[s], 1);
            mbar_init(&empty1[s], BITS == 16 ? 1 : 1 + kNumProducerWarps);
        }
        for (int s = 0; s < kS2; ++s) {
            mbar_init(&full2[s], kNumProducerWarps);
            mbar_init(&empty2[s], 1);
        }
        mbar_init(accbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256 * MSUB);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            prefetch_tmap(&tmap_x);
            prefetch_tmap(&tmap_wq);
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kS1;
                if (kb >= kS1 && !mbar_wait(&empty1[s], (uint32_t)((kb / kS1) - 1) & 1u, a.status)) {
                    atomicExch(abort_flag, 1);
                    break;
                }
                if (*(volatile int*)abort_flag) break;
                mbar_arrive_expect_tx(&full1[s], SL::kStage1);
                uint8_t* As = smem + SL::kOffA + s * SL::kATile;
#pragma unroll
                for (int ms = 0; ms < MSUB; ++ms)
                    tma_load_2d(As + ms * (128 * kBK * 2), &tmap_x, &full1[s], kb * kBK, m0 + 128 * ms);
                if constexpr (BITS == 16)
                    tma_load_2d(smem + SL::kOffWq + s * SL::kWqTile, &tmap_wq, &full1[s], kb * kBK, n0);
                else
                    tma_load_2d(smem + SL::kOffWq + s * SL::kWqTile, &tmap_wq, &full1[s], kb * (kBK * BITS / 32), n0);
                ++issued;
            }
            // drain: wait until the last load into every stage has landed
            for (int kb = issued - 1; kb >= 0 && kb >= issued - kS1; --kb)
                mbar_wait(&full1[kb % kS1], (uint32_t)(kb / kS1) & 1u, a.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = mma_idesc_bf16(128, kBN);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s1 = kb % kS1, s2 = kb % kS2;
                if (!mbar_wait(&full1[s1], (uint32_t)(kb / kS1) & 1u, a.status) ||
                    (BITS != 16 && !mbar_wait(&full2[s2], (uint32_t)(kb / kS2) & 1u, a.status))) {
                    atomicExch(abort_flag, 1);
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + SL::kOffA + s1 * SL::kATile);
                const uint32_t b_addr = BITS == 16 ? smem_u32(smem + SL::kOffWq + s1 * SL::kWqTile)
                                                   : smem_u32(smem + SL::kOffB + s2 * SL::kBTile);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t bdesc = sw128_kmajor_desc(b_addr + kk * 32);
#pragma unroll
                    for (int ms = 0; ms < MSUB; ++ms) {
                        const uint64_t adesc = sw128_kmajor_desc(a_addr + ms * (128 * kBK * 2) + kk * 32);
                        tc_mma_f16(tmem_base + ms * kBN, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                }
                tc_commit(&empty1[s1]);
                if constexpr (BITS != 16) tc_commit(&empty2[s2]);
            }
            tc_commit(accbar);  // completes once every MMA issued above has finished
        }
        __syncwarp();
    } else {
        // ---------------- dequant producers, then epilogue ----------------
        const int i = threadIdx.x - kProducerWarp0 * 32;  // B-tile row 0..255
        const int n = n0 + i;
        const bool nvalid = n < a.N;
        const bool sym = a.symmetric != 0;
        const int kw = a.K * BITS / 32;  // packed words per row
        for (int kb = 0; kb < (BITS == 16 ? 0 : nkb); ++kb) {
            const int s1 = kb % kS1, s2 = kb % kS2;
            if (__any_sync(0xffffffffu, *(volatile int*)abort_flag != 0)) break;
            // group constants for the two 32-k halves of this k block
            const int kbase = kb * kBK;
            const int gA = kbase / a.g, gB = (kbase + 32) / a.g;
            uint8_t* brow = smem + SL::kOffB + s2 * SL::kBTile + i * 128;
            if constexpr (BITS == 16) {
                // no producer work: TMA loads the bf16 B tiles
            } else if constexpr (BITS == 4) {
                GroupConsts cA, cB;
                if (nvalid) {
                    const int64_t ia = (int64_t)n * a.G + gA;
                    cA = make_group_consts(a.scales[ia], sym ? 0 : (int)__half2float(__ushort_as_half(a.zeros[ia])), sym);
                    if (gB != gA && kbase + 32 < a.K) {
                        const int64_t ib = (int64_t)n * a.G + gB;
                        cB = make_group_consts(a.scales[ib], sym ? 0 : (int)__half2float(__ushort_as_half(a.zeros[ib])),
                                               sym);
                    } else {
                        cB = cA;
                    }
                } else {
                    cA = make_group_consts(0x3c00u, 0, sym);
                    cB = cA;
                }
                bool ready = mbar_wait(&full1[s1], (uint32_t)(kb / kS1) & 1u, a.status);
                if (ready && kb >= kS2) ready = mbar_wait(&empty2[s2], (uint32_t)((kb / kS2) - 1) & 1u, a.status);
                if (!__all_sync(0xffffffffu, ready)) {  // warp-uniform give-up
                    if (lane == 0) atomicExch(abort_flag, 1);
                    break;
                }
                // packed row i: 32 bytes, SWIZZLE_32B (16-byte half h stored at h ^ ((i >> 2) & 1))
                const uint8_t* wq = smem + SL::kOffWq + s1 * SL::kWqTile + i * 32;
                const int sw = (i >> 2) & 1;
                const uint4 h0 = *reinterpret_cast<const uint4*>(wq + ((0 ^ sw) << 4));
                const uint4 h1 = *reinterpret_cast<const uint4*>(wq + ((1 ^ sw) << 4));
                const uint32_t words[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty1[s1]);  // packed tile no longer needed by this warp
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t o[4];
                    const bool kval = nvalid && (kb * (kBK / 8) + j) < kw;
                    if (kval) {
                        dequant_word_natural(words[j], j < 4 ? cA : cB, o);
                    } else {
                        o[0] = o[1] = o[2] = o[3] = 0u;
                    }
                    // 16-byte chunk j of a 128-byte row, swizzled by row % 8
                    *reinterpret_cast<uint4*>(brow + ((j ^ (i & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            } else {
                float sA = 0.0f, sB = 0.0f;  // symmetric INT8: scales only
                if (nvalid) {
                    sA = __half2float(__ushort_as_half(a.scales[(int64_t)n * a.G + gA]));
                    sB = (gB != gA && kbase + 32 < a.K) ? __half2float(__ushort_as_half(a.scales[(int64_t)n * a.G + gB]))
                                                         : sA;
                }
                bool ready = mbar_wait(&full1[s1], (uint32_t)(kb / kS1) & 1u, a.status);
                if (ready && kb >= kS2) ready = mbar_wait(&empty2[s2], (uint32_t)((kb / kS2) - 1) & 1u, a.status);
                if (!__all_sync(0xffffffffu, ready)) {  // warp-uniform give-up
                    if (lane == 0) atomicExch(abort_flag, 1);
                    break;
                }
                // packed row i: 64 bytes, SWIZZLE_64B (16-byte chunk h stored at h ^ ((i >> 1) & 3))
                const uint8_t* wq = smem + SL::kOffWq + s1 * SL::kWqTile + i * 64;
                const int sw = (i >> 1) & 3;
                uint32_t words[16];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint4 v = *reinterpret_cast<const uint4*>(wq + ((h ^ sw) << 4));
                    words[4 * h] = v.x;
                    words[4 * h + 1] = v.y;
                    words[4 * h + 2] = v.z;
                    words[4 * h + 3] = v.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty1[s1]);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t o[4] = {0u, 0u, 0u, 0u};
                    if (nvalid && (kb * (kBK / 4) + 2 * j) < kw) {
                        dequant_word_w8(words[2 * j], j < 4 ? sA : sB, o[0], o[1]);
                        dequant_word_w8(words[2 * j + 1], j < 4 ? sA : sB, o[2], o[3]);
                    }
                    *reinterpret_cast<uint4*>(brow + ((j ^ (i & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async_smem();  // make the generic-proxy stores visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&full2[s2]);
        }

        // ---------------- epilogue ----------------
        const bool ok = __all_sync(0xffffffffu, mbar_wait(accbar, 0u, a.status));
        tc_fence_after();
        const int q = warp & 3;              // TMEM lane quadrant this warp may access
        const int h = (warp - kProducerWarp0) >> 2;  // column half
        const bool do_store = ok && !*(volatile int*)abort_flag;
#pragma unroll 1
        for (int ms = 0; ms < MSUB; ++ms) {
            const int m = m0 + 128 * ms + 32 * q + lane;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                const int col0 = h * 128 + cc * 32;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ms * kBN + col0), v);
                tc_wait_ld();
                if (!do_store || m >= a.M) continue;
                const int nb = n0 + col0;
                if (a.y_fp32) {
                    float* yr = static_cast<float*>(a.Y) + (int64_t)m * a.N;
                    if (nb + 32 <= a.N && (a.N & 3) == 0) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            *reinterpret_cast<uint4*>(yr + nb + 4 * j) =
                                make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    } else {
                        for (int j = 0; j < 32; ++j)
                            if (nb + j < a.N) yr[nb + j] = __uint_as_float(v[j]);
                    }
                } else {
                    __nv_bfloat16* yr = static_cast<__nv_bfloat16*>(a.Y) + (int64_t)m * a.N;
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                        pk[j] = bf2_bits(b2);
                    }
                    if (nb + 32 <= a.N && (a.N & 7) == 0) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4*>(yr + nb + 8 * j) =
                                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    } else {
                        for (int j = 0; j < 32; ++j)
                            if (nb + j < a.N)
                                yr[nb + j] = __ushort_as_bfloat16((uint16_t)(pk[j / 2] >> (16 * (j & 1))));
                    }
                }
            }
        }
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // every MMA issued must have completed before the accumulator is freed
        if (lane == 0) mbar_wait(accbar, 0u, a.status);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 256 * MSUB);
    }
}

}  // namespace

namespace {

template <int BITS>
cudaError_t launch_gemm_bits(const GemmArgs& a, int num_sms, cudaStream_t stream) {
    const int n_tiles = (a.N + kBN - 1) / kBN;
    const int m_tiles256 = (a.M + 255) / 256;
    const bool use2 = (int64_t)m_tiles256 * n_tiles >= num_sms;
    constexpr int kWordsPerRowStage = kBK * BITS / 32;
    CUtensorMap tx, tw;
    CUresult cr = encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, (uint64_t)a.K, (uint64_t)a.M,
                                       (uint64_t)a.K * 2, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if constexpr (BITS == 16)
        cr = encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.qweight, (uint64_t)a.K, (uint64_t)a.N,
                                  (uint64_t)a.K * 2, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        cr = encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.qweight, (uint64_t)a.K * BITS / 32,
                                  (uint64_t)a.N, (uint64_t)a.K * BITS / 8, kWordsPerRowStage, kBN,
                                  BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kGemmThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (use2) {
        auto kern = gemm_w4a16_tcgen05_kernel<2, BITS>;
        constexpr int bytes = GemmSmem<2, BITS>::kAlloc;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(m_tiles256 * n_tiles);
        cfg.dynamicSmemBytes = bytes;
        return cudaLaunchKernelEx(&cfg, kern, tx, tw, a);
    }
    auto kern = gemm_w4a16_tcgen05_kernel<1, BITS>;
    constexpr int bytes = GemmSmem<1, BITS>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(((a.M + 127) / 128) * n_tiles);
    cfg.dynamicSmemBytes = bytes;
    return cudaLaunchKernelEx(&cfg, kern, tx, tw, a);
}

static_assert(GemmSmem<2, 4>::kAlloc <= 227 * 1024, "4-bit GEMM shared memory");
static_assert(GemmSmem<2, 8>::kAlloc <= 227 * 1024, "8-bit GEMM shared memory");
static_assert(GemmSmem<2, 16>::kAlloc <= 227 * 1024, "bf16 GEMM shared memory");
static_assert(GemmSmem<1, 16>::kAlloc <= 227 * 1024, "bf16 GEMM shared memory");

}  // namespace

cudaError_t launch_gemm(const GemmArgs& a, int num_sms, const LaunchOptions& opt, cudaStream_t stream) {
    (void)opt;
    if (a.bits == 8) return launch_gemm_bits<8>(a, num_sms, stream);
    if (a.bits == 16) return launch_gemm_bits<16>(a, num_sms, stream);
    return launch_gemm_bits<4>(a, num_sms, stream);
}

}  // namespace wq
