// gemv_kmajor.cu -- W4A16 decode GEMV for a few tokens (M = 2..16) on sm_100a.
//
// y[m, n] = sum_k x_hat[n, k] * x[m, k], x_hat = bf16_rn(s (q - z)), fp32
// accumulation: the fused low-bit path ("path A": packed weights, fused load /
// dequant / matmul, higher-precision accumulation) of "LLM Quantization: GPTQ,
// AWQ, SmoothQuant, FP8, KV Cache (7/10)", section "Without a kernel the
// compression benefit disappears"; decode with a small batch stays bound by
// the weight stream (section "Speed depends on batch and context").
//
// With several tokens the activations are as large as a good part of the
// weights a CTA reads (16 tokens x 4096 k = 128 KB), so they are neither
// staged whole in shared memory nor re-read per tile.  The weights stream
// k-major instead:
// - a CTA owns a run of 16-row blocks (processed in passes of at most
//   kKmMaxRB blocks) and walks K in chunks of 2048 k; a chunk of a pass is one
//   2-D TMA box of 16 rows x 1024 bytes per block, into a ring of slots that
//   thread 0 refills once every warp is done with a chunk;
// - consumer warp w takes k-unit w (128 k) of every chunk, for every row block
//   of the pass: it loads its activation fragments for that k-unit once (from
//   global memory; a chunk ahead for up to 8 tokens), dequantizes each block's
//   16 x 128 tile into m16n8k16 A
//   fragments (the exact split-scale bf16x2 dequant) and issues NT x 8 MMAs
//   (NT = 1 for M <= 8 tokens, 2 for M <= 16) into accumulators that stay in
//   registers for the whole pass;
// - the group constants of the next chunk are fetched while this one is
//   processed and built before the chunk barrier (two buffers);
// - at the end of a pass the partial sums of the 16 k-units are added in a
//   fixed order (warp w + 8 into warp w through shared memory, then the eight
//   sums in warp order): deterministic.
// A lane's fragments follow the k order of the dequant (nibbles p and p + 4 of
// a word share one bf16x2 register); its activation fragments use the same
// order.  Every mbarrier wait is bounded (WQ_DEVFLAG_TIMEOUT).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

constexpr int kKmWarps = 16;                       // warps; one 128-k unit of a chunk each
constexpr int kKmThreads = kKmWarps * 32;          // thread 0 also issues the weight copies
constexpr int kKmChunkK = 128 * kKmWarps;          // 2048 k per chunk
constexpr int kKmChunkWords = kKmChunkK / 8;       // 256 packed words of a row
constexpr int kKmRowBytes = kKmChunkK / 2;         // 1024 bytes of a row per chunk
constexpr int kKmBlockBytes = 16 * kKmRowBytes;    // one 16-row block of a chunk (16 KB)
constexpr int kKmMaxRB = 4;                        // 16-row blocks per pass (accumulators in registers)
constexpr int kKmMaxSlots = 4;
constexpr int kKmSmemBudget = 220 * 1024;
constexpr int kKmMaxItems = 2;                     // group constants per thread per chunk

struct KmLayout {
    int cst_off, red_off, slot_off, total;
};

// bars: full[4]; cst: 16 B per (row, group) of a chunk, two buffers (the next
// chunk's are built while this one's are read); red: fp32 per (warp of the
// upper half, row, token) of a pass, in the same bytes as cst (a pass's last
// chunk barrier frees both buffers, the next pass builds its constants after
// the reduction); slots: 1024-aligned.
__host__ __device__ inline int km_cst_bytes(const KmArgs& a) { return (a.prb * 16 * a.gpc * 16 + 127) & ~127; }
__host__ __device__ inline KmLayout km_layout(const KmArgs& a) {
    KmLayout L;
    L.cst_off = kKmMaxSlots * 8;
    L.red_off = L.cst_off;
    const int cst2 = 2 * km_cst_bytes(a), red = (kKmWarps / 2) * a.prb * 16 * 16 * 4;
    L.slot_off = (L.cst_off + (cst2 > red ? cst2 : red) + 1023) & ~1023;
    L.total = L.slot_off + a.nslots * a.prb * kKmBlockBytes + 1024;  // + base alignment slack
    return L;
}

__device__ __forceinline__ uint4 km_lds(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint4 km_ldg(const void* p) {
    uint4 r;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void km_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Kernel parameters the loops read, pinned in registers once.
struct KmP {
    const uint16_t* X;
    const uint16_t* scales;
    const uint16_t* zeros;
    int M, N, K, G, g_shift, gpc_shift, sym;
};

// B fragments of k-unit ku for the lane (token 8 nt + g8, 32-k slice t4):
// word p of part q is (x[32 t4 + 8 q + p], x[32 t4 + 8 q + p + 4]).
template <int NT>
__device__ __forceinline__ void km_load_x(const KmP& P, int ku, int g8, int t4, uint32_t (&xr)[NT][16]) {
    // tokens past M read token M - 1 (their outputs are discarded); a slice past
    // K (a ragged last k-unit) must be zero, since the weights there are zero
    // codes whose x_hat need not be zero
    const int k0 = ku * 128 + t4 * 32;
    const bool kin = k0 < P.K;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int m = min(nt * 8 + g8, P.M - 1);
        const uint16_t* src = P.X + (int64_t)m * P.K + (kin ? k0 : 0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = km_ldg(src + 8 * q);
            xr[nt][4 * q] = __byte_perm(v.x, v.z, 0x5410);
            xr[nt][4 * q + 1] = __byte_perm(v.x, v.z, 0x7632);
            xr[nt][4 * q + 2] = __byte_perm(v.y, v.w, 0x5410);
            xr[nt][4 * q + 3] = __byte_perm(v.y, v.w, 0x7632);
        }
    }
    if (__any_sync(0xffffffffu, !kin) && !kin) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 16; ++i) xr[nt][i] = 0u;
    }
}

// One 16 x 128 tile for the lane: rows g8 (wa) and g8 + 8 (wa + 8 rows), its
// 32-k slice.  Word q of the slice gives the A fragments of MMAs 2 q and
// 2 q + 1 (register i % 4 of MMA 2 q + i / 4 from nibble pair i / 2 of word q),
// so only one word's fragments are live at a time.
template <int NT>
__device__ __forceinline__ void km_tile(uint32_t wa, uint32_t ca, uint32_t cb, const uint32_t (&xr)[NT][16],
                                        float (&acc)[NT][4]) {
    const uint4 a = km_lds(wa);
    const uint4 b = km_lds(wa + 8 * kKmRowBytes);
    const uint4 ka = km_lds(ca);
    const uint4 kb = km_lds(cb);
    const GroupConsts gca = {ka.x, ka.y, ka.z, ka.w}, gcb = {kb.x, kb.y, kb.z, kb.w};
    const uint32_t va[4] = {a.x, a.y, a.z, a.w}, vb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t f[8];
        f[0] = dequant_pair(va[q], gca);
        f[1] = dequant_pair(vb[q], gcb);
        f[2] = dequant_pair(va[q] >> 4, gca);
        f[3] = dequant_pair(vb[q] >> 4, gcb);
        f[4] = dequant_pair(va[q] >> 8, gca);
        f[5] = dequant_pair(vb[q] >> 8, gcb);
        f[6] = dequant_pair(va[q] >> 12, gca);
        f[7] = dequant_pair(vb[q] >> 12, gcb);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            km_mma(acc[nt], f[0], f[1], f[2], f[3], xr[nt][4 * q], xr[nt][4 * q + 1]);
            km_mma(acc[nt], f[4], f[5], f[6], f[7], xr[nt][4 * q + 2], xr[nt][4 * q + 3]);
        }
    }
}

// The raw scale/zero codes of the (row, group) items of a chunk this thread
// builds (item it = threadIdx.x + i * kKmThreads); fetched a chunk ahead.
struct KmRaw {
    uint16_t s[kKmMaxItems], z[kKmMaxItems];
};
__device__ __forceinline__ void km_fetch_consts(const KmP& P, int row0, int nitems, int chunk, KmRaw& r) {
    const int gk0 = (chunk * kKmChunkK) >> P.g_shift;  // first group of the chunk
#pragma unroll
    for (int i = 0; i < kKmMaxItems; ++i) {
        const int it = (int)threadIdx.x + i * kKmThreads;
        const int rr = it >> P.gpc_shift, gi = it & ((1 << P.gpc_shift) - 1);
        const int row = row0 + rr, grp = gk0 + gi;
        const bool ok = it < nitems && row < P.N && grp < P.G;
        const int64_t idx = (int64_t)row * P.G + grp;
        r.s[i] = ok ? ld_nc_u16(P.scales + idx) : (uint16_t)0;
        r.z[i] = (ok && !P.sym) ? ld_nc_u16(P.zeros + idx) : (uint16_t)0;
    }
}
__device__ __forceinline__ void km_build_consts(const KmP& P, int nitems, const KmRaw& r, uint4* cst) {
#pragma unroll
    for (int i = 0; i < kKmMaxItems; ++i) {
        const int it = (int)threadIdx.x + i * kKmThreads;
        if (it < nitems) {
            // a zero scale code only comes from an item outside the rows or groups
            // (or a zero scale): zero constants, x_hat = 0 either way
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r.s[i] != 0) {
                const GroupConsts k =
                    make_group_consts(r.s[i], P.sym ? 0 : (int)__half2float(__ushort_as_half(r.z[i])), P.sym != 0);
                v = make_uint4(k.s_hi, k.s_lo, k.zm, k.xmask);
            }
            cst[it] = v;
        }
    }
}

// Thread 0: the weight copies of global chunk Q (pass Q / nchunk, chunk Q % nchunk)
// into slot Q % nslots, completing on full[slot].
__device__ __forceinline__ void km_issue(const KmArgs& a, const CUtensorMap* tmap, uint64_t* full, uint8_t* slots,
                                         int Q, int nchunk, int b0, int nb) {
    const int p = Q / nchunk, c = Q - p * nchunk;
    const int pb = min(a.prb, nb - p * a.prb);
    const int row = (b0 + p * a.prb) * 16;
    const int slot = Q % a.nslots;
    uint8_t* dst = slots + (size_t)slot * a.prb * kKmBlockBytes;
    mbar_arrive_expect_tx(&full[slot], (uint32_t)(pb * kKmBlockBytes));
    for (int i = 0; i < pb; ++i) tma_load_2d(dst + i * kKmBlockBytes, tmap, &full[slot], c * kKmChunkWords, row + 16 * i);
}

template <int NT>
__global__ void __launch_bounds__(kKmThreads, 1)
    gemv_kmajor_kernel(const __grid_constant__ CUtensorMap tmap_w, const KmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const KmLayout L = km_layout(a);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint8_t* cst0 = smem + L.cst_off;
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint8_t* slots = smem + L.slot_off;
    const uint32_t slots_s = smem_u32(slots);
    const uint32_t slot_bytes = (uint32_t)(a.prb * kKmBlockBytes);
    const uint32_t cst_bytes = (uint32_t)km_cst_bytes(a);
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the CTA's 16-row blocks [b0, b0 + nb), split evenly over the grid
    const int nblocks = (a.N + 15) / 16;
    const int per = nblocks / (int)gridDim.x, extra = nblocks - per * (int)gridDim.x;
    const int b0 = (int)blockIdx.x * per + min((int)blockIdx.x, extra);
    const int nb = per + ((int)blockIdx.x < extra ? 1 : 0);
    const int prb = pin_i32(a.prb), nslots = pin_i32(a.nslots);
    const int npass = (nb + prb - 1) / prb;
    const int nchunk = (a.K + kKmChunkK - 1) / kKmChunkK;
    const int total = npass * nchunk;

    if (threadIdx.x == 0) {
        for (int i = 0; i < nslots; ++i) mbar_init(&full[i], 1);
        abort_flag = 0;
        fence_mbar_init();
        // the weights do not depend on the previous kernel: the first slots now
        prefetch_tmap(&tmap_w);
        for (int Q = 0; Q < nslots && Q < total; ++Q) km_issue(a, &tmap_w, full, slots, Q, nchunk, b0, nb);
    }
    __syncthreads();
    pdl_launch_dependents();

    KmP P;
    P.X = pin_ptr(static_cast<const uint16_t*>(a.X));
    P.scales = pin_ptr(a.scales);
    P.zeros = pin_ptr(a.zeros);
    P.M = pin_i32(a.M);
    P.N = pin_i32(a.N);
    P.K = pin_i32(a.K);
    P.G = pin_i32(a.G);
    P.g_shift = pin_i32(a.g_shift);
    P.gpc_shift = pin_i32(a.gpc_shift);
    P.sym = pin_i32(a.symmetric);
    void* const Y = pin_ptr(a.Y);
    const int y_fp32 = pin_i32(a.y_fp32);
    const int g8 = lane >> 2, t4 = lane & 3;
    const int gpc = 1 << P.gpc_shift;
    // the lane's slice of every chunk: k offset 128 warp + 32 t4, group gi
    const int gi = min((warp * 128 + t4 * 32) >> P.g_shift, gpc - 1);
    const uint32_t wlane = (uint32_t)(g8 * kKmRowBytes + warp * 64 + t4 * 16);
    const uint32_t clane = 16u * (uint32_t)(g8 * gpc + gi);
    pdl_wait_prior();  // the activations (and y) may belong to the previous kernel

    bool aborted = false;
    int q = 0;
    for (int p = 0; p < npass; ++p) {
        const int pb = min(prb, nb - p * prb);
        const int row0 = (b0 + p * prb) * 16;
        const int nitems = pb * 16 * gpc;
        float acc[kKmMaxRB][NT][4];
#pragma unroll
        for (int rb = 0; rb < kKmMaxRB; ++rb)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[rb][nt][0] = acc[rb][nt][1] = acc[rb][nt][2] = acc[rb][nt][3] = 0.0f;
        // chunk 0's constants (the buffers of the previous pass were released by
        // its closing barrier)
        {
            KmRaw raw;
            km_fetch_consts(P, row0, nitems, 0, raw);
            km_build_consts(P, nitems, raw, reinterpret_cast<uint4*>(cst0));
        }
        // one token tile: the next chunk's activation fragments are loaded a chunk
        // ahead; two: at the start of the chunk (registers)
        constexpr bool kAhead = NT == 1;
        uint32_t xn[NT][16];
        if (kAhead) km_load_x<NT>(P, warp, g8, t4, xn);
        named_sync(1, kKmThreads);
        for (int c = 0; c < nchunk; ++c, ++q) {
            const int slot = q % nslots;
            const int ku = c * kKmWarps + warp;
            const bool more = c + 1 < nchunk;
            uint32_t xr[NT][16];
            if (kAhead) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 16; ++i) xr[nt][i] = xn[nt][i];
                if (more) km_load_x<NT>(P, ku + kKmWarps, g8, t4, xn);
            } else {
                km_load_x<NT>(P, ku, g8, t4, xr);
            }
            KmRaw raw;  // the next chunk's constants, in flight during this chunk
            if (more) km_fetch_consts(P, row0, nitems, c + 1, raw);
            if (!aborted) {
                const uint32_t par = (uint32_t)(q / nslots) & 1u;
                const bool ok = mbar_test_wait(&full[slot], par) || mbar_wait(&full[slot], par, a.status);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) atomicExch(&abort_flag, 1);
                    aborted = true;
                }
            }
            if (!aborted && ku * 128 < P.K) {
                const uint32_t wbase = slots_s + slot * slot_bytes + wlane;
                const uint32_t cbase = smem_u32(cst0) + (uint32_t)(c & 1) * cst_bytes + clane;
#pragma unroll
                for (int rb = 0; rb < kKmMaxRB; ++rb) {
                    if (rb < pb)
                        km_tile<NT>(wbase + rb * kKmBlockBytes, cbase + 16u * (uint32_t)(rb * 16 * gpc),
                                    cbase + 16u * (uint32_t)((rb * 16 + 8) * gpc), xr, acc[rb]);
                }
            }
            if (more)
                km_build_consts(P, nitems, raw, reinterpret_cast<uint4*>(cst0 + ((c + 1) & 1) * cst_bytes));
            // the next chunk's constants are written, and nobody reads this chunk's
            // constants or weights any more: its slot takes chunk q + nslots
            named_sync(1, kKmThreads);
            if (threadIdx.x == 0 && q + nslots < total && !abort_flag) {
                fence_proxy_async_smem();
                km_issue(a, &tmap_w, full, slots, q + nslots, nchunk, b0, nb);
            }
        }
        // ---- the pass's outputs: warps 8..15 park, warps 0..7 add theirs, then
        // the eight sums in warp order ----
        const int prows = prb * 16;
        if (warp >= kKmWarps / 2) {
#pragma unroll
            for (int rb = 0; rb < kKmMaxRB; ++rb) {
                if (rb < pb) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float* r0 = red + ((size_t)(warp - kKmWarps / 2) * prows + rb * 16 + g8) * 16 + nt * 8 + 2 * t4;
                        r0[0] = acc[rb][nt][0];
                        r0[1] = acc[rb][nt][1];
                        r0[8 * 16] = acc[rb][nt][2];
                        r0[8 * 16 + 1] = acc[rb][nt][3];
                    }
                }
            }
        }
        named_sync(1, kKmThreads);
        if (warp < kKmWarps / 2) {
#pragma unroll
            for (int rb = 0; rb < kKmMaxRB; ++rb) {
                if (rb < pb) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float* r0 = red + ((size_t)warp * prows + rb * 16 + g8) * 16 + nt * 8 + 2 * t4;
                        r0[0] = acc[rb][nt][0] + r0[0];
                        r0[1] = acc[rb][nt][1] + r0[1];
                        r0[8 * 16] = acc[rb][nt][2] + r0[8 * 16];
                        r0[8 * 16 + 1] = acc[rb][nt][3] + r0[8 * 16 + 1];
                    }
                }
            }
        }
        named_sync(1, kKmThreads);
        const bool ok = !abort_flag;
        for (int o = threadIdx.x; o < pb * 16 * P.M; o += kKmThreads) {
            const int rr = o / P.M, m = o - rr * P.M;
            const int row = row0 + rr;
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < kKmWarps / 2; ++w) v += red[((size_t)w * prows + rr) * 16 + m];
            if (ok && row < P.N) {
                const int64_t yo = (int64_t)m * P.N + row;
                if (y_fp32)
                    static_cast<float*>(Y)[yo] = v;
                else
                    static_cast<__nv_bfloat16*>(Y)[yo] = __float2bfloat16_rn(v);
            }
        }
        named_sync(1, kKmThreads);  // red is free for the next pass
    }
}

template <int NT>
cudaError_t launch_kmajor(const uint32_t* qweight, KmArgs a, int num_sms, const LaunchOptions& opt,
                          cudaStream_t stream) {
    const int nblocks = (a.N + 15) / 16;
    const int grid = min(num_sms, nblocks);
    a.gpc = a.g >= kKmChunkK ? 1 : kKmChunkK / a.g;
    a.gpc_shift = 0;
    while ((1 << a.gpc_shift) < a.gpc) ++a.gpc_shift;
    // row blocks per pass: at most kKmMaxRB, and few enough that every thread
    // builds at most kKmMaxItems group constants per chunk
    int maxrb = kKmMaxItems * kKmThreads / (16 * a.gpc);
    if (maxrb > kKmMaxRB) maxrb = kKmMaxRB;
    if (maxrb < 1) return cudaErrorNotSupported;
    const int nb_max = (nblocks + grid - 1) / grid;
    const int npass = (nb_max + maxrb - 1) / maxrb;
    a.prb = (nb_max + npass - 1) / npass;
    a.nslots = 0;
    const int fixed = km_layout(a).total;
    int ns = (kKmSmemBudget - fixed) / (a.prb * kKmBlockBytes);
    if (ns > kKmMaxSlots) ns = kKmMaxSlots;
    if (ns < 2) return cudaErrorNotSupported;
    a.nslots = ns;
    const KmLayout L = km_layout(a);
    if (L.total > 227 * 1024) return cudaErrorNotSupported;

    CUtensorMap tmap;
    if (encode_tensor_map_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)(a.K / 8), (uint64_t)a.N,
                             (uint64_t)(a.K / 2), kKmChunkWords, 16, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = gemv_kmajor_kernel<NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kKmThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = opt.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, a);
}

}  // namespace

cudaError_t launch_gemv_kmajor(const uint32_t* qweight, const KmArgs& a, int num_sms, const LaunchOptions& opt,
                               cudaStream_t stream) {
    // whole 2048-k chunks in the tensor map's box, at least one 16-row block
    if (a.M < 1 || a.M > 16 || a.K < kKmChunkK || a.K % 32 != 0 || a.N < 16 || a.g % 32 != 0 || a.g_shift < 0)
        return cudaErrorNotSupported;
    if (a.M <= 8) return launch_kmajor<1>(qweight, a, num_sms, opt, stream);
    return launch_kmajor<2>(qweight, a, num_sms, opt, stream);
}

}  // namespace wq
