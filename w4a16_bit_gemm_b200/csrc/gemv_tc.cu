// gemv_tc.cu -- decode W4A16 GEMV (M = 1, 2) on 5th-generation tensor cores.
//
// y[m, n] = sum_k x_hat[n, k] * x[m, k], x_hat = bf16_rn(s (q - z)), fp32
// accumulation: the fused low-bit path of "LLM Quantization: GPTQ, AWQ,
// SmoothQuant, FP8, KV Cache (7/10)" (section "Without a kernel the
// compression benefit disappears", path A: packed weights -> fused load /
// dequant / matmul -> higher-precision accumulation).
//
// The products run on the tensor pipe with the dequantized weights as the A
// operand in TENSOR MEMORY, so the weights never make a round trip through
// shared memory and the ALU only unpacks and dequantizes.
//
// One M=128 MMA tile = 32 weight rows x 4 k-segments: TMEM lane
// 32*q + 4*r + s holds row (4*r + q) of the tile and segment s.  A "quad" J
// covers k in [256 J, 256 J + 256): segment s owns k in [256 J + 64 s, +64),
// i.e. 8 packed words (two 16-byte loads) per lane and four K=16 MMA steps.
// The B operand (activations) holds one row per (segment, token):
//   B[s*M + m][k'] = x[m][256 J + 64 s + 16 h + perm(k')]  for MMA step 4J + h,
// so D[lane][s*M + m] accumulates segment s of row r for token m; the four
// segments are summed in a fixed order in the epilogue.  Inside each 16-k
// step the k order follows the nibble pairs of the dequant (nibble p and
// p + 4 of a word share one 32-bit TMEM column), and B uses the same order.
//
// Warps: 4 groups of 4 dequant warps (one per TMEM lane quadrant) plus one
// MMA warp per group.  Group g dequantizes the quads J = g (mod 4) of every
// tile into its two A slots (32 TMEM columns each); its four warps arrive on
// a hardware named barrier, the group's MMA warp passes it, issues the four
// MMAs into the group's own accumulator bank and commits the slot's empty
// mbarrier.  Four issuing threads keep the tensor pipe fed (one thread's
// tcgen05.mma issue alone is several times slower), and the named barrier is
// far cheaper than an mbarrier wait for the issuing thread.
//
// Weights: at kernel start one MMA warp streams the CTA's rows into shared
// memory with one 1-D bulk copy per (row, k chunk), completing on one
// mbarrier per (tile, chunk), before the dependency on the previous kernel
// is resolved (programmatic dependent launch).  Rows sit at a pitch of
// K/2 + 16 bytes, and lanes with odd r read their two 16-byte halves in the
// opposite order, so the lane <-> (row, segment) reads hit all eight 16-byte
// bank groups.  Scales and zeros are loaded kPf quads ahead.  The MMA warps
// stage the activations.  Every mbarrier wait is bounded (WQ_DEVFLAG_TIMEOUT).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"
#include "wq_tcgen05.cuh"

namespace wq {
namespace {

constexpr int kTcGroups = 4;
constexpr int kTcDequantWarps = 4 * kTcGroups;
constexpr int kTcWarps = kTcDequantWarps + kTcGroups;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcSlots = 2;             // A slots per group
constexpr int kTcSlotCols = 32;         // four K=16 steps of bf16 A per slot
constexpr int kTcMaxTiles = 4;          // 32-row MMA tiles per CTA
constexpr int kTcMaxChunks = 4;         // k chunks per tile (one weight mbarrier each)
constexpr int kTcDCols = 16;            // MMA N: fp32 accumulator columns per (tile, group) bank
constexpr int kTcTmemCols = 512;        // 256 A columns + up to 4 x 4 x 16 accumulator columns
constexpr int kTcMaxM = 2;              // B rows = 4 * M <= 8
constexpr int kTcGroupBarThreads = 5 * 32;
constexpr int kTcBReadyBar = 1 + 2 * kTcGroups;  // named barrier of the four MMA warps
constexpr int kTcSmemBudget = 220 * 1024;

struct TcLayout {
    int pitch;     // weight row pitch in shared memory (bytes)
    int b_off, w_off, c_off, bar_off, total;
};

// B: K/256 swizzle atoms of 8 rows x 128 B (64 k'), plus one atom of slack
// (the N=16 MMA reads rows 8..15 one atom further; those columns are unused).
// cst: packed group constants, 8 bytes per (row, group), [rows][G].
__host__ __device__ inline TcLayout gemv_tc_layout(int K, int G, int rows_per_cta) {
    TcLayout L;
    L.pitch = K / 2 + 16;
    L.b_off = 0;
    L.w_off = (K / 256 + 1) * 1024;
    L.c_off = L.w_off + ((rows_per_cta * L.pitch + 127) & ~127);
    L.bar_off = L.c_off + ((rows_per_cta * G * 8 + 127) & ~127);
    L.total = L.bar_off + 512 + 1024;  // barriers + alignment slack
    return L;
}

__device__ __forceinline__ void dequant_word_into(uint32_t w, const GroupConsts& gc, uint32_t* out) {
    uint32_t t4[4];
    dequant_word_pairs(w, gc, t4);
    out[0] = t4[0];
    out[1] = t4[1];
    out[2] = t4[2];
    out[3] = t4[3];
}

__global__ void __launch_bounds__(kTcThreads, 1)
    gemv_tc_kernel(const uint32_t* __restrict__ qweight, const GemvArgs a, int rows_per_cta, int nch) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const TcLayout L = gemv_tc_layout(a.K, a.G, rows_per_cta);
    uint8_t* bsm = smem + L.b_off;
    uint8_t* wsm = smem + L.w_off;
    uint2* cst = reinterpret_cast<uint2*>(smem + L.c_off);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.bar_off);  // [group][slot]
    uint64_t* done = empty + kTcGroups * kTcSlots;
    uint64_t* wfull = done + 1;                                       // [tile][chunk]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfull + kTcMaxTiles * kTcMaxChunks);
    __shared__ int abort_flag;
    __shared__ volatile int mma_progress[kTcGroups];  // items whose barrier the MMA warp has passed

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * rows_per_cta;
    const int nrows = min(rows_per_cta, a.N - row0);
    const int T = (nrows + 31) / 32;
    const int rows_t = (nrows + T - 1) / T;  // rows per tile, balanced
    const int Q = a.K / 256;                 // quads per tile
    const int Qc = (Q + nch - 1) / nch;      // quads per weight chunk
    const bool sym = a.symmetric != 0;
    const int M = a.M;
    const uint32_t a_col0 = 0, d_col0 = kTcGroups * kTcSlots * kTcSlotCols;

    // warps 0..15: dequant (group = warp / 4, quadrant = warp % 4); warps 16..19: MMA warp of group warp - 16
    const bool is_mma = warp >= kTcDequantWarps;
    const int grp = is_mma ? warp - kTcDequantWarps : warp >> 2;
    const int pg = grp < Q ? (Q - grp + 3) >> 2 : 0;  // quads per tile owned by the group
    const int nitems = T * pg;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int g = 0; g < kTcGroups; ++g) mma_progress[g] = 0;
        for (int i = 0; i < kTcGroups * kTcSlots; ++i) mbar_init(&empty[i], 1);
        mbar_init(done, kTcGroups);
        for (int i = 0; i < kTcMaxTiles * kTcMaxChunks; ++i) mbar_init(&wfull[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kTcDequantWarps + 1) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    }

    // ---- group constants of the CTA's rows (dequant warps), while the weights are in flight ----
    const int q = warp & 3, r = lane >> 2, s = lane & 3;
    const int rl = 4 * r + q;  // row within a tile
    const bool g_pow2 = a.g_shift >= 0;
    const bool two_groups = (a.g & 63) != 0;  // a 64-k segment may span two groups (g = 32, 96, ...)
    if (!is_mma) {
        const size_t gbase = (size_t)row0 * a.G;
        for (int idx = threadIdx.x; idx < nrows * a.G; idx += kTcDequantWarps * 32) {
            const uint16_t sc = ld_nc_u16(a.scales + gbase + idx);
            const uint16_t zr = sym ? (uint16_t)0 : ld_nc_u16(a.zeros + gbase + idx);
            cst[idx] = pack_consts(sc, sym ? 0 : (int)__half2float(__ushort_as_half(zr)), sym);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (is_mma) {
        // ---------------- MMA warps: weight stream (warp 0) or B staging (warps 1..3), then MMAs ----------------
        if (warp == kTcDequantWarps) {
            // ---- weight stream: one bulk copy per (row, chunk), chunk-major within a tile ----
            if (lane == 0) {
                for (int t = 0; t < T; ++t) {
                    const int rt = min(rows_t, nrows - t * rows_t);
                    for (int c = 0; c < nch; ++c) {
                        const int nq = min(Qc, Q - c * Qc);
                        if (nq > 0) mbar_arrive_expect_tx(&wfull[t * kTcMaxChunks + c], (uint32_t)(rt * nq * 128));
                    }
                }
            }
            __syncwarp();
            for (int t = 0; t < T; ++t) {
                const int rt = min(rows_t, nrows - t * rows_t);
                for (int c = 0; c < nch; ++c) {
                    const int nq = min(Qc, Q - c * Qc);
                    if (nq <= 0) continue;
                    for (int rr = lane; rr < rt; rr += 32) {
                        const int rloc = t * rows_t + rr;
                        const uint8_t* src = reinterpret_cast<const uint8_t*>(qweight) +
                                             (size_t)(row0 + rloc) * (a.K / 2) + (size_t)c * Qc * 128;
                        bulk_copy_g2s(wsm + (size_t)rloc * L.pitch + c * Qc * 128, src, (uint32_t)(nq * 128),
                                      &wfull[t * kTcMaxChunks + c]);
                    }
                }
            }
            if (lane == 0) pdl_launch_dependents();
            pdl_wait_prior();
        } else {
            if (lane == 0) pdl_launch_dependents();
            pdl_wait_prior();  // the activations may come from the previous kernel
            {
                const uint16_t* X = static_cast<const uint16_t*>(a.X);
                const int nwords = a.K / 8;
                const int mt = threadIdx.x - (kTcDequantWarps + 1) * 32;  // MMA warps 1..3
                for (int u = mt; u < M * nwords; u += (kTcGroups - 1) * 32) {
                    const int m = u >= nwords ? 1 : 0, w = u - m * nwords;
                    const uint4 v = *reinterpret_cast<const uint4*>(X + (size_t)m * a.K + 8 * w);
                    const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
                    // k' order inside the word: (x0, x4, x1, x5, x2, x6, x3, x7)
                    uint32_t o[4];
    #pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint32_t lo = (p & 1) ? (xw[p >> 1] >> 16) : (xw[p >> 1] & 0xffffu);
                        const uint32_t hi = (p & 1) ? (xw[2 + (p >> 1)] & 0xffff0000u) : (xw[2 + (p >> 1)] << 16);
                        o[p] = lo | hi;
                    }
                    const int J = w >> 5, o32 = w & 31;
                    const int seg = o32 >> 3, h = (o32 >> 1) & 3, wi = o32 & 1;
                    const int n = seg * M + m;      // B row
                    const int chunk = 2 * h + wi;   // 16-byte chunk of the 128-byte row (step 4J + h)
                    uint8_t* dst = bsm + J * 1024 + n * 128 + ((chunk ^ (n & 7)) << 4);
                    *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                // rows 4M..7 of every atom are read by the MMA but feed unused columns; zero them
                for (int u = mt; u < Q * (8 - 4 * M) * 8; u += (kTcGroups - 1) * 32) {
                    const int atom = u / ((8 - 4 * M) * 8), rem = u - atom * (8 - 4 * M) * 8;
                    const int n = 4 * M + rem / 8, c = rem & 7;
                    *reinterpret_cast<uint4*>(bsm + atom * 1024 + n * 128 + c * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
        }
        named_sync(kTcBReadyBar, kTcGroups * 32);  // B staged by warps 1..3
        const uint32_t idesc = mma_idesc_bf16(128, kTcDCols);
        // descriptor start address field counts 16-byte units: +64 per quad (1 KB), +2 per K=16 step (32 B)
        const uint64_t bdesc0 = sw128_kmajor_desc(smem_u32(bsm));
        const uint32_t a_tm = tmem + a_col0 + kTcSlotCols * kTcSlots * grp;
        uint32_t d_tm = tmem + d_col0 + kTcDCols * grp;  // bank (tile 0, group)
        int J = grp;
        for (int i = 0; i < nitems; ++i) {
            named_sync(1 + 2 * grp + (i & 1), kTcGroupBarThreads);  // the group's four warps wrote slot i % 2
            if (lane == 0) {
                mma_progress[grp] = i + 1;
                tc_fence_after();
                const uint32_t a_slot = a_tm + kTcSlotCols * (i & 1);
                const uint64_t bq = bdesc0 + (uint64_t)(J * 64);
                tc_mma_f16_tmem_a(d_tm, a_slot, bq, idesc, J >= 4 ? 1u : 0u);
                tc_mma_f16_tmem_a(d_tm, a_slot + 8, bq + 2, idesc, 1u);
                tc_mma_f16_tmem_a(d_tm, a_slot + 16, bq + 4, idesc, 1u);
                tc_mma_f16_tmem_a(d_tm, a_slot + 24, bq + 6, idesc, 1u);
                tc_commit(&empty[grp * kTcSlots + (i & 1)]);
            }
            __syncwarp();
            J += 4;
            if (J >= Q) {
                J = grp;
                d_tm += kTcDCols * kTcGroups;  // next tile's bank
            }
        }
        if (lane == 0) tc_commit(done);  // completes once every MMA of this warp has finished
        __syncwarp();
    } else {
        // ---------------- dequant warps ----------------
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t hfirst = (uint32_t)(r & 1) * 16u;  // odd r reads its two halves in the other order
        bool ok = true;
        int t = 0, J = grp, c = 0, c_end = min(Qc, Q);  // weight chunk c holds quads [c * Qc, c_end)
        bool c_ready = false;
        for (int i = 0; i < nitems; ++i) {
            // the weight chunk holding quad J of tile t must have landed
            while (J >= c_end) {
                ++c;
                c_end = min(c_end + Qc, Q);
                c_ready = false;
            }
            if (ok && !c_ready) {
                ok = mbar_wait(&wfull[t * kTcMaxChunks + c], 0, a.status);
                c_ready = true;
            }
            const int rt = min(rows_t, nrows - t * rows_t);
            uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
            if (rl < rt) {
                const uint8_t* base = wsm + (size_t)(t * rows_t + rl) * L.pitch + J * 128 + s * 32;
                const uint4 f = *reinterpret_cast<const uint4*>(base + hfirst);
                const uint4 g = *reinterpret_cast<const uint4*>(base + (16u - hfirst));
                w0 = (r & 1) ? g : f;
                w1 = (r & 1) ? f : g;
            }
            const int slot = i & 1;
            // slot reuse: the MMAs of item i - 2 (issued right after that item's
            // barrier, so this wait is at most one phase behind) must be done.
            // Poll once now; its latency overlaps the first half of the dequant.
            const uint32_t epar = (uint32_t)((i - kTcSlots) >> 1) & 1u;
            const bool early = i < kTcSlots || mbar_test_wait(&empty[grp * kTcSlots + slot], epar);
            const int k0 = 256 * J + 64 * s;
            const uint2* crow = cst + (size_t)(t * rows_t + min(rl, rt - 1)) * a.G;
            const int g0 = g_pow2 ? (k0 >> a.g_shift) : k0 / a.g;
            const GroupConsts gc0 = unpack_consts(crow[g0]);
            uint32_t av[16], bv[16];
            dequant_word_into(w0.x, gc0, av + 0);
            dequant_word_into(w0.y, gc0, av + 4);
            dequant_word_into(w0.z, gc0, av + 8);
            dequant_word_into(w0.w, gc0, av + 12);
            if (ok && !early) ok = mbar_wait(&empty[grp * kTcSlots + slot], epar, a.status);
            if (!__all_sync(0xffffffffu, ok)) ok = false;
            const uint32_t ta = tmem + lane_base + a_col0 + kTcSlotCols * (grp * kTcSlots + slot);
            if (ok) tmem_st_32x32b_x16(ta, av);  // steps 0, 1; in flight during the second half
            GroupConsts gc1 = gc0;
            if (two_groups) gc1 = unpack_consts(crow[g_pow2 ? ((k0 + 32) >> a.g_shift) : (k0 + 32) / a.g]);
            dequant_word_into(w1.x, gc1, bv + 0);
            dequant_word_into(w1.y, gc1, bv + 4);
            dequant_word_into(w1.z, gc1, bv + 8);
            dequant_word_into(w1.w, gc1, bv + 12);
            if (ok) {
                tmem_st_32x32b_x16(ta + 16, bv);  // steps 2, 3
                tc_wait_st();
            }
            tc_fence_before();
            if (!ok && i >= kTcSlots) {
                // after a timed-out wait, still never arrive two uses ahead of the
                // MMA warp on this barrier id (bounded: ~1 s, then give up waiting)
                const uint64_t t0 = global_timer_ns();
                while (mma_progress[grp] < i - 1 && global_timer_ns() - t0 < kWaitLimitNs) {
                }
            }
            named_arrive(1 + 2 * grp + (i & 1), kTcGroupBarThreads);  // always, so the MMA warp never blocks
            J += 4;
            if (J >= Q) {
                J = grp;
                ++t;
                c = 0;
                c_end = min(Qc, Q);
                c_ready = false;
            }
        }
        if (!ok && lane == 0) atomicExch(&abort_flag, 1);

        // ---------------- epilogue: sum the group banks, D -> y ----------------
        const bool fin = __all_sync(0xffffffffu, mbar_wait(done, 0, a.status));
        tc_fence_after();
        pdl_wait_prior();  // y may still be read by the previous kernel
        if (fin) {
            const int ngrp_used = min(kTcGroups, Q);
            for (int tt = grp; tt < T; tt += kTcGroups) {
                float acc[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
                for (int gg = 0; gg < ngrp_used; ++gg) {  // fixed order
                    uint32_t d[8];
                    tmem_ld_32x32b_x8(tmem + lane_base + d_col0 + kTcDCols * (tt * kTcGroups + gg), d);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[c] += __uint_as_float(d[c]);
                }
                const int rt = min(rows_t, nrows - tt * rows_t);
                for (int m = 0; m < M; ++m) {
                    // this lane's segment s, token m sits in column s * M + m
                    const int col = s * M + m;
                    float v = 0.0f;
#pragma unroll
                    for (int cidx = 0; cidx < 8; ++cidx)
                        if (cidx == col) v = acc[cidx];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    if (s == 0 && rl < rt && !abort_flag) {
                        const int row = row0 + tt * rows_t + rl;
                        if (a.y_fp32)
                            static_cast<float*>(a.Y)[(size_t)m * a.N + row] = v;
                        else
                            static_cast<__nv_bfloat16*>(a.Y)[(size_t)m * a.N + row] = __float2bfloat16_rn(v);
                    }
                }
            }
        }
    }
    // every weight copy has completed before the CTA exits (its wait may have been skipped on a
    // timeout or for a chunk no item needed)
    if (warp == kTcDequantWarps && lane < T * kTcMaxChunks) {
        const int c = lane % kTcMaxChunks;  // barrier lane = tile * kTcMaxChunks + c
        if (c < nch && c * Qc < Q) mbar_wait(&wfull[lane], 0, a.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kTcDequantWarps + 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

}  // namespace

cudaError_t launch_gemv_tc(const uint32_t* qweight, const GemvArgs& a, int num_sms, const LaunchOptions& opt,
                           cudaStream_t stream) {
    if (a.M < 1 || a.M > kTcMaxM || a.K % 256 != 0 || a.g % 32 != 0) return cudaErrorNotSupported;
    const int pitch = a.K / 2 + 16;
    const int b_bytes = (a.K / 256 + 1) * 1024;
    int rows_per_cta = (a.N + num_sms - 1) / num_sms;
    const int fit = (kTcSmemBudget - b_bytes - 512 - 1024 - 256) / (pitch + 8 * a.G);
    if (rows_per_cta > fit) rows_per_cta = fit;
    if (rows_per_cta > 32 * kTcMaxTiles) rows_per_cta = 32 * kTcMaxTiles;
    if (rows_per_cta < 1) return cudaErrorNotSupported;
    const TcLayout L = gemv_tc_layout(a.K, a.G, rows_per_cta);
    if (L.total > kTcSmemBudget + 2048) return cudaErrorNotSupported;
    const int grid = (a.N + rows_per_cta - 1) / rows_per_cta;
    // k chunks per tile: about 1 KB of row per chunk copy, at most kTcMaxChunks
    const int Q = a.K / 256;
    int nch = (a.K / 2 + 1023) / 1024;
    if (nch > kTcMaxChunks) nch = kTcMaxChunks;
    if (nch > Q) nch = Q;
    if ((reinterpret_cast<uintptr_t>(qweight) & 15u) != 0 || (reinterpret_cast<uintptr_t>(a.X) & 15u) != 0)
        return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(gemv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = opt.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_tc_kernel, qweight, a, rows_per_cta, nch);
}

}  // namespace wq
