// gemv.cu -- W4A16 decode GEMV (M <= 16) for sm_100a.
//
// y[m, n] = sum_k x_hat[n, k] * x[m, k], x_hat = bf16_rn(s (q - z)), fp32
// accumulation: the "fused load/dequant/matmul" path of "LLM Quantization:
// GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)" (section "Fused low-bit
// kernel"); decode is memory-bound (section "Batch and context"), so the
// kernel is built around streaming the packed weights once at full HBM rate
// while the exact in-register dequantization runs beside the stream.
//
// Design
// - CTA c owns `rows_per_cta` consecutive output rows and all of K (no
//   cross-CTA reduction), processed in `npass` passes of BR <= 64 rows, each
//   pass in T tiles of BRT = ceil(BR/T) <= 16 rows (the MMA's 16 rows).
//   A CTA needs at most ~110 KB of shared memory and 288 threads x <= 112
//   registers, so two CTAs fit on one SM: with programmatic dependent launch
//   the next GEMV in the stream streams its weights while this one computes.
// - A producer warp streams the packed weights with one 2D TMA box per chunk,
//   [BRT rows x 256 words] (1 KB of contiguous codes per row; a chunk is one
//   tile x one 2048-k segment).  Few large requests keep the copy engine far
//   from its per-request issue cost (boxes of many 64-byte row pieces cannot
//   stream at HBM rate).  Rows past N and words past K are zero-filled by the
//   TMA unit; MMA rows BRT..15 of a tile read stale slot rows and their
//   outputs are discarded.
//   Chunks (pass, tile, k segment) flow through a ring of slots with a "full"
//   (TMA bytes) and an "empty" (one arrival per consumer warp) mbarrier.
// - Every consumer warp consumes every chunk in order (the warps split the
//   chunk's 16 k blocks), so a parity wait never runs ahead of a slot phase.
// - Before a pass the consumers precompute, per (row, group), the constants of
//   the exact bf16x2 dequantization (wq_device.cuh) into shared memory, and
//   stage the activations once, permuted into mma.sync B-fragment order.
// - A unit is (16-row tile, 128-wide k block).  A lane reads one 16-byte run
//   (4 words = 32 k) of rows r and r+8 with one LDS.128 each, dequantizes it in
//   registers straight into m16n8k16 A fragments (k order inside a fragment
//   follows the nibble pairs (n, n+4) of a word; the staged activations use
//   the same order, the sum being order-free) and issues the MMAs.  Tokens are
//   the MMA n dimension (8 per n-tile).
// - Partial sums of the consumer warps are reduced in shared memory in a fixed
//   order (deterministic), converted and stored.
// - Weights, scales and zeros are static, so their loads start before
//   griddepcontrol.wait; activations are read and y written only after it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"

namespace wq {
namespace {

constexpr int kNW = 8;                 // consumer warps
constexpr int kThreads = (kNW + 1) * 32;
constexpr int kChunkK = 128;           // k per MMA k block (16 packed words)
constexpr int kSegWords = 256;         // TMA box width: 256 words = 2048 k = 1 KB per row
constexpr int kSegK = kSegWords * 8;
constexpr int kKbPerSeg = kSegK / kChunkK;  // 16
constexpr int kSlotBytes = 16 * kSegWords * 4;  // 16 KB: a 16-row tile x one segment
constexpr int kMaxBR = 64;                      // rows per pass (red buffer size)
constexpr int kMaxSlots = 8;
constexpr int kSmemBudget = 110 * 1024;
constexpr int kXsMaxBytes = 32 * 1024;

__host__ __device__ inline int round_up(int x, int a) { return (x + a - 1) / a * a; }

struct GemvSmemLayout {
    int bar_off, cst_off, xs_off, red_off, slot_off, total;
};

// Constants are 8 bytes per (row, group): {s_hi | s_lo << 16, zm | xmask-half}.
__host__ __device__ inline GemvSmemLayout gemv_smem_layout(const GemvArgs& a) {
    GemvSmemLayout L;
    const int T = (a.BR + 15) / 16;
    L.bar_off = 0;
    L.cst_off = round_up(16 * a.nslots, 128);
    L.xs_off = L.cst_off + round_up(a.BR * a.G * 8, 128);
    L.red_off = L.xs_off + round_up(a.xs_bytes, 128);
    L.slot_off = round_up(L.red_off + kNW * T * 16 * a.M * 4, 1024);
    L.total = L.slot_off + a.nslots * kSlotBytes + 1024;  // + base alignment slack
    return L;
}

__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


// B fragments of one 128-wide k block for token n: the lane's 32 k values
// (k0 .. k0+31), paired to match dequant_word_pairs: MMA i takes
// b01 = (x[L], x[L+4]) and b23 = (x[L+1], x[L+5]) with L = 8*(i/2) + 2*(i%2).
struct BFrag {
    uint32_t b01[8], b23[8];
};

__device__ __forceinline__ void permute_x32(const uint4 v[4], BFrag& f) {
    const uint32_t xw[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                             v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int h = 4 * (i / 2) + (i % 2);
        f.b01[i] = __byte_perm(xw[h], xw[h + 2], 0x5410);
        f.b23[i] = __byte_perm(xw[h], xw[h + 2], 0x7632);
    }
}

__device__ __forceinline__ void load_bfrag_global(BFrag& f, const uint16_t* X, int K, int M, int n, int k0,
                                                  bool kvalid) {
    if (n < M && kvalid) {
        const uint4* p = reinterpret_cast<const uint4*>(X + (int64_t)n * K + k0);
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = p[i];
        permute_x32(v, f);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f.b01[i] = f.b23[i] = 0u;
    }
}

// Staged layout: xs[kb][i][n][tq] (uint4), i = 0..3 holding b01[0..3],
// b01[4..7], b23[0..3], b23[4..7]; consecutive lanes read consecutive 16 B.
__device__ __forceinline__ void load_bfrag_smem(BFrag& f, const uint4* xs, int M, int kb, int n, int tq) {
    if (n < M) {
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = xs[((kb * 4 + i) * M + n) * 4 + tq];
        f.b01[0] = v[0].x; f.b01[1] = v[0].y; f.b01[2] = v[0].z; f.b01[3] = v[0].w;
        f.b01[4] = v[1].x; f.b01[5] = v[1].y; f.b01[6] = v[1].z; f.b01[7] = v[1].w;
        f.b23[0] = v[2].x; f.b23[1] = v[2].y; f.b23[2] = v[2].z; f.b23[3] = v[2].w;
        f.b23[4] = v[3].x; f.b23[5] = v[3].y; f.b23[6] = v[3].z; f.b23[7] = v[3].w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f.b01[i] = f.b23[i] = 0u;
    }
}

__device__ __forceinline__ void store_xs(uint4* xs, int M, int kb, int n, int t4, const BFrag& f) {
    xs[((kb * 4 + 0) * M + n) * 4 + t4] = make_uint4(f.b01[0], f.b01[1], f.b01[2], f.b01[3]);
    xs[((kb * 4 + 1) * M + n) * 4 + t4] = make_uint4(f.b01[4], f.b01[5], f.b01[6], f.b01[7]);
    xs[((kb * 4 + 2) * M + n) * 4 + t4] = make_uint4(f.b23[0], f.b23[1], f.b23[2], f.b23[3]);
    xs[((kb * 4 + 3) * M + n) * 4 + t4] = make_uint4(f.b23[4], f.b23[5], f.b23[6], f.b23[7]);
}

// 8-byte packed constants -> the four bf16x2 words of GroupConsts.
// NCH independent accumulator chains per warp: consecutive MMAs of a unit go
// to different chains, so the MMA result latency is not on the critical path.
template <int NT, int NCH>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 2 : 1)
    gemv_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_w, const GemvArgs a) {
    // The dynamic shared-memory base is only guaranteed 16-byte alignment;
    // round up (the launch adds slack) so TMA destinations are 1024-aligned.
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const GemvSmemLayout L = gemv_smem_layout(a);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    uint64_t* empty = full + a.nslots;
    uint2* cst = reinterpret_cast<uint2*>(smem + L.cst_off);
    uint4* xs = reinterpret_cast<uint4*>(smem + L.xs_off);
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint8_t* slots = smem + L.slot_off;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, BRT = a.BRT;  // tiles per pass, rows per tile (<= 16)
    const int cta_row0 = blockIdx.x * a.rows_per_cta;
    const int total_chunks = a.npass * T * a.nks;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.nslots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kNW);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kNW) {
        // ---------------- producer: TMA weight stream ----------------
        if (lane == 0) {
            prefetch_tmap(&tmap_w);
            for (int c = 0; c < total_chunks; ++c) {
                const int slot = c % a.nslots;
                if (c >= a.nslots &&
                    !mbar_wait(&empty[slot], (uint32_t)((c / a.nslots) - 1) & 1u, a.status)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                const int seg = c % a.nks, pt = c / a.nks;
                const int t = pt % T, pass = pt / T;
                // one box [BRT rows x 256 words] per chunk
                mbar_arrive_expect_tx(&full[slot], (uint32_t)(BRT * kSegWords * 4));
                tma_load_2d(slots + (size_t)slot * kSlotBytes, &tmap_w, &full[slot], seg * kSegWords,
                            cta_row0 + pass * a.BR + t * BRT);
            }
        }
        __syncwarp();
        // let the next kernel in the stream begin its own weight prefetch
        pdl_launch_dependents();
        return;
    }

    // ---------------- consumers ----------------
    const int quad = lane >> 2, tq = lane & 3;
    const int nthreads_c = kNW * 32;
    const uint16_t* X = static_cast<const uint16_t*>(a.X);
    const bool sym = a.symmetric != 0;
    int c = 0;  // next chunk, in the producer's order

    for (int pass = 0; pass < a.npass; ++pass) {
        const int row0 = cta_row0 + pass * a.BR;
        const int nitems = a.BR * a.G;
        // Prologue: all global loads issued before any is used.  Round 0
        // covers kPf (row, group) items per thread; scales/zeros are static,
        // so they are read before griddepcontrol.wait, activations after it.
        constexpr int kPf = 4;
        uint16_t sv[kPf], zv[kPf];
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
            const int i = threadIdx.x + u * nthreads_c;
            sv[u] = 0x3c00u;
            zv[u] = 0;
            if (i < nitems) {
                const int r = i / a.G, row = row0 + r;
                if (row < a.N) {
                    const int64_t gi = (int64_t)row * a.G + (i - r * a.G);
                    sv[u] = a.scales[gi];
                    if (!sym) zv[u] = a.zeros[gi];
                }
            }
        }
        const int nx = (pass == 0 && a.xs_bytes > 0) ? a.nkb * a.M * 4 : 0;
        uint4 xv[4];
        if (pass == 0) {
            pdl_wait_prior();  // activations (and y) may belong to the previous kernel
            if ((int)threadIdx.x < nx) {
                const int it = threadIdx.x;
                const int k0 = ((it >> 2) / a.M) * kChunkK + 32 * (it & 3);
                const uint4* p = reinterpret_cast<const uint4*>(X + (int64_t)((it >> 2) % a.M) * a.K + k0);
#pragma unroll
                for (int q = 0; q < 4; ++q) xv[q] = k0 < a.K ? p[q] : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
            const int i = threadIdx.x + u * nthreads_c;
            if (i < nitems) cst[i] = pack_consts(sv[u], sym ? 0 : (int)__half2float(__ushort_as_half(zv[u])), sym);
        }
        for (int it = threadIdx.x; it < nx; it += nthreads_c) {
            const int t4 = it & 3, n = (it >> 2) % a.M, kb = (it >> 2) / a.M;
            BFrag f;
            if (it == (int)threadIdx.x) {
                permute_x32(xv, f);
            } else {
                const int k0 = kb * kChunkK + 32 * t4;
                load_bfrag_global(f, X, a.K, a.M, n, k0, k0 < a.K);
            }
            store_xs(xs, a.M, kb, n, t4, f);
        }
        for (int i = threadIdx.x + kPf * nthreads_c; i < nitems; i += nthreads_c) {
            const int r = i / a.G, row = row0 + r;
            uint16_t s16 = 0x3c00u, z16 = 0;
            if (row < a.N) {
                const int64_t gi = (int64_t)row * a.G + (i - r * a.G);
                s16 = a.scales[gi];
                if (!sym) z16 = a.zeros[gi];
            }
            cst[i] = pack_consts(s16, sym ? 0 : (int)__half2float(__ushort_as_half(z16)), sym);
        }
        named_sync(1, nthreads_c);

        // red[warp][tile row][m]: this warp's partial sums for the pass
        float* wred = red + (size_t)warp * (T * 16) * a.M;
        bool aborted = false;
        for (int t = 0; t < T; ++t) {
            float acc[NCH][NT][4];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[ch][nt][e] = 0.0f;
            const int ra = t * BRT + quad, rb = ra + 8;  // pass rows of the fragment
            const int ca_row = min(ra, a.BR - 1) * a.G, cb_row = min(rb, a.BR - 1) * a.G;
            for (int seg = 0; seg < a.nks && !aborted; ++seg, ++c) {
                const int slot = c % a.nslots;
                const bool landed = mbar_wait(&full[slot], (uint32_t)(c / a.nslots) & 1u, a.status);
                if (!__all_sync(0xffffffffu, landed)) {
                    if (lane == 0) atomicExch(&abort_flag, 1);
                    aborted = true;
                    break;
                }
                const uint8_t* sp = slots + (size_t)slot * kSlotBytes;
                const int kb_begin = seg * kKbPerSeg;
                const int kb_end = min(a.nkb, kb_begin + kKbPerSeg);
                for (int kb = kb_begin + warp; kb < kb_end; kb += kNW) {
                    const int k0 = kb * kChunkK + 32 * tq;
                    const bool kvalid = k0 < a.K;
                    BFrag bf[NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (a.xs_bytes > 0)
                            load_bfrag_smem(bf[nt], xs, a.M, kb, nt * 8 + quad, tq);
                        else
                            load_bfrag_global(bf[nt], X, a.K, a.M, nt * 8 + quad, k0, kvalid);
                    }
                    // slot rows: BRT x 1 KB (rows >= BRT hold stale data and only feed
                    // discarded MMA rows); this k block at byte (kb - kb_begin) * 64
                    const uint8_t* kp = sp + (kb - kb_begin) * (kChunkK / 2) + tq * 16;
                    const uint4 wa = *reinterpret_cast<const uint4*>(kp + quad * (kSegWords * 4));
                    const uint4 wb = *reinterpret_cast<const uint4*>(kp + (quad + 8) * (kSegWords * 4));
                    GroupConsts ka = {0u, 0u, 0u, 0u}, kc = {0u, 0u, 0u, 0u};
                    if (kvalid) {
                        const int gcol = a.g_shift >= 0 ? (k0 >> a.g_shift) : k0 / a.g;
                        ka = unpack_consts(cst[ca_row + gcol]);
                        kc = unpack_consts(cst[cb_row + gcol]);
                    }
                    // zero constants give x_hat = 0 past K (with zero-filled words)
                    const uint32_t wav[4] = {wa.x, wa.y, wa.z, wa.w}, wbv[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // word j of rows r and r+8 feeds MMAs 2j and 2j+1
                        uint32_t pa[4], pb[4];
                        dequant_word_pairs(wav[j], ka, pa);
                        dequant_word_pairs(wbv[j], kc, pb);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int i = 2 * j + h, p = 2 * h;
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_16816(acc[i % NCH][nt], pa[p], pb[p], pa[p + 1], pb[p + 1], bf[nt].b01[i],
                                          bf[nt].b23[i]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
            }
            // tile done: fold the chains and park this warp's partial sums
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[e] = acc[0][nt][e];
#pragma unroll
                    for (int ch = 1; ch < NCH; ++ch) v[e] += acc[ch][nt][e];
                }
                const int m0 = nt * 8 + 2 * tq;
                const int r = t * 16 + quad;
                if (m0 < a.M) {
                    wred[r * a.M + m0] = v[0];
                    wred[(r + 8) * a.M + m0] = v[2];
                }
                if (m0 + 1 < a.M) {
                    wred[r * a.M + m0 + 1] = v[1];
                    wred[(r + 8) * a.M + m0 + 1] = v[3];
                }
            }
            if (aborted) break;
        }

        named_sync(1, nthreads_c);
        for (int i = threadIdx.x; i < a.BR * a.M; i += nthreads_c) {
            const int m = i / a.BR, r = i - m * a.BR;
            const int row = row0 + r;
            const int rr = (r / BRT) * 16 + (r % BRT);  // row within the red tile layout
            float s = 0.0f;
#pragma unroll
            for (int w = 0; w < kNW; ++w) s += red[((size_t)w * T * 16 + rr) * a.M + m];
            if (row < a.N && !abort_flag) {
                const int64_t o = (int64_t)m * a.N + row;
                if (a.y_fp32)
                    static_cast<float*>(a.Y)[o] = s;
                else
                    static_cast<__nv_bfloat16*>(a.Y)[o] = __float2bfloat16_rn(s);
            }
        }
        named_sync(1, nthreads_c);  // cst / red reused by the next pass
        if (abort_flag) break;
    }
}

// ------------------------------------------------------------------------
// M = 1: dequant on the CUDA cores, products and sums on the tensor pipe
// (fp32 accumulation).  One token fills 1/8 of the m16n8k16 n dimension, but
// the MMA still replaces the per-weight multiply-add and register splitting
// the CUDA cores would otherwise spend on every weight.
// - A CTA's rows are one contiguous byte range of qweight, so the producer
//   moves them with 1D bulk copies of <= 16 KB (the copy engine streams these
//   at HBM rate; many small row pieces it cannot).  A chunk is RC consecutive
//   rows; chunks are resident when they fit, else they cycle through a ring
//   where every consumer warp consumes every chunk in order.
// - Products on the tensor pipe with mma.sync m16n8k16: a unit is (16-row
//   block, 128-k step).  Lane (g, t) = (lane / 4, lane % 4) dequantizes the
//   32-k slice 4 * step + t of rows g and g + 8 (one 16-byte word load per
//   row); its bf16x2 pairs (nibble p, nibble p + 4) are A-fragment registers
//   directly, and the staged activation pairs are the matching B fragments
//   (all 8 columns of B carry the same token, so any column of D is y).
//   Steps are dealt round-robin to 16 consumer warps; each warp parks its
//   per-row partial, and a fixed-order sum per row finishes (deterministic).
// ------------------------------------------------------------------------

constexpr int kM1Warps = 16;
constexpr int kM1Threads = (kM1Warps + 1) * 32;
constexpr int kM1StepK = 128;             // k per unit (4 lanes x 32 k)
constexpr int kM1SmemBudget = 200 * 1024;
constexpr int kM1MaxSlots = 16;
constexpr int kM1CopyPiece = 16384;

struct GemvM1Layout {
    int bar_off, cst_off, xs_off, red_off, slot_off, total;
};

// cst: 16 B per (row, group); xs: 64 B per 32-k slice (activation pairs
// matching the nibble pairs); red: [rows][consumer warps] floats.
__host__ __device__ inline GemvM1Layout gemv_m1_layout(const GemvArgs& a) {
    GemvM1Layout L;
    const int nsl = (a.K + 31) / 32;
    L.bar_off = 0;
    L.cst_off = round_up(16 * a.nslots, 128);
    L.xs_off = L.cst_off + round_up(a.BR * a.G * 16, 128);
    L.red_off = L.xs_off + round_up(nsl * 64, 128);
    L.slot_off = round_up(L.red_off + a.BR * kM1Warps * 4, 1024);
    L.total = L.slot_off + a.nslots * a.slot_bytes + 1024;
    return L;
}

__global__ void __launch_bounds__(kM1Threads, 1)
    gemv_m1_kernel(const uint32_t* __restrict__ qweight, const GemvArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const GemvM1Layout L = gemv_m1_layout(a);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    uint64_t* empty = full + a.nslots;
    uint4* cst = reinterpret_cast<uint4*>(smem + L.cst_off);
    uint4* xs = reinterpret_cast<uint4*>(smem + L.xs_off);
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint8_t* slots = smem + L.slot_off;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * a.rows_per_cta;                 // single pass: BR rows
    const int nrows = min(a.BR, a.N - row0);                      // valid rows of this CTA
    const int RC = a.BRT;                                         // rows per chunk
    const int nch = (nrows + RC - 1) / RC;
    const int64_t row_bytes = (int64_t)a.K / 2;
    const int nsl = (a.K + 31) / 32;
    const int nks = (a.K + kM1StepK - 1) / kM1StepK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.nslots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kM1Warps);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // the next launch may start as soon as SM resources allow: it only streams
    // weights and scales before its own griddepcontrol.wait
    pdl_launch_dependents();

    if (warp == kM1Warps) {
        // ---------------- producer: contiguous bulk copies ----------------
        if (lane == 0) {
            const char* qbytes = reinterpret_cast<const char*>(qweight);
            for (int c = 0; c < nch; ++c) {
                const int slot = c % a.nslots;
                if (c >= a.nslots &&
                    !mbar_wait(&empty[slot], (uint32_t)((c / a.nslots) - 1) & 1u, a.status)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                const int rows = min(RC, nrows - c * RC);
                const int64_t bytes = rows * row_bytes;
                const char* src = qbytes + (int64_t)(row0 + c * RC) * row_bytes;
                uint8_t* dst = slots + (size_t)slot * a.slot_bytes;
                mbar_arrive_expect_tx(&full[slot], (uint32_t)bytes);
                for (int64_t off = 0; off < bytes; off += kM1CopyPiece) {
                    const uint32_t n = (uint32_t)min((int64_t)kM1CopyPiece, bytes - off);
                    bulk_copy_g2s(dst + off, src + off, n, &full[slot]);
                }
            }
        }
        __syncwarp();
        return;
    }

    // ---------------- consumers ----------------
    const int nthreads_c = kM1Warps * 32;
    const uint16_t* X = static_cast<const uint16_t*>(a.X);
    const bool sym = a.symmetric != 0;
    const int nitems = nrows * a.G;
    constexpr int kPf = 4;
    uint16_t sv[kPf], zv[kPf];
#pragma unroll
    for (int u = 0; u < kPf; ++u) {
        const int i = threadIdx.x + u * nthreads_c;
        sv[u] = 0x3c00u;
        zv[u] = 0;
        if (i < nitems) {
            const int64_t gi = (int64_t)row0 * a.G + i;
            sv[u] = a.scales[gi];
            if (!sym) zv[u] = a.zeros[gi];
        }
    }
    pdl_wait_prior();  // activations (and y) may belong to the previous kernel
    uint4 xv[4];
    if ((int)threadIdx.x < nsl) {
        const uint4* p = reinterpret_cast<const uint4*>(X + threadIdx.x * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = p[q];
    }
#pragma unroll
    for (int u = 0; u < kPf; ++u) {
        const int i = threadIdx.x + u * nthreads_c;
        if (i < nitems) {
            const GroupConsts g = make_group_consts(sv[u], sym ? 0 : (int)__half2float(__ushort_as_half(zv[u])), sym);
            cst[i] = make_uint4(g.s_hi, g.s_lo, g.zm, g.xmask);
        }
    }
    // activation slices, paired like the nibbles: (x[8j+p], x[8j+p+4])
    for (int it = threadIdx.x; it < nsl; it += nthreads_c) {
        uint4 v[4];
        if (it == (int)threadIdx.x) {
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = xv[q];
        } else {
            const uint4* p = reinterpret_cast<const uint4*>(X + it * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = p[q];
        }
        const uint32_t xw[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                 v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
        uint32_t pw[16];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                // element e of the slice sits in half (e & 1) of word e >> 1
                const int e0 = 8 * j + p, e1 = 8 * j + p + 4;
                const uint32_t lo = (e0 & 1) ? (xw[e0 >> 1] >> 16) : (xw[e0 >> 1] & 0xffffu);
                const uint32_t hi = (e1 & 1) ? (xw[e1 >> 1] & 0xffff0000u) : (xw[e1 >> 1] << 16);
                pw[4 * j + p] = lo | hi;
            }
        uint4* dst = xs + it * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3]);
    }
    for (int i = threadIdx.x + kPf * nthreads_c; i < nitems; i += nthreads_c) {
        const int64_t gi = (int64_t)row0 * a.G + i;
        const uint16_t s16 = a.scales[gi];
        const uint16_t z16 = sym ? (uint16_t)0 : a.zeros[gi];
        const GroupConsts g = make_group_consts(s16, sym ? 0 : (int)__half2float(__ushort_as_half(z16)), sym);
        cst[i] = make_uint4(g.s_hi, g.s_lo, g.zm, g.xmask);
    }
    named_sync(1, nthreads_c);

    const int g8 = lane >> 2, t4 = lane & 3;
    const GroupConsts zero_consts = {0u, 0u, 0u, 0u};  // x_hat = 0 for rows past the chunk
    uint32_t xr[16];
    int cached_ks = -1;
    for (int c = 0; c < nch; ++c) {
        const int slot = c % a.nslots;
        const bool landed = mbar_wait(&full[slot], (uint32_t)(c / a.nslots) & 1u, a.status);
        if (!__all_sync(0xffffffffu, landed)) {
            if (lane == 0) atomicExch(&abort_flag, 1);
            break;
        }
        const uint8_t* sp = slots + (size_t)slot * a.slot_bytes;
        const int rows = min(RC, nrows - c * RC);
        for (int rb = 0; rb * 16 < rows; ++rb) {
            const int ra = rb * 16 + g8, rbb = ra + 8;  // chunk rows of this lane
            const bool va = ra < rows, vb = rbb < rows;
            float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int ks = warp; ks < nks; ks += kM1Warps) {
                const int s = ks * 4 + t4;  // the lane's 32-k slice
                const bool vs = s < nsl;
                if (ks != cached_ks) {  // activation pairs of the slice: the B fragments
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = vs ? xs[s * 4 + q] : make_uint4(0, 0, 0, 0);
                        xr[4 * q] = v.x; xr[4 * q + 1] = v.y; xr[4 * q + 2] = v.z; xr[4 * q + 3] = v.w;
                    }
                    cached_ks = ks;
                }
                const int gi = a.g_shift >= 0 ? ((s * 32) >> a.g_shift) : (s * 32) / a.g;
                uint4 wa = make_uint4(0, 0, 0, 0), wb = wa;
                GroupConsts ka = zero_consts, kb = zero_consts;
                if (va && vs) {
                    wa = *reinterpret_cast<const uint4*>(sp + ra * row_bytes + s * 16);
                    const uint4 k4 = cst[(c * RC + ra) * a.G + gi];
                    ka = {k4.x, k4.y, k4.z, k4.w};
                }
                if (vb && vs) {
                    wb = *reinterpret_cast<const uint4*>(sp + rbb * row_bytes + s * 16);
                    const uint4 k4 = cst[(c * RC + rbb) * a.G + gi];
                    kb = {k4.x, k4.y, k4.z, k4.w};
                }
                const uint32_t wva[4] = {wa.x, wa.y, wa.z, wa.w}, wvb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t pa[4], pb[4];
                    dequant_word_pairs(wva[j], ka, pa);
                    dequant_word_pairs(wvb[j], kb, pb);
                    mma_16816(d, pa[0], pb[0], pa[1], pb[1], xr[4 * j + 0], xr[4 * j + 1]);
                    mma_16816(d, pa[2], pb[2], pa[3], pb[3], xr[4 * j + 2], xr[4 * j + 3]);
                }
            }
            // d = (D[ra][2t], D[ra][2t+1], D[rb][2t], D[rb][2t+1]); every column holds the token
            if (t4 == 0) {
                if (va) red[(c * RC + ra) * kM1Warps + warp] = d[0];
                if (vb) red[(c * RC + rbb) * kM1Warps + warp] = d[2];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
    named_sync(1, nthreads_c);
    // each row's parked partials (one per consumer warp) summed by one warp in a
    // fixed order (a shuffle tree), so the result is deterministic
    for (int r = warp; r < nrows; r += kM1Warps) {
        float v = lane < kM1Warps ? red[r * kM1Warps + lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && !abort_flag) {
            if (a.y_fp32)
                static_cast<float*>(a.Y)[row0 + r] = v;
            else
                static_cast<__nv_bfloat16*>(a.Y)[row0 + r] = __float2bfloat16_rn(v);
        }
    }
}

cudaError_t launch_gemv_m1(const uint32_t* qweight, GemvArgs a, int num_sms, const LaunchOptions& opt,
                           cudaStream_t stream) {
    // one pass of R rows per CTA; chunks of RC rows (<= 32 KB, at least 1 row)
    const int R = (a.N + num_sms - 1) / num_sms;
    a.npass = 1;
    a.BR = R;
    a.rows_per_cta = R;
    const int64_t row_bytes = a.K / 2;
    int RC = (int)((32 * 1024) / row_bytes);
    if (RC < 1) RC = 1;
    if (RC > R) RC = R;
    a.BRT = RC;
    a.T = (R + RC - 1) / RC;
    a.slot_bytes = round_up((int)(RC * row_bytes), 1024);
    a.xs_bytes = 0;
    const int grid = (a.N + R - 1) / R;
    const int nch = a.T;
    a.nslots = 1;
    const int fixed = gemv_m1_layout(a).slot_off + 16 * kM1MaxSlots;
    int nslots = (kM1SmemBudget - fixed - 1024) / a.slot_bytes;
    if (nslots > kM1MaxSlots) nslots = kM1MaxSlots;
    if (nslots > nch) nslots = nch;
    if (nslots < 2 && nch > 1) nslots = 2;
    if (nslots < 1) nslots = 1;
    a.nslots = nslots;
    const GemvM1Layout L = gemv_m1_layout(a);
    // shapes whose per-CTA constants do not fit run on the MMA kernel instead
    if (L.total > 226 * 1024 || L.slot_off % 1024 != 0 || row_bytes % 16 != 0) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(gemv_m1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kM1Threads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = opt.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_m1_kernel, qweight, a);
}

template <int NT, int NCH>
cudaError_t launch_gemv_variant(const uint32_t* qweight, GemvArgs a, int num_sms, const LaunchOptions& opt,
                                cudaStream_t stream) {
    const int R = (a.N + num_sms - 1) / num_sms;
    a.npass = (R + kMaxBR - 1) / kMaxBR;
    a.BR = (R + a.npass - 1) / a.npass;
    a.rows_per_cta = a.npass * a.BR;
    a.T = (a.BR + 15) / 16;
    a.BRT = (a.BR + a.T - 1) / a.T;  // balanced tiles of <= 16 rows
    a.nkb = (a.K + kChunkK - 1) / kChunkK;
    a.nks = (a.K + kSegK - 1) / kSegK;
    a.pitch = kSegWords * 4;
    a.slot_bytes = kSlotBytes;
    const int T = a.T;
    const int grid = (a.N + a.rows_per_cta - 1) / a.rows_per_cta;
    const int xs = a.nkb * a.M * 256;
    a.xs_bytes = (NT == 1 && xs <= kXsMaxBytes) ? xs : 0;

    // slots: the whole share if it fits the budget, else a ring (>= 2 slots)
    const int total_chunks = a.npass * T * a.nks;
    a.nslots = 1;
    const int fixed = gemv_smem_layout(a).slot_off + 16 * kMaxSlots;
    int nslots = (kSmemBudget - fixed - 1024) / kSlotBytes;
    if (nslots > kMaxSlots) nslots = kMaxSlots;
    if (nslots > total_chunks) nslots = total_chunks;
    if (nslots < 2 && total_chunks > 1) nslots = 2;
    if (nslots < 1) nslots = 1;
    a.nslots = nslots;
    const GemvSmemLayout L = gemv_smem_layout(a);
    if (L.total > 226 * 1024) return cudaErrorInvalidConfiguration;
    if (L.slot_off % 1024 != 0 || L.xs_off % 16 != 0) return cudaErrorInvalidConfiguration;

    CUtensorMap tmap;
    CUresult cr = encode_tensor_map_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)(a.K / 8),
                                       (uint64_t)a.N, (uint64_t)(a.K / 2), kSegWords, (uint32_t)a.BRT,
                                       CU_TENSOR_MAP_SWIZZLE_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;

    auto kern = gemv_w4a16_kernel<NT, NCH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
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

cudaError_t launch_gemv(const uint32_t* qweight, const GemvArgs& base, int num_sms, const LaunchOptions& opt,
                        cudaStream_t stream) {
    // M = 1, 2: the k-split kernels (gemv_ksplit.cu) first (power-of-two g; the
    // CTA's rows within shared memory).  M = 3..16: the k-major kernel
    // (gemv_kmajor.cu: K >= 2048, N >= 16, power-of-two g) first, then the
    // k-split ones; it beats them from M = 3 on (4096x4096 M=8: 7.7 vs 10.9 us,
    // M=3: 7.3 vs 8.0 us) and loses at M = 2 (7.2 vs 5.5 us).  The older kernels serve the rest: for
    // M = 1 with rows up to 8K k the CUDA-core kernel was the faster one (7.0
    // vs 9.0 us at 4096x4096), longer rows and M = 2 run faster on the
    // tensor-memory kernel (15.7 vs 17.6 us at 4096x11008, M = 2: 9.1 vs 10.6 us
    // at 4096x4096).
    auto kmajor = [&]() -> cudaError_t {
        KmArgs k = {};
        k.X = base.X;
        k.scales = base.scales;
        k.zeros = base.zeros;
        k.Y = base.Y;
        k.status = base.status;
        k.M = base.M;
        k.N = base.N;
        k.K = base.K;
        k.G = base.G;
        k.g = base.g;
        k.g_shift = base.g_shift;
        k.symmetric = base.symmetric;
        k.y_fp32 = base.y_fp32;
        return launch_gemv_kmajor(qweight, k, num_sms, opt, stream);
    };
    const bool km_ok = base.M >= 2 && !gemv_kmajor_disabled();
    if (km_ok && base.M >= 3) {
        const cudaError_t e = kmajor();
        if (e != cudaErrorNotSupported) return e;
    }
    if (base.M <= 8 && !gemv_ksplit_disabled()) {
        KsArgs k = {};
        k.X = base.X;
        k.scales = base.scales;
        k.zeros = base.zeros;
        k.Y = base.Y;
        k.status = base.status;
        k.M = base.M;
        k.N = base.N;
        k.K = base.K;
        k.G = base.G;
        k.g = base.g;
        k.g_shift = base.g_shift;
        k.symmetric = base.symmetric;
        k.y_fp32 = base.y_fp32;
        const cudaError_t e = launch_gemv_ksplit(qweight, k, num_sms, opt, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    if (km_ok && base.M < 3) {
        const cudaError_t e = kmajor();
        if (e != cudaErrorNotSupported) return e;
    }
    const bool m1_first = base.M == 1 && base.K < 8192;
    if (m1_first) {
        const cudaError_t e = launch_gemv_m1(qweight, base, num_sms, opt, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    if (base.M <= 2 && !gemv_tc_disabled()) {
        const cudaError_t e = launch_gemv_tc(qweight, base, num_sms, opt, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    if (base.M == 1 && !m1_first) {
        const cudaError_t e = launch_gemv_m1(qweight, base, num_sms, opt, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    if (base.M <= 8) return launch_gemv_variant<1, 4>(qweight, base, num_sms, opt, stream);
    return launch_gemv_variant<2, 4>(qweight, base, num_sms, opt, stream);
}

}  // namespace wq
