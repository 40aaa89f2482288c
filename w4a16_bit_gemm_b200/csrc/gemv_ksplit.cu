// gemv_ksplit.cu -- W4A16 decode GEMV for M <= 8 on sm_100a.
//
// y[m, n] = sum_k x_hat[n, k] * x[m, k], x_hat = bf16_rn(s (q - z)), fp32
// accumulation: the fused low-bit path ("path A": packed weights, fused
// load / dequant / matmul, higher-precision accumulation) of "LLM
// Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)", section
// "Without a kernel the compression benefit disappears".  Decode is bound by
// the weight stream (section "Speed depends on batch and context"), so the
// kernels are organised around three facts of a decode step on B200:
//
// 1. One layer's packed weights are only ~60 KB per SM (4096 x 4096), which
//    HBM delivers in about a microsecond; the launch ramp and the first
//    bytes' latency cost as much.  The weights do not depend on the previous
//    kernel in the stream (only the activations do), so with programmatic
//    dependent launch the next GEMV's CTA becomes resident beside the running
//    one, streams its weights into its own shared memory, builds its group
//    constants and dequantizes most of its tiles, and only then waits for the
//    activations (griddepcontrol.wait).
// 2. The exact dequantization costs ~2.4 instructions per weight on the CUDA
//    cores, as long as the weight stream itself.  Dequantized tiles are kept
//    where a waiting CTA has room for them: in its half of the SM's tensor
//    memory (tcgen05.st / tcgen05.ld used as per-thread storage) and in
//    registers, so that after the wait a warp mostly issues MMAs.
// 3. No MMA row may be padding.  An m16n8k16 tile's 16 A rows are (output
//    row, 128-k unit) pairs: NK = 8 / MT k-units of RG = 2 MT rows.  B column
//    n carries token n % MT of k-unit n / MT, so D[i][n] for A row i and the
//    columns of its own k-unit is a partial sum of one output row; the other
//    columns are discarded.  Row counts only need to be multiples of RG (2 at
//    M = 1), so ~28 rows per SM fill every MMA row, and a warp's 16-byte
//    weight reads of one tile are 512 contiguous bytes of a row (no bank
//    conflicts).
//
// Two kernels share the tile code:
// - gemv_ksplit_res_kernel (every chunk of the CTA's rows resident): 8 warps,
//   two CTAs per SM (2 x 8 warps x 128 registers fills the register file;
//   each SMSP's 16K registers hold four warps).  Thread 0 issues all weight
//   copies at the start; each warp dequantizes its first kKsPre tiles into
//   tensor memory and one more into registers before the wait, one more
//   while the activations are fetched after it, and the rest afterwards.
// - gemv_ksplit_ring_kernel (rows that do not fit): a copy warp streams
//   chunks through a ring of slots; the 8 consumer warps take each chunk's
//   tiles round-robin.
// Each tile's partial sums are parked per (token, row, k-unit) and summed per
// output in a fixed order (deterministic).  Every mbarrier wait is bounded
// (WQ_DEVFLAG_TIMEOUT).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"
#include "wq_kernels.h"
#include "wq_tcgen05.cuh"

namespace wq {
namespace {

constexpr int kKsW = 8;                         // consumer warps
constexpr int kKsCThreads = kKsW * 32;
constexpr int kKsRingThreads = kKsCThreads + 32;  // + the copy warp
constexpr int kKsPiece = 32768;                 // bytes per bulk copy (at most)
constexpr int kKsMaxSlots = 16;
constexpr int kKsChunkTarget = 16384;           // bytes per chunk (rows rounded to the tile)
constexpr int kKsShared2 = 110 * 1024;          // two CTAs per SM
constexpr int kKsShared1 = 220 * 1024;          // one CTA per SM
constexpr int kKsSharedMin = 80 * 1024;         // never three CTAs per SM: two halves of tensor memory
constexpr int kKsTmemCols = 256;                // half of an SM's tensor memory
constexpr int kKsPre = 4;                       // tiles per warp held in tensor memory (128 columns)

struct KsLayout {
    int cst_off, xs_off, red_off, dummy_off, slot_off, total;
};

// Row stride of the partial sums: one float per k-unit, padded to an odd
// count so that lanes summing different rows read different banks.
__host__ __device__ inline int ks_red_pitch(int K) { return ((K + 127) / 128) | 1; }

// bars: full[16], empty[16]; cst: 16 B per (row, group) for the CTA's rows
// plus one zero entry; xs: 64 B per (token, 32-k slice); red: fp32 per
// (token, row, k-unit); dummy: 32 floats; slots: contiguous, then 512 bytes of
// slack for the reads of a ragged last k-unit set.
__host__ __device__ inline KsLayout ks_layout(const KsArgs& a) {
    KsLayout L;
    const int nsl = a.K / 32;
    L.cst_off = 2 * kKsMaxSlots * 8;
    L.xs_off = L.cst_off + (((a.R * a.G + 1) * 16 + 127) & ~127);
    L.red_off = L.xs_off + ((a.M * nsl * 64 + 127) & ~127);
    L.dummy_off = L.red_off + ((a.M * a.R * ks_red_pitch(a.K) * 4 + 127) & ~127);
    L.slot_off = (L.dummy_off + 128 + 1023) & ~1023;
    L.total = L.slot_off + a.nslots * a.slot_bytes + 512 + 1024;  // + base alignment slack
    return L;
}

__device__ __forceinline__ void mma_bf16_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A B with a zero accumulator input (the first MMA of a chain).
__device__ __forceinline__ void mma_bf16_16816_zc(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                  uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint4 ld_global_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// The CTA's share of the rows: row groups of RG split evenly over the grid,
// the first CTAs taking one group more.
template <int RG>
__device__ __forceinline__ void ks_rows(int N, int& row0, int& nrows) {
    const int ngroups = (N + RG - 1) / RG;
    const int per = ngroups / gridDim.x, extra = ngroups - per * gridDim.x;
    row0 = RG * (blockIdx.x * per + min((int)blockIdx.x, extra));
    nrows = min(RG * (per + ((int)blockIdx.x < extra ? 1 : 0)), N - row0);
}

// Per-(row, group) constants of the exact bf16x2 dequant for the CTA's rows,
// plus a zero entry after them (x_hat = 0 for rows and k past the ends).
// Scales and zeros are static, so this runs before the wait; kPf items per
// thread have their loads issued before any is used.
__device__ __forceinline__ void ks_constants(const KsArgs& a, int row0, int nrows, uint4* cst, int tid, int nthr) {
    constexpr int kPf = 4;
    const bool sym = a.symmetric != 0;
    const int nitems = nrows * a.G;
    for (int i0 = tid; i0 < nitems; i0 += kPf * nthr) {
        uint16_t sv[kPf], zv[kPf];
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
            const int i = i0 + u * nthr;
            const int64_t gi = (int64_t)row0 * a.G + i;
            sv[u] = i < nitems ? ld_nc_u16(a.scales + gi) : (uint16_t)0;
            zv[u] = (i < nitems && !sym) ? ld_nc_u16(a.zeros + gi) : (uint16_t)0;
        }
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
            const int i = i0 + u * nthr;
            if (i < nitems) {
                const GroupConsts k = make_group_consts(sv[u], sym ? 0 : (int)__half2float(__ushort_as_half(zv[u])), sym);
                cst[i] = make_uint4(k.s_hi, k.s_lo, k.zm, k.xmask);
            }
        }
    }
    if (tid == 0) cst[nitems] = make_uint4(0, 0, 0, 0);
}

// Activation slices in B-fragment pair order: word p of part q of slice s
// holds (x[32 s + 8 q + p], x[32 s + 8 q + p + 4]), the pairing of
// dequant_word_pairs; stored part-major, xs[(q M + m) nsl + s], so that lanes
// reading consecutive slices hit consecutive 16-byte bank groups.
__device__ __forceinline__ void ks_load_slice(const uint16_t* X, int K, int nsl, int it, uint4 (&v)[4]) {
    const int m = it / nsl, sl = it - m * nsl;
    const uint16_t* src = X + (int64_t)m * K + sl * 32;
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = ld_global_v4(src + 8 * q);
}
__device__ __forceinline__ void ks_stage_slice(int M, int nsl, int it, const uint4 (&v)[4], uint4* xs) {
    const int m = it / nsl, sl = it - m * nsl;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        xs[(q * M + m) * nsl + sl] =
            make_uint4(__byte_perm(v[q].x, v[q].z, 0x5410), __byte_perm(v[q].x, v[q].z, 0x7632),
                       __byte_perm(v[q].y, v[q].w, 0x5410), __byte_perm(v[q].y, v[q].w, 0x7632));
}

// Each output's k-unit partials: eight lanes take every eighth k-unit in
// order, then a three-level shuffle tree (fixed order: deterministic).
// Parameters the epilogue reads, pinned in registers at kernel start.
struct KsOut {
    void* Y;
    int M, N, R, y_fp32;
};
__device__ __forceinline__ KsOut ks_out(const KsArgs& a) {
    KsOut o;
    o.Y = pin_ptr(a.Y);
    o.M = pin_i32(a.M);
    o.N = pin_i32(a.N);
    o.R = pin_i32(a.R);
    o.y_fp32 = pin_i32(a.y_fp32);
    return o;
}

__device__ __forceinline__ void ks_epilogue(const KsOut& o, const float* red, int rp_pitch, int nku, int row0,
                                            int nrows, bool ok) {
    const int part = threadIdx.x & 7, sub = threadIdx.x >> 3;  // 32 outputs per round
    for (int m = 0; m < o.M; ++m) {
        for (int r0 = 0; r0 < nrows; r0 += kKsCThreads / 8) {
            const int r = r0 + sub;
            float v = 0.0f;
            if (r < nrows) {
                const float* rp = red + (m * o.R + r) * rp_pitch;
#pragma unroll 4
                for (int k = part; k < nku; k += 8) v += rp[k];
            }
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            if (ok && r < nrows && part == 0) {
                const int64_t yo = (int64_t)m * o.N + row0 + r;
                if (o.y_fp32)
                    static_cast<float*>(o.Y)[yo] = v;
                else
                    static_cast<__nv_bfloat16*>(o.Y)[yo] = __float2bfloat16_rn(v);
            }
        }
    }
}

// What a lane of a consumer warp needs for every tile: its place in the MMA
// fragments, and the shared-memory addresses of constants, partials and the
// discarded-store sink.
template <int MT>
struct KsLane {
    static constexpr int NK = 8 / MT;  // k-units per MMA tile
    static constexpr int RG = 16 / NK;  // output rows per MMA tile
    static constexpr int RB = 8 / NK;   // row offset of a lane's second A row
    int t4, kidx, rsub, xc;
    bool xv_ok, f0, f1;
    uint32_t red0, red1, dummy, cst_s, zero_cst;
    uint32_t red_keep;  // MT = 1: partial block of the kept column (when f0 || f1)
    int G, g_shift, nsl, row_bytes, rp_pitch;
    const uint4* xsl;  // this lane's token row of part 0 of the staged activations
    int xq;            // part stride of the staged activations (in uint4)

    __device__ __forceinline__ KsLane(const KsArgs& a, int lane, int nrows, const uint4* cst, const uint4* xs,
                                      const float* red, const uint8_t* dummy_p, int rp_pitch_) {
        const int g8 = lane >> 2;
        t4 = lane & 3;
        kidx = g8 % NK;  // the lane's k-unit within a set (its A rows)
        rsub = g8 / NK;  // the lane's first A row within the tile
        xc = g8 / MT;    // the lane's B column: k-unit xc of the set, token g8 % MT
        const int xm = g8 % MT;
        // D columns 2 t4 + e (e = 0, 1) that belong to this lane's own k-unit, and
        // their tokens; MT = 1: at most one of them, MT >= 2: both or neither
        const int n0 = 2 * t4, n1 = 2 * t4 + 1;
        f0 = n0 / MT == kidx && n0 % MT < a.M;
        f1 = n1 / MT == kidx && n1 % MT < a.M;
        rp_pitch = rp_pitch_;
        const uint32_t red_s = smem_u32(red);
        red0 = red_s + 4u * (uint32_t)((n0 % MT) * a.R * rp_pitch);
        red1 = red_s + 4u * (uint32_t)((n1 % MT) * a.R * rp_pitch);
        red_keep = f1 ? red1 : red0;
        dummy = smem_u32(dummy_p) + 4u * lane;
        G = a.G;
        g_shift = a.g_shift;
        nsl = a.K / 32;
        row_bytes = a.K / 2;
        cst_s = smem_u32(cst);
        zero_cst = cst_s + 16u * (uint32_t)(nrows * G);
        xv_ok = xm < a.M;
        xsl = xs + xm * nsl;
        xq = a.M * nsl;
    }

    // A fragments of one tile (the lane's rows at wa_addr and wa_addr + RB
    // rows; constants at ca / cb): f[8 q + i] is register i % 4 of the MMA
    // 2 q + i / 4 (word q of the lane's 32-k slice, nibble pairs (p, p + 4)).
    __device__ __forceinline__ void dequant(uint32_t wa_addr, uint32_t ca, uint32_t cb, uint32_t (&f)[32]) const {
        const uint4 wa = ld_shared_v4(wa_addr);
        const uint4 wb = ld_shared_v4(wa_addr + RB * row_bytes);
        const uint4 ka = ld_shared_v4(ca);
        const uint4 kb = ld_shared_v4(cb);
        const GroupConsts gca = {ka.x, ka.y, ka.z, ka.w}, gcb = {kb.x, kb.y, kb.z, kb.w};
        const uint32_t wva[4] = {wa.x, wa.y, wa.z, wa.w}, wvb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            f[8 * q + 0] = dequant_pair(wva[q], gca);
            f[8 * q + 1] = dequant_pair(wvb[q], gcb);
            f[8 * q + 2] = dequant_pair(wva[q] >> 4, gca);
            f[8 * q + 3] = dequant_pair(wvb[q] >> 4, gcb);
            f[8 * q + 4] = dequant_pair(wva[q] >> 8, gca);
            f[8 * q + 5] = dequant_pair(wvb[q] >> 8, gcb);
            f[8 * q + 6] = dequant_pair(wva[q] >> 12, gca);
            f[8 * q + 7] = dequant_pair(wvb[q] >> 12, gcb);
        }
    }

    // The tile's eight MMAs against the activation fragments xr, and its partials
    // (ro: byte offset of (row, k-unit) in a token's partial block).  ACC4: four
    // accumulators two MMAs deep (the resident kernel, whose MMAs run after the
    // wait), else two accumulators four deep (fewer registers for the ring
    // kernel); either way summed in a fixed order.
    template <bool ACC4 = false>
    __device__ __forceinline__ void mma_flush(const uint32_t (&f)[32], const uint32_t (&xr)[16], uint32_t ro, bool va,
                                              bool vb) const {
        float d0[4], d1[4];
        mma_bf16_16816_zc(d0, f[0], f[1], f[2], f[3], xr[0], xr[1]);
        mma_bf16_16816_zc(d1, f[4], f[5], f[6], f[7], xr[2], xr[3]);
        if constexpr (ACC4) {
            float d2[4], d3[4];
            mma_bf16_16816_zc(d2, f[8], f[9], f[10], f[11], xr[4], xr[5]);
            mma_bf16_16816_zc(d3, f[12], f[13], f[14], f[15], xr[6], xr[7]);
            mma_bf16_16816(d0, f[16], f[17], f[18], f[19], xr[8], xr[9]);
            mma_bf16_16816(d1, f[20], f[21], f[22], f[23], xr[10], xr[11]);
            mma_bf16_16816(d2, f[24], f[25], f[26], f[27], xr[12], xr[13]);
            mma_bf16_16816(d3, f[28], f[29], f[30], f[31], xr[14], xr[15]);
#pragma unroll
            for (int i = 0; i < 4; ++i) d0[i] = (d0[i] + d2[i]) + (d1[i] + d3[i]);
        } else {
#pragma unroll
            for (int q = 1; q < 4; ++q) {
                mma_bf16_16816(d0, f[8 * q], f[8 * q + 1], f[8 * q + 2], f[8 * q + 3], xr[4 * q], xr[4 * q + 1]);
                mma_bf16_16816(d1, f[8 * q + 4], f[8 * q + 5], f[8 * q + 6], f[8 * q + 7], xr[4 * q + 2],
                               xr[4 * q + 3]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) d0[i] += d1[i];
        }
        // D[g8][2 t4 + e] and D[g8 + 8][2 t4 + e]: keep the columns of this lane's k-unit
        const uint32_t rbo = 4u * RB * rp_pitch;
        if constexpr (MT == 1) {
            // va / vb already include whether this lane keeps a column (Walk)
            const float va_v = f1 ? d0[1] : d0[0];
            const float vb_v = f1 ? d0[3] : d0[2];
            const uint32_t rr = red_keep + ro;
            st_shared_f32(va ? rr : dummy, va_v);
            st_shared_f32(vb ? rr + rbo : dummy, vb_v);
        } else {
            st_shared_f32(f0 && va ? red0 + ro : dummy, d0[0]);
            st_shared_f32(f0 && vb ? red0 + ro + rbo : dummy, d0[2]);
            st_shared_f32(f1 && va ? red1 + ro : dummy, d0[1]);
            st_shared_f32(f1 && vb ? red1 + ro + rbo : dummy, d0[3]);
        }
    }

    // Activation fragments of k-unit set j.
    __device__ __forceinline__ void load_x(int j, uint32_t (&xr)[16]) const {
        const int sx = (j * NK + xc) * 4 + t4;
        const bool ok = xv_ok && sx < nsl;
        const int sxc = ok ? sx : 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 v = xsl[q * xq + sxc];
            if (!ok) v = make_uint4(0, 0, 0, 0);
            xr[4 * q] = v.x;
            xr[4 * q + 1] = v.y;
            xr[4 * q + 2] = v.z;
            xr[4 * q + 3] = v.w;
        }
    }

    // The tiles of a warp's run in (k-set major, row-group minor) order, with
    // their addresses advanced by additions only.  For MT = 1, va / vb also hold
    // whether this lane keeps a column at all (its stores go to the sink if not).
    struct Walk {
        int j, gr, rc;           // k-unit set, row group, CTA-local row of A row g8
        uint32_t wa, cc, ro;     // weights, constants (row a), partials offset
        bool kv;                 // the lane's slice lies inside K
        bool va, vb;             // rows a / b exist (and, for MT = 1, the lane keeps a column)
        uint32_t ca, cb;         // constants of rows a / b (or the zero entry)
    };
    __device__ __forceinline__ void walk_set(Walk& w, uint32_t slots_s) const {
        const int kunit = w.j * NK + kidx;
        const int sw = kunit * 4 + t4;
        w.kv = sw < nsl;
        w.rc = w.gr * RG + rsub;
        w.wa = slots_s + (uint32_t)(w.rc * row_bytes + sw * 16);
        w.cc = cst_s + 16u * (uint32_t)(w.rc * G + ((sw * 32) >> g_shift));
        w.ro = 4u * (uint32_t)(w.rc * rp_pitch + kunit);
    }
    // REG: every tile lies inside the rows and K (K a multiple of 128 NK, the
    // CTA's row count a multiple of RG), so only the lane's own keep flag remains.
    template <bool REG>
    __device__ __forceinline__ void walk_valid(Walk& w, int nrows) const {
        const bool keep = MT != 1 || f0 || f1;
        if constexpr (REG) {
            w.ca = w.cc;
            w.cb = w.cc + 16u * RB * G;
            w.va = keep;
            w.vb = keep;
            return;
        }
        w.va = w.kv && w.rc < nrows;
        w.vb = w.kv && w.rc + RB < nrows;
        w.ca = w.va ? w.cc : zero_cst;
        w.cb = w.vb ? w.cc + 16u * RB * G : zero_cst;
        w.va = w.va && keep;
        w.vb = w.vb && keep;
    }
    template <bool REG>
    __device__ __forceinline__ void walk_start(Walk& w, int u, int ngr, uint32_t slots_s, int nrows) const {
        w.j = u / ngr;
        w.gr = u - w.j * ngr;
        walk_set(w, slots_s);
        walk_valid<REG>(w, nrows);
    }
    template <bool REG>
    __device__ __forceinline__ void walk_next(Walk& w, int ngr, uint32_t slots_s, int nrows) const {
        if (++w.gr == ngr) {
            w.gr = 0;
            ++w.j;
            walk_set(w, slots_s);
        } else {
            w.rc += RG;
            w.wa += (uint32_t)(RG * row_bytes);
            w.cc += 16u * (uint32_t)(RG * G);
            w.ro += 4u * (uint32_t)(RG * rp_pitch);
        }
        walk_valid<REG>(w, nrows);
    }

    // Addresses of tile (k-unit set j, row group gr) for the lane: rows past the
    // CTA's and k past the row read stale slot bytes (or the slack) and take the
    // zero constants.  slot_base: smem address of the slot holding CTA-local
    // row crow (the slot's first row).
    __device__ __forceinline__ void tile(uint32_t slot_base, int crow, int gr, int j, int nrows, uint32_t& wa,
                                         uint32_t& ca, uint32_t& cb, uint32_t& ro, bool& va, bool& vb) const {
        const int kunit = j * NK + kidx;
        const int sw = kunit * 4 + t4;  // the lane's 32-k slice
        const int rl = gr * RG + rsub;  // row of A row g8 within the slot (+ RB for g8 + 8)
        const int rc = crow + rl;       // CTA-local row
        const bool kv = sw < nsl;
        va = kv && rc < nrows;
        vb = kv && rc + RB < nrows;
        const uint32_t cidx = (uint32_t)(rc * G + ((sw * 32) >> g_shift));
        wa = slot_base + (uint32_t)(rl * row_bytes + sw * 16);
        ca = va ? cst_s + 16u * cidx : zero_cst;
        cb = vb ? cst_s + 16u * (cidx + RB * G) : zero_cst;
        ro = 4u * (uint32_t)(rc * rp_pitch + kunit);
        if constexpr (MT == 1) {  // the flush expects whether this lane keeps a column folded in
            va = va && (f0 || f1);
            vb = vb && (f0 || f1);
        }
    }
};

// ---------------------------------------------------------------------------
// Every chunk of the CTA's rows resident; tiles dequantized ahead of the wait.
// ---------------------------------------------------------------------------
template <int MT, bool REG>
__global__ void __maxnreg__(128) gemv_ksplit_res_kernel(const uint32_t* __restrict__ qweight, const KsArgs a) {
    using Lane = KsLane<MT>;
    constexpr int RG = Lane::RG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const KsLayout L = ks_layout(a);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint4* cst = reinterpret_cast<uint4*>(smem + L.cst_off);
    uint4* xs = reinterpret_cast<uint4*>(smem + L.xs_off);
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint8_t* slots = smem + L.slot_off;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int row0, nrows;
    ks_rows<RG>(a.N, row0, nrows);
    const int nch = (nrows + a.RC - 1) / a.RC;
    const int row_bytes = a.K / 2;
    const int nsl = a.K / 32;
    const int nku = (a.K + 127) / 128;
    const int rp_pitch = ks_red_pitch(a.K);
    const int J = (nku + Lane::NK - 1) / Lane::NK;  // k-unit sets per row group
    const KsOut out = ks_out(a);
    const uint16_t* Xp = pin_ptr(static_cast<const uint16_t*>(a.X));
    const int Kp = pin_i32(a.K);

    if (threadIdx.x == 0) {
        for (int c = 0; c < nch; ++c) mbar_init(&full[c], 1);
        abort_flag = 0;
        fence_mbar_init();
        // the CTA's rows, one slot per chunk, all requested at once
        const char* src0 = reinterpret_cast<const char*>(qweight) + (int64_t)row0 * row_bytes;
        for (int c = 0; c < nch; ++c) {
            const uint32_t bytes = (uint32_t)(min(a.RC, nrows - c * a.RC) * row_bytes);
            const char* src = src0 + (int64_t)c * a.RC * row_bytes;
            uint8_t* dst = slots + (size_t)c * a.slot_bytes;
            mbar_arrive_expect_tx(&full[c], bytes);
            for (uint32_t off = 0; off < bytes; off += kKsPiece)
                bulk_copy_g2s(dst + off, src + off, min((uint32_t)kKsPiece, bytes - off), &full[c]);
        }
        // the activations into L2 ahead of the wait (L2 is the point of coherence,
        // so a line the previous kernel writes later is still read fresh)
        prefetch_l2_bulk(a.X, (uint32_t)(a.M * a.K * 2));
    }
    // tensor memory is allocated before this CTA lets the next launch start, so a
    // co-resident CTA of a later launch never holds columns this one waits for
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(&tmem_slot, kKsTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    // the next launch only streams its weights, builds constants and dequantizes
    // before its own griddepcontrol.wait, so it may start at once
    pdl_launch_dependents();

    ks_constants(a, row0, nrows, cst, threadIdx.x, kKsCThreads);
    const Lane ln(a, lane, nrows, cst, xs, red, smem + L.dummy_off, rp_pitch);
    const uint32_t slots_s = smem_u32(slots);
    // warp w takes the contiguous run [u0, u1) of the (k-set major, row-group
    // minor) tiles: its first npre in tensor memory (128 columns per warp), the
    // next one in registers (fr) before the wait, the next (f2) while the
    // activations are fetched, the rest after
    const int ngr = (nrows + RG - 1) / RG;
    const int total = ngr * J;
    const int u0 = (warp * total) / kKsW, u1 = ((warp + 1) * total) / kKsW;
    const uint32_t taddr = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
    __syncthreads();  // every constant written

    bool aborted = false;
    {
        bool ok = true;
        for (int c = 0; c < nch; ++c) ok = ok && (mbar_test_wait(&full[c], 0u) || mbar_wait(&full[c], 0u, a.status));
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) atomicExch(&abort_flag, 1);
            aborted = true;
        }
    }
    const int nwork = aborted ? 0 : u1 - u0;
    const int ntm = min(kKsPre, nwork);  // tiles in tensor memory
    typename Lane::Walk w;
    if (nwork > 0) ln.template walk_start<REG>(w, u0, ngr, slots_s, nrows);
    for (int k = 0; k < ntm; ++k) {
        uint32_t f[32];
        ln.dequant(w.wa, w.ca, w.cb, f);
        tmem_st_32x32b_x32(taddr + 32u * k, f);
        ln.template walk_next<REG>(w, ngr, slots_s, nrows);
    }
    tc_wait_st();
    uint32_t fr[32];
    const bool have_fr = ntm < nwork;
    const int fr_j = w.j;
    const uint32_t fr_ro = w.ro;
    const bool fr_va = w.va, fr_vb = w.vb;
    if (have_fr) {
        ln.dequant(w.wa, w.ca, w.cb, fr);
        ln.template walk_next<REG>(w, ngr, slots_s, nrows);
    }

    pdl_wait_prior();  // the activations (and y) may belong to the previous kernel
    const int nst = out.M * nsl;
    uint4 xv0[4];
    if ((int)threadIdx.x < nst) ks_load_slice(Xp, Kp, nsl, threadIdx.x, xv0);
    // one more tile while the first slices are in flight
    uint32_t f2[32];
    const bool have_f2 = ntm + 1 < nwork;
    const int f2_j = w.j;
    const uint32_t f2_ro = w.ro;
    const bool f2_va = w.va, f2_vb = w.vb;
    if (have_f2) {
        ln.dequant(w.wa, w.ca, w.cb, f2);
        ln.template walk_next<REG>(w, ngr, slots_s, nrows);
    }
    if ((int)threadIdx.x < nst) ks_stage_slice(out.M, nsl, threadIdx.x, xv0, xs);
    for (int it = threadIdx.x + kKsCThreads; it < nst; it += kKsCThreads) {
        uint4 v[4];
        ks_load_slice(Xp, Kp, nsl, it, v);
        ks_stage_slice(out.M, nsl, it, v, xs);
    }
    __syncthreads();

    uint32_t xr[16];
    int jx = -1;
    if (have_fr) {
        ln.load_x(fr_j, xr);
        jx = fr_j;
        ln.template mma_flush<true>(fr, xr, fr_ro, fr_va, fr_vb);
    }
    if (have_f2) {
        if (f2_j != jx) {
            ln.load_x(f2_j, xr);
            jx = f2_j;
        }
        ln.template mma_flush<true>(f2, xr, f2_ro, f2_va, f2_vb);
    }
    {
        typename Lane::Walk wt;  // the tensor-memory tiles again, from the start of the run
        if (ntm > 0) ln.template walk_start<REG>(wt, u0, ngr, slots_s, nrows);
        for (int k = 0; k < ntm; ++k) {
            if (wt.j != jx) {
                ln.load_x(wt.j, xr);
                jx = wt.j;
            }
            uint32_t f[32];
            tmem_ld_32x32b_x32(taddr + 32u * k, f);
            tc_wait_ld();
            ln.template mma_flush<true>(f, xr, wt.ro, wt.va, wt.vb);
            ln.template walk_next<REG>(wt, ngr, slots_s, nrows);
        }
    }
    // tensor memory goes back as soon as every warp has read its tiles
    tc_fence_before();
    if (warp == 0) {
        named_sync(2, kKsCThreads);
        tc_fence_after();
        tmem_dealloc(tmem_base, kKsTmemCols);
    } else {
        named_arrive(2, kKsCThreads);
    }
    for (int k = ntm + 2; k < nwork; ++k) {
        if (w.j != jx) {
            ln.load_x(w.j, xr);
            jx = w.j;
        }
        uint32_t f[32];
        ln.dequant(w.wa, w.ca, w.cb, f);
        ln.template mma_flush<true>(f, xr, w.ro, w.va, w.vb);
        ln.template walk_next<REG>(w, ngr, slots_s, nrows);
    }
    __syncthreads();
    ks_epilogue(out, red, rp_pitch, nku, row0, nrows, !abort_flag);
}

// ---------------------------------------------------------------------------
// Rows that do not fit: a copy warp streams chunks through a ring of slots.
// ---------------------------------------------------------------------------
template <int MT>
__global__ void __launch_bounds__(kKsRingThreads, 2)
    gemv_ksplit_ring_kernel(const uint32_t* __restrict__ qweight, const KsArgs a) {
    using Lane = KsLane<MT>;
    constexpr int RG = Lane::RG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const KsLayout L = ks_layout(a);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kKsMaxSlots;
    uint4* cst = reinterpret_cast<uint4*>(smem + L.cst_off);
    uint4* xs = reinterpret_cast<uint4*>(smem + L.xs_off);
    float* red = reinterpret_cast<float*>(smem + L.red_off);
    uint8_t* slots = smem + L.slot_off;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int row0, nrows;
    ks_rows<RG>(a.N, row0, nrows);
    const int nch = (nrows + a.RC - 1) / a.RC;
    const int row_bytes = a.K / 2;
    const int nsl = a.K / 32;
    const int nku = (a.K + 127) / 128;
    const int rp_pitch = ks_red_pitch(a.K);
    const int J = (nku + Lane::NK - 1) / Lane::NK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.nslots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kKsW);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    // tensor memory before the next launch may start (see the resident kernel);
    // only when two CTAs share an SM, so that the parking overlaps a running launch
    const bool pre = a.pre != 0;
    if (pre && warp == 0) {
        __syncwarp();
        tmem_alloc(&tmem_slot, kKsTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = pre ? tmem_slot : 0u;
    pdl_launch_dependents();

    if (warp == kKsW) {
        // ---------------- copy warp: the CTA's rows, chunk by chunk ----------------
        if (lane == 0) {
            const char* src0 = reinterpret_cast<const char*>(qweight) + (int64_t)row0 * row_bytes;
            for (int c = 0; c < nch; ++c) {
                const int slot = c % a.nslots;
                if (c >= a.nslots &&
                    !mbar_wait(&empty[slot], (uint32_t)((c / a.nslots) - 1) & 1u, a.status)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                const uint32_t bytes = (uint32_t)(min(a.RC, nrows - c * a.RC) * row_bytes);
                const char* src = src0 + (int64_t)c * a.RC * row_bytes;
                uint8_t* dst = slots + (size_t)slot * a.slot_bytes;
                mbar_arrive_expect_tx(&full[slot], bytes);
                for (uint32_t off = 0; off < bytes; off += kKsPiece)
                    bulk_copy_g2s(dst + off, src + off, min((uint32_t)kKsPiece, bytes - off), &full[slot]);
            }
            prefetch_l2_bulk(a.X, (uint32_t)(a.M * a.K * 2));
        }
        return;
    }

    // ---------------- consumers ----------------
    ks_constants(a, row0, nrows, cst, threadIdx.x, kKsCThreads);
    const KsOut out = ks_out(a);
    named_sync(1, kKsCThreads);  // constants written
    const Lane ln(a, lane, nrows, cst, xs, red, smem + L.dummy_off, rp_pitch);
    const uint32_t slots_s = smem_u32(slots);
    const uint32_t taddr = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
    auto chunk_units = [&](int c) { return ((min(a.RC, nrows - c * a.RC) + RG - 1) / RG) * J; };
    // the leading chunks whose tiles give every warp at most kKsPre tiles are
    // dequantized into tensor memory before the wait (their slots are released
    // at once, so the copy warp streams further chunks meanwhile)
    int pc = 0;
    for (int tot = 0; pre && pc < nch && tot + chunk_units(pc) <= kKsPre * kKsW; ++pc) tot += chunk_units(pc);
    bool aborted = false;
    int U = warp;  // this warp's next tile, counted over all chunks
    int base = 0;
    int ntm = 0;
    for (int c = 0; c < pc; ++c) {
        const int crow0 = c * a.RC;
        const int units = chunk_units(c);
        const int slot = c % a.nslots;
        if (!aborted) {
            const uint32_t par = (uint32_t)(c / a.nslots) & 1u;
            const bool ok = mbar_test_wait(&full[slot], par) || mbar_wait(&full[slot], par, a.status);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicExch(&abort_flag, 1);
                aborted = true;
            }
            const uint32_t sp = slots_s + (uint32_t)(slot * a.slot_bytes);
            for (; !aborted && U < base + units; U += kKsW) {
                const int gr = (U - base) / J, j = (U - base) - gr * J;
                uint32_t wa, ca, cb, ro;
                bool va, vb;
                ln.tile(sp, crow0, gr, j, nrows, wa, ca, cb, ro, va, vb);
                uint32_t f[32];
                ln.dequant(wa, ca, cb, f);
                tmem_st_32x32b_x32(taddr + 32u * ntm, f);
                ++ntm;
            }
        }
        tc_wait_st();  // the slot is read (and the stores done) before it is released
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        base += units;
    }

    pdl_wait_prior();  // the activations (and y) may belong to the previous kernel
    for (int it = threadIdx.x; it < a.M * nsl; it += kKsCThreads) {
        uint4 v[4];
        ks_load_slice(static_cast<const uint16_t*>(a.X), a.K, nsl, it, v);
        ks_stage_slice(a.M, nsl, it, v, xs);
    }
    named_sync(1, kKsCThreads);  // activations written
    uint32_t xr[16];
    int jx = -1;  // k-unit set whose activation fragments are in xr
    {
        // the tensor-memory tiles, in the order they were stored
        int Ut = warp, bt = 0, k = 0;
        for (int c = 0; c < pc && k < ntm; ++c) {
            const int units = chunk_units(c);
            for (; k < ntm && Ut < bt + units; Ut += kKsW, ++k) {
                const int gr = (Ut - bt) / J, j = (Ut - bt) - gr * J;
                if (j != jx) {
                    ln.load_x(j, xr);
                    jx = j;
                }
                uint32_t wa, ca, cb, ro;
                bool va, vb;
                ln.tile(slots_s, c * a.RC, gr, j, nrows, wa, ca, cb, ro, va, vb);
                uint32_t f[32];
                tmem_ld_32x32b_x32(taddr + 32u * k, f);
                tc_wait_ld();
                ln.mma_flush(f, xr, ro, va, vb);
            }
            bt += units;
        }
    }
    // tensor memory goes back once every consumer warp has read its tiles (the
    // copy warp never touches it, and may still wait for slots these warps free)
    if (pre) {
        tc_fence_before();
        if (warp == 0) {
            named_sync(2, kKsCThreads);
            tc_fence_after();
            tmem_dealloc(tmem_base, kKsTmemCols);
        } else {
            named_arrive(2, kKsCThreads);
        }
    }
    for (int c = pc; c < nch; ++c) {
        const int crow0 = c * a.RC;
        const int units = chunk_units(c);
        const int slot = c % a.nslots;
        // a warp with no tile in this chunk still waits for it: its arrival on
        // `empty` must not count toward an earlier phase
        if (!aborted) {
            const uint32_t par = (uint32_t)(c / a.nslots) & 1u;
            const bool ok = mbar_test_wait(&full[slot], par) || mbar_wait(&full[slot], par, a.status);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicExch(&abort_flag, 1);
                aborted = true;
            }
            const uint32_t sp = slots_s + (uint32_t)(slot * a.slot_bytes);
            int gr = (U - base) / J, j = (U - base) - gr * J;
            for (; !aborted && U < base + units; U += kKsW) {
                if (j != jx) {
                    ln.load_x(j, xr);
                    jx = j;
                }
                uint32_t wa, ca, cb, ro;
                bool va, vb;
                ln.tile(sp, crow0, gr, j, nrows, wa, ca, cb, ro, va, vb);
                uint32_t f[32];
                ln.dequant(wa, ca, cb, f);
                ln.mma_flush(f, xr, ro, va, vb);
                j += kKsW;
                while (j >= J) {
                    j -= J;
                    ++gr;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        base += units;
    }
    named_sync(1, kKsCThreads);
    ks_epilogue(out, red, rp_pitch, nku, row0, nrows, !abort_flag);
}

template <int MT>
cudaError_t launch_ksplit(const uint32_t* qweight, KsArgs a, int num_sms, const LaunchOptions& opt,
                          cudaStream_t stream) {
    constexpr int RG = 2 * MT;
    // one CTA per SM (a second CTA of the same launch on one SM would double
    // that SM's work and set the pace of the whole launch); row groups are
    // split evenly, the first CTAs taking one group more
    const int ngroups = (a.N + RG - 1) / RG;
    const int grid = min(num_sms, ngroups);
    a.R = RG * ((ngroups + grid - 1) / grid);
    const int row_bytes = a.K / 2;
    int RC = kKsChunkTarget / row_bytes / RG * RG;
    if (RC < RG) RC = RG;
    if (RC > a.R) RC = a.R;
    a.RC = RC;
    a.slot_bytes = RC * row_bytes;  // a multiple of 16 (K is a multiple of 32)
    const int nch = (a.R + RC - 1) / RC;
    // every chunk resident with two CTAs per SM: the pre-dequantizing kernel
    a.nslots = nch;
    const bool res = nch <= kKsMaxSlots && ks_layout(a).total <= kKsShared2;
    if (!res) {
        // else a ring: two CTAs per SM when it still holds two chunks, else one
        int budget = kKsShared2;
        for (int pass = 0; pass < 2; ++pass, budget = kKsShared1) {
            a.nslots = 0;
            const int fixed = ks_layout(a).total;
            int ns = (budget - fixed) / a.slot_bytes;
            if (ns > kKsMaxSlots) ns = kKsMaxSlots;
            if (ns > nch) ns = nch;
            if (ns >= 2 || (ns == 1 && nch == 1)) {
                a.nslots = ns;
                break;
            }
        }
        if (a.nslots == 0) return cudaErrorNotSupported;
    }
    const KsLayout L = ks_layout(a);
    if (L.total > 227 * 1024) return cudaErrorNotSupported;
    a.pre = L.total <= kKsShared2 ? 1 : 0;
    // at least kKsSharedMin, so that at most two CTAs share an SM (each takes
    // half of its tensor memory)
    const int smem = L.total > kKsSharedMin ? L.total : kKsSharedMin;
    // every tile inside the rows and K: the resident kernel skips its bounds checks
    const bool reg = a.K % (128 * KsLane<MT>::NK) == 0 && a.N % RG == 0;
    void (*kern)(const uint32_t*, const KsArgs) =
        !res ? gemv_ksplit_ring_kernel<MT> : reg ? gemv_ksplit_res_kernel<MT, true> : gemv_ksplit_res_kernel<MT, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // the whole unified L1/shared array as shared memory, so that two CTAs fit
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(res ? kKsCThreads : kKsRingThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = opt.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, qweight, a);
}

}  // namespace

cudaError_t launch_gemv_ksplit(const uint32_t* qweight, const KsArgs& a, int num_sms, const LaunchOptions& opt,
                               cudaStream_t stream) {
    if (a.M < 1 || a.M > 8 || a.K % 32 != 0 || a.g % 32 != 0 || a.g_shift < 0) return cudaErrorNotSupported;
    if (a.M == 1) return launch_ksplit<1>(qweight, a, num_sms, opt, stream);
    if (a.M == 2) return launch_ksplit<2>(qweight, a, num_sms, opt, stream);
    if (a.M <= 4) return launch_ksplit<4>(qweight, a, num_sms, opt, stream);
    return launch_ksplit<8>(qweight, a, num_sms, opt, stream);
}

}  // namespace wq
