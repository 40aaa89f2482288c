// wq_device.cuh -- device helpers shared by the libwq kernels (sm_100a only).
//
// Exact dequantization in packed bf16x2 arithmetic
// ------------------------------------------------
// x_hat = bf16_rn(s * (q - z)) ("Affine Quantization": x_hat = s(q - z), one
// rounding to the bf16 compute type).  s is fp16 (11 significant bits) and
// d = q - z an integer with |d| <= 15, so s*d has up to 15 significant bits:
// exact in fp32, not in bf16.  Split s = s_hi + s_lo with s_hi = bf16_rn(s);
// then s_lo = s - s_hi is a multiple of ulp16(s) with |s_lo| <= 4 ulp16(s),
// i.e. at most 3 significant bits, so p = d * s_lo (<= 7 bits) is exact in
// bf16, and fma.rn.bf16x2(d, s_hi, p) rounds the exact value d*s_hi + p = d*s
// once: the result equals bf16_rn(s*d) bit for bit.
//
// d itself is produced without integer->float conversion: a nibble placed in
// the low mantissa bits of the bf16 value 128.0 (0x4300) gives 128 + q
// exactly (bf16 spacing at 128 is 1), and (128 + q) - (128 + z) = d is exact.
// Symmetric two's-complement nibbles are first XORed with 8 (offset binary:
// nib ^ 8 = q + 8) and 136 = 128 + 8 is subtracted instead.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace wq {

// ------------------------------------------------------------------------
// bf16x2 helpers (bit-level views)
// ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) {
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ __nv_bfloat162 bits_bf2(uint32_t u) {
    return *reinterpret_cast<__nv_bfloat162*>(&u);
}

// Per-(row, group) constants of the exact dequantization.
struct GroupConsts {
    uint32_t s_hi;   // bf16x2 (s_hi, s_hi)
    uint32_t s_lo;   // bf16x2 (s_lo, s_lo)
    uint32_t zm;     // bf16x2 (128 + z, 128 + z), or 136 for symmetric
    uint32_t xmask;  // 0x43004300 (asym) or 0x43084308 (sym: nibble ^ 8)
};

// s16: fp16 bits of the scale; z: integer zero point (0 for symmetric).
__device__ __forceinline__ GroupConsts make_group_consts(uint16_t s16, int z, bool symmetric) {
    GroupConsts c;
    float s = __half2float(__ushort_as_half(s16));
    __nv_bfloat16 hi = __float2bfloat16_rn(s);
    float lo_f = s - __bfloat162float(hi);  // exact in fp32
    __nv_bfloat16 lo = __float2bfloat16_rn(lo_f);  // exact: <= 3 significant bits
    uint32_t hb = __bfloat16_as_ushort(hi);
    uint32_t lb = __bfloat16_as_ushort(lo);
    c.s_hi = hb | (hb << 16);
    c.s_lo = lb | (lb << 16);
    uint32_t zb = symmetric ? 0x4308u : (0x4300u | (uint32_t)(z & 0xF));
    c.zm = zb | (zb << 16);
    c.xmask = symmetric ? 0x43084308u : 0x43004300u;
    return c;
}

// Exact x_hat for the two nibbles at bits (0..3, 16..19) of `t` after the
// caller shifted them there: returns bf16x2 (x_hat(lo nibble), x_hat(hi nibble)).
__device__ __forceinline__ uint32_t dequant_pair(uint32_t shifted, const GroupConsts& c) {
    uint32_t t = (shifted & 0x000F000Fu) ^ c.xmask;  // 128 + q (offset binary for sym)
    __nv_bfloat162 d = __hsub2(bits_bf2(t), bits_bf2(c.zm));         // q - z, exact
    __nv_bfloat162 p = __hmul2(d, bits_bf2(c.s_lo));                  // exact
    __nv_bfloat162 w = __hfma2(d, bits_bf2(c.s_hi), p);              // one rounding
    return bf2_bits(w);
}

// Group constants packed in 8 bytes: (s_hi, s_lo) and (128 + z, xmask half),
// each bf16 once; unpack_consts replicates them into the bf16x2 form.
__device__ __forceinline__ GroupConsts unpack_consts(uint2 v) {
    GroupConsts c;
    c.s_hi = __byte_perm(v.x, v.x, 0x1010);
    c.s_lo = __byte_perm(v.x, v.x, 0x3232);
    c.zm = __byte_perm(v.y, v.y, 0x1010);
    c.xmask = __byte_perm(v.y, v.y, 0x3232);
    return c;
}

__device__ __forceinline__ uint2 pack_consts(uint16_t s16, int z, bool sym) {
    const GroupConsts g = make_group_consts(s16, z, sym);
    return make_uint2((g.s_hi & 0xffffu) | (g.s_lo << 16), (g.zm & 0xffffu) | (g.xmask << 16));
}

// Dequantize one packed word (8 nibbles, low nibble first).
// out[p] = (x_hat(nibble p), x_hat(nibble p + 4)) for p = 0..3.
__device__ __forceinline__ void dequant_word_pairs(uint32_t w, const GroupConsts& c, uint32_t out[4]) {
    out[0] = dequant_pair(w, c);
    out[1] = dequant_pair(w >> 4, c);
    out[2] = dequant_pair(w >> 8, c);
    out[3] = dequant_pair(w >> 12, c);
}

// Dequantize one packed word into natural k order:
// out[i] = (x_hat(nibble 2i), x_hat(nibble 2i + 1)) for i = 0..3.
__device__ __forceinline__ void dequant_word_natural(uint32_t w, const GroupConsts& c, uint32_t out[4]) {
    uint32_t p[4];
    dequant_word_pairs(w, c, p);
    out[0] = __byte_perm(p[0], p[1], 0x5410);  // (n0, n1)
    out[1] = __byte_perm(p[2], p[3], 0x5410);  // (n2, n3)
    out[2] = __byte_perm(p[0], p[1], 0x7632);  // (n4, n5)
    out[3] = __byte_perm(p[2], p[3], 0x7632);  // (n6, n7)
}

// ------------------------------------------------------------------------
// Status word
// ------------------------------------------------------------------------

__device__ __forceinline__ void raise_flag(uint32_t* status, uint32_t bits) {
    if (status) atomicOr(status, bits);
}

// ------------------------------------------------------------------------
// mbarrier / TMA / fences (inline PTX, sm_90+ forms valid on sm_100a)
// ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_count(uint64_t* bar, uint32_t count) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

// Non-blocking test of an mbarrier phase (no suspend).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase.  Gives up after ~1 s of wall time
// (measured with %globaltimer), raises WQ_DEVFLAG_TIMEOUT and returns false.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr uint32_t kFlagTimeout = 0x4u;

__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, uint32_t* status,
                                                uint64_t limit_ns) {
    // a completed phase is seen by the non-blocking test at once; the blocking
    // try_wait costs the thread hundreds of cycles even then (measured in the
    // GEMM's dequant warps: ~0.6 us per k block across two waits)
    if (mbar_test_wait(bar, parity)) return true;
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = global_timer_ns();
    while (true) {
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) {
            raise_flag(status, kFlagTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
    return mbar_wait_limit(bar, parity, status, kWaitLimitNs);
}

// 2D tiled TMA load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int32_t x,
                                            int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(smem_dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// 1D bulk copy global -> shared (both 16-byte aligned, bytes a multiple of 16),
// completion counted on `bar` (bytes).
__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue, and wait for the previous kernel's memory to be visible.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Hardware named barriers (ids 1..15; id 0 is __syncthreads).  bar.arrive
// counts the calling warp and continues; bar.sync counts it and waits until
// `nthreads` threads have arrived.
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Copies of kernel parameters pinned in registers where they are taken (a
// volatile move is not re-materialised later from the parameter bank).
__device__ __forceinline__ int pin_i32(int v) {
    int r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}
template <typename T>
__device__ __forceinline__ T* pin_ptr(T* p) {
    uint64_t r;
    asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(reinterpret_cast<uint64_t>(p)));
    return reinterpret_cast<T*>(r);
}

__device__ __forceinline__ uint16_t ld_nc_u16(const uint16_t* p) {
    uint16_t r;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

}  // namespace wq
