// w8_device.cuh -- exact dequantization of symmetric INT8 codes to bf16.
//
// x_hat = bf16_rn(s q): the fp16 scale has 11 significant bits and |q| <= 127
// has 7, so the fp32 product is exact and the conversion to bf16 is the only
// rounding.  A code byte b (two's complement) becomes a float without an
// integer conversion: with u = b ^ 0x80 = q + 128, the bit pattern
// 0x4B0000uu is the float 2^23 + u, and subtracting 2^23 + 128 leaves q.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "wq_device.cuh"

namespace wq {

constexpr float kW8Magic = 8388736.0f;  // 2^23 + 128

// One word (4 codes, low byte first) times s -> two bf16x2 pairs.
__device__ __forceinline__ void dequant_word_w8(uint32_t w, float s, uint32_t& p01, uint32_t& p23) {
    const uint32_t u = w ^ 0x80808080u;
    const float f0 = __uint_as_float(__byte_perm(u, 0x4Bu, 0x4550u));
    const float f1 = __uint_as_float(__byte_perm(u, 0x4Bu, 0x4551u));
    const float f2 = __uint_as_float(__byte_perm(u, 0x4Bu, 0x4552u));
    const float f3 = __uint_as_float(__byte_perm(u, 0x4Bu, 0x4553u));
    const float2 q01 = __fadd2_rn(make_float2(f0, f1), make_float2(-kW8Magic, -kW8Magic));
    const float2 q23 = __fadd2_rn(make_float2(f2, f3), make_float2(-kW8Magic, -kW8Magic));
    const float2 x01 = __fmul2_rn(q01, make_float2(s, s));
    const float2 x23 = __fmul2_rn(q23, make_float2(s, s));
    p01 = bf2_bits(__floats2bfloat162_rn(x01.x, x01.y));
    p23 = bf2_bits(__floats2bfloat162_rn(x23.x, x23.y));
}

}  // namespace wq
