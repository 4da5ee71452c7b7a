// qoq_epilogue.cuh -- the FP16 output of the W4A8 layer from its INT32
// sums, shared by every kernel that writes Y, so that all of them round
// alike (and alike with the oracle).
//
// Source: "QServe Guide: W4A8KV4 Quantization for LLM Serving", Deep Dive,
// subsection 1: the INT32 sum is rescaled once by the token scale and the
// channel scale.  Reading where the page is silent: y = fp16(((float)acc *
// s_x) * s_c), each product rounded to FP32; the fused residual adds in
// FP32 and rounds once to FP16; SiLU(g) = g / (1 + exp(-g)) in FP32.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace qoq {

__device__ __forceinline__ uint16_t scale_to_half(int32_t acc, float sx, float sc)
{
    const float y = __fmul_rn(__fmul_rn(__int2float_rn(acc), sx), sc);
    return __half_as_ushort(__float2half_rn(y));
}

// y + r for one FP16 pair: added in FP32, rounded once
__device__ __forceinline__ uint16_t add_half(uint16_t y, uint16_t r)
{
    const float s = __fadd_rn(__half2float(__ushort_as_half(y)), __half2float(__ushort_as_half(r)));
    return __half_as_ushort(__float2half_rn(s));
}

__device__ __forceinline__ uint32_t add_half2(uint32_t y, uint32_t r)
{
    return (uint32_t)add_half((uint16_t)(y & 0xFFFFu), (uint16_t)(r & 0xFFFFu)) |
           ((uint32_t)add_half((uint16_t)(y >> 16), (uint16_t)(r >> 16)) << 16);
}

__device__ __forceinline__ uint16_t silu_mul_half(uint16_t gb, uint16_t ub)
{
    const float g = __half2float(__ushort_as_half(gb));
    const float u = __half2float(__ushort_as_half(ub));
    const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
    return __half_as_ushort(__float2half_rn(__fmul_rn(silu, u)));
}

__device__ __forceinline__ uint32_t silu_mul_half2(uint32_t g, uint32_t u)
{
    return (uint32_t)silu_mul_half((uint16_t)(g & 0xFFFFu), (uint16_t)(u & 0xFFFFu)) |
           ((uint32_t)silu_mul_half((uint16_t)(g >> 16), (uint16_t)(u >> 16)) << 16);
}

}  // namespace qoq
