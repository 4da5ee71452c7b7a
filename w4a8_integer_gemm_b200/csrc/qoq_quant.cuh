// qoq_quant.cuh -- per-token INT8 activation quantization of one row's
// FP16 values, shared by the stand-alone quantizer and the GEMM that
// quantizes its own input.
//
// Source: "QServe Guide: W4A8KV4 Quantization for LLM Serving", Deep Dive,
// subsection 1, the activation equation: s_x = max|x| / 127 per token,
// X8 = round(x / s_x).  Readings where the page is silent: s_x is stored
// as FP16 (round to nearest even) and the stored value is the one used to
// quantize; round is half to even on the IEEE quotient; a zero scale
// quantizes the row to zero; codes are clamped to [-128, 127].
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace qoq {

__device__ __forceinline__ float half_bits_to_float(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t float_to_half_bits(float f)
{
    return __half_as_ushort(__float2half_rn(f));
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// max |x| over the 8 FP16 values of a 16-byte vector
__device__ __forceinline__ float absmax8(const uint4 &v)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = fmaxf(m, fabsf(half_bits_to_float((uint16_t)(w[i] & 0xFFFFu))));
        m = fmaxf(m, fabsf(half_bits_to_float((uint16_t)(w[i] >> 16))));
    }
    return m;
}

// The token scale from the row's max |x|.
__device__ __forceinline__ uint16_t token_scale_bits(float amax)
{
    return float_to_half_bits(__fdiv_rn(amax, 127.0f));
}

__device__ __forceinline__ int quant_x(float x, float sx)
{
    if (sx == 0.0f) return 0;
    return (int)fminf(fmaxf(rintf(__fdiv_rn(x, sx)), -128.0f), 127.0f);
}

// 8 FP16 values -> 8 INT8 codes (in order, lowest address in the lowest byte)
__device__ __forceinline__ uint2 quant8(const uint4 &v, float sx)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (uint32_t)quant_x(half_bits_to_float((uint16_t)(w[i] & 0xFFFFu)), sx) & 0xFFu;
        const uint32_t hi = (uint32_t)quant_x(half_bits_to_float((uint16_t)(w[i] >> 16)), sx) & 0xFFu;
        o[i >> 1] |= (lo | (hi << 8)) << (16 * (i & 1));
    }
    return make_uint2(o[0], o[1]);
}

}  // namespace qoq
