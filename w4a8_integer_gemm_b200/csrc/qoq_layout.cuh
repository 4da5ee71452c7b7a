// qoq_layout.cuh -- the packed UINT4 weight layout and the in-register
// INT4 -> INT8 expansion shared by the GEMM and the dequantization kernel.
//
// Expansion rule ("QServe: Low Bit Width Does Not Guarantee High
// Throughput", section 4, paragraph after the stage-2 equation; paper card
// "QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
// Serving", Key points: multiply first, subtract afterward):
//
//     W8hat = q * s_g - zs,   zs = z * s_g precomputed offline.
//
// Four codes sit in the four byte lanes of a 32-bit register.  The
// protective range gives q*s_g <= 15*16 = 240 < 256 for every code, so one
// 32-bit integer multiply by s_g scales all four lanes without a carry
// between them.  The zero compensation is then subtracted with a +128 bias:
// adding the constant (128 - zs) * 0x01010101 (mod 2^32) yields, in every
// lane, W8hat + 128, which lies in [1, 255] for every code the quantizer
// emits (|W8hat| <= 127), so the 32-bit sum is exactly the four biased bytes
// and no lane borrows from its neighbour.  XOR with 0x80808080 removes the
// bias and leaves four two's-complement INT8 weights.  Per four weights:
// one AND (or one shift and one AND), one IMAD, one XOR.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace qoq {

constexpr int kPanelRows = 128;     // output channels per packed panel (= MMA M)
constexpr int kBlockK = 128;        // K per packed chunk (= one pipeline stage)
constexpr int kSlabK = 32;          // K per 16-byte row slice (= one MMA K step)
constexpr int kSlabBytes = 2048;    // 128 rows x 16 bytes
constexpr int kChunkBytes = 8192;   // 4 slabs of codes
constexpr int kChunkTabBytes = 256; // G = 128: the chunk's s_g[128], then zs[128]

// Bytes from one chunk to the next: with 128-wide groups every chunk
// carries its group's tables right after its codes, so one copy brings
// both; per-channel tables (G = K) are not repeated in the chunks.
__host__ __device__ __forceinline__ int chunk_stride(int G)
{
    return kChunkBytes + (G == kBlockK ? kChunkTabBytes : 0);
}

// Byte offset of chunk (panel p, K block b) in the packed buffer.
__host__ __device__ __forceinline__ size_t chunk_offset(int p, int b, int K, int G)
{
    return ((size_t)p * (size_t)(K / kBlockK) + (size_t)b) * (size_t)chunk_stride(G);
}

// The biased zero-compensation constant for a group, replicated in 4 lanes.
__device__ __forceinline__ uint32_t zero_comp_bias(uint32_t zs)
{
    return (128u - zs) * 0x01010101u;
}

// One packed word (8 codes) -> two words of 4 INT8 weights.  `lo` holds the
// weights of the low nibbles (k0+4w .. k0+4w+3), `hi` those of the high
// nibbles (k0+16+4w .. k0+16+4w+3).
__device__ __forceinline__ void dequant_word(uint32_t v, uint32_t sg, uint32_t bias, uint32_t &lo,
                                             uint32_t &hi)
{
    const uint32_t ql = v & 0x0F0F0F0Fu;
    const uint32_t qh = (v >> 4) & 0x0F0F0F0Fu;
    lo = (ql * sg + bias) ^ 0x80808080u;
    hi = (qh * sg + bias) ^ 0x80808080u;
}

// One 16-byte row slice (32 codes of one channel) -> 8 words holding the
// INT8 weights of k0 .. k0+31 in order (word i = k0+4i .. k0+4i+3, lowest k
// in the lowest byte).
__device__ __forceinline__ void dequant_slab(const uint4 &v, uint32_t sg, uint32_t bias, uint32_t *out)
{
    dequant_word(v.x, sg, bias, out[0], out[4]);
    dequant_word(v.y, sg, bias, out[1], out[5]);
    dequant_word(v.z, sg, bias, out[2], out[6]);
    dequant_word(v.w, sg, bias, out[3], out[7]);
}

}  // namespace qoq
