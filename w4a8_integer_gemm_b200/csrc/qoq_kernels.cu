// qoq_kernels.cu -- the offline weight packer, the per-token activation
// quantizer and the INT8 weight expansion used for inspection.
//
// Sources (by page title):
//   "QServe: Low Bit Width Does Not Guarantee High Throughput", section 4,
//       stage-1 equation (per-channel symmetric INT8 in [-119,119]) and
//       stage-2 equation (group UINT4 with integer scale and zero).
//   "QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
//       Serving" (paper card), Key points: FP16 per-channel scales.
//   "QServe Guide: W4A8KV4 Quantization for LLM Serving", Deep Dive,
//       subsection 1: per-token activation equation.
#include <cuda_fp16.h>

#include "qoq_internal.h"
#include "qoq_layout.cuh"
#include "qoq_ptx.cuh"
#include "qoq_quant.cuh"

namespace qoq {
namespace {

__device__ __forceinline__ int warp_min_i(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_max_i(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Stage 1 for one value: clamp(round(w / sc), -119, 119), IEEE division,
// round half to even; a zero scale quantizes to zero.
__device__ __forceinline__ int stage1(float w, float sc)
{
    if (sc == 0.0f) return 0;
    return (int)fminf(fmaxf(rintf(__fdiv_rn(w, sc)), -119.0f), 119.0f);
}

// Stage 2 code: clamp(round(w8 / s_g) + z, 0, 15).  w8 in [-119,119] and
// s_g in [1,16]: the FP32 quotient is within 2^-20 of the exact rational,
// non-tie quotients lie at least 1/32 from a half, and ties are exact, so
// rintf gives the exact round-half-to-even of the rational.
__device__ __forceinline__ uint32_t stage2_code(int w8, float sgf, int z)
{
    const int v = (int)rintf(__fdiv_rn((float)w8, sgf)) + z;
    return (uint32_t)min(max(v, 0), 15);
}

// ------------------------------------------------------------ packer --
// One warp per output channel n.  Lane l covers k = kc + 4l .. kc + 4l + 3
// of each 128-wide chunk kc.
// Optional outputs for inspection: z_dbg [N][K/G] the zero points, q_dbg
// [N][K] the canonical codes, one per byte.
__global__ void __launch_bounds__(256) pack_kernel(const float *__restrict__ W, int N, int K, int G,
                                                   uint8_t *__restrict__ Wp, uint16_t *__restrict__ s_c,
                                                   uint8_t *__restrict__ s_g, uint8_t *__restrict__ zs,
                                                   uint8_t *__restrict__ z_dbg, uint8_t *__restrict__ q_dbg,
                                                   bool gate_up)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + warp;  // packed row (output channel position)
    if (n >= N) return;
    // the source row: itself, or for a gate/up pair, gate row 64p + r (r < 64)
    // or up row N/2 + 64p + r - 64 of packed panel p
    const int pr = n % kPanelRows, pp = n / kPanelRows;
    const int src = !gate_up ? n : (pr < 64 ? 64 * pp + pr : N / 2 + 64 * pp + pr - 64);
    const float *w = W + (size_t)src * K;

    float amax = 0.0f;
    for (int k = lane * 4; k < K; k += 128) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(w + k));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    amax = warp_max(amax);
    const uint16_t sch = float_to_half_bits(__fdiv_rn(amax, 119.0f));
    const float sc = half_bits_to_float(sch);
    if (lane == 0) s_c[n] = sch;

    const int p = n / kPanelRows, rr = n % kPanelRows;
    for (int g = 0; g < K / G; ++g) {
        const int k_lo = g * G, k_hi = k_lo + G;
        int mn = 0, mx = 0;
        for (int k = k_lo + lane * 4; k < k_hi; k += 128) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(w + k));
            const int a0 = stage1(v.x, sc), a1 = stage1(v.y, sc), a2 = stage1(v.z, sc), a3 = stage1(v.w, sc);
            mn = min(mn, min(min(a0, a1), min(a2, a3)));
            mx = max(mx, max(max(a0, a1), max(a2, a3)));
        }
        mn = warp_min_i(mn);
        mx = warp_max_i(mx);
        const int sg = max(1, (mx - mn + 14) / 15);
        const float sgf = (float)sg;
        const int z = (int)rintf(__fdiv_rn((float)(-mn), sgf));
        if (lane == 0) {
            const size_t ti = ((size_t)p * (K / G) + g) * kPanelRows + rr;
            s_g[ti] = (uint8_t)sg;
            zs[ti] = (uint8_t)(z * sg);
            if (z_dbg) z_dbg[(size_t)n * (K / G) + g] = (uint8_t)z;
            if (G == kBlockK) {  // the copy inside the group's chunk
                uint8_t *tab = Wp + chunk_offset(p, g, K, G) + kChunkBytes;
                tab[rr] = (uint8_t)sg;
                tab[kPanelRows + rr] = (uint8_t)(z * sg);
            }
        }
        for (int kc = k_lo; kc < k_hi; kc += 128) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(w + kc + lane * 4));
            const uint32_t mine = stage2_code(stage1(v.x, sc), sgf, z) | (stage2_code(stage1(v.y, sc), sgf, z) << 8) |
                                  (stage2_code(stage1(v.z, sc), sgf, z) << 16) |
                                  (stage2_code(stage1(v.w, sc), sgf, z) << 24);
            if (q_dbg) *reinterpret_cast<uint32_t *>(q_dbg + (size_t)n * K + kc + lane * 4) = mine;
            // lanes l and l+4 of each group of 8 fill the low and high
            // nibbles of the same packed word
            const uint32_t partner = __shfl_down_sync(0xffffffffu, mine, 4);
            if ((lane & 7) < 4) {
                const int slab = lane >> 3, word = lane & 7;
                uint8_t *dst = Wp + chunk_offset(p, kc / kBlockK, K, G) + slab * kSlabBytes + rr * 16 + word * 4;
                *reinterpret_cast<uint32_t *>(dst) = mine | (partner << 4);
            }
        }
    }
}

// quant_x(x, sx) = clamp(rint(fl(x / sx))) without a division for almost
// every x.  With r = fl(1/sx), qa = fl(x * r) differs from fl(x / sx) by at
// most |x/sx| * 3 * 2^-24 (two roundings of r and qa, one of the quotient):
// under 2.3e-5 where |x/sx| < 128.5, the only quotients the clamp does not
// decide, and under 2^-12 up to |x/sx| = 1365.  So when qa is farther than
// 2^-12 from the nearest half-integer, no half-integer lies between qa and
// fl(x / sx), and both round to the same integer; clamping first to
// [-128, 127] (whose ends are integers) changes neither result, and beyond
// |x/sx| = 1365 both sides clamp alike.  The rounding itself: adding 1.5 * 2^23 to a
// float of magnitude below 2^22 leaves a float of unit spacing, so the sum
// is rounded to an integer, ties to even as rint rounds, and that integer's
// low byte (two's complement) is the low byte of the sum's bits.
constexpr float kRoundMagic = 12582912.0f;        // 1.5 * 2^23
constexpr float kFarFromHalf = 0.499755859375f;   // 1/2 - 2^-12

// 8 FP16 values -> 8 INT8 codes (lowest address in the lowest byte).  The
// rare vector with an element within 2^-12 of a rounding boundary (or any
// vector of a row with s_x = 0) is redone with the IEEE division.
__device__ __forceinline__ uint2 quant8_fast(const uint4 &v, float sx, float rsx)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t y[8];
    bool near = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float c = fminf(fmaxf(half_bits_to_float((uint16_t)(w[i >> 1] >> (16 * (i & 1)))) * rsx, -128.0f),
                              127.0f);
        const float r = c + kRoundMagic;
        near |= fabsf(c - (r - kRoundMagic)) >= kFarFromHalf;
        y[i] = __float_as_uint(r);
    }
    if (near || sx == 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            y[i] = (uint32_t)quant_x(half_bits_to_float((uint16_t)(w[i >> 1] >> (16 * (i & 1)))), sx);
    }
    // the low byte of each: two per half word, then the halves side by side
    const uint32_t a = __byte_perm(y[0], y[1], 0x0040u), b = __byte_perm(y[2], y[3], 0x0040u);
    const uint32_t c = __byte_perm(y[4], y[5], 0x0040u), d = __byte_perm(y[6], y[7], 0x0040u);
    return make_uint2(__byte_perm(a, b, 0x5410u), __byte_perm(c, d, 0x5410u));
}

// max |x| of 8 FP16 values, taken in FP16 (exact), returned as a float
__device__ __forceinline__ float absmax8_h2(const uint4 &v)
{
    __half2 m = __habs2(__halves2half2(__ushort_as_half((uint16_t)v.x), __ushort_as_half((uint16_t)(v.x >> 16))));
    const uint32_t w[3] = {v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 3; ++i)
        m = __hmax2(m, __habs2(__halves2half2(__ushort_as_half((uint16_t)w[i]), __ushort_as_half((uint16_t)(w[i] >> 16)))));
    return fmaxf(__low2float(m), __high2float(m));
}

// ---------------------------------------------------- activation quant --
// One CTA per token row: read the row once (kept in registers up to
// T * CACHE * 8 values), reduce max|x|, then quantize.  Short rows
// (K <= 4096) take a small CTA (128 threads, few registers) so that the
// quantizer of the next layer fits on an SM beside a running GEMM CTA: it
// can then start, and trigger the launch of its own GEMM, before the
// current GEMM ends.  Longer rows take 256 threads with 4 vectors each
// (K <= 8192) or 8 (K <= 16384 in registers), so that every load of the
// row is in flight at once: the quantizer of a large batch is on the
// step's critical path.
// With rowsum non-null it also writes rowsum[m] = sum_k X8[m][k] (INT32).
template <int T, int CACHE>
__global__ void __launch_bounds__(T, T == 128 ? 10 : CACHE <= 4 ? 5 : 4) act_quant_kernel(const uint16_t *__restrict__ X, int K,
                                                                        int8_t *__restrict__ X8,
                                                                        uint16_t *__restrict__ s_x,
                                                                        int32_t *__restrict__ rowsum)
{
    __shared__ float red[T / 32];
    __shared__ int rsum[T / 32];
    // the GEMM that consumes X8 may launch now and start streaming weights;
    // it waits for this grid to finish before it reads X8 or s_x
    grid_launch_dependents();
    // this grid may itself have launched early (programmatic dependent
    // launch): X, and the buffers written below, belong to the kernels
    // before it until they have finished
    grid_dependency_wait();
    const int m = blockIdx.x;
    const uint4 *row = reinterpret_cast<const uint4 *>(X + (size_t)m * K);
    uint2 *out = reinterpret_cast<uint2 *>(X8 + (size_t)m * K);
    const int nvec = K / 8;
    uint4 cache[CACHE];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
        const int idx = threadIdx.x + i * T;
        if (idx < nvec) cache[i] = __ldcs(row + idx);
    }
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
        const int idx = threadIdx.x + i * T;
        if (idx < nvec) amax = fmaxf(amax, absmax8_h2(cache[i]));
    }
    for (int idx = threadIdx.x + CACHE * T; idx < nvec; idx += T)
        amax = fmaxf(amax, absmax8_h2(__ldg(row + idx)));
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < T / 32 ? red[threadIdx.x] : 0.0f;
        v = warp_max(v);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    amax = red[0];
    const uint16_t sxh = token_scale_bits(amax);
    const float sx = half_bits_to_float(sxh);
    const float rsx = sx == 0.0f ? 0.0f : __frcp_rn(sx);
    if (threadIdx.x == 0) s_x[m] = sxh;
    int sum = 0;  // sum of this thread's INT8 codes (rowsum only)
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
        const int idx = threadIdx.x + i * T;
        if (idx < nvec) {
            const uint2 v = quant8_fast(cache[i], sx, rsx);
            out[idx] = v;
            if (rowsum) sum = __dp4a((int)v.y, 0x01010101, __dp4a((int)v.x, 0x01010101, sum));
        }
    }
    for (int idx = threadIdx.x + CACHE * T; idx < nvec; idx += T) {
        const uint2 v = quant8_fast(__ldg(row + idx), sx, rsx);
        out[idx] = v;
        if (rowsum) sum = __dp4a((int)v.y, 0x01010101, __dp4a((int)v.x, 0x01010101, sum));
    }
    if (rowsum) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if ((threadIdx.x & 31) == 0) rsum[threadIdx.x >> 5] = sum;
        __syncthreads();
        if (threadIdx.x == 0) {
            int t = 0;
#pragma unroll
            for (int w = 0; w < T / 32; ++w) t += rsum[w];
            rowsum[m] = t;
        }
    }
}

// ------------------------------------------------- INT8 weight expand --
// One thread per (channel n, 32-wide K slice): the GEMM's dequant routine
// on one 16-byte row slice, written out as 32 INT8 weights.  Like the GEMM,
// it takes 128-wide groups' tables from the chunk and per-channel tables
// from s_g / zs.
__global__ void dequant_kernel(const uint8_t *__restrict__ Wp, const uint8_t *__restrict__ s_g,
                               const uint8_t *__restrict__ zs, int N, int K, int G, int8_t *__restrict__ out)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int slices = K / kSlabK;
    if (idx >= (size_t)N * slices) return;
    const int n = (int)(idx / slices);
    const int k0 = (int)(idx % slices) * kSlabK;
    const uint8_t *chunk = Wp + chunk_offset(n / kPanelRows, k0 / kBlockK, K, G);
    const uint4 v = *reinterpret_cast<const uint4 *>(chunk + ((k0 % kBlockK) / kSlabK) * kSlabBytes +
                                                     (n % kPanelRows) * 16);
    uint32_t sg, zsv;
    if (G == kBlockK) {
        sg = chunk[kChunkBytes + n % kPanelRows];
        zsv = chunk[kChunkBytes + kPanelRows + n % kPanelRows];
    } else {
        const size_t ti = ((size_t)(n / kPanelRows) * (K / G) + k0 / G) * kPanelRows + n % kPanelRows;
        sg = s_g[ti];
        zsv = zs[ti];
    }
    const uint32_t bias = zero_comp_bias(zsv);
    uint32_t w8[8];
    dequant_slab(v, sg, bias, w8);
    uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)n * K + k0);
    dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
    dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
}

// ------------------------------------------- W8A8 yardstick weights --
// One warp per output channel: s_w = fp16(max|W| / 127), then
// W8 = clamp(round(W / s_w), -127, 127) with IEEE division and round half to
// even, using the stored FP16 scale (a zero scale gives a zero row).
__global__ void __launch_bounds__(256) quantize_w8_kernel(const float *__restrict__ W, int N, int K,
                                                          int8_t *__restrict__ W8, uint16_t *__restrict__ s_w)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + warp;
    if (n >= N) return;
    const float *w = W + (size_t)n * K;
    float amax = 0.0f;
    for (int k = lane * 4; k < K; k += 128) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(w + k));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    amax = warp_max(amax);
    const uint16_t bits = float_to_half_bits(__fdiv_rn(amax, 127.0f));
    const float sw = half_bits_to_float(bits);
    if (lane == 0) s_w[n] = bits;
    for (int k = lane * 4; k < K; k += 128) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(w + k));
        const float e[4] = {v.x, v.y, v.z, v.w};
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = sw == 0.0f ? 0 : (int)fminf(fmaxf(rintf(__fdiv_rn(e[i], sw)), -127.0f), 127.0f);
            word |= (uint32_t)(c & 0xFF) << (8 * i);
        }
        *reinterpret_cast<uint32_t *>(W8 + (size_t)n * K + k) = word;
    }
}

// ------------------------------------------------ stand-alone epilogue --
// The output rescaling on INT32 sums that were computed elsewhere (the
// all-reduced partials of a K-split layer): one thread per 8 consecutive
// outputs of a row, 16-byte loads and stores, the GEMM epilogue's rounding
// order.  HBM-bound: 4 + 2 bytes per output.
__global__ void __launch_bounds__(256) epilogue_i32_kernel(const int32_t *__restrict__ acc,
                                                           const uint16_t *__restrict__ s_x,
                                                           const uint16_t *__restrict__ s_c, int M, int N,
                                                           uint16_t *__restrict__ Y)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int per_row = N / 8;
    if (idx >= (size_t)M * per_row) return;
    const int m = (int)(idx / per_row);
    const int n0 = (int)(idx % per_row) * 8;
    const int4 a0 = __ldcs(reinterpret_cast<const int4 *>(acc + (size_t)m * N + n0));
    const int4 a1 = __ldcs(reinterpret_cast<const int4 *>(acc + (size_t)m * N + n0 + 4));
    const uint4 c = __ldg(reinterpret_cast<const uint4 *>(s_c + n0));
    const float sx = half_bits_to_float(__ldg(s_x + m));
    const int av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __fmul_rn(__fmul_rn(__int2float_rn(av[2 * i]), sx),
                                   half_bits_to_float((uint16_t)(cw[i] & 0xFFFFu)));
        const float hi = __fmul_rn(__fmul_rn(__int2float_rn(av[2 * i + 1]), sx),
                                   half_bits_to_float((uint16_t)(cw[i] >> 16)));
        o[i] = (uint32_t)float_to_half_bits(lo) | ((uint32_t)float_to_half_bits(hi) << 16);
    }
    *reinterpret_cast<uint4 *>(Y + (size_t)m * N + n0) = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

cudaError_t launch_pack(const float *W, int N, int K, int G, uint8_t *Wp, uint16_t *s_c, uint8_t *s_g, uint8_t *zs,
                        uint8_t *z_dbg, uint8_t *q_dbg, cudaStream_t stream, bool gate_up)
{
    pack_kernel<<<(N + 7) / 8, 256, 0, stream>>>(W, N, K, G, Wp, s_c, s_g, zs, z_dbg, q_dbg, gate_up);
    return cudaGetLastError();
}

cudaError_t launch_act_quant(const uint16_t *X, int M, int K, int8_t *X8, uint16_t *s_x, int32_t *rowsum,
                             cudaStream_t stream)
{
    // programmatic dependent launch: the CTAs may be scheduled while the
    // previous kernel (for instance the previous layer's GEMM) finishes;
    // they wait for it at the top of the kernel
    const bool wide = K > 4096;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)M);
    cfg.blockDim = dim3(wide ? 256 : 128);
    // (K <= 8192: four vectors per thread, few registers, six CTAs per SM)
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = !wide     ? cudaLaunchKernelEx(&cfg, act_quant_kernel<128, 4>, X, K, X8, s_x, rowsum)
                    : K <= 8192 ? cudaLaunchKernelEx(&cfg, act_quant_kernel<256, 4>, X, K, X8, s_x, rowsum)
                                : cudaLaunchKernelEx(&cfg, act_quant_kernel<256, 8>, X, K, X8, s_x, rowsum);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_quantize_w8(const float *W, int N, int K, int8_t *W8, uint16_t *s_w, cudaStream_t stream)
{
    quantize_w8_kernel<<<(N + 7) / 8, 256, 0, stream>>>(W, N, K, W8, s_w);
    return cudaGetLastError();
}

cudaError_t launch_epilogue_i32(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c, int M, int N,
                                uint16_t *Y, cudaStream_t stream)
{
    const size_t threads = (size_t)M * (N / 8);
    epilogue_i32_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(acc, s_x, s_c, M, N, Y);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t *Wp, const uint8_t *s_g, const uint8_t *zs, int N, int K, int G,
                           int8_t *W8hat, cudaStream_t stream)
{
    const size_t threads = (size_t)N * (K / kSlabK);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    dequant_kernel<<<blocks, 256, 0, stream>>>(Wp, s_g, zs, N, K, G, W8hat);
    return cudaGetLastError();
}

}  // namespace qoq
