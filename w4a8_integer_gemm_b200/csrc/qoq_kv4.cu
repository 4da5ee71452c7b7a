// qoq_kv4.cu -- 4-bit KV cache with SmoothAttention and the decode attention
// that reads it (one new query token per sequence).
//
// Sources (by page title):
//   "QServe: Low Bit Width Does Not Guarantee High Throughput", section 4,
//       the SmoothAttention paragraph: a per-channel factor lambda moves the
//       cached keys' outliers into the query, K' = K / lambda, Q' = Q *
//       lambda (so Q'K'^T = QK^T), lambda = max|K|^alpha with alpha = 0.5.
//   "QServe Guide: W4A8KV4 Quantization for LLM Serving", The Architecture,
//       subsection 3: the smoothed keys and the values are stored as 4-bit
//       integers with per-channel scales.
// Readings where the pages are silent (shared with the CPU oracle): the
// statistics are per (sequence, KV head, channel) over the cached tokens;
// lambda = fp16(max(sqrt(max|K|), 1e-5)); codes are symmetric, s =
// fp16(max|X'| / 7), code = clamp(round(X' / s), -8, 7), stored as the
// nibble code + 8 (channel 2j in the low nibble of byte j of a token row).
//
// The attention folds every per-channel factor into the query once:
// q'[c] = q[c] * lambda[c] * s_k[c] / sqrt(d), so a score is a dot product
// of q' with the raw 4-bit codes; the value scales s_v are applied once to
// the final weighted sum.  Design for B200 (the pages' A100 kernel with
// FP16 QK/SV products is prior art): flash-decoding over token chunks, one
// CTA per (sequence, KV head, chunk) serving the G query heads that share
// the KV head, FP32 products and sums on the CUDA cores, 8-byte coalesced
// loads (a warp reads 4 whole token rows per load), a second small kernel
// combining the chunks.  The path is HBM-bound for G = 1 and bound by the
// FP32 issue rate for larger G (G FMAs per cached element).
#include <cuda_fp16.h>

#include <cstdint>

#include "qoq_internal.h"
#include "qoq_ptx.cuh"
#include "qoq_quant.cuh"

namespace qoq {
namespace {

constexpr int kD = 128;          // head dimension (the channels of one head)
constexpr int kRowBytes = kD / 2;

// ----------------------------------------------------------- cache writer --
// One CTA per (sequence, KV head), one thread per channel.  Keys: lambda,
// K' = K / lambda, s_k, codes; values: s_v, codes.  Offline (filling a
// cache), not on the decode path.
__global__ void __launch_bounds__(kD) kv4_cache_kernel(const uint16_t *__restrict__ K,
                                                       const uint16_t *__restrict__ V, int L,
                                                       uint8_t *__restrict__ K4, uint8_t *__restrict__ V4,
                                                       uint16_t *__restrict__ lam, uint16_t *__restrict__ s_k,
                                                       uint16_t *__restrict__ s_v)
{
    const int c = threadIdx.x;
    const size_t head = blockIdx.x;
    const uint16_t *k = K + head * L * kD;
    const uint16_t *v = V + head * L * kD;
    float mk = 0.0f, mv = 0.0f;
    for (int l = 0; l < L; ++l) {
        mk = fmaxf(mk, fabsf(half_bits_to_float(k[(size_t)l * kD + c])));
        mv = fmaxf(mv, fabsf(half_bits_to_float(v[(size_t)l * kD + c])));
    }
    double lv = sqrt((double)mk);
    if (lv < 1e-5) lv = 1e-5;
    const uint16_t lb = __half_as_ushort(__double2half(lv));
    const float lf = half_bits_to_float(lb);
    float mks = 0.0f;
    for (int l = 0; l < L; ++l) mks = fmaxf(mks, fabsf(__fdiv_rn(half_bits_to_float(k[(size_t)l * kD + c]), lf)));
    const uint16_t skb = float_to_half_bits(__fdiv_rn(mks, 7.0f));
    const uint16_t svb = float_to_half_bits(__fdiv_rn(mv, 7.0f));
    const float skf = half_bits_to_float(skb), svf = half_bits_to_float(svb);
    lam[head * kD + c] = lb;
    s_k[head * kD + c] = skb;
    s_v[head * kD + c] = svb;
    auto code = [](float x, float s) -> uint32_t {
        if (s == 0.0f) return 8u;
        const float r = fminf(fmaxf(rintf(__fdiv_rn(x, s)), -8.0f), 7.0f);
        return (uint32_t)((int)r + 8);
    };
    for (int l = 0; l < L; ++l) {
        const uint32_t ck = code(__fdiv_rn(half_bits_to_float(k[(size_t)l * kD + c]), lf), skf);
        const uint32_t cv = code(half_bits_to_float(v[(size_t)l * kD + c]), svf);
        const uint32_t pk = __shfl_down_sync(0xffffffffu, ck, 1);
        const uint32_t pv = __shfl_down_sync(0xffffffffu, cv, 1);
        if ((c & 1) == 0) {
            K4[(head * L + l) * kRowBytes + c / 2] = (uint8_t)(ck | (pk << 4));
            V4[(head * L + l) * kRowBytes + c / 2] = (uint8_t)(cv | (pv << 4));
        }
    }
}

// 16 nibbles of a 64-bit word -> the codes as floats (nibble - 8).  The
// nibble is placed in the low mantissa bits of 2^23 (exactly 2^23 + n) and
// 2^23 + 8 is subtracted: one logic op and one add per value, exact, at
// full rate (an integer-to-float conversion is a quarter-rate instruction).
__device__ __forceinline__ float nib_to_float(uint32_t w, int i)
{
    return __int_as_float((int)(0x4B000000u | ((w >> (4 * i)) & 0xFu))) - 8388616.0f;
}

__device__ __forceinline__ void unpack16(uint2 w, float *f)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = nib_to_float(w.x, i);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[8 + i] = nib_to_float(w.y, i);
}

constexpr int kThreads = 256;    // 8 warps; a warp covers 4 token rows per step (8 lanes a row)
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 512;      // tokens per CTA: 32 KB of K codes and 32 KB of V codes

__device__ int g_kv4_error;      // non-zero after a bounded wait of this file's kernels ran out

// ------------------------------------------------- attention, one chunk --
// CTA (sequence b, KV head g, chunk s) over tokens [s*kChunk, min(L, ...)):
// the chunk's K and V codes are contiguous in the cache, so one bulk copy
// each brings them into shared memory at the start (64 KB in flight per
// CTA).  Pass 1 scores every token for the G query heads (from shared
// memory), the chunk's softmax numerators follow, pass 2 sums the value
// codes weighted by them.  The chunk's (max, sum, weighted sums) go to the
// workspace for the combine.
template <int G>
__global__ void __launch_bounds__(kThreads) kv4_attn_chunk_kernel(
    const uint16_t *__restrict__ q, const uint8_t *__restrict__ K4, const uint8_t *__restrict__ V4,
    const uint16_t *__restrict__ lam, const uint16_t *__restrict__ s_k, int Hkv, int L,
    float *__restrict__ part)
{
    extern __shared__ __align__(128) uint8_t dyn[];
    uint8_t *ks = dyn;                                   // [kChunk][64] K codes
    uint8_t *vs = dyn + kChunk * kRowBytes;              // [kChunk][64] V codes
    float *sm = reinterpret_cast<float *>(dyn + 2 * kChunk * kRowBytes);   // [G][kChunk]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + G * kChunk);        // K landed, V landed
    __shared__ float red[G][kWarps];
    __shared__ float gmax[G], gsum[G];
    __shared__ float osum[kWarps][G][kD];
    __shared__ int abort_flag;
    const int bh = blockIdx.x;                   // b * Hkv + kv head
    const int b = bh / Hkv, hk = bh % Hkv;
    const int S = gridDim.y, s = blockIdx.y;
    const int l0 = s * kChunk, n = min(L - l0, kChunk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cb = lane & 7;                     // channel block: channels 16*cb .. 16*cb+15
    const int tw = lane >> 3;                    // row within the warp's 4
    const size_t head = (size_t)bh;
    const uint32_t kbar = smem_addr(bars), vbar = smem_addr(bars + 1);
    const uint32_t bytes = (uint32_t)n * kRowBytes;
    if (threadIdx.x == 0) {
        mbar_init(kbar, 1);
        mbar_init(vbar, 1);
        abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_expect_tx(kbar, bytes);
        bulk_load(smem_addr(ks), K4 + (head * L + l0) * kRowBytes, bytes, kbar);
        mbar_arrive_expect_tx(vbar, bytes);
        bulk_load(smem_addr(vs), V4 + (head * L + l0) * kRowBytes, bytes, vbar);
    }
    // the query of each of the G heads, with lambda, s_k and 1/sqrt(d)
    // folded in (while the copies are in flight)
    const float inv_sqrt_d = 0.08838834764831845f;   // 1 / sqrt(128)
    float qf[G][16];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        const size_t qh = ((size_t)b * Hkv * G + (size_t)hk * G + gi) * kD;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = 16 * cb + i;
            const float f = __fmul_rn(__fmul_rn(half_bits_to_float(__ldg(lam + head * kD + c)),
                                                half_bits_to_float(__ldg(s_k + head * kD + c))),
                                      inv_sqrt_d);
            qf[gi][i] = __fmul_rn(half_bits_to_float(__ldg(q + qh + c)), f);
        }
    }
    __syncthreads();
    const uint64_t budget = 2000000000ull;
    bool ok = wait_bounded(kbar, 0u, &abort_flag, budget);
    // pass 1: scores
    const int nr = (n + 4 * kWarps - 1) / (4 * kWarps) * (4 * kWarps);
    for (int t0 = 4 * warp + tw; t0 < nr && ok; t0 += 4 * kWarps) {
        const uint2 w = t0 < n ? *reinterpret_cast<const uint2 *>(ks + t0 * kRowBytes + 8 * cb)
                               : make_uint2(0x88888888u, 0x88888888u);
        float kc[16];
        unpack16(w, kc);
        float acc[G];
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) a = fmaf(qf[gi][i], kc[i], a);
            acc[gi] = a;
        }
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            acc[gi] += __shfl_xor_sync(0xffffffffu, acc[gi], 4);
            acc[gi] += __shfl_xor_sync(0xffffffffu, acc[gi], 2);
            acc[gi] += __shfl_xor_sync(0xffffffffu, acc[gi], 1);
        }
        if (cb == 0 && t0 < n) {
#pragma unroll
            for (int gi = 0; gi < G; ++gi) sm[gi * kChunk + t0] = acc[gi];
        }
    }
    __syncthreads();
    // the chunk's softmax numerators: exp(score - chunk max), and their sum
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        float m = -INFINITY;
        for (int t = threadIdx.x; t < n; t += kThreads) m = fmaxf(m, sm[gi * kChunk + t]);
        m = warp_max(m);
        if (lane == 0) red[gi][warp] = m;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float m = red[threadIdx.x][0];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[threadIdx.x][w]);
        gmax[threadIdx.x] = m;
    }
    __syncthreads();
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        float sum = 0.0f;
        for (int t = threadIdx.x; t < n; t += kThreads) {
            const float p = expf(sm[gi * kChunk + t] - gmax[gi]);
            sm[gi * kChunk + t] = p;
            sum += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) red[gi][warp] = sum;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float t = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t += red[threadIdx.x][w];
        gsum[threadIdx.x] = t;
    }
    // pass 2: the numerator-weighted sums of the value codes
    float acc2[G][16];
#pragma unroll
    for (int gi = 0; gi < G; ++gi)
#pragma unroll
        for (int i = 0; i < 16; ++i) acc2[gi][i] = 0.0f;
    ok = ok && wait_bounded(vbar, 0u, &abort_flag, budget);
    for (int t0 = 4 * warp + tw; t0 < nr && ok; t0 += 4 * kWarps) {
        const uint2 w = t0 < n ? *reinterpret_cast<const uint2 *>(vs + t0 * kRowBytes + 8 * cb)
                               : make_uint2(0x88888888u, 0x88888888u);
        float vc[16];
        unpack16(w, vc);
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            const float p = t0 < n ? sm[gi * kChunk + t0] : 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) acc2[gi][i] = fmaf(p, vc[i], acc2[gi][i]);
        }
    }
    // sum over the warp's 4 row lanes (same channel block), then the warps
#pragma unroll
    for (int gi = 0; gi < G; ++gi)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            acc2[gi][i] += __shfl_xor_sync(0xffffffffu, acc2[gi][i], 8);
            acc2[gi][i] += __shfl_xor_sync(0xffffffffu, acc2[gi][i], 16);
        }
    if (tw == 0) {
#pragma unroll
        for (int gi = 0; gi < G; ++gi)
#pragma unroll
            for (int i = 0; i < 16; ++i) osum[warp][gi][16 * cb + i] = acc2[gi][i];
    }
    __syncthreads();
    // partial record per query head: [max, sum, kD weighted sums]
    float *rec = part + (((size_t)bh * S + s) * G) * (kD + 2);
    for (int e = threadIdx.x; e < G * kD; e += kThreads) {
        const int gi = e / kD, c = e % kD;
        float t = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t += osum[w][gi][c];
        rec[gi * (kD + 2) + 2 + c] = t;
    }
    if (threadIdx.x < G) {
        rec[threadIdx.x * (kD + 2)] = gmax[threadIdx.x];
        rec[threadIdx.x * (kD + 2) + 1] = gsum[threadIdx.x];
    }
    if (threadIdx.x == 0 && abort_flag) {
        // a wait ran out: report it, and let both copies land before leaving
        atomicExch(&g_kv4_error, 1);
        const uint64_t end = global_timer_ns() + 200000000ull;
        while (!mbar_try_wait(kbar, 0u) && global_timer_ns() < end) {
        }
        while (!mbar_try_wait(vbar, 0u) && global_timer_ns() < end) {
        }
    }
}

// ------------------------------------------------------------- combine --
// One CTA per (sequence, query head), one thread per channel: rescale the
// chunks to the global max, divide, apply s_v once, round to FP16.
template <int G>
__global__ void __launch_bounds__(kD) kv4_combine_kernel(const float *__restrict__ part,
                                                         const uint16_t *__restrict__ s_v, int Hkv, int S,
                                                         uint16_t *__restrict__ out)
{
    const int bq = blockIdx.x;                  // b * Hq + query head
    const int Hq = Hkv * G;
    const int b = bq / Hq, h = bq % Hq;
    const int hk = h / G, gi = h % G;
    const size_t bh = (size_t)b * Hkv + hk;
    const int c = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, part[((bh * S + s) * G + gi) * (kD + 2)]);
    float den = 0.0f, num = 0.0f;
    for (int s = 0; s < S; ++s) {
        const float *rec = part + ((bh * S + s) * G + gi) * (kD + 2);
        const float w = expf(rec[0] - M);
        den = fmaf(rec[1], w, den);
        num = fmaf(rec[2 + c], w, num);
    }
    const float sv = half_bits_to_float(__ldg(s_v + bh * kD + c));
    out[(size_t)bq * kD + c] = float_to_half_bits(__fmul_rn(__fdiv_rn(num, den), sv));
}

}  // namespace

size_t kv4_workspace_bytes(int B, int Hq, int Hkv, int L)
{
    const long long S = (L + kChunk - 1) / kChunk;
    return (size_t)B * Hq * S * (kD + 2) * sizeof(float);
}

cudaError_t launch_kv4_cache(const uint16_t *K, const uint16_t *V, int B, int Hkv, int L, uint8_t *K4, uint8_t *V4,
                             uint16_t *lam, uint16_t *s_k, uint16_t *s_v, cudaStream_t stream)
{
    kv4_cache_kernel<<<(unsigned)(B * Hkv), kD, 0, stream>>>(K, V, L, K4, V4, lam, s_k, s_v);
    return cudaGetLastError();
}

template <int G>
static cudaError_t launch_attn_g(const uint16_t *q, const uint8_t *K4, const uint8_t *V4, const uint16_t *lam,
                                 const uint16_t *s_k, const uint16_t *s_v, int B, int Hkv, int L, uint16_t *out,
                                 float *part, cudaStream_t stream)
{
    const int S = (L + kChunk - 1) / kChunk;
    const size_t smem = 2 * (size_t)kChunk * kRowBytes + (size_t)G * kChunk * sizeof(float) + 16;
    auto k1 = kv4_attn_chunk_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k1<<<dim3((unsigned)(B * Hkv), (unsigned)S), kThreads, smem, stream>>>(q, K4, V4, lam, s_k, Hkv, L, part);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    kv4_combine_kernel<G><<<(unsigned)(B * Hkv * G), kD, 0, stream>>>(part, s_v, Hkv, S, out);
    return cudaGetLastError();
}

cudaError_t launch_kv4_attention(const uint16_t *q, const uint8_t *K4, const uint8_t *V4, const uint16_t *lam,
                                 const uint16_t *s_k, const uint16_t *s_v, int B, int Hq, int Hkv, int L,
                                 uint16_t *out, void *workspace, cudaStream_t stream)
{
    float *part = reinterpret_cast<float *>(workspace);
    switch (Hq / Hkv) {
    case 1: return launch_attn_g<1>(q, K4, V4, lam, s_k, s_v, B, Hkv, L, out, part, stream);
    case 2: return launch_attn_g<2>(q, K4, V4, lam, s_k, s_v, B, Hkv, L, out, part, stream);
    case 4: return launch_attn_g<4>(q, K4, V4, lam, s_k, s_v, B, Hkv, L, out, part, stream);
    default: return launch_attn_g<8>(q, K4, V4, lam, s_k, s_v, B, Hkv, L, out, part, stream);
    }
}

cudaError_t read_and_clear_kv4_error(int *value)
{
    *value = 0;
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_kv4_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_kv4_error, &zero, sizeof(int));
    }
    *value = v;
    return e;
}

}  // namespace qoq
