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

// 16 nibbles of a 64-bit word -> the codes as floats (nibble - 8).
__device__ __forceinline__ void unpack16(uint2 w, float *f)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = (float)(int)((w.x >> (4 * i)) & 0xFu) - 8.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) f[8 + i] = (float)(int)((w.y >> (4 * i)) & 0xFu) - 8.0f;
}

constexpr int kThreads = 128;    // 4 warps; a warp covers 4 tokens per load (8 lanes a token)

// ------------------------------------------------- attention, one chunk --
// CTA (sequence b, KV head g, chunk s) over tokens [s*Lc, min(L, (s+1)*Lc)):
// pass 1 scores every token for the G query heads, the chunk's softmax
// numerators follow, pass 2 sums the codes of V weighted by them.  The
// chunk's (max, sum, weighted sums) go to the workspace for the combine.
template <int G>
__global__ void __launch_bounds__(kThreads) kv4_attn_chunk_kernel(
    const uint16_t *__restrict__ q, const uint8_t *__restrict__ K4, const uint8_t *__restrict__ V4,
    const uint16_t *__restrict__ lam, const uint16_t *__restrict__ s_k, int Hkv, int L, int Lc,
    float *__restrict__ part)
{
    extern __shared__ float sm[];                // [G][Lc] scores, then numerators
    __shared__ float red[G][kThreads / 32];
    __shared__ float gmax[G], gsum[G];
    __shared__ float osum[kThreads / 32][G][kD];
    const int bh = blockIdx.x;                   // b * Hkv + kv head
    const int b = bh / Hkv, hk = bh % Hkv;
    const int S = gridDim.y, s = blockIdx.y;
    const int l0 = s * Lc, l1 = min(L, l0 + Lc);
    const int n = l1 - l0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cb = lane & 7;                     // channel block: channels 16*cb .. 16*cb+15
    const int tw = lane >> 3;                    // token within the warp's 4
    const size_t head = (size_t)bh;
    const float inv_sqrt_d = 0.08838834764831845f;   // 1 / sqrt(128)
    // the query of each of the G heads, with lambda, s_k and 1/sqrt(d) folded in
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
    // pass 1: scores
    const uint2 *krow = reinterpret_cast<const uint2 *>(K4 + head * (size_t)L * kRowBytes);
    for (int t0 = 4 * warp + tw; t0 < ((n + 15) & ~15); t0 += 16) {
        const bool live = t0 < n;
        const uint2 w = live ? __ldcs(krow + (size_t)(l0 + t0) * (kRowBytes / 8) + cb) : make_uint2(0x88888888u, 0x88888888u);
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
        if (cb == 0 && live) {
#pragma unroll
            for (int gi = 0; gi < G; ++gi) sm[gi * Lc + t0] = acc[gi];
        }
    }
    __syncthreads();
    // the chunk's softmax numerators: exp(score - chunk max), and their sum
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        float m = -INFINITY;
        for (int t = threadIdx.x; t < n; t += kThreads) m = fmaxf(m, sm[gi * Lc + t]);
        m = warp_max(m);
        if (lane == 0) red[gi][warp] = m;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float m = red[threadIdx.x][0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[threadIdx.x][w]);
        gmax[threadIdx.x] = m;
    }
    __syncthreads();
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        float sum = 0.0f;
        for (int t = threadIdx.x; t < n; t += kThreads) {
            const float p = expf(sm[gi * Lc + t] - gmax[gi]);
            sm[gi * Lc + t] = p;
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
        for (int w = 0; w < kThreads / 32; ++w) t += red[threadIdx.x][w];
        gsum[threadIdx.x] = t;
    }
    // pass 2: the numerator-weighted sums of the value codes
    float acc2[G][16];
#pragma unroll
    for (int gi = 0; gi < G; ++gi)
#pragma unroll
        for (int i = 0; i < 16; ++i) acc2[gi][i] = 0.0f;
    const uint2 *vrow = reinterpret_cast<const uint2 *>(V4 + head * (size_t)L * kRowBytes);
    for (int t0 = 4 * warp + tw; t0 < ((n + 15) & ~15); t0 += 16) {
        const bool live = t0 < n;
        const uint2 w = live ? __ldcs(vrow + (size_t)(l0 + t0) * (kRowBytes / 8) + cb) : make_uint2(0x88888888u, 0x88888888u);
        float vc[16];
        unpack16(w, vc);
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            const float p = live ? sm[gi * Lc + t0] : 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) acc2[gi][i] = fmaf(p, vc[i], acc2[gi][i]);
        }
    }
    // sum over the warp's 4 token lanes (same channel block), then the warps
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
        for (int w = 0; w < kThreads / 32; ++w) t += osum[w][gi][c];
        rec[gi * (kD + 2) + 2 + c] = t;
    }
    if (threadIdx.x < G) {
        rec[threadIdx.x * (kD + 2)] = gmax[threadIdx.x];
        rec[threadIdx.x * (kD + 2) + 1] = gsum[threadIdx.x];
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

// chunk length (tokens, a multiple of 16) for a problem: about two CTAs per
// SM over all (sequence, KV head, chunk), at most 1024 tokens per chunk
static int kv4_chunk(int B, int Hkv, int L)
{
    const long long heads = (long long)B * Hkv;
    long long S = (2 * kMaxCtas + heads - 1) / heads;
    if (S < 1) S = 1;
    long long Lc = (L + S - 1) / S;
    Lc = (Lc + 15) / 16 * 16;
    if (Lc < 64) Lc = 64;
    if (Lc > 1024) Lc = 1024;
    return (int)Lc;
}

size_t kv4_workspace_bytes(int B, int Hq, int Hkv, int L)
{
    const int Lc = kv4_chunk(B, Hkv, L);
    const long long S = (L + Lc - 1) / Lc;
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
    const int Lc = kv4_chunk(B, Hkv, L);
    const int S = (L + Lc - 1) / Lc;
    const size_t smem = (size_t)G * Lc * sizeof(float);
    auto k1 = kv4_attn_chunk_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k1<<<dim3((unsigned)(B * Hkv), (unsigned)S), kThreads, smem, stream>>>(q, K4, V4, lam, s_k, Hkv, L, Lc, part);
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

}  // namespace qoq
