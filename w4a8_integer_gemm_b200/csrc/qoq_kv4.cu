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
// the KV head, the chunk's codes brought into shared memory by bulk copies,
// both products on the tensor cores as warp-level MMAs with the codes
// expanded to FP16 in registers (exact) and the FP32 factors split into
// two FP16 parts, a second small kernel combining the chunks.  The path is
// HBM-bound: the expansion costs about 1.5 instructions per code.
#include <cuda_fp16.h>

#include <atomic>
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

// Two 4-bit codes as an FP16 pair, without conversion instructions.  A
// nibble pair in bits 0-3 and 16-19 of x goes into the mantissa of 1024
// (exactly 1024 + n), and 1032 is subtracted: the codes n - 8, exact.  A
// pair in bits 4-7 and 20-23 lands one hex digit higher (1024 + 16n), and
// 1152 is subtracted: 16 (n - 8), exact, so two of every four nibble pairs
// need no shift; the factor 16 is taken out of the other operand (the
// query) or of the result (the weighted sums).  One logic op and one FP16
// pair subtraction per two codes.
__device__ __forceinline__ uint32_t codes_h2(uint32_t x)
{
    const uint32_t h = (x & 0x000F000Fu) | 0x64006400u;
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64086408u));
    return r;
}

__device__ __forceinline__ uint32_t codes16_h2(uint32_t x)
{
    const uint32_t h = (x & 0x00F000F0u) | 0x64006400u;
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64806480u));
    return r;
}

// D (16 x 8, FP32) += A (16 x 16, FP16, row) * B (16 x 8, FP16, col): the
// warp-level tensor-core product.  Fragment of lane (g = lane / 4, c = lane
// % 4): A rows g and g + 8 at columns 2c, 2c + 1 and 2c + 8, 2c + 9; B
// column g at rows 2c, 2c + 1 and 2c + 8, 2c + 9; D rows g and g + 8 at
// columns 2c, 2c + 1.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kThreads = 256;    // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 512;      // tokens per CTA: 32 KB of K codes and 32 KB of V codes
constexpr int kWarpTok = kChunk / kWarps;   // 64 tokens per warp: four 16-token MMA steps
constexpr int kSub = 128;        // tokens per bulk copy (two warps' share)
constexpr int kNumSub = kChunk / kSub;
constexpr int kPStride = kChunk + 8;        // FP16 elements per row of P (rows 4 banks apart)

__device__ int g_kv4_error;      // non-zero after a bounded wait of this file's kernels ran out

// ------------------------------------------------------------ attention --
// A persistent CTA per resident slot.  The work items are the (sequence, KV
// head, chunk) triples in that order; CTA k of P takes items [k*I/P,
// (k+1)*I/P), so consecutive items mostly share a KV head.  Per item, over
// tokens [s*kChunk, min(L, ...)) of the chunk:
//   - the K and V codes are contiguous in the cache and arrive by bulk
//     copies of 128 tokens, each on its own barrier; the next item's K codes
//     are requested as soon as this item's scores are computed, its V codes
//     once this item's weighted sums are out of shared memory;
//   - both products run on the tensor cores (mma.sync m16n8k16, FP16
//     operands, FP32 sums), eight columns per MMA: up to four query heads,
//     each as a high and a low FP16 part, so that the operands carry
//     FP32-level precision (hi + lo) while the codes are exact in FP16:
//       scores:  S[token][col] = sum_c K[token][c] * q'[col][c]  (A = codes, rows = tokens)
//       values:  O^T[c][col]   = sum_t V[t][c] * p[col][t]       (A = codes^T, rows = channels)
//   - the softmax numerators of the chunk, split the same way, go through
//     shared memory (the score fragment holds tokens by row, the value
//     product needs them by column);
//   - each warp takes 64 tokens in both passes; the warps' weighted sums are
//     added in shared memory (over the V codes, read by then), and the
//     chunk's (max, sum, weighted sums) per query head go to the workspace
//     for the combine.
// The folded query q' of a KV head is built once per change of head: warp h
// folds query head h, scales it by the power of two that brings its largest
// element into [2^13, 2^14) (no FP16 overflow, full precision in the
// parts; the score undoes it exactly) and writes the high and low parts
// into shared memory in the order of the MMA's B fragments.
template <int G>
__global__ void __launch_bounds__(kThreads, G > 4 ? 2 : 3) kv4_attn_kernel(
    const uint16_t *__restrict__ q, const uint8_t *__restrict__ K4, const uint8_t *__restrict__ V4,
    const uint16_t *__restrict__ lam, const uint16_t *__restrict__ s_k, int Hkv, int L, int S, int items,
    float *__restrict__ part)
{
    constexpr int HT = (G + 3) / 4;             // column tiles of 8 (4 heads x hi/lo)
    extern __shared__ __align__(128) uint8_t dyn[];
    uint8_t *ks = dyn;                                   // [kChunk][64] K codes
    uint8_t *vs = dyn + kChunk * kRowBytes;              // [kChunk][64] V codes
    __half *ps = reinterpret_cast<__half *>(dyn + 2 * kChunk * kRowBytes);   // [HT][8][kPStride]
    uint2 *qfrag = reinterpret_cast<uint2 *>(ps + HT * 8 * kPStride);        // [HT][8 steps][32 lanes]
    uint64_t *bars = reinterpret_cast<uint64_t *>(qfrag + HT * 8 * 32);      // K parts, V parts
    float *osum = reinterpret_cast<float *>(vs);         // [kWarps][G][kD], over the V codes once read
    __shared__ float red[kWarps][G], red2[kWarps][G];
    __shared__ float escl[4 * HT];
    __shared__ int abort_flag;
    const int P = gridDim.x;
    const int it_begin = (int)((long long)blockIdx.x * items / P);
    const int it_end = (int)((long long)(blockIdx.x + 1) * items / P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t bar0 = smem_addr(bars);
    auto kbar = [&](int j) { return bar0 + 8u * j; };
    auto vbar = [&](int j) { return bar0 + 8u * (kNumSub + j); };
    // (thread 0) one item's K or V codes, in parts of kSub tokens
    auto issue = [&](int it, bool val) {
        const int bh_ = it / S, s_ = it % S;
        const int l0_ = s_ * kChunk, n_ = min(L - l0_, kChunk);
        const uint8_t *src = (val ? V4 : K4) + ((size_t)bh_ * L + l0_) * kRowBytes;
        uint8_t *dst = val ? vs : ks;
        for (int j = 0; j < kNumSub; ++j) {
            const int rows = max(0, min(n_ - j * kSub, kSub));
            const uint32_t bar = val ? vbar(j) : kbar(j);
            if (rows > 0) {
                mbar_arrive_expect_tx(bar, (uint32_t)rows * kRowBytes);
                bulk_load(smem_addr(dst + j * kSub * kRowBytes), src + (size_t)j * kSub * kRowBytes,
                          (uint32_t)rows * kRowBytes, bar);
            } else {
                mbar_arrive(bar);
            }
        }
    };
    int k_issued = 0, v_issued = 0;              // (thread 0) items whose copies went out
    if (threadIdx.x == 0) {
        for (int j = 0; j < 2 * kNumSub; ++j) mbar_init(bar0 + 8u * j, 1);
        abort_flag = 0;
        fence_mbar_init();
        if (it_begin < it_end) {
            issue(it_begin, false);
            issue(it_begin, true);
            k_issued = v_issued = 1;
        }
    }
    __syncthreads();
    const uint64_t budget = 2000000000ull;
    const float inv_sqrt_d = 0.08838834764831845f;   // 1 / sqrt(128)
    const int T0 = warp * kWarpTok;
    // byte selectors of the value pass (see there): even lanes hold token
    // tA in the first operand, odd lanes in the second
    const uint32_t psel_even[2] = {0x5410u, 0x7632u}, psel_odd[2] = {0x1054u, 0x3276u};
    int cur_bh = -1;
    for (int it = it_begin; it < it_end; ++it) {
        const uint32_t ph = (uint32_t)((it - it_begin) & 1);
        const int bh = it / S, s = it % S;
        const int l0 = s * kChunk, n = min(L - l0, kChunk);
        if (bh != cur_bh) {                      // the same for every thread of the CTA
            cur_bh = bh;
            if (warp < 4 * HT) {
                // query head `warp` (zeros past G): lane l folds channels 4l .. 4l + 3
                float f[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                float m = 0.0f;
                if (warp < G) {
                    const uint2 lw = __ldg(reinterpret_cast<const uint2 *>(lam + (size_t)bh * kD) + lane);
                    const uint2 sw = __ldg(reinterpret_cast<const uint2 *>(s_k + (size_t)bh * kD) + lane);
                    const uint2 qw = __ldg(reinterpret_cast<const uint2 *>(q + ((size_t)bh * G + warp) * kD) + lane);
                    const uint32_t la[2] = {lw.x, lw.y}, sa[2] = {sw.x, sw.y}, qa[2] = {qw.x, qw.y};
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const int sh = 16 * (e4 & 1);
                        const float fold = __fmul_rn(__fmul_rn(half_bits_to_float((uint16_t)(la[e4 >> 1] >> sh)),
                                                               half_bits_to_float((uint16_t)(sa[e4 >> 1] >> sh))),
                                                     inv_sqrt_d);
                        f[e4] = __fmul_rn(half_bits_to_float((uint16_t)(qa[e4 >> 1] >> sh)), fold);
                        m = fmaxf(m, fabsf(f[e4]));
                    }
                }
                m = warp_max(m);
                // m in [2^E, 2^(E+1)) with E its biased exponent field - 127 (a
                // zero or subnormal m takes E = -126); e = E - 13 brings the
                // largest |q'| * 2^-e into [2^13, 2^14), and both powers of
                // two are exact FP32 numbers for e in [-126, 114]
                const int E = max((int)((__float_as_uint(m) >> 23) & 0xFFu), 1) - 127;
                const int e = max(E - 13, -126);
                const float down = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e
                // channel 32c + 8j + i goes to step 2j + h, register r, half hf
                // of lane (column, c), where i = 2h + r + 4hf; the column is
                // the head's slot (high part) or slot + 4 (low part)
                const int t = warp >> 2, slot = warp & 3;
                const int cc = lane >> 3, j = (lane & 7) >> 1, ib = 4 * (lane & 1);
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const int i = ib + e4;
                    const int hf = i >> 2, h = (i & 3) >> 1, r = i & 1;
                    // register 1 meets codes scaled by 16 (codes16_h2): 1/16 here
                    const float x = f[e4] * down * (r ? 0.0625f : 1.0f);
                    const __half hi = __float2half_rn(x);
                    const __half lo = __float2half_rn(x - __half2float(hi));
                    uint16_t *fr = reinterpret_cast<uint16_t *>(qfrag + (t * 8 + 2 * j + h) * 32);
                    fr[(slot * 4 + cc) * 4 + 2 * r + hf] = __half_as_ushort(hi);
                    fr[((slot + 4) * 4 + cc) * 4 + 2 * r + hf] = __half_as_ushort(lo);
                }
                if (lane == 0) escl[warp] = __uint_as_float((uint32_t)(127 + e) << 23);   // 2^e
            }
            __syncthreads();
        }
        // this lane's B fragments (reloaded per item: registers are what
        // bounds the CTAs per SM)
        uint32_t qb[HT][8][2];
        float escale[HT][2];
#pragma unroll
        for (int t = 0; t < HT; ++t) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint2 v = qfrag[(t * 8 + kk) * 32 + lane];
                qb[t][kk][0] = v.x;
                qb[t][kk][1] = v.y;
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) escale[t][i] = escl[4 * t + 2 * (c & 1) + i];
        }
        bool ok = wait_bounded(kbar(T0 / kSub), ph, &abort_flag, budget);
        // pass 1: scores of the warp's 64 tokens (rows g and g + 8 of each
        // 16-token step), all columns; the K codes' word j of lane c's 32
        // channels holds channel 32c + 8j + i in nibble i, and MMA step 2j + h
        // pairs nibbles (2h, 2h + 4) at columns 2c, 2c + 1 and (2h + 1,
        // 2h + 5) at 2c + 8, 2c + 9, the latter scaled by 16 (the order of
        // q' in qb, whose second register carries the factor 1/16)
        float sc[4][HT][4];
#pragma unroll
        for (int st = 0; st < 4; ++st) {
#pragma unroll
            for (int t = 0; t < HT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r) sc[st][t][r] = 0.0f;
            if (!ok) continue;
            const int r0 = T0 + 16 * st + g;
            const uint4 k0 = *reinterpret_cast<const uint4 *>(ks + r0 * kRowBytes + 16 * c);
            const uint4 k1 = *reinterpret_cast<const uint4 *>(ks + (r0 + 8) * kRowBytes + 16 * c);
            const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t x0 = w0[j] >> (8 * h), x1 = w1[j] >> (8 * h);
                    const uint32_t a[4] = {codes_h2(x0), codes_h2(x1), codes16_h2(x0), codes16_h2(x1)};
#pragma unroll
                    for (int t = 0; t < HT; ++t)
                        mma_f16_16816(sc[st][t], a, qb[t][2 * j + h][0], qb[t][2 * j + h][1]);
                }
        }
        // high + low columns (lanes c and c ^ 2), power of two undone; lane c
        // then holds heads 4t + 2(c % 2) + i for rows g and g + 8 of each step
        float lmax[HT][2];
#pragma unroll
        for (int t = 0; t < HT; ++t) lmax[t][0] = lmax[t][1] = -INFINITY;
#pragma unroll
        for (int st = 0; st < 4; ++st)
#pragma unroll
            for (int t = 0; t < HT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int i = r & 1;
                    const int tok = T0 + 16 * st + g + 8 * (r >> 1);
                    const int hq = 4 * t + 2 * (c & 1) + i;
                    const float v = (sc[st][t][r] + __shfl_xor_sync(0xffffffffu, sc[st][t][r], 2)) * escale[t][i];
                    sc[st][t][r] = (tok < n && hq < G) ? v : -INFINITY;
                    lmax[t][i] = fmaxf(lmax[t][i], sc[st][t][r]);
                }
#pragma unroll
        for (int t = 0; t < HT; ++t)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float m = lmax[t][i];
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                const int hq = 4 * t + 2 * (c & 1) + i;
                if (lane < 2 && hq < G) red[warp][hq] = m;
            }
        // the K codes were read through the generic proxy; the next item's
        // bulk copies write them through the async proxy
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0 && it + 1 < it_end && !abort_flag) {
            issue(it + 1, false);
            ++k_issued;
        }
        // the chunk max of each head this lane holds (every lane reads the
        // warps' maxima itself: no second barrier)
        float cmax[HT][2];
#pragma unroll
        for (int t = 0; t < HT; ++t)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int hq = 4 * t + 2 * (c & 1) + i;
                float m = -INFINITY;
                if (hq < G) {
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w][hq]);
                }
                cmax[t][i] = m;
            }
        // the chunk's softmax numerators exp(score - chunk max), their sum,
        // and their high and low FP16 parts at column (c / 2) * 4 + 2(c % 2) + i
        float lsum[HT][2];
#pragma unroll
        for (int t = 0; t < HT; ++t) lsum[t][0] = lsum[t][1] = 0.0f;
#pragma unroll
        for (int st = 0; st < 4; ++st)
#pragma unroll
            for (int t = 0; t < HT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int i = r & 1;
                    const int tok = T0 + 16 * st + g + 8 * (r >> 1);
                    const int hq = 4 * t + 2 * (c & 1) + i;
                    const float p = sc[st][t][r] == -INFINITY ? 0.0f : expf(sc[st][t][r] - cmax[t][i]);
                    lsum[t][i] += p;
                    const __half hi = __float2half_rn(p);
                    ps[(t * 8 + (c >> 1) * 4 + 2 * (c & 1) + i) * kPStride + tok] =
                        c < 2 ? hi : __float2half_rn(p - __half2float(hi));
                }
#pragma unroll
        for (int t = 0; t < HT; ++t)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float v = lsum[t][i];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                const int hq = 4 * t + 2 * (c & 1) + i;
                if (lane < 2 && hq < G) red2[warp][hq] = v;
            }
        // each warp reads back only the numerators of its own 64 tokens
        __syncwarp();
        // pass 2: O^T[channel][column] over the warp's 64 tokens; m-tile mt
        // row g is channel 16g + 2mt (a low nibble), row g + 8 channel
        // 16g + 2mt + 1 (the high nibble of the same byte)
        float o[HT][8][4];
#pragma unroll
        for (int t = 0; t < HT; ++t)
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int r = 0; r < 4; ++r) o[t][mt][r] = 0.0f;
        ok = ok && wait_bounded(vbar(T0 / kSub), ph, &abort_flag, budget);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            if (!ok) break;
            const int tA = T0 + 16 * st + 2 * c;    // tokens tA, tA + 1, tA + 8, tA + 9
            const int odd = c & 1;
            // each load instruction of the warp touches rows of both parities
            // (odd lanes load token tA + 1 first; their byte selectors below
            // take the second operand first, so no register is swapped)
            const uint2 x0 = *reinterpret_cast<const uint2 *>(vs + (tA + odd) * kRowBytes + 8 * g);
            const uint2 x1 = *reinterpret_cast<const uint2 *>(vs + (tA + 1 - odd) * kRowBytes + 8 * g);
            const uint2 y0 = *reinterpret_cast<const uint2 *>(vs + (tA + 8 + odd) * kRowBytes + 8 * g);
            const uint2 y1 = *reinterpret_cast<const uint2 *>(vs + (tA + 9 - odd) * kRowBytes + 8 * g);
            uint32_t pb[HT][2];
#pragma unroll
            for (int t = 0; t < HT; ++t) {
                pb[t][0] = *reinterpret_cast<const uint32_t *>(ps + (t * 8 + g) * kPStride + tA);
                pb[t][1] = *reinterpret_cast<const uint32_t *>(ps + (t * 8 + g) * kPStride + tA + 8);
            }
#pragma unroll
            for (int wi = 0; wi < 2; ++wi) {
                const uint32_t wa = wi ? x0.y : x0.x, wb = wi ? x1.y : x1.x;
                const uint32_t wc = wi ? y0.y : y0.x, wd = wi ? y1.y : y1.x;
#pragma unroll
                for (int bp = 0; bp < 2; ++bp) {
                    // bytes 2bp, 2bp + 1 of token tA (resp. tA + 8) over those
                    // of tA + 1 (tA + 9)
                    const uint32_t sel = odd ? psel_odd[bp] : psel_even[bp];
                    const uint32_t xab = __byte_perm(wa, wb, sel), xcd = __byte_perm(wc, wd, sel);
                    const int mt = 4 * wi + 2 * bp;
                    // rows g + 8 (the high nibbles) come out scaled by 16
                    const uint32_t xab8 = xab >> 8, xcd8 = xcd >> 8;
                    const uint32_t a0[4] = {codes_h2(xab), codes16_h2(xab), codes_h2(xcd), codes16_h2(xcd)};
                    const uint32_t a1[4] = {codes_h2(xab8), codes16_h2(xab8), codes_h2(xcd8), codes16_h2(xcd8)};
#pragma unroll
                    for (int t = 0; t < HT; ++t) {
                        mma_f16_16816(o[t][mt], a0, pb[t][0], pb[t][1]);
                        mma_f16_16816(o[t][mt + 1], a1, pb[t][0], pb[t][1]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < HT; ++t)
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    o[t][mt][r] += __shfl_xor_sync(0xffffffffu, o[t][mt][r], 2);
                    if (r >= 2) o[t][mt][r] *= 0.0625f;   // rows g + 8: codes scaled by 16
                }
        __syncthreads();   // every warp is done with the V codes
        // high + low columns, then the warps' sums in shared memory
#pragma unroll
        for (int t = 0; t < HT; ++t)
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int hq = 4 * t + 2 * c + (r & 1);
                    if (c < 2 && hq < G) osum[(warp * G + hq) * kD + 16 * g + 2 * mt + (r >> 1)] = o[t][mt][r];
                }
        __syncthreads();
        // partial record per query head: [max, sum, kD weighted sums]
        float *rec = part + (size_t)it * G * (kD + 2);
        for (int e = threadIdx.x; e < G * kD; e += kThreads) {
            const int gi = e / kD, ch = e % kD;
            float t = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) t += osum[(w * G + gi) * kD + ch];
            rec[gi * (kD + 2) + 2 + ch] = t;
        }
        if (threadIdx.x < G) {
            float t = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) t += red2[w][threadIdx.x];
            float m = red[0][threadIdx.x];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[w][threadIdx.x]);
            rec[threadIdx.x * (kD + 2)] = m;
            rec[threadIdx.x * (kD + 2) + 1] = t;
        }
        // the V codes' bytes were used through the generic proxy; the next
        // item's bulk copies write them through the async proxy
        fence_proxy_async_smem();
        if (__syncthreads_or(abort_flag != 0)) break;
        if (threadIdx.x == 0 && it + 1 < it_end) {
            issue(it + 1, true);
            ++v_issued;
        }
    }
    if (threadIdx.x == 0 && abort_flag) {
        // a wait ran out: report it, and let every copy issued land before
        // leaving (the last item issued on each barrier completes its phase
        // last)
        atomicExch(&g_kv4_error, 1);
        const uint64_t end = global_timer_ns() + 200000000ull;
        for (int j = 0; j < kNumSub; ++j) {
            if (k_issued > 0)
                while (!mbar_try_wait(kbar(j), (uint32_t)((k_issued - 1) & 1)) && global_timer_ns() < end) {
                }
            if (v_issued > 0)
                while (!mbar_try_wait(vbar(j), (uint32_t)((v_issued - 1) & 1)) && global_timer_ns() < end) {
                }
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
    const float *rec0 = part + (bh * S * G + gi) * (kD + 2);   // chunk s at rec0 + s * G * (kD + 2)
    const size_t step = (size_t)G * (kD + 2);
    float M = -INFINITY;
    for (int s = 0; s < S; s += 8) {
        float m[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) m[u] = s + u < S ? rec0[(s + u) * step] : -INFINITY;
#pragma unroll
        for (int u = 0; u < 8; ++u) M = fmaxf(M, m[u]);
    }
    float den = 0.0f, num = 0.0f;
    for (int s = 0; s < S; s += 8) {
        float mx[8], sm[8], x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bool in = s + u < S;
            mx[u] = in ? rec0[(s + u) * step] : -INFINITY;
            sm[u] = in ? rec0[(s + u) * step + 1] : 0.0f;
            x[u] = in ? rec0[(s + u) * step + 2 + c] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float w = s + u < S ? expf(mx[u] - M) : 0.0f;
            den = fmaf(sm[u], w, den);
            num = fmaf(x[u], w, num);
        }
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

// SMs of the current device, looked up once per device.
static int kv4_sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int G>
static cudaError_t launch_attn_g(const uint16_t *q, const uint8_t *K4, const uint8_t *V4, const uint16_t *lam,
                                 const uint16_t *s_k, const uint16_t *s_v, int B, int Hkv, int L, uint16_t *out,
                                 float *part, cudaStream_t stream)
{
    constexpr int HT = (G + 3) / 4;
    const int S = (L + kChunk - 1) / kChunk;
    const long long items = (long long)B * Hkv * S;
    const size_t smem = 2 * (size_t)kChunk * kRowBytes + (size_t)HT * 8 * kPStride * sizeof(__half) +
                        (size_t)HT * 8 * 32 * sizeof(uint2) + 2 * kNumSub * sizeof(uint64_t);
    auto k1 = kv4_attn_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // all of the unified L1/shared storage as shared memory: three CTAs
    // (two for G = 8) per SM keep their copies in flight together
    e = cudaFuncSetAttribute(k1, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k1, kThreads, smem);
    if (e != cudaSuccess) return e;
    const long long slots = (long long)kv4_sm_count() * (per_sm > 0 ? per_sm : 1);
    const int grid = (int)(items < slots ? items : slots);
    k1<<<grid, kThreads, smem, stream>>>(q, K4, V4, lam, s_k, Hkv, L, S, (int)items, part);
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
