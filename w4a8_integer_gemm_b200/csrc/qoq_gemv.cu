// qoq_gemv.cu -- the W4A8 layer for a handful of tokens (M <= 8) with
// warp-level tensor-core products.
//
// The layer is the same as the GEMM's ("QServe: Low Bit Width Does Not
// Guarantee High Throughput", section 4, progressive quantization; "QServe
// Guide: W4A8KV4 Quantization for LLM Serving", Deep Dive, subsection 1):
// the UINT4 codes expand to INT8 in registers (W8hat = q * s_g - zs), the
// products W8hat * X8 add up in INT32, and the sum is rescaled once per
// output, y = fp16(((float)acc * s_x) * s_c).  Only the kernel differs: with
// M <= 8 tokens the layer is bound by the weight stream from HBM (N*K/2
// bytes against 2*M*N*K operations) and by each launch's fixed costs, so it
// runs without the GEMM's machinery: no tensor memory, no barrier rings, no
// stream-K handoff.  Each CTA reads its channels' weights once with
// coalesced loads, and the next layer's CTAs fit beside this layer's on an
// SM (programmatic dependent launch).
//
// CTA: 16 output channels (one MMA tile) and all of K, or for small N (too
// few channel groups to give every SM three CTAs) a 1/2 or 1/4 share of the
// K blocks, the shares' INT32 sums added through distributed shared memory
// in a cluster; its 8 warps take the 128-wide K blocks in turn.  The
// products are warp-level INT8 MMAs (m16n8k32, INT32 sums) with the tokens
// as the 8-wide N dimension, so up to 8 tokens cost one MMA per 32 K per 16
// channels, whatever M is.  The packed
// layout feeds the A fragment directly.  The MMA's K index is mapped onto
// the block so that lane (g, c) reads whole 16-byte slices: in K step s it
// supplies, for rows g and g + 8, word s of slice c, whose low and high
// nibbles are K values 32c + 4s .. +3 and 32c + 16 + 4s .. +3 (the A
// fragment's two K groups), and X8 supplies the same K values (B).  Each
// lane thus loads two 16-byte slices of weights and two of X8 per block.  The
// weights of a warp's first K block are requested before the wait on the
// preceding kernel (they do not depend on it); every later block one block
// ahead.  The warps' INT32 sums are added in shared memory.
#include <cuda_fp16.h>

#include <cstdint>

#include "qoq_epilogue.cuh"
#include "qoq_internal.h"
#include "qoq_layout.cuh"
#include "qoq_ptx.cuh"
#include "qoq_quant.cuh"

namespace qoq {
namespace {

constexpr int kGvWarps = 8;
constexpr int kGvThreads = 32 * kGvWarps;

struct GemvArgs {
    const int8_t *X8;
    int ldx;              // X8 row stride in bytes
    const uint16_t *s_x;
    const uint8_t *Wp;
    const uint16_t *s_c;
    const uint8_t *s_g;   // per-channel tables (G = K); G = 128 keeps them in the chunks
    const uint8_t *zs;
    uint16_t *Y;
    int32_t *acc_dbg;     // INT32 sums [M][N] (kEpiI32: the only output)
    const uint16_t *R;    // kEpiResidual: Y = fp16(y + R)
    int epi;
    int M, N, K, G;
};

// D (16 x 8, INT32) += A (16 x 32, INT8, row) * B (32 x 8, INT8, col).
// Lane (g = lane / 4, c = lane % 4): A rows g and g + 8 at K 4c..4c+3 (a0,
// a1) and 16+4c..16+4c+3 (a2, a3); B column g at the same K; D rows g and
// g + 8 at columns 2c, 2c + 1.
__device__ __forceinline__ void mma_s8_16832(int32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One K block of this lane's two rows (g and g + 8 of the CTA's 16): the
// rows' 16-byte slice c (32 K values), and with 128-wide groups the rows'
// s_g and zs bytes.
struct Block {
    uint4 w[2];   // [row g, g + 8]
    uint32_t sg[2], zs[2];
};

template <bool PG>
__device__ __forceinline__ void load_block(const GemvArgs &a, int panel, int r0, int g, int c, int b, Block &blk)
{
    const uint8_t *ch = a.Wp + chunk_offset(panel, b, a.K, a.G);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = r0 + 8 * h + g;
        blk.w[h] = __ldg(reinterpret_cast<const uint4 *>(ch + c * kSlabBytes + row * 16));
        if constexpr (PG) {
            blk.sg[h] = __ldg(ch + kChunkBytes + row);
            blk.zs[h] = __ldg(ch + kChunkBytes + kPanelRows + row);
        }
    }
}

// NT: token tiles of 8 (M <= 8 NT; the layer calls use one); PG: 128-wide
// groups (tables in the chunks), else per-channel tables; S: CTAs (a
// cluster) that split the K blocks of one channel group, their INT32 sums
// added through distributed shared memory by the cluster's first CTA.
template <int NT, bool PG, int S>
__global__ void __launch_bounds__(kGvThreads, 4) w4a8_gemv_kernel(GemvArgs a)
{
    __shared__ int32_t red[kGvWarps][16][8 * NT];   // [warp][channel][token]
    __shared__ int32_t part[16][8 * NT];            // the CTA's sums
    // the next kernel in the stream may launch now; it waits for this grid
    // before it reads anything this kernel writes
    grid_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int q = S > 1 ? (int)cluster_ctarank() : 0;   // this CTA's share of the K blocks
    const int n0 = (blockIdx.x / S) * 16;
    const int panel = n0 / kPanelRows, r0 = n0 % kPanelRows;
    const int nb = a.K / kBlockK;
    uint32_t sg[2] = {0, 0}, bias[2] = {0, 0};
    if constexpr (!PG) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = n0 + 8 * h + g;
            sg[h] = __ldg(a.s_g + n);
            bias[h] = zero_comp_bias(__ldg(a.zs + n));
        }
    }
    int32_t acc[NT][4];
#pragma unroll
    for (int u = 0; u < NT; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[u][i] = 0;
    constexpr int kStep = kGvWarps * S;
    // weights two K blocks ahead of the products
    Block cur, nxt;
    int b = q * kGvWarps + warp;
    if (b < nb) load_block<PG>(a, panel, r0, g, c, b, cur);
    if (b + kStep < nb) load_block<PG>(a, panel, r0, g, c, b + kStep, nxt);
    grid_dependency_wait();  // X8 and s_x come from the preceding kernel
    for (; b < nb; b += kStep) {
        Block nx2;
        if (b + 2 * kStep < nb) load_block<PG>(a, panel, r0, g, c, b + 2 * kStep, nx2);
        uint32_t gs[2], bs[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            gs[h] = PG ? cur.sg[h] : sg[h];
            bs[h] = PG ? zero_comp_bias(cur.zs[h]) : bias[h];
        }
        // B: token g + 8u, the 32 K values of slice c (zero past M)
        uint4 xl[NT], xh[NT];
#pragma unroll
        for (int u = 0; u < NT; ++u) {
            const int m = g + 8 * u;
            if (m < a.M) {
                const uint4 *xr = reinterpret_cast<const uint4 *>(a.X8 + (size_t)m * a.ldx + b * kBlockK + c * kSlabK);
                xl[u] = __ldg(xr);
                xh[u] = __ldg(xr + 1);
            } else {
                xl[u] = xh[u] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        const uint32_t w0[4] = {cur.w[0].x, cur.w[0].y, cur.w[0].z, cur.w[0].w};
        const uint32_t w1[4] = {cur.w[1].x, cur.w[1].y, cur.w[1].z, cur.w[1].w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            // MMA K step s: lane c supplies word s of slice c, i.e. K values
            // 32c + 4s .. +3 (low nibbles) and 32c + 16 + 4s .. +3 (high
            // nibbles), and the same K values of X8
            uint32_t af[4];
            dequant_word(w0[s], gs[0], bs[0], af[0], af[2]);   // row g
            dequant_word(w1[s], gs[1], bs[1], af[1], af[3]);   // row g + 8
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                const uint32_t xlo[4] = {xl[u].x, xl[u].y, xl[u].z, xl[u].w};
                const uint32_t xhi[4] = {xh[u].x, xh[u].y, xh[u].z, xh[u].w};
                mma_s8_16832(acc[u], af, xlo[s], xhi[s]);
            }
        }
        cur = nxt;
        nxt = nx2;
    }
    // the warps' sums: lane (g, c) holds rows (channels) g and g + 8,
    // columns (tokens) 8u + 2c and 8u + 2c + 1
#pragma unroll
    for (int u = 0; u < NT; ++u) {
        red[warp][g][8 * u + 2 * c] = acc[u][0];
        red[warp][g][8 * u + 2 * c + 1] = acc[u][1];
        red[warp][g + 8][8 * u + 2 * c] = acc[u][2];
        red[warp][g + 8][8 * u + 2 * c + 1] = acc[u][3];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * a.M; e += kGvThreads) {
        const int m = e >> 4, ch = e & 15;
        int32_t s = 0;
#pragma unroll
        for (int w = 0; w < kGvWarps; ++w) s += red[w][ch][m];
        part[ch][m] = s;
    }
    if constexpr (S > 1) cluster_sync_all();   // every CTA's sums are in its shared memory
    else __syncthreads();
    // outputs (the cluster's first CTA): thread i takes channel i % 16 of
    // tokens i / 16, i / 16 + 16, ...
    for (int e = threadIdx.x; e < 16 * a.M && q == 0; e += kGvThreads) {
        const int m = e >> 4, ch = e & 15;
        int32_t s = part[ch][m];
#pragma unroll
        for (int r = 1; r < S; ++r) s += (int32_t)ld_shared_cluster_u32(mapa_shared(smem_addr(&part[ch][m]), r));
        const int n = n0 + ch;
        const size_t o = (size_t)m * a.N + n;
        if (a.acc_dbg) a.acc_dbg[o] = s;
        if (a.epi != kEpiI32) {
            uint16_t y = scale_to_half(s, half_bits_to_float(__ldg(a.s_x + m)), half_bits_to_float(__ldg(a.s_c + n)));
            if (a.epi == kEpiResidual) y = add_half(y, a.R[o]);   // a plain load: R may be Y itself
            a.Y[o] = y;
        }
    }
    // the other CTAs' shared memory stays until the first one has read it
    if constexpr (S > 1) cluster_sync_all();
}

template <int NT, int S>
cudaError_t launch_nts(const GemvArgs &a, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.N / 16 * S));
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (S > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = S;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cudaError_t e = a.G == kBlockK ? cudaLaunchKernelEx(&cfg, w4a8_gemv_kernel<NT, true, S>, a)
                                   : cudaLaunchKernelEx(&cfg, w4a8_gemv_kernel<NT, false, S>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// K split over S CTAs (1, 2 or 4) so that the grid gives every SM at least
// about three CTAs: 16-channel groups alone are too few for small N.
template <int NT>
cudaError_t launch_nt(const GemvArgs &a, cudaStream_t stream)
{
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long groups = a.N / 16;
    int S = 1;
    while (S < 4 && groups * S < 3LL * sms) S *= 2;
    if (S == 1) return launch_nts<NT, 1>(a, stream);
    if (S == 2) return launch_nts<NT, 2>(a, stream);
    return launch_nts<NT, 4>(a, stream);
}

}  // namespace

bool gemv_applies(int M, int N, int epi, bool one_launch, int sms)
{
    return M >= 1 && M <= kGemvMaxM && epi != kEpiSiluMul && !one_launch && (long long)(N / 16) <= 8LL * sms;
}

cudaError_t launch_gemv(const int8_t *X8, int ldx, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int G, uint16_t *Y,
                        int32_t *acc_dbg, int epi, const uint16_t *R, cudaStream_t stream)
{
    GemvArgs a;
    a.X8 = X8;
    a.ldx = ldx > 0 ? ldx : K;
    a.s_x = s_x;
    a.Wp = Wp;
    a.s_c = s_c;
    a.s_g = s_g;
    a.zs = zs;
    a.Y = Y;
    a.acc_dbg = acc_dbg;
    a.R = R;
    a.epi = epi;
    a.M = M;
    a.N = N;
    a.K = K;
    a.G = G;
    return launch_nt<1>(a, stream);
}

}  // namespace qoq
