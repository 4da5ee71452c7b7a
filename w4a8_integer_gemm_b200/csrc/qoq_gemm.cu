// qoq_gemm.cu -- the W4A8 GEMM for sm_100a: packed UINT4 weights expanded
// to INT8 in registers, tcgen05 kind::i8 MMA into TMEM INT32 accumulators,
// FP16 per-token x per-channel scaling in the epilogue.
//
// Sources (by page title):
//   "QServe Guide: W4A8KV4 Quantization for LLM Serving", The Architecture,
//       subsection 2: INT8 x INT8 tensor-core products, INT32 accumulation,
//       output scales applied once after the products; Deep Dive,
//       subsection 1, output rescaling equation.
//   "QServe: Low Bit Width Does Not Guarantee High Throughput", section 4:
//       in-register INT4 -> INT8 (multiply by the integer group scale, then
//       subtract the precomputed zero compensation).
//
// Design (B200-first; the pages' A100/L40S register-fed mma.sync design is
// prior art only):
//   * Swap-AB: the 128 output channels of a weight panel are the MMA's M
//     (A operand), the tokens are its N (B operand, BN = 16..256).  Decode
//     shapes (M <= 64) therefore waste no tensor-core rows on padding tokens.
//     Beyond 64 tokens the tile narrows while tiles would be few and
//     widely shared (gemm_block_n).
//   * Persistent grid, one CTA per SM, stream-K schedule: the sequence of
//     (output tile, KST-wide K block) units is cut into equal contiguous
//     ranges, one per CTA, so every SM streams the same number of weight
//     bytes.  When the tiles alone fill 70-100% of the SMs each CTA takes
//     one whole tile instead and nothing is split.  A tile whose K loop is
//     split across CTAs is finished by its
//     first contributor (the CTA whose range holds the tile's first unit:
//     for it the tile is the last one it works on).  Every later
//     contributor works on the tile first, publishes its INT32 partial
//     (exact in any order) and counts it: every lane adds 1 with release
//     semantics after its own stores, so the count covers every lane's
//     bytes.  The finisher's lanes each wait (acquire, bounded) for the
//     full count, add the partials to their accumulators and run the
//     epilogue.  No contributor waits for anything while it still has work,
//     so the waits cannot form a cycle.
//   * Warpgroups (384 or 512 threads):
//       warp 0      weight producer: per stage one bulk copy of the stage's
//                   packed chunks with their group tables; also TMEM.
//       warp 1      MMA issuer (one thread): one barrier wait, KST/32
//                   tcgen05.mma (K = 32) and one tcgen05.commit per stage.
//       warp 2      X8 producer: tiled TMA loads of the activation tiles,
//                   completing on this CTA's own x8full barrier (CTA 1 of
//                   a pair: on CTA 0's x8peer, which it arms itself).  It
//                   and the epilogue alone wait for the preceding kernel
//                   (programmatic dependent launch), so weights stream in
//                   and are dequantized while that kernel still runs.
//       dequant     one or two groups of four warps (two for tiles up to 64
//                   tokens, taking alternate stages): thread r owns output
//                   channel r of the panel, reads its packed bytes with
//                   128-bit shared loads, expands them to INT8 in registers
//                   and stores them as the MMA's A operand -- into TMEM
//                   with tcgen05.st (default), or into shared memory in the
//                   128-byte-swizzled K-major layout.
//       epilogue    one or two groups of four warps (two for 256-token
//                   tiles, one per 128 tokens): tcgen05.ld of the INT32
//                   accumulators, FP32 scaling, FP16 stores; split tiles as
//                   above.  In the one-launch layer call they first
//                   quantize the token rows.
//   * Rings: a weight ring (packed chunks and tables of a K block, freed
//     as soon as the dequant warps hold them in registers; with two dequant
//     groups each slot belongs to one group); an X8/A ring
//     (slot s holds the X8 tiles of a K block in shared memory and its
//     dequantized weights in A slot s; the MMA waits for the dequant warps'
//     barrier and for the X8 copies' own barrier, and one commit frees
//     both); and one or two TMEM accumulators, so the MMAs of the next tile
//     need not wait for the epilogue of the last one.  Every copy completes
//     on a barrier that only its issuer's arrival and its own bytes
//     complete, so an aborted CTA can wait for exactly its own copies.
//   * CTA pairs (256-token tiles): a cluster of two CTAs computes a
//     256-channel tile with one M = 256 MMA per K step (cta_group::2);
//     each CTA dequantizes its own 128-channel panel into its TMEM and
//     loads half of the X8 tile, CTA 0 issues the MMAs and multicasts the
//     commits, and the other CTA's dequant warps and X8 copies arrive on
//     CTA 0's barriers.
//   * Every wait is bounded (per wait, global timer); on expiry the CTA
//     stops, waits for its own in-flight copies (on their own barriers) and
//     MMAs, frees TMEM, and raises the device error flag that
//     qoq_device_error() reports.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "qoq_internal.h"
#include "qoq_epilogue.cuh"
#include "qoq_layout.cuh"
#include "qoq_ptx.cuh"
#include "qoq_quant.cuh"

namespace qoq {

__device__ int g_dev_error;  // non-zero after a bounded wait ran out

struct GemmArgs {
    const uint8_t *Wp;
    const uint8_t *s_g;
    const uint8_t *zs;
    const uint16_t *s_x;
    const uint16_t *s_c;
    uint16_t *Y;
    int32_t *acc_dbg;
    int32_t *ws_cnt;   // [kMaxCtas][4] arrival counters, at the start of the workspace
    int32_t *ws_part;  // [cta][BN/16][4][128][4] INT32 partial tile, after the counters
    // The one-launch layer call (X non-null): the kernel first quantizes the FP16 rows
    // of X into X8 / s_x itself, then reads them as in the plain GEMM.
    const uint16_t *X;
    int8_t *X8w;       // = the X8 the tensor map reads
    uint16_t *s_xw;    // = s_x
    int32_t *ws_ready; // token rows quantized and stored (one-launch layer call)
    int32_t *ws_done;  // CTAs finished; the last one resets both counters
    // Output-side fusion (kEpiPlain, kEpiResidual, kEpiSiluMul): with
    // kEpiResidual Y = fp16(y + R) for the layer output y; with kEpiSiluMul
    // the packed panels hold 64 gate then 64 up channels and Y[m][j] =
    // fp16(silu(g) * u) over N/2 columns.  ldy is Y's row stride.
    int epi;
    const uint16_t *R;
    int ldy;
    int M, N, K, G;
    int m_tiles;
    int ks;            // K / KST units per tile
    int ngroups;       // K / G
    int total;         // tiles * ks units
    unsigned long long timeout_ns;  // longest any one wait may last
};

// Weight stages issued by the setup thread before the CTA-wide barrier.
constexpr int kPrologueStages = 2;

// Warpgroups: producers and MMA issuer (warps 0-3), kDq dequant groups of
// four warps that take the stages in turn, and the epilogue (the last four
// warps).  Token tiles up to 64 wide use two dequant groups (512 threads,
// 128 registers each): there the dequantization, not the MMA, bounds a
// stage, and one group's barrier waits and TMEM stores overlap the other's
// arithmetic.  Wider tiles keep one group (384 threads, 168 registers) for
// their larger epilogue.
// The W8A8 yardstick (W8) has no dequantization: its INT8 weights go
// straight from HBM into the MMA's A slots.
// Half-SM CTAs (HALF) keep one group, for registers.
__host__ __device__ constexpr int dequant_groups(int BN, bool W8 = false, bool HALF = false)
{
    return W8 ? 0 : (BN <= 64 && !HALF) ? 2 : 1;
}
// 256-token tiles drain their accumulator with two epilogue warpgroups (one
// per 128 tokens): with one accumulator in TMEM the MMAs of the next tile
// wait for the epilogue, so its length is lost tensor time.
__host__ __device__ constexpr int epilogue_groups(int BN) { return BN == 256 ? 2 : 1; }
__host__ __device__ constexpr int gemm_threads(int BN, bool W8 = false, bool HALF = false)
{
    return 128 * (1 + dequant_groups(BN, W8, HALF) + epilogue_groups(BN));
}

__host__ __device__ constexpr uint32_t pow2_cols(uint32_t c)
{
    return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512;
}

// PAIR: a 2-CTA cluster computes a 256-channel x BN-token tile with one
// M = 256 MMA per K step (tcgen05 cta_group::2): each CTA dequantizes its
// own 128-channel panel into its TMEM and holds half of the X8 tile.
// HALF: a CTA that takes at most half of an SM (registers, shared memory,
// tensor memory), so that the next GEMM's CTA can be resident beside it and
// stream and dequantize its weights while this one finishes (token tiles up
// to 64, K blocks of 128).
// W8: the W8A8 yardstick: INT8 weights [N][K] loaded by 2-D tiled TMA into
// shared-memory A slots (one per X8 slot, SW == SX), no weight ring and no
// dequant warps.
template <int BN, int KST, int SW, int SX, bool A_TMEM, bool PAIR = false, bool HALF = false, bool W8 = false>
struct GemmCfg {
    static constexpr int kChunks = KST / kBlockK;        // packed 8 KB chunks per K block
    static constexpr int kXRows = PAIR ? BN / 2 : BN;    // token rows of X8 this CTA holds
    static constexpr int kXTile = kXRows * 128;          // one [rows][128 B] swizzled X8 tile
    static constexpr int kXSlot = kChunks * kXTile;      // X8 tiles of one K block
    static constexpr int kATile = 128 * 128;             // one [128][128 B] swizzled A tile
    static constexpr int kABytes = A_TMEM ? 0 : kChunks * kATile;
    // one W slot: the K block's packed chunks, each followed by its group
    // tables when G = 128 (the layout of the packed buffer itself)
    static constexpr int kWSlot = W8 ? 0 : kChunks * (kChunkBytes + kChunkTabBytes);
    // shared memory: [X8 ring][A ring (A in shared memory only)][W ring][barriers]
    static constexpr int kAOff = SX * kXSlot;
    static constexpr int kWOff = kAOff + SX * kABytes;
    static constexpr int kStgOff = kWOff + SW * kWSlot;  // per epilogue warp: 16 tokens x 32 channels FP16
    static constexpr int kBarOff = kStgOff + 4 * 1024 * epilogue_groups(BN);
    static constexpr uint32_t kACols = KST / 4;          // TMEM columns of one A slot
    // two accumulators (the MMAs of the next tile run while the epilogue
    // drains the last one) wherever TMEM has room for them
    static constexpr int kAccBufs = (2 * BN + (A_TMEM ? SX * (int)kACols : 0) <= 512) ? 2 : 1;
    static constexpr int kNumBars = 2 * SW + 4 * SX + 2 * kAccBufs + 2;
    static constexpr int kUsed = kBarOff + kNumBars * 8 + 16;  // + TMEM base, abort flag, peer count
    // full CTAs: at least ~120 KB so that exactly one CTA (and one TMEM
    // allocation) lives on each SM; +1024 for manual alignment of the
    // dynamic base
    static constexpr int kSmemBytes = (HALF || kUsed > 120 * 1024 ? kUsed : 120 * 1024) + 1024;
    static constexpr uint32_t kACol0 = kAccBufs * BN;    // first TMEM column of the A ring
    static constexpr uint32_t kTmemCols = pow2_cols(kACol0 + (A_TMEM ? SX * kACols : 0));
    static constexpr int kSx = (BN + 31) / 32;           // s_x registers per lane
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(KST == 128 || KST == 256, "K block");
    static_assert(BN + (A_TMEM ? SX * kACols : 0) <= 512, "TMEM columns");
    static_assert(kUsed <= 227 * 1024, "shared memory");
    static_assert(SW <= 32 && SX <= 32, "ring bookkeeping masks");
    // The dequant groups take the K blocks in turn, and a group waits on a
    // weight slot by phase parity.  With a ring depth that the groups do not
    // divide, the slot's previous fill belongs to the other group and may
    // still be in flight; its pending phase then reads as this fill's
    // completed one (unless SW >= SX + 2, when the group's own previous A-slot
    // wait already proves that fill consumed).  The kernel keeps the simpler
    // sufficient rule: each weight slot belongs to one group.
    static_assert(W8 || SW % dequant_groups(BN, W8, HALF) == 0, "each weight slot belongs to one dequant group");
    static_assert(!W8 || (!A_TMEM && !PAIR && !HALF && SW == SX), "W8A8: A slots in shared memory, one per X8 slot");
    static_assert(kXSlot % 1024 == 0 && kAOff % 1024 == 0 && kWOff % 1024 == 0, "swizzle atoms");
    // two half CTAs per SM: 228 KB of shared memory (1 KB reserved per CTA)
    // and 512 TMEM columns between them
    static_assert(!HALF || (kSmemBytes <= 113 * 1024 && kTmemCols <= 256 && !PAIR && A_TMEM), "half CTA");
};

// The CTA whose stream-K range contains unit i (ranges: [c*T/P, (c+1)*T/P)).
__device__ __forceinline__ int cta_of(int i, int P, int T)
{
    return (int)((((long long)i + 1) * P - 1) / T);
}

__device__ __forceinline__ int range_begin(int c, int P, int T)
{
    return (int)((long long)c * T / P);
}

// Waits without the shared abort check; used only to drain in-flight work
// on the way out of an aborted CTA.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns)
{
    const uint64_t end = global_timer_ns() + budget_ns;
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() > end) break;
    }
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wait (acquire, bounded) until *p >= want; false on timeout or abort, and
// a timeout raises the CTA's abort flag.
__device__ __forceinline__ bool wait_count_gpu(const int *p, int want, volatile int *abort, uint64_t budget_ns)
{
    if (ld_acquire_gpu(p) >= want) return true;
    const uint64_t start = global_timer_ns();
    while (ld_acquire_gpu(p) < want) {
        if (*abort) return false;
        if (global_timer_ns() - start > budget_ns) {
            *abort = 1;
            return false;
        }
        __nanosleep(100);
    }
    return true;
}

__device__ __forceinline__ void red_release_gpu_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// FP16 outputs (and optionally the INT32 accumulators; with kEpiI32 only
// those) of the 16
// consecutive tokens m0.. of chunk `cc` for this lane's channel n0 + lane.
// The token scales come from the lanes' registers: lane l of sx holds
// s_x[m0 - 16*(cc&1) + l].  The warp stages its 16 x 32 block in its own
// 1 KB of shared memory ([token][32 channels], 64 bytes per token) and then
// writes Y with 16-byte stores: in store j, lane l writes token 8*j + l/4,
// channels 8*(l%4) .. 8*(l%4)+7.
//
// Output-side fusion happens on the staged FP16 values, so the layer's own
// output is rounded exactly as without it:
//   residual: each stored value becomes fp16((float)y + (float)R[m][n]);
//   SiLU-gated pair: the four epilogue warps of the group (quarters 0-1 hold
//     gate channels, 2-3 the up channels of the same outputs) meet at a
//     named barrier; quarters 0-1 read the up values from the staging block
//     two warps on and store fp16(silu(g) * u), silu in FP32 with IEEE
//     division; a second barrier frees the staging blocks for the next chunk.
// (The rounding of each step is in qoq_epilogue.cuh.)
__device__ __forceinline__ void store_outputs(const GemmArgs &a, uint8_t *stg, int m0, int cc, int n0, int lane,
                                              float sc, float sx, const int32_t *acc, int quarter, int bar_id)
{
    if (a.epi == kEpiI32) {
        // INT32 partial sums only (the K-split layer scales them after its
        // all-reduce)
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (m0 + q < a.M) a.acc_dbg[(size_t)(m0 + q) * a.N + n0 + lane] = acc[q];
        return;
    }
    __syncwarp();  // the previous chunk's reads of the staging block are done
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const float sxq = __shfl_sync(0xffffffffu, sx, (cc & 1) * 16 + q);
        *reinterpret_cast<uint16_t *>(stg + q * 64 + lane * 2) = scale_to_half(acc[q], sxq, sc);
    }
    __syncwarp();
    if (a.epi == kEpiSiluMul) {
        named_barrier(bar_id, 128);  // the group's four warps have staged their chunk
        if (quarter < 2) {
            // output column of this warp's first gate channel: 64 per panel
            const int o0 = (n0 / 128) * 64 + quarter * 32;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int q = 8 * j + (lane >> 2);
                const int m = m0 + q;
                const uint4 g = *reinterpret_cast<const uint4 *>(stg + q * 64 + (lane & 3) * 16);
                const uint4 u = *reinterpret_cast<const uint4 *>(stg + 2048 + q * 64 + (lane & 3) * 16);
                const uint4 v = make_uint4(silu_mul_half2(g.x, u.x), silu_mul_half2(g.y, u.y),
                                           silu_mul_half2(g.z, u.z), silu_mul_half2(g.w, u.w));
                if (m < a.M) *reinterpret_cast<uint4 *>(a.Y + (size_t)m * a.ldy + o0 + (lane & 3) * 8) = v;
            }
        }
        named_barrier(bar_id, 128);  // the up values have been read
    } else {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int q = 8 * j + (lane >> 2);
            const int m = m0 + q;
            uint4 v = *reinterpret_cast<const uint4 *>(stg + q * 64 + (lane & 3) * 16);
            if (m < a.M) {
                const size_t o = (size_t)m * a.ldy + n0 + (lane & 3) * 8;
                if (a.epi == kEpiResidual) {
                    // a plain load: R may be Y itself (this thread reads o before it writes o)
                    const uint4 r = *reinterpret_cast<const uint4 *>(a.R + o);
                    v = make_uint4(add_half2(v.x, r.x), add_half2(v.y, r.y), add_half2(v.z, r.z), add_half2(v.w, r.w));
                }
                *reinterpret_cast<uint4 *>(a.Y + o) = v;
            }
        }
    }
    if (a.acc_dbg) {
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (m0 + q < a.M) a.acc_dbg[(size_t)(m0 + q) * a.N + n0 + lane] = acc[q];
    }
}

// The accumulator columns [c0, c0 + W) of this thread's TMEM lane, W = 16,
// 32 or 64, in one load.
template <int W>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t *v)
{
    if constexpr (W == 64) {
        tmem_ld64(taddr, v);
    } else if constexpr (W == 32) {
        tmem_ld32(taddr, v);
    } else {
        uint32_t (&r)[16] = *reinterpret_cast<uint32_t(*)[16]>(v);
        tmem_ld16(taddr, r);
    }
}

template <int BN, int KST, int SW, int SX, bool A_TMEM, bool PAIR, bool HALF, bool W8>
__global__ void __launch_bounds__(gemm_threads(BN, W8, HALF), HALF ? 2 : 1)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const GemmArgs a)
{
    using C = GemmCfg<BN, KST, SW, SX, A_TMEM, PAIR, HALF, W8>;
    static_assert(!PAIR || (A_TMEM && BN == 256), "pairs: 256-token tiles, A in TMEM");
    constexpr int kCh = C::kChunks;
    constexpr int kDq = dequant_groups(BN, W8, HALF);
    constexpr int kEpiWarp0 = 4 + 4 * kDq;  // first epilogue warp
    constexpr int kEpi = epilogue_groups(BN);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar0 = sbase + C::kBarOff;
    // W ring (packed weights + group tables of one K block):
    //   wfull (bulk copy landed), wempty (the dequant warps have read it)
    // X8/A ring (X8 tiles in shared memory, dequantized weights in A slot):
    //   afull (the 4 dequant warps of the stage -- of each CTA of a pair --
    //   have written the A slot),
    //   x8full (this CTA's X8 tiles have landed: the X8 producer's arrival
    //   plus its own copies' bytes, and nothing else, so the producer can
    //   always wait for its own copies),
    //   x8peer (pairs, in CTA 0): CTA 1's X8 half has landed -- CTA 1's
    //   producer's remote arrival (with the half's bytes expected) plus its
    //   copies' bytes, and nothing else,
    //   xaempty (the MMAs reading the slot have completed: both the X8
    //   slot and the A slot are free)
    auto wfull_bar = [&](int s) { return bar0 + 8u * s; };
    auto wempty_bar = [&](int s) { return bar0 + 8u * (SW + s); };
    auto afull_bar = [&](int s) { return bar0 + 8u * (2 * SW + s); };
    auto xaempty_bar = [&](int s) { return bar0 + 8u * (2 * SW + SX + s); };
    // accumulator b: accfull (its tile's MMAs are done), accempty (the
    // epilogue has read it)
    auto accfull_bar = [&](int b) { return bar0 + 8u * (2 * SW + 2 * SX + b); };
    auto accempty_bar = [&](int b) { return bar0 + 8u * (2 * SW + 2 * SX + C::kAccBufs + b); };
    const uint32_t mmadone_bar = bar0 + 8u * (2 * SW + 2 * SX + 2 * C::kAccBufs);
    auto x8full_bar = [&](int s) { return mmadone_bar + 16u + 8u * s; };
    auto x8peer_bar = [&](int s) { return mmadone_bar + 16u + 8u * (SX + s); };
    // one-launch layer call: every token row of X8 and s_x is in memory (the X8
    // producer, the one thread of the CTA that polls the grid-wide count,
    // passes it on to the epilogue warps)
    const uint32_t xready_bar = mmadone_bar + 8u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kBarOff + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // (pairs, CTA 0) the number of X8 stages CTA 1 issued, written by CTA 1
    uint32_t *peer_count = tmem_slot + 2;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Scheduling state, computed first: its reads of the kernel parameters
    // start filling the constant cache while the prologue below runs.
    // Stream-K schedules CTAs, or CTA pairs (PAIR: both CTAs of a cluster
    // take the same range; `rank` picks the panel and the X8 half).
    const int cta = blockIdx.x;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const int P = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
    const int sched = PAIR ? (cta >> 1) : cta;  // index among the scheduled units
    const int T = a.total;
    const int i_begin = range_begin(sched, P, T);
    const int i_end = range_begin(sched + 1, P, T);
    const int ks = a.ks;
    // the weight panel of tile t held by this CTA
    auto panel_of = [&](int t) { return PAIR ? 2 * (t / a.m_tiles) + (int)rank : t / a.m_tiles; };
    // the CTA of scheduled unit c that holds this CTA's panel
    auto cta_index = [&](int c) { return PAIR ? 2 * c + (int)rank : c; };
    // the MMA's barriers live in CTA 0 of a pair
    auto leader = [&](uint32_t bar) { return PAIR ? mapa_shared(bar, 0) : bar; };

    // ring slots a producer has filled, and the phase parity of each slot's
    // latest fill (drained on the way out of an aborted CTA)
    uint32_t issued = 0, issued_par = 0;
    // The weight copy of unit u (tile u / ks, K block u % ks) into W slot s:
    // the kCh chunks of the K block are contiguous in the packed buffer,
    // with their group tables when G = 128, so one bulk copy brings them.
    const bool per_group = (a.G == kBlockK);
    const int cstride = chunk_stride(a.G);
    auto issue_weights = [&](int u, int s, uint32_t ph) {
        const int t = u / ks;
        const int kb = u - t * ks;
        const int n_tile = panel_of(t);
        if constexpr (W8) {
            // W8A8: the K block's [128 channels][KST] INT8 tile, straight
            // into A slot s (128-byte swizzled K-major, as the MMA reads it)
            mbar_arrive_expect_tx(wfull_bar(s), (uint32_t)C::kABytes);
#pragma unroll
            for (int c = 0; c < kCh; ++c)
                tma_load_2d(sbase + C::kAOff + s * C::kABytes + c * C::kATile, &tmap_w, (kb * kCh + c) * kBlockK,
                            n_tile * kPanelRows, wfull_bar(s));
        } else {
            const uint32_t st = sbase + C::kWOff + s * C::kWSlot;
            const uint32_t bytes = (uint32_t)(kCh * cstride);
            mbar_arrive_expect_tx(wfull_bar(s), bytes);
            bulk_load(st, a.Wp + chunk_offset(n_tile, kb * kCh, a.K, a.G), bytes, wfull_bar(s));
        }
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
    };
    // the first stages go out before anything else (no slot is taken yet);
    // only a few, since the whole CTA waits for this thread at the barrier
    const int n_pro = min(min(SW, kPrologueStages), i_end - i_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(wfull_bar(s), 1);
            mbar_init(wempty_bar(s), 4);     // 4 dequant warps
        }
        for (int s = 0; s < SX; ++s) {
            // 4 dequant warps (of each CTA of a pair; unused in W8A8)
            mbar_init(afull_bar(s), PAIR ? 8 : 4);
            mbar_init(xaempty_bar(s), 1);    // MMA commit
            mbar_init(x8full_bar(s), 1);     // this CTA's X8 producer, plus its bytes
            mbar_init(x8peer_bar(s), 1);     // (pairs) CTA 1's X8 producer
        }
        for (int b = 0; b < C::kAccBufs; ++b) {
            mbar_init(accfull_bar(b), 1);
            mbar_init(accempty_bar(b), 4 * kEpi * (PAIR ? 2 : 1));   // the epilogue warps (of each CTA)
        }
        mbar_init(mmadone_bar, 1);
        mbar_init(xready_bar, 1);
        *abort_flag = 0;
        *peer_count = 0;
        fence_mbar_init();
        // weights stream from here on, while the rest of the CTA sets up
        for (int j = 0; j < n_pro; ++j) {
            issue_weights(i_begin + j, j, 0u);
        }
    }
    if (threadIdx.x == 64) prefetch_tmap(&tmap_x);
    if constexpr (W8) {
        if (threadIdx.x == 32) prefetch_tmap(&tmap_w);
    }
    // The next kernel in the stream may launch now; whatever it reads from
    // this GEMM it must read after its own griddepcontrol.wait.
    grid_launch_dependents();
    if (warp == 0) {
        __syncwarp();
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    // a pair: both CTAs' barriers are initialized before either arrives remotely
    if constexpr (PAIR) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t budget = a.timeout_ns;
    // waits on the X8/A ring and the accumulators (in a pair, the phases
    // may be completed by the other CTA's arrivals or the MMA's multicast
    // commits; the tcgen05 fences around the waits order the tensor-memory
    // accesses, as with one CTA)
    auto wait_x = [&](uint32_t bar, uint32_t parity) { return wait_bounded(bar, parity, abort_flag, budget); };

    if (warp == 0) {
        // ---------------------------------------------- weight producer --
        // (the first n_pro units were issued before the CTA-wide barrier)
        if (lane == 0) {
            int s = n_pro == SW ? 0 : n_pro;
            uint32_t ph = (n_pro == SW) ? 1u : 0u;
            for (int u = i_begin + n_pro; u < i_end; ++u) {
                // a weight slot is free once the dequant warps have read it
                // (W8A8: once the MMAs reading the A slot have completed)
                if (!wait_bounded(W8 ? xaempty_bar(s) : wempty_bar(s), ph ^ 1u, abort_flag, budget)) break;
                issue_weights(u, s, ph);
                if (++s == SW) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------- X8 producer --
        if (lane == 0) {
            grid_dependency_wait();  // X8 comes from the preceding kernel
            bool ok = true;
            if (a.X) {
                // one-launch layer call: X8 is written by this grid's epilogue warps
                ok = wait_count_gpu(a.ws_ready, a.M, abort_flag, budget);
                fence_proxy_async_global();
                if (ok) mbar_arrive(xready_bar);
            }
            int s = 0;
            uint32_t ph = 0;
            uint32_t n_peer = 0;  // (CTA 1 of a pair) stages issued
            for (int i = i_begin; i < i_end && ok;) {
                const int t = i / ks;
                const int ks1 = min(ks, i_end - t * ks);
                const int m_tile = t % a.m_tiles;
                for (int kb = i - t * ks; kb < ks1; ++kb) {
                    if (!wait_x(xaempty_bar(s), ph ^ 1u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = sbase + s * C::kXSlot;
                    if (rank == 0) {
                        // this CTA's token rows of the tile (a pair: its
                        // half), completing on its own x8full
                        mbar_arrive_expect_tx(x8full_bar(s), C::kXSlot);
#pragma unroll
                        for (int c = 0; c < kCh; ++c)
                            tma_load_2d(st + c * C::kXTile, &tmap_x, (kb * kCh + c) * kBlockK, m_tile * BN,
                                        x8full_bar(s));
                    } else {
                        // CTA 1 of a pair: its half completes on CTA 0's
                        // x8peer, which only this arrival and these bytes
                        // complete
                        mbar_arrive_expect_tx_cluster(leader(x8peer_bar(s)), C::kXSlot);
                        ++n_peer;
#pragma unroll
                        for (int c = 0; c < kCh; ++c)
                            tma_load_2d_pair(st + c * C::kXTile, &tmap_x, (kb * kCh + c) * kBlockK,
                                             m_tile * BN + C::kXRows, leader(x8peer_bar(s)));
                    }
                    issued |= 1u << s;
                    issued_par = (issued_par & ~(1u << s)) | (ph << s);
                    if (++s == SX) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                i = t * ks + ks1;
            }
            // CTA 1 of a pair tells CTA 0 how many stages it issued (read
            // after the cluster barrier at the end, when no more are issued)
            if constexpr (PAIR) {
                if (rank == 1) st_shared_cluster_u32(mapa_shared(smem_addr(peer_count), 0), n_peer);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer --
        if (lane == 0 && (!PAIR || rank == 0)) {  // a pair's MMAs are issued by CTA 0
            const uint32_t idesc = PAIR ? idesc_i8_m256(BN) : idesc_i8_m128(BN);
            int s = 0;
            uint32_t ph = 0;
            int ab = 0;          // accumulator of the current tile
            uint32_t accph = 0;  // its phase parity
            bool ok = true;
            for (int i = i_begin; i < i_end && ok;) {
                const int t = i / ks;
                const int ks0 = i - t * ks;
                const int ks1 = min(ks, i_end - t * ks);
                if (!wait_x(accempty_bar(ab), accph ^ 1u)) break;
                tc_fence_after();
                const uint32_t dacc = tmem_base + (uint32_t)(ab * BN);
                for (int kb = ks0; kb < ks1; ++kb) {
                    // the stage is ready: its A slot written (W8A8: its weight
                    // tile landed) and its X8 tiles landed (a pair: both halves)
                    if (!wait_x(W8 ? wfull_bar(s) : afull_bar(s), ph) || !wait_x(x8full_bar(s), ph)) {
                        ok = false;
                        break;
                    }
                    if constexpr (PAIR) {
                        if (!wait_x(x8peer_bar(s), ph)) {  // CTA 1's half
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint32_t st = sbase + s * C::kXSlot;
#pragma unroll
                    for (int j = 0; j < 4 * kCh; ++j) {
                        const uint32_t acc = (kb > ks0 || j > 0) ? 1u : 0u;
                        const uint64_t bdesc = smem_desc_sw128(st + (j >> 2) * C::kXTile) + 2 * (j & 3);
                        if constexpr (PAIR) {
                            mma_i8_ts_pair(dacc, tmem_base + C::kACol0 + s * C::kACols + j * 8, bdesc, idesc, acc);
                        } else if constexpr (A_TMEM) {
                            mma_i8_ts(dacc, tmem_base + C::kACol0 + s * C::kACols + j * 8, bdesc, idesc, acc);
                        } else {
                            const uint64_t adesc =
                                smem_desc_sw128(sbase + C::kAOff + s * C::kABytes + (j >> 2) * C::kATile) + 2 * (j & 3);
                            mma_i8_ss(dacc, adesc, bdesc, idesc, acc);
                        }
                    }
                    if constexpr (PAIR) {
                        mma_commit_pair(xaempty_bar(s), 0x3);
                    } else {
                        mma_commit(xaempty_bar(s));
                    }
                    if (++s == SX) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                if constexpr (PAIR) {
                    mma_commit_pair(accfull_bar(ab), 0x3);
                } else {
                    mma_commit(accfull_bar(ab));
                }
                if (++ab == C::kAccBufs) {
                    ab = 0;
                    accph ^= 1u;
                }
                i = t * ks + ks1;
            }
            // all MMAs this thread issued have completed once this arrives
            if constexpr (PAIR) {
                mma_commit_pair(mmadone_bar, 0x1);
            } else {
                mma_commit(mmadone_bar);
            }
            drain_wait(mmadone_bar, 0, 200000000ull);
        }
    } else if (warp >= 4 && warp < kEpiWarp0) {
      if constexpr (!W8) {
        // ------------------------------------------------------ dequant --
        // With two groups of four warps, group 0 takes the CTA's even
        // stages and group 1 the odd ones.
        const int grp = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // output channel within the panel
        int sw = 0, sx = 0;
        uint32_t pw = 0, px = 0;
        // per-channel tables (G = K) come from global memory, one byte each
        // per tile; the next tile's are fetched while this one runs
        uint32_t pc_sg = 0, pc_zs = 0, nx_sg = 0, nx_zs = 0;
        int t_cur = -1, t_nx = -1;
        auto load_tab = [&](int t, uint32_t &sgv, uint32_t &zsv) {
            const size_t o = (size_t)panel_of(t) * kPanelRows + r;
            sgv = __ldg(a.s_g + o);
            zsv = __ldg(a.zs + o);
        };
        if (!per_group && i_begin < i_end) {
            t_nx = i_begin / ks;
            load_tab(t_nx, nx_sg, nx_zs);
        }
        for (int u = i_begin; u < i_end; ++u) {
            if ((u - i_begin) % kDq == grp) {
                if (!per_group) {
                    const int t = u / ks;
                    if (t != t_cur) {
                        if (t == t_nx) {
                            pc_sg = nx_sg;
                            pc_zs = nx_zs;
                        } else {
                            load_tab(t, pc_sg, pc_zs);
                        }
                        t_cur = t;
                        t_nx = ((t + 1) * ks < i_end) ? t + 1 : -1;
                        if (t_nx >= 0) load_tab(t_nx, nx_sg, nx_zs);
                    }
                }
                if (!wait_bounded(wfull_bar(sw), pw, abort_flag, budget)) break;
                const uint8_t *wsl = smem + C::kWOff + sw * C::kWSlot;
                uint4 v[kCh][4];
                uint32_t sg[kCh], zsv[kCh];
#pragma unroll
                for (int c = 0; c < kCh; ++c) {
                    const uint8_t *chunk = wsl + c * cstride;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        v[c][j] = *reinterpret_cast<const uint4 *>(chunk + j * kSlabBytes + r * 16);
                    if (per_group) {
                        sg[c] = chunk[kChunkBytes + r];
                        zsv[c] = chunk[kChunkBytes + kPanelRows + r];
                    } else {
                        sg[c] = pc_sg;
                        zsv[c] = pc_zs;
                    }
                }
                // The next bulk copy into this slot writes through the async
                // proxy: order these generic-proxy reads before it, then
                // release the slot.
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(wempty_bar(sw));  // the weight slot may be refilled now
                // A slot sx is free once the MMAs of its previous use have
                // completed; the X8 tiles need not have landed (the MMA
                // issuer waits for those on afull)
                if (!wait_x(xaempty_bar(sx), px ^ 1u)) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < kCh; ++c) {
                    const uint32_t sgc = sg[c];
                    const uint32_t bias = zero_comp_bias(zsv[c]);
                    uint32_t w8[32];
#pragma unroll
                    for (int j = 0; j < 4; ++j) dequant_slab(v[c][j], sgc, bias, &w8[8 * j]);
                    if constexpr (A_TMEM) {
                        tmem_st32(tmem_base + ((uint32_t)(quarter * 32) << 16) + C::kACol0 + sx * C::kACols + c * 32,
                                  w8);
                    } else {
                        uint8_t *arow = smem + C::kAOff + sx * C::kABytes + c * C::kATile + r * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<uint4 *>(arow + ((q ^ (r & 7)) << 4)) =
                                make_uint4(w8[4 * q], w8[4 * q + 1], w8[4 * q + 2], w8[4 * q + 3]);
                    }
                }
                if constexpr (A_TMEM) {
                    tmem_wait_st();
                    tc_fence_before();
                } else {
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) {
                        mbar_arrive_cluster(leader(afull_bar(sx)));
                    } else {
                        mbar_arrive(afull_bar(sx));
                    }
                }
            }
            if (++sw == SW) {
                sw = 0;
                pw ^= 1u;
            }
            if (++sx == SX) {
                sx = 0;
                px ^= 1u;
            }
        }
      }
    } else if (warp >= kEpiWarp0) {
        // ----------------------------------------------------- epilogue --
        const int quarter = warp & 3;
        const int eg = (warp - kEpiWarp0) >> 2;  // epilogue group: which 16-token chunks it drains
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16);
        uint8_t *stg = smem + C::kStgOff + (eg * 4 + quarter) * 1024;  // this warp's output staging block
        int ab = 0;          // accumulator of the current tile
        uint32_t accph = 0;  // its phase parity
        grid_dependency_wait();  // s_x (or X) comes from the preceding kernel
        if (a.X && eg == 0) {
            // Fused call: the four epilogue warps of each CTA quantize token
            // rows cta, cta + P, ... together (128 threads per row, the
            // loads of a row in flight at once), then every lane waits until
            // all rows are done: any token's X8 tiles and s_x may be needed.
            const int et = threadIdx.x - kEpiWarp0 * 32;           // 0..127
            float *rowmax = reinterpret_cast<float *>(smem + C::kStgOff);  // [4], in warp 0's staging block
            const int nvec = a.K / 8;
            constexpr int kCache = 4;  // 16-byte vectors per thread held across the two passes (K <= 4096)
            for (int row = cta; row < a.M; row += (int)gridDim.x) {  // (epilogue group 0)
                const uint4 *src = reinterpret_cast<const uint4 *>(a.X + (size_t)row * a.K);
                uint4 cache[kCache];
                float amax = 0.0f;
#pragma unroll
                for (int c = 0; c < kCache; ++c) {
                    const int v = et + c * 128;
                    cache[c] = v < nvec ? __ldcg(src + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int c = 0; c < kCache; ++c) amax = fmaxf(amax, absmax8(cache[c]));
                for (int v0 = et + kCache * 128; v0 < nvec; v0 += 4 * 128) {
                    uint4 t[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) t[c] = (v0 + c * 128 < nvec) ? __ldcg(src + v0 + c * 128) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < 4; ++c) amax = fmaxf(amax, absmax8(t[c]));
                }
                amax = warp_max(amax);
                if (lane == 0) rowmax[warp - kEpiWarp0] = amax;
                named_barrier(1, 128);
                amax = fmaxf(fmaxf(rowmax[0], rowmax[1]), fmaxf(rowmax[2], rowmax[3]));
                named_barrier(1, 128);  // rowmax is free for the next row
                const uint16_t sxh = token_scale_bits(amax);
                const float sxf = half_bits_to_float(sxh);
                uint2 *dst = reinterpret_cast<uint2 *>(a.X8w + (size_t)row * a.K);
#pragma unroll
                for (int c = 0; c < kCache; ++c) {
                    const int v = et + c * 128;
                    if (v < nvec) dst[v] = quant8(cache[c], sxf);
                }
                for (int v0 = et + kCache * 128; v0 < nvec; v0 += 4 * 128) {
                    uint4 t[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) t[c] = (v0 + c * 128 < nvec) ? __ldcg(src + v0 + c * 128) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (v0 + c * 128 < nvec) dst[v0 + c * 128] = quant8(t[c], sxf);
                }
                if (et == 0) a.s_xw[row] = sxh;
                // the X8 tiles are read back by TMA (the async proxy); after
                // the barrier one release covers the row's stores by all 128
                // threads (one count per row keeps the polled line quiet)
                fence_proxy_async_global();
                named_barrier(1, 128);
                if (et == 0) red_release_gpu_add(a.ws_ready, 1);
            }
        }
        if (a.X) {
            // every row is done once the X8 producer has seen the count; on
            // a timeout the flag stops every role
            wait_x(xready_bar, 0u);
        }
        for (int i = i_begin; i < i_end;) {
            const int t = i / ks;
            const int ks0 = i - t * ks;
            const int ks1 = min(ks, i_end - t * ks);
            const int m_tile = t % a.m_tiles;
            const int n_tile = panel_of(t);
            const int n = n_tile * kPanelRows + r;
            const int m0 = m_tile * BN;
            const int nchunks = (min(BN, a.M - m0) + 15) >> 4;  // 16-token chunks that exist
            // this epilogue group's chunks
            const int ch_lo = eg * (BN / 16 / kEpi);
            const int ch_hi = min(nchunks, ch_lo + BN / 16 / kEpi);
            const bool partial = !(ks0 == 0 && ks1 == ks);
            // token scales of this tile, one per lane per 32 tokens
            float sx_reg[C::kSx];
#pragma unroll
            for (int q = 0; q < C::kSx; ++q) {
                const int m = m0 + q * 32 + lane;
                sx_reg[q] = (a.epi != kEpiI32 && q * 32 + lane < BN && m < a.M) ? half_bits_to_float(__ldcg(a.s_x + m))
                                                                                   : 0.0f;
            }
            const float sc = a.epi != kEpiI32 ? half_bits_to_float(__ldg(a.s_c + n)) : 0.0f;
            // (scheduled units: CTAs, or CTA pairs; cta_index maps one to
            // the CTA that holds this CTA's panel)
            const int c_lo = partial ? cta_of(t * ks, P, T) : sched;
            const bool finisher = partial && c_lo == sched;   // this CTA completes a split tile
            const int c_hi = finisher ? cta_of(t * ks + ks - 1, P, T) : sched;
            // A finisher's split tile is the last tile of its range, and the
            // other contributors published their parts at the start of
            // theirs: wait for the count and sum their partials now, while
            // this CTA's own MMAs for the tile are still running.
            bool ready = true;
            constexpr bool kPresum = (BN <= 64) && !HALF;  // (registers: 64 per thread in a half CTA)
            // accumulator columns per TMEM load (16 where the pre-summed
            // partials of a 64-wide tile already hold 64 registers); 64 for
            // the 256-token tiles, so that each epilogue warp has its last
            // columns in registers (and the accumulator back with the MMA)
            // after one group of four chunks instead of three groups of two
            constexpr int kGrp = HALF ? 16 : BN < 64 ? BN : (kPresum ? 16 : 64);
            int32_t pre[kPresum ? BN : 1];
            if (finisher) {
                // Every lane of every later contributor counts its own
                // stores (32 per contributor and quarter); every lane here
                // acquires the count itself before it reads the partials.
                int *counter = a.ws_cnt + (cta * kEpi + eg) * 4 + quarter;
                const int want = 32 * (c_hi - sched);
                if (ld_acquire_gpu(counter) < want) {
                    const uint64_t start = global_timer_ns();
                    while (ld_acquire_gpu(counter) < want) {
                        if (*abort_flag || global_timer_ns() - start > budget) {
                            *abort_flag = 1;
                            ready = false;
                            break;
                        }
                    }
                }
                ready = __all_sync(0xffffffffu, ready);
                __syncwarp();  // every lane has seen the full count
                if (lane == 0 && ready) *counter = 0;  // ready for the next call
                if constexpr (kPresum) {
#pragma unroll
                    for (int q = 0; q < BN; ++q) pre[q] = 0;
                    if (ready) {
#pragma unroll 1
                        for (int c2 = sched + 1; c2 <= c_hi; ++c2) {
                            const int4 *src =
                                reinterpret_cast<const int4 *>(a.ws_part + (size_t)cta_index(c2) * BN * kPanelRows);
                            int4 ld[BN / 4];
#pragma unroll
                            for (int cc = 0; cc < BN / 16; ++cc)
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    ld[cc * 4 + j] = (cc < nchunks) ? __ldcg(src + (size_t)(cc * 4 + j) * kPanelRows + r)
                                                                    : make_int4(0, 0, 0, 0);
#pragma unroll
                            for (int j = 0; j < BN / 4; ++j) {
                                pre[4 * j] += ld[j].x;
                                pre[4 * j + 1] += ld[j].y;
                                pre[4 * j + 2] += ld[j].z;
                                pre[4 * j + 3] += ld[j].w;
                            }
                        }
                    }
                }
            }
            if (!wait_x(accfull_bar(ab), accph)) break;
            tc_fence_after();
            const uint32_t tacc = trow + (uint32_t)(ab * BN);
            // the accumulator goes back to the MMA as soon as its last
            // columns are in registers
            bool released = false;
            auto release_acc = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) {
                        mbar_arrive_cluster(leader(accempty_bar(ab)));
                    } else {
                        mbar_arrive(accempty_bar(ab));
                    }
                }
                released = true;
            };
            if (partial && !finisher) {
                // a later contributor: publish the partial, count it, done
                int4 *my_part = reinterpret_cast<int4 *>(a.ws_part + (size_t)cta * BN * kPanelRows);
#pragma unroll 1
                for (int g0 = ch_lo; g0 < ch_hi; g0 += kGrp / 16) {
                    uint32_t v[kGrp];
                    tmem_load_cols<kGrp>(tacc + g0 * 16, v);
                    if (g0 + kGrp / 16 >= ch_hi) release_acc();
#pragma unroll
                    for (int u = 0; u < kGrp / 16; ++u) {
                        if (g0 + u < ch_hi) {
                            int4 *dst = my_part + (size_t)(g0 + u) * 4 * kPanelRows + r;
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                dst[j * kPanelRows] = make_int4((int)v[16 * u + 4 * j], (int)v[16 * u + 4 * j + 1],
                                                   (int)v[16 * u + 4 * j + 2], (int)v[16 * u + 4 * j + 3]);
                        }
                    }
                }
                if (!released) release_acc();
                // each lane's release covers its own partial stores
                red_release_gpu_add(a.ws_cnt + (cta_index(c_lo) * kEpi + eg) * 4 + quarter, 1);
            } else {
                // a whole tile, or a split tile this CTA finishes
                if (ready) {
#pragma unroll 1
                    for (int g0 = ch_lo; g0 < ch_hi; g0 += kGrp / 16) {
                    uint32_t vg[kGrp];
                    tmem_load_cols<kGrp>(tacc + g0 * 16, vg);
                    if (g0 + kGrp / 16 >= ch_hi) release_acc();
                    if constexpr (!kPresum) {
                        if (finisher) {
                            // the later contributors' partials of this group
                            // of chunks, all loads of a contributor in flight
#pragma unroll 1
                            for (int c2 = sched + 1; c2 <= c_hi; ++c2) {
                                const int4 *src = reinterpret_cast<const int4 *>(
                                    a.ws_part + (size_t)cta_index(c2) * BN * kPanelRows);
                                int4 ld[kGrp / 4];
#pragma unroll
                                for (int u = 0; u < kGrp / 16; ++u)
#pragma unroll
                                    for (int j = 0; j < 4; ++j)
                                        ld[u * 4 + j] = (g0 + u < ch_hi)
                                                            ? __ldcg(src + (size_t)((g0 + u) * 4 + j) * kPanelRows + r)
                                                            : make_int4(0, 0, 0, 0);
#pragma unroll
                                for (int j = 0; j < kGrp / 4; ++j) {
                                    vg[4 * j] += (uint32_t)ld[j].x;
                                    vg[4 * j + 1] += (uint32_t)ld[j].y;
                                    vg[4 * j + 2] += (uint32_t)ld[j].z;
                                    vg[4 * j + 3] += (uint32_t)ld[j].w;
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kGrp / 16; ++u) {
                        const int cc = g0 + u;
                        if (cc >= ch_hi) break;
                        int32_t acc[16];
#pragma unroll
                        for (int q = 0; q < 16; ++q) acc[q] = (int32_t)vg[16 * u + q];
                        if constexpr (kPresum) {
                            if (finisher) {
#pragma unroll
                                for (int q = 0; q < 16; ++q) {
                                    // pre[] is indexed by a runtime chunk: select with unrolled compares
                                    int32_t add = 0;
#pragma unroll
                                    for (int c3 = 0; c3 < BN / 16; ++c3)
                                        if (c3 == cc) add = pre[c3 * 16 + q];
                                    acc[q] += add;
                                }
                            }
                        }
                        float sxr = sx_reg[0];
#pragma unroll
                        for (int q = 1; q < C::kSx; ++q)
                            if ((cc >> 1) == q) sxr = sx_reg[q];
                        store_outputs(a, stg, m0 + cc * 16, cc, n - lane, lane, sc, sxr, acc, quarter, 2 + eg);
                    }
                    }
                }
                if (!released) release_acc();
            }
            if (++ab == C::kAccBufs) {
                ab = 0;
                accph ^= 1u;
            }
            i = t * ks + ks1;
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    // An aborted CTA first lets its producers' own copies land: each waits on
    // barriers whose phase only its own arrival and its own copies' bytes
    // complete, so an issued copy cannot be missed (the bound is a last
    // resort that a landing copy never reaches).
    if (*abort_flag) {
        if (threadIdx.x == 0) {
            atomicExch(&g_dev_error, 1);
            for (int q = 0; q < SW; ++q)
                if (issued & (1u << q)) drain_wait(wfull_bar(q), (issued_par >> q) & 1u, 200000000ull);
        } else if (threadIdx.x == 64 && rank == 0) {
            for (int q = 0; q < SX; ++q)
                if (issued & (1u << q)) drain_wait(x8full_bar(q), (issued_par >> q) & 1u, 200000000ull);
        }
    }
    if constexpr (PAIR) {
        // CTA 0's MMAs write both CTAs' TMEM and the CTAs arrive on each
        // other's barriers: neither leaves before both are done.  After this
        // barrier neither CTA issues anything.
        cluster_sync_all();
        // CTA 1's X8 copies complete on CTA 0's x8peer, each phase armed by
        // CTA 1 itself: the latest phase of every slot CTA 1 used completes
        // exactly when its copy has landed.  If either CTA stopped early,
        // CTA 0 waits for those (CTA 1 stated their number before the
        // barrier) and CTA 1 waits at a second barrier until then; both read
        // the same two flags, so both take the same branch.
        const bool any_abort =
            *abort_flag || ld_shared_cluster_u32(mapa_shared(smem_addr((void *)abort_flag), rank ^ 1u)) != 0;
        if (any_abort) {
            if (rank == 0 && threadIdx.x == 64) {
                const uint32_t n1 = *reinterpret_cast<volatile uint32_t *>(peer_count);
                for (uint32_t q = 0; q < (uint32_t)SX && q < n1; ++q) {
                    // stage j = the last one CTA 1 issued into slot q
                    const uint32_t j = q + (n1 - 1 - q) / SX * SX;
                    drain_wait(x8peer_bar((int)q), (j / SX) & 1u, 200000000ull);
                }
            }
            cluster_sync_all();
        }
    }
    tc_fence_after();
    if (a.X && threadIdx.x == 0) {
        // every CTA is past its waits on ws_ready: the last one to get here
        // leaves both counters at zero for the next call
        if (atomicAdd(a.ws_done, 1) == (int)gridDim.x - 1) {
            *a.ws_ready = 0;
            *a.ws_done = 0;
        }
    }
    if (warp == 0) {
        __syncwarp();
        if constexpr (PAIR) {
            tmem_dealloc_pair(tmem_base, C::kTmemCols);
        } else {
            tmem_dealloc(tmem_base, C::kTmemCols);
        }
    }
}

// Self-test of the failure path: one thread waits, bounded, on an mbarrier
// phase that nothing completes, exactly as the GEMM's roles wait; when the
// budget runs out it raises the device error flag and returns.
__global__ void stuck_wait_kernel(unsigned long long budget_ns)
{
    __shared__ __align__(8) unsigned long long bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!wait_bounded(smem_addr(&bar), 0u, &abort_flag, budget_ns)) atomicExch(&g_dev_error, 1);
    }
}

// ----------------------------------------------------------------- host --

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

template <int BN, int KST, int SW, int SX, bool A_TMEM, bool PAIR = false, bool HALF = false, bool W8 = false>
cudaError_t launch_cfg(const CUtensorMap &tmap, const GemmArgs &args, int grid, cudaStream_t stream,
                       const CUtensorMap *tmap_w = nullptr)
{
    using C = GemmCfg<BN, KST, SW, SX, A_TMEM, PAIR, HALF, W8>;
    auto kern = w4a8_gemm_kernel<BN, KST, SW, SX, A_TMEM, PAIR, HALF, W8>;
    // the shared-memory opt-in is per device and per kernel: set it once
    static std::atomic<unsigned long long> opted_in{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(opted_in.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        // all of the unified L1/shared storage as shared memory, so that two
        // half CTAs (or a GEMM CTA and a neighbour) fit on one SM
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        opted_in.fetch_or(bit, std::memory_order_acq_rel);
    }
    // programmatic dependent launch: the GEMM may start (and stream weights)
    // while the kernel before it in the stream -- normally the activation
    // quantizer -- is still running; the kernel waits for it before it
    // touches X8 or s_x.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(gemm_threads(BN, W8, HALF));
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (PAIR) {
        // CTA pairs: clusters of two consecutive CTAs
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 2;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    e = cudaLaunchKernelEx(&cfg, kern, tmap, tmap_w ? *tmap_w : tmap, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Ring depths per token-tile width and K block: the X8/A ring as deep as
// the TMEM next to the accumulator allows (A in TMEM) or shared memory
// allows (A in shared memory); the weight ring fills the rest of the
// ~227 KB of shared memory, since it is what streams from HBM.
template <bool A_TMEM>
cudaError_t dispatch(int BN, int KST, bool pair, bool half, const CUtensorMap &tmap, const GemmArgs &args,
                     int grid, cudaStream_t stream)
{
    if constexpr (A_TMEM) {
        // half CTAs (two per SM, consecutive GEMMs overlap): one dequant
        // group, 256-wide K blocks, rings sized to half the SM
        if (half) {
            switch (BN) {
            case 16: return launch_cfg<16, 256, 4, 3, true, false, true>(tmap, args, grid, stream);
            case 32: return launch_cfg<32, 256, 4, 3, true, false, true>(tmap, args, grid, stream);
            default: return launch_cfg<64, 256, 4, 2, true, false, true>(tmap, args, grid, stream);
            }
        }
        // 256-token tiles on CTA pairs: half the X8 tile per CTA, so a ring
        // of 8 stages fits beside 10 weight stages
        if (pair) {
            if (KST == 256) return launch_cfg<256, 256, 5, 4, true, true>(tmap, args, grid, stream);
            return launch_cfg<256, 128, 10, 8, true, true>(tmap, args, grid, stream);
        }
    }
    if (KST == 256) {
        switch (BN) {
        case 16: return launch_cfg<16, 256, A_TMEM ? 10 : 6, A_TMEM ? 7 : 3, A_TMEM>(tmap, args, grid, stream);
        case 32: return launch_cfg<32, 256, A_TMEM ? 8 : 6, A_TMEM ? 7 : 3, A_TMEM>(tmap, args, grid, stream);
        default: return launch_cfg<64, 256, A_TMEM ? 8 : 4, A_TMEM ? 5 : 2, A_TMEM>(tmap, args, grid, stream);
        }
    }
    switch (BN) {
    case 16: return launch_cfg<16, 128, A_TMEM ? 16 : 12, A_TMEM ? 8 : 4, A_TMEM>(tmap, args, grid, stream);
    case 32: return launch_cfg<32, 128, A_TMEM ? 16 : 12, A_TMEM ? 8 : 4, A_TMEM>(tmap, args, grid, stream);
    case 64: return launch_cfg<64, 128, A_TMEM ? 16 : 12, A_TMEM ? 8 : 4, A_TMEM>(tmap, args, grid, stream);
    case 128: return launch_cfg<128, 128, A_TMEM ? 10 : 10, A_TMEM ? 8 : 3, A_TMEM>(tmap, args, grid, stream);
    default: return launch_cfg<256, 128, A_TMEM ? 6 : 8, A_TMEM ? 5 : 3, A_TMEM>(tmap, args, grid, stream);
    }
}

// The W8A8 yardstick: A and X8 slots in pairs (one stage each), as many as
// shared memory holds.
cudaError_t dispatch_w8(int BN, int KST, const CUtensorMap &tmap, const CUtensorMap &tmap_w, const GemmArgs &args,
                        int grid, cudaStream_t stream)
{
    if (KST == 256) {
        switch (BN) {
        case 16: return launch_cfg<16, 256, 5, 5, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
        case 32: return launch_cfg<32, 256, 5, 5, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
        default: return launch_cfg<64, 256, 4, 4, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
        }
    }
    switch (BN) {
    case 16: return launch_cfg<16, 128, 8, 8, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
    case 32: return launch_cfg<32, 128, 8, 8, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
    case 64: return launch_cfg<64, 128, 8, 8, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
    case 128: return launch_cfg<128, 128, 6, 6, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
    default: return launch_cfg<256, 128, 4, 4, false, false, false, true>(tmap, args, grid, stream, &tmap_w);
    }
}

std::atomic<int> g_cta_pairs{1};
std::atomic<int> g_half_ctas{0};
std::atomic<int> g_gemv{1};
std::atomic<int> g_narrow_tiles{1};

// SMs of the current device, looked up once per device.
int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kMaxCtas;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = kMaxCtas;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// K depth of one pipeline stage: two packed chunks when K allows it and the
// token tile leaves room for enough stages, else one.

}  // namespace

cudaError_t launch_stuck_wait(unsigned long long budget_ns, cudaStream_t stream)
{
    stuck_wait_kernel<<<1, 32, 0, stream>>>(budget_ns);
    return cudaGetLastError();
}

void set_cta_pairs(bool enable)
{
    g_cta_pairs.store(enable ? 1 : 0);
}

void set_narrow_tiles(bool enable)
{
    g_narrow_tiles.store(enable ? 1 : 0);
}

void set_half_ctas(bool enable)
{
    g_half_ctas.store(enable ? 1 : 0);
}

void set_gemv(bool enable)
{
    g_gemv.store(enable ? 1 : 0);
}

// Token tile width.  Up to 128 tokens one tile covers M.  Beyond that,
// 256-token tiles unless they are so few that stream-K shares each among
// many CTAs: every extra CTA on a tile costs a full INT32 partial that the
// finishing CTA reads back, while a narrower tile costs another pass over
// the weights.  Narrower tiles are taken (down to 64 tokens) while a tile
// would be shared by four or more CTAs, or, for a short K (<= 4096, where
// the partials weigh most against the K loop), by two or more.
static int block_n_for(int M, int N, int K, bool narrow)
{
    int bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    if (bn < 128 || !narrow) return bn;
    // 65..128 tokens: two 64-token tiles per panel where they fit the SMs
    // one tile per CTA (no stream-K split, as for decode); measured 11%
    // faster at M = 128, K = N = 8192 (the same rule for 129..256 tokens
    // with 128-token tiles was slower than the CTA pairs)
    if (bn == 128 && 2LL * (N / kPanelRows) <= kMaxCtas) return 64;
    for (;;) {
        const long long tiles = (long long)((M + bn - 1) / bn) * (N / kPanelRows);
        const bool wide_split = tiles * 4 <= kMaxCtas || (K <= 4096 && tiles * 2 <= kMaxCtas);
        if (bn == 64 || !wide_split) return bn;
        bn /= 2;
    }
}

// The most stream-K units a tile width can give: 128-wide K blocks (the
// narrowest stage any configuration uses), so that sizes derived from it
// hold for every stage width, CTA pairs and half CTAs included.
static long long units_for(int M, int N, int K, int BN)
{
    return (long long)((M + BN - 1) / BN) * (N / kPanelRows) * (K / 128);
}

int gemm_block_n(int M, int N, int K)
{
    return block_n_for(M, N, K, g_narrow_tiles.load(std::memory_order_relaxed) != 0);
}

bool gemm_shape_supported(int M, int N, int K)
{
    // the most units either tile choice can give (the narrowest tile)
    return units_for(M, N, K, block_n_for(M, N, K, true)) < (1ll << 31);
}

// Sized for both tile choices (narrowing on or off), so that a workspace
// stays valid across qoq_set_gemm_narrow_tiles: the widest tile's partial
// times the most CTAs either choice launches.
size_t gemm_workspace_bytes(int M, int N, int K)
{
    const int bn_wide = block_n_for(M, N, K, false);
    const int bn_narrow = block_n_for(M, N, K, true);
    const long long units = std::max(units_for(M, N, K, bn_wide), units_for(M, N, K, bn_narrow));
    const long long grid = std::min<long long>(kMaxCtas, units);
    return kCounterBytes + (size_t)grid * bn_wide * kPanelRows * sizeof(int32_t);
}

cudaError_t launch_gemm(const int8_t *X8, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int G, uint16_t *Y,
                        int32_t *acc_dbg, void *workspace, bool a_in_tmem, cudaStream_t stream, int *tmap_status,
                        const uint16_t *X, int epi, const uint16_t *R, int ldx, const int8_t *W8)
{
    *tmap_status = 0;
    // a few tokens: the matrix-vector kernel on the CUDA cores
    if (W8 == nullptr && g_gemv.load(std::memory_order_relaxed) && gemv_applies(M, N, epi, X != nullptr, sm_count()))
        return launch_gemv(X8, ldx, s_x, Wp, s_c, s_g, zs, M, N, K, G, Y, acc_dbg, epi, R, stream);
    const int BN = gemm_block_n(M, N, K);
    // W8A8 yardstick: INT8 weights in shared-memory A slots, single CTAs
    const bool w8 = W8 != nullptr;
    if (w8) a_in_tmem = false;
    // 256-token tiles run on CTA pairs (one M = 256 MMA over two weight
    // panels, each CTA holding half of the X8 tile) when N allows it, with
    // 256-wide K stages where K allows them
    const bool pair = a_in_tmem && g_cta_pairs.load(std::memory_order_relaxed) && BN == 256 && N % 256 == 0;
    // token tiles up to 64 in half CTAs (two per SM) when selected
    const bool half = a_in_tmem && !pair && BN <= 64 && K % 256 == 0 && g_half_ctas.load(std::memory_order_relaxed);
    const int KST = (pair && K % 256 == 0) ? 256 : (BN <= 64 && K % 256 == 0) ? 256 : 128;
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) {
        *tmap_status = -1;
        return cudaErrorNotSupported;
    }
    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    // X8 rows are ldx bytes apart (K, or the full row of a K-split layer's slice)
    const cuuint64_t gstride[1] = {(cuuint64_t)(ldx > 0 ? ldx : K)};
    const cuuint32_t box[2] = {(cuuint32_t)kBlockK, (cuuint32_t)(pair ? BN / 2 : BN)};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(X8), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *tmap_status = (int)r;
        return cudaErrorInvalidValue;
    }
    CUtensorMap tmap_w;
    if (w8) {
        // [N][K] INT8 weights, [128 channels][128 K] boxes, 128-byte swizzle
        const cuuint64_t wdim[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t wstride[1] = {(cuuint64_t)K};
        const cuuint32_t wbox[2] = {(cuuint32_t)kBlockK, (cuuint32_t)kPanelRows};
        r = enc(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(W8), wdim, wstride, wbox, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            *tmap_status = (int)r;
            return cudaErrorInvalidValue;
        }
    }
    const int sms = sm_count();
    // stream-K units: (tile, K block) per CTA, or per CTA pair
    const long long units = pair ? (long long)((M + BN - 1) / BN) * (N / 256) * (K / KST)
                                 : (long long)((M + BN - 1) / BN) * (N / kPanelRows) * (K / KST);
    // Stream-K over the SMs, except when the tiles alone fill at least 70%
    // of them: then one whole tile per CTA (or pair), so that no tile is
    // split and no CTA waits at the end for another's partial sums (the
    // decode projections: 112 tiles on 148 SMs).
    const long long slots = pair ? std::min(kMaxCtas, sms) / 2 : std::min(kMaxCtas, sms);
    const long long tiles = units / (K / KST);
    const long long sched_units = (tiles <= slots && tiles * 10 >= slots * 7) ? tiles : std::min(slots, units);
    const long long grid = pair ? 2 * sched_units : sched_units;

    GemmArgs args;
    args.Wp = Wp;
    args.s_g = s_g;
    args.zs = zs;
    args.s_x = s_x;
    args.s_c = s_c;
    args.Y = Y;
    args.acc_dbg = acc_dbg;
    args.epi = epi;
    args.R = R;
    args.ldy = (epi == kEpiSiluMul) ? N / 2 : N;
    args.ws_cnt = reinterpret_cast<int32_t *>(workspace);
    args.X = X;
    args.X8w = const_cast<int8_t *>(X8);
    args.s_xw = const_cast<uint16_t *>(s_x);
    args.ws_ready = args.ws_cnt + kFusedReadyWord;
    args.ws_done = args.ws_cnt + kFusedDoneWord;
    args.ws_part = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(workspace) + kCounterBytes);
    args.M = M;
    args.N = N;
    args.K = K;
    args.G = G;
    args.m_tiles = (M + BN - 1) / BN;
    args.ks = K / KST;
    args.ngroups = K / G;
    args.total = (int)units;
    args.timeout_ns = 2000000000ull;  // 2 s for one wait: far beyond any legitimate one
    if (w8) return dispatch_w8(BN, KST, tmap, tmap_w, args, (int)grid, stream);
    return a_in_tmem ? dispatch<true>(BN, KST, pair, half, tmap, args, (int)grid, stream)
                     : dispatch<false>(BN, KST, false, false, tmap, args, (int)grid, stream);
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, int *value)
{
    *value = 0;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int));
    }
    *value = v;
    return e;
}

}  // namespace qoq
