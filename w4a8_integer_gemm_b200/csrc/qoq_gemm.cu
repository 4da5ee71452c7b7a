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
//     (A operand), the tokens are its N (B operand, 16..256).  Decode shapes
//     (M <= 64) therefore waste no tensor-core rows on padding tokens.
//   * Persistent grid, one CTA per SM, stream-K schedule: the sequence of
//     (output tile, 128-wide K block) units is cut into equal contiguous
//     ranges, one per CTA, so every SM streams the same number of weight
//     bytes.  Tiles whose K loop is split across CTAs meet as INT32 partials
//     in a workspace (exact in any order); the last contributor, found with
//     a counter per split tile and 32-channel quarter, reduces them and runs
//     the epilogue.  A split tile is the last tile of the first CTA that
//     contributes to it, so the counters are indexed by that CTA: a fixed
//     region at the start of the workspace, whatever the shape, which every
//     call leaves at zero.
//   * Warp roles (320 threads):
//       warp 0      TMA producer: per stage one tiled TMA of the X8 tile
//                   (128-byte swizzle), one 8 KB bulk copy of the packed
//                   weight chunk and two 128-byte bulk copies of the group
//                   tables into a shared-memory ring.
//       warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 32 each)
//                   per stage, tcgen05.commit frees ring slots.
//       warps 2-5   dequant: thread r owns output channel r of the panel,
//                   reads its 64 packed bytes with four 128-bit shared loads,
//                   expands them to 128 INT8 weights in registers, and
//                   stores them as the MMA's A operand -- into TMEM with
//                   tcgen05.st (default), or into shared memory in the
//                   128-byte-swizzled K-major layout.
//       warps 6-9   epilogue: tcgen05.ld of the INT32 accumulators, FP32
//                   scaling, FP16 stores (or INT32 partials for split tiles).
//   * Every mbarrier wait is bounded by a global-timer deadline; on expiry
//     the CTA stops, drains its own in-flight copies and MMAs, frees TMEM,
//     and raises the device error flag that qoq_device_error() reports.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "qoq_internal.h"
#include "qoq_layout.cuh"
#include "qoq_ptx.cuh"

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
    int32_t *ws_part;  // [cta][2 slots][BN][128] INT32 partial tiles, after the counters
    int M, N, K, G;
    int m_tiles, ks;        // ks = K / 128 stages per tile
    long long total;        // tiles * ks units
    unsigned long long timeout_ns;  // longest any one wait may last
#ifdef QOQ_TRACE
    unsigned long long *trace;  // [cta][256] global-timer marks (trace builds only)
#endif
};

// Timeline marks for the trace build (compiled out otherwise).
#ifdef QOQ_TRACE
// slot 255 holds the CTA's global-timer entry time; the other marks are SM
// clock cycles since the CTA's entry
#define QOQ_MARK(idx)                                                                              \
    do {                                                                                           \
        if (a.trace) a.trace[(size_t)blockIdx.x * 256 + (idx)] = clock64() - trace_t0;             \
    } while (0)
#else
#define QOQ_MARK(idx) \
    do {              \
    } while (0)
#endif

__host__ __device__ constexpr uint32_t pow2_cols(uint32_t c)
{
    return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512;
}

template <int BN, int STAGES, int ASTAGES, bool A_TMEM>
struct GemmCfg {
    static constexpr int kXBytes = BN * 128;  // X8 tile: BN tokens x 128 k
    static constexpr int kWBytes = kChunkBytes;
    static constexpr int kTabBytes = 256;  // s_g[128] then zs[128]
    static constexpr int kStageBytes = ((kXBytes + kWBytes + kTabBytes + 1023) / 1024) * 1024;
    static constexpr int kABytes = A_TMEM ? 0 : 128 * 128;  // dequantized tile in smem
    static constexpr int kBarOff = STAGES * kStageBytes + ASTAGES * kABytes;
    static constexpr int kNumBars = 3 * STAGES + 2 * ASTAGES + 3;
    static constexpr int kUsed = kBarOff + kNumBars * 8 + 16;
    // at least ~120 KB so that exactly one CTA (and one TMEM allocation)
    // lives on each SM; +1024 for manual alignment of the dynamic base
    static constexpr int kSmemBytes = (kUsed > 120 * 1024 ? kUsed : 120 * 1024) + 1024;
    static constexpr uint32_t kAccCols = BN;
    static constexpr uint32_t kACol0 = BN;  // first TMEM column of the A ring
    static constexpr uint32_t kTmemCols = pow2_cols(BN + (A_TMEM ? ASTAGES * 32 : 0));
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(BN + (A_TMEM ? ASTAGES * 32 : 0) <= 512, "TMEM columns");
    static_assert(kUsed <= 227 * 1024, "shared memory");
};

// The CTA whose stream-K range contains unit i.
__device__ __forceinline__ long long cta_of(long long i, long long P, long long T)
{
    return ((i + 1) * P - 1) / T;
}

__device__ __forceinline__ long long range_begin(long long c, long long P, long long T)
{
    return c * T / P;
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

__device__ __forceinline__ float half_bits_to_float(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t scale_to_half(int32_t acc, float sx, float sc)
{
    const float y = __fmul_rn(__fmul_rn(__int2float_rn(acc), sx), sc);
    return __half_as_ushort(__float2half_rn(y));
}

// FP16 outputs (and optionally the INT32 accumulators) of 16 consecutive
// tokens m0.. for channel n; tokens beyond M are skipped.
__device__ __forceinline__ void store_outputs(const GemmArgs &a, int m0, int n, float sc, const int32_t *acc)
{
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const int m = m0 + q;
        if (m < a.M) {
            const float sx = half_bits_to_float(__ldg(a.s_x + m));
            a.Y[(size_t)m * a.N + n] = scale_to_half(acc[q], sx, sc);
            if (a.acc_dbg) a.acc_dbg[(size_t)m * a.N + n] = acc[q];
        }
    }
}

template <int BN, int STAGES, int ASTAGES, bool A_TMEM>
__global__ void __launch_bounds__(320, 1)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmArgs a)
{
    using C = GemmCfg<BN, STAGES, ASTAGES, A_TMEM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar0 = sbase + C::kBarOff;
    // per ring slot: fullw (weights + tables landed), fullx (X8 tile landed),
    // empty (dequant warps and the MMA are done with the slot)
    auto fullw_bar = [&](int s) { return bar0 + 8u * s; };
    auto fullx_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto empty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
    auto afull_bar = [&](int t) { return bar0 + 8u * (3 * STAGES + t); };
    auto aempty_bar = [&](int t) { return bar0 + 8u * (3 * STAGES + ASTAGES + t); };
    const uint32_t accfull_bar = bar0 + 8u * (3 * STAGES + 2 * ASTAGES);
    const uint32_t accempty_bar = accfull_bar + 8u;
    const uint32_t mmadone_bar = accfull_bar + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kBarOff + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

#ifdef QOQ_TRACE
    const long long trace_t0 = clock64();
    if (threadIdx.x == 0 && a.trace) a.trace[(size_t)blockIdx.x * 256 + 255] = global_timer_ns();
#endif
    if (threadIdx.x == 0) {
        QOQ_MARK(0);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(fullw_bar(s), 1);
            mbar_init(fullx_bar(s), 1);
            mbar_init(empty_bar(s), 1 + 4);  // MMA commit + 4 dequant warps
        }
        for (int t = 0; t < ASTAGES; ++t) {
            mbar_init(afull_bar(t), 4);
            mbar_init(aempty_bar(t), 1);
        }
        mbar_init(accfull_bar, 1);
        mbar_init(accempty_bar, 4);
        mbar_init(mmadone_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_x);
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (threadIdx.x == 0) QOQ_MARK(1);
    int trace_j = 0;  // per-role stage counter for the timeline marks
    (void)trace_j;
    const uint64_t deadline = a.timeout_ns;  // budget of any single wait

    const long long P = gridDim.x;
    const long long T = a.total;
    const long long cta = blockIdx.x;
    const long long i_begin = range_begin(cta, P, T);
    const long long i_end = range_begin(cta + 1, P, T);
    const int ks = a.ks;
    // ring slots the producer has filled, and the phase parity of each
    // slot's latest fill (drained on the way out of an aborted CTA)
    uint32_t issued = 0, issued_par = 0;
    int issued_x_none = 0;  // set when the producer stopped before any X8 load

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            // The X8 tiles come from the kernel that precedes this one in the
            // stream (programmatic dependent launch): the weights of the first
            // STAGES slots stream in before that kernel has finished, the X8
            // loads of those slots are issued once it has.
            int n_issued = 0;
            bool x_ready = false;
            int pend_kb[STAGES], pend_m[STAGES];
            auto load_x = [&](int slot, int kb, int m_tile) {
                mbar_arrive_expect_tx(fullx_bar(slot), C::kXBytes);
                tma_load_2d(sbase + slot * C::kStageBytes, &tmap_x, kb * kBlockK, m_tile * BN, fullx_bar(slot));
            };
            auto release_x = [&]() {
                grid_dependency_wait();
                QOQ_MARK(144);
                x_ready = true;
                for (int j = 0; j < n_issued; ++j) {
                    load_x(j, pend_kb[j], pend_m[j]);
                    if (j < 16) QOQ_MARK(160 + j);
                }
            };
            for (long long i = i_begin; i < i_end && ok;) {
                const long long t = i / ks;
                const int ks0 = (int)(i - t * ks);
                const int ks1 = (int)min((long long)ks, i_end - t * ks);
                const int m_tile = (int)(t % a.m_tiles);
                const int n_tile = (int)(t / a.m_tiles);
                for (int kb = ks0; kb < ks1; ++kb) {
                    if (!x_ready && n_issued == STAGES) release_x();  // every slot waits for X8
                    if (trace_j < 8) QOQ_MARK(216 + trace_j);
                    if (!wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, deadline)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = sbase + s * C::kStageBytes;
                    const int g = (kb * kBlockK) / a.G;
                    if (trace_j < 16) QOQ_MARK(180 + trace_j);
                    mbar_arrive_expect_tx(fullw_bar(s), C::kWBytes + C::kTabBytes);
                    bulk_load(st + C::kXBytes, a.Wp + chunk_offset(n_tile, kb, a.K), C::kWBytes, fullw_bar(s));
                    if (trace_j < 16) QOQ_MARK(200 + trace_j);
                    const size_t toff = (size_t)g * a.N + (size_t)n_tile * kPanelRows;
                    bulk_load(st + C::kXBytes + C::kWBytes, a.s_g + toff, 128, fullw_bar(s));
                    bulk_load(st + C::kXBytes + C::kWBytes + 128, a.zs + toff, 128, fullw_bar(s));
                    if (trace_j < 32) QOQ_MARK(16 + trace_j);
                    ++trace_j;
                    if (x_ready) {
                        load_x(s, kb, m_tile);
                    } else {
                        pend_kb[n_issued] = kb;
                        pend_m[n_issued] = m_tile;
                        ++n_issued;
                    }
                    issued |= 1u << s;
                    issued_par = (issued_par & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                i = t * ks + ks1;
            }
            if (ok && !x_ready) release_x();
            if (!x_ready) issued_x_none = 1;
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t idesc = idesc_i8_m128(BN);
            int s = 0, ta = 0;
            uint32_t ph = 0, aph = 0, accph = 0;
            bool ok = true;
            for (long long i = i_begin; i < i_end && ok;) {
                const long long t = i / ks;
                const int ks0 = (int)(i - t * ks);
                const int ks1 = (int)min((long long)ks, i_end - t * ks);
                if (!wait_bounded(accempty_bar, accph ^ 1u, abort_flag, deadline)) break;
                tc_fence_after();
                for (int kb = ks0; kb < ks1; ++kb) {
                    if (trace_j < 8) QOQ_MARK(224 + trace_j);
                    if (!wait_bounded(fullx_bar(s), ph, abort_flag, deadline)) {
                        ok = false;
                        break;
                    }
                    if (trace_j < 8) QOQ_MARK(232 + trace_j);
                    if (!wait_bounded(afull_bar(ta), aph, abort_flag, deadline)) {
                        ok = false;
                        break;
                    }
                    if (trace_j < 8) QOQ_MARK(240 + trace_j);
                    tc_fence_after();
                    const uint64_t bdesc = smem_desc_sw128(sbase + s * C::kStageBytes);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t acc = (kb > ks0 || j > 0) ? 1u : 0u;
                        if constexpr (A_TMEM) {
                            mma_i8_ts(tmem_base, tmem_base + C::kACol0 + ta * 32 + j * 8, bdesc + 2 * j, idesc, acc);
                        } else {
                            const uint64_t adesc =
                                smem_desc_sw128(sbase + STAGES * C::kStageBytes + ta * C::kABytes);
                            mma_i8_ss(tmem_base, adesc + 2 * j, bdesc + 2 * j, idesc, acc);
                        }
                    }
                    if (trace_j < 8) QOQ_MARK(248 + trace_j);
                    mma_commit(empty_bar(s));
                    mma_commit(aempty_bar(ta));
                    if (trace_j < 32) QOQ_MARK(80 + trace_j);
                    ++trace_j;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (++ta == ASTAGES) {
                        ta = 0;
                        aph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(accfull_bar);
                accph ^= 1u;
                i = t * ks + ks1;
            }
            // all MMAs this thread issued have completed once this arrives
            mma_commit(mmadone_bar);
            drain_wait(mmadone_bar, 0, 200000000ull);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------ dequant --
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // output channel within the panel
        int s = 0, ta = 0;
        uint32_t ph = 0, aph = 0;
        bool ok = true;
        for (long long i = i_begin; i < i_end && ok;) {
            const long long t = i / ks;
            const int ks0 = (int)(i - t * ks);
            const int ks1 = (int)min((long long)ks, i_end - t * ks);
            for (int kb = ks0; kb < ks1; ++kb) {
                if (!wait_bounded(fullw_bar(s), ph, abort_flag, deadline)) {
                    ok = false;
                    break;
                }
                if (warp == 2 && lane == 0 && trace_j < 32) QOQ_MARK(112 + trace_j);
                const uint8_t *st = smem + s * C::kStageBytes;
                const uint8_t *sw = st + C::kXBytes;
                uint4 v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4 *>(sw + j * kSlabBytes + r * 16);
                const uint32_t sg = st[C::kXBytes + C::kWBytes + r];
                const uint32_t zsv = st[C::kXBytes + C::kWBytes + 128 + r];
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(s));
                if (!wait_bounded(aempty_bar(ta), aph ^ 1u, abort_flag, deadline)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t bias = zero_comp_bias(zsv);
                uint32_t w8[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) dequant_slab(v[j], sg, bias, &w8[8 * j]);
                if constexpr (A_TMEM) {
                    tmem_st32(tmem_base + ((uint32_t)(quarter * 32) << 16) + C::kACol0 + ta * 32, w8);
                    tmem_wait_st();
                    tc_fence_before();
                } else {
                    uint8_t *arow = smem + STAGES * C::kStageBytes + ta * C::kABytes + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(arow + ((c ^ (r & 7)) << 4)) =
                            make_uint4(w8[4 * c], w8[4 * c + 1], w8[4 * c + 2], w8[4 * c + 3]);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(afull_bar(ta));
                if (warp == 2 && lane == 0 && trace_j < 32) QOQ_MARK(48 + trace_j);
                ++trace_j;
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
                if (++ta == ASTAGES) {
                    ta = 0;
                    aph ^= 1u;
                }
            }
            i = t * ks + ks1;
        }
    } else {
        // ----------------------------------------------------- epilogue --
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16);
        uint32_t accph = 0;
        const long long first_tile = i_begin / ks;
        grid_dependency_wait();  // s_x comes from the preceding kernel
        for (long long i = i_begin; i < i_end;) {
            const long long t = i / ks;
            const int ks0 = (int)(i - t * ks);
            const int ks1 = (int)min((long long)ks, i_end - t * ks);
            const int m_tile = (int)(t % a.m_tiles);
            const int n_tile = (int)(t / a.m_tiles);
            const int n = n_tile * kPanelRows + r;
            const int m0 = m_tile * BN;
            const int live = min(BN, a.M - m0);      // token columns that exist
            const int nchunks = (live + 15) >> 4;     // 16-column chunks holding them
            const bool partial = !(ks0 == 0 && ks1 == ks);
            if (!wait_bounded(accfull_bar, accph, abort_flag, deadline)) break;
            if (warp == 6 && lane == 0 && trace_j < 4) QOQ_MARK(145 + trace_j);
            tc_fence_after();
            if (!partial) {
                const float sc = half_bits_to_float(a.s_c[n]);
#pragma unroll 1
                for (int cc = 0; cc < nchunks; ++cc) {
                    uint32_t v[16];
                    tmem_ld16(trow + cc * 16, v);
                    store_outputs(a, m0 + cc * 16, n, sc, reinterpret_cast<const int32_t *>(v));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(accempty_bar);
            } else {
                // Partial tile: 16 consecutive columns of one channel are 64
                // contiguous bytes, [chunk][channel][16] per slot.
                const int slot = (t == first_tile) ? 0 : 1;
                int4 *part = reinterpret_cast<int4 *>(a.ws_part + (size_t)(cta * 2 + slot) * BN * kPanelRows);
#pragma unroll 1
                for (int cc = 0; cc < nchunks; ++cc) {
                    uint32_t v[16];
                    tmem_ld16(trow + cc * 16, v);
                    int4 *dst = part + ((size_t)cc * kPanelRows + r) * 4;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_int4((int)v[4 * j], (int)v[4 * j + 1], (int)v[4 * j + 2], (int)v[4 * j + 3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(accempty_bar);
                // publish this partial, then count arrivals for the quarter
                __threadfence();
                __syncwarp();
                const long long c_lo = cta_of(t * ks, P, T);
                const long long c_hi = cta_of(t * ks + ks - 1, P, T);
                int *counter = a.ws_cnt + c_lo * 4 + quarter;
                int last = 0;
                if (lane == 0) {
                    const int old = atomicAdd(counter, 1);
                    last = (old == (int)(c_hi - c_lo));
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
                    const float sc = half_bits_to_float(a.s_c[n]);
                    const int nc = (int)(c_hi - c_lo + 1);
#pragma unroll 1
                    for (int cc = 0; cc < nchunks; ++cc) {
                        int32_t sum[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) sum[j] = 0;
                        // up to 4 contributors per batch: all 16 loads are in
                        // flight before the first add
#pragma unroll 1
                        for (int b = 0; b < nc; b += 4) {
                            int4 ld[4][4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                if (b + u < nc) {
                                    const long long c2 = c_lo + b + u;
                                    const int sl = (t == range_begin(c2, P, T) / ks) ? 0 : 1;
                                    const int4 *src = reinterpret_cast<const int4 *>(
                                                          a.ws_part + (size_t)(c2 * 2 + sl) * BN * kPanelRows) +
                                                      ((size_t)cc * kPanelRows + r) * 4;
#pragma unroll
                                    for (int j = 0; j < 4; ++j) ld[u][j] = __ldcg(src + j);
                                } else {
#pragma unroll
                                    for (int j = 0; j < 4; ++j) ld[u][j] = make_int4(0, 0, 0, 0);
                                }
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u)
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    sum[4 * j] += ld[u][j].x;
                                    sum[4 * j + 1] += ld[u][j].y;
                                    sum[4 * j + 2] += ld[u][j].z;
                                    sum[4 * j + 3] += ld[u][j].w;
                                }
                        }
                        store_outputs(a, m0 + cc * 16, n, sc, sum);
                    }
                    if (lane == 0) *counter = 0;  // ready for the next call
                    if (warp == 6 && lane == 0 && trace_j < 4) QOQ_MARK(155 + trace_j);
                }
            }
            if (warp == 6 && lane == 0 && trace_j < 4) QOQ_MARK(150 + trace_j);
            ++trace_j;
            accph ^= 1u;
            i = t * ks + ks1;
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) QOQ_MARK(2);
    if (threadIdx.x == 0 && *abort_flag) {
        atomicExch(&g_dev_error, 1);
        // thread 0 is the producer: let its own copies land before exit
        for (int q = 0; q < STAGES; ++q)
            if (issued & (1u << q)) {
                drain_wait(fullw_bar(q), (issued_par >> q) & 1u, 200000000ull);
                if (!issued_x_none) drain_wait(fullx_bar(q), (issued_par >> q) & 1u, 200000000ull);
            }
    }
    if (warp == 0) {
        __syncwarp();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ----------------------------------------------------------------- host --
#ifdef QOQ_TRACE
extern unsigned long long *g_trace_buffer;
#endif

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

template <int BN, int STAGES, int ASTAGES, bool A_TMEM>
cudaError_t launch_cfg(const CUtensorMap &tmap, const GemmArgs &args, int grid, cudaStream_t stream)
{
    using C = GemmCfg<BN, STAGES, ASTAGES, A_TMEM>;
    auto kern = w4a8_gemm_kernel<BN, STAGES, ASTAGES, A_TMEM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the GEMM may start (and stream weights)
    // while the kernel before it in the stream -- normally the activation
    // quantizer -- is still running; the kernel waits for it before it
    // touches X8 or s_x.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tmap, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <bool A_TMEM>
cudaError_t dispatch(int BN, const CUtensorMap &tmap, const GemmArgs &args, int grid, cudaStream_t stream)
{
    switch (BN) {
    // TMEM A ring: as many 32-column slots as fit next to the accumulator
    // in a power-of-two allocation (256 columns for BN <= 64, else 512)
    case 16: return launch_cfg<16, A_TMEM ? 16 : 12, A_TMEM ? 7 : 2, A_TMEM>(tmap, args, grid, stream);
    case 32: return launch_cfg<32, A_TMEM ? 14 : 11, A_TMEM ? 7 : 2, A_TMEM>(tmap, args, grid, stream);
    case 64: return launch_cfg<64, A_TMEM ? 11 : 9, A_TMEM ? 6 : 2, A_TMEM>(tmap, args, grid, stream);
    case 128: return launch_cfg<128, A_TMEM ? 7 : 6, A_TMEM ? 7 : 2, A_TMEM>(tmap, args, grid, stream);
    default: return launch_cfg<256, 4, A_TMEM ? 4 : 2, A_TMEM>(tmap, args, grid, stream);
    }
}

long long gemm_units(int M, int N, int K, int BN)
{
    const long long m_tiles = (M + BN - 1) / BN;
    return m_tiles * (long long)(N / kPanelRows) * (long long)(K / kBlockK);
}

}  // namespace

int gemm_block_n(int M)
{
    return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
}

size_t gemm_workspace_bytes(int M, int N, int K)
{
    const int BN = gemm_block_n(M);
    const long long units = gemm_units(M, N, K, BN);
    const long long grid = std::min<long long>(kMaxCtas, units);
    return kCounterBytes + (size_t)grid * 2 * BN * kPanelRows * sizeof(int32_t);
}

cudaError_t launch_gemm(const int8_t *X8, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int G, uint16_t *Y,
                        int32_t *acc_dbg, void *workspace, bool a_in_tmem, cudaStream_t stream, int *tmap_status)
{
    *tmap_status = 0;
    const int BN = gemm_block_n(M);
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) {
        *tmap_status = -1;
        return cudaErrorNotSupported;
    }
    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)kBlockK, (cuuint32_t)BN};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(X8), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *tmap_status = (int)r;
        return cudaErrorInvalidValue;
    }
    int dev = 0, sms = kMaxCtas;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = gemm_units(M, N, K, BN);
    const long long grid = std::min<long long>(std::min(kMaxCtas, sms), units);

    GemmArgs args;
    args.Wp = Wp;
    args.s_g = s_g;
    args.zs = zs;
    args.s_x = s_x;
    args.s_c = s_c;
    args.Y = Y;
    args.acc_dbg = acc_dbg;
    args.ws_cnt = reinterpret_cast<int32_t *>(workspace);
    args.ws_part = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(workspace) + kCounterBytes);
    args.M = M;
    args.N = N;
    args.K = K;
    args.G = G;
    args.m_tiles = (M + BN - 1) / BN;
    args.ks = K / kBlockK;
    args.total = units;
    args.timeout_ns = 2000000000ull;  // 2 s for one wait: far beyond any legitimate one
#ifdef QOQ_TRACE
    args.trace = g_trace_buffer;
#endif
    return a_in_tmem ? dispatch<true>(BN, tmap, args, (int)grid, stream)
                     : dispatch<false>(BN, tmap, args, (int)grid, stream);
}

#ifdef QOQ_TRACE
unsigned long long *g_trace_buffer = nullptr;
#endif

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
