// qoq_internal.h -- host-side launchers behind the C ABI (C++ linkage, not
// exported).  Arguments have been validated by the caller (qoq_api.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace qoq {

// Upper bound on the persistent GEMM grid (B200 has 148 SMs); also sizes
// the split-tile workspace, so the workspace size does not depend on the
// device a query runs on.
constexpr int kMaxCtas = 148;

// The split-tile counters (kMaxCtas x 4 int32) occupy this many bytes at the
// start of every GEMM workspace; the INT32 partial tiles follow.
constexpr size_t kCounterBytes = 8192;
// split-tile counters: kMaxCtas CTAs x 2 epilogue groups x 4 quarters
static_assert(kMaxCtas * 2 * 4 * 4 <= kCounterBytes - 64, "counter region");

// z_dbg and q_dbg may be null (optional inspection outputs).  With gate_up
// set, W holds a gate/up pair ([N/2 gate rows; N/2 up rows]) and packed
// panel p takes gate rows 64p..64p+63 then up rows 64p..64p+63.
cudaError_t launch_pack(const float *W, int N, int K, int G, uint8_t *Wp, uint16_t *s_c, uint8_t *s_g,
                        uint8_t *zs, uint8_t *z_dbg, uint8_t *q_dbg, cudaStream_t stream, bool gate_up = false);

// rowsum may be null.
cudaError_t launch_act_quant(const uint16_t *X, int M, int K, int8_t *X8, uint16_t *s_x, int32_t *rowsum,
                             cudaStream_t stream);

cudaError_t launch_dequant(const uint8_t *Wp, const uint8_t *s_g, const uint8_t *zs, int N, int K, int G,
                           int8_t *W8hat, cudaStream_t stream);

// Tile width along M (tokens) the GEMM uses for a given M.
int gemm_block_n(int M, int N, int K);

// False when the shape has more work units than the GEMM's 32-bit
// scheduling arithmetic covers.
bool gemm_shape_supported(int M, int N, int K);

size_t gemm_workspace_bytes(int M, int N, int K);

// One bounded wait that nothing completes (the failure-path self-test).
cudaError_t launch_stuck_wait(unsigned long long budget_ns, cudaStream_t stream);

// Whether 256-token tiles run on CTA pairs (2-SM MMA); default on.
void set_cta_pairs(bool enable);

// Whether few, widely shared 256/128-token tiles give way to narrower ones;
// default on.
void set_narrow_tiles(bool enable);

// Whether token tiles up to 64 run in half-SM CTAs (two per SM, so that
// consecutive GEMMs overlap).
void set_half_ctas(bool enable);
// Up to kGemvMaxM tokens: the decode kernel (warp-level MMAs, the default)
// or the tensor-core GEMM.
constexpr int kGemvMaxM = 8;
void set_gemv(bool enable);

// Word offsets, in the workspace's counter region, of the two counters of
// the one-launch layer call (after the split-tile counters of up to kMaxCtas CTAs).
constexpr int kFusedReadyWord = 2000;
constexpr int kFusedDoneWord = 2001;
// Largest M for which the layer call can quantize inside the GEMM kernel.
constexpr int kFusedMaxRows = kMaxCtas;

// ldx: bytes between rows of X8 (0 means K).  W8 non-null: the W8A8
// yardstick, INT8 weights [N][K] in place of the packed ones (Wp, s_g, zs
// unused; s_c holds the weights' per-channel scales).
// Returns cudaSuccess or the launch / tensor-map error.  `tmap_status`
// receives the driver status of the tensor-map encode (0 on success).
// With X non-null the kernel first quantizes X into X8 and s_x (the one-launch
// call); otherwise it reads them.
// Output-side fusion kinds of the GEMM epilogue (the values of
// qoq_epilogue_kind in qoq.h).
constexpr int kEpiPlain = 0;
constexpr int kEpiResidual = 1;
constexpr int kEpiSiluMul = 2;
// (internal) INT32 sums only, into acc_dbg: the partial GEMM of a K-split layer
constexpr int kEpiI32 = 3;

// W8A8 yardstick weights: per-channel symmetric INT8, s_w = fp16(max|W|/127).
cudaError_t launch_quantize_w8(const float *W, int N, int K, int8_t *W8, uint16_t *s_w, cudaStream_t stream);

// Y[m][n] = fp16(((float)acc[m][n] * s_x[m]) * s_c[n]) over [M][N].
cudaError_t launch_epilogue_i32(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c, int M, int N,
                                uint16_t *Y, cudaStream_t stream);

cudaError_t launch_gemm(const int8_t *X8, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int G, uint16_t *Y,
                        int32_t *acc_dbg, void *workspace, bool a_in_tmem, cudaStream_t stream,
                        int *tmap_status, const uint16_t *X = nullptr, int epi = kEpiPlain,
                        const uint16_t *R = nullptr, int ldx = 0, const int8_t *W8 = nullptr);


// KV4 cache (head dimension 128): per (sequence, KV head) lambda, s_k, s_v
// and the packed 4-bit codes of K' = K / lambda and V.
cudaError_t launch_kv4_cache(const uint16_t *K, const uint16_t *V, int B, int Hkv, int L, uint8_t *K4, uint8_t *V4,
                             uint16_t *lam, uint16_t *s_k, uint16_t *s_v, cudaStream_t stream);
// Decode attention over a KV4 cache: chunk kernel, then combine kernel.
size_t kv4_workspace_bytes(int B, int Hq, int Hkv, int L);
cudaError_t launch_kv4_attention(const uint16_t *q, const uint8_t *K4, const uint8_t *V4, const uint16_t *lam,
                                 const uint16_t *s_k, const uint16_t *s_v, int B, int Hq, int Hkv, int L,
                                 uint16_t *out, void *workspace, cudaStream_t stream);

// Device error flag of the current device: read and clear (synchronous).
cudaError_t read_and_clear_device_error(cudaStream_t stream, int *value);
// The KV4 kernels' own flag (read after that synchronization).
cudaError_t read_and_clear_kv4_error(int *value);

// The argument checks every GEMM entry point shares (qoq_api.cu).
bool valid_nk(int N, int K);
bool valid_group(int K, int G);
bool aligned16(const void *p);
// Where the GEMM keeps its dequantized tile (qoq_set_gemm_a_in_tmem).
bool gemm_a_in_tmem();
// QOQ_OK when the current device is compute capability 10.0 (cached per device).
int check_device();

// The decode kernel for M <= kGemvMaxM tokens (same inputs, outputs and
// rounding as launch_gemm; no workspace).  gemv_applies says whether a call
// takes it: not the SiLU-gated pair, not the one-launch layer call, and not
// N above 8 channel groups of 16 per SM, where the GEMM's bulk-copy weight
// stream is faster than the decode kernel's loads.
bool gemv_applies(int M, int N, int epi, bool one_launch, int sms);
cudaError_t launch_gemv(const int8_t *X8, int ldx, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int G, uint16_t *Y,
                        int32_t *acc_dbg, int epi, const uint16_t *R, cudaStream_t stream);

}  // namespace qoq
