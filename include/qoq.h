/*
 * qoq.h -- C ABI of libqoq.so, the B200 (sm_100a) QoQ W4A8 linear layer
 *
 *     Y = diag(s_x) * (X8 * W8hat^T) * diag(s_c)
 *
 * X8 holds per-token INT8 activations, and W8hat is the INT8 weight that
 * progressive group quantization produces. The steps are:
 *   - stage 1: per-channel symmetric INT8 in the protective range [-119,119];
 *   - stage 2: group-wise UINT4 codes q with an integer scale s_g and a zero z.
 * At run time the kernel expands each code to INT8 as q*s_g - z*s_g. It
 * multiplies on INT8 tensor cores and accumulates in INT32. The FP16 scales
 * are applied once, after the K loop.
 *
 * Sources, by page title:
 *   "QServe: Low Bit Width Does Not Guarantee High Throughput", section 4
 *       "Formalization and procedure": the stage-1 and stage-2 equations, and
 *       the paragraph after them (multiply by the integer scale first, then
 *       subtract the precomputed zero compensation).
 *   "QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
 *       Serving" (paper card), Key points: FP16 per-channel scales; the
 *       protective range; multiply first, subtract afterward.
 *   "QServe Guide: W4A8KV4 Quantization for LLM Serving":
 *       - Deep Dive, subsection 1: the per-token activation equation and the
 *         output rescaling equation;
 *       - The Architecture, subsection 2: INT8 tensor-core products with
 *         INT32 accumulation, and scales applied after the products.
 *
 * Conventions shared by every call:
 *   - Pointers marked "device" are CUDA device pointers on the current
 *     device. The caller allocates and owns every buffer. The library
 *     allocates no memory.
 *   - FP16 values cross the ABI as uint16_t bit patterns (IEEE binary16).
 *   - Matrices are dense row-major with no strides. W and Y follow the
 *     PyTorch Linear convention: a row of W is an output channel.
 *   - `stream` is a cudaStream_t passed as void*. NULL means the legacy
 *     default stream. Every call that launches work is asynchronous on that
 *     stream.
 *   - Every call returns a qoq_status. Argument checks run on the host
 *     before anything is launched. A failed check returns
 *     QOQ_ERR_INVALID_ARG and launches nothing.
 *   - Shape limits, checked on every call:
 *       - M >= 0. M == 0 is a valid empty problem: it returns QOQ_OK and
 *         launches nothing.
 *       - N is a multiple of 128, from 128 to 1048576.
 *       - K is a multiple of 128, from 128 to 65536. The INT32 accumulator
 *         then cannot overflow: |acc| <= K*128*127 < 2^31.
 *       - group_size is 128 (g128) or K (per-channel).
 *       - Pointers are 16-byte aligned.
 *   - The library needs a B200-class GPU (compute capability 10.0). On any
 *     other device a call returns QOQ_ERR_UNSUPPORTED.
 */
#ifndef QOQ_H
#define QOQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QOQ_API __attribute__((visibility("default")))
#else
#define QOQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QOQ_OK = 0,
    QOQ_ERR_INVALID_ARG = -1,   /* a shape, pointer or size failed the checks above */
    QOQ_ERR_UNSUPPORTED = -2,   /* the current device is not compute capability 10.0 */
    QOQ_ERR_CUDA = -3,          /* a CUDA runtime call or a launch failed */
    QOQ_ERR_TIMEOUT = -4,       /* a kernel's bounded wait ran out (see qoq_device_error) */
    QOQ_ERR_SCRATCH_TOO_SMALL = -5 /* qoq_w4a8_gemm_noalloc: the shape needs more scratch
                                      than the built-in buffer holds */
} qoq_status;

/* Short English text for a status code. The string is static. */
QOQ_API const char *qoq_status_string(int status);

/* ------------------------------------------------------------------------
 * Packed weight layout: the "Blackwell interleaved UINT4" layout
 * ------------------------------------------------------------------------
 * Wp holds one 4-bit code per weight, grouped into chunks, one per
 * (128-channel panel p, 128-wide K block b). Chunks are ordered p-major, S
 * bytes apart:
 *     chunk(p, b) starts at byte (p * (K/128) + b) * S,
 *     S = 8192 + 256 when group_size == 128, S = 8192 when group_size == K.
 * The first 8192 bytes of a chunk hold its codes. With group_size == 128
 * the chunk covers exactly one group, and bytes 8192..8319 hold that
 * group's s_g for channels r = 0..127 of the panel, bytes 8320..8447 its
 * zs (the same values as in the s_g and zs arrays below): one copy brings
 * a stage's codes and tables together.
 * The codes of a chunk form 4 slabs of 2048 bytes, one per 32-wide K slice j. Inside slab
 * j, channel r (0..127 within the panel) owns the 16 bytes at j*2048 + r*16.
 * Those 16 bytes are 4 little-endian 32-bit words. For word w (0..3),
 * byte i (0..3), with k0 = 128*b + 32*j:
 *     low nibble  = q[n][k0 + 4*w + i]
 *     high nibble = q[n][k0 + 16 + 4*w + i]
 * So one AND of a word with 0x0F0F0F0F gives four consecutive codes in four
 * byte lanes, and one shift plus one AND gives the next four.
 *
 * The group tables are also written as arrays, panel-major, one byte per
 * entry: for channel n in panel p = n/128 (r = n%128) and group
 * g = k/group_size,
 *     s_g[(p*(K/group_size) + g)*128 + r]  the integer group scale (1..16),
 *     zs [(p*(K/group_size) + g)*128 + r]  the zero compensation z*s_g (0..240).
 * The GEMM reads per-channel tables (group_size == K) from these arrays and
 * 128-wide groups' tables from the chunks. s_c[n] is the FP16 channel scale.
 */

/* Bytes of Wp for an N x K weight: N*K/2, plus N*K/64 for the tables the
 * chunks carry when group_size == 128. Returns 0 when N or K is not a
 * positive multiple of 128 or group_size is neither 128 nor K. */
QOQ_API size_t qoq_packed_weight_bytes(int N, int K, int group_size);

/* Progressive group quantization and packing (the offline step).
 *
 * Sources: "QServe: Low Bit Width Does Not Guarantee High Throughput",
 * section 4, stage-1 and stage-2 equations; FP16 scales per the paper card's
 * Key points. Choices where the pages are silent:
 *   - round is half to even;
 *   - s_c = fp16(max|W_n| / 119), and the stored FP16 value is the one used
 *     to quantize;
 *   - per group: mn = min(0, min W8) and mx = max(0, max W8);
 *     s_g = max(1, ceil((mx - mn)/15)); z = round(-mn/s_g);
 *     q = clamp(round(W8/s_g) + z, 0, 15).
 *   - A row whose scale rounds to FP16 zero quantizes to all zeros.
 *   - W must be finite. Entries with |W| >= 65520*119 make s_c infinite.
 *
 *   W      device, float32 [N][K], read only.
 *   Wp     device, qoq_packed_weight_bytes(N, K, group_size) bytes, written in the
 *          packed layout above.
 *   s_c    device, uint16_t [N] FP16 bits, written.
 *   s_g    device, uint8_t [N/128][K/group_size][128], written.
 *   zs     device, uint8_t [N/128][K/group_size][128], written.
 *   z_dbg  device, uint8_t [N][K/group_size], or NULL. When given, the zero
 *          points z (0..15) are written there, channel-major (inspection and
 *          parity tests; the GEMM needs only zs).
 *   q_dbg  device, uint8_t [N][K], or NULL (16-byte aligned when given).
 *          When given, the canonical codes q (0..15) are written there, one
 *          per byte, in the natural [n][k] order (inspection and parity).
 * The result is deterministic and bit-identical on every call.
 */
QOQ_API int qoq_pack_weights(const float *W, int N, int K, int group_size,
                     uint8_t *Wp, uint16_t *s_c, uint8_t *s_g, uint8_t *zs,
                     uint8_t *z_dbg, uint8_t *q_dbg, void *stream);

/* Packs a gate/up projection pair for the SiLU-gated epilogue of
 * qoq_w4a8_gemm_fused (the pages have no counterpart: it is the layout the
 * fused MLP activation needs, not part of the method).
 *
 *   W      device, float32 [N][K]: rows 0..N/2-1 are the gate projection's
 *          output channels, rows N/2..N-1 the up projection's (the order of
 *          a fused gate/up weight). N is a multiple of 128.
 * The quantization is exactly qoq_pack_weights' (per output channel, so the
 * row order does not change any value). Only the placement differs: packed
 * panel p (rows 128p..128p+127 of Wp, s_c, s_g and zs) holds gate channels
 * 64p..64p+63 followed by up channels 64p..64p+63, so that one tile of the
 * GEMM holds both halves of 64 outputs. Outputs, sizes and limits as for
 * qoq_pack_weights (there are no debug outputs). */
QOQ_API int qoq_pack_weights_gate_up(const float *W, int N, int K, int group_size,
                             uint8_t *Wp, uint16_t *s_c, uint8_t *s_g, uint8_t *zs,
                             void *stream);

/* Per-token symmetric INT8 activation quantization.
 *
 * Source: "QServe Guide: W4A8KV4 Quantization for LLM Serving", Deep Dive,
 * subsection 1, the activation equation. For each row m:
 *     s_x[m] = fp16(max_k |X[m][k]| / 127)
 *     X8[m][k] = clamp(round(X[m][k] / s_x[m]), -128, 127)
 * The division is IEEE FP32 and round is half to even. A row whose scale
 * rounds to FP16 zero gives all zeros.
 *
 *   X      device, uint16_t [M][K] FP16 bits, read only. Must be finite.
 *   X8     device, int8_t [M][K], written.
 *   s_x    device, uint16_t [M] FP16 bits, written.
 *   rowsum device, int32_t [M], or NULL (4-byte aligned when given). When
 *          given, rowsum[m] = sum_k X8[m][k] is written there. It is the term
 *          a zero point multiplies when the zero compensation is applied after
 *          the products instead of before them; qoq_w4a8_gemm subtracts z*s_g
 *          from the weights before the products (multiply first, subtract
 *          afterward), so it takes no rowsum.
 * K follows the GEMM limits above (multiple of 128, at most 65536).
 */
QOQ_API int qoq_quant_act_per_token(const uint16_t *X, int M, int K,
                            int8_t *X8, uint16_t *s_x, int32_t *rowsum, void *stream);

/* Bytes of scratch workspace qoq_w4a8_gemm needs for this shape.
 *
 * The GEMM splits the K loop of some output tiles across SMs so that every
 * SM streams the same number of weight bytes. The INT32 partial sums of a
 * split tile meet in this workspace. The sum is exact in any order.
 * Layout: the first 8192 bytes hold arrival counters (the same region for
 * every shape); the partial tiles follow. Rules:
 *   - a fresh workspace must be zero-filled once before its first use;
 *   - every completed call leaves the counters at zero again, so one
 *     workspace serves any sequence of shapes on one stream;
 *   - after a call that returned QOQ_ERR_TIMEOUT from qoq_device_error,
 *     zero-fill the workspace again.
 * The size covers both token-tile rules of qoq_set_gemm_narrow_tiles, so a
 * workspace stays valid when that setting changes.
 * Returns 0 for an invalid shape. */
QOQ_API size_t qoq_gemm_workspace_bytes(int M, int N, int K, int group_size);

/* The W4A8 GEMM with its epilogue.
 *
 * Sources: "QServe Guide: W4A8KV4 Quantization for LLM Serving", The
 * Architecture, subsection 2, and Deep Dive, subsection 1, the output
 * rescaling equation. For every m < M and n < N:
 *     W8hat[n][k] = q[n][k]*s_g[g][n] - zs[g][n]            (INT8)
 *     acc[m][n]   = sum_k X8[m][k] * W8hat[n][k]           (INT32, exact)
 *     Y[m][n]     = fp16( ((float)acc * (float)s_x[m]) * (float)s_c[n] )
 * The FP32 products are rounded in that order, with no fused multiply-add.
 *
 *   X8, s_x      device, from qoq_quant_act_per_token.
 *   Wp, s_c, s_g, zs
 *                device, from qoq_pack_weights with the same N, K and
 *                group_size.
 *   Y            device, uint16_t [M][N] FP16 bits, written.
 *   acc_dbg      device int32_t [M][N], or NULL. When given, the raw INT32
 *                accumulators are written there too (used for parity tests).
 *   workspace    device, at least qoq_gemm_workspace_bytes(M, N, K,
 *                group_size) bytes, prepared as described above. Two calls
 *                that may run at the same time must not share a workspace.
 *   workspace_bytes  the size of that buffer. A smaller size is rejected.
 * The kernel's internal waits are bounded. If one runs out, the kernel
 * stops early and sets a device error flag; qoq_device_error reports it.
 */
QOQ_API int qoq_w4a8_gemm(const int8_t *X8, const uint16_t *s_x,
                  const uint8_t *Wp, const uint16_t *s_c,
                  const uint8_t *s_g, const uint8_t *zs,
                  int M, int N, int K, int group_size,
                  uint16_t *Y, int32_t *acc_dbg,
                  void *workspace, size_t workspace_bytes, void *stream);

/* Output-side fusion in the GEMM's epilogue (the pages stop at the layer's
 * FP16 output, "QServe Guide: W4A8KV4 Quantization for LLM Serving", The
 * Architecture, subsection 2; these are the operations that follow it in a
 * transformer block, done on the layer's FP16 values before they leave the
 * SM). The layer's own output y[m][n] is rounded exactly as qoq_w4a8_gemm
 * rounds it; then:
 *   QOQ_EPILOGUE_NONE      Y = y (the same as qoq_w4a8_gemm).
 *   QOQ_EPILOGUE_RESIDUAL  Y[m][n] = fp16((float)y[m][n] + (float)R[m][n]):
 *                          a residual add, the same bits as an FP16 add after
 *                          the layer.
 *   QOQ_EPILOGUE_SILU_MUL  Wp, s_c, s_g, zs from qoq_pack_weights_gate_up;
 *                          with g = y of gate channel j and u = y of up
 *                          channel j, Y[m][j] = fp16(silu(g) * u) for
 *                          j < N/2, silu(g) = g / (1 + exp(-g)) in FP32 with
 *                          IEEE division. Y is [M][N/2].
 */
typedef enum {
    QOQ_EPILOGUE_NONE = 0,
    QOQ_EPILOGUE_RESIDUAL = 1,
    QOQ_EPILOGUE_SILU_MUL = 2
} qoq_epilogue_kind;

/* The GEMM of qoq_w4a8_gemm with an output-side fusion.
 *   epilogue   a qoq_epilogue_kind; other values give QOQ_ERR_INVALID_ARG.
 *   residual   device, uint16_t [M][N] FP16 bits, read; required (16-byte
 *              aligned) for QOQ_EPILOGUE_RESIDUAL, ignored otherwise. It may
 *              be the same buffer as Y (each element is read before it is
 *              written, by the same thread).
 *   Y          device, uint16_t FP16 bits, written: [M][N], or [M][N/2] for
 *              QOQ_EPILOGUE_SILU_MUL.
 * Every other argument, limit and workspace rule as for qoq_w4a8_gemm (no
 * acc_dbg). */
QOQ_API int qoq_w4a8_gemm_fused(const int8_t *X8, const uint16_t *s_x,
                        const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs,
                        int M, int N, int K, int group_size, int epilogue,
                        const uint16_t *residual, uint16_t *Y,
                        void *workspace, size_t workspace_bytes, void *stream);

/* The INT32 inner products alone: acc[m][n] = sum_k X8[m][k] * W8hat[n][k]
 * for m < M, n < N, over this call's K (the GEMM of qoq_w4a8_gemm without
 * its output scaling).
 *
 * Source: "QServe Guide: W4A8KV4 Quantization for LLM Serving", The
 * Architecture, subsection 2 (INT8 x INT8 products accumulated in INT32).
 * It is the per-GPU step of a row-parallel (K-split) layer: each GPU holds a
 * K slice of the weights (a multiple of the group size), computes these
 * partial sums, the GPUs add them (an INT32 sum is exact in any order), and
 * qoq_epilogue_i32 applies the scales once.
 *   X8, ldx          device, int8_t: row m of this GPU's K slice starts at
 *                    X8 + m*ldx (ldx >= K, a multiple of 16), so a slice of
 *                    a full [M][K_total] activation matrix is passed without
 *                    a copy (X8 = base + k0, ldx = K_total).
 *   Wp, s_g, zs      device, the packed slice (see the K-split helpers of the
 *                    Python binding for slicing a packed weight).
 *   acc              device, int32_t [M][N], written.
 *   workspace, workspace_bytes  as for qoq_w4a8_gemm.
 * Limits as for qoq_w4a8_gemm. */
QOQ_API int qoq_w4a8_gemm_i32(const int8_t *X8, int ldx, const uint8_t *Wp, const uint8_t *s_g,
                      const uint8_t *zs, int M, int N, int K, int group_size, int32_t *acc,
                      void *workspace, size_t workspace_bytes, void *stream);

/* The output rescaling on INT32 sums computed elsewhere:
 *     Y[m][n] = fp16( ((float)acc[m][n] * (float)s_x[m]) * (float)s_c[n] )
 * rounded exactly as qoq_w4a8_gemm's epilogue.
 * Source: "QServe Guide: W4A8KV4 Quantization for LLM Serving", Deep Dive,
 * subsection 1, the output rescaling equation.
 *   acc    device, int32_t [M][N] (for a K-split layer: the summed partials).
 *   s_x    device, uint16_t [M] FP16 bits; s_c device, uint16_t [N] FP16 bits.
 *   Y      device, uint16_t [M][N] FP16 bits, written.
 * N is a multiple of 128 (at most 1048576); M >= 0 (0 launches nothing). */
QOQ_API int qoq_epilogue_i32(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c,
                     int M, int N, uint16_t *Y, void *stream);

/* ------------------------------------------------------------------------
 * The W8A8 yardstick (the pages have no kernel for it; they use W8A8 as the
 * INT8-peak side of their roofline argument, "QServe: Low Bit Width Does Not
 * Guarantee High Throughput", section 2 "Motivation", Figure 3). The same
 * GEMM kernel with 8-bit weights loaded by TMA straight into the tensor
 * cores' operand slots: no unpacking and no dequantization, twice the weight
 * bytes. Comparing it with qoq_w4a8_gemm measures what the 4-bit stream saves
 * at small M and what the dequantization costs at large M.
 * ------------------------------------------------------------------------ */

/* Per-channel symmetric INT8 weights: s_w[n] = fp16(max_k |W[n][k]| / 127),
 * W8[n][k] = clamp(round(W[n][k] / s_w[n]), -127, 127), IEEE division, round
 * half to even, with the stored FP16 scale; a zero scale gives a zero row.
 *   W    device, float32 [N][K], read only (finite).
 *   W8   device, int8_t [N][K], written.
 *   s_w  device, uint16_t [N] FP16 bits, written.
 * N and K follow the GEMM limits. */
QOQ_API int qoq_quantize_weights_w8(const float *W, int N, int K, int8_t *W8, uint16_t *s_w,
                            void *stream);

/* Y[m][n] = fp16( ((float)acc * s_x[m]) * s_w[n] ), acc = sum_k X8[m][k] * W8[n][k]
 * (INT32, exact), the epilogue of qoq_w4a8_gemm.
 *   X8, s_x   device, from qoq_quant_act_per_token.
 *   W8, s_w   device, from qoq_quantize_weights_w8.
 *   Y         device, uint16_t [M][N] FP16 bits, written.
 *   acc_dbg   device int32_t [M][N] or NULL: the raw INT32 sums.
 *   workspace, workspace_bytes  as for qoq_w4a8_gemm, sized by
 *             qoq_gemm_workspace_bytes(M, N, K, 128).
 * Limits as for qoq_w4a8_gemm. */
QOQ_API int qoq_w8a8_gemm(const int8_t *X8, const uint16_t *s_x, const int8_t *W8, const uint16_t *s_w,
                  int M, int N, int K, uint16_t *Y, int32_t *acc_dbg,
                  void *workspace, size_t workspace_bytes, void *stream);

/* The whole W4A8 linear layer in one call: the per-token quantization of
 * qoq_quant_act_per_token followed by qoq_w4a8_gemm.
 *
 * Sources: as for those two calls; the result is bit-identical to calling
 * them in sequence (the pages describe the two steps as one layer).
 *
 *   X        device, uint16_t [M][K] FP16 bits, read only.
 *   X8, s_x  device, written exactly as qoq_quant_act_per_token writes them
 *            (int8_t [M][K]; uint16_t [M] FP16 bits, 16-byte aligned).
 *   Wp, s_c, s_g, zs, Y, workspace, workspace_bytes
 *            as for qoq_w4a8_gemm (the same workspace rules; this call also
 *            leaves the workspace's counters at zero).
 * By default the call launches the quantizer and the GEMM back to back on
 * the stream (programmatic dependent launch: the GEMM streams its weights
 * while the quantizer runs). With qoq_set_linear_in_kernel_quant(1) and
 * M <= 148 it is one launch instead: the GEMM's epilogue warps quantize the
 * rows (one row per SM) and publish each finished row with a release
 * operation, and the GEMM's loads of X8 and s_x wait (bounded) until every
 * row is done. Limits: as for qoq_w4a8_gemm.
 */
QOQ_API int qoq_w4a8_linear(const uint16_t *X, int M, int N, int K, int group_size,
                    const uint8_t *Wp, const uint16_t *s_c,
                    const uint8_t *s_g, const uint8_t *zs,
                    int8_t *X8, uint16_t *s_x, uint16_t *Y,
                    void *workspace, size_t workspace_bytes, void *stream);

/* The same GEMM as qoq_w4a8_gemm, for callers that cannot allocate memory.
 *
 * The paper has no counterpart to this call. It exists because some callers
 * cannot hand qoq_w4a8_gemm a scratch workspace:
 *   - code inside an inference engine's execute/enqueue step, where
 *     allocating is forbidden or would synchronize the device (cudaFree
 *     waits for all outstanding work, and cudaMalloc can too);
 *   - plug-ins that have no allocator of their own;
 *   - real-time paths that must never enter the allocator.
 *
 * This entry point keeps the GEMM's scratch in a fixed 16 MiB
 * (QOQ_NOALLOC_SCRATCH_BYTES) buffer in the library's own device image:
 *   - every GPU that loads the library holds that buffer until the process
 *     exits;
 *   - the call itself allocates nothing, through CUDA or any other library;
 *   - the caller still provides every input and the output Y, with the
 *     layouts, limits and checks of qoq_w4a8_gemm (there is no acc_dbg).
 *
 * Scratch rules:
 *   - a shape whose qoq_gemm_workspace_bytes exceeds
 *     QOQ_NOALLOC_SCRATCH_BYTES is rejected with QOQ_ERR_SCRATCH_TOO_SMALL.
 *     Token counts up to 128 fit for every N and K;
 *   - every call on a device shares the one buffer, which keeps the last
 *     call's contents. Each call first clears the part that must start at
 *     zero (an asynchronous memset on `stream`, not an allocation);
 *   - two calls whose work can overlap on the GPU (different streams, or
 *     concurrent graph branches) race on the buffer and give undefined
 *     results. Serialize them.
 *
 * The first call on each device looks up the buffer's device address, with
 * that device current, and caches it. Make that first call before any
 * stream capture that should contain this entry point. */
#define QOQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
QOQ_API int qoq_w4a8_gemm_noalloc(const int8_t *X8, const uint16_t *s_x,
                                  const uint8_t *Wp, const uint16_t *s_c,
                                  const uint8_t *s_g, const uint8_t *zs,
                                  int M, int N, int K, int group_size,
                                  uint16_t *Y, void *stream);

/* ------------------------------------------------------------------------
 * KV4 decode attention with SmoothAttention
 * ------------------------------------------------------------------------
 * Sources: "QServe: Low Bit Width Does Not Guarantee High Throughput",
 * section 4 (SmoothAttention: K' = K / lambda, Q' = Q * lambda, so
 * Q'K'^T = QK^T, with lambda = max|K|^alpha, alpha = 0.5); "QServe Guide:
 * W4A8KV4 Quantization for LLM Serving", The Architecture, subsection 3
 * (the smoothed keys and the values stored as 4-bit integers with
 * per-channel scale factors). Choices where the pages are silent:
 *   - statistics per (sequence, KV head, channel), over the cached tokens;
 *   - lambda = fp16(max(sqrt(max_l |K[l][c]|), 1e-5));
 *   - K'[l][c] = K / lambda (FP32); s = fp16(max_l |X'| / 7); code =
 *     clamp(round(X' / s), -8, 7), round half to even, for X' = K' (s_k)
 *     and X' = V (s_v); a zero scale gives zero codes.
 * Layouts (head dimension d = 128):
 *   K, V      FP16 [B][Hkv][L][d];   q, out   FP16 [B][Hq][d];
 *   K4, V4    uint8 [B][Hkv][L][d/2]: byte j of a token row holds channel
 *             2j (low nibble) and 2j+1 (high nibble), each as code + 8;
 *   lam, s_k, s_v   FP16 bits [B][Hkv][d].
 * Query head h attends with KV head h / (Hq / Hkv) (grouped-query
 * attention; Hq / Hkv in {1, 2, 4, 8}).
 */

/* Fills a KV4 cache from FP16 keys and values (the cache writer).
 * B >= 0 (0 does nothing), 1 <= Hkv <= 1024, 1 <= L <= 2^20, d = 128;
 * 16-byte aligned pointers. */
QOQ_API int qoq_kv4_cache_quantize(const uint16_t *K, const uint16_t *V, int B, int Hkv, int L, int d,
                           uint8_t *K4, uint8_t *V4, uint16_t *lam, uint16_t *s_k, uint16_t *s_v,
                           void *stream);

/* Bytes of scratch qoq_kv4_decode_attention needs (per-chunk partial
 * results); 0 for an invalid or empty shape. */
QOQ_API size_t qoq_kv4_attention_workspace_bytes(int B, int Hq, int Hkv, int L, int d);

/* Attention of one new query token per sequence over its L cached tokens:
 *   score[l] = sum_c (q[c] * lam[c]) * (s_k[c] * code_k[l][c]) / sqrt(d)
 *   p = softmax(score);  out[c] = sum_l p[l] * s_v[c] * code_v[l][c]
 * rounded to FP16 once. The kernel folds lam, s_k and 1/sqrt(d) into the
 * query and s_v into the final sum. Both products run on the tensor cores
 * with the codes exact in FP16 and each FP32 factor (the folded query, the
 * softmax numerators) split into two FP16 parts, summed in FP32: within
 * 2 FP16 ulp (plus 1e-3 of the output row's largest value) of the binary64
 * result.
 *   workspace   device, qoq_kv4_attention_workspace_bytes bytes, any
 *               contents (every call overwrites what it reads).
 * Limits as for qoq_kv4_cache_quantize, plus Hq a multiple of Hkv. */
QOQ_API int qoq_kv4_decode_attention(const uint16_t *q, const uint8_t *K4, const uint8_t *V4,
                             const uint16_t *lam, const uint16_t *s_k, const uint16_t *s_v,
                             int B, int Hq, int Hkv, int L, int d, uint16_t *out,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Expands the packed codes to the INT8 weights the GEMM multiplies,
 * W8hat[n][k] = q*s_g - zs. It runs the same device routine as the GEMM's
 * in-register dequantization. Use it for parity tests and inspection; it is
 * not on the hot path.
 *   W8hat  device, int8_t [N][K], written. */
QOQ_API int qoq_dequant_weights_i8(const uint8_t *Wp, const uint8_t *s_g, const uint8_t *zs,
                           int N, int K, int group_size, int8_t *W8hat, void *stream);

/* Selects where the GEMM keeps the dequantized weight tile before it feeds
 * the tensor cores:
 *   1 (default): tensor memory (TMEM), read by the MMA as its A operand;
 *   0: shared memory.
 * The choice applies to later GEMM calls from every thread. Results are
 * identical either way. Returns QOQ_ERR_INVALID_ARG for other values. */
QOQ_API int qoq_set_gemm_a_in_tmem(int enable);

/* Selects whether 256-token tiles (M > 128) run on pairs of SMs when the
 * weight tile is in TMEM and N is a multiple of 256:
 *   1 (default): two CTAs of a cluster compute a 256-channel tile with one
 *      M = 256 tensor-core instruction per K step (tcgen05 cta_group::2),
 *      each holding half of the activation tile, which halves the
 *      activation traffic per SM;
 *   0: one CTA per 128-channel tile.
 * The choice applies to later GEMM calls from every thread. Results are
 * identical either way. Returns QOQ_ERR_INVALID_ARG for other values. */
QOQ_API int qoq_set_gemm_cta_pairs(int enable);

/* Selects the CTA size for token tiles up to 64 (decode):
 *   1: half-SM CTAs (at most half of an SM's registers, shared memory and
 *      tensor memory, 128-wide K stages), so that the CTA of the next GEMM
 *      on the stream can be resident beside the current one and stream and
 *      dequantize its weights while the current one finishes;
 *   0 (default): one CTA per SM with deeper rings and 256-wide K stages.
 * The choice applies to later GEMM calls from every thread. Results are
 * identical either way. Returns QOQ_ERR_INVALID_ARG for other values. */
QOQ_API int qoq_set_gemm_half_ctas(int enable);

/* Selects the kernel for M <= 8 tokens (decode):
 *   1 (default): a decode kernel without the GEMM's per-launch machinery:
 *      the codes expand to INT8 in registers as in the GEMM, straight into
 *      the fragments of warp-level INT8 MMAs (m16n8k32, INT32 sums, the
 *      tokens as the 8-wide N dimension); each CTA owns 16 output channels
 *      and all of K, so no tensor memory, barrier ring or split-tile handoff
 *      is set up per launch;
 *   0: the tensor-core GEMM with a 16-token tile.
 * It does not apply to the SiLU-gated gate/up epilogue, to the one-launch
 * layer call, or to N above 128 channels per SM (18944 on 148 SMs), where
 * the GEMM's bulk-copy weight stream is faster; those keep the GEMM. For
 * small N the decode kernel splits K over a cluster of 2 or 4 CTAs. The choice applies to later GEMM calls
 * from every thread. Results are identical either way. Returns
 * QOQ_ERR_INVALID_ARG for other values. */
QOQ_API int qoq_set_gemm_gemv(int enable);

/* Selects the token-tile width rule for M > 64:
 *   1 (default): 256 tokens per tile (128 for M <= 128), narrowed to 128 and
 *      then 64 while the tiles are so few that stream-K would share each
 *      among four or more CTAs (two or more when K <= 4096); every extra
 *      CTA on a tile adds one INT32 partial tile that the finishing CTA
 *      reads back;
 *   0: the tile covers min(M, 256) tokens rounded up to 128 or 256.
 * qoq_gemm_workspace_bytes covers both rules, so a workspace stays valid
 * when this changes. The choice applies to later GEMM calls from every
 * thread. Results are identical either way. Returns QOQ_ERR_INVALID_ARG
 * for other values. */
QOQ_API int qoq_set_gemm_narrow_tiles(int enable);

/* Selects how qoq_w4a8_linear runs for M <= 148:
 *   0 (default): the quantizer kernel, then the GEMM kernel;
 *   1: one GEMM launch that quantizes its own rows (see qoq_w4a8_linear).
 * On B200, chains of decode-sized layers measured 0.5-3.8 us per layer
 * faster with two kernels: one row per SM, all waited for by every SM,
 * costs more than the quantizer's own launch. The choice applies to later
 * calls from every thread. Results are identical either way. Returns
 * QOQ_ERR_INVALID_ARG for other values. */
QOQ_API int qoq_set_linear_in_kernel_quant(int enable);

/* Self-test of the failure path (the pages have no counterpart). Launches
 * one thread that waits on a barrier phase nothing completes, with the same
 * bounded wait every GEMM role uses and a budget of timeout_ns (1 us ..
 * 100 ms) instead of the GEMM's 2 s. When the budget runs out the kernel
 * raises the device error flag and returns normally: nothing traps, and the
 * context stays usable. A following qoq_device_error therefore reports
 * QOQ_ERR_TIMEOUT (and clears the flag). Returns QOQ_ERR_INVALID_ARG for a
 * budget outside the range. */
QOQ_API int qoq_selftest_wait_timeout(unsigned long long timeout_ns, void *stream);

/* Synchronizes `stream`, then reads and clears the device error flag of
 * the current device.
 *   Returns QOQ_OK when no kernel reported a problem.
 *   Returns QOQ_ERR_TIMEOUT when a bounded wait in a GEMM ran out. The CUDA
 *     context stays usable, but the outputs of that call are undefined.
 *   Returns QOQ_ERR_CUDA when the synchronization itself failed. */
QOQ_API int qoq_device_error(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QOQ_H */
