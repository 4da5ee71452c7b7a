// qoq_api.cu -- the extern "C" entry points declared in include/qoq.h:
// argument validation on the host, then the call's launches (one per call,
// two for the layer call in its default form).
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/qoq.h"
#include "qoq_internal.h"
#include "qoq_layout.cuh"

static_assert(QOQ_EPILOGUE_NONE == qoq::kEpiPlain && QOQ_EPILOGUE_RESIDUAL == qoq::kEpiResidual &&
                  QOQ_EPILOGUE_SILU_MUL == qoq::kEpiSiluMul,
              "epilogue kinds");

namespace {

std::atomic<int> g_a_in_tmem{1};
std::atomic<int> g_linear_in_kernel_quant{0};

constexpr int kMaxK = 65536;
constexpr int kMaxN = 1 << 20;
constexpr int kMaxM = 1 << 24;

int from_cuda(cudaError_t e)
{
    return e == cudaSuccess ? QOQ_OK : QOQ_ERR_CUDA;
}

}  // namespace

namespace qoq {

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool valid_nk(int N, int K)
{
    return N >= 128 && N <= kMaxN && N % 128 == 0 && K >= 128 && K <= kMaxK && K % 128 == 0;
}

bool valid_group(int K, int G)
{
    return G == 128 || G == K;
}

bool gemm_a_in_tmem()
{
    return g_a_in_tmem.load() != 0;
}

// Compute capability 10.0 check for the current device, cached per device.
int check_device()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
    if (dev < 0 || dev >= 64) return QOQ_ERR_UNSUPPORTED;
    int c = cache[dev].load();
    if (c == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return QOQ_ERR_CUDA;
        c = (major == 10 && minor == 0) ? 1 : -1;
        cache[dev].store(c);
    }
    return c == 1 ? QOQ_OK : QOQ_ERR_UNSUPPORTED;
}

}  // namespace qoq

using qoq::aligned16;
using qoq::check_device;
using qoq::valid_group;
using qoq::valid_nk;

extern "C" {

const char *qoq_status_string(int status)
{
    switch (status) {
    case QOQ_OK: return "ok";
    case QOQ_ERR_INVALID_ARG: return "invalid argument (shape, alignment, pointer or workspace size)";
    case QOQ_ERR_UNSUPPORTED: return "unsupported device (needs compute capability 10.0, sm_100a)";
    case QOQ_ERR_CUDA: return "CUDA runtime or launch error";
    case QOQ_ERR_TIMEOUT: return "a bounded device wait ran out; outputs of that call are undefined";
    case QOQ_ERR_SCRATCH_TOO_SMALL: return "shape needs more scratch than the built-in no-alloc buffer holds";
    default: return "unknown status";
    }
}

size_t qoq_packed_weight_bytes(int N, int K, int group_size)
{
    if (!valid_nk(N, K) || !valid_group(K, group_size)) return 0;
    return (size_t)(N / qoq::kPanelRows) * (size_t)(K / qoq::kBlockK) * (size_t)qoq::chunk_stride(group_size);
}

int qoq_pack_weights(const float *W, int N, int K, int group_size, uint8_t *Wp, uint16_t *s_c, uint8_t *s_g,
                     uint8_t *zs, uint8_t *z_dbg, uint8_t *q_dbg, void *stream)
{
    if (!valid_nk(N, K) || !valid_group(K, group_size)) return QOQ_ERR_INVALID_ARG;
    if (!W || !Wp || !s_c || !s_g || !zs) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(Wp) || !aligned16(s_c) || !aligned16(s_g) || !aligned16(zs) ||
        (q_dbg && !aligned16(q_dbg)))
        return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(
        qoq::launch_pack(W, N, K, group_size, Wp, s_c, s_g, zs, z_dbg, q_dbg, (cudaStream_t)stream));
}

int qoq_pack_weights_gate_up(const float *W, int N, int K, int group_size, uint8_t *Wp, uint16_t *s_c,
                             uint8_t *s_g, uint8_t *zs, void *stream)
{
    if (!valid_nk(N, K) || !valid_group(K, group_size)) return QOQ_ERR_INVALID_ARG;
    if (!W || !Wp || !s_c || !s_g || !zs) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(Wp) || !aligned16(s_c) || !aligned16(s_g) || !aligned16(zs))
        return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_pack(W, N, K, group_size, Wp, s_c, s_g, zs, nullptr, nullptr,
                                      (cudaStream_t)stream, true));
}

int qoq_quant_act_per_token(const uint16_t *X, int M, int K, int8_t *X8, uint16_t *s_x, int32_t *rowsum,
                            void *stream)
{
    if (M < 0 || M > kMaxM || K < 128 || K > kMaxK || K % 128 != 0) return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X || !X8 || !s_x || !aligned16(X) || !aligned16(X8) || !aligned16(s_x) ||
        (rowsum && (reinterpret_cast<uintptr_t>(rowsum) & 3u)))
        return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_act_quant(X, M, K, X8, s_x, rowsum, (cudaStream_t)stream));
}

size_t qoq_gemm_workspace_bytes(int M, int N, int K, int group_size)
{
    if (M < 1 || M > kMaxM || !valid_nk(N, K) || !valid_group(K, group_size)) return 0;
    if (!qoq::gemm_shape_supported(M, N, K)) return 0;
    return qoq::gemm_workspace_bytes(M, N, K);
}

int qoq_w4a8_gemm(const int8_t *X8, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                  const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int group_size, uint16_t *Y,
                  int32_t *acc_dbg, void *workspace, size_t workspace_bytes, void *stream)
{
    if (M < 0 || M > kMaxM || !valid_nk(N, K) || !valid_group(K, group_size)) return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X8 || !s_x || !Wp || !s_c || !s_g || !zs || !Y || !workspace) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(X8) || !aligned16(s_x) || !aligned16(Wp) || !aligned16(s_c) || !aligned16(s_g) ||
        !aligned16(zs) || !aligned16(Y) || !aligned16(workspace) || (acc_dbg && !aligned16(acc_dbg)))
        return QOQ_ERR_INVALID_ARG;
    if (!qoq::gemm_shape_supported(M, N, K)) return QOQ_ERR_INVALID_ARG;
    if (workspace_bytes < qoq::gemm_workspace_bytes(M, N, K)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    int tmap_status = 0;
    cudaError_t e = qoq::launch_gemm(X8, s_x, Wp, s_c, s_g, zs, M, N, K, group_size, Y, acc_dbg, workspace,
                                     qoq::gemm_a_in_tmem(), (cudaStream_t)stream, &tmap_status);
    if (tmap_status == -1) return QOQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

int qoq_w4a8_gemm_fused(const int8_t *X8, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                        const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int group_size, int epilogue,
                        const uint16_t *residual, uint16_t *Y, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    if (M < 0 || M > kMaxM || !valid_nk(N, K) || !valid_group(K, group_size)) return QOQ_ERR_INVALID_ARG;
    if (epilogue != QOQ_EPILOGUE_NONE && epilogue != QOQ_EPILOGUE_RESIDUAL && epilogue != QOQ_EPILOGUE_SILU_MUL)
        return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X8 || !s_x || !Wp || !s_c || !s_g || !zs || !Y || !workspace) return QOQ_ERR_INVALID_ARG;
    if (epilogue == QOQ_EPILOGUE_RESIDUAL && (!residual || !aligned16(residual))) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(X8) || !aligned16(s_x) || !aligned16(Wp) || !aligned16(s_c) || !aligned16(s_g) ||
        !aligned16(zs) || !aligned16(Y) || !aligned16(workspace))
        return QOQ_ERR_INVALID_ARG;
    if (!qoq::gemm_shape_supported(M, N, K)) return QOQ_ERR_INVALID_ARG;
    if (workspace_bytes < qoq::gemm_workspace_bytes(M, N, K)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    int tmap_status = 0;
    cudaError_t e = qoq::launch_gemm(X8, s_x, Wp, s_c, s_g, zs, M, N, K, group_size, Y, nullptr, workspace,
                                     qoq::gemm_a_in_tmem(), (cudaStream_t)stream, &tmap_status, nullptr, epilogue,
                                     epilogue == QOQ_EPILOGUE_RESIDUAL ? residual : nullptr);
    if (tmap_status == -1) return QOQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

int qoq_w4a8_gemm_i32(const int8_t *X8, int ldx, const uint8_t *Wp, const uint8_t *s_g, const uint8_t *zs, int M,
                      int N, int K, int group_size, int32_t *acc, void *workspace, size_t workspace_bytes,
                      void *stream)
{
    if (M < 0 || M > kMaxM || !valid_nk(N, K) || !valid_group(K, group_size)) return QOQ_ERR_INVALID_ARG;
    if (ldx < K || ldx % 16 != 0) return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X8 || !Wp || !s_g || !zs || !acc || !workspace) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(X8) || !aligned16(Wp) || !aligned16(s_g) || !aligned16(zs) || !aligned16(acc) ||
        !aligned16(workspace))
        return QOQ_ERR_INVALID_ARG;
    if (!qoq::gemm_shape_supported(M, N, K)) return QOQ_ERR_INVALID_ARG;
    if (workspace_bytes < qoq::gemm_workspace_bytes(M, N, K)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    int tmap_status = 0;
    // no scales are read and no FP16 output is written: acc receives the sums
    cudaError_t e = qoq::launch_gemm(X8, nullptr, Wp, nullptr, s_g, zs, M, N, K, group_size, nullptr, acc,
                                     workspace, qoq::gemm_a_in_tmem(), (cudaStream_t)stream, &tmap_status, nullptr,
                                     qoq::kEpiI32, nullptr, ldx);
    if (tmap_status == -1) return QOQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

int qoq_epilogue_i32(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c, int M, int N, uint16_t *Y,
                     void *stream)
{
    if (M < 0 || M > kMaxM || N < 128 || N > kMaxN || N % 128 != 0) return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!acc || !s_x || !s_c || !Y || !aligned16(acc) || !aligned16(s_c) || !aligned16(Y))
        return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_epilogue_i32(acc, s_x, s_c, M, N, Y, (cudaStream_t)stream));
}

int qoq_quantize_weights_w8(const float *W, int N, int K, int8_t *W8, uint16_t *s_w, void *stream)
{
    if (!valid_nk(N, K)) return QOQ_ERR_INVALID_ARG;
    if (!W || !W8 || !s_w || !aligned16(W) || !aligned16(W8) || !aligned16(s_w)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_quantize_w8(W, N, K, W8, s_w, (cudaStream_t)stream));
}

int qoq_w8a8_gemm(const int8_t *X8, const uint16_t *s_x, const int8_t *W8, const uint16_t *s_w, int M, int N, int K,
                  uint16_t *Y, int32_t *acc_dbg, void *workspace, size_t workspace_bytes, void *stream)
{
    if (M < 0 || M > kMaxM || !valid_nk(N, K)) return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X8 || !s_x || !W8 || !s_w || !Y || !workspace) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(X8) || !aligned16(s_x) || !aligned16(W8) || !aligned16(s_w) || !aligned16(Y) ||
        !aligned16(workspace) || (acc_dbg && !aligned16(acc_dbg)))
        return QOQ_ERR_INVALID_ARG;
    if (!qoq::gemm_shape_supported(M, N, K)) return QOQ_ERR_INVALID_ARG;
    if (workspace_bytes < qoq::gemm_workspace_bytes(M, N, K)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    int tmap_status = 0;
    cudaError_t e = qoq::launch_gemm(X8, s_x, nullptr, s_w, nullptr, nullptr, M, N, K, 128, Y, acc_dbg, workspace,
                                     false, (cudaStream_t)stream, &tmap_status, nullptr, qoq::kEpiPlain, nullptr, 0,
                                     W8);
    if (tmap_status == -1) return QOQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

static bool valid_kv4(int B, int Hq, int Hkv, int L, int d)
{
    if (B < 0 || B > (1 << 16) || Hkv < 1 || Hkv > 1024 || Hq < Hkv || Hq % Hkv != 0 || d != 128) return false;
    const int G = Hq / Hkv;
    return (G == 1 || G == 2 || G == 4 || G == 8) && L >= 1 && L <= (1 << 20);
}

int qoq_kv4_cache_quantize(const uint16_t *K, const uint16_t *V, int B, int Hkv, int L, int d, uint8_t *K4,
                           uint8_t *V4, uint16_t *lam, uint16_t *s_k, uint16_t *s_v, void *stream)
{
    if (!valid_kv4(B, Hkv, Hkv, L, d)) return QOQ_ERR_INVALID_ARG;
    if (B == 0) return QOQ_OK;
    if (!K || !V || !K4 || !V4 || !lam || !s_k || !s_v) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(K) || !aligned16(V) || !aligned16(K4) || !aligned16(V4) || !aligned16(lam) || !aligned16(s_k) ||
        !aligned16(s_v))
        return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_kv4_cache(K, V, B, Hkv, L, K4, V4, lam, s_k, s_v, (cudaStream_t)stream));
}

size_t qoq_kv4_attention_workspace_bytes(int B, int Hq, int Hkv, int L, int d)
{
    if (!valid_kv4(B, Hq, Hkv, L, d) || B == 0) return 0;
    return qoq::kv4_workspace_bytes(B, Hq, Hkv, L);
}

int qoq_kv4_decode_attention(const uint16_t *q, const uint8_t *K4, const uint8_t *V4, const uint16_t *lam,
                             const uint16_t *s_k, const uint16_t *s_v, int B, int Hq, int Hkv, int L, int d,
                             uint16_t *out, void *workspace, size_t workspace_bytes, void *stream)
{
    if (!valid_kv4(B, Hq, Hkv, L, d)) return QOQ_ERR_INVALID_ARG;
    if (B == 0) return QOQ_OK;
    if (!q || !K4 || !V4 || !lam || !s_k || !s_v || !out || !workspace) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(K4) || !aligned16(V4) || !aligned16(lam) || !aligned16(s_k) || !aligned16(s_v) ||
        !aligned16(out) || !aligned16(workspace))
        return QOQ_ERR_INVALID_ARG;
    if (workspace_bytes < qoq::kv4_workspace_bytes(B, Hq, Hkv, L)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(
        qoq::launch_kv4_attention(q, K4, V4, lam, s_k, s_v, B, Hq, Hkv, L, out, workspace, (cudaStream_t)stream));
}

int qoq_w4a8_linear(const uint16_t *X, int M, int N, int K, int group_size, const uint8_t *Wp,
                    const uint16_t *s_c, const uint8_t *s_g, const uint8_t *zs, int8_t *X8, uint16_t *s_x,
                    uint16_t *Y, void *workspace, size_t workspace_bytes, void *stream)
{
    if (M < 0 || M > kMaxM || !valid_nk(N, K) || !valid_group(K, group_size) || K > kMaxK)
        return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X || !X8 || !s_x || !Wp || !s_c || !s_g || !zs || !Y || !workspace) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(X8) || !aligned16(s_x) || !aligned16(Wp) || !aligned16(s_c) ||
        !aligned16(s_g) || !aligned16(zs) || !aligned16(Y) || !aligned16(workspace))
        return QOQ_ERR_INVALID_ARG;
    if (!qoq::gemm_shape_supported(M, N, K)) return QOQ_ERR_INVALID_ARG;
    if (workspace_bytes < qoq::gemm_workspace_bytes(M, N, K)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    int tmap_status = 0;
    // The quantizer and the GEMM as two kernels (default), or, up to one
    // row per SM and when selected, one GEMM launch that quantizes its own
    // input (same results).
    const bool in_kernel = g_linear_in_kernel_quant.load() != 0 && M <= qoq::kFusedMaxRows;
    if (!in_kernel) {
        const cudaError_t eq = qoq::launch_act_quant(X, M, K, X8, s_x, nullptr, (cudaStream_t)stream);
        if (eq != cudaSuccess) return from_cuda(eq);
    }
    cudaError_t e = qoq::launch_gemm(X8, s_x, Wp, s_c, s_g, zs, M, N, K, group_size, Y, nullptr, workspace,
                                     qoq::gemm_a_in_tmem(), (cudaStream_t)stream, &tmap_status,
                                     in_kernel ? X : nullptr);
    if (tmap_status == -1) return QOQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

int qoq_dequant_weights_i8(const uint8_t *Wp, const uint8_t *s_g, const uint8_t *zs, int N, int K, int group_size,
                           int8_t *W8hat, void *stream)
{
    if (!valid_nk(N, K) || !valid_group(K, group_size)) return QOQ_ERR_INVALID_ARG;
    if (!Wp || !s_g || !zs || !W8hat || !aligned16(Wp) || !aligned16(W8hat)) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_dequant(Wp, s_g, zs, N, K, group_size, W8hat, (cudaStream_t)stream));
}

int qoq_set_gemm_a_in_tmem(int enable)
{
    if (enable != 0 && enable != 1) return QOQ_ERR_INVALID_ARG;
    g_a_in_tmem.store(enable);
    return QOQ_OK;
}

int qoq_selftest_wait_timeout(unsigned long long timeout_ns, void *stream)
{
    if (timeout_ns < 1000ull || timeout_ns > 100000000ull) return QOQ_ERR_INVALID_ARG;
    const int dev = check_device();
    if (dev != QOQ_OK) return dev;
    return from_cuda(qoq::launch_stuck_wait(timeout_ns, (cudaStream_t)stream));
}

int qoq_set_gemm_cta_pairs(int enable)
{
    if (enable != 0 && enable != 1) return QOQ_ERR_INVALID_ARG;
    qoq::set_cta_pairs(enable != 0);
    return QOQ_OK;
}

int qoq_set_gemm_half_ctas(int enable)
{
    if (enable != 0 && enable != 1) return QOQ_ERR_INVALID_ARG;
    qoq::set_half_ctas(enable != 0);
    return QOQ_OK;
}

int qoq_set_gemm_gemv(int enable)
{
    if (enable != 0 && enable != 1) return QOQ_ERR_INVALID_ARG;
    qoq::set_gemv(enable != 0);
    return QOQ_OK;
}

int qoq_set_gemm_narrow_tiles(int enable)
{
    if (enable != 0 && enable != 1) return QOQ_ERR_INVALID_ARG;
    qoq::set_narrow_tiles(enable != 0);
    return QOQ_OK;
}

int qoq_set_linear_in_kernel_quant(int enable)
{
    if (enable != 0 && enable != 1) return QOQ_ERR_INVALID_ARG;
    g_linear_in_kernel_quant.store(enable);
    return QOQ_OK;
}


int qoq_device_error(void *stream)
{
    int v = 0, w = 0;
    if (qoq::read_and_clear_device_error((cudaStream_t)stream, &v) != cudaSuccess) return QOQ_ERR_CUDA;
    if (qoq::read_and_clear_kv4_error(&w) != cudaSuccess) return QOQ_ERR_CUDA;
    return (v || w) ? QOQ_ERR_TIMEOUT : QOQ_OK;
}

}  // extern "C"
