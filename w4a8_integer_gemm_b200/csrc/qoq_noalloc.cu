// qoq_noalloc.cu -- a GEMM entry point that allocates nothing.
//
// qoq_w4a8_gemm needs a caller-provided scratch workspace for the INT32
// partial sums of output tiles whose K loop is split across SMs.  Some
// callers cannot provide one: code running inside an inference engine's
// execute/enqueue step, where allocating is forbidden or would synchronize
// the device (cudaFree waits for all work; cudaMalloc can too), plug-ins
// that have no allocator of their own, and real-time paths that must never
// touch the allocator.  For them, qoq_w4a8_gemm_noalloc runs the same kernel
// with its scratch in a fixed buffer that lives in this library's device
// image.  The buffer is a file-scope __device__ array: every GPU that loads
// the library holds its 16 MiB until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qoq.h"
#include "qoq_internal.h"

namespace {

constexpr size_t kScratchBytes = QOQ_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// On the host, g_noalloc_scratch names a host-side stand-in, not device
// memory: the kernel must be given the address the runtime reports for the
// current device.  Looked up once per device, with that device current.
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return QOQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QOQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return QOQ_OK;
}

}  // namespace

extern "C" {

int qoq_w4a8_gemm_noalloc(const int8_t *X8, const uint16_t *s_x, const uint8_t *Wp, const uint16_t *s_c,
                          const uint8_t *s_g, const uint8_t *zs, int M, int N, int K, int group_size,
                          uint16_t *Y, void *stream)
{
    // the same shape and pointer checks as qoq_w4a8_gemm (shared code)
    if (M < 0 || M > (1 << 24) || !qoq::valid_nk(N, K) || !qoq::valid_group(K, group_size))
        return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (!X8 || !s_x || !Wp || !s_c || !s_g || !zs || !Y) return QOQ_ERR_INVALID_ARG;
    if (!qoq::aligned16(X8) || !qoq::aligned16(s_x) || !qoq::aligned16(Wp) || !qoq::aligned16(s_c) ||
        !qoq::aligned16(s_g) || !qoq::aligned16(zs) || !qoq::aligned16(Y))
        return QOQ_ERR_INVALID_ARG;
    const size_t need = qoq_gemm_workspace_bytes(M, N, K, group_size);
    if (need == 0) return QOQ_ERR_INVALID_ARG;
    if (need > kScratchBytes) return QOQ_ERR_SCRATCH_TOO_SMALL;
    const int dev = qoq::check_device();
    if (dev != QOQ_OK) return dev;

    void *scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != QOQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // The split-tile counters must start at zero.  Completed calls leave
    // them at zero, but a call that timed out may not have, so clear them
    // every time (a memset, not an allocation).
    if (cudaMemsetAsync(scratch, 0, qoq::kCounterBytes, s) != cudaSuccess) return QOQ_ERR_CUDA;
    int tmap_status = 0;
    const cudaError_t e = qoq::launch_gemm(X8, s_x, Wp, s_c, s_g, zs, M, N, K, group_size, Y, nullptr, scratch,
                                           qoq::gemm_a_in_tmem(), s, &tmap_status);
    if (tmap_status == -1) return QOQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? QOQ_OK : QOQ_ERR_CUDA;
}

}  // extern "C"
