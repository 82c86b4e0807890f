// qlin_noalloc.cu -- w8a8_linear_noalloc: the W8A8 layer with its scratch in a
// fixed buffer that lives inside libqlin.so, for callers that cannot hand the
// library any device memory of their own.
//
// Who needs it: hosts that must not allocate device memory on the call path
// (a runtime that reserved all GPU memory up front for its own pool, a
// latency-critical serving loop that forbids allocator calls after start-up,
// or plain C callers with no allocator to borrow scratch from).  w8a8_linear
// needs M*K bytes of int8 activations plus M floats of scales between its two
// kernels; this variant keeps them in the static array below instead of a
// caller workspace.
#include <mutex>

#include "qlin_common.cuh"

namespace qlin {
namespace {

// Capacity of the built-in scratch (qx int8 [M][K], 256-byte aligned, then
// s_x fp32 [M]).  Each GPU that loads the library holds this memory until the
// process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices];

// Device address of the scratch array on the current device, after the same
// sm_100 check every entry point makes.  Looked up on the first call made with
// that device current (kept only once the lookup succeeded, so a failed first
// attempt is retried on the next call); the host-side symbol itself is only a
// stand-in and must never reach a kernel.
qlin_status scratch_address(void** out)
{
    DeviceInfo info;
    const qlin_status s = current_device(info);
    if (s != QLIN_OK)
        return s;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QLIN_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return QLIN_ERR_CUDA;
        }
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return QLIN_OK;
}

}  // namespace
}  // namespace qlin

extern "C" {

qlin_status w8a8_linear_noalloc(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const int8_t* w,
                                const float* scale_w, int64_t N, const void* bias, void* y, void* stream)
{
    if (!x || !w || !scale_w || !y || M <= 0 || N <= 0 || K <= 0)
        return QLIN_ERR_INVALID_ARG;
    // the problem must fit in the built-in scratch; nothing is launched otherwise
    const size_t need = qlin_workspace_size(QLIN_OP_W8A8, M, N, K, 0, 0);
    if (need > qlin::kNoAllocScratchBytes)
        return QLIN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const qlin_status s = qlin::scratch_address(&scratch);
    if (s != QLIN_OK)
        return s;
    // qx and s_x are fully rewritten by the activation quantiser before the GEMM
    // reads them, so nothing needs clearing between calls.
    return w8a8_linear(x, x_dt, M, K, w, scale_w, N, bias, y, scratch, qlin::kNoAllocScratchBytes, stream);
}

}  // extern "C"
