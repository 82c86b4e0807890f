// qlin_abi.cu -- the extern "C" boundary of libqlin.so: argument validation,
// device checks, workspace sizing and dispatch to the kernel launchers.
// No exception crosses this file's functions; every failure is a qlin_status.
#include <mutex>

#include "qlin_common.cuh"

namespace qlin {

// Device status word: kernels OR kStatusTimeout into it when a bounded wait
// gives up; qlin_get_device_status() reads and clears it.
__device__ unsigned g_device_status;

// k_quant.cu: the per-row int8 quantiser launched as a programmatic dependent of the stream's
// previous kernel (its CTAs may be placed early and wait before touching memory); it also lets
// the next kernel start its prologue early.
cudaError_t launch_quantize_int8_rows_dependent(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, int8_t* q,
                                                float* scale, cudaStream_t st, const DeviceInfo& dev);
// k_tc_gemm.cu: the CTA tile of the int8 tcgen05 GEMM, mt sub-tiles of 128 tokens by bn columns.
void tc_tile_shape(TcOp op, int64_t M, int64_t N, int64_t sms, int& mt, int& bn);

namespace {

constexpr int kMaxDevices = 64;

struct DeviceSlot {
    std::once_flag once;
    qlin_status state = QLIN_ERR_DEVICE;
    DeviceInfo info = {0, nullptr};
};

DeviceSlot g_slots[kMaxDevices];

}  // namespace

// Checks (once per device) that the current device is an sm_100 part, and
// records its SM count and the address of the status word.  Must run with
// that device current, outside stream capture (the first call per device).
qlin_status current_device(DeviceInfo& out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QLIN_ERR_DEVICE;
    }
    DeviceSlot& slot = g_slots[dev];
    std::call_once(slot.once, [&slot, dev]() {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
            cudaGetLastError();
            slot.state = QLIN_ERR_DEVICE;
            return;
        }
        if (prop.major != 10 || prop.minor != 0) {
            slot.state = QLIN_ERR_DEVICE;
            return;
        }
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            slot.state = QLIN_ERR_CUDA;
            return;
        }
        slot.info.sm_count = prop.multiProcessorCount;
        slot.info.status = static_cast<unsigned*>(p);
        slot.state = QLIN_OK;
    });
    out = slot.info;
    return slot.state;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(qlin_dtype d) { return d == QLIN_F32 || d == QLIN_BF16 || d == QLIN_F16; }
size_t dtype_size(qlin_dtype d) { return d == QLIN_F32 ? 4 : 2; }
bool bits_ok(int b) { return (b >= 1 && b <= 6) || b == 8; }
bool group_ok(int g) { return g == 32 || g == 64 || g == 128; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

qlin_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess)
        return QLIN_OK;
    cudaGetLastError();  // clear a non-sticky launch error
    return e == cudaErrorNotSupported ? QLIN_ERR_UNSUPPORTED : QLIN_ERR_CUDA;
}

// Shape/type rules common to the affine-format calls.
qlin_status check_affine(int64_t N, int64_t K, int bits, int g, qlin_dtype p_dt)
{
    if (N <= 0 || K <= 0 || N > INT32_MAX || K > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!bits_ok(bits) || !group_ok(g) || !dtype_ok(p_dt))
        return QLIN_ERR_UNSUPPORTED;
    if (K % g != 0)
        return QLIN_ERR_INVALID_ARG;
    return QLIN_OK;
}

}  // namespace
}  // namespace qlin

using namespace qlin;

namespace qlin {
// self-test of the bounded-wait path (k_selftest.cu): one wait that runs out after limit_ns.
cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t st, const DeviceInfo& dev);
}  // namespace qlin

extern "C" {

const char* qlin_status_string(qlin_status s)
{
    switch (s) {
    case QLIN_OK: return "QLIN_OK";
    case QLIN_ERR_INVALID_ARG: return "QLIN_ERR_INVALID_ARG: invalid argument";
    case QLIN_ERR_UNSUPPORTED: return "QLIN_ERR_UNSUPPORTED: unsupported bits/group/dtype combination";
    case QLIN_ERR_MISALIGNED: return "QLIN_ERR_MISALIGNED: pointer or row pitch not 16-byte aligned";
    case QLIN_ERR_DEVICE: return "QLIN_ERR_DEVICE: no sm_100 CUDA device current";
    case QLIN_ERR_CUDA: return "QLIN_ERR_CUDA: CUDA runtime error";
    case QLIN_ERR_TIMEOUT: return "QLIN_ERR_TIMEOUT: a bounded device wait expired";
    case QLIN_ERR_WORKSPACE: return "QLIN_ERR_WORKSPACE: workspace missing or too small";
    }
    return "QLIN_ERR_?: unknown status";
}

int qlin_version(void) { return 1 * 10000 + 0 * 100 + 0; }

qlin_status qlin_int8_gemm_tile(qlin_op op, int64_t M, int64_t N, int sm_count, int* tokens, int* columns)
{
    if ((op != QLIN_OP_W8A8 && op != QLIN_OP_W4A8) || M < 1 || N < 1 || sm_count < 1 || !tokens || !columns)
        return QLIN_ERR_INVALID_ARG;
    int mt = 1, bn = 256;
    tc_tile_shape(op == QLIN_OP_W4A8 ? TC_W4A8 : TC_W8A8, M, N, sm_count, mt, bn);
    *tokens = 128 * mt;
    *columns = bn;
    return QLIN_OK;
}

size_t qlin_workspace_size(qlin_op op, int64_t M, int64_t N, int64_t K, int bits, int group_size)
{
    if (M <= 0 || K <= 0)
        return 0;
    switch (op) {
    case QLIN_OP_W8A8:
    case QLIN_OP_W4A8: return align256((size_t)M * (size_t)K) + align256((size_t)M * 4);
    case QLIN_OP_PERGROUP:
        return (N > 0 && (group_size == 64 || group_size == 128 || group_size == 256) && K % group_size == 0)
                   ? tc_affine_workspace(M, N, K, group_size)
                   : 0;
    case QLIN_OP_MATMUL:
        // the tensor-core prefill (M > 16, 4-bit codes): fp16 x and group parameters, scales
        return (M > 16 && bits == 4 && N > 0 && group_size > 0 && K % group_size == 0)
                   ? tc_affine_workspace(M, N, K, group_size)
                   : 0;
    default: return 0;
    }
}

qlin_status qlin_quantize(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int bits, int group_size,
                          uint32_t* codes, void* scales, void* biases, qlin_dtype param_dt, void* stream)
{
    if (!w || !codes || !scales || !biases)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(w_dt))
        return QLIN_ERR_UNSUPPORTED;
    qlin_status s = check_affine(N, K, bits, group_size, param_dt);
    if (s != QLIN_OK)
        return s;
    DeviceInfo dev;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    return from_cuda(launch_affine_quantize(w, w_dt, N, K, bits, group_size, codes, scales, biases, param_dt,
                                            static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_dequantize(const uint32_t* codes, const void* scales, const void* biases, qlin_dtype param_dt,
                            int64_t N, int64_t K, int bits, int group_size, void* w_out, qlin_dtype out_dt,
                            void* stream)
{
    if (!codes || !scales || !biases || !w_out)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(out_dt))
        return QLIN_ERR_UNSUPPORTED;
    qlin_status s = check_affine(N, K, bits, group_size, param_dt);
    if (s != QLIN_OK)
        return s;
    // one word's outputs go out as 8- or 16-byte vector stores
    if (!aligned16(w_out) || (reinterpret_cast<uintptr_t>(codes) & 3u) != 0)
        return QLIN_ERR_MISALIGNED;
    DeviceInfo dev;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    return from_cuda(launch_affine_dequantize(codes, scales, biases, param_dt, N, K, bits, group_size, w_out, out_dt,
                                              static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_matmul(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const uint32_t* codes,
                        const void* scales, const void* biases, qlin_dtype param_dt, int64_t N, int bits,
                        int group_size, const void* bias, void* y, void* workspace, size_t ws_bytes, void* stream)
{
    if (!x || !codes || !scales || !biases || !y || M <= 0 || M > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(x_dt))
        return QLIN_ERR_UNSUPPORTED;
    qlin_status s = check_affine(N, K, bits, group_size, param_dt);
    if (s != QLIN_OK)
        return s;
    // the specialized paths: power-of-two widths (not 2 bits in groups of 32), fp32 / bf16 operands,
    // TMA-loaded rows (16-byte pitch); the tensor-core prefill also takes fp16 x.  Everything else
    // runs the general decode kernel, which needs 4-byte aligned codes and 16-byte x rows.
    const bool tma_rows = aligned16(codes) && (K * bits / 8) % 16 == 0;
    const bool prefill = M > 16 && bits == 4 && param_dt == QLIN_BF16 && tma_rows;
    const bool special = (bits == 2 || bits == 4 || bits == 8) && !(bits == 2 && group_size == 32) &&
                         x_dt != QLIN_F16 && param_dt != QLIN_F16 && tma_rows;
    if (!aligned16(x) || (K * (int64_t)dtype_size(x_dt)) % 16 != 0 || (reinterpret_cast<uintptr_t>(codes) & 3u) != 0)
        return QLIN_ERR_MISALIGNED;
    DeviceInfo dev;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    if (prefill) {
        const size_t need = qlin_workspace_size(QLIN_OP_MATMUL, M, N, K, bits, group_size);
        if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return QLIN_ERR_WORKSPACE;
        TcGemmArgs t = {};
        t.M = M;
        t.N = N;
        t.K = K;
        t.a = x;
        t.b = codes;
        t.out = y;
        t.bias = bias;
        t.scales = scales;
        t.biases = biases;
        t.g = group_size;
        t.bits = bits;
        t.x_dt = x_dt;
        t.workspace = workspace;
        return from_cuda(launch_tc_affine(t, static_cast<cudaStream_t>(stream), dev));
    }
    AffineGemvArgs a;
    a.x = x;
    a.x_dt = x_dt;
    a.M = M;
    a.K = K;
    a.N = N;
    a.codes = codes;
    a.scales = scales;
    a.biases = biases;
    a.p_dt = param_dt;
    a.bits = bits;
    a.g = group_size;
    a.bias = bias;
    a.y = y;
    return from_cuda(special ? launch_affine_gemv(a, static_cast<cudaStream_t>(stream), dev)
                             : launch_affine_gemv_any(a, static_cast<cudaStream_t>(stream), dev));
}

qlin_status bitlinear_matmul(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const uint8_t* packed, int64_t N,
                             const float* weight_scale, int invert_weight_scale, const void* bias, void* y,
                             void* stream)
{
    if (!x || !packed || !weight_scale || !y || M <= 0 || K <= 0 || N <= 0 || M > INT32_MAX || K > INT32_MAX ||
        N > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (N % 4 != 0 || K % 16 != 0)
        return QLIN_ERR_INVALID_ARG;
    if (x_dt != QLIN_BF16)
        return QLIN_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(packed))
        return QLIN_ERR_MISALIGNED;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    BitlinearArgs a;
    a.x = x;
    a.x_dt = x_dt;
    a.M = M;
    a.K = K;
    a.N = N;
    a.packed = packed;
    a.weight_scale = weight_scale;
    a.invert = invert_weight_scale ? 1 : 0;
    a.bias = bias;
    a.y = y;
    if (M > 16)  // prefill: the tcgen05 GEMM reads the packed weights once per 256-token tile
        return from_cuda(launch_tc_bitlinear(a, static_cast<cudaStream_t>(stream), dev));
    return from_cuda(launch_bitlinear_gemv(a, static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_quantize_int8_rows(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, int8_t* q, float* scale,
                                    void* stream)
{
    if (!w || !q || !scale || R <= 0 || C <= 0 || R > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(w_dt))
        return QLIN_ERR_UNSUPPORTED;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    return from_cuda(
        launch_quantize_int8_rows(w, w_dt, R, C, q, scale, static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_pack_int4_cols(const void* w, qlin_dtype w_dt, int64_t K, int64_t N, uint8_t* packed, float* scale,
                                void* stream)
{
    if (!w || !packed || !scale || K <= 0 || N <= 0 || K % 2 != 0 || N > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(w_dt))
        return QLIN_ERR_UNSUPPORTED;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    return from_cuda(launch_pack_int4_cols(w, w_dt, K, N, packed, scale, static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_quantize_weight_int8(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, double clip_percentile,
                                     int8_t* q, float* scale, void* stream)
{
    if (!w || !q || !scale || R <= 0 || C <= 0 || R > INT32_MAX || C > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(w_dt))
        return QLIN_ERR_UNSUPPORTED;
    if (clip_percentile > 100.0 || clip_percentile != clip_percentile)
        return QLIN_ERR_INVALID_ARG;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    if (clip_percentile < 0.0)  // no clip: the absmax rule
        return from_cuda(
            launch_quantize_int8_rows(w, w_dt, R, C, q, scale, static_cast<cudaStream_t>(stream), dev));
    if (C > 32768)  // the row is held in shared memory
        return QLIN_ERR_UNSUPPORTED;
    // numpy converts the percentile to the row's float32 before dividing by 100
    return from_cuda(launch_quantize_weight_int8_clip(w, w_dt, R, C, (float)clip_percentile, q, scale,
                                                      static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_quantize_int8_groups(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int group_size,
                                     int8_t* q, float* scale_w, void* stream)
{
    if (!w || !q || !scale_w || N <= 0 || K <= 0 || N > INT32_MAX || K > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(w_dt) || !(group_size == 64 || group_size == 128 || group_size == 256))
        return QLIN_ERR_UNSUPPORTED;
    if (K % group_size != 0)
        return QLIN_ERR_INVALID_ARG;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    return from_cuda(
        launch_quantize_int8_groups(w, w_dt, N, K, group_size, q, scale_w, static_cast<cudaStream_t>(stream), dev));
}

qlin_status pergroup_linear(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const int8_t* w,
                            const float* scale_w, int64_t N, int group_size, const void* bias, void* y,
                            void* workspace, size_t ws_bytes, void* stream)
{
    if (!x || !w || !scale_w || !y || M <= 0 || N <= 0 || K <= 0 || M > INT32_MAX || N > INT32_MAX ||
        K > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (!dtype_ok(x_dt) || !(group_size == 64 || group_size == 128 || group_size == 256))
        return QLIN_ERR_UNSUPPORTED;
    if (K % group_size != 0)
        return QLIN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || K % 16 != 0)
        return QLIN_ERR_MISALIGNED;
    const size_t need = qlin_workspace_size(QLIN_OP_PERGROUP, M, N, K, 8, group_size);
    if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return QLIN_ERR_WORKSPACE;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    if (M == 1 && x_dt == QLIN_BF16) {  // the FP-activation branch as a weight-resident decode GEMV
        AffineGemvArgs a;
        a.x = x;
        a.x_dt = x_dt;
        a.M = M;
        a.K = K;
        a.N = N;
        a.codes = reinterpret_cast<const uint32_t*>(w);
        a.scales = scale_w;
        a.biases = scale_w;  // not read
        a.p_dt = QLIN_F32;
        a.bits = 8;
        a.g = group_size;
        a.bias = bias;
        a.y = y;
        a.pergroup = 1;
        const cudaError_t e = launch_affine_dec(a, static_cast<cudaStream_t>(stream), dev);
        if (e != cudaErrorNotSupported)
            return from_cuda(e);
    }
    TcGemmArgs t = {};
    t.M = M;
    t.N = N;
    t.K = K;
    t.a = x;
    t.b = w;
    t.out = y;
    t.bias = bias;
    t.scales = scale_w;
    t.biases = nullptr;
    t.g = group_size;
    t.bits = 8;
    t.x_dt = x_dt;
    t.pergroup = 1;
    t.workspace = workspace;
    return from_cuda(launch_tc_affine(t, static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_int8_matmul_int32(const int8_t* a, const int8_t* b, int64_t M, int64_t N, int64_t K, int32_t* c,
                                   void* stream)
{
    if (!a || !b || !c || M <= 0 || N <= 0 || K <= 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (K % 16 != 0)
        return QLIN_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(c))
        return QLIN_ERR_MISALIGNED;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    TcGemmArgs t = {};
    t.M = M;
    t.N = N;
    t.K = K;
    t.a = a;
    t.b = b;
    t.out = c;
    return from_cuda(launch_tc_gemm(TC_I8_RAW, t, static_cast<cudaStream_t>(stream), dev));
}

namespace {

// Shared body of the W8A8 / W4A8 layers: per-token int8 activation quant
// into the workspace, then the tcgen05 GEMM with the scaled epilogue.
qlin_status int_linear(TcOp op, const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const void* w,
                       const float* scale_w, int64_t N, const void* bias, void* y, void* workspace, size_t ws_bytes,
                       void* stream)
{
    if (!x || !w || !scale_w || !y || M <= 0 || N <= 0 || K <= 0 || M > INT32_MAX || N > INT32_MAX ||
        K > INT32_MAX)
        return QLIN_ERR_INVALID_ARG;
    if (op == TC_W4A8 ? (K % 32 != 0 || N % 16 != 0) : (K % 16 != 0))
        return QLIN_ERR_INVALID_ARG;
    if (x_dt != QLIN_BF16 && x_dt != QLIN_F16)  // y and bias take x's 16-bit dtype
        return QLIN_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w) || !aligned16(y))
        return QLIN_ERR_MISALIGNED;
    const size_t need = qlin_workspace_size(op == TC_W4A8 ? QLIN_OP_W4A8 : QLIN_OP_W8A8, M, N, K, 0, 0);
    if (!workspace || ws_bytes < need || !aligned16(workspace))
        return QLIN_ERR_WORKSPACE;
    DeviceInfo dev;
    qlin_status s;
    if ((s = current_device(dev)) != QLIN_OK)
        return s;
    int8_t* qx = static_cast<int8_t*>(workspace);
    float* sx = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256((size_t)M * (size_t)K));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the quantiser lets the next kernel start its prologue (fetching the layer's weights) early;
    // ahead of a tcgen05 GEMM it is also placed early itself, behind the stream's previous kernel
    cudaError_t e = M > 16 ? launch_quantize_int8_rows_dependent(x, x_dt, M, K, qx, sx, st, dev)
                           : launch_quantize_int8_rows(x, x_dt, M, K, qx, sx, st, dev, true);
    if (e != cudaSuccess)
        return from_cuda(e);
    if (M <= 16) {  // decode: weight-streaming GEMV on int8 mma.sync
        W8GemvArgs g;
        g.qx = qx;
        g.s_x = sx;
        g.w = static_cast<const int8_t*>(w);
        g.s_w = scale_w;
        g.bias = bias;
        g.y = y;
        g.M = M;
        g.K = K;
        g.N = N;
        g.out_f16 = x_dt == QLIN_F16;
        return from_cuda(op == TC_W8A8 ? launch_w8_gemv(g, st, dev) : launch_w4_gemv(g, st, dev));
    }
    TcGemmArgs t = {};
    t.M = M;
    t.N = N;
    t.K = K;
    t.a = qx;
    t.b = w;
    t.out = y;
    t.s_x = sx;
    t.s_w = scale_w;
    t.bias = bias;
    t.x_dt = x_dt;
    return from_cuda(launch_tc_gemm(op, t, st, dev));
}

}  // namespace

qlin_status w8a8_linear(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const int8_t* w, const float* scale_w,
                        int64_t N, const void* bias, void* y, void* workspace, size_t ws_bytes, void* stream)
{
    return int_linear(TC_W8A8, x, x_dt, M, K, w, scale_w, N, bias, y, workspace, ws_bytes, stream);
}

qlin_status w4a8_linear(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const uint8_t* packed_w,
                        const float* scale_w, int64_t N, const void* bias, void* y, void* workspace, size_t ws_bytes,
                        void* stream)
{
    return int_linear(TC_W4A8, x, x_dt, M, K, packed_w, scale_w, N, bias, y, workspace, ws_bytes, stream);
}

qlin_status qlin_selftest_wait_timeout(unsigned limit_us, void* stream)
{
    if (limit_us == 0 || limit_us > 2000000u)
        return QLIN_ERR_INVALID_ARG;
    DeviceInfo dev;
    qlin_status s = current_device(dev);
    if (s != QLIN_OK)
        return s;
    return from_cuda(launch_wait_timeout_selftest((unsigned long long)limit_us * 1000ull,
                                                  static_cast<cudaStream_t>(stream), dev));
}

qlin_status qlin_get_device_status(void* stream)
{
    DeviceInfo dev;
    qlin_status s = current_device(dev);
    if (s != QLIN_OK)
        return s;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return QLIN_ERR_CUDA;
    }
    unsigned word = 0;
    if (cudaMemcpy(&word, dev.status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return QLIN_ERR_CUDA;
    }
    if (word != 0) {
        const unsigned zero = 0;
        cudaMemcpy(dev.status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        return QLIN_ERR_TIMEOUT;
    }
    return QLIN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- tensor maps (host)
#include <cudaTypedefs.h>

namespace qlin {

bool encode_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t dim0, uint64_t dim1,
                    uint64_t pitch_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle)
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    if (!fn)
        return false;
    cuuint64_t dims[2] = {dim0, dim1};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box0, box1};
    cuuint32_t estr[2] = {1, 1};
    return fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace qlin
