// k_affine_any.cu -- the MLX affine layer for every code width and dtype the specialized
// decode kernels do not cover: 1, 3, 5 and 6 bits (codes straddling 32-bit words), 2 bits with
// groups of 32, and fp16 activations or group parameters.
//
//   y[m,n] = sum_k x[m,k] * w_hat[n,k] + bias[n],  w_hat[n,k] = fma(q[n,k], s[n,k/g], b[n,k/g])
//   [nuvec-nn QuantizedLinear: forward and dequantized_weight; bits 1..6, 8]
//
// A row's codes are one LSB-first bitstream (code k at bits k*b .. k*b+b-1 of the row's words), so
// eight consecutive codes are b whole bytes.  One warp per RW output rows: lane l takes codes
// 8l .. 8l+7 of each 256-code span, reads the 1-3 words that hold their b bytes (the warp's loads
// cover the span's 32b bytes once), builds w_hat in fp32 exactly as the dequantizer does, and
// multiplies it into up to MT tokens whose 8 x values it reads once per span for all RW rows.
// Memory-bound at small M; this is the general path, the specialized ones are faster.
#include "qlin_common.cuh"

namespace qlin {
namespace {

QLIN_DEV void load_x8(const float* p, float (&v)[8])
{
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
QLIN_DEV void load_x8(const __nv_bfloat16* p, float (&v)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
QLIN_DEV void load_x8(const __half* p, float (&v)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

struct AnyParams {
    const void* x;  // [M][K] of XT, this launch's first token
    const uint32_t* codes;  // [N][K*BITS/32]
    const void* scales;     // [N][K/g] of PT
    const void* biases;
    const void* bias;       // [N] of XT or null
    void* y;                // [M][N] of XT, this launch's first token
    int M, K, N, g;
};

constexpr int kAnyWarps = 8;

template <typename XT, typename PT, int BITS, int MT, int RW>
__global__ void __launch_bounds__(kAnyWarps * 32) affine_any_kernel(const AnyParams p)
{
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nbase = ((int)blockIdx.x * kAnyWarps + warp) * RW;
    if (nbase >= p.N)
        return;  // warp-uniform
    const XT* x = static_cast<const XT*>(p.x);
    const PT* sc = static_cast<const PT*>(p.scales);
    const PT* bi = static_cast<const PT*>(p.biases);
    const int64_t wpr = (int64_t)p.K * BITS / 32;  // words per row
    const int ng = p.K / p.g;
    float acc[MT][RW];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int r = 0; r < RW; ++r)
            acc[m][r] = 0.f;

    for (int base = 0; base < p.K; base += 256) {
        const int k0 = base + 8 * lane;
        if (k0 < p.K) {  // K is a multiple of 32: a lane's eight codes are all in or all out
            // byte offset of the eight codes in the row, the word holding the first, the bit shift
            const int bo = k0 / 8 * BITS;
            const int wi = bo >> 2;
            const int sh = 8 * (bo & 3);
            float wh[RW][8];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int n = nbase + r < p.N ? nbase + r : p.N - 1;  // rows past N compute, never store
                const uint32_t* row = p.codes + (int64_t)n * wpr + wi;
                // the codes' bits sh .. sh + 8 BITS - 1 of row[0..2]; only the words they reach are read
                const uint32_t w0 = __ldg(row);
                const uint32_t w1 = sh + 8 * BITS > 32 ? __ldg(row + 1) : 0u;
                const uint32_t w2 = sh + 8 * BITS > 64 ? __ldg(row + 2) : 0u;
                const uint64_t v = (uint64_t)__funnelshift_r(w0, w1, sh) |
                                   ((uint64_t)__funnelshift_r(w1, w2, sh) << 32);
                const float s = to_float(sc[(int64_t)n * ng + k0 / p.g]);
                const float b = to_float(bi[(int64_t)n * ng + k0 / p.g]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    wh[r][i] = __fmaf_rn((float)((uint32_t)(v >> (BITS * i)) & MASK), s, b);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < p.M) {
                    float xv[8];
                    load_x8(x + (int64_t)m * p.K + k0, xv);
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            acc[m][r] = fmaf(xv[i], wh[r][i], acc[m][r]);
                }
            }
        }
    }
    // warp sums; lane (m * RW + r) % 32 keeps the total of (m, r)
    float keep = 0.f;
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            float t = acc[m][r];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                t += __shfl_xor_sync(0xffffffffu, t, off);
            if (lane == (m * RW + r) % 32)
                keep = t;
        }
    if (lane < MT * RW) {
        const int m = lane / RW, n = nbase + lane % RW;
        if (m < p.M && n < p.N) {
            float out = keep;
            if (p.bias)
                out += to_float(static_cast<const XT*>(p.bias)[n]);
            static_cast<XT*>(p.y)[(int64_t)m * p.N + n] = from_float<XT>(out);
        }
    }
}

template <typename XT, typename PT, int BITS, int MT>
cudaError_t any_launch_rw(const AnyParams& prm, cudaStream_t st, const DeviceInfo& dev)
{
    // the widest warp tile that still gives every SM a CTA
    const int n = prm.N;
    if ((n + kAnyWarps * 4 - 1) / (kAnyWarps * 4) >= dev.sm_count)
        affine_any_kernel<XT, PT, BITS, MT, 4><<<(n + kAnyWarps * 4 - 1) / (kAnyWarps * 4), kAnyWarps * 32, 0, st>>>(prm);
    else if ((n + kAnyWarps * 2 - 1) / (kAnyWarps * 2) >= dev.sm_count)
        affine_any_kernel<XT, PT, BITS, MT, 2><<<(n + kAnyWarps * 2 - 1) / (kAnyWarps * 2), kAnyWarps * 32, 0, st>>>(prm);
    else
        affine_any_kernel<XT, PT, BITS, MT, 1><<<(n + kAnyWarps - 1) / kAnyWarps, kAnyWarps * 32, 0, st>>>(prm);
    return cudaGetLastError();
}

template <typename XT, typename PT, int BITS>
cudaError_t any_launch_m(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    for (int64_t m0 = 0; m0 < a.M; m0 += 8) {
        const int mc = (int)(a.M - m0 < 8 ? a.M - m0 : 8);
        AnyParams prm;
        prm.x = static_cast<const XT*>(a.x) + m0 * a.K;
        prm.codes = a.codes;
        prm.scales = a.scales;
        prm.biases = a.biases;
        prm.bias = a.bias;
        prm.y = static_cast<XT*>(a.y) + m0 * a.N;
        prm.M = mc;
        prm.K = (int)a.K;
        prm.N = (int)a.N;
        prm.g = a.g;
        cudaError_t e;
        if (mc == 1)
            e = any_launch_rw<XT, PT, BITS, 1>(prm, st, dev);
        else if (mc == 2)
            e = any_launch_rw<XT, PT, BITS, 2>(prm, st, dev);
        else if (mc <= 4)
            e = any_launch_rw<XT, PT, BITS, 4>(prm, st, dev);
        else
            e = any_launch_rw<XT, PT, BITS, 8>(prm, st, dev);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

template <typename XT, typename PT>
cudaError_t any_launch_b(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    switch (a.bits) {
    case 1: return any_launch_m<XT, PT, 1>(a, st, dev);
    case 2: return any_launch_m<XT, PT, 2>(a, st, dev);
    case 3: return any_launch_m<XT, PT, 3>(a, st, dev);
    case 4: return any_launch_m<XT, PT, 4>(a, st, dev);
    case 5: return any_launch_m<XT, PT, 5>(a, st, dev);
    case 6: return any_launch_m<XT, PT, 6>(a, st, dev);
    default: return any_launch_m<XT, PT, 8>(a, st, dev);
    }
}

template <typename XT>
cudaError_t any_launch_p(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    switch (a.p_dt) {
    case QLIN_F32: return any_launch_b<XT, float>(a, st, dev);
    case QLIN_BF16: return any_launch_b<XT, __nv_bfloat16>(a, st, dev);
    default: return any_launch_b<XT, __half>(a, st, dev);
    }
}

}  // namespace

cudaError_t launch_affine_gemv_any(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    switch (a.x_dt) {
    case QLIN_F32: return any_launch_p<float>(a, st, dev);
    case QLIN_BF16: return any_launch_p<__nv_bfloat16>(a, st, dev);
    default: return any_launch_p<__half>(a, st, dev);
    }
}

}  // namespace qlin
