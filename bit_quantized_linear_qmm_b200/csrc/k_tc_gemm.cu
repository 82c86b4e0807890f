// k_tc_gemm.cu -- prefill-regime GEMMs on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory), sm_100a.
//
//   raw int8:  c[m,n] = sum_k a[m,k] * b[n,k]                (int32, exact)
//              [cider/ops.py int8_matmul_int32]
//   W8A8:      y[m,n] = acc * s_x[m] * s_w[n] + bias[n]      (acc = qx . w, int32)
//              [cider/ops.py perchannel_linear]
//   W4A8:      y[m,n] = acc * s_x[m] * s_w[n] (+ bias[n]),   acc = qx . (c - 8)
//              [cider/ops.py w4a8_linear, pack_weight_int4]
//   affine:    y[m,n] = sum_k x[m,k] * bf16(fma(q, s, b)) + bias[n]
//              [nuvec-nn QuantizedLinear, forward; cider/ops.py pergroup_linear
//               docstring, dequantize]
//
// One CTA computes a 128 x 128 output tile:
//   warp 0       TMA producer: A tiles (and B, or the packed B source) into a
//                shared-memory ring, 128-byte swizzle, mbarrier completion.
//   warp 1       allocates 128 TMEM columns; one thread issues tcgen05.mma
//                (M = 128, N = 128, K = 32 int8 / 16 bf16 per instruction) and
//                tcgen05.commit releases each stage when its MMAs are done.
//   warps 2..5   epilogue: tcgen05.ld of the fp32/int32 accumulator (each warp
//                owns 32 TMEM lanes = 32 output rows), scales, bias, stores.
//   warps 6..13  (W4A8, affine) transform the packed B source into the
//                K-major swizzled operand layout: nibbles -> int8 (c - 8), or
//                codes -> bf16(fma(q, scale, bias)) in fp32 (the dequantized
//                weight, rounded once to bf16), then fence.proxy.async.
// Every mbarrier wait is bounded; on expiry the kernel records the timeout,
// skips the remaining work, and always frees its TMEM.
#include "qlin_common.cuh"

namespace qlin {
namespace {

constexpr int kBM = 128;      // output rows (tokens) per CTA
constexpr int kBN = 128;      // output columns (features) per CTA
constexpr int kTmemCols = 128;

enum BSource { B_TMA_I8 = 0, B_W4 = 1, B_AFFINE4 = 2 };
enum Epi { E_I32 = 0, E_SCALED = 1, E_BIAS = 2 };

__host__ __device__ constexpr int rup(int a, int b) { return (a + b - 1) / b * b; }

template <int BSRC>
struct TcCfg {
    static constexpr bool I8 = BSRC != B_AFFINE4;          // kind::i8 (s32) or kind::f16 (bf16 -> f32)
    static constexpr int KE = I8 ? 128 : 64;                // K elements per stage (128 bytes of A)
    static constexpr int A_BYTES = kBM * 128;
    static constexpr int B_BYTES = kBN * 128;
    static constexpr int RAW_BYTES = BSRC == B_W4 ? (KE / 2) * kBN : (BSRC == B_AFFINE4 ? kBN * (KE / 2) : 0);
    static constexpr int STAGE = rup(A_BYTES + B_BYTES + RAW_BYTES, 1024);
    static constexpr int NS = BSRC == B_TMA_I8 ? 6 : 5;
    static constexpr int XW = BSRC == B_TMA_I8 ? 0 : 8;     // transform warps
    static constexpr int THREADS = (6 + XW) * 32;
    static constexpr uint32_t IDESC =
        (I8 ? (2u << 4) : (1u << 4)) |                      // D: s32 / f32
        (1u << 7) | (1u << 10) |                            // A, B: s8 / bf16 (signed)
        ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);  // K-major A and B
    struct Bars {
        uint64_t full[NS];
        uint64_t bready[NS];
        uint64_t empty[NS];
        uint64_t accf;
        uint32_t tmem;
        int abort_flag;
    };
    static constexpr int SMEM = NS * STAGE + (int)sizeof(Bars) + 1024;
};

struct TcParams {
    CUtensorMap tm_a;  // A [M][K], box {128 B, 128 rows}, 128-byte swizzle
    CUtensorMap tm_b;  // int8 B [N][K] (box {128 B, 128 rows}, swizzled) | packed int4 [K/2][N]
                       // (box {128 B, 64 rows}) | affine code bytes [N][K/2] (box {32 B, 128 rows})
    int M, N, K;
    void* out;
    const float* s_x;
    const float* s_w;
    const __nv_bfloat16* bias;
    const __nv_bfloat16* scales;
    const __nv_bfloat16* biases;
    int g;
    unsigned* status;
};

QLIN_DEV void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

QLIN_DEV uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int BSRC, int EPI>
__global__ void __launch_bounds__(TcCfg<BSRC>::THREADS, 1) tc_gemm_kernel(const __grid_constant__ TcParams p)
{
    using Cfg = TcCfg<BSRC>;
    using Bars = typename Cfg::Bars;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars& bars = *reinterpret_cast<Bars*>(smem + Cfg::NS * Cfg::STAGE);
    auto A = [&](int s) { return smem + s * Cfg::STAGE; };
    auto B = [&](int s) { return smem + s * Cfg::STAGE + Cfg::A_BYTES; };
    auto RAW = [&](int s) { return smem + s * Cfg::STAGE + Cfg::A_BYTES + Cfg::B_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
    const int nk = (p.K + Cfg::KE - 1) / Cfg::KE;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.bready[s], Cfg::XW > 0 ? Cfg::XW : 1);
            mbar_init(&bars.empty[s], 1);
        }
        mbar_init(&bars.accf, 1);
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1)
        tmem_alloc(&bars.tmem, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            pdl_launch_dependents();
            pdl_wait_prior_grids();  // A (activations) may come from the previous kernel
            int issued = 0;
            for (int it = 0; it < nk; ++it) {
                const int slot = it % Cfg::NS;
                if (it >= Cfg::NS &&
                    (!mbar_wait_bounded(&bars.empty[slot], ((it / Cfg::NS) & 1) ^ 1, p.status) ||
                     *reinterpret_cast<volatile int*>(&bars.abort_flag))) {
                    bars.abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(&bars.full[slot],
                                      Cfg::A_BYTES + (BSRC == B_TMA_I8 ? Cfg::B_BYTES : Cfg::RAW_BYTES));
                tma_load_2d(A(slot), &p.tm_a, it * Cfg::KE, m0, &bars.full[slot]);
                if constexpr (BSRC == B_TMA_I8)
                    tma_load_2d(B(slot), &p.tm_b, it * 128, n0, &bars.full[slot]);
                else if constexpr (BSRC == B_W4)
                    tma_load_2d(RAW(slot), &p.tm_b, n0, it * (Cfg::KE / 2), &bars.full[slot]);
                else
                    tma_load_2d(RAW(slot), &p.tm_b, it * (Cfg::KE / 2), n0, &bars.full[slot]);
                ++issued;
            }
            for (int it = issued - Cfg::NS < 0 ? 0 : issued - Cfg::NS; it < issued; ++it)
                mbar_wait_bounded(&bars.full[it % Cfg::NS], (it / Cfg::NS) & 1, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int it = 0; it < nk && ok; ++it) {
                const int slot = it % Cfg::NS;
                const unsigned par = (it / Cfg::NS) & 1;
                ok = mbar_wait_bounded(&bars.full[slot], par, p.status);
                if (ok && Cfg::XW > 0)
                    ok = mbar_wait_bounded(&bars.bready[slot], par, p.status);
                if (!ok) {
                    bars.abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(A(slot)), b0 = smem_u32(B(slot));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma<Cfg::I8>(tmem, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32), Cfg::IDESC,
                                    (it | kk) != 0 ? 1u : 0u);
                tc_commit(&bars.empty[slot]);
            }
            tc_commit(&bars.accf);  // also fires when nothing was issued
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const bool ok = mbar_wait_bounded(&bars.accf, 0, p.status);
        tc_fence_after();
        pdl_wait_prior_grids();  // scales / bias / out may be touched by the previous kernel
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row = m0 + 32 * q + lane;
        float sx = 0.f;
        if constexpr (EPI == E_SCALED)
            sx = (row < p.M) ? p.s_x[row] : 0.f;
#pragma unroll 1
        for (int c = 0; c < kBN / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(c * 16), r);
            const int n = n0 + c * 16;
            if (!ok || row >= p.M || n >= p.N)
                continue;
            // vector stores need the row pitch aligned: N % 4 (int32) / N % 8 (bf16)
            const bool full16 = n + 16 <= p.N && (p.N % (EPI == E_I32 ? 4 : 8)) == 0;
            if constexpr (EPI == E_I32) {
                int32_t* o = static_cast<int32_t*>(p.out) + (size_t)row * p.N + n;
                if (full16) {
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<uint4*>(o + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
                } else {
                    for (int j = 0; j < 16 && n + j < p.N; ++j)
                        o[j] = (int32_t)r[j];
                }
            } else {
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int nj = n + j < p.N ? n + j : p.N - 1;
                    float a;
                    if constexpr (EPI == E_SCALED)
                        a = fmaf((float)(int32_t)r[j], sx * __ldg(p.s_w + nj), 0.f);
                    else
                        a = __uint_as_float(r[j]);
                    if (p.bias)
                        a += __bfloat162float(p.bias[nj]);
                    v[j] = a;
                }
                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.N + n;
                if (full16) {
                    *reinterpret_cast<uint4*>(o) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                    *reinterpret_cast<uint4*>(o + 8) =
                        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15]));
                } else {
                    for (int j = 0; j < 16 && n + j < p.N; ++j)
                        o[j] = __float2bfloat16_rn(v[j]);
                }
            }
        }
    } else if constexpr (Cfg::XW > 0) {
        // ------------------------------------------------------------ B transform
        const int tt = threadIdx.x - 6 * 32;  // 0 .. 255
        const int r = tt & (kBN - 1);         // operand row (output column n0 + r)
        const int half = tt >> 7;             // which 64 bytes of the 128-byte K slice
        const int ng = p.K / (p.g > 0 ? p.g : 1);
        const int nrow = min(n0 + r, p.N - 1);
        pdl_wait_prior_grids();  // the packed weights' parameters may come from the previous kernel
        for (int it = 0; it < nk; ++it) {
            const int slot = it % Cfg::NS;
            if (!mbar_wait_bounded(&bars.full[slot], (it / Cfg::NS) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            uint8_t* dst = B(slot);
            if constexpr (BSRC == B_W4) {
                // raw[i][n]: k-pair row i (k = 2i high nibble, 2i+1 low), column n; 64 rows x 128 bytes
                const uint8_t* raw = RAW(slot);
#pragma unroll
                for (int u = 4 * half; u < 4 * half + 4; ++u) {  // 16-byte unit: k = 16u .. 16u+15
                    uint32_t wd[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t b0 = raw[(8 * u + 2 * w) * kBN + r];
                        const uint32_t b1 = raw[(8 * u + 2 * w + 1) * kBN + r];
                        const uint32_t v = (b0 >> 4) | ((b0 & 15u) << 8) | ((b1 >> 4) << 16) | ((b1 & 15u) << 24);
                        wd[w] = (v + 0x78787878u) ^ 0x80808080u;  // each nibble c -> int8 c - 8
                    }
                    st_shared_v4(dst + swz128(r, u), wd[0], wd[1], wd[2], wd[3]);
                }
            } else {
                // raw[n][32 bytes]: 64 LSB-first 4-bit codes of row n, k = k0 .. k0+63
                const int kbase = it * Cfg::KE + 32 * half;  // first k of this thread's 32 codes
                const uint4 cw = *reinterpret_cast<const uint4*>(RAW(slot) + r * 32 + 16 * half);
                const int gi = min(kbase, p.K - 1) / p.g;
                const float s = __bfloat162float(p.scales[(size_t)nrow * ng + gi]);
                const float b = __bfloat162float(p.biases[(size_t)nrow * ng + gi]);
                const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {  // word w: k = kbase + 8w .. +7 -> unit 4 half + w
                    uint32_t o[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t w0 = words[w] >> (8 * j);
                        const float q0 = __uint_as_float(0x4B000000u | (w0 & 15u)) - 8388608.0f;
                        const float q1 = __uint_as_float(0x4B000000u | ((w0 >> 4) & 15u)) - 8388608.0f;
                        o[j] = pack_bf16x2(__fmaf_rn(q0, s, b), __fmaf_rn(q1, s, b));
                    }
                    // k beyond K: zero weights (the activations there are zero too)
                    if (kbase + 8 * w >= p.K)
                        o[0] = o[1] = o[2] = o[3] = 0u;
                    st_shared_v4(dst + swz128(r, 4 * half + w), o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.bready[slot]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemCols);
}

template <int BSRC, int EPI>
cudaError_t launch_t(const TcParams& prm, int M, int N, cudaStream_t st)
{
    using Cfg = TcCfg<BSRC>;
    auto kern = tc_gemm_kernel<BSRC, EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + kBN - 1) / kBN), (unsigned)((M + kBM - 1) / kBM), 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)Cfg::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

}  // namespace

cudaError_t launch_tc_gemm(TcOp op, const TcGemmArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    TcParams prm;
    prm.M = (int)a.M;
    prm.N = (int)a.N;
    prm.K = (int)a.K;
    prm.out = a.out;
    prm.s_x = a.s_x;
    prm.s_w = a.s_w;
    prm.bias = static_cast<const __nv_bfloat16*>(a.bias);
    prm.scales = static_cast<const __nv_bfloat16*>(a.scales);
    prm.biases = static_cast<const __nv_bfloat16*>(a.biases);
    prm.g = a.g;
    prm.status = dev.status;
    const bool bf16_a = op == TC_AFFINE4;
    const uint64_t a_pitch = (uint64_t)a.K * (bf16_a ? 2 : 1);
    if (!encode_tmap_2d(&prm.tm_a, bf16_a ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a,
                        (uint64_t)a.K, (uint64_t)a.M, a_pitch, bf16_a ? 64 : 128, kBM))
        return cudaErrorInvalidValue;
    bool ok;
    switch (op) {
    case TC_I8_RAW:
    case TC_W8A8:
        ok = encode_tmap_2d(&prm.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b, (uint64_t)a.K, (uint64_t)a.N,
                            (uint64_t)a.K, 128, kBN);
        break;
    case TC_W4A8:
        ok = encode_tmap_2d(&prm.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b, (uint64_t)a.N, (uint64_t)(a.K / 2),
                            (uint64_t)a.N, kBN, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
        break;
    default:
        ok = encode_tmap_2d(&prm.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b, (uint64_t)(a.K / 2), (uint64_t)a.N,
                            (uint64_t)(a.K / 2), 32, kBN, CU_TENSOR_MAP_SWIZZLE_NONE);
        break;
    }
    if (!ok)
        return cudaErrorInvalidValue;
    switch (op) {
    case TC_I8_RAW: return launch_t<B_TMA_I8, E_I32>(prm, prm.M, prm.N, st);
    case TC_W8A8: return launch_t<B_TMA_I8, E_SCALED>(prm, prm.M, prm.N, st);
    case TC_W4A8: return launch_t<B_W4, E_SCALED>(prm, prm.M, prm.N, st);
    default: return launch_t<B_AFFINE4, E_BIAS>(prm, prm.M, prm.N, st);
    }
}

}  // namespace qlin
