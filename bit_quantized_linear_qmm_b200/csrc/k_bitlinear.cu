// k_bitlinear.cu -- BitLinear ternary decode GEMV (M <= 16 per launch) for sm_100a.
//
//   y[m, r + j*N/4] = s * sum_k x[m,k] * (((P[r,k] >> 2j) & 3) - 1) + bias[r + j*N/4]
//   [mlx_lm bitlinear_layers.py, make_bitlinear_kernel (kernel source: the
//    code of field j of byte P[r, k] is output row r + j*N/4, weight code - 1,
//    the tensor scale multiplied in or its reciprocal multiplied in);
//    BitLinear.__call__]
//
// Design (B200; a decode layer is a few MB of packed weights and sits in a
// chain of dependent layers, so the time per layer is the latency of the
// work that must follow the previous layer, not the weight stream):
//  * One CTA per SM (148 on B200) and the packed rows split evenly over them
//    (6 or 7 rows of 8 per CTA at N = 4096): no spare CTAs, so the next
//    layer's CTAs -- released early by programmatic dependent launch -- land
//    exactly one per SM and no SM runs two CTAs of one layer.  Layers with
//    more than 8 rows per SM use 8-row CTAs in waves instead.
//  * Before griddepcontrol.wait (the weights do not depend on the previous
//    kernel) each lane copies its 16-byte pieces of the first 8 chunks of its
//    packed row into shared memory with cp.async and waits for them to land:
//    an explicit completion, so the weight fetch cannot slip behind the
//    dependency wait (a plain read-only register load may be scheduled after
//    it, which was measured to cost ~1 us per layer).  x, the weight scale,
//    the bias and y are touched only after the wait; x streams through a
//    4-deep register ring, the staged weights are read back with conflict-free
//    16-byte shared loads, and chunks beyond the first 8 (K > 4096) stream
//    through registers.
//  * Decode, per 32-bit word (4 consecutive k of one packed row, 16
//    weights): two PRMTs place bytes (k, k+1) and (k+2, k+3) in the low byte
//    of each 16-bit half; one LOP3 per field pair masks the field into the
//    mantissa of the bf16 constant 128 (0x4300) -- 128 + 4^j c, exact -- and
//    one bf16x2 FMA turns that into exactly c - 1.  Field 3 (bits 6-7) lands
//    on the exponent's low bit: the pattern is 128, 192, 256, 384 for codes
//    0..3, the FMA maps it to -1, 0, 1, 3 and a bf16x2 min with 2 gives code
//    3 its weight 2.  A code-1 weight is an exact zero, so every product is
//    exact and only the fp32 accumulation and the final rounding spend the
//    error budget.
//  * The MACs run on the tensor cores with mma.sync m16n8k16 (A = weights:
//    rows g and g + 8 of the 16 are fields {0, 2} / {1, 3} of packed row g,
//    B = 8 tokens of x); partial tiles of the 8 warps (which split K) are
//    summed through shared memory, scaled, biased and rounded once.
//  * Compiled with QLIN_TRACE (a separate trace build of the library), thread
//    0 of every CTA records %globaltimer at the steps of the kernel so the
//    time of a chained layer can be broken down.
#include "qlin_common.cuh"

namespace qlin {

#ifdef QLIN_TRACE
// [slot][cta][8]: start, weights issued, wait returned, first chunk done,
// main loop done, end, (unused), smid.  Host side: qlin_trace_read().
constexpr int kTraceSlots = 1024;
constexpr int kTraceCtas = 512;
__device__ unsigned long long g_bl_trace[(size_t)kTraceSlots * kTraceCtas * 8];
#endif

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 8;       // packed rows per MMA tile row group (lane groups)
constexpr int kChunk = 64;     // k per chunk (4 lanes x 16 bytes)
constexpr int kRing = 8;       // chunks of weights a lane holds in registers

struct BitParams {
    const uint8_t* packed;  // [R][K]
    const __nv_bfloat16* x;  // [M][K]
    const float* weight_scale;
    const __nv_bfloat16* bias;  // [N] or null
    __nv_bfloat16* y;           // [M][N]
    int M, K, N, R;
    int invert;
    int spread;  // 1: rows split evenly over the grid; 0: 8-row CTAs
    int trace_slot;
};

QLIN_DEV uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// 16-byte asynchronous global -> shared copy (L2 only); src_bytes = 0 writes zeros.
QLIN_DEV void cp_async16(void* smem_dst, const void* src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}

// Waits until every cp.async this thread issued has landed in shared memory.
QLIN_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

QLIN_DEV uint32_t bf16x2_min(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// bf16x2 constants: field j of a byte masked into 0x4300 (= 128) reads 128 + 4^j c
constexpr uint32_t kMagic = 0x43004300u;
constexpr uint32_t kScale0 = 0x3F803F80u, kBias0 = 0xC301C301u;  // j = 0: (128 + c) - 129
constexpr uint32_t kScale1 = 0x3E803E80u, kBias1 = 0xC204C204u;  // j = 1: (128 + 4c) / 4 - 33
constexpr uint32_t kScale2 = 0x3D803D80u, kBias2 = 0xC110C110u;  // j = 2: (128 + 16c) / 16 - 9
constexpr uint32_t kScale3 = 0x3C803C80u, kBias3 = 0xC040C040u;  // j = 3: {128,192,256,384} / 64 - 3
constexpr uint32_t kTwo = 0x40004000u;                            // code 3 -> weight 2

// One 32-bit word (bytes k..k+3 of one packed row) -> the A registers of the two
// m16n8k16 tiles: f[0..3] fields {0, 2}, f[4..7] fields {1, 3}; each register a bf16
// pair (k, k+1) or (k+2, k+3) of one field.
QLIN_DEV void decode_word(uint32_t raw, uint32_t* f)
{
    const uint32_t lo = prmt(raw, 0u, 0x0100u);  // bytes k, k+1 in the low byte of each half
    const uint32_t hi = prmt(raw, 0u, 0x0302u);  // bytes k+2, k+3
    f[0] = bf16x2_fma(lop3_and_or(lo, 0x00030003u, kMagic), kScale0, kBias0);
    f[1] = bf16x2_fma(lop3_and_or(lo, 0x00300030u, kMagic), kScale2, kBias2);
    f[2] = bf16x2_fma(lop3_and_or(hi, 0x00030003u, kMagic), kScale0, kBias0);
    f[3] = bf16x2_fma(lop3_and_or(hi, 0x00300030u, kMagic), kScale2, kBias2);
    f[4] = bf16x2_fma(lop3_and_or(lo, 0x000C000Cu, kMagic), kScale1, kBias1);
    f[5] = bf16x2_min(bf16x2_fma(lop3_and_or(lo, 0x00C000C0u, kMagic), kScale3, kBias3), kTwo);
    f[6] = bf16x2_fma(lop3_and_or(hi, 0x000C000Cu, kMagic), kScale1, kBias1);
    f[7] = bf16x2_min(bf16x2_fma(lop3_and_or(hi, 0x00C000C0u, kMagic), kScale3, kBias3), kTwo);
}

#ifdef QLIN_TRACE
#define BL_TRACE(i) \
    do { if (threadIdx.x == 0) tr[i] = globaltimer_ns(); } while (0)
#else
#define BL_TRACE(i) \
    do { } while (0)
#endif

// NT token tiles of 8 (M <= 8 * NT); XD-deep x ring.  MY > 0: every warp has exactly MY
// whole 64-k chunks (K = 512 * MY, MY <= kRing), held in registers in one round and
// processed as straight-line code; MY = 0: any K (K % 16 == 0), in rounds of kRing
// chunks with the weights refilled as they are used.
template <int NT, int XD, int MY>
__global__ void __launch_bounds__(kThreads, 2) bitlinear_kernel(const __grid_constant__ BitParams p)
{
    constexpr bool FAST = MY > 0;
    static_assert(kRing % XD == 0, "x ring depth must divide the register round");
    __shared__ float red[kWarps * NT * 8 * 32];
    __shared__ uint4 wst[kRing][kWarps][32];  // first round of weights: [chunk][warp][lane]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
#ifdef QLIN_TRACE
    unsigned long long tr[8] = {};
#endif
    BL_TRACE(0);
    pdl_launch_dependents();

    const int r0 = p.spread ? (int)((long long)blockIdx.x * p.R / gridDim.x) : (int)blockIdx.x * kRows;
    const int r1 = p.spread ? (int)((long long)(blockIdx.x + 1) * p.R / gridDim.x) : min(r0 + kRows, p.R);
    const bool row_ok = r0 + gid < r1;
    const uint8_t* wrow = p.packed + (size_t)(row_ok ? r0 + gid : r0) * p.K + 16 * tig;
    const int nch = (p.K + kChunk - 1) / kChunk;
    const int my = FAST ? MY : nch > warp ? (nch - 1 - warp) / kWarps + 1 : 0;  // chunks of this warp
    auto chunk_k = [&](int ci) { return (warp + ci * kWarps) * kChunk; };

    auto load_w = [&](uint4& dst, int ci) {
        if (row_ok && ci < my && (FAST || chunk_k(ci) + 16 * tig < p.K))  // ci < MY is compile-time when FAST
            dst = ldg_stream_v4(wrow + chunk_k(ci));
        else
            dst = make_uint4(0u, 0u, 0u, 0u);
    };
    auto load_x = [&](uint4 (&dst)[NT][2], int ci) {
        const int k = chunk_k(ci) + 16 * tig;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int m = 8 * t + gid;
            if constexpr (FAST) {
                // token rows past M read row 0 and are zeroed with a mask: no divergent branch in
                // the straight-line loop (ci < MY is compile-time here)
                const uint32_t keep = m < p.M ? 0xFFFFFFFFu : 0u;
                const __nv_bfloat16* src = p.x + (size_t)(m < p.M ? m : 0) * p.K + k;
                if (ci < my) {
                    const uint4 a = ldg_cg_v4(src), b = ldg_cg_v4(src + 8);
                    dst[t][0] = make_uint4(a.x & keep, a.y & keep, a.z & keep, a.w & keep);
                    dst[t][1] = make_uint4(b.x & keep, b.y & keep, b.z & keep, b.w & keep);
                } else {
                    dst[t][0] = dst[t][1] = make_uint4(0u, 0u, 0u, 0u);
                }
            } else if (ci < my && m < p.M && k < p.K) {
                const __nv_bfloat16* src = p.x + (size_t)m * p.K + k;
                dst[t][0] = ldg_cg_v4(src);
                dst[t][1] = ldg_cg_v4(src + 8);
            } else {
                dst[t][0] = dst[t][1] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };

    // first round: global -> shared, completed before the dependency wait
#pragma unroll
    for (int j = 0; j < kRing; ++j) {
        if (j < (FAST ? MY : kRing)) {
            const bool ok = row_ok && j < my && (FAST || chunk_k(j) + 16 * tig < p.K);
            cp_async16(&wst[j][warp][lane], ok ? wrow + chunk_k(j) : p.packed, ok ? 16 : 0);
        }
    }
    cp_async_wait_all();
    BL_TRACE(1);
    pdl_wait_prior_grids();  // x, the weight scale, the bias and y may belong to the previous kernel
    BL_TRACE(2);
    uint4 wr[FAST ? 1 : kRing];  // later rounds (general path): register ring
    if constexpr (!FAST) {
#pragma unroll
        for (int j = 0; j < kRing; ++j)
            load_w(wr[j], j + kRing);
    }
    uint4 xb[XD][NT][2];
#pragma unroll
    for (int d = 0; d < XD; ++d)
        load_x(xb[d], d);
    const float ws = *p.weight_scale;

    // with one token tile, two accumulator sets (even / odd words) keep four MMA chains per warp
    constexpr int AS = NT == 1 ? 2 : 1;
    float acc[2][AS][NT][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int h = 0; h < AS; ++h)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[a][h][t][e] = 0.f;

    auto chunk = [&](const uint4& w4, const uint4 (&xv)[NT][2]) {
        uint32_t f[4][8];  // word i: k = chunk + 16 tig + 4i .. +3
        decode_word(w4.x, f[0]);
        decode_word(w4.y, f[1]);
        decode_word(w4.z, f[2]);
        decode_word(w4.w, f[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint4& xh = xv[t][i >> 1];
                const uint32_t b0 = (i & 1) ? xh.z : xh.x;  // (x_k, x_k+1)
                const uint32_t b1 = (i & 1) ? xh.w : xh.y;  // (x_k+2, x_k+3)
                const uint32_t a02[4] = {f[i][0], f[i][1], f[i][2], f[i][3]};
                const uint32_t a13[4] = {f[i][4], f[i][5], f[i][6], f[i][7]};
                mma_bf16_16816(acc[0][i % AS][t], a02, b0, b1);
                mma_bf16_16816(acc[1][i % AS][t], a13, b0, b1);
            }
        }
    };

    if constexpr (FAST) {
#pragma unroll
        for (int j = 0; j < MY; ++j) {
            chunk(wst[j][warp][lane], xb[j % XD]);
            if (j == 0)
                BL_TRACE(3);
            if (j + XD < MY)
                load_x(xb[j % XD], j + XD);
        }
    } else {
#pragma unroll
        for (int j = 0; j < kRing; ++j) {  // round 0 from shared memory
            if (j < my)
                chunk(wst[j][warp][lane], xb[j % XD]);
            if (j == 0)
                BL_TRACE(3);
            load_x(xb[j % XD], j + XD);
        }
        const int rounds = (my + kRing - 1) / kRing;
        for (int rd = 1; rd < rounds; ++rd) {  // later rounds from the register ring
#pragma unroll
            for (int j = 0; j < kRing; ++j) {
                const int ci = rd * kRing + j;
                if (ci < my)
                    chunk(wr[j], xb[j % XD]);
                load_x(xb[j % XD], ci + XD);
                load_w(wr[j], ci + kRing);
            }
        }
    }
    BL_TRACE(4);

    // sum the 8 warps' partial tiles; v = t * 8 + a * 4 + e
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                red[((warp * NT + t) * 8 + a * 4 + e) * 32 + lane] =
                    acc[a][0][t][e] + (AS > 1 ? acc[a][AS - 1][t][e] : 0.f);
    __syncthreads();
    const float scale = p.invert ? __frcp_rn(ws) : ws;  // 1/ws rounded once, as a division would
#pragma unroll
    for (int q = 0; q < NT; ++q) {
        const int idx = q * kThreads + threadIdx.x;
        const int v = idx >> 5, ln = idx & 31;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            sum += red[(w * NT * 8 + v) * 32 + ln];
        const int t = v >> 3, a = (v >> 2) & 1, e = v & 3;
        const int pr = r0 + (ln >> 2);
        const int m = 8 * t + 2 * (ln & 3) + (e & 1);
        if (pr < r1 && m < p.M) {
            const int n = pr + (a + 2 * (e >> 1)) * p.R;
            float out = sum * scale;
            if (p.bias)
                out += __bfloat162float(p.bias[n]);
            p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(out);
        }
    }
#ifdef QLIN_TRACE
    BL_TRACE(5);
    if (threadIdx.x == 0 && p.trace_slot >= 0 && blockIdx.x < kTraceCtas) {
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        tr[7] = smid;
        unsigned long long* dst = g_bl_trace + ((size_t)p.trace_slot * kTraceCtas + blockIdx.x) * 8;
        for (int i = 0; i < 8; ++i)
            dst[i] = tr[i];
    }
#endif
}

template <typename Kern>
cudaError_t launch_pdl_bl(Kern kern, dim3 grid, cudaStream_t st, const BitParams& prm)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

#ifdef QLIN_TRACE
int g_trace_next = 0;  // host: next trace slot (launches past kTraceSlots are not recorded)
#endif

}  // namespace

cudaError_t launch_bitlinear_gemv(const BitlinearArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    const int R = (int)(a.N / 4);
    // rows split evenly over one CTA per SM while that keeps at most 8 per CTA, else 8-row CTAs
    const bool spread = R <= kRows * dev.sm_count;
    const int grid = spread ? (R < dev.sm_count ? R : dev.sm_count) : (R + kRows - 1) / kRows;
    // whole chunks, the same count for every warp: straight-line kernels for K = 512 * MY
    const int my = a.K % (kChunk * kWarps) == 0 ? (int)(a.K / (kChunk * kWarps)) : 0;
    const int fast = (my == 1 || my == 2 || my == 4 || my == 8) ? my : 0;
    for (int64_t m0 = 0; m0 < a.M; m0 += 16) {
        const int mc = (int)(a.M - m0 < 16 ? a.M - m0 : 16);
        BitParams prm;
        prm.packed = a.packed;
        prm.x = static_cast<const __nv_bfloat16*>(a.x) + m0 * a.K;
        prm.weight_scale = a.weight_scale;
        prm.bias = static_cast<const __nv_bfloat16*>(a.bias);
        prm.y = static_cast<__nv_bfloat16*>(a.y) + m0 * a.N;
        prm.M = mc;
        prm.K = (int)a.K;
        prm.N = (int)a.N;
        prm.R = R;
        prm.invert = a.invert;
        prm.spread = spread ? 1 : 0;
#ifdef QLIN_TRACE
        prm.trace_slot = g_trace_next < kTraceSlots ? g_trace_next++ : -1;
#else
        prm.trace_slot = -1;
#endif
        cudaError_t e;
        const dim3 g((unsigned)grid);
        if (mc <= 8) {
            switch (fast) {
            case 8: e = launch_pdl_bl(bitlinear_kernel<1, 4, 8>, g, st, prm); break;
            case 4: e = launch_pdl_bl(bitlinear_kernel<1, 4, 4>, g, st, prm); break;
            case 2: e = launch_pdl_bl(bitlinear_kernel<1, 2, 2>, g, st, prm); break;
            case 1: e = launch_pdl_bl(bitlinear_kernel<1, 1, 1>, g, st, prm); break;
            default: e = launch_pdl_bl(bitlinear_kernel<1, 4, 0>, g, st, prm); break;
            }
        } else {
            switch (fast) {
            case 8: e = launch_pdl_bl(bitlinear_kernel<2, 2, 8>, g, st, prm); break;
            case 4: e = launch_pdl_bl(bitlinear_kernel<2, 2, 4>, g, st, prm); break;
            case 2: e = launch_pdl_bl(bitlinear_kernel<2, 2, 2>, g, st, prm); break;
            case 1: e = launch_pdl_bl(bitlinear_kernel<2, 1, 1>, g, st, prm); break;
            default: e = launch_pdl_bl(bitlinear_kernel<2, 2, 0>, g, st, prm); break;
            }
        }
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace qlin

#ifdef QLIN_TRACE
// Trace build only: copies the recorded timestamps ([slot][cta][8] uint64) to a host
// buffer and clears the slot counter; returns the number of slots recorded.
extern "C" int qlin_trace_read(void* host, size_t bytes)
{
    const int used = qlin::g_trace_next;
    const size_t need = (size_t)used * qlin::kTraceCtas * 8 * sizeof(unsigned long long);
    if (host && bytes >= need && need > 0 &&
        cudaMemcpyFromSymbol(host, qlin::g_bl_trace, need) != cudaSuccess)
        return -1;
    qlin::g_trace_next = 0;
    return used;
}

extern "C" int qlin_trace_ctas(void) { return qlin::kTraceCtas; }
#endif
