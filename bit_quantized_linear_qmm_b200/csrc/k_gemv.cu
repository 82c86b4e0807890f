// k_gemv.cu -- decode-regime (M <= 16) quantized GEMV kernels for sm_100a.
//
//   affine:    y[m,n] = sum_k x[m,k] * (q[n,k]*s[n,k/g] + b[n,k/g]) + bias[n]
//              [nuvec-nn QuantizedLinear, forward / fields weight, scales,
//               biases; cider/ops.py pergroup_linear docstring, dequantize]
//   bitlinear: y[m, r + j*N/4] = scale * sum_k x[m,k] * (((P[r,k] >> 2j) & 3) - 1) + bias
//              [mlx_lm bitlinear_layers.py, make_bitlinear_kernel, BitLinear.__call__]
//
// Design (B200, HBM- and latency-bound):
//  * A CTA owns 64 output rows x a K-range.  K is split over the CTAs of a
//    thread-block cluster; each CTA pushes its fp32 partial tile into the
//    leader CTA's shared memory (st.shared::cluster) and arrives on the
//    leader's mbarrier; the leader sums, adds the layer bias and stores y.
//    No workspace, no atomics in global memory, one cluster barrier.
//  * One producer thread streams the tile through a 4-stage shared-memory
//    ring with 2-D tensor-map TMA (cp.async.bulk.tensor, 128-byte swizzle,
//    completion on mbarriers): one instruction moves a 128-byte column block
//    of all 64 weight rows, one a 128-byte column block of all tokens of x
//    (tokens >= M and bytes past the row end arrive as zeros).  With
//    programmatic dependent launch the first stages' weights are prefetched
//    into L2 before griddepcontrol.wait, so back-to-back layers overlap one
//    kernel's DRAM fetch with the previous kernel's tail.
//  * Eight consumer warps (4 row tiles of 16 rows x 2 K-lanes) dequantise in
//    registers and run the MACs on the tensor cores with the legacy
//    mma.sync.m16n8k16 (weights as the 16-row A operand, x as the n=8 B
//    operand, fp32 accumulation).
//  * affine: codes become bf16 with one LOP3 per pair: (w >> s) & 0x000F000F
//    | 0x43004300 is the bf16 pair (128 + q_i, 128 + q_j), exact.  The 128
//    offset and the group bias fold out per group with the group sums of x,
//    which an MMA against an all-ones A operand produces:
//      y = sum_g [ s_g * D'_g + (b_g - 128 s_g) * X_g ],
//      D'_g = sum_{k in g} (q_k + 128) x_k,  X_g = sum_{k in g} x_k.
//    (8-bit codes use no offset: bf16 holds 0..255 exactly.)  Because a dot
//    product over a group does not depend on the order of k, each lane pairs
//    codes in the order the LOP3 yields them and permutes x to match (PRMT).
//  * bitlinear: (c + 128) pairs from the same LOP3, then one bf16x2 add of
//    -129 gives the exact weights c - 1, so a code-1 weight contributes an
//    exact zero.
//  * Every mbarrier wait is bounded (qlin::kWaitLimitNs); on expiry the
//    kernel records the timeout in the status word, stops issuing copies,
//    waits (bounded) for its copies in flight and runs to completion.
#include "qlin_common.cuh"

namespace qlin {
namespace {

constexpr int kRowTiles = 4;                       // 16-row MMA tiles per CTA
constexpr int kKLanes = 2;                         // consumer warps sharing a row tile along K
constexpr int kConsumerWarps = kRowTiles * kKLanes;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;    // + one producer warp
constexpr int kRowsPerCta = 16 * kRowTiles;
constexpr int kStages = 4;
constexpr int kMaxCluster = 8;
constexpr int kRedStride = kRowsPerCta + 4;        // padded row of the partial tile (bank spread)

__host__ __device__ constexpr int round_up(int a, int b) { return (a + b - 1) / b * b; }

struct alignas(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t reduce;  // leader: one arrival per CTA of the cluster
    int abort_flag;
};

QLIN_DEV bool volatile_abort(Barriers& b) { return *reinterpret_cast<volatile int*>(&b.abort_flag) != 0; }

QLIN_DEV void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory"); }

QLIN_DEV uint32_t pair_lo(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410); }  // (a.lo, b.lo)
QLIN_DEV uint32_t pair_hi(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632); }  // (a.hi, b.hi)

constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;      // (1.0, 1.0)
constexpr uint32_t kMinus129Bf16x2 = 0xC301C301u;  // (-129.0, -129.0)

QLIN_DEV uint32_t bf16x2_add(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Split fp32 pairs into bf16 hi/lo parts: x = hi + lo + O(2^-17 |x|).
QLIN_DEV void split_f32_pair(float a, float b, uint32_t& hi, uint32_t& lo)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    float ra = __fsub_rn(a, __low2float(h));
    float rb = __fsub_rn(b, __high2float(h));
    __nv_bfloat162 l = __floats2bfloat162_rn(ra, rb);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

// ---------------------------------------------------------------- producer

// Run by the whole producer warp; lane 0 streams `nst` stages: issue(it, slot)
// issues the TMA loads of stage `it`, prefetch(it) the L2 prefetches of its
// weights, stage_bytes(it) is what the full barrier expects.  Before
// griddepcontrol.wait only L2 prefetches of weights are issued (coherent
// with any earlier kernel's writes); every load into shared memory follows
// the wait.
template <typename IssueFn, typename PFn, typename BytesFn>
QLIN_DEV void producer_loop(Barriers& bars, int nst, unsigned* status, IssueFn issue, PFn prefetch,
                            BytesFn stage_bytes)
{
    if ((threadIdx.x & 31) == 0) {
        const int pre = nst < kStages ? nst : kStages;
        const int npf = nst < 2 * kStages ? nst : 2 * kStages;
        for (int it = 0; it < npf; ++it)
            prefetch(it);
        pdl_wait_prior_grids();
        for (int it = 0; it < pre; ++it) {
            mbar_arrive_expect_tx(&bars.full[it], stage_bytes(it));
            issue(it, it);
        }
        pdl_launch_dependents();
        int issued = pre;
        for (int it = pre; it < nst; ++it) {
            const int slot = it % kStages;
            if (!mbar_wait_bounded(&bars.empty[slot], ((it / kStages) & 1) ^ 1, status) || volatile_abort(bars))
                break;
            mbar_arrive_expect_tx(&bars.full[slot], stage_bytes(it));
            issue(it, slot);
            ++issued;
        }
        // Drain: no TMA load may still target this CTA's shared memory at exit.
        for (int it = issued - kStages < 0 ? 0 : issued - kStages; it < issued; ++it)
            mbar_wait_bounded(&bars.full[it % kStages], (it / kStages) & 1, status);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- cluster reduction

// Called by all kThreads threads.  Consumers have accumulated this CTA's
// partial tile in red[token * kRedStride + row].  Every CTA pushes it into
// slot `rank` of the leader's recv buffer and arrives on the leader's reduce
// barrier; the leader's consumers wait for all S slots, sum them and call
// store(token, row, value).
template <typename StoreFn>
QLIN_DEV void cluster_reduce(Barriers& bars, float* red, float* recv, int M, int S, unsigned* status,
                             StoreFn store)
{
    const int rank = blockIdx.x;  // the cluster spans gridDim.x
    cluster_wait();               // every CTA's barriers are initialised before any remote access
    if (threadIdx.x >= kConsumerThreads)
        return;
    consumer_bar();  // red complete
    const int tile = M * kRowsPerCta;
    const uint32_t dst = map_shared_rank(smem_u32(recv + rank * tile), 0);
    for (int e4 = threadIdx.x; e4 < tile / 4; e4 += kConsumerThreads) {
        const int e = e4 * 4;
        const int tok = e / kRowsPerCta, r = e % kRowsPerCta;
        const float* src = red + tok * kRedStride + r;
        st_shared_cluster_v4(dst + 16u * (uint32_t)e4, make_float4(src[0], src[1], src[2], src[3]));
    }
    consumer_bar();  // all of this CTA's pushes issued
    if (threadIdx.x == 0)
        mbar_remote_arrive_cluster(map_shared_rank(smem_u32(&bars.reduce), 0));
    if (rank != 0)
        return;
    if (!mbar_wait_cluster_bounded(&bars.reduce, 0, status))
        return;
    pdl_wait_prior_grids();  // (already satisfied) no global write before the prior grid completed
    for (int e = threadIdx.x; e < tile; e += kConsumerThreads) {
        float v = 0.f;
        for (int q = 0; q < S; ++q)
            v += recv[q * tile + e];
        store(e / kRowsPerCta, e % kRowsPerCta, v);
    }
}

QLIN_DEV void init_barriers(Barriers& bars, int S)
{
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], kConsumerWarps);
        }
        mbar_init(&bars.reduce, (unsigned)S);
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    cluster_arrive_relaxed();
}

// ---------------------------------------------------------------- affine decode kernel

template <int BITS, int G, typename XT, typename PT, int NT>
struct AffineCfg {
    static constexpr int KST = 1024 / BITS > 256 ? 1024 / BITS : 256;  // k per stage
    static constexpr int NWB = KST * BITS / 8 / 128;       // 128-byte weight boxes per stage
    static constexpr int XE = 128 / (int)sizeof(XT);       // x elements per 128-byte box row
    static constexpr int NXB = KST / XE;                   // x boxes per stage
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = NWB * kRowsPerCta * 128;
    static constexpr int X_STAGE = NXB * MMAX * 128;
    static constexpr int STAGE = W_STAGE + X_STAGE;       // multiple of 1024
    static constexpr int CPW = 32 / BITS;                  // codes per 32-bit word
    static constexpr int WPG = G * BITS / 32;              // words per row per group
    static constexpr int WPL = WPG / 4;                    // words per lane per row per group
    static constexpr int NP = CPW / 2;                     // bf16 pairs per word
    static constexpr int MAX_GROUPS = 64;                  // param groups per row kept in smem
    static constexpr int PARAMS_PER_THREAD = kRowsPerCta * MAX_GROUPS / kConsumerThreads;
    static_assert(WPL >= 1, "group too small for the decode lane mapping");
    static_assert(STAGE % 1024 == 0, "swizzled boxes need 1024-byte alignment");
    // bf16 holds 0..255 exactly but not 128 + q for q >= 128: 8-bit codes go unbiased
    static constexpr float OFFSET = BITS == 8 ? 0.0f : 128.0f;
    static constexpr int RED = MMAX * kRedStride * 4;
    static constexpr int recv_bytes(int S) { return S * MMAX * kRowsPerCta * 4; }
    static constexpr int smem_bytes(int gstride, int S)
    {
        return kStages * STAGE + round_up(kRowsPerCta * gstride * 8, 16) + RED + recv_bytes(S) +
               (int)sizeof(Barriers) + 1024;
    }
};

struct AffineParams {
    CUtensorMap tm_w;  // codes as bytes [N][K*BITS/8], box {128 B, 64 rows}
    CUtensorMap tm_x;  // x [M][K], box {128 B, 8*NT tokens}
    const uint8_t* codes;  // bytes of the uint32 words
    const void* x;
    const void* scales;
    const void* biases;
    const void* bias;
    void* y;
    int M, K, N;
    int k_per_split;  // multiple of KST
    int gstride;      // groups per row held in the smem parameter block (k_per_split / G)
    unsigned* status;
};

// A-operand registers of one mma from the packed words of rows gid (w0) and
// gid+8 (w1); `part` selects the code pairs.
template <int BITS>
QLIN_DEV void make_a_regs(uint32_t w0, uint32_t w1, int part, uint32_t (&a)[4])
{
    if constexpr (BITS == 4) {
        // pairs (q_j, q_{j+4}) from (w >> 4j) & 0x000F000F; part 0 uses j = 0, 1; part 1 uses j = 2, 3
        const int s0 = 8 * part, s1 = 8 * part + 4;
        a[0] = lop3_and_or(w0 >> s0, 0x000F000Fu, 0x43004300u);
        a[1] = lop3_and_or(w1 >> s0, 0x000F000Fu, 0x43004300u);
        a[2] = lop3_and_or(w0 >> s1, 0x000F000Fu, 0x43004300u);
        a[3] = lop3_and_or(w1 >> s1, 0x000F000Fu, 0x43004300u);
    } else if constexpr (BITS == 2) {
        // pairs (q_j, q_{j+8}) from (w >> 2j) & 0x00030003; part p uses j = 2p, 2p+1
        const int s0 = 4 * part, s1 = 4 * part + 2;
        a[0] = lop3_and_or(w0 >> s0, 0x00030003u, 0x43004300u);
        a[1] = lop3_and_or(w1 >> s0, 0x00030003u, 0x43004300u);
        a[2] = lop3_and_or(w0 >> s1, 0x00030003u, 0x43004300u);
        a[3] = lop3_and_or(w1 >> s1, 0x00030003u, 0x43004300u);
    } else {
        // 8-bit: four codes per word; pairs (q0, q2), (q1, q3); byte -> 0x4B0000qq is the
        // fp32 2^23 + q, minus 2^23 = q (exact, and exact in bf16)
        auto pr = [](uint32_t w, uint32_t sel_lo, uint32_t sel_hi) {
            const float lo = __uint_as_float(prmt(w, 0x4B000000u, sel_lo)) - 8388608.0f;
            const float hi = __uint_as_float(prmt(w, 0x4B000000u, sel_hi)) - 8388608.0f;
            __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
            return *reinterpret_cast<uint32_t*>(&h);
        };
        (void)part;
        a[0] = pr(w0, 0x7440u, 0x7442u);
        a[1] = pr(w1, 0x7440u, 0x7442u);
        a[2] = pr(w0, 0x7441u, 0x7443u);
        a[3] = pr(w1, 0x7441u, 0x7443u);
    }
}

// x element offset `kl` (stage-relative) of token `tok` inside the stage's
// swizzled x boxes (each box: MMAX token rows of 128 bytes).
template <typename XT, int MMAX>
QLIN_DEV const uint8_t* x_addr(const uint8_t* xst, int tok, int kl)
{
    constexpr int XE = 128 / (int)sizeof(XT);
    const int b = kl / XE;
    const int o = (kl % XE) * (int)sizeof(XT);
    return xst + b * (MMAX * 128) + swz128(tok, o >> 4) + (o & 15);
}

// B-operand pairs for one word of one token (the word's CPW activations
// starting at stage offset kl); hi/lo parts for fp32 activations.  Tokens
// beyond M read the zeros the TMA wrote.
template <int BITS, typename XT, int NP, int MMAX>
QLIN_DEV void load_b_pairs(const uint8_t* xst, int tok, int kl, uint32_t (&bx)[NP], uint32_t (&bxl)[NP])
{
    uint32_t raw[NP], rawl[NP];
    if constexpr (sizeof(XT) == 2) {
        if constexpr (NP == 2) {  // 4 activations = 8 bytes
            const uint2 v = *reinterpret_cast<const uint2*>(x_addr<XT, MMAX>(xst, tok, kl));
            raw[0] = v.x; raw[1] = v.y;
        } else {                  // NP/4 units of 16 bytes
#pragma unroll
            for (int u = 0; u < NP / 4; ++u) {
                const uint4 v = *reinterpret_cast<const uint4*>(x_addr<XT, MMAX>(xst, tok, kl + 8 * u));
                raw[4 * u] = v.x; raw[4 * u + 1] = v.y; raw[4 * u + 2] = v.z; raw[4 * u + 3] = v.w;
            }
        }
#pragma unroll
        for (int q = 0; q < NP; ++q)
            rawl[q] = 0u;
    } else {
#pragma unroll
        for (int u = 0; u < NP / 2; ++u) {  // 4 floats per 16-byte unit
            const float4 v = *reinterpret_cast<const float4*>(x_addr<XT, MMAX>(xst, tok, kl + 4 * u));
            split_f32_pair(v.x, v.y, raw[2 * u], rawl[2 * u]);
            split_f32_pair(v.z, v.w, raw[2 * u + 1], rawl[2 * u + 1]);
        }
    }
    // raw[q] = (x_{2q}, x_{2q+1}); re-pair to match the A side
    if constexpr (BITS == 4) {
        bx[0] = pair_lo(raw[0], raw[2]);   // (x0, x4)
        bx[1] = pair_hi(raw[0], raw[2]);   // (x1, x5)
        bx[2] = pair_lo(raw[1], raw[3]);   // (x2, x6)
        bx[3] = pair_hi(raw[1], raw[3]);   // (x3, x7)
        bxl[0] = pair_lo(rawl[0], rawl[2]);
        bxl[1] = pair_hi(rawl[0], rawl[2]);
        bxl[2] = pair_lo(rawl[1], rawl[3]);
        bxl[3] = pair_hi(rawl[1], rawl[3]);
    } else if constexpr (BITS == 2) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // (x_{2i}, x_{2i+8}), (x_{2i+1}, x_{2i+9})
            bx[2 * i] = pair_lo(raw[i], raw[i + 4]);
            bx[2 * i + 1] = pair_hi(raw[i], raw[i + 4]);
            bxl[2 * i] = pair_lo(rawl[i], rawl[i + 4]);
            bxl[2 * i + 1] = pair_hi(rawl[i], rawl[i + 4]);
        }
    } else {
        bx[0] = pair_lo(raw[0], raw[1]);   // (x0, x2)
        bx[1] = pair_hi(raw[0], raw[1]);   // (x1, x3)
        bxl[0] = pair_lo(rawl[0], rawl[1]);
        bxl[1] = pair_hi(rawl[0], rawl[1]);
    }
}

// 32-bit word `wi` (stage-relative) of local row `row` in the swizzled weight
// boxes (each box: kRowsPerCta rows of 128 bytes).
QLIN_DEV uint32_t w_word(const uint8_t* wst, int rows, int row, int wi)
{
    const int b = wi >> 5, w = wi & 31;
    return *reinterpret_cast<const uint32_t*>(wst + b * (rows * 128) + swz128(row, w >> 2) + ((w & 3) << 2));
}

template <int BITS, int G, typename XT, typename PT, int NT>
__global__ void __launch_bounds__(kThreads, 2) affine_gemv_kernel(const __grid_constant__ AffineParams p)
{
    using Cfg = AffineCfg<BITS, G, XT, PT, NT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    const int params_bytes = round_up(kRowsPerCta * p.gstride * 8, 16);
    float2* params = reinterpret_cast<float2*>(smem + kStages * Cfg::STAGE);
    float* red = reinterpret_cast<float*>(smem + kStages * Cfg::STAGE + params_bytes);
    float* recv = red + Cfg::RED / 4;
    Barriers& bars = *reinterpret_cast<Barriers*>(reinterpret_cast<uint8_t*>(recv) + Cfg::recv_bytes(gridDim.x));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = gridDim.x;
    const int split = blockIdx.x;  // == rank in the cluster
    const int n0 = blockIdx.y * kRowsPerCta;
    const int kbeg = split * p.k_per_split;
    const int kend = min(p.K, kbeg + p.k_per_split);
    const int nst = kend > kbeg ? (kend - kbeg + Cfg::KST - 1) / Cfg::KST : 0;
    const int rows_valid = min(kRowsPerCta, p.N - n0);
    const int M = p.M;

    init_barriers(bars, S);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer warp
        producer_loop(
            bars, nst, p.status,
            [&](int it, int slot) {
                const int k0 = kbeg + it * Cfg::KST;
                uint8_t* wst = stages + slot * Cfg::STAGE;
                uint8_t* xst = wst + Cfg::W_STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_load_2d(wst + b * (kRowsPerCta * 128), &p.tm_w, k0 * BITS / 8 + b * 128, n0,
                                &bars.full[slot]);
#pragma unroll
                for (int b = 0; b < Cfg::NXB; ++b)
                    tma_load_2d(xst + b * (Cfg::MMAX * 128), &p.tm_x, k0 + b * Cfg::XE, 0, &bars.full[slot]);
            },
            [&](int it) {
                const int k0 = kbeg + it * Cfg::KST;
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_prefetch_2d(&p.tm_w, k0 * BITS / 8 + b * 128, n0);
            },
            [&](int) { return (unsigned)Cfg::STAGE; });
    } else {
        // ------------------------------------------------ consumer warps
        // zero the partial tile; group parameters of this CTA's rows and K-range -> smem as
        // {s, b - OFFSET s}: all loads issued before any store (one round trip)
        for (int e = threadIdx.x; e < Cfg::RED / 4; e += kConsumerThreads)
            red[e] = 0.f;
        {
            const int g0 = kbeg / G;
            const int ng = (kend - kbeg) / G;
            const int gpr = p.K / G;
            const PT* sc = static_cast<const PT*>(p.scales);
            const PT* bi = static_cast<const PT*>(p.biases);
            PT sv[Cfg::PARAMS_PER_THREAD], bv[Cfg::PARAMS_PER_THREAD];
#pragma unroll
            for (int i = 0; i < Cfg::PARAMS_PER_THREAD; ++i) {
                const int e = threadIdx.x + i * kConsumerThreads;
                const int r = e / ng, gl = e % ng;
                if (r < rows_valid && e < kRowsPerCta * ng && gl == 0) {
                    prefetch_l2(sc + (size_t)(n0 + r) * gpr + g0);
                    prefetch_l2(bi + (size_t)(n0 + r) * gpr + g0);
                }
            }
            pdl_wait_prior_grids();
#pragma unroll
            for (int i = 0; i < Cfg::PARAMS_PER_THREAD; ++i) {
                const int e = threadIdx.x + i * kConsumerThreads;
                const int r = e / ng, gl = e % ng;
                if (r < rows_valid && e < kRowsPerCta * ng) {
                    sv[i] = sc[(size_t)(n0 + r) * gpr + g0 + gl];
                    bv[i] = bi[(size_t)(n0 + r) * gpr + g0 + gl];
                }
            }
#pragma unroll
            for (int i = 0; i < Cfg::PARAMS_PER_THREAD; ++i) {
                const int e = threadIdx.x + i * kConsumerThreads;
                const int r = e / ng, gl = e % ng;
                if (e < kRowsPerCta * ng) {
                    float s = 0.f, b = 0.f;
                    if (r < rows_valid) {
                        s = to_float(sv[i]);
                        b = to_float(bv[i]);
                    }
                    params[r * p.gstride + gl] = make_float2(s, fmaf(-Cfg::OFFSET, s, b));
                }
            }
        }
        consumer_bar();

        const int gid = lane >> 2, tig = lane & 3;
        const int rt = warp % kRowTiles, kl_lane = warp / kRowTiles;
        const int row0 = rt * 16 + gid;  // local rows row0, row0 + 8
        float acc[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[t][i] = 0.f;
        const uint32_t ones[4] = {kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2};
        for (int it = 0; it < nst; ++it) {
            const int slot = it % kStages;
            if (!mbar_wait_bounded(&bars.full[slot], (it / kStages) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            const uint8_t* wst = stages + slot * Cfg::STAGE;
            const uint8_t* xst = wst + Cfg::W_STAGE;
            const int kst = min(Cfg::KST, kend - (kbeg + it * Cfg::KST));
            const int groups = kst / G;
            for (int gl = kl_lane; gl < groups; gl += kKLanes) {
                float d[NT][4], dx[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        d[t][i] = dx[t][i] = 0.f;
#pragma unroll
                for (int j = 0; j < Cfg::WPL; ++j) {
                    const int wi = gl * Cfg::WPG + j * 4 + tig;  // word index in the stage row
                    const uint32_t w0 = w_word(wst, kRowsPerCta, row0, wi);
                    const uint32_t w1 = w_word(wst, kRowsPerCta, row0 + 8, wi);
                    const int kl = wi * Cfg::CPW;                // k offset of the word in the stage
                    uint32_t bx[NT][Cfg::NP], bxl[NT][Cfg::NP];
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        load_b_pairs<BITS, XT, Cfg::NP, Cfg::MMAX>(xst, t * 8 + gid, kl, bx[t], bxl[t]);
#pragma unroll
                    for (int part = 0; part < Cfg::NP / 2; ++part) {
                        uint32_t a[4];
                        make_a_regs<BITS>(w0, w1, part, a);
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            mma_bf16_16816(d[t], a, bx[t][2 * part], bx[t][2 * part + 1]);
                            mma_bf16_16816(dx[t], ones, bx[t][2 * part], bx[t][2 * part + 1]);
                            if constexpr (sizeof(XT) == 4) {
                                mma_bf16_16816(d[t], a, bxl[t][2 * part], bxl[t][2 * part + 1]);
                                mma_bf16_16816(dx[t], ones, bxl[t][2 * part], bxl[t][2 * part + 1]);
                            }
                        }
                    }
                }
                // group epilogue: acc += s * D' + (b - OFFSET s) * X
                const int gidx = it * (Cfg::KST / G) + gl;
                const float2 pr0 = params[row0 * p.gstride + gidx];
                const float2 pr1 = params[(row0 + 8) * p.gstride + gidx];
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    acc[t][0] = fmaf(pr0.x, d[t][0], fmaf(pr0.y, dx[t][0], acc[t][0]));
                    acc[t][1] = fmaf(pr0.x, d[t][1], fmaf(pr0.y, dx[t][1], acc[t][1]));
                    acc[t][2] = fmaf(pr1.x, d[t][2], fmaf(pr1.y, dx[t][2], acc[t][2]));
                    acc[t][3] = fmaf(pr1.x, d[t][3], fmaf(pr1.y, dx[t][3], acc[t][3]));
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.empty[slot]);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int c0 = t * 8 + 2 * tig;
            atomicAdd(&red[c0 * kRedStride + row0], acc[t][0]);
            atomicAdd(&red[(c0 + 1) * kRedStride + row0], acc[t][1]);
            atomicAdd(&red[c0 * kRedStride + row0 + 8], acc[t][2]);
            atomicAdd(&red[(c0 + 1) * kRedStride + row0 + 8], acc[t][3]);
        }
    }
    using OT = XT;
    const OT* bias = static_cast<const OT*>(p.bias);
    OT* y = static_cast<OT*>(p.y);
    cluster_reduce(bars, red, recv, M, S, p.status, [&](int tok, int r, float v) {
        if (r < rows_valid) {
            if (bias)
                v += to_float(bias[n0 + r]);
            y[(size_t)tok * p.N + n0 + r] = from_float<OT>(v);
        }
    });
}

// ---------------------------------------------------------------- BitLinear decode kernel

template <int NT>
struct BitCfg {
    static constexpr int PROWS = kRowsPerCta / 4;   // packed rows per CTA (16) -> 64 output rows
    static constexpr int KST = 512;                 // k (bytes per packed row) per stage
    static constexpr int NWB = KST / 128;           // 128-byte weight boxes per stage
    static constexpr int NXB = KST * 2 / 128;       // 128-byte x boxes per stage
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = NWB * PROWS * 128;
    static constexpr int X_STAGE = NXB * MMAX * 128;
    static constexpr int STAGE = W_STAGE + X_STAGE;
    static_assert(STAGE % 1024 == 0, "swizzled boxes need 1024-byte alignment");
    static constexpr int RED = MMAX * kRedStride * 4;
    static constexpr int recv_bytes(int S) { return S * MMAX * kRowsPerCta * 4; }
    static constexpr int smem_bytes(int S) { return kStages * STAGE + RED + recv_bytes(S) + (int)sizeof(Barriers) + 1024; }
};

struct BitParams {
    CUtensorMap tm_w;  // packed [N/4][K] bytes, box {128 B, 16 rows}
    CUtensorMap tm_x;  // x [M][K] bf16, box {64 elements, 8*NT tokens}
    const uint8_t* packed;
    const __nv_bfloat16* x;
    const float* weight_scale;
    const __nv_bfloat16* bias;
    __nv_bfloat16* y;
    int M, K, N, R;  // R = N / 4
    int k_per_split;
    int invert;
    unsigned* status;
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 2) bitlinear_gemv_kernel(const __grid_constant__ BitParams p)
{
    using Cfg = BitCfg<NT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    float* red = reinterpret_cast<float*>(smem + kStages * Cfg::STAGE);
    float* recv = red + Cfg::RED / 4;
    Barriers& bars = *reinterpret_cast<Barriers*>(reinterpret_cast<uint8_t*>(recv) + Cfg::recv_bytes(gridDim.x));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = gridDim.x;
    const int split = blockIdx.x;
    const int p0 = blockIdx.y * Cfg::PROWS;
    const int kbeg = split * p.k_per_split;
    const int kend = min(p.K, kbeg + p.k_per_split);
    const int nst = kend > kbeg ? (kend - kbeg + Cfg::KST - 1) / Cfg::KST : 0;
    const int M = p.M;

    init_barriers(bars, S);

    if (warp == kConsumerWarps) {
        producer_loop(
            bars, nst, p.status,
            [&](int it, int slot) {
                const int k0 = kbeg + it * Cfg::KST;
                uint8_t* wst = stages + slot * Cfg::STAGE;
                uint8_t* xst = wst + Cfg::W_STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_load_2d(wst + b * (Cfg::PROWS * 128), &p.tm_w, k0 + b * 128, p0, &bars.full[slot]);
#pragma unroll
                for (int b = 0; b < Cfg::NXB; ++b)
                    tma_load_2d(xst + b * (Cfg::MMAX * 128), &p.tm_x, k0 + b * 64, 0, &bars.full[slot]);
            },
            [&](int it) {
                const int k0 = kbeg + it * Cfg::KST;
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_prefetch_2d(&p.tm_w, k0 + b * 128, p0);
            },
            [&](int) { return (unsigned)Cfg::STAGE; });
    } else {
        for (int e = threadIdx.x; e < Cfg::RED / 4; e += kConsumerThreads)
            red[e] = 0.f;
        consumer_bar();
        const int gid = lane >> 2, tig = lane & 3;
        const int rt = warp % kRowTiles, kl_lane = warp / kRowTiles;
        const int prow = rt * 4 + (gid & 3);  // local packed row of both A rows of this lane
        const int sh0 = 2 * (gid >> 2);       // field j of A row gid; row gid+8 uses j+2
        // two accumulator sets (even / odd steps) halve the MMA dependency chain
        float acc[2][NT][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc[h][t][i] = 0.f;
        for (int it = 0; it < nst; ++it) {
            const int slot = it % kStages;
            if (!mbar_wait_bounded(&bars.full[slot], (it / kStages) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            const uint8_t* wst = stages + slot * Cfg::STAGE;
            const uint8_t* xst = wst + Cfg::W_STAGE;
            const int kst = min(Cfg::KST, kend - (kbeg + it * Cfg::KST));
            const int steps = kst / 16;
            const int s_half = (steps + 1) / 2;
            const int s_beg = kl_lane * s_half;
            const int s_end = min(steps, s_beg + s_half);
            // one k16 step: A from the word of this lane, B from x; accumulates into acc_h
            auto step = [&](int s, float (&acc_h)[NT][4]) {
                const int wi = s * 4 + tig;  // word of 4 bytes (k = 4 wi .. 4 wi + 3)
                const uint32_t w = w_word(wst, Cfg::PROWS, prow, wi);
                uint32_t a[4];
                // (c + 128) pairs, then + (-129, -129): the exact weights c - 1.
                // row gid: field j = sh0 / 2, pairs (k, k+2) and (k+1, k+3); row gid+8: field j + 2
                a[0] = bf16x2_add(lop3_and_or(w >> sh0, 0x00030003u, 0x43004300u), kMinus129Bf16x2);
                a[2] = bf16x2_add(lop3_and_or(w >> (sh0 + 8), 0x00030003u, 0x43004300u), kMinus129Bf16x2);
                a[1] = bf16x2_add(lop3_and_or(w >> (sh0 + 4), 0x00030003u, 0x43004300u), kMinus129Bf16x2);
                a[3] = bf16x2_add(lop3_and_or(w >> (sh0 + 12), 0x00030003u, 0x43004300u), kMinus129Bf16x2);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    // tokens >= M read the zeros the TMA wrote
                    const uint2 v = *reinterpret_cast<const uint2*>(
                        x_addr<__nv_bfloat16, Cfg::MMAX>(xst, t * 8 + gid, 4 * wi));
                    mma_bf16_16816(acc_h[t], a, pair_lo(v.x, v.y), pair_hi(v.x, v.y));  // (x_k, x_{k+2}), (x_{k+1}, x_{k+3})
                }
            };
            int s = s_beg;
#pragma unroll 2
            for (; s + 1 < s_end; s += 2) {
                step(s, acc[0]);
                step(s + 1, acc[1]);
            }
            if (s < s_end)
                step(s, acc[0]);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.empty[slot]);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int c0 = t * 8 + 2 * tig;
            const int r0 = rt * 16 + gid;
            atomicAdd(&red[c0 * kRedStride + r0], acc[0][t][0] + acc[1][t][0]);
            atomicAdd(&red[(c0 + 1) * kRedStride + r0], acc[0][t][1] + acc[1][t][1]);
            atomicAdd(&red[c0 * kRedStride + r0 + 8], acc[0][t][2] + acc[1][t][2]);
            atomicAdd(&red[(c0 + 1) * kRedStride + r0 + 8], acc[0][t][3] + acc[1][t][3]);
        }
    }
    pdl_wait_prior_grids();  // weight_scale may come from an earlier kernel
    const float ws = *p.weight_scale;
    const float scale = p.invert ? __fdiv_rn(1.0f, ws) : ws;
    cluster_reduce(bars, red, recv, M, S, p.status, [&](int tok, int i, float v) {
        // local row i: row tile i / 16; A row ii = i % 16 -> packed row 4 (i / 16) + ii % 4, field ii / 4
        const int ii = i % 16;
        const int pr = p0 + (i / 16) * 4 + (ii & 3);
        if (pr < p.R) {
            const int n = pr + (ii >> 2) * p.R;
            v *= scale;
            if (p.bias)
                v += __bfloat162float(p.bias[n]);
            p.y[(size_t)tok * p.N + n] = __float2bfloat16_rn(v);
        }
    });
}

// ---------------------------------------------------------------- launch helpers

struct SplitPlan {
    int S;
    int k_per_split;
};

SplitPlan plan_splits(int tiles, int K, int kst, int sm_count, int max_k_per_split)
{
    const int nst = (K + kst - 1) / kst;
    int S = (2 * sm_count + tiles - 1) / tiles;
    S = S < 1 ? 1 : (S > kMaxCluster ? kMaxCluster : S);
    const int min_s = (K + max_k_per_split - 1) / max_k_per_split;
    if (S < min_s)
        S = min_s;
    if (S > nst)
        S = nst;
    const int sps = (nst + S - 1) / S;
    SplitPlan pl;
    pl.S = (nst + sps - 1) / sps;
    pl.k_per_split = sps * kst;
    return pl;
}

template <typename Kern, typename Params>
cudaError_t launch_cluster(Kern kern, dim3 grid, int smem, int cluster_x, cudaStream_t st, const Params& prm)
{
    if (cluster_x > kMaxCluster)
        return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int BITS, int G, typename XT, typename PT, int NT>
cudaError_t affine_launch_t(const AffineGemvArgs& a, int m0, int mcount, cudaStream_t st, const DeviceInfo& dev)
{
    using Cfg = AffineCfg<BITS, G, XT, PT, NT>;
    const int tiles = (int)((a.N + kRowsPerCta - 1) / kRowsPerCta);
    const SplitPlan pl = plan_splits(tiles, (int)a.K, Cfg::KST, dev.sm_count, Cfg::MAX_GROUPS * G);
    if (pl.k_per_split / G > Cfg::MAX_GROUPS)
        return cudaErrorNotSupported;
    AffineParams prm;
    prm.codes = reinterpret_cast<const uint8_t*>(a.codes);
    prm.x = static_cast<const uint8_t*>(a.x) + (size_t)m0 * a.K * sizeof(XT);
    prm.scales = a.scales;
    prm.biases = a.biases;
    prm.bias = a.bias;
    prm.y = static_cast<uint8_t*>(a.y) + (size_t)m0 * a.N * sizeof(XT);
    prm.M = mcount;
    prm.K = (int)a.K;
    prm.N = (int)a.N;
    prm.k_per_split = pl.k_per_split;
    prm.gstride = pl.k_per_split / G;
    prm.status = dev.status;
    const uint64_t row_bytes = (uint64_t)a.K * BITS / 8;
    if (!encode_tmap_2d(&prm.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, row_bytes, (uint64_t)a.N, row_bytes, 128,
                        kRowsPerCta) ||
        !encode_tmap_2d(&prm.tm_x, sizeof(XT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        prm.x, (uint64_t)a.K, (uint64_t)mcount, (uint64_t)a.K * sizeof(XT), Cfg::XE, Cfg::MMAX))
        return cudaErrorInvalidValue;
    return launch_cluster(affine_gemv_kernel<BITS, G, XT, PT, NT>, dim3(pl.S, tiles, 1),
                          Cfg::smem_bytes(prm.gstride, pl.S), pl.S, st, prm);
}

template <int BITS, int G, typename XT, typename PT>
cudaError_t affine_launch_nt(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    for (int64_t m0 = 0; m0 < a.M; m0 += 16) {
        const int mc = (int)(a.M - m0 < 16 ? a.M - m0 : 16);
        cudaError_t e = mc <= 8 ? affine_launch_t<BITS, G, XT, PT, 1>(a, (int)m0, mc, st, dev)
                                : affine_launch_t<BITS, G, XT, PT, 2>(a, (int)m0, mc, st, dev);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

template <int BITS, typename XT, typename PT>
cudaError_t affine_launch_g(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    switch (a.g) {
    case 32:
        if constexpr (BITS == 2)
            return cudaErrorNotSupported;
        else
            return affine_launch_nt<BITS, 32, XT, PT>(a, st, dev);
    case 64: return affine_launch_nt<BITS, 64, XT, PT>(a, st, dev);
    default: return affine_launch_nt<BITS, 128, XT, PT>(a, st, dev);
    }
}

template <typename XT, typename PT>
cudaError_t affine_launch_b(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    switch (a.bits) {
    case 2: return affine_launch_g<2, XT, PT>(a, st, dev);
    case 4: return affine_launch_g<4, XT, PT>(a, st, dev);
    default: return affine_launch_g<8, XT, PT>(a, st, dev);
    }
}

}  // namespace

cudaError_t launch_affine_gemv(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    if (a.x_dt == QLIN_BF16)
        return a.p_dt == QLIN_BF16 ? affine_launch_b<__nv_bfloat16, __nv_bfloat16>(a, st, dev)
                                   : affine_launch_b<__nv_bfloat16, float>(a, st, dev);
    return a.p_dt == QLIN_BF16 ? affine_launch_b<float, __nv_bfloat16>(a, st, dev)
                               : affine_launch_b<float, float>(a, st, dev);
}

cudaError_t launch_bitlinear_gemv(const BitlinearArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    const int R = (int)(a.N / 4);
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
        prm.status = dev.status;
        cudaError_t e;
        const int tiles = (R + BitCfg<1>::PROWS - 1) / BitCfg<1>::PROWS;
        const SplitPlan pl = plan_splits(tiles, (int)a.K, BitCfg<1>::KST, dev.sm_count, 1 << 30);
        prm.k_per_split = pl.k_per_split;
        if (!encode_tmap_2d(&prm.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.packed, (uint64_t)a.K, (uint64_t)R,
                            (uint64_t)a.K, 128, BitCfg<1>::PROWS) ||
            !encode_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, prm.x, (uint64_t)a.K, (uint64_t)mc,
                            (uint64_t)a.K * 2, 64, mc <= 8 ? 8 : 16))
            return cudaErrorInvalidValue;
        if (mc <= 8)
            e = launch_cluster(bitlinear_gemv_kernel<1>, dim3(pl.S, tiles, 1), BitCfg<1>::smem_bytes(pl.S), pl.S, st,
                               prm);
        else
            e = launch_cluster(bitlinear_gemv_kernel<2>, dim3(pl.S, tiles, 1), BitCfg<2>::smem_bytes(pl.S), pl.S, st,
                               prm);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace qlin
