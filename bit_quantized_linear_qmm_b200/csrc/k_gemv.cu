// k_gemv.cu -- decode-regime (M <= 16) quantized GEMV kernels for sm_100a:
// the MLX-affine layer and the weight-streaming halves of W8A8 / W4A8.
// (BitLinear's decode kernel is in k_bitlinear.cu.)
//
//   affine:    y[m,n] = sum_k x[m,k] * (q[n,k]*s[n,k/g] + b[n,k/g]) + bias[n]
//              [nuvec-nn QuantizedLinear, forward / fields weight, scales,
//               biases; cider/ops.py pergroup_linear docstring, dequantize]
//
// Design (B200, HBM- and latency-bound):
//  * A CTA owns a block of output rows over the whole of K (about one CTA
//    per SM), so the only reduction is inside the CTA: no clusters, no
//    workspace, no global atomics.  A small footprint leaves room on each SM
//    for the next kernel in the stream, which programmatic dependent launch
//    releases at once.
//  * affine: one producer thread streams the block through a shared-memory
//    ring with 2-D tensor-map TMA (cp.async.bulk.tensor, 128-byte swizzle,
//    completion on mbarriers): one instruction moves a 128-byte column block
//    of all the CTA's weight rows, one the same columns of the M token rows
//    of x (the remaining token rows of the ring stay zero).  The weights of
//    the first stages (and the group parameters) are fetched before
//    griddepcontrol.wait, the next stages prefetched into L2, so a layer's
//    DRAM fetch overlaps the previous layer's tail.  Eight consumer warps
//    take whole groups round robin; each covers all the CTA's 16-row tiles,
//    so every x fragment serves them all.
//  * The MACs run on the tensor cores with the legacy mma.sync (weights as
//    the 16-row A operand, x as the n=8 B operand, fp32 accumulation);
//    partial tiles are summed through shared memory.
//  * affine: codes become bf16 with one LOP3 per pair: (w >> s) & 0x000F000F
//    | 0x43004300 is the bf16 pair (128 + q_i, 128 + q_j), exact.  The 128
//    offset and the group bias fold out per group with the group sums of x,
//    which an MMA against an all-ones A operand produces:
//      y = sum_g [ s_g * D'_g + (b_g - 128 s_g) * X_g ],
//      D'_g = sum_{k in g} (q_k + 128) x_k,  X_g = sum_{k in g} x_k.
//    (8-bit codes use no offset: bf16 holds 0..255 exactly.)  Because a dot
//    product over a group does not depend on the order of k, each lane pairs
//    codes in the order the LOP3 yields them and permutes x to match (PRMT).
//  * Every mbarrier wait is bounded (qlin::kWaitLimitNs); on expiry the
//    kernel records the timeout in the status word, stops issuing copies,
//    waits (bounded) for its copies in flight and runs to completion.
#include "qlin_common.cuh"

namespace qlin {
namespace {

constexpr int kRowTiles = 4;                       // 16-row MMA tiles per CTA
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;    // + one producer warp
constexpr int kRowsPerCta = 16 * kRowTiles;
constexpr int kStages = 12;                         // barrier slots; a kernel uses NS <= kStages
constexpr int kRingBytes = 80 * 1024;               // stage ring budget: two CTAs still fit per SM
constexpr int kRedStride = kRowsPerCta + 4;        // padded row of the partial tile (bank spread)

__host__ __device__ constexpr int round_up(int a, int b) { return (a + b - 1) / b * b; }

struct alignas(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int abort_flag;
};

QLIN_DEV bool volatile_abort(Barriers& b) { return *reinterpret_cast<volatile int*>(&b.abort_flag) != 0; }

QLIN_DEV void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory"); }

QLIN_DEV uint32_t pair_lo(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410); }  // (a.lo, b.lo)
QLIN_DEV uint32_t pair_hi(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632); }  // (a.hi, b.hi)

constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;      // (1.0, 1.0)

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
template <int NS, typename WFn, typename XFn, typename PFn, typename BytesFn>
QLIN_DEV void producer_loop(Barriers& bars, int nst, unsigned* status, WFn issue_w, XFn issue_x, PFn prefetch,
                            BytesFn stage_bytes)
{
    if ((threadIdx.x & 31) == 0) {
        // let the next kernel in the stream start its own prologue on whatever
        // SM room is left
        pdl_launch_dependents();
        const int pre = nst < NS ? nst : NS;
        const int npf = nst < 2 * NS ? nst : 2 * NS;
        // the layer's constant weights: the first NS stages straight into the
        // ring, the next NS into L2, all before the dependency wait
        for (int it = 0; it < pre; ++it) {
            mbar_arrive_expect_tx(&bars.full[it], stage_bytes(it));
            issue_w(it, it);
        }
        for (int it = pre; it < npf; ++it)
            prefetch(it);
        pdl_wait_prior_grids();
        for (int it = 0; it < pre; ++it)
            issue_x(it, it);
        int issued = pre;
        for (int it = pre; it < nst; ++it) {
            const int slot = it % NS;
            if (!mbar_wait_bounded(&bars.empty[slot], ((it / NS) & 1) ^ 1, status) || volatile_abort(bars))
                break;
            mbar_arrive_expect_tx(&bars.full[slot], stage_bytes(it));
            issue_w(it, slot);
            issue_x(it, slot);
            ++issued;
        }
        // Drain: no TMA load may still target this CTA's shared memory at exit.
        for (int it = issued - NS < 0 ? 0 : issued - NS; it < issued; ++it)
            mbar_wait_bounded(&bars.full[it % NS], (it / NS) & 1, status);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- CTA reduction

// Sums, over the consumer warps that cover the same rows, the F fragment
// values each lane holds (val(j)) and writes them to red[token * kRedStride +
// row] (pos(rg, j, lane, row, token)).  Warp w covers row group w % RG.  The
// stage ring (idle once every warp has left the main loop) is the scratch;
// no shared-memory atomics.
template <int F, int RG, typename ValFn, typename PosFn>
QLIN_DEV void cta_reduce(float* scratch, float* red, ValFn val, PosFn pos)
{
    constexpr int KL = kConsumerWarps / RG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    consumer_bar();  // every consumer warp is done with the stage ring
#pragma unroll
    for (int j = 0; j < F; ++j)
        scratch[(warp * F + j) * 32 + lane] = val(j);
    consumer_bar();
    for (int e = threadIdx.x; e < RG * F * 32; e += kConsumerThreads) {
        const int rg = e / (F * 32), j = (e / 32) % F, ln = e % 32;
        float v = 0.f;
#pragma unroll
        for (int k = 0; k < KL; ++k)
            v += scratch[((k * RG + rg) * F + j) * 32 + ln];
        int row, tok;
        pos(rg, j, ln, row, tok);
        red[tok * kRedStride + row] = v;
    }
}

QLIN_DEV void init_barriers(Barriers& bars)
{
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], kConsumerWarps);
        }
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
}

// Zeroes the token rows [m0, MMAX) of every x box of every stage: the TMA
// only writes the first M rows, and tokens past M must read as zero.
QLIN_DEV void zero_x_tail(uint8_t* stages, int ns, int stage_bytes, int w_stage, int nxb, int mmax, int m0)
{
    const int per_box = (mmax - m0) * 128 / 16;  // 16-byte units
    const int total = ns * nxb * per_box;
    for (int e = threadIdx.x; e < total; e += kConsumerThreads) {
        const int s = e / (nxb * per_box), b = (e / per_box) % nxb, u = e % per_box;
        *reinterpret_cast<uint4*>(stages + s * stage_bytes + w_stage + b * (mmax * 128) + m0 * 128 + u * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// ---------------------------------------------------------------- affine decode kernel

template <int BITS, int G, typename XT, typename PT, int NT, int RT>
struct AffineCfg {
    static constexpr int ROWS = 16 * RT;                   // output rows per CTA
    static constexpr int KST = 1024 / BITS > 256 ? 1024 / BITS : 256;  // k per stage
    static constexpr int NWB = KST * BITS / 8 / 128;       // 128-byte weight boxes per stage
    static constexpr int XE = 128 / (int)sizeof(XT);       // x elements per 128-byte box row
    static constexpr int NXB = KST / XE;                   // x boxes per stage
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = NWB * ROWS * 128;
    static constexpr int X_STAGE = NXB * MMAX * 128;
    static constexpr int STAGE = W_STAGE + X_STAGE;       // multiple of 1024
    static constexpr int NS = (kRingBytes / STAGE) < 2 ? 2 : ((kRingBytes / STAGE) > kStages ? kStages : (kRingBytes / STAGE));
    static constexpr int CPW = 32 / BITS;                  // codes per 32-bit word
    static constexpr int WPG = G * BITS / 32;              // words per row per group
    static constexpr int WPL = WPG / 4;                    // words per lane per row per group
    static constexpr int NP = CPW / 2;                     // bf16 pairs per word
    static constexpr int GPS = KST / G;                    // groups per full stage
    static_assert(WPL >= 1, "group too small for the decode lane mapping");
    static_assert(STAGE % 1024 == 0, "swizzled boxes need 1024-byte alignment");
    // bf16 holds 0..255 exactly but not 128 + q for q >= 128: 8-bit codes go unbiased
    static constexpr float OFFSET = BITS == 8 ? 0.0f : 128.0f;
    static constexpr int RED = MMAX * kRedStride * 4;
    static constexpr int params_bytes(int groups) { return round_up(ROWS * groups * 8, 16); }
    static constexpr int smem_bytes(int groups)
    {
        return NS * STAGE + params_bytes(groups) + RED + (int)sizeof(Barriers) + 1024;
    }
};

struct AffineParams {
    CUtensorMap tm_w;  // codes as bytes [N][K*BITS/8], box {128 B, ROWS rows}
    CUtensorMap tm_x;  // x [M][K], box {128 B, M tokens}
    const void* scales;
    const void* biases;
    const void* bias;
    void* y;
    int M, K, N;
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

template <int BITS, int G, typename XT, typename PT, int NT, int RT>
__global__ void __launch_bounds__(kThreads, 2) affine_gemv_kernel(const __grid_constant__ AffineParams p)
{
    using Cfg = AffineCfg<BITS, G, XT, PT, NT, RT>;
    constexpr int ROWS = Cfg::ROWS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    const int ng = p.K / G;  // groups per row
    float2* params = reinterpret_cast<float2*>(smem + Cfg::NS * Cfg::STAGE);
    float* red = reinterpret_cast<float*>(smem + Cfg::NS * Cfg::STAGE + Cfg::params_bytes(ng));
    Barriers& bars = *reinterpret_cast<Barriers*>(reinterpret_cast<uint8_t*>(red) + Cfg::RED);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * ROWS;
    const int nst = (p.K + Cfg::KST - 1) / Cfg::KST;
    const int rows_valid = min(ROWS, p.N - n0);
    const int M = p.M;

    init_barriers(bars);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer warp
        producer_loop<Cfg::NS>(
            bars, nst, p.status,
            [&](int it, int slot) {
                uint8_t* wst = stages + slot * Cfg::STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_load_2d(wst + b * (ROWS * 128), &p.tm_w, it * Cfg::KST * BITS / 8 + b * 128, n0,
                                &bars.full[slot]);
            },
            [&](int it, int slot) {
                uint8_t* xst = stages + slot * Cfg::STAGE + Cfg::W_STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NXB; ++b)
                    tma_load_2d(xst + b * (Cfg::MMAX * 128), &p.tm_x, it * Cfg::KST + b * Cfg::XE, 0, &bars.full[slot]);
            },
            [&](int it) {
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_prefetch_2d(&p.tm_w, it * Cfg::KST * BITS / 8 + b * 128, n0);
            },
            [&](int) { return (unsigned)(Cfg::W_STAGE + Cfg::NXB * M * 128); });
    } else {
        // ------------------------------------------------ consumer warps
        zero_x_tail(stages, Cfg::NS, Cfg::STAGE, Cfg::W_STAGE, Cfg::NXB, Cfg::MMAX, M);
        // group parameters of the CTA's rows -> smem as {s, b - OFFSET s}.  They are constants of
        // the layer, like the packed weights, so they are read before griddepcontrol.wait: one
        // 16-byte vector per thread and batch (the CTA's parameters are contiguous).
        {
            const PT* sc = static_cast<const PT*>(p.scales) + (size_t)n0 * ng;
            const PT* bi = static_cast<const PT*>(p.biases) + (size_t)n0 * ng;
            constexpr int VE = 16 / (int)sizeof(PT);
            const int total = rows_valid * ng;
            const bool vec = ((reinterpret_cast<uintptr_t>(sc) | reinterpret_cast<uintptr_t>(bi)) & 15u) == 0;
#pragma unroll 4
            for (int c = threadIdx.x; c * VE < ROWS * ng; c += kConsumerThreads) {
                const int e0 = c * VE;
                float sv[VE], bv[VE];
                if (vec && e0 + VE <= total) {
                    const uint4 s4 = ldg_stream_v4(sc + e0), b4 = ldg_stream_v4(bi + e0);
                    const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w}, bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                    for (int e = 0; e < VE; ++e) {
                        if constexpr (sizeof(PT) == 2) {  // bf16: two per word, low half first
                            sv[e] = __uint_as_float((sw[e >> 1] >> (16 * (e & 1))) << 16);
                            bv[e] = __uint_as_float((bw[e >> 1] >> (16 * (e & 1))) << 16);
                        } else {
                            sv[e] = __uint_as_float(sw[e]);
                            bv[e] = __uint_as_float(bw[e]);
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < VE; ++e) {
                        sv[e] = e0 + e < total ? to_float(sc[e0 + e]) : 0.f;
                        bv[e] = e0 + e < total ? to_float(bi[e0 + e]) : 0.f;
                    }
                }
#pragma unroll
                for (int e = 0; e < VE; ++e)
                    if (e0 + e < ROWS * ng)
                        params[e0 + e] = make_float2(sv[e], fmaf(-Cfg::OFFSET, sv[e], bv[e]));
            }
        }
        pdl_wait_prior_grids();  // x, y and the bias may belong to the previous kernel
        consumer_bar();

        // every warp covers all RT row tiles (sharing each x fragment and the
        // group-sum MMA among them) and takes whole groups round robin
        const int gid = lane >> 2, tig = lane & 3;
        float acc[RT][NT][4];
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[i][t][e] = 0.f;
        const uint32_t ones[4] = {kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2};
        for (int it = 0; it < nst; ++it) {
            const int slot = it % Cfg::NS;
            if (!mbar_wait_bounded(&bars.full[slot], (it / Cfg::NS) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            const uint8_t* wst = stages + slot * Cfg::STAGE;
            const uint8_t* xst = wst + Cfg::W_STAGE;
            const int kst = min(Cfg::KST, p.K - it * Cfg::KST);
            const int groups = kst / G;
            for (int gl = (warp - it * Cfg::GPS % kConsumerWarps + kConsumerWarps) % kConsumerWarps; gl < groups;
                 gl += kConsumerWarps) {
                float d[RT][NT][4], dx[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dx[t][e] = 0.f;
#pragma unroll
                    for (int i = 0; i < RT; ++i)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            d[i][t][e] = 0.f;
                }
#pragma unroll
                for (int j = 0; j < Cfg::WPL; ++j) {
                    const int wi = gl * Cfg::WPG + j * 4 + tig;  // word index in the stage row
                    uint32_t w[RT][2];
#pragma unroll
                    for (int i = 0; i < RT; ++i) {
                        w[i][0] = w_word(wst, ROWS, i * 16 + gid, wi);
                        w[i][1] = w_word(wst, ROWS, i * 16 + gid + 8, wi);
                    }
                    const int kl = wi * Cfg::CPW;  // k offset of the word in the stage
                    uint32_t bx[NT][Cfg::NP], bxl[NT][Cfg::NP];
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        load_b_pairs<BITS, XT, Cfg::NP, Cfg::MMAX>(xst, t * 8 + gid, kl, bx[t], bxl[t]);
#pragma unroll
                    for (int part = 0; part < Cfg::NP / 2; ++part) {
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            mma_bf16_16816(dx[t], ones, bx[t][2 * part], bx[t][2 * part + 1]);
                            if constexpr (sizeof(XT) == 4)
                                mma_bf16_16816(dx[t], ones, bxl[t][2 * part], bxl[t][2 * part + 1]);
                        }
#pragma unroll
                        for (int i = 0; i < RT; ++i) {
                            uint32_t a[4];
                            make_a_regs<BITS>(w[i][0], w[i][1], part, a);
#pragma unroll
                            for (int t = 0; t < NT; ++t) {
                                mma_bf16_16816(d[i][t], a, bx[t][2 * part], bx[t][2 * part + 1]);
                                if constexpr (sizeof(XT) == 4)
                                    mma_bf16_16816(d[i][t], a, bxl[t][2 * part], bxl[t][2 * part + 1]);
                            }
                        }
                    }
                }
                // group epilogue: acc += s * D' + (b - OFFSET s) * X
                const int gidx = it * Cfg::GPS + gl;
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const int row = i * 16 + gid;
                    const float2 pr0 = params[row * ng + gidx];
                    const float2 pr1 = params[(row + 8) * ng + gidx];
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        acc[i][t][0] = fmaf(pr0.x, d[i][t][0], fmaf(pr0.y, dx[t][0], acc[i][t][0]));
                        acc[i][t][1] = fmaf(pr0.x, d[i][t][1], fmaf(pr0.y, dx[t][1], acc[i][t][1]));
                        acc[i][t][2] = fmaf(pr1.x, d[i][t][2], fmaf(pr1.y, dx[t][2], acc[i][t][2]));
                        acc[i][t][3] = fmaf(pr1.x, d[i][t][3], fmaf(pr1.y, dx[t][3], acc[i][t][3]));
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.empty[slot]);
        }
        cta_reduce<RT * NT * 4, 1>(
            reinterpret_cast<float*>(stages), red,
            [&](int j) { return acc[j / (NT * 4)][(j / 4) % NT][j % 4]; },
            [&](int, int j, int ln, int& row, int& tok) {
                const int i = j / (NT * 4), t = (j / 4) % NT, e = j % 4;
                row = i * 16 + (ln >> 2) + (e >= 2 ? 8 : 0);
                tok = t * 8 + 2 * (ln & 3) + (e & 1);
            });
        consumer_bar();
        using OT = XT;
        const OT* bias = static_cast<const OT*>(p.bias);
        OT* y = static_cast<OT*>(p.y);
        for (int e = threadIdx.x; e < M * ROWS; e += kConsumerThreads) {
            const int tok = e / ROWS, r = e % ROWS;
            if (r < rows_valid) {
                float v = red[tok * kRedStride + r];
                if (bias)
                    v += to_float(bias[n0 + r]);
                y[(size_t)tok * p.N + n0 + r] = from_float<OT>(v);
            }
        }
    }
}

// ---------------------------------------------------------------- W8A8 decode kernel

// y[m,n] = (float)(sum_k qx[m,k] * w[n,k]) * s_x[m] * s_w[n] + bias[n]
// [cider/ops.py perchannel_linear], M <= 16.  The same pipeline as the affine
// decode kernel (TMA stage ring fed by one producer thread, the weights of the
// first stages fetched before griddepcontrol.wait), with no dequantisation:
// int8 weights and int8 activations go straight into mma.m16n8k32.s8 (int32
// accumulation, exact).  Warps take k32 steps round robin; the partial int32
// tiles are summed in any order (exact) through shared memory.
template <int NT, int RT>
struct W8Cfg {
    static constexpr int ROWS = 16 * RT;
    static constexpr int KST = RT == 4 ? 256 : 512;  // k per stage (a ring of at least 3 stages)
    static constexpr int NWB = KST / 128;            // 128-byte weight boxes per stage
    static constexpr int NXB = KST / 128;            // 128-byte x boxes per stage
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = NWB * ROWS * 128;
    static constexpr int X_STAGE = NXB * MMAX * 128;
    static constexpr int STAGE = W_STAGE + X_STAGE;  // multiple of 1024
    static constexpr int NS = (kRingBytes / STAGE) < 2 ? 2 : ((kRingBytes / STAGE) > kStages ? kStages : (kRingBytes / STAGE));
    static constexpr int SMEM = NS * STAGE + (int)sizeof(Barriers) + 1024;
    static_assert(STAGE % 1024 == 0, "swizzled boxes need 1024-byte alignment");
    static_assert(kConsumerWarps * RT * NT * 4 * 32 * 4 <= NS * STAGE, "reduction scratch fits the ring");
};

struct W8Params {
    CUtensorMap tm_w;  // w [N][K] int8, box {128 B, ROWS rows}
    CUtensorMap tm_x;  // qx [M][K] int8, box {128 B, M rows}
    const float* s_x;
    const float* s_w;
    const unsigned short* bias;  // [N] bf16, or fp16 when out_f16
    unsigned short* y;           // [M][N] bf16, or fp16 when out_f16
    int out_f16;
    int M, K, N;
    unsigned* status;
};

template <int NT, int RT>
__global__ void __launch_bounds__(kThreads, 2) w8_gemv_kernel(const __grid_constant__ W8Params p)
{
    using Cfg = W8Cfg<NT, RT>;
    constexpr int ROWS = Cfg::ROWS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    Barriers& bars = *reinterpret_cast<Barriers*>(smem + Cfg::NS * Cfg::STAGE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * ROWS;
    const int nst = (p.K + Cfg::KST - 1) / Cfg::KST;
    const int M = p.M;

    init_barriers(bars);

    if (warp == kConsumerWarps) {
        producer_loop<Cfg::NS>(
            bars, nst, p.status,
            [&](int it, int slot) {
                uint8_t* wst = stages + slot * Cfg::STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_load_2d(wst + b * (ROWS * 128), &p.tm_w, it * Cfg::KST + b * 128, n0, &bars.full[slot]);
            },
            [&](int it, int slot) {
                uint8_t* xst = stages + slot * Cfg::STAGE + Cfg::W_STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NXB; ++b)
                    tma_load_2d(xst + b * (Cfg::MMAX * 128), &p.tm_x, it * Cfg::KST + b * 128, 0, &bars.full[slot]);
            },
            [&](int it) {
#pragma unroll
                for (int b = 0; b < Cfg::NWB; ++b)
                    tma_prefetch_2d(&p.tm_w, it * Cfg::KST + b * 128, n0);
            },
            [&](int) { return (unsigned)(Cfg::W_STAGE + Cfg::NXB * M * 128); });
    } else {
        // ------------------------------------------------ consumer warps
        zero_x_tail(stages, Cfg::NS, Cfg::STAGE, Cfg::W_STAGE, Cfg::NXB, Cfg::MMAX, M);
        consumer_bar();
        const int gid = lane >> 2, tig = lane & 3;
        int acc[RT][NT][4];
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[i][t][e] = 0;
        for (int it = 0; it < nst; ++it) {
            const int slot = it % Cfg::NS;
            if (!mbar_wait_bounded(&bars.full[slot], (it / Cfg::NS) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            const uint8_t* wst = stages + slot * Cfg::STAGE;
            const uint8_t* xst = wst + Cfg::W_STAGE;
            // k past K reads the zeros the TMA wrote, in both operands
            const int steps = (min(Cfg::KST, p.K - it * Cfg::KST) + 31) / 32;
            for (int st = warp; st < steps; st += kConsumerWarps) {
                const int wi = st * 8;  // first 32-bit word of this k32 step in the stage row
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    b0[t] = *reinterpret_cast<const uint32_t*>(x_addr<int8_t, Cfg::MMAX>(xst, t * 8 + gid, 32 * st + 4 * tig));
                    b1[t] = *reinterpret_cast<const uint32_t*>(
                        x_addr<int8_t, Cfg::MMAX>(xst, t * 8 + gid, 32 * st + 16 + 4 * tig));
                }
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    uint32_t a[4];
                    a[0] = w_word(wst, ROWS, i * 16 + gid, wi + tig);
                    a[1] = w_word(wst, ROWS, i * 16 + gid + 8, wi + tig);
                    a[2] = w_word(wst, ROWS, i * 16 + gid, wi + 4 + tig);
                    a[3] = w_word(wst, ROWS, i * 16 + gid + 8, wi + 4 + tig);
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        mma_s8_16832(acc[i][t], a, b0[t], b1[t]);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.empty[slot]);
        }
        // sum the warps' partial tiles (int32: exact in any order); the idle stage ring is the scratch
        consumer_bar();
        int* scratch = reinterpret_cast<int*>(stages);
        constexpr int V = RT * NT * 4;
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    scratch[(warp * V + (i * NT + t) * 4 + e) * 32 + lane] = acc[i][t][e];
        consumer_bar();
        pdl_wait_prior_grids();  // s_x comes from the activation quantiser; y and bias after it too
        for (int idx = threadIdx.x; idx < V * 32; idx += kConsumerThreads) {
            const int v = idx >> 5, ln = idx & 31;
            int sum = 0;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w)
                sum += scratch[(w * V + v) * 32 + ln];
            const int i = v / (NT * 4), t = (v / 4) % NT, e = v % 4;
            const int row = i * 16 + (ln >> 2) + (e >= 2 ? 8 : 0);
            const int tok = t * 8 + 2 * (ln & 3) + (e & 1);
            const int n = n0 + row;
            if (tok < M && n < p.N) {
                float out = (float)sum * (p.s_x[tok] * p.s_w[n]);
                if (p.bias)
                    out += h16_to_float(p.bias[n], p.out_f16);
                p.y[(size_t)tok * p.N + n] = to_h16(out, p.out_f16);
            }
        }
    }
}

// ---------------------------------------------------------------- W4A8 decode kernel

// y[m,n] = (float)(sum_k qx[m,k] * (c[k,n] - 8)) * s_x[m] * s_w[n] (+ bias[n])
// [cider/ops.py w4a8_linear, pack_weight_int4], M <= 16.  The packed weights
// are [K/2][N] bytes (N contiguous, high nibble = even k); a CTA streams a
// 64-column strip through the TMA stage ring (boxes of 64 bytes x 256 k-pair
// rows).  Per k32 step a lane reads four 32-bit words -- columns 4g .. 4g+3 of
// k-pair rows 4t .. 4t+3 -- and turns them with PRMT into the int8 A
// fragments of two 16-row tiles (columns 4g, 4g+1 and 4g+2, 4g+3 as rows g,
// g+8), each nibble c as 16 (c - 8) (bit 3 flipped, kept in the high half of
// the byte); the MMA's k slots 4t .. 4t+3 / 16+4t .. 16+4t+3 stand for
// k = 8t .. 8t+3 / 8t+4 .. 8t+7, so x is one 8-byte read.  The exact int32
// sum is shifted back by 4 bits in the epilogue.
template <int NT>
struct W4Cfg {
    static constexpr int COLS = 64;                   // output columns per CTA
    static constexpr int KP = 256;                    // k-pair rows per stage (512 k)
    static constexpr int KST = 2 * KP;
    static constexpr int NXB = KST / 128;             // 128-byte x boxes per stage
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = KP * COLS;         // 16 KB
    static constexpr int X_STAGE = NXB * MMAX * 128;
    static constexpr int STAGE = W_STAGE + X_STAGE;   // multiple of 1024
    static constexpr int NS = (kRingBytes / STAGE) < 2 ? 2 : ((kRingBytes / STAGE) > kStages ? kStages : (kRingBytes / STAGE));
    static constexpr int V = 2 * NT * 4;              // accumulators per lane
    static constexpr int SMEM = NS * STAGE + (int)sizeof(Barriers) + 1024;
    static_assert(STAGE % 1024 == 0, "swizzled x boxes need 1024-byte alignment");
    static_assert(kConsumerWarps * V * 32 * 4 <= NS * STAGE, "reduction scratch fits the ring");
};

struct W4Params {
    CUtensorMap tm_w;  // packed [K/2][N] bytes, box {64 B, 256 rows}, no swizzle
    CUtensorMap tm_x;  // qx [M][K] int8, box {128 B, M rows}
    const float* s_x;
    const float* s_w;
    const unsigned short* bias;  // [N] bf16, or fp16 when out_f16
    unsigned short* y;           // [M][N] bf16, or fp16 when out_f16
    int out_f16;
    int M, K, N;
    unsigned* status;
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 2) w4_gemv_kernel(const __grid_constant__ W4Params p)
{
    using Cfg = W4Cfg<NT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    Barriers& bars = *reinterpret_cast<Barriers*>(smem + Cfg::NS * Cfg::STAGE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = blockIdx.x * Cfg::COLS;
    const int nst = (p.K + Cfg::KST - 1) / Cfg::KST;
    const int M = p.M;

    init_barriers(bars);

    if (warp == kConsumerWarps) {
        producer_loop<Cfg::NS>(
            bars, nst, p.status,
            [&](int it, int slot) {
                tma_load_2d(stages + slot * Cfg::STAGE, &p.tm_w, c0, it * Cfg::KP, &bars.full[slot]);
            },
            [&](int it, int slot) {
                uint8_t* xst = stages + slot * Cfg::STAGE + Cfg::W_STAGE;
#pragma unroll
                for (int b = 0; b < Cfg::NXB; ++b)
                    tma_load_2d(xst + b * (Cfg::MMAX * 128), &p.tm_x, it * Cfg::KST + b * 128, 0, &bars.full[slot]);
            },
            [&](int it) { tma_prefetch_2d(&p.tm_w, c0, it * Cfg::KP); },
            [&](int) { return (unsigned)(Cfg::W_STAGE + Cfg::NXB * M * 128); });
    } else {
        // ------------------------------------------------ consumer warps
        zero_x_tail(stages, Cfg::NS, Cfg::STAGE, Cfg::W_STAGE, Cfg::NXB, Cfg::MMAX, M);
        consumer_bar();
        const int gid = lane >> 2, tig = lane & 3;
        const int cg = warp & 1;   // 32-column group of the strip
        const int kw = warp >> 1;  // k32 steps kw, kw + 4, ... of every stage
        int acc[2][NT][4];
#pragma unroll
        for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[t2][t][e] = 0;
        for (int it = 0; it < nst; ++it) {
            const int slot = it % Cfg::NS;
            if (!mbar_wait_bounded(&bars.full[slot], (it / Cfg::NS) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            const uint32_t* raw32 = reinterpret_cast<const uint32_t*>(stages + slot * Cfg::STAGE);
            const uint8_t* xst = stages + slot * Cfg::STAGE + Cfg::W_STAGE;
            // k past K: the TMA wrote zero codes and zero activations
            const int steps = (min(Cfg::KST, p.K - it * Cfg::KST) + 31) / 32;
            for (int st = kw; st < steps; st += 4) {
                uint32_t W[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    W[j] = raw32[(16 * st + 4 * tig + j) * (Cfg::COLS / 4) + 8 * cg + gid];
                uint32_t a[2][4];  // [tile][fragment register]
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // k-pair rows (0,1) -> slots 4t.., rows (2,3) -> slots 16+4t..
#pragma unroll
                    for (int t2 = 0; t2 < 2; ++t2) {  // tile: columns (4g, 4g+1) or (4g+2, 4g+3)
                        const uint32_t x = prmt(W[2 * h], W[2 * h + 1], t2 ? 0x7362u : 0x5140u) ^ 0x88888888u;
                        const uint32_t hi = x & 0xF0F0F0F0u;         // even k
                        const uint32_t lo = (x << 4) & 0xF0F0F0F0u;  // odd k
                        a[t2][2 * h] = prmt(hi, lo, 0x5140u);        // row g
                        a[t2][2 * h + 1] = prmt(hi, lo, 0x7362u);    // row g + 8
                    }
                }
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const uint2 xb = *reinterpret_cast<const uint2*>(x_addr<int8_t, Cfg::MMAX>(xst, t * 8 + gid, 32 * st + 8 * tig));
#pragma unroll
                    for (int t2 = 0; t2 < 2; ++t2) {
                        const uint32_t fa[4] = {a[t2][0], a[t2][1], a[t2][2], a[t2][3]};
                        mma_s8_16832(acc[t2][t], fa, xb.x, xb.y);
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.empty[slot]);
        }
        // sum the partial tiles of the four k warps of each column group (int32, exact)
        consumer_bar();
        int* scratch = reinterpret_cast<int*>(stages);
        constexpr int V = Cfg::V;
#pragma unroll
        for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    scratch[(warp * V + (t2 * NT + t) * 4 + e) * 32 + lane] = acc[t2][t][e];
        consumer_bar();
        pdl_wait_prior_grids();  // s_x comes from the activation quantiser; y and bias after it too
        for (int idx = threadIdx.x; idx < 2 * V * 32; idx += kConsumerThreads) {
            const int g2 = idx / (V * 32), v = (idx / 32) % V, ln = idx & 31;
            int sum = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                sum += scratch[((2 * q + g2) * V + v) * 32 + ln];
            const int t2 = v / (NT * 4), t = (v / 4) % NT, e = v % 4;
            const int col = c0 + 32 * g2 + 4 * (ln >> 2) + 2 * t2 + (e >= 2 ? 1 : 0);
            const int tok = t * 8 + 2 * (ln & 3) + (e & 1);
            if (tok < M && col < p.N) {
                float out = (float)(sum >> 4) * (p.s_x[tok] * p.s_w[col]);
                if (p.bias)
                    out += h16_to_float(p.bias[col], p.out_f16);
                p.y[(size_t)tok * p.N + col] = to_h16(out, p.out_f16);
            }
        }
    }
}

// ---------------------------------------------------------------- launch helpers

template <typename Kern, typename Params>
cudaError_t launch_pdl(Kern kern, dim3 grid, int smem, cudaStream_t st, const Params& prm)
{
    if (smem > 227 * 1024)
        return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int BITS, int G, typename XT, typename PT, int NT, int RT>
cudaError_t affine_launch_t(const AffineGemvArgs& a, int m0, int mcount, cudaStream_t st, const DeviceInfo& dev,
                            bool dry)
{
    using Cfg = AffineCfg<BITS, G, XT, PT, NT, RT>;
    (void)dev;
    // the CTA's group parameters live in shared memory beside the ring: long rows of small
    // groups do not fit (the caller then takes the general kernel)
    if (Cfg::smem_bytes((int)(a.K / G)) > 227 * 1024)
        return cudaErrorNotSupported;
    if (dry)
        return cudaSuccess;
    AffineParams prm;
    const void* x = static_cast<const uint8_t*>(a.x) + (size_t)m0 * a.K * sizeof(XT);
    prm.scales = a.scales;
    prm.biases = a.biases;
    prm.bias = a.bias;
    prm.y = static_cast<uint8_t*>(a.y) + (size_t)m0 * a.N * sizeof(XT);
    prm.M = mcount;
    prm.K = (int)a.K;
    prm.N = (int)a.N;
    prm.status = dev.status;
    const uint64_t row_bytes = (uint64_t)a.K * BITS / 8;
    if (!encode_tmap_2d(&prm.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, row_bytes, (uint64_t)a.N, row_bytes, 128,
                        Cfg::ROWS) ||
        !encode_tmap_2d(&prm.tm_x, sizeof(XT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        x, (uint64_t)a.K, (uint64_t)mcount, (uint64_t)a.K * sizeof(XT), Cfg::XE, (uint32_t)mcount))
        return cudaErrorInvalidValue;
    const int ctas = (int)((a.N + Cfg::ROWS - 1) / Cfg::ROWS);
    return launch_pdl(affine_gemv_kernel<BITS, G, XT, PT, NT, RT>, dim3(ctas, 1, 1), Cfg::smem_bytes((int)(a.K / G)),
                      st, prm);
}

template <int BITS, int G, typename XT, typename PT>
cudaError_t affine_launch_nt(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev, bool dry)
{
    // 64-row CTAs when that still gives about one CTA per SM, 32-row CTAs, or 16-row CTAs (two
    // working CTAs per SM) when even 32-row CTAs would leave SMs idle
    const bool wide = a.N / 64 >= dev.sm_count;
    const bool narrow = a.N / 32 < dev.sm_count;
    for (int64_t m0 = 0; m0 < a.M; m0 += 16) {
        const int mc = (int)(a.M - m0 < 16 ? a.M - m0 : 16);
        cudaError_t e;
        if (mc <= 8 && sizeof(XT) == 2)
            e = wide     ? affine_launch_t<BITS, G, XT, PT, 1, 4>(a, (int)m0, mc, st, dev, dry)
                : narrow ? affine_launch_t<BITS, G, XT, PT, 1, 1>(a, (int)m0, mc, st, dev, dry)
                         : affine_launch_t<BITS, G, XT, PT, 1, 2>(a, (int)m0, mc, st, dev, dry);
        else if (mc <= 8)
            e = affine_launch_t<BITS, G, XT, PT, 1, 2>(a, (int)m0, mc, st, dev, dry);
        else if (narrow && sizeof(XT) == 2)
            e = affine_launch_t<BITS, G, XT, PT, 2, 1>(a, (int)m0, mc, st, dev, dry);
        else
            e = affine_launch_t<BITS, G, XT, PT, 2, 2>(a, (int)m0, mc, st, dev, dry);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

template <int BITS, typename XT, typename PT>
cudaError_t affine_launch_g(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev, bool dry)
{
    switch (a.g) {
    case 32:
        if constexpr (BITS == 2)
            return cudaErrorNotSupported;
        else
            return affine_launch_nt<BITS, 32, XT, PT>(a, st, dev, dry);
    case 64: return affine_launch_nt<BITS, 64, XT, PT>(a, st, dev, dry);
    default: return affine_launch_nt<BITS, 128, XT, PT>(a, st, dev, dry);
    }
}

template <typename XT, typename PT>
cudaError_t affine_launch_b(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev, bool dry)
{
    switch (a.bits) {
    case 2: return affine_launch_g<2, XT, PT>(a, st, dev, dry);
    case 4: return affine_launch_g<4, XT, PT>(a, st, dev, dry);
    default: return affine_launch_g<8, XT, PT>(a, st, dev, dry);
    }
}

}  // namespace

cudaError_t launch_affine_gemv(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    auto run = [&](bool dry) {
        if (a.x_dt == QLIN_BF16)
            return a.p_dt == QLIN_BF16 ? affine_launch_b<__nv_bfloat16, __nv_bfloat16>(a, st, dev, dry)
                                       : affine_launch_b<__nv_bfloat16, float>(a, st, dev, dry);
        return a.p_dt == QLIN_BF16 ? affine_launch_b<float, __nv_bfloat16>(a, st, dev, dry)
                                   : affine_launch_b<float, float>(a, st, dev, dry);
    };
    // layers whose codes fit in shared memory over the SMs: the resident-weight kernel
    const cudaError_t ed = launch_affine_dec(a, st, dev);
    if (ed != cudaErrorNotSupported)
        return ed;
    // every launch of the call checked first, so that a call runs wholly on one kernel
    const cudaError_t e = run(true);
    if (e == cudaErrorNotSupported)
        return launch_affine_gemv_any(a, st, dev);
    return e != cudaSuccess ? e : run(false);
}

cudaError_t launch_w8_gemv(const W8GemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    const bool wide = a.N / 64 >= dev.sm_count;  // 64-row CTAs when they still fill the GPU
    for (int64_t m0 = 0; m0 < a.M; m0 += 16) {
        const int mc = (int)(a.M - m0 < 16 ? a.M - m0 : 16);
        W8Params prm;
        prm.s_x = a.s_x + m0;
        prm.s_w = a.s_w;
        prm.bias = static_cast<const unsigned short*>(a.bias);
        prm.y = static_cast<unsigned short*>(a.y) + m0 * a.N;
        prm.out_f16 = a.out_f16;
        prm.M = mc;
        prm.K = (int)a.K;
        prm.N = (int)a.N;
        prm.status = dev.status;
        const int rows = mc <= 8 && wide ? 64 : 32;
        if (!encode_tmap_2d(&prm.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.K,
                            128, (uint32_t)rows) ||
            !encode_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qx + m0 * a.K, (uint64_t)a.K, (uint64_t)mc,
                            (uint64_t)a.K, 128, (uint32_t)mc))
            return cudaErrorInvalidValue;
        const dim3 grid((unsigned)((a.N + rows - 1) / rows), 1, 1);
        cudaError_t e;
        if (mc <= 8 && wide)
            e = launch_pdl(w8_gemv_kernel<1, 4>, grid, W8Cfg<1, 4>::SMEM, st, prm);
        else if (mc <= 8)
            e = launch_pdl(w8_gemv_kernel<1, 2>, grid, W8Cfg<1, 2>::SMEM, st, prm);
        else
            e = launch_pdl(w8_gemv_kernel<2, 2>, grid, W8Cfg<2, 2>::SMEM, st, prm);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}


cudaError_t launch_w4_gemv(const W8GemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    for (int64_t m0 = 0; m0 < a.M; m0 += 16) {
        const int mc = (int)(a.M - m0 < 16 ? a.M - m0 : 16);
        W4Params prm;
        prm.s_x = a.s_x + m0;
        prm.s_w = a.s_w;
        prm.bias = static_cast<const unsigned short*>(a.bias);
        prm.y = static_cast<unsigned short*>(a.y) + m0 * a.N;
        prm.out_f16 = a.out_f16;
        prm.M = mc;
        prm.K = (int)a.K;
        prm.N = (int)a.N;
        prm.status = dev.status;
        if (!encode_tmap_2d(&prm.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w, (uint64_t)a.N, (uint64_t)(a.K / 2),
                            (uint64_t)a.N, W4Cfg<1>::COLS, W4Cfg<1>::KP, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qx + m0 * a.K, (uint64_t)a.K, (uint64_t)mc,
                            (uint64_t)a.K, 128, (uint32_t)mc))
            return cudaErrorInvalidValue;
        const dim3 grid((unsigned)((a.N + W4Cfg<1>::COLS - 1) / W4Cfg<1>::COLS), 1, 1);
        const cudaError_t e = mc <= 8 ? launch_pdl(w4_gemv_kernel<1>, grid, W4Cfg<1>::SMEM, st, prm)
                                      : launch_pdl(w4_gemv_kernel<2>, grid, W4Cfg<2>::SMEM, st, prm);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace qlin
