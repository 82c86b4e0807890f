// k_gemv.cu -- decode-regime (M <= 16) quantized GEMV kernels for sm_100a.
//
//   affine:    y[m,n] = sum_k x[m,k] * (q[n,k]*s[n,k/g] + b[n,k/g]) + bias[n]
//              [nuvec-nn QuantizedLinear, forward / fields weight, scales,
//               biases; cider/ops.py pergroup_linear docstring, dequantize]
//   bitlinear: y[m, r + j*N/4] = scale * sum_k x[m,k] * (((P[r,k] >> 2j) & 3) - 1) + bias
//              [mlx_lm bitlinear_layers.py, make_bitlinear_kernel, BitLinear.__call__]
//
// Design (B200, HBM-bound):
//  * A CTA owns a tile of 64 output rows x a K-range.  K is split over the
//    CTAs of a thread-block cluster; their fp32 partial tiles are summed
//    through distributed shared memory (no workspace, no atomics).
//  * One producer warp streams the tile through a 4-stage shared-memory ring
//    with 1-D bulk copies (cp.async.bulk, one per weight row and per token
//    row of x, completion on mbarriers).  Four consumer warps dequantise in
//    registers and run the MACs on the tensor cores with the legacy
//    mma.sync.m16n8k16 (weights as the 16-row A operand, x as the n=8 B
//    operand, fp32 accumulation), which keeps the ALU cost per code below
//    one instruction.
//  * Codes become bf16 with one LOP3 per pair: (word >> s) & 0x000F000F |
//    0x43004300 is the bf16 pair (128 + q_i, 128 + q_j), exact.  The 128
//    offset and the group bias are folded out per group with the group sums
//    of x, which an extra MMA against an all-ones A operand produces:
//      y = sum_g [ s_g * D'_g + (b_g - 128 s_g) * X_g ],
//      D'_g = sum_{k in g} (q_k + 128) x_k,  X_g = sum_{k in g} x_k.
//    Because the dot product over a group does not depend on the order of
//    k, each lane pairs codes in the order the LOP3 produces them and
//    permutes x to match (PRMT), instead of reordering the codes.
//  * Every mbarrier wait is bounded (qlin::kWaitLimitNs); on expiry the
//    kernel records QLIN timeout status, stops issuing copies, waits
//    (bounded) for its copies in flight and runs to completion.
#include "qlin_common.cuh"

namespace qlin {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kRowsPerCta = 16 * kConsumerWarps;
constexpr int kStages = 4;

__host__ __device__ constexpr int round_up(int a, int b) { return (a + b - 1) / b * b; }

// ---------------------------------------------------------------- shared pieces

struct alignas(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int abort_flag;
};

QLIN_DEV bool volatile_abort(Barriers& b) { return *reinterpret_cast<volatile int*>(&b.abort_flag) != 0; }

// x pairs for a 4-code word position: from regs X01=(x0,x1), X45=(x4,x5) etc.
QLIN_DEV uint32_t pair_lo(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410); }  // (a.lo, b.lo)
QLIN_DEV uint32_t pair_hi(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632); }  // (a.hi, b.hi)

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

constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;  // (1.0, 1.0)

// Producer: streams `nst` stages.  Lane 0 waits for free slots and arms the
// full barrier; every lane issues a share of the row copies.
template <typename IssueFn>
QLIN_DEV void producer_loop(Barriers& bars, int nst, unsigned* status, IssueFn issue)
{
    const int lane = threadIdx.x & 31;
    int issued = 0;
    for (int it = 0; it < nst; ++it) {
        const int slot = it % kStages;
        int ok = 1;
        if (lane == 0) {
            ok = mbar_wait_bounded(&bars.empty[slot], ((it / kStages) & 1) ^ 1, status) ? 1 : 0;
            if (ok && volatile_abort(bars))
                ok = 0;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok)
            break;
        issue(it, slot, lane);  // lane 0 arms full[slot] first, then __syncwarp, then copies
        ++issued;
    }
    // Drain: no bulk copy may still target this CTA's shared memory at exit.
    if (lane == 0) {
        for (int it = issued - kStages < 0 ? 0 : issued - kStages; it < issued; ++it)
            mbar_wait_bounded(&bars.full[it % kStages], (it / kStages) & 1, status);
    }
}

// ---------------------------------------------------------------- affine decode kernel

template <int BITS, int G, typename XT, typename PT, int NT>
struct AffineCfg {
    static constexpr int KST = 256;                        // k per stage
    static constexpr int RB = KST * BITS / 8;              // weight bytes per row per stage
    static constexpr int RBP = RB + 16;                    // padded smem row stride
    static constexpr int XB = KST * (int)sizeof(XT);       // x bytes per token per stage
    // token-row padding that keeps the x loads of one warp phase on distinct banks
    static constexpr int XBP = XB + (sizeof(XT) == 4 ? 16 : (BITS == 4 ? 64 : (BITS == 2 ? 16 : 32)));
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = kRowsPerCta * RBP;
    static constexpr int X_STAGE = MMAX * XBP;
    static constexpr int STAGE = round_up(W_STAGE + X_STAGE, 128);
    static constexpr int CPW = 32 / BITS;                  // codes per 32-bit word
    static constexpr int WPG = G * BITS / 32;              // words per row per group
    static constexpr int WPL = WPG / 4;                    // words per lane per row per group
    static constexpr int MAX_GROUPS = 64;                  // groups of params kept in smem per CTA
    static_assert(WPL >= 1, "group too small for the decode lane mapping");
    // bf16 holds 0..255 exactly but not 128 + q for q >= 128: 8-bit codes go unbiased
    static constexpr float OFFSET = BITS == 8 ? 0.0f : 128.0f;
    static constexpr int RED = MMAX * kRowsPerCta * 4;
    static constexpr int smem_bytes(int gstride)
    {
        return kStages * STAGE + kRowsPerCta * gstride * 8 + RED + (int)sizeof(Barriers) + 128;
    }
};

struct AffineParams {
    const uint8_t* codes;  // bytes of the uint32 words
    const void* x;
    const void* scales;
    const void* biases;
    const void* bias;
    void* y;
    int M, K, N;
    int k_per_split;      // multiple of KST
    int gstride;          // groups per row held in the smem parameter block (k_per_split / G)
    unsigned* status;
};

// Builds the A-operand registers for one mma from packed words of rows gid
// (w0) and gid+8 (w1); `part` selects which pairs of the word.
template <int BITS>
QLIN_DEV void make_a_regs(uint32_t w0, uint32_t w1, int part, uint32_t (&a)[4])
{
    if constexpr (BITS == 4) {
        // pairs (q_j, q_{j+4}) from (w >> 4j) & 0x000F000F; mma part 0 uses j=0,1; part 1 uses j=2,3
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
        // 8-bit: four codes per word; pairs (q0,q2), (q1,q3), exact q via an fp32 magic number
        auto pr = [](uint32_t w, uint32_t sel) {
            // byte -> 0x4B0000qq, the fp32 2^23 + q; minus 2^23 = q (exact, and exact in bf16)
            const float lo = __uint_as_float(prmt(w, 0x4B000000u, sel & 0xffffu)) - 8388608.0f;
            const float hi = __uint_as_float(prmt(w, 0x4B000000u, sel >> 16)) - 8388608.0f;
            __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
            return *reinterpret_cast<uint32_t*>(&h);
        };
        // selectors: byte i of w into byte 0, zero bytes (index 4,5 of 0x4B000000 = 0x00), 0x4B (index 7)
        const uint32_t sel02 = (0x7440u + 0u) | ((0x7440u + 2u) << 16);
        const uint32_t sel13 = (0x7440u + 1u) | ((0x7440u + 3u) << 16);
        (void)part;
        a[0] = pr(w0, sel02);
        a[1] = pr(w1, sel02);
        a[2] = pr(w0, sel13);
        a[3] = pr(w1, sel13);
    }
}

template <int BITS, int G, typename XT, typename PT, int NT>
__global__ void __launch_bounds__(kThreads) affine_gemv_kernel(const AffineParams p)
{
    using Cfg = AffineCfg<BITS, G, XT, PT, NT>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t* stages = smem;
    float2* params = reinterpret_cast<float2*>(smem + kStages * Cfg::STAGE);
    const int params_bytes = kRowsPerCta * p.gstride * 8;
    float* red = reinterpret_cast<float*>(smem + kStages * Cfg::STAGE + params_bytes);
    Barriers& bars = *reinterpret_cast<Barriers*>(smem + kStages * Cfg::STAGE + params_bytes + Cfg::RED);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;  // == rank in the cluster
    const int n0 = blockIdx.y * kRowsPerCta;
    const int kbeg = split * p.k_per_split;
    const int kend = min(p.K, kbeg + p.k_per_split);
    const int nst = kend > kbeg ? (kend - kbeg + Cfg::KST - 1) / Cfg::KST : 0;
    const int rows_valid = min(kRowsPerCta, p.N - n0);
    const int M = p.M;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], kConsumerWarps);
        }
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer warp
        const size_t row_pitch = (size_t)p.K * BITS / 8;
        const uint8_t* xb = static_cast<const uint8_t*>(p.x);
        producer_loop(bars, nst, p.status, [&](int it, int slot, int ln) {
            const int k0 = kbeg + it * Cfg::KST;
            const int kst = min(Cfg::KST, kend - k0);
            const unsigned wbytes = (unsigned)(kst * BITS / 8);
            const unsigned xbytes = (unsigned)(kst * (int)sizeof(XT));
            uint8_t* wst = stages + slot * Cfg::STAGE;
            uint8_t* xst = wst + Cfg::W_STAGE;
            if (ln == 0)
                mbar_arrive_expect_tx(&bars.full[slot], rows_valid * wbytes + M * xbytes);
            __syncwarp();
            for (int r = ln; r < rows_valid; r += 32)
                bulk_g2s(wst + r * Cfg::RBP, p.codes + (size_t)(n0 + r) * row_pitch + (size_t)k0 * BITS / 8, wbytes,
                         &bars.full[slot]);
            for (int m = ln; m < M; m += 32)
                bulk_g2s(xst + m * Cfg::XBP, xb + ((size_t)m * p.K + k0) * sizeof(XT), xbytes, &bars.full[slot]);
        });
    } else {
        // ------------------------------------------------ consumer warps
        // group parameters of this CTA's rows and K-range -> smem as {s, b - 128 s}
        const int g0 = kbeg / G;
        const int ng = (kend - kbeg) / G;
        const int gpr = p.K / G;
        const PT* sc = static_cast<const PT*>(p.scales);
        const PT* bi = static_cast<const PT*>(p.biases);
        for (int e = threadIdx.x; e < kRowsPerCta * ng; e += kConsumerWarps * 32) {
            const int r = e / ng, gl = e % ng;
            float s = 0.f, b = 0.f;
            if (r < rows_valid) {
                s = to_float(sc[(size_t)(n0 + r) * gpr + g0 + gl]);
                b = to_float(bi[(size_t)(n0 + r) * gpr + g0 + gl]);
            }
            params[r * p.gstride + gl] = make_float2(s, fmaf(-Cfg::OFFSET, s, b));
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");

        const int gid = lane >> 2, tig = lane & 3;
        const int row0 = warp * 16 + gid;  // local rows row0, row0 + 8
        float acc[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[t][i] = 0.f;
        const uint32_t ones[4] = {kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2};
        bool aborted = false;
        for (int it = 0; it < nst; ++it) {
            const int slot = it % kStages;
            if (!mbar_wait_bounded(&bars.full[slot], (it / kStages) & 1, p.status)) {
                aborted = true;
                bars.abort_flag = 1;
                break;
            }
            const uint8_t* wst = stages + slot * Cfg::STAGE;
            const uint8_t* xst = wst + Cfg::W_STAGE;
            const uint32_t* wr0 = reinterpret_cast<const uint32_t*>(wst + row0 * Cfg::RBP);
            const uint32_t* wr1 = reinterpret_cast<const uint32_t*>(wst + (row0 + 8) * Cfg::RBP);
            const int kst = min(Cfg::KST, kend - (kbeg + it * Cfg::KST));
            const int groups = kst / G;
            for (int gl = 0; gl < groups; ++gl) {
                float d[NT][4], dx[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        d[t][i] = dx[t][i] = 0.f;
#pragma unroll
                for (int j = 0; j < Cfg::WPL; ++j) {
                    const int wi = gl * Cfg::WPG + j * 4 + tig;  // word index in the stage row
                    const uint32_t w0 = wr0[wi];
                    const uint32_t w1 = wr1[wi];
                    const int kl = wi * Cfg::CPW;                // k offset of the word in the stage
                    // B operand registers: bx[t][q] for the word's codes, paired as the A side pairs them
                    constexpr int NP = Cfg::CPW / 2;             // bf16 pairs per word (4-bit: 4, 2-bit: 8, 8-bit: 2)
                    uint32_t bx[NT][NP];
                    uint32_t bxl[NT][NP];                        // low parts when x is fp32
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const int tok = t * 8 + gid;
                        uint32_t raw[NP];                        // (x_{2i}, x_{2i+1}) as bf16 pairs
                        uint32_t rawl[NP];
                        if (tok < M) {
                            if constexpr (sizeof(XT) == 2) {
                                const uint32_t* xp = reinterpret_cast<const uint32_t*>(xst + tok * Cfg::XBP + kl * 2);
                                if constexpr (NP == 4) {
                                    const uint4 v = *reinterpret_cast<const uint4*>(xp);
                                    raw[0] = v.x; raw[1] = v.y; raw[2] = v.z; raw[3] = v.w;
                                } else if constexpr (NP == 8) {
                                    const uint4 v0 = reinterpret_cast<const uint4*>(xp)[0];
                                    const uint4 v1 = reinterpret_cast<const uint4*>(xp)[1];
                                    raw[0] = v0.x; raw[1] = v0.y; raw[2] = v0.z; raw[3] = v0.w;
                                    raw[4] = v1.x; raw[5] = v1.y; raw[6] = v1.z; raw[7] = v1.w;
                                } else {
                                    const uint2 v = *reinterpret_cast<const uint2*>(xp);
                                    raw[0] = v.x; raw[1] = v.y;
                                }
#pragma unroll
                                for (int q = 0; q < NP; ++q)
                                    rawl[q] = 0u;
                            } else {
                                const float* xp = reinterpret_cast<const float*>(xst + tok * Cfg::XBP + kl * 4);
#pragma unroll
                                for (int q = 0; q < NP; q += 2) {
                                    const float4 v = reinterpret_cast<const float4*>(xp)[q / 2];
                                    split_f32_pair(v.x, v.y, raw[q], rawl[q]);
                                    split_f32_pair(v.z, v.w, raw[q + 1], rawl[q + 1]);
                                }
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < NP; ++q)
                                raw[q] = rawl[q] = 0u;
                        }
                        // re-pair to match the A side
                        if constexpr (BITS == 4) {
                            // codes pairs (0,4),(1,5),(2,6),(3,7): raw[q] = (x_{2q}, x_{2q+1})
                            bx[t][0] = pair_lo(raw[0], raw[2]);   // (x0, x4)
                            bx[t][1] = pair_hi(raw[0], raw[2]);   // (x1, x5)
                            bx[t][2] = pair_lo(raw[1], raw[3]);   // (x2, x6)
                            bx[t][3] = pair_hi(raw[1], raw[3]);   // (x3, x7)
                            bxl[t][0] = pair_lo(rawl[0], rawl[2]);
                            bxl[t][1] = pair_hi(rawl[0], rawl[2]);
                            bxl[t][2] = pair_lo(rawl[1], rawl[3]);
                            bxl[t][3] = pair_hi(rawl[1], rawl[3]);
                        } else if constexpr (BITS == 2) {
                            // pairs (j, j+8): raw[i] = (x_{2i}, x_{2i+1}); (x_{2i}, x_{2i+8}) = lo(raw[i], raw[i+4])
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                bx[t][2 * i] = pair_lo(raw[i], raw[i + 4]);
                                bx[t][2 * i + 1] = pair_hi(raw[i], raw[i + 4]);
                                bxl[t][2 * i] = pair_lo(rawl[i], rawl[i + 4]);
                                bxl[t][2 * i + 1] = pair_hi(rawl[i], rawl[i + 4]);
                            }
                        } else {
                            // 8-bit pairs (0,2),(1,3)
                            bx[t][0] = pair_lo(raw[0], raw[1]);
                            bx[t][1] = pair_hi(raw[0], raw[1]);
                            bxl[t][0] = pair_lo(rawl[0], rawl[1]);
                            bxl[t][1] = pair_hi(rawl[0], rawl[1]);
                        }
                    }
                    // MMAs: each part consumes 2 pairs per row
#pragma unroll
                    for (int part = 0; part < NP / 2; ++part) {
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
                // group epilogue: acc += s * D' + (b - 128 s) * X
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
        (void)aborted;
        // partial tile -> smem [token][row]
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int c0 = t * 8 + 2 * tig;
            red[c0 * kRowsPerCta + row0] = acc[t][0];
            red[(c0 + 1) * kRowsPerCta + row0] = acc[t][1];
            red[c0 * kRowsPerCta + row0 + 8] = acc[t][2];
            red[(c0 + 1) * kRowsPerCta + row0 + 8] = acc[t][3];
        }
    }
    // ---------------------------------------------------- split-K reduction through DSMEM
    __syncwarp();
    cluster_sync();
    if (warp < kConsumerWarps) {
        const int S = gridDim.x;
        const uint32_t red_local = smem_u32(red);
        using OT = XT;
        const OT* bias = static_cast<const OT*>(p.bias);
        OT* y = static_cast<OT*>(p.y);
        for (int e = split * (kConsumerWarps * 32) + threadIdx.x; e < M * kRowsPerCta;
             e += S * kConsumerWarps * 32) {
            const int tok = e / kRowsPerCta, r = e % kRowsPerCta;
            float v = 0.f;
            for (int q = 0; q < S; ++q)
                v += ld_shared_cluster_f32(map_shared_rank(red_local + 4u * (uint32_t)e, (unsigned)q));
            if (r < rows_valid) {
                if (bias)
                    v += to_float(bias[n0 + r]);
                y[(size_t)tok * p.N + n0 + r] = from_float<OT>(v);
            }
        }
    }
    cluster_sync();
}

// ---------------------------------------------------------------- BitLinear decode kernel

template <int NT>
struct BitCfg {
    static constexpr int PROWS = kRowsPerCta / 4;   // packed rows per CTA (16) -> 64 output rows
    static constexpr int KST = 512;                 // k (bytes per packed row) per stage
    static constexpr int RBP = KST + 16;
    static constexpr int XB = KST * 2;
    static constexpr int XBP = XB + 32;
    static constexpr int MMAX = 8 * NT;
    static constexpr int W_STAGE = PROWS * RBP;
    static constexpr int X_STAGE = MMAX * XBP;
    static constexpr int STAGE = round_up(W_STAGE + X_STAGE, 128);
    static constexpr int RED = MMAX * kRowsPerCta * 4;
    static constexpr int SMEM = kStages * STAGE + RED + (int)sizeof(Barriers) + 128;
};

struct BitParams {
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
__global__ void __launch_bounds__(kThreads) bitlinear_gemv_kernel(const BitParams p)
{
    using Cfg = BitCfg<NT>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t* stages = smem;
    float* red = reinterpret_cast<float*>(smem + kStages * Cfg::STAGE);
    Barriers& bars = *reinterpret_cast<Barriers*>(smem + kStages * Cfg::STAGE + Cfg::RED);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int p0 = blockIdx.y * Cfg::PROWS;
    const int kbeg = split * p.k_per_split;
    const int kend = min(p.K, kbeg + p.k_per_split);
    const int nst = kend > kbeg ? (kend - kbeg + Cfg::KST - 1) / Cfg::KST : 0;
    const int prows_valid = min(Cfg::PROWS, p.R - p0);
    const int M = p.M;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], kConsumerWarps);
        }
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        producer_loop(bars, nst, p.status, [&](int it, int slot, int ln) {
            const int k0 = kbeg + it * Cfg::KST;
            const int kst = min(Cfg::KST, kend - k0);
            uint8_t* wst = stages + slot * Cfg::STAGE;
            uint8_t* xst = wst + Cfg::W_STAGE;
            if (ln == 0)
                mbar_arrive_expect_tx(&bars.full[slot], prows_valid * kst + M * kst * 2);
            __syncwarp();
            for (int r = ln; r < prows_valid; r += 32)
                bulk_g2s(wst + r * Cfg::RBP, p.packed + (size_t)(p0 + r) * p.K + k0, (unsigned)kst, &bars.full[slot]);
            for (int m = ln; m < M; m += 32)
                bulk_g2s(xst + m * Cfg::XBP, p.x + (size_t)m * p.K + k0, (unsigned)(kst * 2), &bars.full[slot]);
        });
    } else {
        const int gid = lane >> 2, tig = lane & 3;
        const int prow = warp * 4 + (gid & 3);  // local packed row of both A rows of this lane
        const int sh0 = 2 * (gid >> 2);         // field j of A row gid; row gid+8 uses j+2
        float acc[NT][4], ax[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[t][i] = ax[t][i] = 0.f;
        const uint32_t ones[4] = {kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2};
        for (int it = 0; it < nst; ++it) {
            const int slot = it % kStages;
            if (!mbar_wait_bounded(&bars.full[slot], (it / kStages) & 1, p.status)) {
                bars.abort_flag = 1;
                break;
            }
            const uint8_t* wst = stages + slot * Cfg::STAGE;
            const uint8_t* xst = wst + Cfg::W_STAGE;
            const uint32_t* wr = reinterpret_cast<const uint32_t*>(wst + prow * Cfg::RBP);
            const int kst = min(Cfg::KST, kend - (kbeg + it * Cfg::KST));
            const int steps = kst / 16;
#pragma unroll 4
            for (int s = 0; s < steps; ++s) {
                const int wi = s * 4 + tig;  // word of 4 bytes (k = 4 wi .. 4 wi + 3)
                const uint32_t w = wr[wi];
                uint32_t a[4];
                // row gid: field j = sh0/2; pairs (k, k+2) and (k+1, k+3)
                a[0] = lop3_and_or(w >> sh0, 0x00030003u, 0x43004300u);
                a[2] = lop3_and_or(w >> (sh0 + 8), 0x00030003u, 0x43004300u);
                a[1] = lop3_and_or(w >> (sh0 + 4), 0x00030003u, 0x43004300u);
                a[3] = lop3_and_or(w >> (sh0 + 12), 0x00030003u, 0x43004300u);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const int tok = t * 8 + gid;
                    uint32_t b0 = 0u, b1 = 0u;
                    if (tok < M) {
                        const uint2 v = *reinterpret_cast<const uint2*>(xst + tok * Cfg::XBP + wi * 8);
                        b0 = pair_lo(v.x, v.y);  // (x_k, x_{k+2})
                        b1 = pair_hi(v.x, v.y);  // (x_{k+1}, x_{k+3})
                    }
                    mma_bf16_16816(acc[t], a, b0, b1);
                    mma_bf16_16816(ax[t], ones, b0, b1);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.empty[slot]);
        }
        // partial = sum x*(c+128) - 129 * sum x = sum x*(c-1)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int c0 = t * 8 + 2 * tig;
            const int r0 = warp * 16 + gid;
            red[c0 * kRowsPerCta + r0] = fmaf(-129.0f, ax[t][0], acc[t][0]);
            red[(c0 + 1) * kRowsPerCta + r0] = fmaf(-129.0f, ax[t][1], acc[t][1]);
            red[c0 * kRowsPerCta + r0 + 8] = fmaf(-129.0f, ax[t][2], acc[t][2]);
            red[(c0 + 1) * kRowsPerCta + r0 + 8] = fmaf(-129.0f, ax[t][3], acc[t][3]);
        }
    }
    __syncwarp();
    cluster_sync();
    if (warp < kConsumerWarps) {
        const int S = gridDim.x;
        const uint32_t red_local = smem_u32(red);
        const float ws = *p.weight_scale;
        const float scale = p.invert ? __fdiv_rn(1.0f, ws) : ws;
        for (int e = split * (kConsumerWarps * 32) + threadIdx.x; e < M * kRowsPerCta;
             e += S * kConsumerWarps * 32) {
            const int tok = e / kRowsPerCta, i = e % kRowsPerCta;
            // local A row i of warp w: packed row 4w + (i%16)%4, field (i%16)/4
            const int w = i / 16, ii = i % 16;
            const int pr = p0 + w * 4 + (ii & 3);
            const int j = ii >> 2;
            float v = 0.f;
            for (int q = 0; q < S; ++q)
                v += ld_shared_cluster_f32(map_shared_rank(red_local + 4u * (uint32_t)e, (unsigned)q));
            if (pr < p.R) {
                const int n = pr + j * p.R;
                v *= scale;
                if (p.bias)
                    v += __bfloat162float(p.bias[n]);
                p.y[(size_t)tok * p.N + n] = __float2bfloat16_rn(v);
            }
        }
    }
    cluster_sync();
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
    S = S < 1 ? 1 : (S > 8 ? 8 : S);
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
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    if (cluster_x > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess)
            return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int BITS, int G, typename XT, typename PT, int NT>
cudaError_t affine_launch_t(const AffineGemvArgs& a, int m0, int mcount, cudaStream_t st, const DeviceInfo& dev)
{
    using Cfg = AffineCfg<BITS, G, XT, PT, NT>;
    const int tiles = (int)((a.N + kRowsPerCta - 1) / kRowsPerCta);
    const SplitPlan pl = plan_splits(tiles, (int)a.K, Cfg::KST, dev.sm_count, Cfg::MAX_GROUPS * G);
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
    return launch_cluster(affine_gemv_kernel<BITS, G, XT, PT, NT>, dim3(pl.S, tiles, 1),
                          Cfg::smem_bytes(prm.gstride), pl.S, st, prm);
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
        if (mc <= 8)
            e = launch_cluster(bitlinear_gemv_kernel<1>, dim3(pl.S, tiles, 1), BitCfg<1>::SMEM, pl.S, st, prm);
        else
            e = launch_cluster(bitlinear_gemv_kernel<2>, dim3(pl.S, tiles, 1), BitCfg<2>::SMEM, pl.S, st, prm);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace qlin
