// k_affine_dec.cu -- MLX-affine decode GEMV for up to 8 tokens per launch (one for 2-bit codes),
// bf16 activations, 2-, 4- or 8-bit codes, on layers whose codes fit in shared memory when spread
// over the SMs: up to 32 output rows per SM (N <= 4736 on B200) with 8 warps, up to 128 with 16
// warps when the codes fill more than half of an SM's shared memory (the Llama-7B layers: 4096 ->
// 4096, 11008 -> 4096, 4096 -> 11008).  Other layers and more tokens take the ring-streaming
// kernel (k_gemv.cu).
//
//   y[m,n] = sum_g [ s[n,g] * sum_{k in g} x[m,k] q[n,k] + b[n,g] * sum_{k in g} x[m,k] ] + bias[n]
//   [nuvec-nn QuantizedLinear: forward, dequantized_weight (w = scale q + bias per group)]
//
// The same kernel runs the one-token branch of the per-group INT8 layer [cider/ops.py
// pergroup_linear: M == 1 -> per-group MV, FP activation, weight dequant on the fly]: an int8
// weight c is the 8-bit code c ^ 0x80 = c + 128 with the group's scale s and bias -128 s, the
// scales read from their group-major [K/g, N] layout.
//
// Design (B200; a decode layer is a few MB and sits in a chain of dependent layers, so the
// weight fetch has to overlap the previous layer and what follows the dependency wait has to be
// short):
//  * One CTA per SM, the output rows split evenly over them (27-28 rows at N = 4096).  Before
//    griddepcontrol.wait one warp issues a bulk copy (cp.async.bulk, no tensor map) per row of the
//    CTA's codes into shared memory and every thread copies a slice of the rows' group scales and
//    biases (cp.async, 4 bytes): the layer's whole weight is on its way before the previous kernel
//    has finished.  Under about 100 registers a thread and half the shared memory, the next
//    layer's CTA fits beside this one (8 warps) and does the same while this one computes; a CTA
//    whose codes fill more than half the shared memory cannot share the SM, and runs 16 warps
//    (measured 4-8 % faster there than 8: more warps to hide the loop's latency).
//  * After the wait the CTA copies the launch's token rows of x into shared memory (one round
//    trip) and the layer bias too, so neither the main loop nor the epilogue waits on memory.
//  * Rows sit in shared memory at a pitch of 16 * WPL (mod 128) bytes (16 for WPL = 8), WPL the
//    words a lane takes per row and group: the vector code loads of a warp fall in distinct banks.
//  * Warps split the row tiles (16 rows, two per warp) and the groups (round robin).  Lane
//    (gid, tig) takes the tig-th quarter of each group of rows gid and gid + 8 (WPL consecutive
//    words, one vector load), and MMA j takes word j of every lane: one m16n8k16 MMA always covers
//    16 codes of a single group.  The loop body is branch-free (a tile past the CTA's rows is
//    computed and dropped); two accumulator chains per tile; a one-token launch folds only the D
//    values of token 0.
//  * Codes become bf16 with one LOP3 per pair -- (w >> b j) & mask | 0x4300 is (128 + q_j,
//    128 + q_j'), exact -- (8-bit codes go through fp32: 0..255 are exact in bf16) and x is
//    permuted with PRMT to the same pairing.  An MMA against an all-ones A operand gives the group
//    sums of x, so per group and row
//        acc += s * D'_g + (b - 128 s) * X_g,   D'_g = sum (128 + q) x,  X_g = sum x
//    (no 128 offset for 8-bit codes): every product is exact, only fp32 sums round.
//  * Measured on B200: mma.sync m16n8k16 issues once per ~8.7 cycles per SM sub-partition; with
//    two warps per sub-partition the loop is bound by the MMA and decode dependency chains, not
//    by the pipe.  (Alternatives measured slower: a second register set loading a group ahead --
//    the register count then keeps the next layer's CTA off the SM; group sums of x computed once
//    per CTA by the threads instead of the all-ones MMA, with 8 and with 16 warps; four accumulator
//    chains; one tile per warp; 16 warps on layers that can share the SM.)
//  * Partial sums of the warps that share rows meet in shared memory (the code area, once every
//    warp has left the main loop); the bias is added in fp32 and y rounded once to bf16.
//  * The bulk copies complete on an mbarrier whose wait is bounded (qlin::kWaitLimitNs): on expiry
//    the kernel records the timeout, waits once more (bounded) for the copies and writes nothing.
#include "qlin_common.cuh"

namespace qlin {
namespace {

constexpr int kDecWarpsMax = 16;
constexpr int kTPW = 2;  // 16-row tiles per warp
constexpr uint32_t kOnes = 0x3F803F80u;  // bf16 (1, 1)

struct DecParams {
    const uint8_t* codes;        // [N][rowbytes]
    const void* scales;          // [N][NG] bf16 or fp32
    const void* biases;
    const __nv_bfloat16* x;      // [M][K] (this launch's tokens)
    const __nv_bfloat16* bias;   // [N] or null
    __nv_bfloat16* y;            // [M][N]
    int M, K, N, NG;
    int rowbytes, pitch;         // code bytes per row; shared-memory row pitch (16 mod 128)
    int rows_max, T, RG, KG;     // rows per CTA at most, 16-row tiles, warp row groups x group split
    int W;                       // warps per CTA (8 or 16)
    int p_f32;                   // group parameters are fp32 (else bf16)
    int pg;                      // per-group INT8: int8 codes, fp32 scales [NG][N], bias -128 s
    int code_bytes, x_bytes, param_bytes, aux_bytes;  // shared-memory areas
    int xpitch;                  // shared-memory pitch of an x row
    unsigned* status;
    int trace_slot;
};

#ifdef QLIN_TRACE
// [slot][cta][8]: start, weights issued, wait returned, x and weights landed, main loop done,
// end, (unused), smid.  Host side: qlin_trace_read_dec().
constexpr int kDecTraceSlots = 1024;
constexpr int kDecTraceCtas = 512;
__device__ unsigned long long g_dec_trace[(size_t)kDecTraceSlots * kDecTraceCtas * 8];
int g_dec_trace_next = 0;
#define DEC_TRACE(i) \
    do { if (threadIdx.x == 0) tr[i] = globaltimer_ns(); } while (0)
#else
#define DEC_TRACE(i) \
    do { } while (0)
#endif

QLIN_DEV void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

QLIN_DEV void cp_async4(void* dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

QLIN_DEV void cp_async_wait_all_dec() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// bf16 pair i of a code word: (q_i, q_{i + CPW/2}), each + 128 for 2 / 4 bits, exact for 8 bits
template <int BITS>
QLIN_DEV uint32_t code_pair(uint32_t w, int i)
{
    if constexpr (BITS == 4) {
        return lop3_and_or(w >> (4 * i), 0x000F000Fu, 0x43004300u);
    } else if constexpr (BITS == 2) {
        return lop3_and_or(w >> (2 * i), 0x00030003u, 0x43004300u);
    } else {
        // bytes i and i + 2 -> fp32 2^23 + q -> q (exact) -> bf16 pair (exact: q <= 255)
        const float lo = __uint_as_float(prmt(w, 0x4B000000u, 0x7440u + (uint32_t)i)) - 8388608.0f;
        const float hi = __uint_as_float(prmt(w, 0x4B000000u, 0x7442u + (uint32_t)i)) - 8388608.0f;
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
}

// ONE: a one-token launch.  W warps: 8 while the CTA leaves room on the SM for the next layer's
// CTA (its weight fetch then overlaps this layer), 16 when its codes alone fill more than half of
// the SM's shared memory (no overlap is possible; more warps hide the loop's latency instead).
template <int BITS, int G, int NT, bool ONE, int W>
__global__ void __launch_bounds__(W * 32, 1) affine_dec_kernel(const __grid_constant__ DecParams p)
{
    constexpr int kDecThreads = W * 32;
    static_assert(!ONE || NT == 1, "one token fits one token tile");
    constexpr int CPW = 32 / BITS;          // codes per word
    constexpr int WPL = G * BITS / 128;     // words per lane per row per group
    constexpr int WPG = 4 * WPL;            // words per row per group
    constexpr int SUB = CPW / 4;            // MMAs per word
    constexpr int XW = CPW >= 8 ? CPW / 8 : 1;  // 16-byte x pieces per word and token tile
    constexpr float OFF = BITS == 8 ? 0.0f : 128.0f;
    static_assert(WPL >= 1, "group too small for the lane mapping");

    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t* codes_s = smem_raw;
    uint8_t* x_s = smem_raw + p.code_bytes;
    uint8_t* params_s = x_s + p.x_bytes;
    float* bias_s = reinterpret_cast<float*>(params_s + p.param_bytes);  // [rows_max] layer bias
    uint64_t* bar = reinterpret_cast<uint64_t*>(params_s + p.param_bytes + p.aux_bytes);
#ifdef QLIN_TRACE
    unsigned long long tr[8] = {};
#endif
    DEC_TRACE(0);
    __shared__ int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int r0 = (int)((long long)blockIdx.x * p.N / gridDim.x);
    const int r1 = (int)((long long)(blockIdx.x + 1) * p.N / gridDim.x);
    const int rows = r1 - r0;
    const int psz = p.p_f32 ? 4 : 2;

    pdl_launch_dependents();
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        abort_s = 0;
    }
    __syncthreads();
    // the layer's constant weights, all before the dependency wait
    if (warp == 0) {
        if (lane == 0)
            mbar_arrive_expect_tx(bar, (unsigned)(rows * p.rowbytes));
        __syncwarp();
        for (int r = lane; r < rows; r += 32)
            bulk_g2s(codes_s + (size_t)r * p.pitch, p.codes + (size_t)(r0 + r) * p.rowbytes, (unsigned)p.rowbytes,
                     bar);
    }
    if (p.pg) {  // group-major fp32 scales -> [row][NG], one element per copy (consecutive rows)
        const float* sg = static_cast<const float*>(p.scales);
        float* ss = reinterpret_cast<float*>(params_s);
        for (int e = tid; e < rows * p.NG; e += kDecThreads) {
            const int g = e / rows, r = e % rows;
            cp_async4(ss + r * p.NG + g, sg + (size_t)g * p.N + r0 + r);
        }
    } else {
        const int words = rows * p.NG * psz / 4;  // scales block, then biases block
        const size_t off = (size_t)r0 * p.NG * psz;
        const uint8_t* sg = static_cast<const uint8_t*>(p.scales) + off;
        const uint8_t* bg = static_cast<const uint8_t*>(p.biases) + off;
        uint8_t* ss = params_s;
        uint8_t* bs = params_s + (size_t)p.rows_max * p.NG * psz;
        for (int e = tid; e < words; e += kDecThreads) {
            cp_async4(ss + 4 * e, sg + 4 * e);
            cp_async4(bs + 4 * e, bg + 4 * e);
        }
    }
    DEC_TRACE(1);
    pdl_wait_prior_grids();  // x, the layer bias and y may belong to the previous kernel
    DEC_TRACE(2);
    {
        const int per_row = p.K * 2 / 16;  // 16-byte pieces of an x row
        for (int e = tid; e < p.M * per_row; e += kDecThreads) {
            const int m = e / per_row, c = e % per_row;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(x_s + (size_t)m * p.xpitch + 16 * c)),
                         "l"(p.x + (size_t)m * p.K + 8 * c)
                         : "memory");
        }
        for (int r = tid; r < rows; r += kDecThreads)  // the layer bias, off the end of the critical path
            bias_s[r] = p.bias ? __bfloat162float(p.bias[r0 + r]) : 0.f;
    }

    const int rg = warp / p.KG, kg = warp % p.KG;
    // both tiles are always computed (branch-free code schedules better); a tile past T reads the
    // last allocated rows and its results are never stored
    int trow[kTPW];
#pragma unroll
    for (int t = 0; t < kTPW; ++t)
        trow[t] = min(16 * (kTPW * rg + t), 16 * p.T - 16);
    // warps past RG x KG (when RG does not divide W) have no work
    const int ngw = (warp < p.RG * p.KG && p.NG > kg) ? (p.NG - 1 - kg) / p.KG + 1 : 0;  // groups of this warp

    if (!mbar_wait_bounded(bar, 0, p.status))
        abort_s = 1;
    cp_async_wait_all_dec();
    __syncthreads();
    DEC_TRACE(3);
    if (abort_s) {
        if (tid == 0)
            mbar_wait_bounded(bar, 0, p.status);  // no copy may still be landing at exit
        return;
    }

    // One group per iteration: its code words (tile, row half, word) and x words, and two
    // independent accumulator chains per tile.
    using CodeBuf = uint32_t[kTPW][2][WPL];
    using XBuf = uint4[NT][WPL][XW];
    auto load_group = [&](int gl, CodeBuf& cw, XBuf& xv) {
        const int gi = kg + p.KG * gl;
#pragma unroll
        for (int t = 0; t < kTPW; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = trow[t] + gid + 8 * h;
                const uint8_t* src = codes_s + (size_t)row * p.pitch + 4 * (gi * WPG + tig * WPL);
                if constexpr (WPL == 1) {
                    cw[t][h][0] = *reinterpret_cast<const uint32_t*>(src);
                } else if constexpr (WPL == 2) {
                    const uint2 v = *reinterpret_cast<const uint2*>(src);
                    cw[t][h][0] = v.x;
                    cw[t][h][1] = v.y;
                } else {
#pragma unroll
                    for (int q = 0; q < WPL / 4; ++q) {
                        const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * q);
                        cw[t][h][4 * q] = v.x;
                        cw[t][h][4 * q + 1] = v.y;
                        cw[t][h][4 * q + 2] = v.z;
                        cw[t][h][4 * q + 3] = v.w;
                    }
                }
            }
        if constexpr (BITS == 8) {
            if (p.pg) {  // int8 weights c read as the unsigned codes c ^ 0x80 = c + 128
#pragma unroll
                for (int t = 0; t < kTPW; ++t)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int j = 0; j < WPL; ++j)
                            cw[t][h][j] ^= 0x80808080u;
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            // token rows past M read row 0 and are zeroed with a mask (no branch)
            const int m = 8 * nt + gid;
            const uint32_t keep = m < p.M ? 0xFFFFFFFFu : 0u;
            const uint8_t* src = x_s + (size_t)(m < p.M ? m : 0) * p.xpitch + 2 * CPW * (gi * WPG + tig * WPL);
#pragma unroll
            for (int j = 0; j < WPL; ++j)
#pragma unroll
                for (int c = 0; c < XW; ++c) {
                    if constexpr (CPW >= 8) {
                        const uint4 v = *reinterpret_cast<const uint4*>(src + 2 * CPW * j + 16 * c);
                        xv[nt][j][c] = make_uint4(v.x & keep, v.y & keep, v.z & keep, v.w & keep);
                    } else {  // 8-bit: four codes, 8 bytes of x
                        const uint2 v = *reinterpret_cast<const uint2*>(src + 2 * CPW * j);
                        xv[nt][j][c] = make_uint4(v.x & keep, v.y & keep, 0u, 0u);
                    }
                }
        }
    };

    float tot[kTPW][NT][4];
#pragma unroll
    for (int t = 0; t < kTPW; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                tot[t][nt][e] = 0.f;
    const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};

    auto compute_group = [&](int gl, const CodeBuf& cw, const XBuf& xv) {
        const int gi = kg + p.KG * gl;
        constexpr int CH = 2;  // independent accumulator chains
        float ga[kTPW][NT][CH][4], xa[NT][CH][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < CH; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xa[nt][c][e] = 0.f;
#pragma unroll
                    for (int t = 0; t < kTPW; ++t)
                        ga[t][nt][c][e] = 0.f;
                }
#pragma unroll
        for (int j = 0; j < WPL; ++j) {
#pragma unroll
            for (int i = 0; i < SUB; ++i) {
                const int ch = (j * SUB + i) % CH;
                // x pairs in the codes' pairing: (x_2i, x_2i+CPW/2), (x_2i+1, x_2i+1+CPW/2)
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t xw[CPW / 2];
#pragma unroll
                    for (int c = 0; c < XW; ++c) {
                        xw[4 * c] = xv[nt][j][c].x;
                        xw[4 * c + 1] = xv[nt][j][c].y;
                        if constexpr (CPW / 2 > 2) {
                            xw[4 * c + 2] = xv[nt][j][c].z;
                            xw[4 * c + 3] = xv[nt][j][c].w;
                        }
                    }
                    b0[nt] = prmt(xw[i], xw[i + CPW / 4], 0x5410u);
                    b1[nt] = prmt(xw[i], xw[i + CPW / 4], 0x7632u);
                    mma_bf16_16816(xa[nt][ch], ones, b0[nt], b1[nt]);
                }
#pragma unroll
                for (int t = 0; t < kTPW; ++t) {
                    const uint32_t a[4] = {code_pair<BITS>(cw[t][0][j], 2 * i), code_pair<BITS>(cw[t][1][j], 2 * i),
                                           code_pair<BITS>(cw[t][0][j], 2 * i + 1),
                                           code_pair<BITS>(cw[t][1][j], 2 * i + 1)};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_bf16_16816(ga[t][nt][ch], a, b0[nt], b1[nt]);
                }
            }
        }
        // group done: scale, offset and group bias of each row; D value e is row gid + 8 (e >> 1),
        // token 8 nt + 2 tig + (e & 1) -- a one-token launch needs only e = 0, 2 (token 0 in tig 0)
        float xs[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                xs[nt][e] = xa[nt][0][e] + xa[nt][1][e];
#pragma unroll
        for (int t = 0; t < kTPW; ++t) {
            // rows past the CTA's own read the last row's parameters (never stored)
            const int ra = min(trow[t] + gid, p.rows_max - 1);
            const int rb = min(trow[t] + gid + 8, p.rows_max - 1);
            float sa, ba, sb, bb;
            if (p.p_f32) {
                const float* S_ = reinterpret_cast<const float*>(params_s);
                const float* B_ = S_ + (size_t)p.rows_max * p.NG;
                sa = S_[ra * p.NG + gi];
                ba = B_[ra * p.NG + gi];
                sb = S_[rb * p.NG + gi];
                bb = B_[rb * p.NG + gi];
            } else {
                const __nv_bfloat16* S_ = reinterpret_cast<const __nv_bfloat16*>(params_s);
                const __nv_bfloat16* B_ = S_ + (size_t)p.rows_max * p.NG;
                sa = __bfloat162float(S_[ra * p.NG + gi]);
                ba = __bfloat162float(B_[ra * p.NG + gi]);
                sb = __bfloat162float(S_[rb * p.NG + gi]);
                bb = __bfloat162float(B_[rb * p.NG + gi]);
            }
            if (p.pg) {  // w = s (c ^ 0x80) - 128 s for the int8 weight c
                ba = -128.0f * sa;
                bb = -128.0f * sb;
            } else {
                ba = fmaf(-OFF, sa, ba);
                bb = fmaf(-OFF, sb, bb);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (ONE && (e & 1))
                        continue;
                    const float s_ = e < 2 ? sa : sb, b_ = e < 2 ? ba : bb;
                    const float d = ga[t][nt][0][e] + ga[t][nt][1][e];
                    tot[t][nt][e] = fmaf(s_, d, fmaf(b_, xs[nt][e], tot[t][nt][e]));
                }
        }
    };

    // (one register set: a second one to load a group ahead measured slower -- the register
    // count then keeps the next layer's CTA off the SM)
    CodeBuf cw;
    XBuf xv;
    for (int gl = 0; gl < ngw; ++gl) {
        load_group(gl, cw, xv);
        compute_group(gl, cw, xv);
    }
    DEC_TRACE(4);

    // partial sums of the KG warps of each row group meet in shared memory (the code area)
    __syncthreads();
    float* red = reinterpret_cast<float*>(codes_s);  // [warp][t][nt][e][lane]
#pragma unroll
    for (int t = 0; t < kTPW; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                red[(((warp * kTPW + t) * NT + nt) * 4 + e) * 32 + lane] = tot[t][nt][e];
    __syncthreads();
    const int per_rg = kTPW * NT * 4 * 32;
    for (int idx = tid; idx < p.RG * per_rg; idx += kDecThreads) {
        const int rgi = idx / per_rg, rem = idx % per_rg;
        const int t = rem / (NT * 4 * 32), nt = (rem / (4 * 32)) % NT, e = (rem / 32) % 4, ln = rem % 32;
        const int row = 16 * (kTPW * rgi + t) + (ln >> 2) + 8 * (e >> 1);
        const int m = 8 * nt + 2 * (ln & 3) + (e & 1);
        if (row >= rows || m >= p.M)
            continue;
        float v = 0.f;
        for (int k = 0; k < p.KG; ++k)
            v += red[((((rgi * p.KG + k) * kTPW + t) * NT + nt) * 4 + e) * 32 + ln];
        const int n = r0 + row;
        v += bias_s[row];
        p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(v);
    }
#ifdef QLIN_TRACE
    __syncthreads();
    DEC_TRACE(5);
    if (threadIdx.x == 0 && p.trace_slot >= 0 && blockIdx.x < kDecTraceCtas) {
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        tr[7] = smid;
        unsigned long long* dst = g_dec_trace + ((size_t)p.trace_slot * kDecTraceCtas + blockIdx.x) * 8;
        for (int i = 0; i < 8; ++i)
            dst[i] = tr[i];
    }
#endif
}

template <typename Kern>
cudaError_t launch_dec(Kern kern, unsigned grid, int warps, int smem, cudaStream_t st, const DecParams& prm)
{
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3((unsigned)(32 * warps), 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int BITS, int G>
cudaError_t dec_launch_nt(const DecParams& prm, unsigned grid, int smem, cudaStream_t st)
{
    if (prm.W == 16)
        return prm.M == 1 ? launch_dec(affine_dec_kernel<BITS, G, 1, true, 16>, grid, 16, smem, st, prm)
                          : launch_dec(affine_dec_kernel<BITS, G, 1, false, 16>, grid, 16, smem, st, prm);
    return prm.M == 1 ? launch_dec(affine_dec_kernel<BITS, G, 1, true, 8>, grid, 8, smem, st, prm)
                      : launch_dec(affine_dec_kernel<BITS, G, 1, false, 8>, grid, 8, smem, st, prm);
}

// Plans the launch; false when the layer is outside this kernel (the caller then takes another).
bool affine_dec_plan(const AffineGemvArgs& a, const DeviceInfo& dev, int& grid, int& smem, DecParams* out)
{
    if (a.x_dt != QLIN_BF16 || !(a.bits == 2 || a.bits == 4 || a.bits == 8) ||
        !(a.g == 32 || a.g == 64 || a.g == 128) || a.g * a.bits < 128)
        return false;
    if (a.p_dt != QLIN_BF16 && a.p_dt != QLIN_F32)
        return false;
    if (a.pergroup && (a.bits != 8 || a.p_dt != QLIN_F32))
        return false;
    const int64_t NG = a.K / a.g;
    if (a.p_dt == QLIN_BF16 && NG % 2 != 0)  // 4-byte copies of whole rows of bf16 parameters
        return false;
    if ((reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases)) & 3u)
        return false;
    const int64_t rowbytes = a.K * a.bits / 8;
    if (rowbytes % 16 != 0 || (reinterpret_cast<uintptr_t>(a.codes) & 15u) != 0)
        return false;
    if (a.M > 8 || (a.bits == 2 && a.M > 1))  // the ring-streaming kernel measured faster there
        return false;
    grid = (int)(a.N >= 16LL * dev.sm_count ? dev.sm_count : (a.N + 15) / 16);
    const int rows_max = (int)((a.N + grid - 1) / grid);
    const int T = (rows_max + 15) / 16;
    if (T > 8)
        return false;
    const int RG = (T + kTPW - 1) / kTPW;  // row groups of kTPW tiles; KG = warps / RG share each
    // code rows at 16 * WPL (mod 128): a warp's vector loads of 8 rows fall in distinct banks
    const int wpl = a.g * a.bits / 128;
    const int ct = wpl >= 8 ? 16 : 16 * wpl;
    const int pitch = (int)(rowbytes + ((ct - rowbytes % 128) + 128) % 128);
    const int mmax = (int)a.M;
    const int red = kDecWarpsMax * kTPW * 4 * 32 * 4;
    int code_bytes = 16 * T * pitch;  // tiles past T are never read
    code_bytes = code_bytes > red ? code_bytes : red;
    // x rows at a pitch that spreads the 16-byte loads of a warp's token rows over the banks
    const int xrow = (int)(a.K * 2);
    const int xt = a.bits == 4 ? 64 : a.bits == 2 ? 16 : 32;
    const int xpitch = xrow + ((xt - xrow % 128) + 128) % 128;
    const int x_bytes = mmax * xpitch;
    const int psz = a.p_dt == QLIN_F32 ? 4 : 2;
    const int param_bytes = (int)((2LL * rows_max * NG * psz + 15) / 16 * 16);
    const int aux_bytes = (rows_max * 4 + 15) / 16 * 16;
    smem = code_bytes + x_bytes + param_bytes + aux_bytes + 16;
    // 8 warps while two CTAs fit on an SM (the next layer's fetch overlaps this one); else 16.
    // More than one row group of two tiles on 8 warps measured slower than the ring kernel.
    const int W = 2 * smem <= 227 * 1024 ? 8 : 16;
    if (W == 8 && T > 2)
        return false;
    if (smem > 227 * 1024)
        return false;
    if (out) {
        DecParams& p = *out;
        p.codes = reinterpret_cast<const uint8_t*>(a.codes);
        p.scales = a.scales;
        p.biases = a.biases;
        p.bias = static_cast<const __nv_bfloat16*>(a.bias);
        p.K = (int)a.K;
        p.N = (int)a.N;
        p.NG = (int)NG;
        p.rowbytes = (int)rowbytes;
        p.pitch = pitch;
        p.rows_max = rows_max;
        p.T = T;
        p.RG = RG;
        p.KG = W / RG;
        p.W = W;
        p.p_f32 = a.p_dt == QLIN_F32;
        p.pg = a.pergroup;
        p.code_bytes = code_bytes;
        p.x_bytes = x_bytes;
        p.param_bytes = param_bytes;
        p.aux_bytes = aux_bytes;
        p.xpitch = xpitch;
        p.status = dev.status;
    }
    return true;
}

}  // namespace

cudaError_t launch_affine_dec(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    DecParams prm;
    int grid = 0, smem = 0;
    if (!affine_dec_plan(a, dev, grid, smem, &prm))
        return cudaErrorNotSupported;
    {  // one launch: M <= 8
        prm.x = static_cast<const __nv_bfloat16*>(a.x);
        prm.y = static_cast<__nv_bfloat16*>(a.y);
        prm.M = (int)a.M;
#ifdef QLIN_TRACE
        prm.trace_slot = g_dec_trace_next < kDecTraceSlots ? g_dec_trace_next++ : -1;
#else
        prm.trace_slot = -1;
#endif
        cudaError_t e;
        switch (a.bits * 1000 + a.g) {
        case 2064: e = dec_launch_nt<2, 64>(prm, grid, smem, st); break;
        case 2128: e = dec_launch_nt<2, 128>(prm, grid, smem, st); break;
        case 4032: e = dec_launch_nt<4, 32>(prm, grid, smem, st); break;
        case 4064: e = dec_launch_nt<4, 64>(prm, grid, smem, st); break;
        case 4128: e = dec_launch_nt<4, 128>(prm, grid, smem, st); break;
        case 8032: e = dec_launch_nt<8, 32>(prm, grid, smem, st); break;
        case 8064: e = dec_launch_nt<8, 64>(prm, grid, smem, st); break;
        default: e = dec_launch_nt<8, 128>(prm, grid, smem, st); break;
        }
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace qlin

#ifdef QLIN_TRACE
// Trace build only: copies the affine decode kernel's timestamps ([slot][cta][8] uint64) to a host
// buffer and clears the slot counter; returns the number of slots recorded.
extern "C" int qlin_trace_read_dec(void* host, size_t bytes)
{
    const int used = qlin::g_dec_trace_next;
    const size_t need = (size_t)used * qlin::kDecTraceCtas * 8 * sizeof(unsigned long long);
    if (host && bytes >= need && need > 0 && cudaMemcpyFromSymbol(host, qlin::g_dec_trace, need) != cudaSuccess)
        return -1;
    qlin::g_dec_trace_next = 0;
    return used;
}
#endif
