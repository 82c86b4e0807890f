// k_tc_affine.cu -- affine-format prefill GEMM on the 5th-generation tensor
// cores with the dequantised weights as the tensor-memory A operand, sm_100a.
//
//   y[m,n] = sum_k x[m,k] * (s[n,k/g] q[n,k] + b[n,k/g]) + bias[n]
//   [nuvec-nn QuantizedLinear, forward; cider/ops.py pergroup_linear docstring, dequantize]
//
// Operands are fp16, so that every product is within 2^-11 of the exact one
// (a bf16 operand would allow 2^-8): a preparation kernel writes, into the
// caller's workspace,
//   x16[m,k] = fp16(x[m,k] 2^-E_m)          E_m: max_k |x[m,k]| 2^-E_m in [2^14, 2^15)
//   s16, b16 = fp16(s 2^-F_n), fp16(b 2^-F_n)  F_n: max_g (|b| + (2^bits-1)|s|) 2^-F_n in [2^14, 2^15)
// (exact for bf16 inputs in fp16's normal range: the power-of-two factors keep
// them there and rule out overflow), and the GEMM forms each weight as
// fp16(s16 q + b16) -- the exact value, rounded once -- and scales the fp32
// accumulator by 2^(E_m + F_n) in the epilogue.
//
// Each tile computes the transposed product  yT[128 weight rows][256 tokens] =
// W^ . xT  as one M = 128, N = 256 MMA per 16-wide k step.  The dequantised
// weights never touch shared memory: transform threads (two per weight row,
// 32 k each per stage) read the 4-bit codes straight from global memory, turn
// a code pair into f16x2 in registers and write 16 columns each into tensor
// memory with tcgen05.st; the tensor core reads them there (tcgen05.mma with
// A in TMEM).  Shared memory carries only the x tile (TMA, 128-byte swizzle):
// a stage moves 32 KB in and 32 KB out of it for 128 x 256 x 64 MACs, and
// each dequantised weight serves 256 tokens.
//
// Warp roles (persistent: one CTA per SM walks tiles in a grouped order):
//   warp 0       TMA producer of the x ring (32 KB stages, expect-tx mbarriers)
//   warp 1       allocates 512 TMEM columns: the accumulator (256 columns) at
//                0, the A ring (8 stages x 32 columns) at 256; one thread
//                issues the MMAs and commits ring releases
//   warps 2..9   transform: warp w writes TMEM lanes 32 (w % 4) .. +31, k half
//                (w - 2) / 4 of each stage; the codes of a stage are loaded
//                four stages ahead, the group parameters in 8-group windows
//                with the next window in flight; a stage's tensor-memory store
//                completes while the next stage is decoded
//   warps 10..17 epilogue: warp w reads token half (w - 10) / 4 of lanes
//                32 (w % 4) .. +31: tcgen05.ld, * 2^(E_m + F_n) + bias[n], bf16 stores
// Every mbarrier wait is bounded; on expiry the kernel records the timeout,
// every role stops, the MMA thread waits for its MMAs in flight, and TMEM is
// always freed.
#include "qlin_common.cuh"

namespace qlin {

#ifdef QLIN_TRACE
// Trace build: %globaltimer per CTA and tile of the last launch -- [cta][tile][4]: the MMA thread
// starts the tile (its accumulator free), has issued the tile's last MMA, the epilogue (warp 10)
// sees the accumulator complete, hands it back.  Host side: qlin_trace_read_ts().
constexpr int kTsTraceCtas = 160;
constexpr int kTsTraceTiles = 16;
__device__ unsigned long long g_ts_trace[kTsTraceCtas * kTsTraceTiles * 4];
#define TS_TRACE(ti, i)                                                                             \
    do {                                                                                            \
        if ((int)blockIdx.x < kTsTraceCtas && (ti) < kTsTraceTiles)                                 \
            g_ts_trace[((int)blockIdx.x * kTsTraceTiles + (ti)) * 4 + (i)] = globaltimer_ns();      \
    } while (0)
#else
#define TS_TRACE(ti, i) \
    do {                \
    } while (0)
#endif

namespace {

constexpr int kTW = 128;            // weight rows (outputs n) per tile: MMA M
constexpr int kKE = 64;             // k per stage (128 bytes of bf16 x)
constexpr int kACols = kKE / 2;     // TMEM columns of one A stage (two bf16 per column)
constexpr int kXformWarps = 8;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kXformWarps + kEpiWarps) * 32;
constexpr int kTmemCols = 512;
constexpr int kXStagesMax = 6, kAStagesMax = 8;
// Code formats of the A operand: CB = 4, the MLX affine 4-bit codes with a group scale and bias;
// CB = 8, signed int8 weights with a group scale (the per-group INT8 format).  A transform thread
// covers 32 k of one weight row per stage: 4 * CB bytes of codes, kept kCodePF(CB) stages ahead in
// its slots of a cp.async ring of 24 KB.
// CB = 2 is the BitLinear ternary format: packed bytes [N/4, K], field j of byte [r, k] the code
// of output r + j N/4; a tile's 128 A rows are 32 packed rows x 4 fields (TMEM lane quarter q =
// field q), each transform thread reads 32 bytes of its packed row per stage and keeps its field.
// Its weights {-1, 0, 1, 2} are exact in bf16, so that format runs bf16 A and B straight from the
// caller's x (no preparation kernel, no workspace) and scales by the weight scale in the epilogue.
template <int CB> struct CodeFmt {
    static constexpr int kBytes = CB == 2 ? 32 : 4 * CB;     // code bytes per thread per stage
    static constexpr int kCopies = kBytes / 16;              // 16-byte copies per stage
    static constexpr int kPF = CB == 4 ? 6 : 3;              // stages in flight
    static constexpr bool kTernary = CB == 2;
    static constexpr int kKPerCopy = CB == 4 ? 32 : 16;      // k covered by one 16-byte copy
};
constexpr int kGroupT = 4;          // token tiles that walk the weight tiles together

// per transform thread, kPF stages of its code bytes: [stage][copy][transform thread] x 16 bytes
constexpr int kCodeRing = 6 * kXformWarps * 32 * 16;
static_assert(CodeFmt<4>::kPF * CodeFmt<4>::kCopies <= 6 && CodeFmt<8>::kPF * CodeFmt<8>::kCopies <= 6, "ring");

struct Bars {
    uint64_t xfull[kXStagesMax];
    uint64_t xempty[kXStagesMax];
    uint64_t afull[kAStagesMax];
    uint64_t aempty[kAStagesMax];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t mma_done;
    uint32_t tmem;
    int abort_flag;
    int epi_abort;  // written by epilogue warps only: their common break decision
};
// Tile shapes.  TT = 256 tokens: one 256-column accumulator, an 8-stage A ring and a 6-stage x
// ring.  TT = 384 tokens: two 192-column accumulators (two MMAs of N = 192 per 16-wide k step on
// the same A stage, so each decoded weight serves 384 tokens), a 4-stage A ring and a 4-stage x
// ring of two 192-row boxes per stage -- for shapes where it takes fewer rounds of tiles over the
// SMs (the weight decode, not the MMA, bounds a stage).
template <int TT> struct TsCfg {
    static constexpr int kTT = TT;                        // tokens per tile
    static constexpr int kNMma = TT == 384 ? 2 : 1;       // MMAs (accumulators) per 16-wide k step
    static constexpr int kNT = TT / kNMma;                // MMA N; also the x TMA box rows
    static constexpr int kXStages = TT == 384 ? 4 : 6;    // x ring depth
    static constexpr int kAStages = TT == 384 ? 4 : 8;    // TMEM A ring depth
    static constexpr int kXBytes = TT * 128;              // one x stage
    static constexpr int kAccCols = TT;                   // A ring starts here
    static constexpr int kTokScaleBytes = TT * 4;         // the epilogue's token scales of a tile
    static constexpr int kSmem = kXStages * kXBytes + kCodeRing + kTokScaleBytes + (int)sizeof(Bars) + 1024;
    // kind::f16: D f32, A and B f16 (format 0; bf16 = format 1 for the ternary format), both
    // K-major, N = kNT, M = 128
    static constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kNT >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    static constexpr uint32_t kIdescBf16 = kIdesc | (1u << 7) | (1u << 10);
    static_assert(TT == 256 || TT == 384, "tile widths");
    static_assert(kXStages <= kXStagesMax && kAStages <= kAStagesMax, "barrier slots");
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static_assert(kAccCols + kAStages * kACols <= kTmemCols, "tensor memory");
    static_assert(kNT % 16 == 0 && kNT <= 256 && (kNT * 128) % 1024 == 0, "MMA N and box alignment");
};

struct TsParams {
    CUtensorMap tm_x;                 // x16 [M][K] fp16 (workspace), box {64, 256}, 128-byte swizzle
    const uint8_t* codes;             // [N][K/2]: LSB-first 4-bit codes
    const unsigned short* scales;     // fp16 bits [N][K/g]: s 2^-F_n (workspace)
    const unsigned short* biases;     //                      b 2^-F_n
    const float* tok_scale;           // [M] 2^E_m
    const float* row_scale;           // [N] 2^F_n
    const void* bias;                 // [N] or null, the output dtype
    void* out;                        // [M][N] of out_dt (fp32, bf16 or fp16)
    int out_dt;                       // a qlin_dtype; also the dtype of bias
    int M, N, K;
    int g_shift, ng;                  // log2 g, K / g
    int tiles_t, tiles_w;
    const float* weight_scale;        // ternary format: device scalar (multiplied, or its reciprocal)
    int invert;
    int R;                            // ternary format: packed rows N / 4
    int vec_params;                   // parameter rows allow 16-byte loads of 8 groups
    unsigned* status;
};

QLIN_DEV uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

QLIN_DEV uint32_t bf16x2_min(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

QLIN_DEV uint32_t f16x2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T (kind::f16), one thread.
QLIN_DEV void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

// 16 registers per thread -> this warp's 32 TMEM lanes, 16 consecutive columns.
QLIN_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

QLIN_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16-byte asynchronous global -> shared copy (L2 only); src_bytes = 0 writes zeros.
QLIN_DEV void cp_async16(void* smem_dst, const void* src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
QLIN_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's committed copy groups are still in flight.
template <int N>
QLIN_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

QLIN_DEV bool aborted(int* flag) { return *reinterpret_cast<volatile int*>(flag) != 0; }

// Grouped tile order: kGroupT consecutive token tiles walk the weight tiles together.
QLIN_DEV void tile_coords(int t, int tiles_t, int tiles_w, int& tt, int& wt)
{
    const int per_group = kGroupT * tiles_w;
    const int grp = t / per_group;
    const int first = grp * kGroupT;
    const int gt = min(kGroupT, tiles_t - first);
    const int r = t - grp * per_group;
    tt = first + r % gt;
    wt = r / gt;
}

template <int CB, int TT>
__global__ void __launch_bounds__(kThreads, 1) tc_affine_ts_kernel(const __grid_constant__ TsParams p)
{
    using F = CodeFmt<CB>;
    using C = TsCfg<TT>;
    constexpr int kTT = C::kTT, kXStages = C::kXStages, kAStages = C::kAStages, kXBytes = C::kXBytes;
    constexpr int kAccCols = C::kAccCols;
    constexpr int kCodePF = F::kPF;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint4* code_ring = reinterpret_cast<uint4*>(smem + kXStages * kXBytes);
    float* tok_s = reinterpret_cast<float*>(smem + kXStages * kXBytes + kCodeRing);
    Bars& bars = *reinterpret_cast<Bars*>(smem + kXStages * kXBytes + kCodeRing + C::kTokScaleBytes);
    auto X = [&](int s) { return smem + s * kXBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = (p.K + kKE - 1) / kKE;
    const int tiles = p.tiles_t * p.tiles_w;
    const int my_tiles = tiles > (int)blockIdx.x ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_tiles * nk;  // stages this CTA runs

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(&bars.xfull[s], 1);
            mbar_init(&bars.xempty[s], 1);
        }
        for (int a = 0; a < kAStages; ++a) {
            mbar_init(&bars.afull[a], kXformWarps);
            mbar_init(&bars.aempty[a], 1);
        }
        mbar_init(&bars.acc_full, 1);
        mbar_init(&bars.acc_empty, kEpiWarps);
        mbar_init(&bars.mma_done, 1);
        bars.abort_flag = 0;
        bars.epi_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1)
        tmem_alloc(&bars.tmem, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ x producer
        if (lane == 0) {
            pdl_launch_dependents();
            pdl_wait_prior_grids();  // x may come from the previous kernel
            int it = 0, slot = 0;
            unsigned ph = 0u;
            bool ok = true;
            for (int ti = 0; ti < my_tiles && ok; ++ti) {
                int tt, wt;
                tile_coords((int)blockIdx.x + ti * (int)gridDim.x, p.tiles_t, p.tiles_w, tt, wt);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    if ((it >= kXStages && !mbar_wait_bounded(&bars.xempty[slot], ph ^ 1u, p.status)) ||
                        aborted(&bars.abort_flag)) {
                        bars.abort_flag = 1;
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars.xfull[slot], kXBytes);
#pragma unroll
                    for (int b = 0; b < C::kNMma; ++b)  // boxes of kNT token rows
                        tma_load_2d(X(slot) + b * C::kNT * 128, &p.tm_x, kb * kKE, tt * kTT + b * C::kNT,
                                    &bars.xfull[slot]);
                    if (++slot == kXStages) {
                        slot = 0;
                        ph ^= 1u;
                    }
                }
            }
            // drain: no copy may still be landing in this CTA's shared memory at exit
            for (int j = it - kXStages < 0 ? 0 : it - kXStages; j < it; ++j)
                mbar_wait_bounded(&bars.xfull[j % kXStages], (j / kXStages) & 1, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int xs = 0, as = 0;
            unsigned xph = 0u, aph = 0u;
            bool ok = true;
            for (int ti = 0; ti < my_tiles && ok; ++ti) {
                // the epilogue has read the previous tile's accumulators
                ok = mbar_wait_bounded(&bars.acc_empty, (unsigned)(ti & 1) ^ 1u, p.status);
                tc_fence_after();
                TS_TRACE(ti, 0);
                for (int kb = 0; kb < nk && ok; ++kb) {
                    ok = mbar_wait_bounded(&bars.xfull[xs], xph, p.status) &&
                         mbar_wait_bounded(&bars.afull[as], aph, p.status);
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t b0 = smem_u32(X(xs));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                        for (int b = 0; b < C::kNMma; ++b)  // accumulator b: tokens b kNT .. +kNT-1
                            tc_mma_ts(tmem + (uint32_t)(b * C::kNT), tmem + (uint32_t)(kAccCols + as * kACols + kk * 8),
                                      umma_desc_sw128(b0 + b * C::kNT * 128 + kk * 32),
                                      CodeFmt<CB>::kTernary ? C::kIdescBf16 : C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    tc_commit(&bars.xempty[xs]);
                    tc_commit(&bars.aempty[as]);
                    if (++xs == kXStages) {
                        xs = 0;
                        xph ^= 1u;
                    }
                    if (++as == kAStages) {
                        as = 0;
                        aph ^= 1u;
                    }
                }
                TS_TRACE(ti, 1);
                if (ok)
                    tc_commit(&bars.acc_full);  // fires when this tile's MMAs are done
            }
            if (!ok)
                bars.abort_flag = 1;
            // every MMA issued has completed before TMEM is released
            tc_commit(&bars.mma_done);
            mbar_wait_bounded(&bars.mma_done, 0, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + kXformWarps) {
        // ------------------------------------------------------------ weight transform
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int kh = (warp - 2) >> 2;     // 32-k half of each stage
        const int r = 32 * q + lane;        // weight row within the tile
        const size_t pitch = (size_t)p.K * F::kBytes / 32;  // bytes per code row (kBytes per 32 k)
        pdl_wait_prior_grids();  // the weights' parameters may come from the previous kernel

        auto row_of = [&](int ti) {  // the code row this thread reads in tile ti
            int tt, wt;
            tile_coords((int)blockIdx.x + ti * (int)gridDim.x, p.tiles_t, p.tiles_w, tt, wt);
            if constexpr (F::kTernary)
                return min(wt * 32 + lane, p.R - 1);
            else
                return min(wt * kTW + r, p.N - 1);
        };
        // codes of stage (ti, kb) for this thread: F::kBytes bytes (32 k) of row n, copied kCodePF
        // stages ahead into this thread's slots of the shared-memory ring with cp.async (one commit
        // group per stage, so the wait before a stage's decode is explicit); a half stage past K or
        // a stage past the last tile is written as zeros (zero codes meet the zero-filled x columns)
        int lti = 0, lkb = 0;
        const uint8_t* lrow = my_tiles > 0 ? p.codes + (size_t)row_of(0) * pitch + F::kBytes * kh : p.codes;
        uint4* my_ring = code_ring + (warp - 2) * 32 + lane;  // copy c of slot j: my_ring[(j * kCopies + c) * 256]
        auto load_next = [&](int slot) {
#pragma unroll
            for (int c = 0; c < F::kCopies; ++c) {  // each copy is in range or zero-filled on its own
                const bool in = lti < my_tiles && lkb * kKE + 32 * kh + c * F::kKPerCopy < p.K;
                cp_async16(my_ring + (slot * F::kCopies + c) * kXformWarps * 32,
                           in ? lrow + (size_t)lkb * (F::kBytes * 2) + 16 * c : p.codes, in ? 16 : 0);
            }
            cp_async_commit();
            if (lti < my_tiles && ++lkb == nk) {
                lkb = 0;
                if (++lti < my_tiles)
                    lrow = p.codes + (size_t)row_of(lti) * pitch + F::kBytes * kh;
            }
        };

        // group parameters of this thread's row in windows of 8 groups (16 bytes of scales, 16 of
        // biases); the window after the current one is always in flight
        const int nwin = (p.ng + 7) / 8;
        auto win_load = [&](int ti, int win, uint4& S, uint4& B) {
            if (ti >= my_tiles)
                return;
            const size_t off = (size_t)row_of(ti) * p.ng + 8 * win;
            if (p.vec_params) {
                S = __ldg(reinterpret_cast<const uint4*>(p.scales + off));
                B = __ldg(reinterpret_cast<const uint4*>(p.biases + off));
            } else {
                uint32_t sv[4], bv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int g0 = 8 * win + 2 * e;
                    const uint32_t slo = g0 < p.ng ? __ldg(p.scales + off + 2 * e) : 0u;
                    const uint32_t shi = g0 + 1 < p.ng ? __ldg(p.scales + off + 2 * e + 1) : 0u;
                    const uint32_t blo = g0 < p.ng ? __ldg(p.biases + off + 2 * e) : 0u;
                    const uint32_t bhi = g0 + 1 < p.ng ? __ldg(p.biases + off + 2 * e + 1) : 0u;
                    sv[e] = slo | (shi << 16);
                    bv[e] = blo | (bhi << 16);
                }
                S = make_uint4(sv[0], sv[1], sv[2], sv[3]);
                B = make_uint4(bv[0], bv[1], bv[2], bv[3]);
            }
        };
        uint4 curS = make_uint4(0u, 0u, 0u, 0u), curB = curS, nxtS = curS, nxtB = curS;
        int cur_ti = 0, cur_win = -1;
        // f16x2 (s, s) and (b, b) of this thread's 32 k of stage (ti, kb)
        auto params_for = [&](int ti, int kb, uint32_t& s2, uint32_t& b2) {
            const int gi = min(kb * kKE + 32 * kh, p.K - 1) >> p.g_shift;
            const int win = gi >> 3;
            if (ti != cur_ti || win != cur_win) {
                if (cur_win < 0) {
                    win_load(ti, win, curS, curB);
                } else {
                    curS = nxtS;
                    curB = nxtB;
                }
                cur_ti = ti;
                cur_win = win;
                if (win + 1 < nwin)
                    win_load(ti, win + 1, nxtS, nxtB);
                else
                    win_load(ti + 1, 0, nxtS, nxtB);
            }
            const int sub = gi & 7;
            const uint32_t sw = (sub >> 1) == 0 ? curS.x : (sub >> 1) == 1 ? curS.y : (sub >> 1) == 2 ? curS.z : curS.w;
            const uint32_t bw = (sub >> 1) == 0 ? curB.x : (sub >> 1) == 1 ? curB.y : (sub >> 1) == 2 ? curB.z : curB.w;
            const uint32_t sv = (sw >> (16 * (sub & 1))) & 0xFFFFu, bv = (bw >> (16 * (sub & 1))) & 0xFFFFu;
            s2 = sv | (sv << 16);
            b2 = bv | (bv << 16);
        };

#pragma unroll
        for (int j = 0; j < kCodePF; ++j)
            load_next(j);
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAccCols + 16 * kh);
        // ternary format: this warp keeps field q (mask, and the bf16x2 scale / bias that map
        // 128 + 4^q c to c - 1)
        const uint32_t tmask = 0x00030003u << (2 * q);
        const uint32_t tscale = q == 0 ? 0x3F803F80u : q == 1 ? 0x3E803E80u : q == 2 ? 0x3D803D80u : 0x3C803C80u;
        const uint32_t tbias = q == 0 ? 0xC301C301u : q == 1 ? 0xC204C204u : q == 2 ? 0xC110C110u : 0xC040C040u;
        int ti = 0, kb = 0, as = 0, pend_as = -1;
        unsigned aph = 0u;
        bool ok = true;
        // the tensor-memory store of a stage is published (wait, fence, arrive) after the next stage
        // has been decoded, so its latency overlaps that work
        auto publish = [&]() {
            if (pend_as >= 0) {
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars.afull[pend_as]);
                pend_as = -1;
            }
        };
        for (int base = 0; base < total && ok; base += kCodePF) {
#pragma unroll
            for (int j = 0; j < kCodePF; ++j) {
                if (base + j >= total || !ok)
                    break;
                uint32_t s2 = 0u, b2 = 0u;
                if constexpr (!F::kTernary)
                    params_for(ti, kb, s2, b2);
                // a pair of codes (q, q') of one byte becomes f16x2 in four instructions: PRMT puts
                // the byte (low half) and the byte of w >> 1 (high half) in place, one LOP3 makes the
                // exact fp16 (1024 + q, 1024 + 8 q'), one f16x2 FMA recovers (q, q') exactly, and one
                // gives fp16(s q + b), the exact value rounded once.  Column c holds k = 2c, 2c + 1.
                cp_async_wait<kCodePF - 1>();  // this stage's copy (the oldest in flight) has landed
                uint32_t o[16];
                if constexpr (CB == 4) {
                    const uint4 cbj = my_ring[j * kXformWarps * 32];
                    const uint32_t words[4] = {cbj.x, cbj.y, cbj.z, cbj.w};
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t w1 = words[w] >> 1;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t sel = (uint32_t)(e | (e << 4) | ((4 + e) << 8) | ((4 + e) << 12));
                            const uint32_t v = lop3_and_or(prmt(words[w], w1, sel), 0x0078000Fu, 0x64006400u);
                            const uint32_t qq = f16x2_fma(v, 0x30003C00u, 0xD800E400u);  // (1, 1/8), (-1024, -128)
                            o[4 * w + e] = f16x2_fma(qq, s2, b2);
                        }
                    }
                } else if constexpr (F::kTernary) {
                    // field q of each byte, k in order: PRMT puts bytes (k, k+1) in the low byte of each
                    // bf16 half, one LOP3 masks the field into the mantissa of 128 (0x4300) -- 128 + 4^q c,
                    // exact -- one bf16x2 FMA gives c - 1 exactly, and a min with 2 keeps code 3 at weight
                    // 2 (field 3 lands on the exponent's low bit: 128, 192, 256, 384 -> -1, 0, 1, 3)
                    const uint4 c0 = my_ring[(2 * j) * kXformWarps * 32];
                    const uint4 c1 = my_ring[(2 * j + 1) * kXformWarps * 32];
                    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t v = lop3_and_or(prmt(words[w], 0u, h ? 0x0302u : 0x0100u), tmask, 0x43004300u);
                            o[2 * w + h] = bf16x2_min(bf16x2_fma(v, tscale, tbias), 0x40004000u);
                        }
                    }
                } else {
                    // int8 weights, k in order: the pair (k, k+1) of a byte pair becomes the exact fp16
                    // (1024 + (b ^ 0x80)) per half with one PRMT; one FMA subtracts 1152, leaving the
                    // signed byte exactly, and one multiply gives fp16(s w), rounded once
                    const uint4 c0 = my_ring[(2 * j) * kXformWarps * 32];
                    const uint4 c1 = my_ring[(2 * j + 1) * kXformWarps * 32];
                    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        const uint32_t u = words[w] ^ 0x80808080u;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t v = prmt(u, 0x64646464u, h ? 0x4342u : 0x4140u);
                            const uint32_t qq = f16x2_fma(v, 0x3C003C00u, 0xE480E480u);  // 1, -1152
                            o[2 * w + h] = f16x2_fma(qq, s2, 0u);
                        }
                    }
                }
                load_next(j);  // the stage kCodePF ahead, into the slot just read
                publish();
                if (!mbar_wait_bounded(&bars.aempty[as], aph ^ 1u, p.status) || aborted(&bars.abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_st16(lane_base + (uint32_t)(as * kACols), o);
                pend_as = as;
                if (++as == kAStages) {
                    as = 0;
                    aph ^= 1u;
                }
                if (++kb == nk) {
                    kb = 0;
                    ++ti;
                }
            }
        }
        if (ok)
            publish();
        cp_async_wait<0>();  // no copy may still be landing in shared memory at exit
        tmem_wait_st();  // no store may be in flight when TMEM is released
        if (!ok)
            bars.abort_flag = 1;
    } else {
        // ------------------------------------------------------------ epilogue
        // Everything a tile's epilogue reads from global memory -- the token scales (into shared
        // memory, one per thread), the bias and the row scale -- is fetched before it waits for the
        // tile's accumulator, so those loads overlap the MMAs instead of following them.
        const int q = warp & 3;                        // TMEM lane quarter this warp may access
        const int th = (warp - 2 - kXformWarps) >> 2;  // token half
        const int et = threadIdx.x - (2 + kXformWarps) * 32;  // 0 .. 255 among the epilogue threads
        auto epi_bar = [] { asm volatile("bar.sync 2, %0;" ::"n"(kEpiWarps * 32) : "memory"); };
        pdl_wait_prior_grids();  // bias / out may be touched by the previous kernel
        for (int ti = 0; ti < my_tiles; ++ti) {
            int tt, wt;
            tile_coords((int)blockIdx.x + ti * (int)gridDim.x, p.tiles_t, p.tiles_w, tt, wt);
            const int m0 = tt * kTT + th * (kTT / 2);
            // output row of TMEM lane 32 q + lane: ternary -> packed row 32 wt + lane, field q
            const int n = F::kTernary ? wt * 32 + lane + q * p.R : wt * kTW + 32 * q + lane;
            const bool n_ok = F::kTernary ? wt * 32 + lane < p.R : n < p.N;
            float bn = 0.f;
            if (p.bias && n_ok)
                bn = p.out_dt == QLIN_F32    ? static_cast<const float*>(p.bias)[n]
                     : p.out_dt == QLIN_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.bias)[n])
                                             : __half2float(static_cast<const __half*>(p.bias)[n]);
            float rs = 0.f;
            if (n_ok) {
                if constexpr (F::kTernary) {
                    const float ws = *p.weight_scale;
                    rs = p.invert ? __frcp_rn(ws) : ws;  // 1/ws rounded once, as a division would
                } else {
                    rs = p.row_scale[n];
                }
            }
            if constexpr (!F::kTernary) {  // the tile's token scales (zero past the last token)
                for (int i = et; i < kTT; i += kEpiWarps * 32)
                    tok_s[i] = tt * kTT + i < p.M ? __ldg(p.tok_scale + tt * kTT + i) : 0.f;
            }
            epi_bar();  // the tile's token scales are in shared memory
            // the epilogue warps meet at named barriers, so they break together: a warp whose wait
            // failed (or that saw another role stop) records it in epi_abort, which only they write,
            // and all of them read it after the next barrier
            if (!mbar_wait_bounded(&bars.acc_full, (unsigned)(ti & 1), p.status) || aborted(&bars.abort_flag))
                bars.epi_abort = 1;
            epi_bar();
            if (*reinterpret_cast<volatile int*>(&bars.epi_abort)) {
                bars.abort_flag = 1;
                break;
            }
            tc_fence_after();
            if (warp == 2 + kXformWarps && lane == 0)
                TS_TRACE(ti, 2);
            const uint32_t acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(th * (kTT / 2));
            const size_t o0 = (size_t)m0 * p.N + n;
            // chunk c = 16 tokens of this warp's token half: its accumulators are scaled by
            // 2^E_m 2^F_n (an exact power of two: one rounding in the fma), biased and stored
            auto chunk_out = [&](int c, const uint32_t (&v)[16]) {
                if (!n_ok)
                    return;
                float ts[16];  // token scales of the chunk, times the row scale
                if constexpr (F::kTernary) {
#pragma unroll
                    for (int u = 0; u < 16; ++u)
                        ts[u] = rs;
                } else {
                    const float4* tsp = reinterpret_cast<const float4*>(tok_s + th * (kTT / 2) + c * 16);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 t4 = tsp[u];
                        ts[4 * u] = t4.x * rs;
                        ts[4 * u + 1] = t4.y * rs;
                        ts[4 * u + 2] = t4.z * rs;
                        ts[4 * u + 3] = t4.w * rs;
                    }
                }
                // tokens of the chunk that exist (all 16 except in the last token tile); the output
                // dtype and the token bound are settled once per chunk, the address advances by N
                const int mleft = p.M - (m0 + c * 16);
                const int cnt = mleft < 16 ? mleft : 16;
                const size_t step = (size_t)p.N;
                if (p.out_dt == QLIN_BF16) {
                    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + o0 + (size_t)(c * 16) * step;
                    if (cnt == 16) {
#pragma unroll
                        for (int j = 0; j < 16; ++j, o += step)
                            *o = __float2bfloat16_rn(fmaf(__uint_as_float(v[j]), ts[j], bn));
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j, o += step)
                            if (j < cnt)
                                *o = __float2bfloat16_rn(fmaf(__uint_as_float(v[j]), ts[j], bn));
                    }
                } else if (p.out_dt == QLIN_F16) {
                    __half* o = static_cast<__half*>(p.out) + o0 + (size_t)(c * 16) * step;
#pragma unroll
                    for (int j = 0; j < 16; ++j, o += step)
                        if (j < cnt)
                            *o = __float2half_rn(fmaf(__uint_as_float(v[j]), ts[j], bn));
                } else {
                    float* o = static_cast<float*>(p.out) + o0 + (size_t)(c * 16) * step;
#pragma unroll
                    for (int j = 0; j < 16; ++j, o += step)
                        if (j < cnt)
                            *o = fmaf(__uint_as_float(v[j]), ts[j], bn);
                }
            };
            // two chunks per tensor-memory round trip; the accumulator is handed back to the MMA
            // thread as soon as the last loads have landed, before their chunks are written out
#pragma unroll 1
            for (int c = 0; c < kTT / 32; c += 2) {
                uint32_t v0[16], v1[16];
                tmem_ld16_nowait(acc + (uint32_t)(c * 16), v0);
                tmem_ld16_nowait(acc + (uint32_t)((c + 1) * 16), v1);
                tmem_wait_ld();
                if (c + 2 >= kTT / 32) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars.acc_empty);
                    if (warp == 2 + kXformWarps && lane == 0)
                        TS_TRACE(ti, 3);
                }
                chunk_out(c, v0);
                chunk_out(c + 1, v1);
            }
            epi_bar();  // every epilogue warp is done with this tile's token scales
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemCols);
}


// Power-of-two exponent that brings a magnitude bound v (> 0) into [2^14, 2^15).
QLIN_DEV int prep_shift(float v)
{
    if (!(v > 0.f) || !isfinite(v))
        return 0;
    const int e = ilogbf(v) - 14;
    return e < -120 ? -120 : e > 120 ? 120 : e;
}

QLIN_DEV float block_max(float v, float* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            m = fmaxf(m, red[w]);
        red[32] = m;
    }
    __syncthreads();
    return red[32];
}

// 8 consecutive x values (16-byte aligned) as fp32.
QLIN_DEV void load8(const __nv_bfloat16* p, float (&v)[8])
{
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
QLIN_DEV void load8(const __half* p, float (&v)[8])
{
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
QLIN_DEV void load8(const float* p, float (&v)[8])
{
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Blocks [0, M): token rows of x -> x16 and tok_scale (16-byte loads and stores; a row of up to
// 256 * 8 * VPT values is held in registers between the max and the conversion).
//   QX = 0: x16 = fp16(x 2^-E_m), tok_scale = 2^E_m (the activations as they are);
//   QX = 1: the per-token int8 quantiser -- s = max|x| / 127 (zero -> 1), q = clip(round(x / s),
//           -128, 127) with an IEEE division -- stored as exact fp16 integers, tok_scale = s.
// Blocks [M, M + ceil(N / 8)): one warp per weight row -> fp16 group scales (and biases) scaled by
// 2^-F_n, row_scale = 2^F_n:
//   PG = 0: affine bf16 scales / biases [N][ng], bound max_g |b| + qmax |s|;
//   PG = 1: per-group int8 scales, fp32 [ng][N] (group-major), bound 128 max_g |s|; no biases.
// K % 8 == 0.
template <typename XT, int VPT, int QX, int PG>
__global__ void __launch_bounds__(256) affine_prefill_prep_kernel(
    const XT* __restrict__ x, int M, int K, const void* __restrict__ scales,
    const __nv_bfloat16* __restrict__ biases, int N, int ng, float qmax, __half* __restrict__ x16,
    __half* __restrict__ s16, __half* __restrict__ b16, float* __restrict__ tok_scale, float* __restrict__ row_scale)
{
    pdl_launch_dependents();  // the GEMM waits for this kernel before reading anything it writes
    __shared__ float red[33];
    if ((int)blockIdx.x < M) {
        const int m = blockIdx.x;
        const XT* row = x + (size_t)m * K;
        const int n8 = K / 8;
        float v[VPT][8];
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int c = (int)threadIdx.x + i * 256;
            if (c < n8) {
                load8(row + 8 * c, v[i]);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    mx = fmaxf(mx, fabsf(v[i][e]));
            }
        }
        for (int c = (int)threadIdx.x + VPT * 256; c < n8; c += 256) {  // rows longer than the registers hold
            float t[8];
            load8(row + 8 * c, t);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                mx = fmaxf(mx, fabsf(t[e]));
        }
        const float amax = block_max(mx, red);
        int e = 0;
        float sq = 1.f;
        if constexpr (QX) {
            sq = __fdiv_rn(amax, 127.0f);
            if (sq == 0.f)
                sq = 1.f;
        } else {
            e = prep_shift(amax);
        }
        auto conv = [&](float t) {
            if constexpr (QX)
                return fminf(fmaxf(rintf(__fdiv_rn(t, sq)), -128.f), 127.f);
            else
                return ldexpf(t, -e);
        };
        auto store8 = [&](int c, const float (&t)[8]) {
            uint32_t h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __half2 p2 = __floats2half2_rn(conv(t[2 * i]), conv(t[2 * i + 1]));
                h[i] = *reinterpret_cast<const uint32_t*>(&p2);
            }
            *reinterpret_cast<uint4*>(x16 + (size_t)m * K + 8 * c) = make_uint4(h[0], h[1], h[2], h[3]);
        };
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int c = (int)threadIdx.x + i * 256;
            if (c < n8)
                store8(c, v[i]);
        }
        for (int c = (int)threadIdx.x + VPT * 256; c < n8; c += 256) {
            float t[8];
            load8(row + 8 * c, t);
            store8(c, t);
        }
        if (threadIdx.x == 0)
            tok_scale[m] = QX ? sq : ldexpf(1.f, e);
        return;
    }
    const int n = ((int)blockIdx.x - M) * 8 + (int)(threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (n >= N)
        return;
    auto scale_at = [&](int gi) {
        if constexpr (PG)
            return static_cast<const float*>(scales)[(size_t)gi * N + n];
        else
            return __bfloat162float(static_cast<const __nv_bfloat16*>(scales)[(size_t)n * ng + gi]);
    };
    float bound = 0.f;
    for (int gi = lane; gi < ng; gi += 32) {
        if constexpr (PG)
            bound = fmaxf(bound, 128.f * fabsf(scale_at(gi)));
        else
            bound = fmaxf(bound, fabsf(__bfloat162float(biases[(size_t)n * ng + gi])) + qmax * fabsf(scale_at(gi)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        bound = fmaxf(bound, __shfl_xor_sync(0xffffffffu, bound, o));
    const int f = prep_shift(bound);
    for (int gi = lane; gi < ng; gi += 32) {
        s16[(size_t)n * ng + gi] = __float2half_rn(ldexpf(scale_at(gi), -f));
        if constexpr (!PG)
            b16[(size_t)n * ng + gi] = __float2half_rn(ldexpf(__bfloat162float(biases[(size_t)n * ng + gi]), -f));
    }
    if (lane == 0)
        row_scale[n] = ldexpf(1.f, f);
}

}  // namespace

size_t tc_affine_workspace(int64_t M, int64_t N, int64_t K, int g)
{
    auto a256 = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t ng = (size_t)(K / g);
    const size_t mt = (size_t)(M + 255) / 256 * 256;  // token scales (the epilogue reads none past M)
    return a256((size_t)M * K * 2) + 2 * a256((size_t)N * ng * 2) + a256(mt * 4) + a256((size_t)N * 4);
}

namespace {

// 384-token tiles when they take fewer rounds of tiles over the SMs than 256-token ones (e.g.
// 2048 tokens x 112 weight tiles: 5 rounds instead of 7), else 256
int tile_tokens(int64_t M, int tiles_w, const DeviceInfo& dev)
{
    auto rounds = [&](int tt) { return ((M + tt - 1) / tt * tiles_w + dev.sm_count - 1) / dev.sm_count; };
    return rounds(384) < rounds(256) ? 384 : 256;
}

template <int TT>
cudaError_t launch_ts(void (*kern)(TsParams), const TsParams& prm, cudaStream_t st, const DeviceInfo& dev)
{
    constexpr int kSmem = TsCfg<TT>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess)
        return e;
    const int tiles = prm.tiles_t * prm.tiles_w;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles < dev.sm_count ? tiles : dev.sm_count), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

}  // namespace

cudaError_t launch_tc_bitlinear(const BitlinearArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    TsParams prm = {};
    prm.codes = a.packed;
    prm.scales = nullptr;
    prm.biases = nullptr;
    prm.tok_scale = nullptr;
    prm.row_scale = nullptr;
    prm.bias = a.bias;
    prm.out = a.y;
    prm.out_dt = QLIN_BF16;
    prm.M = (int)a.M;
    prm.N = (int)a.N;
    prm.K = (int)a.K;
    prm.R = (int)(a.N / 4);
    prm.g_shift = 0;
    prm.ng = 1;
    prm.tiles_w = (prm.R + 31) / 32;
    const int tt = tile_tokens(a.M, prm.tiles_w, dev);
    prm.tiles_t = (int)((a.M + tt - 1) / tt);
    prm.vec_params = 0;
    prm.weight_scale = a.weight_scale;
    prm.invert = a.invert;
    prm.status = dev.status;
    if (!encode_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.K, (uint64_t)a.M,
                        (uint64_t)a.K * 2, kKE, tt == 384 ? TsCfg<384>::kNT : TsCfg<256>::kNT))
        return cudaErrorInvalidValue;
    return tt == 384 ? launch_ts<384>(tc_affine_ts_kernel<2, 384>, prm, st, dev)
                     : launch_ts<256>(tc_affine_ts_kernel<2, 256>, prm, st, dev);
}

cudaError_t launch_tc_affine(const TcGemmArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    // workspace: x16 [M][K], s16 / b16 [N][ng] (fp16), tok_scale [M rounded up to 256 tokens],
    // row_scale [N] (fp32) -- the layout tc_affine_workspace sizes
    auto a256 = [](size_t v) { return (v + 255) & ~size_t(255); };
    const int ng = (int)(a.K / a.g);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    __half* x16 = reinterpret_cast<__half*>(ws);
    __half* s16 = reinterpret_cast<__half*>(ws + a256((size_t)a.M * a.K * 2));
    __half* b16 = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(s16) + a256((size_t)a.N * ng * 2));
    float* tok_scale = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(b16) + a256((size_t)a.N * ng * 2));
    const size_t mt = (size_t)(a.M + 255) / 256 * 256;
    float* row_scale = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(tok_scale) + a256(mt * 4));
    {
        const unsigned blocks = (unsigned)(a.M + (a.N + 7) / 8);
        const float qmax = (float)((1 << a.bits) - 1);
        const __nv_bfloat16* bb = static_cast<const __nv_bfloat16*>(a.biases);
        // (activation handling, parameter format) x (x dtype)
        const int form = (a.pergroup && a.M > 1 ? 2 : 0) | (a.pergroup ? 1 : 0);
#define QLIN_PREP(XT, QX, PG)                                                                                   \
    affine_prefill_prep_kernel<XT, 2, QX, PG><<<blocks, 256, 0, st>>>(static_cast<const XT*>(a.a), (int)a.M,    \
                                                                      (int)a.K, a.scales, bb, (int)a.N, ng, qmax, \
                                                                      x16, s16, b16, tok_scale, row_scale)
#define QLIN_PREP_X(QX, PG)                                                                                     \
    switch (a.x_dt) {                                                                                           \
    case QLIN_F32: QLIN_PREP(float, QX, PG); break;                                                             \
    case QLIN_BF16: QLIN_PREP(__nv_bfloat16, QX, PG); break;                                                    \
    default: QLIN_PREP(__half, QX, PG); break;                                                                  \
    }
        switch (form) {
        case 0: QLIN_PREP_X(0, 0); break;
        case 1: QLIN_PREP_X(0, 1); break;
        default: QLIN_PREP_X(1, 1); break;
        }
#undef QLIN_PREP_X
#undef QLIN_PREP
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    TsParams prm;
    prm.codes = static_cast<const uint8_t*>(a.b);
    prm.scales = reinterpret_cast<const unsigned short*>(s16);
    prm.biases = reinterpret_cast<const unsigned short*>(a.pergroup ? s16 : b16);  // read, unused, for int8
    prm.tok_scale = tok_scale;
    prm.row_scale = row_scale;
    prm.bias = a.bias;
    prm.out = a.out;
    prm.out_dt = a.x_dt;
    prm.M = (int)a.M;
    prm.N = (int)a.N;
    prm.K = (int)a.K;
    prm.g_shift = 0;
    while ((1 << prm.g_shift) < a.g)
        ++prm.g_shift;
    prm.ng = (int)(a.K / a.g);
    prm.tiles_w = (int)((a.N + kTW - 1) / kTW);
    const int tt = tile_tokens(a.M, prm.tiles_w, dev);
    prm.tiles_t = (int)((a.M + tt - 1) / tt);
    prm.vec_params = prm.ng % 8 == 0;  // workspace rows are then 16-byte aligned
    prm.status = dev.status;
    if (!encode_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)a.K, (uint64_t)a.M,
                        (uint64_t)a.K * 2, kKE, tt == 384 ? TsCfg<384>::kNT : TsCfg<256>::kNT))
        return cudaErrorInvalidValue;
    prm.weight_scale = nullptr;
    prm.invert = 0;
    prm.R = 0;
    if (tt == 384)
        return launch_ts<384>(a.bits == 8 ? tc_affine_ts_kernel<8, 384> : tc_affine_ts_kernel<4, 384>, prm, st, dev);
    return launch_ts<256>(a.bits == 8 ? tc_affine_ts_kernel<8, 256> : tc_affine_ts_kernel<4, 256>, prm, st, dev);
}

}  // namespace qlin

#ifdef QLIN_TRACE
// Trace build only: the prefill GEMM's per-tile timestamps of the last launch ([cta][tile][4]
// uint64, see g_ts_trace); returns the number of CTAs and tiles recorded per CTA as 1000 c + t.
extern "C" int qlin_trace_read_ts(void* host, size_t bytes)
{
    const size_t need = sizeof(qlin::g_ts_trace);
    if (!host || bytes < need || cudaMemcpyFromSymbol(host, qlin::g_ts_trace, need) != cudaSuccess)
        return -1;
    return qlin::kTsTraceCtas * 1000 + qlin::kTsTraceTiles;
}
#endif
