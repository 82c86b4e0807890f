// k_tc_gemm.cu -- prefill-regime GEMMs on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory), sm_100a.
//
//   raw int8:  c[m,n] = sum_k a[m,k] * b[n,k]                (int32, exact)
//              [cider/ops.py int8_matmul_int32]
//   W8A8:      y[m,n] = acc * s_x[m] * s_w[n] + bias[n]      (acc = qx . w, int32)
//              [cider/ops.py perchannel_linear]
//   W4A8:      y[m,n] = acc * s_x[m] * s_w[n] (+ bias[n]),   acc = qx . (c - 8)
//              [cider/ops.py w4a8_linear, pack_weight_int4]
//
// Persistent, warp-specialised kernel: one CTA per SM walks MT*128 x BN output
// tiles (128 x 256; or, when there are too few tiles to fill the GPU, 128 x 128,
// 128 x 112 or 256 x 112, two 128-token sub-tiles sharing each weight stage) in a
// grouped order: kGroupM M-tiles walk the N-tiles together, so each weight
// tile is fetched from HBM about once and reused from L2.
//   warp 0       TMA producer: A tiles and the B source (int8 B or packed
//                int4) into a shared-memory ring, mbarrier completion
//                (expect-tx).
//   warp 1       allocates two accumulators of MT x BN TMEM columns; one thread
//                issues tcgen05.mma (kind::i8, M = 128, N = BN, K = 32 per
//                instruction, once per sub-tile); tcgen05.commit frees ring
//                slots and transformed B buffers when their MMAs are done, and
//                publishes each finished accumulator to the epilogue.
//   warps 2..    4 MT epilogue warps: tcgen05.ld of one accumulator (warp w owns
//                TMEM lanes 32 (w % 4) .. +31 = 32 output rows of one sub-tile)
//                while the MMAs of the next tile fill the other one; scales,
//                bias, 16-byte stores.
//   then         (W4A8) BN transform threads turn the packed source into an
//                MN-major 128-byte-swizzled operand in a 2-deep buffer: a
//                packed row of k-pairs [K/2][N] is already N-contiguous, so
//                each 16-byte chunk becomes one 16-byte chunk of K row 2i
//                (high nibbles) and one of K row 2i + 1 (low nibbles), no
//                transposition; nibble c -> int8 16 (c - 8) (the epilogue
//                shifts the exact int32 sum back by 4 bits).
//                fence.proxy.async publishes the operand to the tensor core.
// Every mbarrier wait is bounded; on expiry the kernel records the timeout,
// every role stops, the MMA thread waits for its MMAs in flight, and TMEM is
// always freed.
#include "qlin_common.cuh"

namespace qlin {
namespace {

constexpr int kBM = 128;    // output rows (tokens) per tile
constexpr int kGroupM = 8;  // M-tiles that walk the N dimension together
constexpr int kEpiWarps = 4;
constexpr int kSmemBudget = 200 * 1024;
#ifndef QLIN_TC_BDEPTH
#define QLIN_TC_BDEPTH 2
#endif
constexpr int kBDepth = QLIN_TC_BDEPTH;  // transformed-B buffers

enum BSource { B_TMA_I8 = 0, B_W4 = 1 };
enum Epi { E_I32 = 0, E_SCALED = 1 };

__host__ __device__ constexpr int rup(int a, int b) { return (a + b - 1) / b * b; }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }

template <int BSRC, int BN, int MT>
struct TcCfg {
    static constexpr int KE = 128;                          // K elements per stage (128 bytes of A)
    static constexpr int XW = BSRC == B_TMA_I8 ? 0 : BN / 32;  // transform warps: one thread per B column
    static constexpr int B_ATOM = 128 * 128;                // MN-major B: one 128-column atom over K = 128
    static constexpr int TM = MT * kBM;                     // tokens per CTA tile: MT sub-tiles of 128
    static constexpr int EW = MT * kEpiWarps;               // epilogue warps: one per (sub-tile, lane quarter)
    static constexpr int A_BYTES = TM * 128;
    static constexpr int B_BYTES = BN * 128;                // one K-major swizzled B operand
    static constexpr int RAW_BYTES = BSRC == B_W4 ? (KE / 2) * BN : B_BYTES;
    static constexpr int SLOT = rup(A_BYTES + RAW_BYTES, 1024);
    static constexpr int BRING = XW > 0 ? kBDepth * B_BYTES : 0;  // transformed B ring
    static constexpr int NS = cmin(8, (kSmemBudget - BRING) / SLOT);
    static constexpr int THREADS = (2 + EW + XW) * 32;
    static constexpr int ACC_COLS = rup(BN, 128);             // TMEM columns between two accumulators
    static constexpr int TMEM_COLS = 2 * MT * ACC_COLS;       // 2 buffers x MT sub-tiles
    static constexpr uint32_t IDESC =
        (2u << 4) |                                         // D: s32
        (1u << 7) | (1u << 10) |                            // A, B: s8 (signed)
        (BSRC == B_W4 ? (1u << 16) : 0u) |                  // B MN-major (W4A8), else K-major
        ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);  // K-major A
    struct Bars {
        uint64_t full[NS];
        uint64_t empty[NS];
        uint64_t bfull[kBDepth];
        uint64_t bempty[kBDepth];
        uint64_t acc_full[2];
        uint64_t acc_empty[2];
        uint64_t mma_done;
        uint32_t tmem;
        int abort_flag;
    };
    static constexpr int SMEM = NS * SLOT + BRING + (int)sizeof(Bars) + 1024;
    static_assert(NS >= 2, "ring too shallow");
    static_assert(TMEM_COLS <= 512, "tensor memory");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct TcParams {
    CUtensorMap tm_a;  // A [M][K] int8, box {128 B, 128 rows}, 128-byte swizzle
    CUtensorMap tm_b;  // int8 B [N][K] (box {128 B, BN rows}, swizzled) | packed int4 [K/2][N]
                       // (box {BN B, 64 rows})
    int M, N, K;
    int tiles_m, tiles_n;
    void* out;
    const float* s_x;
    const float* s_w;
    const unsigned short* bias;     // [N] bf16, or fp16 when out_f16
    int out_f16;                    // y and bias are fp16 (else bf16)
    int vec_sw, vec_bias, vec_out;  // 16-byte alignment of s_w, bias and out
    unsigned* status;
};

QLIN_DEV void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Grouped tile order: kGroupM consecutive M-tiles walk the N-tiles together.
QLIN_DEV void tile_coords(int t, int tiles_m, int tiles_n, int& mt, int& nt)
{
    const int per_group = kGroupM * tiles_n;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int gm = min(kGroupM, tiles_m - first_m);
    const int r = t - grp * per_group;
    mt = first_m + r % gm;
    nt = r / gm;
}

QLIN_DEV bool aborted(int* flag) { return *reinterpret_cast<volatile int*>(flag) != 0; }

template <int BSRC, int EPI, int BN, int MT>
__global__ void __launch_bounds__(TcCfg<BSRC, BN, MT>::THREADS, 1) tc_gemm_kernel(const __grid_constant__ TcParams p)
{
    using Cfg = TcCfg<BSRC, BN, MT>;
    using Bars = typename Cfg::Bars;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars& bars = *reinterpret_cast<Bars*>(smem + Cfg::NS * Cfg::SLOT + Cfg::BRING);
    auto A = [&](int s) { return smem + s * Cfg::SLOT; };
    auto RAW = [&](int s) { return smem + s * Cfg::SLOT + Cfg::A_BYTES; };  // B itself for int8 B
    auto BT = [&](int b) { return smem + Cfg::NS * Cfg::SLOT + b * Cfg::B_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = (p.K + Cfg::KE - 1) / Cfg::KE;
    const int tiles = p.tiles_m * p.tiles_n;
    // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int my_tiles = tiles > (int)blockIdx.x ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_tiles * nk;  // ring stages this CTA runs
    // 128-token sub-tiles of M-tile mt that hold rows (those wholly past M are neither loaded nor
    // multiplied)
    auto subtiles = [&](int mt) { return min(MT, (p.M - mt * Cfg::TM + kBM - 1) / kBM); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], 1);
        }
        for (int b = 0; b < kBDepth; ++b) {
            mbar_init(&bars.bfull[b], Cfg::XW > 0 ? Cfg::XW : 1);
            mbar_init(&bars.bempty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.acc_full[b], 1);
            mbar_init(&bars.acc_empty[b], Cfg::EW);
        }
        mbar_init(&bars.mma_done, 1);
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1)
        tmem_alloc(&bars.tmem, Cfg::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            pdl_launch_dependents();
            auto load_b = [&](int slot, int kb, int nt) {
                if constexpr (BSRC == B_TMA_I8)
                    tma_load_2d(RAW(slot), &p.tm_b, kb * 128, nt * BN, &bars.full[slot]);
                else
                    tma_load_2d(RAW(slot), &p.tm_b, nt * BN, kb * (Cfg::KE / 2), &bars.full[slot]);
            };
            // W8A8 / W4A8: a layer's weights are not written by the previous kernels of the stream
            // (the ordering rule), so the first stages' weight boxes go out before the dependency
            // wait and stream while the activation quantiser runs; the raw int8 GEMM's B may be
            // an activation and waits first
            auto load_a = [&](int slot, int kb, int mt, int ms) {
                for (int m = 0; m < ms; ++m)
                    tma_load_2d(A(slot) + m * (kBM * 128), &p.tm_a, kb * Cfg::KE, mt * Cfg::TM + m * kBM,
                                &bars.full[slot]);
            };
            int pre = 0, mt0 = 0, nt0 = 0;
            if (EPI == E_SCALED && my_tiles > 0) {
                tile_coords((int)blockIdx.x, p.tiles_m, p.tiles_n, mt0, nt0);
                pre = nk < Cfg::NS ? nk : Cfg::NS;
                for (int kb = 0; kb < pre; ++kb) {
                    mbar_arrive_expect_tx(&bars.full[kb], subtiles(mt0) * (kBM * 128) + Cfg::RAW_BYTES);
                    load_b(kb, kb, nt0);
                }
            }
            pdl_wait_prior_grids();  // A (activations) may come from the previous kernel
            for (int kb = 0; kb < pre; ++kb)
                load_a(kb, kb, mt0, subtiles(mt0));
            int it = 0;
            for (int ti = 0; ti < my_tiles && !aborted(&bars.abort_flag); ++ti) {
                int mt, nt;
                tile_coords((int)blockIdx.x + ti * (int)gridDim.x, p.tiles_m, p.tiles_n, mt, nt);
                const int ms = subtiles(mt);
                int kb = 0;
                for (; kb < nk; ++kb, ++it) {
                    if (it < pre)
                        continue;  // issued above (the first stages of tile 0)
                    const int slot = it % Cfg::NS;
                    if (it >= Cfg::NS && !mbar_wait_bounded(&bars.empty[slot], ((it / Cfg::NS) & 1) ^ 1, p.status)) {
                        bars.abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars.full[slot], ms * (kBM * 128) + Cfg::RAW_BYTES);
                    load_a(slot, kb, mt, ms);
                    load_b(slot, kb, nt);
                }
                if (kb < nk)
                    break;
            }
            // drain: no copy may still be landing in this CTA's shared memory at exit
            for (int j = it - Cfg::NS < 0 ? 0 : it - Cfg::NS; j < it; ++j)
                mbar_wait_bounded(&bars.full[j % Cfg::NS], (j / Cfg::NS) & 1, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int ti = 0; ti < my_tiles && ok; ++ti) {
                const int buf = ti & 1;
                int mt, nt;
                tile_coords((int)blockIdx.x + ti * (int)gridDim.x, p.tiles_m, p.tiles_n, mt, nt);
                const int ms = subtiles(mt);
                ok = mbar_wait_bounded(&bars.acc_empty[buf], ((ti >> 1) & 1) ^ 1, p.status);
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * MT * Cfg::ACC_COLS);
                for (int kb = 0; kb < nk && ok; ++kb, ++it) {
                    const int slot = it % Cfg::NS;
                    ok = mbar_wait_bounded(&bars.full[slot], (it / Cfg::NS) & 1, p.status);
                    if (ok && Cfg::XW > 0)
                        ok = mbar_wait_bounded(&bars.bfull[it % kBDepth], (it / kBDepth) & 1, p.status);
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(A(slot));
                    const uint32_t b0 = smem_u32(Cfg::XW > 0 ? BT(it % kBDepth) : RAW(slot));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // K = 32 per instruction: 32 bytes along a K-major row, or 32 rows (4 swizzle
                        // groups of 1024 bytes) of the MN-major W4A8 operand; every sub-tile of
                        // tokens multiplies the same B operand
                        const uint64_t bd = Cfg::XW > 0 ? umma_desc_sw128_mn(b0 + kk * 4096, Cfg::B_ATOM)
                                                        : umma_desc_sw128(b0 + kk * 32);
#pragma unroll
                        for (int m = 0; m < MT; ++m)
                            if (m < ms)
                                tc_mma<true>(acc + (uint32_t)(m * Cfg::ACC_COLS),
                                             umma_desc_sw128(a0 + m * (kBM * 128) + kk * 32), bd, Cfg::IDESC,
                                             (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&bars.empty[slot]);
                    if (Cfg::XW > 0)
                        tc_commit(&bars.bempty[it % kBDepth]);
                }
                tc_commit(&bars.acc_full[buf]);  // fires when this tile's MMAs are done
            }
            if (!ok)
                bars.abort_flag = 1;
            // every MMA issued has completed before TMEM is released
            tc_commit(&bars.mma_done);
            mbar_wait_bounded(&bars.mma_done, 0, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + Cfg::EW) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int msub = (warp - 2) / kEpiWarps;  // token sub-tile this warp reads back
        pdl_wait_prior_grids();  // scales / bias / out may be touched by the previous kernel
        for (int ti = 0; ti < my_tiles; ++ti) {
            const int buf = ti & 1;
            if (!mbar_wait_bounded(&bars.acc_full[buf], (ti >> 1) & 1, p.status) || aborted(&bars.abort_flag)) {
                bars.abort_flag = 1;
                break;
            }
            tc_fence_after();
            int mt, nt;
            tile_coords((int)blockIdx.x + ti * (int)gridDim.x, p.tiles_m, p.tiles_n, mt, nt);
            const int row = mt * Cfg::TM + msub * kBM + 32 * q + lane;
            const bool row_ok = row < p.M;
            float sx = 0.f;
            if constexpr (EPI == E_SCALED)
                sx = row_ok ? p.s_x[row] : 0.f;
            const uint32_t acc =
                tmem + (uint32_t)((buf * MT + msub) * Cfg::ACC_COLS) + ((uint32_t)(32 * q) << 16);
            // a sub-tile wholly past M was not multiplied: nothing to read back
            const int ncols = msub < subtiles(mt) ? BN / 16 : 0;
#pragma unroll 1
            for (int c = 0; c < ncols; ++c) {
                const int n = nt * BN + c * 16;
                // 16 whole columns with 16-byte aligned rows: vector loads and stores
                const bool full16 = n + 16 <= p.N && p.vec_out && (p.N % (EPI == E_I32 ? 4 : 8)) == 0;
                float sw[16], bb[16];
                if constexpr (EPI != E_I32) {
                    // column constants first, so their latency overlaps the TMEM load
                    if (n < p.N) {
                        if (full16 && EPI == E_SCALED && p.vec_sw) {
                            const float4* s4 = reinterpret_cast<const float4*>(p.s_w + n);
#pragma unroll
                            for (int j4 = 0; j4 < 4; ++j4) {
                                const float4 v = __ldg(s4 + j4);
                                sw[4 * j4] = v.x;
                                sw[4 * j4 + 1] = v.y;
                                sw[4 * j4 + 2] = v.z;
                                sw[4 * j4 + 3] = v.w;
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                sw[j] = EPI == E_SCALED ? __ldg(p.s_w + min(n + j, p.N - 1)) : 1.f;
                        }
                        if (p.bias && full16 && p.vec_bias) {
                            const uint4* b4 = reinterpret_cast<const uint4*>(p.bias + n);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint4 v = __ldg(b4 + h);
                                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    bb[8 * h + 2 * j] = h16_to_float(w4[j], p.out_f16);
                                    bb[8 * h + 2 * j + 1] = h16_to_float(w4[j] >> 16, p.out_f16);
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                bb[j] = p.bias ? h16_to_float(p.bias[min(n + j, p.N - 1)], p.out_f16) : 0.f;
                        }
                    }
                }
                uint32_t r[16];
                tmem_ld16(acc + (uint32_t)(c * 16), r);
                if (!row_ok || n >= p.N)
                    continue;
                if constexpr (EPI == E_I32) {
                    int32_t* o = static_cast<int32_t*>(p.out) + (size_t)row * p.N + n;
                    if (full16) {
#pragma unroll
                        for (int j = 0; j < 16; j += 4)
                            *reinterpret_cast<uint4*>(o + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (n + j < p.N)
                                o[j] = (int32_t)r[j];
                    }
                } else {
                    float v[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float a;
                        if constexpr (EPI == E_SCALED)  // W4 operands are 16 (c - 8): exact shift back
                            a = (float)((int32_t)r[j] >> (BSRC == B_W4 ? 4 : 0)) * (sx * sw[j]);
                        else
                            a = __uint_as_float(r[j]);
                        v[j] = a + bb[j];
                    }
                    unsigned short* o = static_cast<unsigned short*>(p.out) + (size_t)row * p.N + n;
                    const int f16 = p.out_f16;
                    if (full16) {
                        *reinterpret_cast<uint4*>(o) =
                            make_uint4(pack_h16x2(v[0], v[1], f16), pack_h16x2(v[2], v[3], f16),
                                       pack_h16x2(v[4], v[5], f16), pack_h16x2(v[6], v[7], f16));
                        *reinterpret_cast<uint4*>(o + 8) =
                            make_uint4(pack_h16x2(v[8], v[9], f16), pack_h16x2(v[10], v[11], f16),
                                       pack_h16x2(v[12], v[13], f16), pack_h16x2(v[14], v[15], f16));
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (n + j < p.N)
                                o[j] = to_h16(v[j], f16);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.acc_empty[buf]);
        }
    } else if constexpr (Cfg::XW > 0) {
        // ------------------------------------------------------------ B transform
        const int tt = threadIdx.x - (2 + Cfg::EW) * 32;  // 0 .. BN - 1
        constexpr int CPR = BN / 16;                        // 16-byte chunks per packed row
        constexpr int UNITS = 64 * CPR / (32 * Cfg::XW);    // chunks per thread per stage
        static_assert(UNITS * 32 * Cfg::XW == 64 * CPR, "transform split");
        const uint32_t kHi = 0xF0F0F0F0u, kSign = 0x80808080u;
        pdl_wait_prior_grids();  // (a stage is complete only once its activations have landed too)
        // one stage: RAW(slot) -> BT(it % kBDepth)
        // ring positions of stage it: slot / phase of the code ring, buffer / phase of the operand ring
        int slot = 0, bslot = 0;
        unsigned fph = 0u, bph = 0u;
        auto stage = [&]() -> bool {
            if (!mbar_wait_bounded(&bars.full[slot], fph, p.status) ||
                !mbar_wait_bounded(&bars.bempty[bslot], bph ^ 1u, p.status) || aborted(&bars.abort_flag))
                return false;
            uint8_t* dst = BT(bslot);
            const uint8_t* raw = RAW(slot);
            // raw[i][n]: packed row i (k = 2i high nibble, 2i + 1 low) of column n, 64 rows x BN bytes.
            // Consecutive lanes take consecutive 16-byte chunks of a row, so every 8-lane phase of a
            // store writes 8 distinct swizzle chunks of one K row.
            uint4 v[UNITS];
#pragma unroll
            for (int u = 0; u < UNITS; ++u)
                v[u] = *reinterpret_cast<const uint4*>(raw + 16 * (tt + u * 32 * Cfg::XW));
#pragma unroll
            for (int u = 0; u < UNITS; ++u) {
                const int idx = tt + u * 32 * Cfg::XW;
                const int i = idx / CPR, c = idx % CPR;
                const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    hi[j] = (w[j] & kHi) ^ kSign;         // k = 2i:     16 (c - 8)
                    lo[j] = ((w[j] << 4) & kHi) ^ kSign;  // k = 2i + 1
                }
                // MN-major swizzled operand: K row r of atom a at a * 16 KB + (r / 8) * 1024 + (r % 8) * 128
                uint8_t* at = dst + (c >> 3) * Cfg::B_ATOM + (i >> 2) * 1024;
                const int r0 = (2 * i) & 7;
                st_shared_v4(at + r0 * 128 + (((c & 7) ^ r0) << 4), hi[0], hi[1], hi[2], hi[3]);
                st_shared_v4(at + (r0 + 1) * 128 + (((c & 7) ^ (r0 + 1)) << 4), lo[0], lo[1], lo[2], lo[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.bfull[bslot]);
            if (++slot == Cfg::NS) {
                slot = 0;
                fph ^= 1u;
            }
            if (++bslot == kBDepth) {
                bslot = 0;
                bph ^= 1u;
            }
            return true;
        };
        bool ok = true;
        for (int it = 0; it < total && ok; ++it)
            ok = stage();
        if (!ok)
            bars.abort_flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

template <int BSRC, int EPI, int BN, int MT>
cudaError_t launch_t(TcParams& prm, cudaStream_t st, const DeviceInfo& dev)
{
    using Cfg = TcCfg<BSRC, BN, MT>;
    auto kern = tc_gemm_kernel<BSRC, EPI, BN, MT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess)
        return e;
    prm.tiles_m = (prm.M + Cfg::TM - 1) / Cfg::TM;
    prm.tiles_n = (prm.N + BN - 1) / BN;
    const int tiles = prm.tiles_m * prm.tiles_n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles < dev.sm_count ? tiles : dev.sm_count), 1, 1);
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

bool encode_b(TcOp op, CUtensorMap* tm, const TcGemmArgs& a, int bn)
{
    switch (op) {
    case TC_I8_RAW:
    case TC_W8A8:
        return encode_tmap_2d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.K,
                              128, (uint32_t)bn);
    default:  // TC_W4A8
        return encode_tmap_2d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b, (uint64_t)a.N, (uint64_t)(a.K / 2),
                              (uint64_t)a.N, (uint32_t)bn, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
}

template <int BN, int MT>
cudaError_t launch_bn(TcOp op, TcParams& prm, cudaStream_t st, const DeviceInfo& dev)
{
    switch (op) {
    case TC_I8_RAW: return launch_t<B_TMA_I8, E_I32, BN, MT>(prm, st, dev);
    case TC_W8A8: return launch_t<B_TMA_I8, E_SCALED, BN, MT>(prm, st, dev);
    default: return launch_t<B_W4, E_SCALED, BN, MT>(prm, st, dev);  // TC_W4A8
    }
}

template <int MT>
cudaError_t launch_i8_112(TcOp op, TcParams& prm, cudaStream_t st, const DeviceInfo& dev)
{
    if (op == TC_I8_RAW)
        return launch_t<B_TMA_I8, E_I32, 112, MT>(prm, st, dev);
    return launch_t<B_TMA_I8, E_SCALED, 112, MT>(prm, st, dev);
}

bool aligned16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// The CTA tile of an M x N output on sms SMs: mt sub-tiles of 128 tokens by bn columns.
void tc_tile_shape(TcOp op, int64_t M, int64_t N, int64_t sms, int& mt, int& bn)
{
    // 128 x 256 tiles when they still give every SM a tile. Otherwise the tile shape, MT sub-tiles
    // of 128 tokens by BN columns, with the least estimated time per SM: (tile rounds) x (the
    // longer of a K stage's tensor-core work and the time one SM takes to draw the stage's operand
    // bytes from L2). At these shapes the intake of one SM, about 65 GB/s, is the bound whether
    // 148 or 74 SMs are busy, so the bytes a tile draws per K step (MT x 128 token rows plus the
    // weight rows) decide: e.g. for 8192 x 8192 weights, 128 x 112 tiles at 256 tokens (148 tiles,
    // 240 rows each) and 256 x 112 tiles at 384 or 512 tokens (148 tiles, 368 rows each, instead
    // of two rounds of 240). Two sub-tiles share each weight stage between two accumulators.
    mt = 1;
    bn = 256;
    if (((M + kBM - 1) / kBM) * ((N + 255) / 256) < sms) {
        constexpr double kMmaNs = 128.0 * 128 * 2 / 21.5e3;  // ns per token x column of one stage (int8)
        constexpr double kIntakeNs = 128.0 / 65.0;           // ns per operand row of one stage, one SM
        double best = 0;
        for (int m = 1; m <= 2; ++m)
            for (int w : {256, 128, 112}) {
                // two sub-tiles with 112-column int8 B tiles only (the other two-sub-tile shapes
                // were slower wherever they were measured)
                if ((w == 112 && op == TC_W4A8) || (m == 2 && w != 112))
                    continue;
                const int64_t tiles = ((M + m * kBM - 1) / (m * kBM)) * ((N + w - 1) / w);
                const int64_t rounds = (tiles + sms - 1) / sms;
                const double rows = m * kBM + (op == TC_W4A8 ? w / 2 : w);
                const double mma = kMmaNs * m * w, intake = kIntakeNs * rows;
                const double t = (double)rounds * (mma > intake ? mma : intake);
                if (best == 0 || t < best) {
                    best = t;
                    mt = m;
                    bn = w;
                }
            }
    }
}

cudaError_t launch_tc_gemm(TcOp op, const TcGemmArgs& a, cudaStream_t st, const DeviceInfo& dev)
{
    TcParams prm;
    prm.M = (int)a.M;
    prm.N = (int)a.N;
    prm.K = (int)a.K;
    prm.out = a.out;
    prm.s_x = a.s_x;
    prm.s_w = a.s_w;
    prm.bias = static_cast<const unsigned short*>(a.bias);
    prm.out_f16 = a.x_dt == QLIN_F16;
    prm.vec_sw = aligned16p(a.s_w);
    prm.vec_bias = aligned16p(a.bias);
    prm.vec_out = aligned16p(a.out);
    prm.status = dev.status;
    if (!encode_tmap_2d(&prm.tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K,
                        128, kBM))
        return cudaErrorInvalidValue;
    int mt, bn;
    tc_tile_shape(op, a.M, a.N, dev.sm_count, mt, bn);
    if (!encode_b(op, &prm.tm_b, a, bn))
        return cudaErrorInvalidValue;
    if (bn == 256)
        return launch_bn<256, 1>(op, prm, st, dev);
    if (bn == 112)
        return mt == 2 ? launch_i8_112<2>(op, prm, st, dev) : launch_i8_112<1>(op, prm, st, dev);
    return launch_bn<128, 1>(op, prm, st, dev);
}

}  // namespace qlin
