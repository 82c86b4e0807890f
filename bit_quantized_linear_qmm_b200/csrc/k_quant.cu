// k_quant.cu -- quantisers and the dequantiser (bandwidth-bound, bit-exact).
//
//  * affine group quantize / dequantize of the MLX format
//    [nuvec-nn QuantizedLinear: from_linear, dequantized_weight;
//     cider/ops.py pergroup_linear docstring: quantize and dequantize formulas]
//  * per-row symmetric int8 (weights and per-token activations)
//    [cider/ops.py quantize_weight_int8; quant_a of perchannel_linear / w4a8_linear]
//  * per-column int4 with zero point 8, two codes per byte
//    [cider/ops.py pack_weight_int4]
//
// Every quantisation decision is taken in fp32 with IEEE operations that
// cannot be contracted (__fsub_rn / __fdiv_rn / __fmaf_rn) and rintf (round
// half to even), so codes match the CPU reference bit for bit.
#include "qlin_common.cuh"

#include <type_traits>

namespace qlin {
namespace {

template <typename T> struct Vec;  // loads of N consecutive elements as floats

QLIN_DEV float load_elem(const float* p, int64_t i) { return p[i]; }
QLIN_DEV float load_elem(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }
QLIN_DEV float load_elem(const __half* p, int64_t i) { return __half2float(p[i]); }

// 16 consecutive elements from a 16-byte aligned address, as floats
QLIN_DEV void load16(const float* p, float (&v)[16])
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(p) + q);
        v[4 * q] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
    }
}
QLIN_DEV float lo_half_to_float(uint32_t u, const __nv_bfloat16*) { return __uint_as_float(u << 16); }
QLIN_DEV float hi_half_to_float(uint32_t u, const __nv_bfloat16*) { return __uint_as_float(u & 0xffff0000u); }
QLIN_DEV float lo_half_to_float(uint32_t u, const __half*)
{
    return __half2float(__ushort_as_half((unsigned short)(u & 0xffffu)));
}
QLIN_DEV float hi_half_to_float(uint32_t u, const __half*) { return __half2float(__ushort_as_half((unsigned short)(u >> 16))); }
template <typename T>
QLIN_DEV void load16(const T* p, float (&v)[16])  // bf16 / fp16: element 2j in the low half of word j
{
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + q);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * q + 2 * j] = lo_half_to_float(w4[j], p);
            v[8 * q + 2 * j + 1] = hi_half_to_float(w4[j], p);
        }
    }
}

// rint(d / s) of the quotient rounded once, as an IEEE single division rounds it, for s > 0.
// With r = 1/s and m = d * r each rounded once, m = q (1 + e1)(1 + e2) for the exact quotient q
// and |e1|, |e2| <= 2^-24, while the rounded quotient is q (1 + e3), |e3| <= 2^-24: the two differ
// by less than 1.8e-7 |q|, under 1e-4 while |m| < 512.  rint changes value only at half-integers,
// so rint(m) is rint of the rounded quotient whenever m lies more than 1e-4 from a half-integer,
// i.e. whenever its distance to the nearest integer, |m - rint(m)| (exact for |m| < 2^23), is
// under 0.4999; within that band (and for |m| >= 512) the division itself is done.  r must come
// from a normal s (fast = false otherwise, and every element divides): r is then finite and both
// roundings are relative.
QLIN_DEV bool rcp_ok(float s) { return s >= 1.17549435e-38f && s <= 8.0e37f; }  // s and 1/s normal
QLIN_DEV float rint_div(float d, float s, float r, bool fast)
{
    if (fast) {
        const float m = __fmul_rn(d, r);
        const float t = rintf(m);
        if (fabsf(__fsub_rn(m, t)) < 0.4999f && fabsf(m) < 512.0f)
            return t;
    }
    return rintf(__fdiv_rn(d, s));
}

// ---------------------------------------------------------------- affine quantize
// G/16 lanes per group, each holding 16 consecutive values (16-byte loads) and storing its own
// 16 codes as whole words (2-, 4- and 8-bit codes; 16-byte aligned weights).  The matrix is a flat
// run of N*K/G groups: the parameters [N][K/G] and the code words [N][K*BITS/32] follow the same
// order.  The group's lanes find its min and max with G/16 - 1 butterfly steps.
template <typename TW, typename TP, int BITS, int G>
__global__ void __launch_bounds__(256) affine_quantize_vec_kernel(const TW* __restrict__ w, int64_t groups,
                                                                  uint32_t* __restrict__ codes,
                                                                  TP* __restrict__ scales, TP* __restrict__ biases)
{
    constexpr int LPG = G / 16;               // lanes per group
    constexpr int WPT = 16 * BITS / 32;       // code words per lane
    constexpr float QMAX = float((1 << BITS) - 1);
    static_assert(BITS == 2 || BITS == 4 || BITS == 8, "whole words per lane");
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t gi = t / LPG;
    const int sub = (int)(t % LPG);
    // lanes past the last group (in the last warp only) work on the last group and store nothing,
    // so that every lane takes part in the butterfly
    const bool ok = gi < groups;
    const int64_t gq = ok ? gi : groups - 1;
    float v[16];
    load16(w + gq * G + 16 * sub, v);
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) {
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    float scale = __fdiv_rn(__fsub_rn(mx, mn), QMAX);
    float bias = mn;
    scale = to_float(from_float<TP>(scale));
    bias = to_float(from_float<TP>(bias));
    if (scale == 0.0f)
        scale = 1.0f;
    if (ok && sub == 0) {
        scales[gi] = from_float<TP>(scale);
        biases[gi] = from_float<TP>(bias);
    }
    uint32_t word[WPT];
#pragma unroll
    for (int j = 0; j < WPT; ++j)
        word[j] = 0u;
    const float rs = __frcp_rn(scale);
    const bool fast = rcp_ok(scale);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float q = rint_div(__fsub_rn(v[i], bias), scale, rs, fast);
        q = fminf(fmaxf(q, 0.0f), QMAX);
        word[i * BITS / 32] |= static_cast<uint32_t>(q) << ((i * BITS) % 32);
    }
    if (ok) {
        uint32_t* dst = codes + gi * (G * BITS / 32) + sub * WPT;
#pragma unroll
        for (int j = 0; j < WPT; ++j)
            dst[j] = word[j];
    }
}

// One warp per (row, group).  Lane l holds CPL = g/32 consecutive values.
template <typename TW, typename TP, int BITS, int G>
__global__ void __launch_bounds__(256) affine_quantize_kernel(const TW* __restrict__ w, int64_t N, int64_t K,
                                                              uint32_t* __restrict__ codes, TP* __restrict__ scales,
                                                              TP* __restrict__ biases)
{
    constexpr int CPL = G / 32;          // codes per lane
    constexpr int CPW = 32 / BITS;       // codes per word
    constexpr int LPW = CPW / CPL;       // lanes sharing one word
    constexpr float QMAX = float((1 << BITS) - 1);
    const int64_t groups_per_row = K / G;
    const int64_t gid = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (gid >= N * groups_per_row)
        return;
    const int lane = threadIdx.x & 31;
    const int64_t n = gid / groups_per_row;
    const int64_t gi = gid % groups_per_row;
    const TW* wg = w + n * K + gi * G + lane * CPL;
    float v[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        v[i] = load_elem(wg, i);
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < CPL; ++i) {
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    float scale = __fdiv_rn(__fsub_rn(mx, mn), QMAX);
    float bias = mn;
    scale = to_float(from_float<TP>(scale));
    bias = to_float(from_float<TP>(bias));
    if (scale == 0.0f)
        scale = 1.0f;
    if (lane == 0) {
        scales[n * groups_per_row + gi] = from_float<TP>(scale);
        biases[n * groups_per_row + gi] = from_float<TP>(bias);
    }
    uint32_t part = 0;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        float t = rintf(__fdiv_rn(__fsub_rn(v[i], bias), scale));
        t = fminf(fmaxf(t, 0.0f), QMAX);
        const int k_in_word = (lane * CPL + i) % CPW;
        part |= static_cast<uint32_t>(t) << (BITS * k_in_word);
    }
#pragma unroll
    for (int off = 1; off < LPW; off <<= 1)
        part |= __shfl_xor_sync(0xffffffffu, part, off);
    if (lane % LPW == 0) {
        const int64_t words_per_row = K * BITS / 32;
        codes[n * words_per_row + gi * (G * BITS / 32) + (lane * CPL) / CPW] = part;
    }
}

// ---------------------------------------------------------------- affine dequantize
// One thread per packed word, in flat form: code c of the [N][K] matrix is field c % CPW of word
// c / CPW and belongs to group c / G of the [N][K/G] parameters (K is a multiple of G), and out[c]
// is its value -- no row / column arithmetic.  A word never straddles a group (CPW <= G).
template <typename TP, typename TO, int BITS, int G>
__global__ void __launch_bounds__(256) affine_dequantize_kernel(const uint32_t* __restrict__ codes,
                                                                const TP* __restrict__ scales,
                                                                const TP* __restrict__ biases, int64_t total,
                                                                TO* __restrict__ out)
{
    constexpr int CPW = 32 / BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c0 = idx * CPW;
        const float s = to_float(scales[c0 / G]);
        const float b = to_float(biases[c0 / G]);
        const uint32_t word = __ldg(codes + idx);
        TO vals[CPW];
#pragma unroll
        for (int i = 0; i < CPW; ++i)
            vals[i] = from_float<TO>(__fmaf_rn(static_cast<float>((word >> (BITS * i)) & MASK), s, b));
        // CPW * sizeof(TO) is 8..64 bytes and out + c0 is aligned to it.
        constexpr int BYTES = CPW * (int)sizeof(TO);
        TO* dst = out + c0;
        if constexpr (BYTES >= 16) {
#pragma unroll
            for (int c = 0; c < BYTES / 16; ++c)
                reinterpret_cast<uint4*>(dst)[c] = reinterpret_cast<const uint4*>(vals)[c];
        } else {
            *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(vals);
        }
    }
}

// ---------------------------------------------------------------- affine quantize, 3 / 5 / 6 bits
// A row's codes form one LSB-first bitstream (code k at bits k*BITS ..), so a code may continue in
// the next word; a group of G codes fills exactly WPG = G*BITS/32 whole words.  One warp per
// (row, group) as above: lane l packs its CPL codes into v (bits l*CPL*BITS ..), and word j of the
// group is the warp-wide OR of every lane's part that falls inside it.
template <typename TW, typename TP, int BITS, int G>
__global__ void __launch_bounds__(256) affine_quantize_odd_kernel(const TW* __restrict__ w, int64_t N, int64_t K,
                                                                  uint32_t* __restrict__ codes,
                                                                  TP* __restrict__ scales, TP* __restrict__ biases)
{
    constexpr int CPL = G / 32;
    constexpr int NB = CPL * BITS;  // bits per lane, at most 24
    constexpr int WPG = G * BITS / 32;
    constexpr float QMAX = float((1 << BITS) - 1);
    const int64_t groups_per_row = K / G;
    const int64_t gid = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (gid >= N * groups_per_row)
        return;
    const int lane = threadIdx.x & 31;
    const int64_t n = gid / groups_per_row;
    const int64_t gi = gid % groups_per_row;
    const TW* wg = w + n * K + gi * G + lane * CPL;
    float v[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        v[i] = load_elem(wg, i);
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < CPL; ++i) {
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    float scale = to_float(from_float<TP>(__fdiv_rn(__fsub_rn(mx, mn), QMAX)));
    const float bias = to_float(from_float<TP>(mn));
    if (scale == 0.0f)
        scale = 1.0f;
    if (lane == 0) {
        scales[n * groups_per_row + gi] = from_float<TP>(scale);
        biases[n * groups_per_row + gi] = from_float<TP>(bias);
    }
    uint32_t part = 0;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        float t = rintf(__fdiv_rn(__fsub_rn(v[i], bias), scale));
        t = fminf(fmaxf(t, 0.0f), QMAX);
        part |= static_cast<uint32_t>(t) << (BITS * i);
    }
    const int o = lane * NB;  // first bit of this lane's part within the group
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < WPG; ++j) {
        const int lo = 32 * j;
        uint32_t c = 0;
        if (o >= lo && o < lo + 32)
            c = part << (o - lo);  // the part starts in word j (its high bits may spill over)
        else if (o < lo && o + NB > lo)
            c = part >> (lo - o);  // the part started in word j-1 and ends in word j
        const uint32_t word = __reduce_or_sync(0xffffffffu, c);
        if (lane == j)
            mine = word;
    }
    if (lane < WPG)
        codes[n * (K * BITS / 32) + gi * WPG + lane] = mine;
}

// Dequantize for widths whose codes straddle words: one thread per 32 codes, which are BITS
// whole words of one group (groups are multiples of 32 codes).
template <typename TP, typename TO, int BITS>
__global__ void __launch_bounds__(256) affine_dequantize_odd_kernel(const uint32_t* __restrict__ codes,
                                                                    const TP* __restrict__ scales,
                                                                    const TP* __restrict__ biases, int64_t N,
                                                                    int64_t K, int g, TO* __restrict__ out)
{
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    const int64_t chunks_per_row = K / 32;
    const int64_t total = N * chunks_per_row;
    const int64_t groups_per_row = K / g;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / chunks_per_row;
        const int64_t k0 = (idx % chunks_per_row) * 32;
        const float s = to_float(scales[n * groups_per_row + k0 / g]);
        const float b = to_float(biases[n * groups_per_row + k0 / g]);
        uint32_t wd[BITS];
#pragma unroll
        for (int i = 0; i < BITS; ++i)
            wd[i] = __ldg(codes + idx * BITS + i);  // the row's words k0*BITS/32 ..; rows are whole chunks
        __align__(16) TO vals[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int bp = i * BITS, wi = bp / 32, sh = bp % 32;
            uint32_t q = wd[wi] >> sh;
            if (sh + BITS > 32)
                q |= wd[wi + 1] << (32 - sh);
            vals[i] = from_float<TO>(__fmaf_rn(static_cast<float>(q & MASK), s, b));
        }
        // 64 or 128 bytes at out + n*K + k0, a multiple of 64 bytes from the 16-byte aligned base
        uint4* dst = reinterpret_cast<uint4*>(out + n * K + k0);
#pragma unroll
        for (int c = 0; c < 32 * (int)sizeof(TO) / 16; ++c)
            dst[c] = reinterpret_cast<const uint4*>(vals)[c];
    }
}

// ---------------------------------------------------------------- per-row int8
// The symmetric int8 code clamp(rint(x / s), -128, 127) of an element with |x| <= amax, s = amax /
// 127 rounded once (or 1 for amax = 0), r = 1/s rounded once.  On the multiply path (rint_div's
// argument, with s and 1/s normal) |x r| <= 127 (1 + 3 2^-24), so the code already lies in
// [-127, 127] and needs no clamp; the division path clamps (a NaN element gives
// fminf(fmaxf(NaN, -128), 127) = -128, as the division form always did).
QLIN_DEV int sym_code(float x, float s, float r, bool fast)
{
    if (fast) {
        const float m = __fmul_rn(x, r);
        const float t = rintf(m);
        if (fabsf(__fsub_rn(m, t)) < 0.4999f)
            return (int)t;
    }
    return (int)fminf(fmaxf(rintf(__fdiv_rn(x, s)), -128.0f), 127.0f);
}

// four int8 codes -> one word, code i in byte i
QLIN_DEV uint32_t pack4(int a, int b, int c, int d)
{
    return prmt(prmt((uint32_t)a, (uint32_t)b, 0x0040u), prmt((uint32_t)c, (uint32_t)d, 0x0040u), 0x5410u);
}

// the row's absmax over the block (NW warps) from each thread's partial
template <int NW = 8>
QLIN_DEV float block_amax(float amax, float* red)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x / 32] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < NW; ++i)
        amax = fmaxf(amax, red[i]);
    return amax;
}

// eight bf16 of a 16-byte piece -> four code words pair: codes of elements 0..3 and 4..7.
// The multiply path is tested once for the whole piece (one branch, not eight): when every
// product lies clear of a half-integer its codes are those sym_code gives; otherwise every
// element goes through sym_code.
QLIN_DEV uint2 sym_codes8(const uint4& v, float s, float r, bool fast)
{
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        x[i] = __uint_as_float((i & 1) ? (u[i / 2] & 0xffff0000u) : (u[i / 2] << 16));
    int c[8];
    if (fast) {
        bool clear = true;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float m = __fmul_rn(x[i], r);
            const float t = rintf(m);
            clear &= fabsf(__fsub_rn(m, t)) < 0.4999f;
            c[i] = (int)t;
        }
        if (clear)
            return make_uint2(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        c[i] = sym_code(x[i], s, r, fast);
    return make_uint2(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
}

QLIN_DEV float amax8(const uint4& v, float amax)
{
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        amax = fmaxf(amax, fabsf(__uint_as_float(u[i] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(u[i] & 0xffff0000u)));
    }
    return amax;
}

// One block (256 threads) per row: absmax, then quantise (second read comes from L1/L2).
template <typename TW>
__global__ void __launch_bounds__(256) quantize_int8_rows_kernel(const TW* __restrict__ w, int64_t C,
                                                                 int8_t* __restrict__ q, float* __restrict__ scale,
                                                                 int release)
{
    if (release)
        pdl_launch_dependents();
    pdl_wait_prior_grids();  // w and the outputs belong to the stream's earlier kernels until they complete
    __shared__ float red[8];
    const int64_t r = blockIdx.x;
    const TW* row = w + r * C;
    float amax = 0.0f;
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x)
        amax = fmaxf(amax, fabsf(load_elem(row, c)));
    amax = block_amax(amax, red);
    float s = __fdiv_rn(amax, 127.0f);
    if (s == 0.0f)
        s = 1.0f;
    if (threadIdx.x == 0)
        scale[r] = s;
    int8_t* qrow = q + r * C;
    const float rs = __frcp_rn(s);
    const bool fast = rcp_ok(s);
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x)
        qrow[c] = static_cast<int8_t>(sym_code(load_elem(row, c), s, rs, fast));
}

// Single-pass variant for bf16 rows with C % 8 == 0 and C <= NT * 8 * VPT: each
// thread keeps its VPT 16-byte pieces of the row in registers between the
// absmax reduction and the quantisation, so the row is read from memory once.
// A launch of few rows takes NT = 512 or 1024 threads per row: a thread's
// dependent chain (load, absmax, codes) is then a few pieces long, and the
// GPU holds enough warps to hide its latency.
template <int NT, int VPT>
__global__ void __launch_bounds__(NT) quantize_int8_rows_bf16_reg_kernel(const __nv_bfloat16* __restrict__ w,
                                                                        int64_t C, int8_t* __restrict__ q,
                                                                        float* __restrict__ scale, int release)
{
    if (release)
        pdl_launch_dependents();
    pdl_wait_prior_grids();  // w and the outputs belong to the stream's earlier kernels until they complete
    __shared__ float red[NT / 32];
    const int64_t r = blockIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(w + r * C);
    const int C8 = (int)(C / 8);
    uint4 v[VPT];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int c = (int)threadIdx.x + j * NT;
        v[j] = c < C8 ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
        amax = amax8(v[j], amax);
    }
    amax = block_amax<NT / 32>(amax, red);
    float s = __fdiv_rn(amax, 127.0f);
    if (s == 0.0f)
        s = 1.0f;
    if (threadIdx.x == 0)
        scale[r] = s;
    uint2* qrow = reinterpret_cast<uint2*>(q + r * C);
    const float rs = __frcp_rn(s);
    const bool fast = rcp_ok(s);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int c = (int)threadIdx.x + j * NT;
        if (c < C8)
            qrow[c] = sym_codes8(v[j], s, rs, fast);
    }
}

// Vectorised variant for bf16 rows with C % 8 == 0 (16-byte loads, 8-byte stores).
__global__ void __launch_bounds__(256) quantize_int8_rows_bf16x8_kernel(const __nv_bfloat16* __restrict__ w,
                                                                        int64_t C, int8_t* __restrict__ q,
                                                                        float* __restrict__ scale, int release)
{
    if (release)
        pdl_launch_dependents();
    pdl_wait_prior_grids();  // w and the outputs belong to the stream's earlier kernels until they complete
    __shared__ float red[8];
    const int64_t r = blockIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(w + r * C);
    const int64_t C8 = C / 8;
    float amax = 0.0f;
    for (int64_t c = threadIdx.x; c < C8; c += blockDim.x)
        amax = amax8(__ldg(row + c), amax);
    amax = block_amax(amax, red);
    float s = __fdiv_rn(amax, 127.0f);
    if (s == 0.0f)
        s = 1.0f;
    if (threadIdx.x == 0)
        scale[r] = s;
    uint2* qrow = reinterpret_cast<uint2*>(q + r * C);
    const float rs = __frcp_rn(s);
    const bool fast = rcp_ok(s);
    for (int64_t c = threadIdx.x; c < C8; c += blockDim.x)
        qrow[c] = sym_codes8(__ldg(row + c), s, rs, fast);
}

// ---------------------------------------------------------------- per-column int4
// Block = 32 columns x 8 row slices.
// ---------------------------------------------------------------- per-row int8 with a percentile clip
// One CTA per row [cider/ops.py quantize_weight_int8, clip_percentile]: the clip is the
// linear-interpolated percentile of |w| at h = (C - 1) p / 100, which needs only the order
// statistics v_(j) and v_(j+1), j = floor(h).  |w| of the row is held in shared memory as uint32
// bit patterns (non-negative floats order like their bits).  First one pass builds a 2048-bin
// histogram of the top 11 bits (the exponent and three mantissa bits) and a block scan finds the
// bin B holding rank j; when B holds at most 256 values they are gathered and ranked by counting
// (v_(j) and, inside B, v_(j+1); past B, v_(j+1) is the smallest value of a higher bin, a minimum
// taken in the same gather pass).  A denser bin takes the general route: a radix select (four
// passes of a 256-bin histogram of one byte, most significant first, over the values that match
// the bytes found so far), with v_(j+1) = v_(j) again when more than j + 1 values are <= it, else
// the smallest value above it.  Both routes select on the same bit patterns.  The interpolation runs in float32 with every operation rounded
// separately (as numpy does it for a float32 row), 0 -> max |w|; then scale = clip / 127 (zero ->
// 1), w clipped to [-clip, clip], q = clip(round(w / scale), -128, 127) with IEEE divisions.
template <typename TW>
__global__ void __launch_bounds__(256) quantize_weight_int8_clip_kernel(const TW* __restrict__ w, int64_t C,
                                                                       float pct, int8_t* __restrict__ q,
                                                                       float* __restrict__ scale)
{
    extern __shared__ uint32_t sv[];  // [C] fp32 bit patterns of w (|w| is the pattern & 0x7FFFFFFF)
    __shared__ unsigned hist[256];
    __shared__ unsigned hist11[2048];  // by the top 11 bits of the pattern (bit 31 is 0)
    __shared__ uint32_t cand[256];     // the values of bin B (fast route)
    __shared__ unsigned wsum[8];
    __shared__ uint32_t sel_s, rank_s;
    __shared__ unsigned cnt_le_s;
    __shared__ uint32_t next_s, max_s, vj_s, vj1_s;
    __shared__ unsigned fbin_s, frank_s, fcnt_s, gcount_s;
    __shared__ float row_clip_s, scale_s;
    const int n = (int)C;
    const TW* row = w + (int64_t)blockIdx.x * C;
    uint32_t mx = 0u;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const uint32_t b = __float_as_uint(to_float(row[i]));
        sv[i] = b;
        mx = max(mx, b & 0x7FFFFFFFu);
    }
    // the rank of v_(j): j = floor((n - 1) q) when that is below n - 1 (else the maximum is used)
    const float qq = __fdiv_rn(pct, 100.0f);
    const float h = __fmul_rn((float)(n - 1), qq);
    const bool interior = h < (float)(n - 1);
    const int j = interior ? (int)floorf(h) : n - 1;
    if (threadIdx.x == 0) {
        sel_s = 0u;
        rank_s = (uint32_t)j;
        max_s = 0u;
        next_s = 0xFFFFFFFFu;
        cnt_le_s = 0u;
        gcount_s = 0u;
        fcnt_s = 0xFFFFFFFFu;
    }
    for (int b = threadIdx.x; b < 2048; b += blockDim.x)
        hist11[b] = 0u;
    __syncthreads();
    atomicMax(&max_s, mx);
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        atomicAdd(&hist11[(sv[i] & 0x7FFFFFFFu) >> 20], 1u);
    __syncthreads();
    {  // block scan of the bins (thread t: bins 8t .. 8t+7) to the bin holding rank j
        unsigned c8[8], tot = 0u;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            c8[b] = hist11[8 * threadIdx.x + b];
            tot += c8[b];
        }
        const int ln = threadIdx.x & 31, wp = threadIdx.x >> 5;
        unsigned inc = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned t = __shfl_up_sync(0xffffffffu, inc, o);
            if (ln >= o)
                inc += t;
        }
        if (ln == 31)
            wsum[wp] = inc;
        __syncthreads();
        for (int k = 0; k < wp; ++k)
            inc += wsum[k];
        const unsigned excl = inc - tot, r = (unsigned)j;
        if (r >= excl && r < inc) {  // exactly one thread
            unsigned rr = r - excl;
            int b = 0;
            for (; b < 7; ++b) {
                if (rr < c8[b])
                    break;
                rr -= c8[b];
            }
            fbin_s = 8u * threadIdx.x + (unsigned)b;
            frank_s = rr;
            fcnt_s = c8[b];
        }
    }
    __syncthreads();
    const bool fast = fcnt_s <= 256u;  // the same for every thread
    if (fast) {
        const uint32_t B = fbin_s;
        uint32_t nx = 0xFFFFFFFFu;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t v = sv[i] & 0x7FFFFFFFu;
            if ((v >> 20) == B)
                cand[atomicAdd(&gcount_s, 1u)] = v;
            else if ((v >> 20) > B)
                nx = min(nx, v);
        }
        atomicMin(&next_s, nx);
        __syncthreads();
        const unsigned cn = fcnt_s, rr = frank_s;
        if (threadIdx.x < cn) {  // rank by counting: v sits at ranks [less, less + eq) of bin B
            const uint32_t e = cand[threadIdx.x];
            unsigned less = 0u, eq = 0u;
            for (unsigned u = 0; u < cn; ++u) {
                const uint32_t o = cand[u];
                less += o < e ? 1u : 0u;
                eq += o == e ? 1u : 0u;
            }
            if (less <= rr && rr < less + eq)
                vj_s = e;
            if (rr + 1 < cn && less <= rr + 1 && rr + 1 < less + eq)
                vj1_s = e;
        }
        if (threadIdx.x == 0 && rr + 1 >= cn)
            vj1_s = next_s;  // v_(j+1) is the smallest value of a higher bin
        __syncthreads();
    }
    // radix select of v_(j), one byte per pass from the top (bins denser than 256 values)
    for (int pass = 3; pass >= 0 && !fast; --pass) {
        const int sh = 8 * pass;
        const uint32_t hi_mask = pass == 3 ? 0u : 0xFFFFFFFFu << (sh + 8);
        for (int b = threadIdx.x; b < 256; b += blockDim.x)
            hist[b] = 0u;
        __syncthreads();
        const uint32_t prefix = sel_s;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t v = sv[i] & 0x7FFFFFFFu;
            if ((v & hi_mask) == prefix) {
                // one shared atomic per distinct byte in the warp (the top bytes of a row's |w|
                // are nearly all equal: per-lane atomics would serialise)
                const uint32_t key = (v >> sh) & 0xFFu;
                const unsigned peers = __match_any_sync(__activemask(), key);
                if ((threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1))
                    atomicAdd(&hist[key], (unsigned)__popc(peers));
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {  // the bucket holding rank_s among the matching values: a warp scan
            const int ln = threadIdx.x;
            unsigned c[8], tot = 0u;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                c[b] = hist[8 * ln + b];
                tot += c[b];
            }
            unsigned inc = tot;  // inclusive prefix of the lanes' bin totals
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned t = __shfl_up_sync(0xffffffffu, inc, o);
                if (ln >= o)
                    inc += t;
            }
            const uint32_t r = rank_s;
            const unsigned excl = inc - tot;
            __syncwarp();
            if (r >= excl && r < inc) {  // exactly one lane: rank_s < the matching count
                uint32_t rr = r - excl;
                int b = 0;
                for (; b < 7; ++b) {
                    if (rr < c[b])
                        break;
                    rr -= c[b];
                }
                sel_s = prefix | ((uint32_t)(8 * ln + b) << sh);
                rank_s = rr;
            }
        }
        __syncthreads();
    }
    if (!fast) {
        // v_(j+1): vj again when more than j + 1 values are <= vj, else the smallest value above it
        const uint32_t vj = sel_s;
        unsigned c = 0u;
        uint32_t nx = 0xFFFFFFFFu;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t v = sv[i] & 0x7FFFFFFFu;
            c += v <= vj ? 1u : 0u;
            if (v > vj)
                nx = min(nx, v);
        }
        atomicAdd(&cnt_le_s, c);
        atomicMin(&next_s, nx);
        __syncthreads();
        if (threadIdx.x == 0) {
            vj_s = vj;
            vj1_s = cnt_le_s > (unsigned)(j + 1) ? vj : next_s;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t vj = vj_s;
        float r;
        if (!interior) {
            r = __uint_as_float(vj);  // the largest value
        } else {
            const uint32_t vj1 = vj1_s;
            const float t = __fsub_rn(h, floorf(h));
            const float a = __uint_as_float(vj), b = __uint_as_float(vj1);
            const float d = __fsub_rn(b, a);
            r = t < 0.5f ? __fadd_rn(a, __fmul_rn(d, t)) : __fsub_rn(b, __fmul_rn(d, __fsub_rn(1.0f, t)));
        }
        if (r == 0.0f)
            r = __uint_as_float(max_s);  // max |w|
        float sc = __fdiv_rn(r, 127.0f);
        if (sc == 0.0f)
            sc = 1.0f;
        row_clip_s = r;
        scale_s = sc;
        scale[blockIdx.x] = sc;
    }
    __syncthreads();
    const float rc = row_clip_s, sc = scale_s;
    const float rsc = __frcp_rn(sc);
    const bool mul_ok = rcp_ok(sc);
    for (int c = threadIdx.x; c < n; c += blockDim.x) {  // the row from shared memory
        const float v = fminf(fmaxf(__uint_as_float(sv[c]), -rc), rc);
        q[(int64_t)blockIdx.x * C + c] = (int8_t)sym_code(v, sc, rsc, mul_ok);
    }
}

// ---------------------------------------------------------------- per-group int8 (pergroup_linear's format)
// One warp per (row n, group): the int8 rule per group of g inputs -- scale = max |w| / 127 (zero
// -> 1), q = clip(round(w / scale), -128, 127), IEEE divisions -- with the scales stored
// group-major, scale_w[grp * N + n] [cider/ops.py pergroup_linear, Args].
template <typename TW, int G>
__global__ void __launch_bounds__(256) quantize_int8_groups_kernel(const TW* __restrict__ w, int64_t N, int64_t K,
                                                                  int8_t* __restrict__ q, float* __restrict__ scale_w)
{
    constexpr int PER = G / 32;
    const int64_t item = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int64_t ng = K / G;
    if (item >= N * ng)
        return;
    const int lane = threadIdx.x & 31;
    const int64_t n = item / ng, grp = item % ng;
    const TW* src = w + n * K + grp * G;
    float v[PER];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        v[i] = to_float(src[i * 32 + lane]);
        amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float sc = __fdiv_rn(amax, 127.0f);
    if (sc == 0.f)
        sc = 1.f;
    const float rsc = __frcp_rn(sc);
    const bool fast = rcp_ok(sc);
#pragma unroll
    for (int i = 0; i < PER; ++i)
        q[n * K + grp * G + i * 32 + lane] = (int8_t)sym_code(v[i], sc, rsc, fast);
    if (lane == 0)
        scale_w[grp * N + n] = sc;
}

// The same with G/16 lanes per group, 16 consecutive values each (16-byte loads, one 16-byte store
// of the lane's int8 codes); 16-byte aligned w and q.
template <typename TW, int G>
__global__ void __launch_bounds__(256) quantize_int8_groups_vec_kernel(const TW* __restrict__ w, int64_t N, int64_t K,
                                                                      int8_t* __restrict__ q,
                                                                      float* __restrict__ scale_w)
{
    constexpr int LPG = G / 16;
    const int64_t ng = K / G, groups = N * ng;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t gi = t / LPG;
    const int sub = (int)(t % LPG);
    // lanes past the last group take part in the butterfly on the last group and store nothing
    const bool ok = gi < groups;
    const int64_t gq = ok ? gi : groups - 1;
    float v[16];
    load16(w + gq * G + 16 * sub, v);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
        amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float sc = __fdiv_rn(amax, 127.0f);
    if (sc == 0.f)
        sc = 1.f;
    const float rsc = __frcp_rn(sc);
    const bool fast = rcp_ok(sc);
    int c[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        c[i] = sym_code(v[i], sc, rsc, fast);
    const uint32_t word[4] = {pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]),
                              pack4(c[8], c[9], c[10], c[11]), pack4(c[12], c[13], c[14], c[15])};
    if (ok) {
        *reinterpret_cast<uint4*>(q + gi * G + 16 * sub) = make_uint4(word[0], word[1], word[2], word[3]);
        if (sub == 0)
            scale_w[(gi % ng) * N + gi / ng] = sc;
    }
}

template <typename TW>
__global__ void __launch_bounds__(256) pack_int4_cols_kernel(const TW* __restrict__ w, int64_t K, int64_t N,
                                                             uint8_t* __restrict__ packed, float* __restrict__ scale)
{
    __shared__ float red[8][32];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int64_t n = (int64_t)blockIdx.x * 32 + tx;
    float amax = 0.0f;
    if (n < N)
        for (int64_t k = ty; k < K; k += 8)
            amax = fmaxf(amax, fabsf(load_elem(w, k * N + n)));
    red[ty][tx] = amax;
    __syncthreads();
    amax = red[0][tx];
#pragma unroll
    for (int i = 1; i < 8; ++i)
        amax = fmaxf(amax, red[i][tx]);
    float s = __fdiv_rn(amax, 7.0f);
    if (s == 0.0f)
        s = 1.0f;
    if (n >= N)
        return;
    if (ty == 0)
        scale[n] = s;
    const float rs = __frcp_rn(s);
    const bool fast = rcp_ok(s);
    for (int64_t i = ty; i < K / 2; i += 8) {
        uint32_t c[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float t = __fadd_rn(rint_div(load_elem(w, (2 * i + h) * N + n), s, rs, fast), 8.0f);
            t = fminf(fmaxf(t, 0.0f), 15.0f);
            c[h] = static_cast<uint32_t>(t);
        }
        packed[i * N + n] = static_cast<uint8_t>((c[0] << 4) | c[1]);
    }
}

template <typename TW, typename TP, int BITS>
cudaError_t quantize_dispatch_g(const TW* w, int64_t N, int64_t K, int g, uint32_t* codes, TP* s, TP* b,
                                cudaStream_t st)
{
    const int64_t groups = N * (K / g);
    const unsigned blocks = (unsigned)((groups + 7) / 8);
    // power-of-two widths never straddle a word: lanes share whole words
    constexpr bool pow2 = (BITS & (BITS - 1)) == 0;
    if constexpr (BITS == 2 || BITS == 4 || BITS == 8) {
        if ((reinterpret_cast<uintptr_t>(w) & 15u) == 0) {  // groups start 16-byte aligned (g >= 32)
            const int64_t threads = groups * (g / 16);
            const unsigned vb = (unsigned)((threads + 255) / 256);
            switch (g) {
            case 32: affine_quantize_vec_kernel<TW, TP, BITS, 32><<<vb, 256, 0, st>>>(w, groups, codes, s, b); break;
            case 64: affine_quantize_vec_kernel<TW, TP, BITS, 64><<<vb, 256, 0, st>>>(w, groups, codes, s, b); break;
            default: affine_quantize_vec_kernel<TW, TP, BITS, 128><<<vb, 256, 0, st>>>(w, groups, codes, s, b); break;
            }
            return cudaGetLastError();
        }
    }
    switch (g) {
    case 32:
        if constexpr (pow2)
            affine_quantize_kernel<TW, TP, BITS, 32><<<blocks, 256, 0, st>>>(w, N, K, codes, s, b);
        else
            affine_quantize_odd_kernel<TW, TP, BITS, 32><<<blocks, 256, 0, st>>>(w, N, K, codes, s, b);
        break;
    case 64:
        if constexpr (pow2)
            affine_quantize_kernel<TW, TP, BITS, 64><<<blocks, 256, 0, st>>>(w, N, K, codes, s, b);
        else
            affine_quantize_odd_kernel<TW, TP, BITS, 64><<<blocks, 256, 0, st>>>(w, N, K, codes, s, b);
        break;
    default:
        if constexpr (pow2)
            affine_quantize_kernel<TW, TP, BITS, 128><<<blocks, 256, 0, st>>>(w, N, K, codes, s, b);
        else
            affine_quantize_odd_kernel<TW, TP, BITS, 128><<<blocks, 256, 0, st>>>(w, N, K, codes, s, b);
        break;
    }
    return cudaGetLastError();
}

template <typename TW, typename TP>
cudaError_t quantize_dispatch_b(const void* w, int64_t N, int64_t K, int bits, int g, uint32_t* codes, void* s,
                                void* b, cudaStream_t st)
{
    const TW* wp = static_cast<const TW*>(w);
    TP* sp = static_cast<TP*>(s);
    TP* bp = static_cast<TP*>(b);
    switch (bits) {
    case 1: return quantize_dispatch_g<TW, TP, 1>(wp, N, K, g, codes, sp, bp, st);
    case 2: return quantize_dispatch_g<TW, TP, 2>(wp, N, K, g, codes, sp, bp, st);
    case 3: return quantize_dispatch_g<TW, TP, 3>(wp, N, K, g, codes, sp, bp, st);
    case 4: return quantize_dispatch_g<TW, TP, 4>(wp, N, K, g, codes, sp, bp, st);
    case 5: return quantize_dispatch_g<TW, TP, 5>(wp, N, K, g, codes, sp, bp, st);
    case 6: return quantize_dispatch_g<TW, TP, 6>(wp, N, K, g, codes, sp, bp, st);
    default: return quantize_dispatch_g<TW, TP, 8>(wp, N, K, g, codes, sp, bp, st);
    }
}

template <typename TW>
cudaError_t quantize_dispatch_p(const void* w, int64_t N, int64_t K, int bits, int g, uint32_t* codes, void* s,
                                void* b, qlin_dtype p_dt, cudaStream_t st)
{
    switch (p_dt) {
    case QLIN_F32: return quantize_dispatch_b<TW, float>(w, N, K, bits, g, codes, s, b, st);
    case QLIN_BF16: return quantize_dispatch_b<TW, __nv_bfloat16>(w, N, K, bits, g, codes, s, b, st);
    default: return quantize_dispatch_b<TW, __half>(w, N, K, bits, g, codes, s, b, st);
    }
}

template <typename TP, typename TO>
cudaError_t dequantize_dispatch(const uint32_t* codes, const void* s, const void* b, int64_t N, int64_t K, int bits,
                                int g, void* out, cudaStream_t st, const DeviceInfo& dev)
{
    const int64_t cap = (int64_t)dev.sm_count * 16;
    const int64_t words = N * K * bits / 32;
    const int64_t want = (bits & (bits - 1)) == 0 ? (words + 255) / 256 : (N * (K / 32) + 255) / 256;
    const unsigned blocks = (unsigned)(want < cap ? want : cap);
    const TP* sp = static_cast<const TP*>(s);
    const TP* bp = static_cast<const TP*>(b);
    TO* op = static_cast<TO*>(out);
    auto pow2 = [&](auto bits_c) {
        constexpr int B = decltype(bits_c)::value;
        switch (g) {
        case 32: affine_dequantize_kernel<TP, TO, B, 32><<<blocks, 256, 0, st>>>(codes, sp, bp, words, op); break;
        case 64: affine_dequantize_kernel<TP, TO, B, 64><<<blocks, 256, 0, st>>>(codes, sp, bp, words, op); break;
        default: affine_dequantize_kernel<TP, TO, B, 128><<<blocks, 256, 0, st>>>(codes, sp, bp, words, op); break;
        }
    };
    switch (bits) {
    case 1: affine_dequantize_odd_kernel<TP, TO, 1><<<blocks, 256, 0, st>>>(codes, sp, bp, N, K, g, op); break;
    case 2: pow2(std::integral_constant<int, 2>{}); break;
    case 3: affine_dequantize_odd_kernel<TP, TO, 3><<<blocks, 256, 0, st>>>(codes, sp, bp, N, K, g, op); break;
    case 4: pow2(std::integral_constant<int, 4>{}); break;
    case 5: affine_dequantize_odd_kernel<TP, TO, 5><<<blocks, 256, 0, st>>>(codes, sp, bp, N, K, g, op); break;
    case 6: affine_dequantize_odd_kernel<TP, TO, 6><<<blocks, 256, 0, st>>>(codes, sp, bp, N, K, g, op); break;
    default: pow2(std::integral_constant<int, 8>{}); break;
    }
    return cudaGetLastError();
}

template <typename TP>
cudaError_t dequantize_dispatch_o(const uint32_t* codes, const void* s, const void* b, int64_t N, int64_t K,
                                  int bits, int g, void* out, qlin_dtype o_dt, cudaStream_t st, const DeviceInfo& dev)
{
    switch (o_dt) {
    case QLIN_F32: return dequantize_dispatch<TP, float>(codes, s, b, N, K, bits, g, out, st, dev);
    case QLIN_BF16: return dequantize_dispatch<TP, __nv_bfloat16>(codes, s, b, N, K, bits, g, out, st, dev);
    default: return dequantize_dispatch<TP, __half>(codes, s, b, N, K, bits, g, out, st, dev);
    }
}

}  // namespace

cudaError_t launch_affine_quantize(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int bits, int g,
                                   uint32_t* codes, void* scales, void* biases, qlin_dtype p_dt, cudaStream_t st,
                                   const DeviceInfo&)
{
    switch (w_dt) {
    case QLIN_F32: return quantize_dispatch_p<float>(w, N, K, bits, g, codes, scales, biases, p_dt, st);
    case QLIN_BF16: return quantize_dispatch_p<__nv_bfloat16>(w, N, K, bits, g, codes, scales, biases, p_dt, st);
    default: return quantize_dispatch_p<__half>(w, N, K, bits, g, codes, scales, biases, p_dt, st);
    }
}

cudaError_t launch_affine_dequantize(const uint32_t* codes, const void* scales, const void* biases, qlin_dtype p_dt,
                                     int64_t N, int64_t K, int bits, int g, void* out, qlin_dtype o_dt,
                                     cudaStream_t st, const DeviceInfo& dev)
{
    switch (p_dt) {
    case QLIN_F32: return dequantize_dispatch_o<float>(codes, scales, biases, N, K, bits, g, out, o_dt, st, dev);
    case QLIN_BF16:
        return dequantize_dispatch_o<__nv_bfloat16>(codes, scales, biases, N, K, bits, g, out, o_dt, st, dev);
    default: return dequantize_dispatch_o<__half>(codes, scales, biases, N, K, bits, g, out, o_dt, st, dev);
    }
}

// One row per CTA.  With release_dependents (the activation quantiser of an int8 linear) the CTAs
// let the next kernel of the call start its prologue early -- that kernel waits before reading q
// and scale.  With as_dependent the launch is itself a programmatic dependent of the stream's
// previous kernel: its CTAs may be placed while that kernel runs and wait (griddepcontrol.wait)
// before touching memory.  (Behind the decode GEMVs that made the pair of calls slower: 20.3
// against 18.0 us at 16 tokens, K = N = 8192; behind the tcgen05 GEMMs it hides the launch.)
template <typename... KArgs, typename... Args>
static cudaError_t launch_rows(void (*kern)(KArgs...), int64_t R, int nt, cudaStream_t st, bool pdl, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)R, 1, 1);
    cfg.blockDim = dim3((unsigned)nt, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

static cudaError_t launch_quantize_int8_rows_as(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, int8_t* q,
                                         float* scale, cudaStream_t st, const DeviceInfo& dev, bool release_dependents,
                                         bool as_dependent)
{
    const int rel = release_dependents ? 1 : 0;
    const bool pdl = as_dependent;
    const bool vec = w_dt == QLIN_BF16 && C % 8 == 0 && (reinterpret_cast<uintptr_t>(w) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(q) & 7) == 0;
    const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(w);
    const int64_t C8 = C / 8, sms = dev.sm_count;
    if (vec && R <= 2 * sms && C8 <= 1024 * 4) {  // few rows: 1024 threads per row
        if (C8 <= 1024)
            return launch_rows(quantize_int8_rows_bf16_reg_kernel<1024, 1>, R, 1024, st, pdl, wb, C, q, scale, rel);
        if (C8 <= 2048)
            return launch_rows(quantize_int8_rows_bf16_reg_kernel<1024, 2>, R, 1024, st, pdl, wb, C, q, scale, rel);
        return launch_rows(quantize_int8_rows_bf16_reg_kernel<1024, 4>, R, 1024, st, pdl, wb, C, q, scale, rel);
    }
    if (vec && R <= 4 * sms && C8 <= 512 * 8) {
        if (C8 <= 1024)
            return launch_rows(quantize_int8_rows_bf16_reg_kernel<512, 2>, R, 512, st, pdl, wb, C, q, scale, rel);
        if (C8 <= 2048)
            return launch_rows(quantize_int8_rows_bf16_reg_kernel<512, 4>, R, 512, st, pdl, wb, C, q, scale, rel);
        return launch_rows(quantize_int8_rows_bf16_reg_kernel<512, 8>, R, 512, st, pdl, wb, C, q, scale, rel);
    }
    if (vec && C8 <= 256 * 4)
        return launch_rows(quantize_int8_rows_bf16_reg_kernel<256, 4>, R, 256, st, pdl, wb, C, q, scale, rel);
    if (vec && C8 <= 256 * 8)
        return launch_rows(quantize_int8_rows_bf16_reg_kernel<256, 8>, R, 256, st, pdl, wb, C, q, scale, rel);
    if (vec)
        return launch_rows(quantize_int8_rows_bf16x8_kernel, R, 256, st, pdl, wb, C, q, scale, rel);
    if (w_dt == QLIN_BF16)
        return launch_rows(quantize_int8_rows_kernel<__nv_bfloat16>, R, 256, st, pdl, wb, C, q, scale, rel);
    if (w_dt == QLIN_F16)
        return launch_rows(quantize_int8_rows_kernel<__half>, R, 256, st, pdl, static_cast<const __half*>(w), C, q,
                           scale, rel);
    return launch_rows(quantize_int8_rows_kernel<float>, R, 256, st, pdl, static_cast<const float*>(w), C, q, scale,
                       rel);
}

cudaError_t launch_quantize_int8_rows(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, int8_t* q, float* scale,
                                      cudaStream_t st, const DeviceInfo& dev, bool release_dependents)
{
    return launch_quantize_int8_rows_as(w, w_dt, R, C, q, scale, st, dev, release_dependents, false);
}

cudaError_t launch_quantize_int8_rows_dependent(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, int8_t* q,
                                                float* scale, cudaStream_t st, const DeviceInfo& dev)
{
    return launch_quantize_int8_rows_as(w, w_dt, R, C, q, scale, st, dev, true, true);
}

cudaError_t launch_quantize_weight_int8_clip(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, float pct,
                                             int8_t* q, float* scale, cudaStream_t st, const DeviceInfo&)
{
    const size_t smem = (size_t)C * 4;  // the row's |w| bit patterns
    auto run = [&](auto* typed) {
        using TW = std::remove_const_t<std::remove_pointer_t<decltype(typed)>>;
        cudaError_t e = cudaFuncSetAttribute(quantize_weight_int8_clip_kernel<TW>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        quantize_weight_int8_clip_kernel<TW><<<(unsigned)R, 256, smem, st>>>(typed, C, pct, q, scale);
        return cudaGetLastError();
    };
    switch (w_dt) {
    case QLIN_F32: return run(static_cast<const float*>(w));
    case QLIN_BF16: return run(static_cast<const __nv_bfloat16*>(w));
    default: return run(static_cast<const __half*>(w));
    }
}

cudaError_t launch_quantize_int8_groups(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int g, int8_t* q,
                                        float* scale_w, cudaStream_t st, const DeviceInfo&)
{
    const bool vec = ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(q)) & 15u) == 0;
    const unsigned blocks = (unsigned)((N * (K / g) + 7) / 8);
    const unsigned vblocks = (unsigned)((N * (K / g) * (g / 16) + 255) / 256);
#define QLIN_QG(TW, G)                                                                                               \
    do {                                                                                                             \
        if (vec)                                                                                                     \
            quantize_int8_groups_vec_kernel<TW, G>                                                                   \
                <<<vblocks, 256, 0, st>>>(static_cast<const TW*>(w), N, K, q, scale_w);                              \
        else                                                                                                         \
            quantize_int8_groups_kernel<TW, G><<<blocks, 256, 0, st>>>(static_cast<const TW*>(w), N, K, q, scale_w); \
    } while (0)
    if (w_dt == QLIN_BF16) {
        if (g == 64) QLIN_QG(__nv_bfloat16, 64); else if (g == 128) QLIN_QG(__nv_bfloat16, 128); else QLIN_QG(__nv_bfloat16, 256);
    } else if (w_dt == QLIN_F16) {
        if (g == 64) QLIN_QG(__half, 64); else if (g == 128) QLIN_QG(__half, 128); else QLIN_QG(__half, 256);
    } else {
        if (g == 64) QLIN_QG(float, 64); else if (g == 128) QLIN_QG(float, 128); else QLIN_QG(float, 256);
    }
#undef QLIN_QG
    return cudaGetLastError();
}

cudaError_t launch_pack_int4_cols(const void* w, qlin_dtype w_dt, int64_t K, int64_t N, uint8_t* packed, float* scale,
                                  cudaStream_t st, const DeviceInfo&)
{
    const unsigned blocks = (unsigned)((N + 31) / 32);
    if (w_dt == QLIN_BF16)
        pack_int4_cols_kernel<__nv_bfloat16>
            <<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w), K, N, packed, scale);
    else if (w_dt == QLIN_F16)
        pack_int4_cols_kernel<__half><<<blocks, 256, 0, st>>>(static_cast<const __half*>(w), K, N, packed, scale);
    else
        pack_int4_cols_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(w), K, N, packed, scale);
    return cudaGetLastError();
}

}  // namespace qlin
