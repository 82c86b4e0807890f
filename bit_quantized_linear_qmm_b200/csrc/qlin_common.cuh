// qlin_common.cuh -- shared device helpers of the sm_100a kernels (inline PTX
// for mbarriers, tensor-map TMA, tcgen05 and the legacy warp MMA) and the internal launch
// interface between the C ABI (qlin_abi.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "qlin.h"

#define QLIN_DEV __device__ __forceinline__

namespace qlin {

// Bit set in the device status word when a bounded wait gave up.
constexpr unsigned kStatusTimeout = 1u;
// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// ---------------------------------------------------------------- small device utilities

QLIN_DEV unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

QLIN_DEV uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <typename T> QLIN_DEV float to_float(T v);
template <> QLIN_DEV float to_float<float>(float v) { return v; }
template <> QLIN_DEV float to_float<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> QLIN_DEV float to_float<__half>(__half v) { return __half2float(v); }

template <typename T> QLIN_DEV T from_float(float v);
template <> QLIN_DEV float from_float<float>(float v) { return v; }
template <> QLIN_DEV __nv_bfloat16 from_float<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> QLIN_DEV __half from_float<__half>(float v) { return __float2half_rn(v); }

// 16-bit output / bias values of the int8 layers: bf16, or fp16 when f16 is set (the dtype of x)
QLIN_DEV float h16_to_float(uint32_t u, int f16)
{
    return f16 ? __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu))) : __uint_as_float(u << 16);
}
QLIN_DEV uint32_t pack_h16x2(float lo, float hi, int f16)
{
    if (f16) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}
QLIN_DEV unsigned short to_h16(float v, int f16)
{
    return f16 ? __half_as_ushort(__float2half_rn(v)) : __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// ---------------------------------------------------------------- mbarrier

QLIN_DEV void mbar_init(uint64_t* bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

QLIN_DEV void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

QLIN_DEV void mbar_arrive(uint64_t* bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

QLIN_DEV void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

#ifndef QLIN_MBAR_SUSPEND_NS
#define QLIN_MBAR_SUSPEND_NS 1000000u
#endif
// Suspends the thread (up to a hint of 1 ms, or until the phase completes)
// instead of spinning, so waiting warps leave the issue slots to the others.
QLIN_DEV bool mbar_try_wait(uint64_t* bar, unsigned parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(QLIN_MBAR_SUSPEND_NS)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up after
// kWaitLimitNs, sets the timeout bit in *status and returns false.
QLIN_DEV bool mbar_wait_bounded(uint64_t* bar, unsigned parity, unsigned* status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------- 16-byte global loads

// Read-only streaming data that is not kept in L1, and
// data another kernel may have written (cached in L2 only).
QLIN_DEV uint4 ldg_stream_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

QLIN_DEV uint4 ldg_cg_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// ---------------------------------------------------------------- tensor-map TMA (2-D tiles)

// Loads the 2-D box at (c0, c1) of `tmap` (a __grid_constant__ kernel
// parameter) into shared memory, completing as transaction bytes on `bar`.
// c0 * element size must be a multiple of 16 bytes.  Out-of-range elements
// of the box are written as zeros.
QLIN_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* tmap, int c0, int c1, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// L2 prefetch of the same box (a hint; coherent with earlier writes).
QLIN_DEV void tma_prefetch_2d(const CUtensorMap* tmap, int c0, int c1)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

// Byte offset of the 16-byte unit `unit` (0..7) of row `row` inside a box
// written with CU_TENSOR_MAP_SWIZZLE_128B whose rows are 128 bytes (box
// base 1024-byte aligned): units are XOR-permuted by row mod 8.
QLIN_DEV int swz128(int row, int unit) { return row * 128 + ((unit ^ (row & 7)) << 4); }

// ---------------------------------------------------------------- tcgen05 (5th-generation tensor cores, TMEM)

QLIN_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
QLIN_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Whole warp: allocate `ncols` TMEM columns (power of two >= 32); the base
// address is written to *dst (shared memory).
QLIN_DEV void tmem_alloc(uint32_t* dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

QLIN_DEV void tmem_dealloc(uint32_t base, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, one elected thread.  KIND is
// "f16" (bf16/f16 inputs, f32 accumulate) or "i8" (s8/u8 inputs, s32).
template <bool I8>
QLIN_DEV void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate)
{
    if constexpr (I8)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
            : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
QLIN_DEV void tc_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 16 consecutive 32-bit TMEM columns -> 16 registers per thread.
QLIN_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// The same load without the wait: several loads may be in flight before one tmem_wait_ld().
QLIN_DEV void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
QLIN_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand tile written with the
// 128-byte swizzle (rows of 128 bytes, 8-row groups 1024 bytes apart).
QLIN_DEV uint64_t umma_desc_sw128(uint32_t smem_addr)
{
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Shared-memory matrix descriptor of an MN-major operand tile written with the
// 128-byte swizzle: each K row holds 128 consecutive M / N bytes, 8-row groups
// are 1024 bytes apart (SBO) and successive 128-byte M / N atoms lbo bytes
// apart (LBO).
QLIN_DEV uint64_t umma_desc_sw128_mn(uint32_t smem_addr, uint32_t lbo)
{
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Make this thread's generic-proxy shared-memory writes visible to the
// async proxy (TMA, tensor cores).
QLIN_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- programmatic dependent launch

QLIN_DEV void pdl_wait_prior_grids()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

QLIN_DEV void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- warp MMA (m16n8k16 bf16, m16n8k32 s8)

QLIN_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

QLIN_DEV void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

QLIN_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

QLIN_DEV uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv)
{
    // (a & mask) | orv
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));
    return r;
}

}  // namespace qlin

// ---------------------------------------------------------------- internal launch interface
// Each launcher validates nothing (qlin_abi.cu did) and returns the launch status.
namespace qlin {

struct DeviceInfo {
    int sm_count;
    unsigned* status;  // device status word
};

// The current device's DeviceInfo after a one-time check that it is an sm_100
// part (QLIN_ERR_DEVICE otherwise); defined in qlin_abi.cu.
qlin_status current_device(DeviceInfo& out);

// Host: encodes a 2-D tiled tensor map (row-major [dim1][dim0] elements,
// row pitch `pitch_bytes`) with box {box0, box1}, 128-byte swizzle, zero
// fill (or the given swizzle).  Returns false if the driver entry point is unavailable or rejects
// the description.
bool encode_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t dim0, uint64_t dim1,
                    uint64_t pitch_bytes, uint32_t box0, uint32_t box1,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

cudaError_t launch_affine_quantize(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int bits, int g,
                                   uint32_t* codes, void* scales, void* biases, qlin_dtype p_dt,
                                   cudaStream_t st, const DeviceInfo& dev);
cudaError_t launch_affine_dequantize(const uint32_t* codes, const void* scales, const void* biases,
                                     qlin_dtype p_dt, int64_t N, int64_t K, int bits, int g, void* out,
                                     qlin_dtype o_dt, cudaStream_t st, const DeviceInfo& dev);
cudaError_t launch_quantize_int8_rows(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, int8_t* q,
                                      float* scale, cudaStream_t st, const DeviceInfo& dev, bool release_dependents = false);
cudaError_t launch_quantize_weight_int8_clip(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, float pct,
                                             int8_t* q, float* scale, cudaStream_t st, const DeviceInfo& dev);
cudaError_t launch_quantize_int8_groups(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int g, int8_t* q,
                                        float* scale_w, cudaStream_t st, const DeviceInfo& dev);
cudaError_t launch_pack_int4_cols(const void* w, qlin_dtype w_dt, int64_t K, int64_t N, uint8_t* packed,
                                  float* scale, cudaStream_t st, const DeviceInfo& dev);

struct AffineGemvArgs {
    const void* x;
    qlin_dtype x_dt;
    int64_t M, K, N;
    const uint32_t* codes;
    const void* scales;
    const void* biases;
    qlin_dtype p_dt;
    int bits, g;
    const void* bias;
    void* y;
    // per-group INT8 at one token (pergroup_linear's FP-activation branch): codes are the int8
    // weights [N][K], scales the fp32 [K/g][N] group-major scale_w, no biases; only
    // launch_affine_dec takes it
    int pergroup = 0;
};
cudaError_t launch_affine_gemv(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev);
// all codes in shared memory, one CTA per SM (k_affine_dec.cu); cudaErrorNotSupported for
// layers outside it (x not bf16, codes too large for shared memory, ...), launching nothing
cudaError_t launch_affine_dec(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev);
// any width 1..6, 8 and any dtypes (k_affine_any.cu); 4-byte aligned codes, 16-byte aligned x rows
cudaError_t launch_affine_gemv_any(const AffineGemvArgs& a, cudaStream_t st, const DeviceInfo& dev);

// int8 decode GEMV (M <= 16): y = (float)(qx . w) * s_x[m] * s_w[n] + bias[n], bf16 out
struct W8GemvArgs {
    const int8_t* qx;  // [M][K]
    const float* s_x;  // [M]
    const int8_t* w;   // [N][K] int8 (W8), or packed [K/2][N] bytes (W4)
    const float* s_w;  // [N]
    const void* bias;  // [N] or NULL, bf16 (fp16 when out_f16)
    void* y;           // [M][N], bf16 (fp16 when out_f16)
    int64_t M, K, N;
    int out_f16;
};
cudaError_t launch_w8_gemv(const W8GemvArgs& a, cudaStream_t st, const DeviceInfo& dev);
// int4 decode GEMV (M <= 16): the same arguments, w = packed [K/2][N] bytes
cudaError_t launch_w4_gemv(const W8GemvArgs& a, cudaStream_t st, const DeviceInfo& dev);

struct BitlinearArgs {
    const void* x;
    qlin_dtype x_dt;
    int64_t M, K, N;
    const uint8_t* packed;
    const float* weight_scale;
    int invert;
    const void* bias;
    void* y;
};
cudaError_t launch_bitlinear_gemv(const BitlinearArgs& a, cudaStream_t st, const DeviceInfo& dev);
// BitLinear with M > 16 on the tcgen05 GEMM (k_tc_affine.cu; bf16 x, bf16 weights exact)
cudaError_t launch_tc_bitlinear(const BitlinearArgs& a, cudaStream_t st, const DeviceInfo& dev);

}  // namespace qlin

namespace qlin {

// tcgen05 GEMM launches: int8 (k_tc_gemm.cu) and affine 4-bit (k_tc_affine.cu).
// A is [M][K] row-major (int8, or bf16 x for the affine GEMM), the output [M][N]
// row-major.
struct TcGemmArgs {
    int64_t M, N, K;
    const void* a;            // int8 (qx / raw a) or bf16 (x)
    const void* b;            // int8 w [N][K], packed int4 [K/2][N] or affine codes [N][K*bits/32]
    void* out;                // int32 or bf16 [M][N]
    const float* s_x;         // [M] (W8A8 / W4A8)
    const float* s_w;         // [N] (W8A8 / W4A8)
    const void* bias;         // bf16 [N] or null
    const void* scales;       // affine: bf16 [N][K/g]
    const void* biases;
    int g;
    int bits;                 // affine code width (8 with pergroup)
    int x_dt;                 // affine / per-group: dtype of x, bias and y (a qlin_dtype)
    int pergroup;             // per-group int8 weights [N][K], fp32 scales [K/g][N] (group-major), no biases
    void* workspace;          // affine prefill: tc_affine_workspace() bytes, 256-byte aligned
};
enum TcOp { TC_I8_RAW = 0, TC_W8A8 = 1, TC_W4A8 = 2 };
cudaError_t launch_tc_gemm(TcOp op, const TcGemmArgs& a, cudaStream_t st, const DeviceInfo& dev);
// affine 4-bit prefill with the dequantised weights as the TMEM A operand (k_tc_affine.cu):
// x bf16 [M][K], codes [N][K/2], bf16 scales / biases [N][K/g], out bf16 [M][N].
cudaError_t launch_tc_affine(const TcGemmArgs& a, cudaStream_t st, const DeviceInfo& dev);
// bytes of workspace launch_tc_affine needs (fp16 x and group parameters, token and row scales)
size_t tc_affine_workspace(int64_t M, int64_t N, int64_t K, int g);

}  // namespace qlin
