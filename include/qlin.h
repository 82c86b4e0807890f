/*
 * qlin.h -- C ABI of libqlin.so: quantized linear layers on an NVIDIA B200
 * (sm_100a), computed straight from packed low-bit weights.
 *
 *     y = x * dequant(Wq)^T + bias
 *
 * Formats (cited by page title and section):
 *   - MLX affine groups [docs.rs nuvec-nn 0.1.0 "Struct QuantizedLinear",
 *     fields weight / scales / biases / group_size / bits; cider/ops.py
 *     pergroup_linear docstring, quantize/dequantize formulas]:
 *     codes uint32 [N, K*bits/32], element k of a row in bits
 *     bits*(k mod 32/bits) of word k*bits/32 (LSB first); one scale and one
 *     bias per group of group_size inputs, [N, K/group_size];
 *     w = q*scale + bias.
 *   - BitLinear ternary [mlx_lm/models/bitlinear_layers.py,
 *     make_bitlinear_kernel and class BitLinear]: uint8 [N/4, K]; bits 2j..2j+1
 *     of byte [r, k] hold the code of output row r + j*N/4; w = code - 1; one
 *     tensor scale, multiplied in, or its reciprocal multiplied in.
 *   - per-row symmetric INT8 [cider/ops.py quantize_weight_int8,
 *     perchannel_linear]: int8 [N, K] + fp32 scale [N].
 *   - per-column INT4 [cider/ops.py pack_weight_int4, w4a8_linear]: uint8
 *     [K/2, N], high nibble = even k, low nibble = odd k, w = (code - 8) *
 *     scale[n].
 *
 * Conventions for every entry point:
 *   - Tensors are caller-owned DEVICE pointers, row-major and contiguous.
 *     The library never allocates device memory: scratch, where an operation
 *     needs it, comes from the caller's `workspace` (size from
 *     qlin_workspace_size()).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise, except qlin_get_device_status().
 *   - Ordering on a stream: the GEMV / GEMM kernels of qlin_matmul,
 *     bitlinear_matmul and qlin_int8_matmul_int32, and the second kernel of
 *     w8a8_linear, w8a8_linear_noalloc, w4a8_linear, pergroup_linear and of
 *     qlin_matmul's prefill path (after its preparation kernel), use programmatic
 *     dependent launch: each releases the next kernel of the stream as soon
 *     as it starts, so in an unbroken run of such calls several kernels can
 *     be resident at once.  Each fetches its layer constants -- packed
 *     weights and group scales / biases -- BEFORE waiting for its
 *     predecessors (x, the BitLinear weight scale, the layer bias and y only
 *     after the wait, by which time every earlier kernel of the stream has
 *     completed).  Rule: the packed weights and group parameters of a call
 *     must not be written by ANY earlier call of the same run.  A run ends at
 *     every other operation on the stream -- a quantize, dequantize or pack
 *     call, the activation quantiser that opens a w8a8 / w4a8 call of at
 *     most 16 tokens, the preparation kernel that opens a qlin_matmul
 *     prefill, a copy, an event wait, another library's kernel -- because
 *     such an operation starts only after everything before it has
 *     completed.  The activation quantiser of a w8a8 / w4a8 call of more
 *     than 16 tokens is itself a programmatic dependent: it waits for its
 *     predecessors before it reads x or writes anything, but it does not
 *     end the run.  (The activation quantiser and the preparation kernel let
 *     the second kernel of their own call start early: it fetches the call's
 *     weights meanwhile and reads the quantiser's or preparation's output
 *     only after its wait.)
 *   - Every call validates its arguments before launching anything and
 *     returns a qlin_status; nothing is launched when it is not QLIN_OK.
 *     No C++ exception crosses this interface.
 *   - The device is the CUDA device current on the calling thread; it must
 *     be an sm_100 GPU (QLIN_ERR_DEVICE otherwise).
 *   - Pointers that the kernels stream with bulk copies (codes, packed
 *     weights, x, int8 weights) must be 16-byte aligned and their row pitch a
 *     multiple of 16 bytes; otherwise QLIN_ERR_MISALIGNED.
 *   - Floating-point results use fp32 accumulation; integer codes and int32
 *     accumulations are exact.
 */
#ifndef QLIN_H_
#define QLIN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QLIN_OK = 0,
    QLIN_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, shape rule broken */
    QLIN_ERR_UNSUPPORTED = 2,  /* bits / group_size / dtype combination not provided */
    QLIN_ERR_MISALIGNED = 3,   /* a pointer or row pitch breaks the 16-byte rule */
    QLIN_ERR_DEVICE = 4,       /* no CUDA device, or not sm_100 */
    QLIN_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    QLIN_ERR_TIMEOUT = 6,      /* a bounded on-device wait gave up (see qlin_get_device_status) */
    QLIN_ERR_WORKSPACE = 7     /* workspace missing or smaller than qlin_workspace_size() */
} qlin_status;

typedef enum {
    QLIN_F32 = 0,
    QLIN_BF16 = 1,
    QLIN_F16 = 2               /* IEEE binary16 */
} qlin_dtype;

typedef enum {
    QLIN_OP_MATMUL = 0,     /* qlin_matmul */
    QLIN_OP_BITLINEAR = 1,  /* bitlinear_matmul */
    QLIN_OP_W8A8 = 2,       /* w8a8_linear */
    QLIN_OP_W4A8 = 3,       /* w4a8_linear */
    QLIN_OP_PERGROUP = 4    /* pergroup_linear */
} qlin_op;

/* Human-readable name of a status code (static storage, never NULL). */
const char* qlin_status_string(qlin_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int qlin_version(void);

/*
 * Bytes of device workspace `op` needs for the given sizes (0 = none).
 * bits / group_size matter only for QLIN_OP_MATMUL and may be 0 otherwise.
 */
size_t qlin_workspace_size(qlin_op op, int64_t M, int64_t N, int64_t K, int bits, int group_size);

/*
 * The CTA tile the int8 tensor-core GEMM takes for an M x N output on a GPU
 * of sm_count SMs: *tokens = 128 or 256 rows, *columns = 256, 128 or 112.
 * This GEMM serves qlin_int8_matmul_int32 and w8a8_linear / w4a8_linear
 * above 16 tokens.  op: QLIN_OP_W8A8 for int8 weights (also the raw int8
 * GEMM), QLIN_OP_W4A8 for packed int4 weights.  With fewer 128 x 256 tiles
 * than SMs, the shape minimises (tile rounds) x (operand rows one SM draws
 * per K step): one SM's intake from L2 bounds these shapes.  A 256-row tile
 * is two 128-token sub-tiles sharing each weight stage.  A pure host
 * function: no device call, any thread.  QLIN_ERR_INVALID_ARG for another
 * op, M < 1, N < 1, sm_count < 1 or a NULL output.
 */
qlin_status qlin_int8_gemm_tile(qlin_op op, int64_t M, int64_t N, int sm_count, int* tokens, int* columns);

/*
 * Affine group quantisation of a dense weight [nuvec-nn QuantizedLinear,
 * from_linear; cider/ops.py pergroup_linear docstring, quantize formula].
 * Per group of `group_size` consecutive inputs of one output row:
 *   scale = (max - min) / (2^bits - 1), bias = min  (fp32; min-max choice),
 *   both rounded to param_dt; a stored scale of 0 becomes 1;
 *   q = clip(round_half_even((w - bias) / scale), 0, 2^bits - 1) from the
 *   STORED scale and bias, fp32 subtract and IEEE divide.
 * w: [N, K] of w_dt.  codes: uint32 [N, K*bits/32]; a row is one
 * LSB-first bitstream, code k at bits k*bits .. k*bits+bits-1 of the row
 * read as a little-endian sequence of 32-bit words, so for 3, 5 and 6 bits a
 * code may continue in the next word (a group of group_size codes is always
 * whole words).  scales, biases: [N, K/group_size] of param_dt.  bits in
 * {1, 2, 3, 4, 5, 6, 8}; group_size in {32, 64, 128}; K % group_size == 0;
 * every dtype (fp32, bf16, fp16) for w and the parameters.  Bit-exact with
 * the CPU reference.
 */
qlin_status qlin_quantize(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int bits,
                          int group_size, uint32_t* codes, void* scales, void* biases,
                          qlin_dtype param_dt, void* stream);

/*
 * Dequantised weight [nuvec-nn QuantizedLinear, dequantized_weight; cider
 * pergroup_linear docstring, dequantize formula]: w_out[n, k] =
 * fma(q, scale, bias) in fp32, rounded once to out_dt.  w_out: [N, K],
 * 16-byte aligned; codes 4-byte aligned.  Widths and dtypes as
 * qlin_quantize.  Bit-exact with the CPU reference.
 */
qlin_status qlin_dequantize(const uint32_t* codes, const void* scales, const void* biases,
                            qlin_dtype param_dt, int64_t N, int64_t K, int bits, int group_size,
                            void* w_out, qlin_dtype out_dt, void* stream);

/*
 * Quantized linear layer [nuvec-nn QuantizedLinear, forward: x W^T + b
 * computed from the packed weight, its scales and biases].
 * x: [M, K] of x_dt (which is also the dtype of bias and y).  bias: [N] or
 * NULL.  y: [M, N].  M <= 16 runs the decode kernel (bulk-copy streamed
 * codes, register dequantisation, tensor-core MACs, partial sums reduced
 * inside the CTA).  M > 16 with 4-bit codes and bf16 parameters (x bf16 or
 * fp32) runs the prefill GEMM: a preparation kernel writes x and the group
 * parameters as fp16 into `workspace`, each token row and each weight row
 * scaled by a power of two that keeps it in fp16's range (undone exactly in
 * the epilogue), and the GEMM dequantises the codes to fp16(s q + b) in
 * registers, writes them to tensor memory as the A operand of tcgen05 MMA
 * and accumulates in fp32 in tensor memory -- every product within 2^-11 of
 * the exact one.  Other M > 16 calls run the decode kernel on 16-token
 * slices.  The decode kernel and the prefill GEMM take 2-, 4- and 8-bit
 * codes whose rows are 16-byte aligned ((K*bits/8) % 16 == 0, codes 16-byte
 * aligned), fp32 or bf16 x and parameters (the prefill also fp16 x), and not
 * 2 bits in groups of 32.  Every other call -- widths 1, 3, 5, 6, fp16
 * activations or parameters at M <= 16, rows whose group parameters do not
 * fit the decode kernel's shared memory (long K in small groups) -- runs a
 * general decode kernel (eight codes per lane, fp32 dequantisation exactly
 * as qlin_dequantize, fp32 accumulation; slower).  x: 16-byte aligned;
 * codes: 4-byte aligned (QLIN_ERR_MISALIGNED otherwise).  workspace: at
 * least qlin_workspace_size(QLIN_OP_MATMUL, M, N, K, bits, group_size)
 * bytes, 256-byte aligned (QLIN_ERR_WORKSPACE otherwise) when the call runs
 * the prefill; NULL is accepted when that size is 0 (M <= 16, or bits != 4).
 */
qlin_status qlin_matmul(const void* x, qlin_dtype x_dt, int64_t M, int64_t K,
                        const uint32_t* codes, const void* scales, const void* biases,
                        qlin_dtype param_dt, int64_t N, int bits, int group_size,
                        const void* bias, void* y, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * BitLinear ternary layer [mlx_lm bitlinear_layers.py, make_bitlinear_kernel
 * and BitLinear.__call__]:
 *   y[m, r + j*N/4] = s * sum_k x[m, k] * (((packed[r, k] >> 2j) & 3) - 1) + bias
 * with s = invert_weight_scale ? 1/weight_scale[0] : weight_scale[0] (an fp32
 * reciprocal, then a multiply).  x: [M, K] of x_dt; packed: uint8 [N/4, K];
 * weight_scale: DEVICE pointer to one fp32; bias: [N] of x_dt or NULL (added
 * in fp32 before the single rounding to x_dt); y: [M, N] of x_dt.
 * Requires N % 4 == 0 and K % 16 == 0.
 */
qlin_status bitlinear_matmul(const void* x, qlin_dtype x_dt, int64_t M, int64_t K,
                             const uint8_t* packed, int64_t N, const float* weight_scale,
                             int invert_weight_scale, const void* bias, void* y, void* stream);

/*
 * Per-row symmetric int8 quantisation [cider/ops.py quantize_weight_int8]:
 * scale[r] = max_c |w[r, c]| / 127 (zero -> 1), q = clip(round_half_even(w /
 * scale), -128, 127).  Used for weights (rows = output features) and, with
 * the same rule, for activations (rows = tokens; the pages' quant_a).
 * w: [R, C] of w_dt (fp32, bf16 or fp16); q: int8 [R, C]; scale: fp32 [R].
 * Bit-exact.
 */
qlin_status qlin_quantize_int8_rows(const void* w, qlin_dtype w_dt, int64_t R, int64_t C,
                                    int8_t* q, float* scale, void* stream);

/*
 * Per-column int4 with zero point 8 [cider/ops.py pack_weight_int4]:
 * scale[n] = max_k |w[k, n]| / 7 (zero -> 1), c = clip(round_half_even(w /
 * scale) + 8, 0, 15); packed[i, n] = (c[2i, n] << 4) | c[2i+1, n].
 * w: [K, N] of w_dt (K even); packed: uint8 [K/2, N]; scale: fp32 [N].
 * Bit-exact.
 */
qlin_status qlin_pack_int4_cols(const void* w, qlin_dtype w_dt, int64_t K, int64_t N,
                                uint8_t* packed, float* scale, void* stream);

/*
 * Raw int8 x int8 -> int32 product [cider/ops.py int8_matmul_int32]:
 * c[m, n] = sum_k a[m, k] * b[n, k], exact (callers keep |c| < 2^31).
 * a: int8 [M, K]; b: int8 [N, K]; c: int32 [M, N].  K % 16 == 0.
 */
qlin_status qlin_int8_matmul_int32(const int8_t* a, const int8_t* b, int64_t M, int64_t N,
                                   int64_t K, int32_t* c, void* stream);

/*
 * W8A8 linear [cider/ops.py perchannel_linear]: y = dequant(quant_a(x) @
 * w^T) + bias, quant_a = per-token qlin_quantize_int8_rows of x (kept in the
 * workspace), int32 accumulation, then y = acc * s_x[m] * scale_w[n] + bias
 * in fp32 and one rounding to x_dt.  x: [M, K] of x_dt, bf16 or fp16
 * (QLIN_ERR_UNSUPPORTED for fp32); w: int8 [N, K];
 * scale_w: fp32 [N]; bias: [N] of x_dt or NULL; y: [M, N] of x_dt.
 * K % 16 == 0.  workspace >= qlin_workspace_size(QLIN_OP_W8A8, M, N, K, 0, 0).
 * M <= 16 runs a weight-streaming GEMV (int8 mma.sync), larger M the tcgen05
 * GEMM (int32 accumulation in tensor memory).
 */
qlin_status w8a8_linear(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const int8_t* w,
                        const float* scale_w, int64_t N, const void* bias, void* y,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * W4A8 linear [cider/ops.py w4a8_linear]: y = dequant(quant_a(x) @
 * unpack4(w)), unpack4 reading code c[k, n] from packed[k/2, n] (high
 * nibble for even k) with weight c - 8; int32 accumulation; y = acc *
 * s_x[m] * scale_w[n] (+ bias, an extension: the page has none) rounded to
 * x_dt.  packed: uint8 [K/2, N]; other arguments as w8a8_linear.
 * K % 32 == 0, N % 16 == 0.  M <= 16 runs a weight-streaming GEMV, larger M
 * the tcgen05 GEMM (the nibbles are converted to int8 in shared memory).
 */
qlin_status w4a8_linear(const void* x, qlin_dtype x_dt, int64_t M, int64_t K,
                        const uint8_t* packed_w, const float* scale_w, int64_t N,
                        const void* bias, void* y, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * Per-row symmetric INT8 weight quantisation with an optional percentile clip
 * [cider/ops.py quantize_weight_int8, clip_percentile]: clip_percentile < 0
 * (the page's None) is the absmax rule of qlin_quantize_int8_rows; 0 <= p <=
 * 100 sets clip = the linear-interpolated p-th percentile of |w| over the row
 * (numpy's default percentile method, in float32 as numpy computes it on a
 * float32 row), replaced by max |w| when 0; scale = clip / 127 (zero -> 1);
 * w clipped to [-clip, clip]; q = clip(round_half_even(w / scale), -128, 127).
 * w: [R, C] of w_dt; q: int8 [R, C]; scale: fp32 [R].  The clip path holds a
 * row in shared memory (a histogram of its top bits, then a count or a radix
 * select inside the bin, finds the two order statistics the interpolation
 * needs): C <= 32768 (QLIN_ERR_UNSUPPORTED otherwise);
 * p > 100 or NaN -> QLIN_ERR_INVALID_ARG.  Bit-exact.
 */
qlin_status qlin_quantize_weight_int8(const void* w, qlin_dtype w_dt, int64_t R, int64_t C, double clip_percentile,
                                     int8_t* q, float* scale, void* stream);

/*
 * Per-group symmetric INT8 weight quantisation, the weight format of
 * pergroup_linear [cider/ops.py pergroup_linear, Args: "INT8 weights [N, K]
 * int8 (per-group symmetric quantized)", scales [num_groups, N]]: per group of
 * group_size consecutive inputs of a row, scale = max |w| / 127 (fp32, zero ->
 * 1) and q = clip(round_half_even(w / scale), -128, 127) -- the rule of
 * qlin_quantize_int8_rows per group.  w: [N, K] of w_dt; q: int8 [N, K];
 * scale_w: fp32 [K/group_size, N], group-major (scale_w[g * N + n]).
 * group_size in {64, 128, 256}; K % group_size == 0.  Bit-exact.
 */
qlin_status qlin_quantize_int8_groups(const void* w, qlin_dtype w_dt, int64_t N, int64_t K, int group_size,
                                     int8_t* q, float* scale_w, void* stream);

/*
 * Per-group INT8 linear [cider/ops.py pergroup_linear: Args, and "Dispatches
 * internally: M > 1 -> per-group GEMM (activation quantize + INT8 TensorOps),
 * M == 1 -> per-group MV (FP activation, weight dequant on-the-fly)"]:
 *   M == 1: y[n] = sum_g scale_w[g, n] * sum_{k in g} x[k] * w[n, k] + bias[n]
 *   M > 1:  y[m, n] = s_x[m] * sum_g scale_w[g, n] * sum_{k in g} qx[m, k] * w[n, k] + bias[n],
 *           qx, s_x = the per-token int8 quantisation of x (the qlin_quantize_int8_rows rule)
 * x: [M, K] of x_dt (also the dtype of bias and y); w: int8 [N, K];
 * scale_w: fp32 [K/group_size, N] (group-major); bias: [N] or NULL; y: [M, N].
 * group_size in {64, 128, 256}; K % 16 == 0.  Both branches run the tcgen05
 * GEMM of the affine prefill: a preparation kernel writes x (M == 1, scaled
 * by a power of two) or its int8 quantisation (M > 1) and the group scales as
 * fp16 into `workspace`, and the GEMM forms each weight as fp16(scale w),
 * rounded once (every product within 2^-11 of the exact one).  workspace: at
 * least qlin_workspace_size(QLIN_OP_PERGROUP, M, N, K, 8, group_size) bytes,
 * 256-byte aligned.
 */
qlin_status pergroup_linear(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const int8_t* w,
                            const float* scale_w, int64_t N, int group_size, const void* bias, void* y,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * W8A8 linear without caller memory (no counterpart on the source pages).
 * Same operation, arguments and results as w8a8_linear, for callers that
 * cannot give the library device memory: a host that reserved the GPU's
 * memory for its own pool, a serving loop that allows no allocator calls
 * after start-up, or a C program with nothing to borrow scratch from.  The
 * per-token int8 activations and their scales live in an 8 MiB buffer built
 * into libqlin.so (each GPU that loads the library holds it until exit);
 * the call itself allocates and frees nothing.
 *   - Limit: qlin_workspace_size(QLIN_OP_W8A8, M, N, K, 0, 0) must be at most
 *     8 MiB (M*K rounded up to 256 bytes, plus 4*M rounded up to 256);
 *     larger problems return QLIN_ERR_WORKSPACE and launch nothing.
 *   - The buffer's device address is looked up on the first call made with
 *     a given device current (after the same sm_100 check as every other
 *     call; a lookup that fails is retried on the next call); make that
 *     first call before any stream capture on that device.
 *   - All calls share the one buffer and it keeps the last call's contents
 *     (every call rewrites what it reads, so nothing needs clearing).  Calls
 *     that may run at the same time on the GPU -- on different streams, or
 *     from different host threads -- race on it; serialise them.
 */
qlin_status w8a8_linear_noalloc(const void* x, qlin_dtype x_dt, int64_t M, int64_t K, const int8_t* w,
                                const float* scale_w, int64_t N, const void* bias, void* y, void* stream);

/*
 * Synchronises `stream`, then reports (and clears) the library's device
 * status word: QLIN_ERR_TIMEOUT if a bounded on-device wait in any kernel
 * gave up since the last call, QLIN_ERR_CUDA if the stream holds an error,
 * QLIN_OK otherwise.
 */
qlin_status qlin_get_device_status(void* stream);

/*
 * Self-test of the bounded-wait path: launches one kernel on `stream` that
 * waits on an on-chip barrier nothing completes, gives up after `limit_us`
 * microseconds (1 .. 2,000,000, else QLIN_ERR_INVALID_ARG), sets the timeout
 * bit of the device status word and returns; the next
 * qlin_get_device_status() then reports QLIN_ERR_TIMEOUT, and the library
 * stays usable.  Nothing faults, nothing is left running.
 */
qlin_status qlin_selftest_wait_timeout(unsigned limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QLIN_H_ */
