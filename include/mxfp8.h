/*
 * mxfp8.h -- C-ABI of libmxfp8.so, the B200 (sm_100a) MXFP8 W8A8 linear layer.
 *
 * The layer is the one the quantized Wan2.2 A14B transformer runs for its 400
 * block linears (model card "Wan2.2-I2V-A14B-Lightning . MXFP8 (AutoRound
 * OptRTN)", sections "Quantization Details" and "Coverage per transformer"):
 * weights are FP8 E4M3 codes with one E8M0 scale per 32 consecutive input
 * channels, activations are quantized the same way at run time, and the
 * output adds an F16 bias.
 *
 * Conventions for every entry point
 *  - Shapes: Y[M,N] = X[M,K] . W[N,K]^T (+ bias[N]).  All matrices are
 *    row-major with K contiguous; W is stored out x in, like nn.Linear.
 *  - Memory: every pointer is DEVICE memory owned by the caller, 16-byte
 *    aligned unless stated otherwise.  The library allocates nothing.
 *  - Streams: work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) of the current device and returns without waiting.
 *    Only mxfp8_device_status() synchronizes.
 *  - Errors: every call returns an mxfp8_status and never aborts.  Bad
 *    arguments are rejected before anything is launched.  A launch failure
 *    returns MXFP8_ERR_CUDA.  A kernel whose pipeline wait gave up (a bounded
 *    wait, several seconds) records MXFP8_ERR_TIMEOUT in a device status word
 *    read by mxfp8_device_status().
 *
 * Number formats
 *  - E4M3 code: OCP 8-bit float, 1 sign, 4 exponent bits (bias 7), 3 mantissa
 *    bits, no infinities, 0x7F/0xFF = NaN, largest finite 448.
 *  - E8M0 scale byte b: the power of two 2^(b-127); 0xFF = NaN.
 *  - A 32-element block x gets e = floor(log2(max|x|)) - 8 clamped to
 *    [-127, 127] (e = -127 for an all-zero block), and codes
 *    RNE_satfinite(x / 2^e): nearest, ties to even, magnitudes >= 448
 *    saturate to 448.  A block holding Inf/NaN gets scale 0xFF, codes 0x7F.
 *
 * Scale-factor layouts (mxfp8_sf_layout)
 *  - MXFP8_SF_ROWMAJOR: byte (r, b) at r*(K/32) + b.  For inspection.
 *  - MXFP8_SF_TCGEN05: the layout the tensor cores read.  Rows are padded to
 *    a multiple of 128, 32-blocks to a multiple of 4; the matrix is cut into
 *    512-byte atoms of 128 rows x 4 blocks, stored atom-row-major
 *    (atom (i, j) at ((i * ceil(K/128)) + j) * 512); inside an atom, byte
 *    (r, b) sits at (r % 32) * 16 + (r / 32) * 4 + b.  Padding bytes are 0.
 */
#ifndef MXFP8_H
#define MXFP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *mxfp8_stream_t; /* same type as cudaStream_t */

typedef enum {
    MXFP8_OK = 0,
    MXFP8_ERR_ARG = 1,     /* null pointer, bad layout, negative size */
    MXFP8_ERR_ALIGN = 2,   /* pointer or leading dimension misaligned */
    MXFP8_ERR_SHAPE = 3,   /* K or N not a supported multiple, too large */
    MXFP8_ERR_CUDA = 4,    /* a CUDA runtime call or launch failed */
    MXFP8_ERR_TIMEOUT = 5  /* a kernel's bounded pipeline wait gave up */
} mxfp8_status;

typedef enum {
    MXFP8_SF_ROWMAJOR = 0,
    MXFP8_SF_TCGEN05 = 1
} mxfp8_sf_layout;

/* Elementwise function applied to a layer's BF16 output before it is
 * quantized for the next layer (mxfp8_gemm_quantize_out). */
typedef enum {
    MXFP8_ACT_NONE = 0,
    MXFP8_ACT_GELU_TANH = 1   /* as mxfp8_gelu_tanh_bf16 */
} mxfp8_activation;

/* Human-readable name of a status.  Static storage; never NULL. */
const char *mxfp8_status_str(mxfp8_status s);

/*
 * Bytes of the E8M0 scale array for a [rows, K] operand in `layout`
 * (K % 32 == 0).  ROWMAJOR: rows*K/32.  TCGEN05: ceil(rows/128) *
 * ceil(K/128) * 512.  Returns 0 for invalid arguments.
 */
size_t mxfp8_scale_bytes(int64_t rows, int64_t K, int layout);

/*
 * Dynamic activation quantization (model card, "Coverage per transformer":
 * "activations are dynamically quantized to MXFP8 at runtime";
 * quantization_config.json: act_data_type mx_fp, act_group_size 32,
 * act_sym true, act_dynamic true).
 *
 *   X       BF16 [M, K], row stride ldx elements (ldx >= K, ldx % 8 == 0)
 *   codes   E4M3 [M, K], row stride K (written)
 *   scales  E8M0, mxfp8_scale_bytes(M, K, layout) bytes (written, padding 0)
 * Requires K % 32 == 0, M >= 0 (M == 0 is a no-op).  X 16-byte aligned,
 * codes 8-byte aligned, scales 4-byte aligned.
 */
mxfp8_status mxfp8_quantize(const void *X, int64_t M, int64_t K, int64_t ldx,
                            void *codes, void *scales, int layout,
                            mxfp8_stream_t stream);

/*
 * Offline weight quantization by plain round-to-nearest (the model card's
 * "Weights are stored as FP8 E4M3 with per-32 E8M0 scales"; quantization_config
 * bits 8, data_type mx_fp, group_size 32, sym true).  Same rule as above,
 * applied to FP32 weights directly.
 *
 *   W       FP32 [N, K] (row stride K), 16-byte aligned
 *   Wq      E4M3 [N, K] (written), Wscale E8M0 mxfp8_scale_bytes(N, K, layout)
 */
mxfp8_status mxfp8_quantize_weight_f32(const float *W, int64_t N, int64_t K,
                                       void *Wq, void *Wscale, int layout,
                                       mxfp8_stream_t stream);

/* Workspace bytes mxfp8_linear needs for M rows of K: the activation codes
 * (rounded up to 256 bytes) plus their TCGEN05 scales. */
size_t mxfp8_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * The quantized linear layer: quantize X (as mxfp8_quantize, TCGEN05 layout,
 * into `workspace`), then the block-scaled GEMM with FP32 accumulation and
 * the epilogue Y = BF16_RNE(acc + F32(bias)) (model card, "Performance
 * Profile": "linear (MXFP8 W8A8)"; "Coverage per transformer": F16 biases).
 *
 *   X       BF16 [M, K], row stride K
 *   Wq      E4M3 [N, K]; Wscale E8M0 in MXFP8_SF_TCGEN05 layout for [N, K]
 *   bias    F16 [N] or NULL (no bias)
 *   Y       BF16 [M, N], row stride N (written)
 *   workspace  >= mxfp8_linear_workspace_bytes(M, K) bytes, 256-byte aligned;
 *              overwritten; must not be in use by other work on the GPU.
 * Requires K % 128 == 0, N % 8 == 0, N > 0, M >= 0.
 */
mxfp8_status mxfp8_linear(const void *X, int64_t M, int64_t K,
                          const void *Wq, const void *Wscale, int64_t N,
                          const void *bias, void *Y,
                          void *workspace, size_t ws_bytes,
                          mxfp8_stream_t stream);

/*
 * The GEMM + epilogue alone, on operands already quantized (both scale
 * arrays in MXFP8_SF_TCGEN05 layout).  Xq [M, K] E4M3, Wq [N, K] E4M3,
 * bias F16 [N] or NULL, Y BF16 [M, N].  Same requirements as mxfp8_linear.
 */
mxfp8_status mxfp8_gemm_prequant(const void *Xq, const void *Xscale, int64_t M, int64_t K,
                                 const void *Wq, const void *Wscale, int64_t N,
                                 const void *bias, void *Y, mxfp8_stream_t stream);

/*
 * GELU, tanh form, between ffn.net.0.proj and ffn.net.2 (the pages leave its
 * form open; this is the tanh approximation
 * 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), evaluated in FP32 as
 * x / (1 + exp(-2u)) with the hardware's approximate exp2 and reciprocal
 * (relative error below 2^-16 before rounding), BF16 in and out, rounded to
 * nearest even: within one BF16 ulp of the exact function).
 *   X, Y    BF16 [n] (Y may equal X), 16-byte aligned, n % 8 == 0.
 */
mxfp8_status mxfp8_gelu_tanh_bf16(const void *X, void *Y, int64_t n, mxfp8_stream_t stream);

/*
 * The GEMM with the next linear's activation quantization in its epilogue
 * (the optional fusion of the quantizer into the previous layer's epilogue,
 * e.g. ffn.net.0.proj -> GELU -> ffn.net.2 of the model card's "Coverage per
 * transformer").  The layer's BF16 output is not written; the result is
 * bit-identical to
 *     mxfp8_gemm_prequant(..., Y)
 *     [mxfp8_gelu_tanh_bf16(Y, Y)]               when act == MXFP8_ACT_GELU_TANH
 *     mxfp8_quantize(Y, M, N, N, Yq, Yscale, MXFP8_SF_TCGEN05)
 * which it replaces, saving Y's BF16 write and the two passes over it.
 *
 *   Xq, Xscale, Wq, Wscale, bias   as mxfp8_gemm_prequant
 *   act     MXFP8_ACT_NONE or MXFP8_ACT_GELU_TANH
 *   Yq      E4M3 codes [M, N], row stride N (written), 16-byte aligned
 *   Yscale  E8M0 scales of [M, N] in MXFP8_SF_TCGEN05 layout,
 *           mxfp8_scale_bytes(M, N, MXFP8_SF_TCGEN05) bytes (written,
 *           padding rows included), 16-byte aligned
 * Requires K % 128 == 0 and N % 128 == 0 (the next linear's K), N > 0,
 * M >= 0.  Errors as mxfp8_gemm_prequant; MXFP8_ERR_ARG for an unknown act.
 */
mxfp8_status mxfp8_gemm_quantize_out(const void *Xq, const void *Xscale, int64_t M, int64_t K,
                                     const void *Wq, const void *Wscale, int64_t N,
                                     const void *bias, int act, void *Yq, void *Yscale,
                                     mxfp8_stream_t stream);

/*
 * mxfp8_linear for callers that cannot allocate device memory.  The pages
 * have no counterpart of this entry point; it exists for users of this
 * library.  mxfp8_linear needs a workspace for the quantized activations;
 * some callers cannot provide one -- code running inside another runtime's
 * launch hook where allocation is not allowed, or a process whose memory
 * allocator already holds all of the GPU's memory, so that cudaMalloc (which
 * also synchronizes the device) would fail or stall other streams.  This
 * variant uses a fixed scratch array inside the library instead and
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library call).
 *
 *   Same arguments, requirements and results as mxfp8_linear, minus the
 *   workspace.  The activation codes must fit MXFP8_NOALLOC_MAX_CODE_BYTES
 *   (M * K <= 32 MiB, e.g. M <= 6553 rows at K = 5120) and their scales
 *   MXFP8_NOALLOC_MAX_SCALE_BYTES; larger problems return MXFP8_ERR_SHAPE
 *   before anything is launched.
 *   Memory: the scratch is a 34 MiB device array that every GPU which loads
 *   the library keeps until the process exits.
 *   First call on a device: looks up the scratch's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture.  cudaDeviceReset invalidates the
 *   cached address: after resetting a device, do not call this entry point
 *   on it again in the same process.
 *   Concurrency: all calls on a device share the one scratch array, which
 *   keeps the last call's contents.  Calls whose work overlaps on the GPU
 *   (different streams, or different host threads without ordering) race on
 *   it and give wrong results; order them on one stream.  Nothing in the
 *   scratch needs clearing between calls.
 */
#define MXFP8_NOALLOC_MAX_CODE_BYTES (32ll << 20)
#define MXFP8_NOALLOC_MAX_SCALE_BYTES (2ll << 20)
#define MXFP8_NOALLOC_SCRATCH_BYTES (MXFP8_NOALLOC_MAX_CODE_BYTES + MXFP8_NOALLOC_MAX_SCALE_BYTES)
mxfp8_status mxfp8_linear_noalloc(const void *X, int64_t M, int64_t K,
                                  const void *Wq, const void *Wscale, int64_t N,
                                  const void *bias, void *Y, mxfp8_stream_t stream);

/*
 * Synchronizes `stream`, then reads and clears the library's device status
 * word on the current device.  Returns MXFP8_ERR_TIMEOUT if a kernel gave up
 * a pipeline wait since the last call, MXFP8_ERR_CUDA if the stream reports
 * an error, MXFP8_OK otherwise.
 */
mxfp8_status mxfp8_device_status(mxfp8_stream_t stream);

/* Which kernel family's bounded wait mxfp8_selftest_wait_timeout exercises. */
typedef enum {
    MXFP8_SELFTEST_GEMM = 0,           /* the block-scaled / per-channel FP8 GEMM */
    MXFP8_SELFTEST_NVFP4_GEMM = 1,     /* the NVFP4 GEMM: the same kernel family and wait as 0 */
    MXFP8_SELFTEST_ROWWISE_QUANT = 2   /* the per-channel FP8 activation quantizer */
} mxfp8_selftest;

/*
 * Failure-path self-test: launches one thread that waits, with that kernel
 * family's bounded wait, on an mbarrier that nothing arrives at.  After
 * timeout_ns (1 .. 10^10) the wait gives up and records the timeout in the
 * status word, so the next mxfp8_device_status() returns MXFP8_ERR_TIMEOUT
 * (and clears it) while the context stays usable.  Nothing else is in flight
 * in the test kernel.  Bad `which` or timeout: MXFP8_ERR_ARG.
 */
mxfp8_status mxfp8_selftest_wait_timeout(int which, uint64_t timeout_ns, mxfp8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXFP8_H */
