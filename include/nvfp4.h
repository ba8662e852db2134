/*
 * nvfp4.h -- NVFP4 W4A4 linear layer, C-ABI of libmxfp8.so.
 *
 * The NVFP4 format of the page "Wan2.2 I2V A14B, four-step 720p: native
 * LightX2V FP8 and NVFP4" (section "Conversion and compatibility"): packed
 * E2M1 weights with E4M3 block scales, an FP32 input_global_scale and an
 * FP32 alpha, weights entering the quantizer as BF16.  The page names the
 * fields, not the arithmetic; this library computes (binary32 throughout):
 *
 *   per 16-element block of a row, with the tensor's global scale g:
 *     s = UE4M3(RN(amax * RN(g / 6)))   E4M3 value used unsigned, nearest
 *                                       even, saturating at 448
 *     q = E2M1(RN(x * RN(g / dec(s))))  nearest even, saturating at 6;
 *                                       s = 0 gives q = +-0
 *   dequantized value q * dec(s) / g; the layer computes
 *     Y[m, n] = BF16_RNE(alpha * sum_k (qx dec(sx)) (qw dec(sw)) + F32(bias[n]))
 *   with alpha = 1 / (g_x * g_w) and FP32 accumulation.  The GEMM runs the
 *   block-scaled 4-bit tensor-core kind (tcgen05.mma kind::mxf4nvf4,
 *   16-element UE4M3 scales): the packed codes are its operands as stored
 *   and the scale atoms below are its scale layout; the epilogue applies
 *   alpha and the bias.
 *
 * Global scales live in device memory (one binary32 per tensor), so the
 * whole path runs on the GPU with no host round trip: nvfp4_amax_* measures
 * a tensor and nvfp4_global_scale_from_amax turns its amax into
 * g = RN(448 * 6 / amax), which gives the tensor's largest block the
 * largest scale (g = 1 when amax is 0 or not finite, or the quotient
 * overflows).  For activations the page calibrates input_global_scale
 * offline; any finite g > 0 may be passed.  The GEMM forms alpha from the
 * two global scales itself.
 *
 * Layouts: codes [rows, K/2] bytes, two E2M1 codes per byte, element 2i in
 * the low nibble; scales in the tensor-core layout of mxfp8.h with 16-element
 * blocks: 512-byte atoms of 128 rows x 4 blocks (64 K elements), atom (i, j)
 * at (i * ceil(K/64) + j) * 512, row r / block b inside at (r % 32) * 16 +
 * ((r / 32) % 4) * 4 + b % 4; padding rows and blocks are written as 0.
 * Ownership, streams and errors as in mxfp8.h.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include "mxfp8.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of the scale array for rows x K (K % 16 == 0), 0 on bad arguments. */
size_t nvfp4_scale_bytes(int64_t rows, int64_t K);

/*
 * amax of a tensor of n elements (n % 16 == 0, 16-byte aligned) into the
 * device float *amax (4-byte aligned).  The FP32 variant measures the values
 * after rounding to BF16, as the weight quantizer sees them.
 */
mxfp8_status nvfp4_amax_bf16(const void *X, int64_t n, float *amax, mxfp8_stream_t stream);
mxfp8_status nvfp4_amax_f32(const float *W, int64_t n, float *amax, mxfp8_stream_t stream);

/*
 * Global scale from an amax, both single device floats (4-byte aligned):
 * *global_scale = RN(448 * 6 / *amax) in binary32, or 1 when *amax is 0 or
 * not finite or the quotient overflows.  Null pointer: MXFP8_ERR_ARG.
 */
mxfp8_status nvfp4_global_scale_from_amax(const float *amax, float *global_scale, mxfp8_stream_t stream);

/*
 * Quantize BF16 activations X [M, K] (row stride ldx, ldx % 8 == 0, X 16-byte
 * aligned) with the global scale *global_scale (a device float, finite and
 * > 0, 4-byte aligned): codes [M, K/2] (8-byte aligned), scales
 * nvfp4_scale_bytes(M, K) bytes (4-byte aligned).  K % 16 == 0.
 */
mxfp8_status nvfp4_quantize_bf16(const void *X, int64_t M, int64_t K, int64_t ldx, const float *global_scale,
                                 void *codes, void *scales, mxfp8_stream_t stream);

/* Weights: FP32 W [N, K] rounded to BF16 (nearest even), then as above. */
mxfp8_status nvfp4_quantize_weight_f32(const float *W, int64_t N, int64_t K, const float *global_scale, void *Wq,
                                       void *Wscale, mxfp8_stream_t stream);

/*
 * The GEMM and epilogue on quantized operands: Xq [M, K/2] and Wq [N, K/2]
 * packed codes with their scales (nvfp4_scale_bytes of [M, K] and [N, K]),
 * the global scales the two operands were quantized with (device floats,
 * finite and > 0, 4-byte aligned; the kernel forms alpha = 1 / (g_x g_w) as
 * a binary32 rounding of the FP64 quotient), bias F16 [N] or NULL, Y BF16
 * [M, N] (written).  Requires K % 64 == 0, N % 8 == 0, N > 0, M >= 0, every
 * other pointer 16-byte aligned.
 */
mxfp8_status nvfp4_gemm(const void *Xq, const void *Xscale, int64_t M, int64_t K, const void *Wq,
                        const void *Wscale, int64_t N, const float *x_global_scale, const float *w_global_scale,
                        const void *bias, void *Y, mxfp8_stream_t stream);

/* Workspace bytes nvfp4_linear needs: the activation codes (rounded up to
 * 256 bytes) and their scales. */
size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * The whole layer: nvfp4_quantize_bf16 of X (row stride K) with the
 * activation global scale *x_global_scale into `workspace`, then nvfp4_gemm
 * with the weights' global scale *w_global_scale (both device floats).
 * workspace: >= nvfp4_linear_workspace_bytes(M, K) bytes, 256-byte aligned,
 * overwritten.  Requirements as nvfp4_gemm.
 */
mxfp8_status nvfp4_linear(const void *X, int64_t M, int64_t K, const float *x_global_scale, const void *Wq,
                          const void *Wscale, int64_t N, const float *w_global_scale, const void *bias, void *Y,
                          void *workspace, size_t ws_bytes, mxfp8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
