/*
 * fp8_rowwise.h -- per-channel FP8 W8A8 linear layer, C-ABI of libmxfp8.so.
 *
 * The per-channel FP8 scheme of "Model Quantization Techniques" (LightX2V),
 * section "Quantization Modes" (fp8-vllm / fp8-sgl: FP8 channel-symmetric
 * weights, FP8 channel-dynamic symmetric activations), with the activation
 * rule of section "MiniMax-H3 FP8 with FP16 Accumulation" (dynamic row-wise
 * quantization, scale = max(abs(x)) / qmax) and qmax = 448 for FP32
 * accumulation (section "MiniMax-H3 Video VAE Encoder Conv3D"); the weights
 * carry "per-output-channel FP32 scales" (page "Wan2.2 I2V A14B, four-step
 * 720p: native LightX2V FP8 and NVFP4", section "Conversion and
 * compatibility").
 *
 *   s[r]    = amax_k |X[r, k]| / 448                 (binary32 division)
 *   q[r, k] = E4M3(X[r, k] / s[r])                   (binary32 division, then
 *             round to nearest even, saturating at +-448; s = 0 -> q = +-0)
 *   Y[m, n] = BF16_RNE( sx[m] sw[n] sum_k q_x[m, k] q_w[n, k] + F32(bias[n]) )
 *             (FP32 accumulation)
 *
 * Layouts: row-major, K contiguous; codes E4M3 bytes [rows, K]; scales FP32
 * [rows] (one per token for activations, one per output channel for
 * weights).  Ownership, streams and errors as in mxfp8.h: the caller owns
 * every buffer and the stream, nothing is allocated or synchronized, failures
 * are returned as mxfp8_status before anything is launched.
 */
#ifndef FP8_ROWWISE_H
#define FP8_ROWWISE_H

#include "mxfp8.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Largest K the row-wise quantizers accept. */
#define FP8RW_MAX_K 16384

/*
 * Dynamic per-token quantization of BF16 activations.
 *   X       BF16 [M, K], row stride ldx >= K elements, 16-byte aligned,
 *           ldx * 2 % 16 == 0
 *   codes   E4M3 [M, K] (written), 8-byte aligned
 *   scales  FP32 [M] (written), 4-byte aligned
 * Requires K % 8 == 0, 0 < K <= FP8RW_MAX_K, M >= 0.
 */
mxfp8_status fp8rw_quantize_bf16(const void *X, int64_t M, int64_t K, int64_t ldx, void *codes,
                                 float *scales, mxfp8_stream_t stream);

/*
 * Per-output-channel quantization of FP32 weights W [N, K] (row stride K,
 * 16-byte aligned) -> Wq E4M3 [N, K] (4-byte aligned), Wscale FP32 [N].
 * Requires K % 4 == 0, 0 < K <= FP8RW_MAX_K.
 */
mxfp8_status fp8rw_quantize_weight_f32(const float *W, int64_t N, int64_t K, void *Wq, float *Wscale,
                                       mxfp8_stream_t stream);

/*
 * The GEMM and epilogue on quantized operands: Xq E4M3 [M, K] with Xscale
 * FP32 [M]; Wq E4M3 [N, K] with Wscale FP32 [N] (16-byte aligned); bias F16
 * [N] or NULL; Y BF16 [M, N] (written).  Requires K % 128 == 0, N % 8 == 0,
 * N > 0, M >= 0, every pointer 16-byte aligned.
 */
mxfp8_status fp8rw_gemm(const void *Xq, const float *Xscale, int64_t M, int64_t K, const void *Wq,
                        const float *Wscale, int64_t N, const void *bias, void *Y, mxfp8_stream_t stream);

/* Workspace bytes fp8rw_linear needs: the activation codes (rounded up to
 * 256 bytes) and the FP32 row scales. */
size_t fp8rw_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * The whole layer: fp8rw_quantize_bf16 of X (row stride K) into `workspace`,
 * then fp8rw_gemm.  workspace: >= fp8rw_linear_workspace_bytes(M, K) bytes,
 * 256-byte aligned, overwritten.  Requirements as fp8rw_gemm and
 * K <= FP8RW_MAX_K.
 */
mxfp8_status fp8rw_linear(const void *X, int64_t M, int64_t K, const void *Wq, const float *Wscale, int64_t N,
                          const void *bias, void *Y, void *workspace, size_t ws_bytes, mxfp8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8_ROWWISE_H */
