/*
 * mxfp8_capi.cu -- the C-ABI entry points declared in include/mxfp8.h:
 * argument checks, then kernel launches on the caller's stream.
 */
#include <cuda_runtime.h>
#include <cstdint>

#include "fp8_rowwise.h"
#include "mxfp8.h"
#include "nvfp4.h"

namespace mx {
cudaError_t launch_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, uint8_t *Q, uint8_t *S,
                            bool sf_tc, cudaStream_t stream);
cudaError_t launch_gelu(const void *X, void *Y, int64_t n, cudaStream_t stream);
int launch_gemm(const void *Xq, const void *Xs, int64_t M, int64_t K, const void *Wq, const void *Ws, int64_t N,
                const void *bias, void *Y, int epi, void *S, cudaStream_t stream, unsigned long long timeout_ns,
                cudaError_t *err, const float *gx = nullptr, const float *gw = nullptr);
cudaError_t launch_nvfp4_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, const float *g,
                                  uint8_t *Q, uint8_t *S, cudaStream_t stream);
cudaError_t launch_nvfp4_amax(const void *X, bool f32_in, int64_t n, unsigned int *out, cudaStream_t stream);
cudaError_t launch_nvfp4_global_scale(const float *amax, float *g, cudaStream_t stream);
cudaError_t read_and_clear_status(unsigned int *out);
cudaError_t launch_fp8_rowwise_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, uint8_t *Q,
                                        float *S, cudaStream_t stream, unsigned long long timeout_ns);
cudaError_t read_and_clear_rw_status(unsigned int *out);
cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t stream);
cudaError_t launch_rw_wait_selftest(unsigned long long limit_ns, cudaStream_t stream);
} // namespace mx

namespace {

/* Bound for every pipeline wait inside the GEMM kernel. */
constexpr unsigned long long kWaitLimitNs = 4000000000ull;

/* Largest extents the kernels index with 32-bit tile arithmetic. */
constexpr int64_t kMaxRows = (int64_t)1 << 30;
constexpr int64_t kMaxK = (int64_t)1 << 20;

bool aligned(const void *p, uintptr_t a)
{
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

size_t round_up(size_t v, size_t a)
{
    return (v + a - 1) / a * a;
}

mxfp8_status quantize_args(const void *X, int64_t M, int64_t K, int64_t ldx, const void *codes, const void *scales,
                           int layout, size_t in_elem_bytes)
{
    if (!X || !codes || !scales)
        return M == 0 ? MXFP8_OK : MXFP8_ERR_ARG;
    if (layout != MXFP8_SF_ROWMAJOR && layout != MXFP8_SF_TCGEN05)
        return MXFP8_ERR_ARG;
    if (M < 0 || K <= 0 || ldx < K)
        return MXFP8_ERR_ARG;
    if (K % 32 != 0 || M > kMaxRows || K > kMaxK)
        return MXFP8_ERR_SHAPE;
    if (!aligned(X, 16) || (ldx * (int64_t)in_elem_bytes) % 16 != 0 || !aligned(codes, 8) || !aligned(scales, 4))
        return MXFP8_ERR_ALIGN;
    return MXFP8_OK;
}

mxfp8_status gemm_args(const void *A, const void *As, int64_t M, int64_t K, const void *Wq, const void *Ws,
                       int64_t N, const void *bias, const void *Y)
{
    if (M < 0 || K <= 0 || N <= 0)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!A || !As || !Wq || !Ws || !Y)
        return MXFP8_ERR_ARG;
    if (K % 128 != 0 || N % 8 != 0 || M > kMaxRows || N > kMaxRows || K > kMaxK)
        return MXFP8_ERR_SHAPE;
    if (!aligned(A, 16) || !aligned(As, 16) || !aligned(Wq, 16) || !aligned(Ws, 16) || !aligned(Y, 16) ||
        (bias && !aligned(bias, 16)))
        return MXFP8_ERR_ALIGN;
    return MXFP8_OK;
}

mxfp8_status from_cuda(cudaError_t e)
{
    return e == cudaSuccess ? MXFP8_OK : MXFP8_ERR_CUDA;
}

} // namespace

extern "C" {

const char *mxfp8_status_str(mxfp8_status s)
{
    switch (s) {
    case MXFP8_OK:
        return "MXFP8_OK";
    case MXFP8_ERR_ARG:
        return "MXFP8_ERR_ARG: invalid argument (null pointer, bad layout or negative size)";
    case MXFP8_ERR_ALIGN:
        return "MXFP8_ERR_ALIGN: pointer or leading dimension not aligned";
    case MXFP8_ERR_SHAPE:
        return "MXFP8_ERR_SHAPE: unsupported shape (K % 32, K % 128 for the GEMM, N % 8, size limits)";
    case MXFP8_ERR_CUDA:
        return "MXFP8_ERR_CUDA: a CUDA call or kernel launch failed";
    case MXFP8_ERR_TIMEOUT:
        return "MXFP8_ERR_TIMEOUT: a kernel gave up a bounded pipeline wait";
    }
    return "MXFP8_ERR_UNKNOWN";
}

size_t mxfp8_scale_bytes(int64_t rows, int64_t K, int layout)
{
    if (rows < 0 || K <= 0 || K % 32 != 0)
        return 0;
    if (layout == MXFP8_SF_ROWMAJOR)
        return (size_t)rows * (size_t)(K / 32);
    if (layout == MXFP8_SF_TCGEN05)
        return (size_t)((rows + 127) / 128) * (size_t)((K + 127) / 128) * 512u;
    return 0;
}

mxfp8_status mxfp8_quantize(const void *X, int64_t M, int64_t K, int64_t ldx, void *codes, void *scales, int layout,
                            mxfp8_stream_t stream)
{
    mxfp8_status st = quantize_args(X, M, K, ldx, codes, scales, layout, 2);
    if (st != MXFP8_OK || M == 0)
        return st;
    return from_cuda(mx::launch_quantize(X, false, M, K, ldx, static_cast<uint8_t *>(codes),
                                         static_cast<uint8_t *>(scales), layout == MXFP8_SF_TCGEN05,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

mxfp8_status mxfp8_quantize_weight_f32(const float *W, int64_t N, int64_t K, void *Wq, void *Wscale, int layout,
                                       mxfp8_stream_t stream)
{
    mxfp8_status st = quantize_args(W, N, K, K, Wq, Wscale, layout, 4);
    if (st != MXFP8_OK || N == 0)
        return st;
    return from_cuda(mx::launch_quantize(W, true, N, K, K, static_cast<uint8_t *>(Wq), static_cast<uint8_t *>(Wscale),
                                         layout == MXFP8_SF_TCGEN05, reinterpret_cast<cudaStream_t>(stream)));
}

size_t mxfp8_linear_workspace_bytes(int64_t M, int64_t K)
{
    if (M < 0 || K <= 0 || K % 32 != 0)
        return 0;
    return round_up((size_t)M * (size_t)K, 256) + mxfp8_scale_bytes(M, K, MXFP8_SF_TCGEN05);
}

mxfp8_status mxfp8_gemm_prequant(const void *Xq, const void *Xscale, int64_t M, int64_t K, const void *Wq,
                                 const void *Wscale, int64_t N, const void *bias, void *Y, mxfp8_stream_t stream)
{
    mxfp8_status st = gemm_args(Xq, Xscale, M, K, Wq, Wscale, N, bias, Y);
    if (st != MXFP8_OK || M == 0)
        return st;
    cudaError_t e;
    int r = mx::launch_gemm(Xq, Xscale, M, K, Wq, Wscale, N, bias, Y, 0, nullptr,
                            reinterpret_cast<cudaStream_t>(stream), kWaitLimitNs, &e);
    if (r == 1)
        return MXFP8_ERR_CUDA; /* tensor map could not be encoded */
    return r == 0 ? MXFP8_OK : from_cuda(e);
}

mxfp8_status mxfp8_gemm_quantize_out(const void *Xq, const void *Xscale, int64_t M, int64_t K, const void *Wq,
                                     const void *Wscale, int64_t N, const void *bias, int act, void *Yq,
                                     void *Yscale, mxfp8_stream_t stream)
{
    if (act != MXFP8_ACT_NONE && act != MXFP8_ACT_GELU_TANH)
        return MXFP8_ERR_ARG;
    mxfp8_status st = gemm_args(Xq, Xscale, M, K, Wq, Wscale, N, bias, Yq);
    if (st != MXFP8_OK || M == 0)
        return st;
    if (!Yscale)
        return MXFP8_ERR_ARG;
    if (N % 128 != 0)
        return MXFP8_ERR_SHAPE;
    if (!aligned(Yscale, 16))
        return MXFP8_ERR_ALIGN;
    cudaError_t e;
    int r = mx::launch_gemm(Xq, Xscale, M, K, Wq, Wscale, N, bias, Yq, act == MXFP8_ACT_GELU_TANH ? 2 : 1, Yscale,
                            reinterpret_cast<cudaStream_t>(stream), kWaitLimitNs, &e);
    if (r == 1)
        return MXFP8_ERR_CUDA;
    return r == 0 ? MXFP8_OK : from_cuda(e);
}

mxfp8_status mxfp8_linear(const void *X, int64_t M, int64_t K, const void *Wq, const void *Wscale, int64_t N,
                          const void *bias, void *Y, void *workspace, size_t ws_bytes, mxfp8_stream_t stream)
{
    if (M < 0 || K <= 0 || N <= 0)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!X || !workspace)
        return MXFP8_ERR_ARG;
    if (K % 128 != 0)
        return MXFP8_ERR_SHAPE;
    if (!aligned(workspace, 256) || !aligned(X, 16))
        return MXFP8_ERR_ALIGN;
    if (ws_bytes < mxfp8_linear_workspace_bytes(M, K))
        return MXFP8_ERR_ARG;
    uint8_t *codes = static_cast<uint8_t *>(workspace);
    uint8_t *scales = codes + round_up((size_t)M * (size_t)K, 256);
    mxfp8_status st = gemm_args(codes, scales, M, K, Wq, Wscale, N, bias, Y);
    if (st != MXFP8_OK)
        return st;
    st = mxfp8_quantize(X, M, K, K, codes, scales, MXFP8_SF_TCGEN05, stream);
    if (st != MXFP8_OK)
        return st;
    return mxfp8_gemm_prequant(codes, scales, M, K, Wq, Wscale, N, bias, Y, stream);
}

mxfp8_status mxfp8_gelu_tanh_bf16(const void *X, void *Y, int64_t n, mxfp8_stream_t stream)
{
    if (n < 0)
        return MXFP8_ERR_ARG;
    if (n == 0)
        return MXFP8_OK;
    if (!X || !Y)
        return MXFP8_ERR_ARG;
    if (n % 8 != 0)
        return MXFP8_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(Y, 16))
        return MXFP8_ERR_ALIGN;
    return from_cuda(mx::launch_gelu(X, Y, n, reinterpret_cast<cudaStream_t>(stream)));
}

/* ---------------------------------------------------- per-channel FP8 */

mxfp8_status fp8rw_quantize_bf16(const void *X, int64_t M, int64_t K, int64_t ldx, void *codes, float *scales,
                                 mxfp8_stream_t stream)
{
    if (M < 0 || K <= 0 || ldx < K)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!X || !codes || !scales)
        return MXFP8_ERR_ARG;
    if (K % 8 != 0 || K > FP8RW_MAX_K || M > kMaxRows)
        return MXFP8_ERR_SHAPE;
    if (!aligned(X, 16) || (ldx * 2) % 16 != 0 || !aligned(codes, 8) || !aligned(scales, 4))
        return MXFP8_ERR_ALIGN;
    return from_cuda(mx::launch_fp8_rowwise_quantize(X, false, M, K, ldx, static_cast<uint8_t *>(codes), scales,
                                                     reinterpret_cast<cudaStream_t>(stream), kWaitLimitNs));
}

mxfp8_status fp8rw_quantize_weight_f32(const float *W, int64_t N, int64_t K, void *Wq, float *Wscale,
                                       mxfp8_stream_t stream)
{
    if (N < 0 || K <= 0)
        return MXFP8_ERR_ARG;
    if (N == 0)
        return MXFP8_OK;
    if (!W || !Wq || !Wscale)
        return MXFP8_ERR_ARG;
    if (K % 4 != 0 || K > FP8RW_MAX_K || N > kMaxRows)
        return MXFP8_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(Wq, 4) || !aligned(Wscale, 4))
        return MXFP8_ERR_ALIGN;
    return from_cuda(mx::launch_fp8_rowwise_quantize(W, true, N, K, K, static_cast<uint8_t *>(Wq), Wscale,
                                                     reinterpret_cast<cudaStream_t>(stream), kWaitLimitNs));
}

mxfp8_status fp8rw_gemm(const void *Xq, const float *Xscale, int64_t M, int64_t K, const void *Wq,
                        const float *Wscale, int64_t N, const void *bias, void *Y, mxfp8_stream_t stream)
{
    mxfp8_status st = gemm_args(Xq, Xscale, M, K, Wq, Wscale, N, bias, Y);
    if (st != MXFP8_OK || M == 0)
        return st;
    cudaError_t e;
    int r = mx::launch_gemm(Xq, Xscale, M, K, Wq, Wscale, N, bias, Y, 3, nullptr,
                            reinterpret_cast<cudaStream_t>(stream), kWaitLimitNs, &e);
    if (r == 1)
        return MXFP8_ERR_CUDA;
    return r == 0 ? MXFP8_OK : from_cuda(e);
}

size_t fp8rw_linear_workspace_bytes(int64_t M, int64_t K)
{
    if (M < 0 || K <= 0)
        return 0;
    return round_up((size_t)M * (size_t)K, 256) + (size_t)M * sizeof(float);
}

mxfp8_status fp8rw_linear(const void *X, int64_t M, int64_t K, const void *Wq, const float *Wscale, int64_t N,
                          const void *bias, void *Y, void *workspace, size_t ws_bytes, mxfp8_stream_t stream)
{
    if (M < 0 || K <= 0 || N <= 0)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!X || !workspace)
        return MXFP8_ERR_ARG;
    if (K % 128 != 0 || K > FP8RW_MAX_K)
        return MXFP8_ERR_SHAPE;
    if (!aligned(workspace, 256) || !aligned(X, 16))
        return MXFP8_ERR_ALIGN;
    if (ws_bytes < fp8rw_linear_workspace_bytes(M, K))
        return MXFP8_ERR_ARG;
    uint8_t *codes = static_cast<uint8_t *>(workspace);
    float *scales = reinterpret_cast<float *>(codes + round_up((size_t)M * (size_t)K, 256));
    mxfp8_status st = gemm_args(codes, scales, M, K, Wq, Wscale, N, bias, Y);
    if (st != MXFP8_OK)
        return st;
    st = fp8rw_quantize_bf16(X, M, K, K, codes, scales, stream);
    if (st != MXFP8_OK)
        return st;
    return fp8rw_gemm(codes, scales, M, K, Wq, Wscale, N, bias, Y, stream);
}

/* --------------------------------------------------------------- NVFP4 */

size_t nvfp4_scale_bytes(int64_t rows, int64_t K)
{
    if (rows < 0 || K <= 0 || K % 16 != 0)
        return 0;
    return (size_t)((rows + 127) / 128) * (size_t)((K + 63) / 64) * 512u;
}

static mxfp8_status nvfp4_amax_any(const void *X, bool f32, int64_t n, float *amax, mxfp8_stream_t stream)
{
    if (n < 0 || !amax)
        return MXFP8_ERR_ARG;
    if (n > 0 && !X)
        return MXFP8_ERR_ARG;
    if (n % 16 != 0)
        return MXFP8_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(amax, 4))
        return MXFP8_ERR_ALIGN;
    return from_cuda(mx::launch_nvfp4_amax(X, f32, n, reinterpret_cast<unsigned int *>(amax),
                                           reinterpret_cast<cudaStream_t>(stream)));
}

mxfp8_status nvfp4_amax_bf16(const void *X, int64_t n, float *amax, mxfp8_stream_t stream)
{
    return nvfp4_amax_any(X, false, n, amax, stream);
}

mxfp8_status nvfp4_amax_f32(const float *W, int64_t n, float *amax, mxfp8_stream_t stream)
{
    return nvfp4_amax_any(W, true, n, amax, stream);
}

mxfp8_status nvfp4_global_scale_from_amax(const float *amax, float *global_scale, mxfp8_stream_t stream)
{
    if (!amax || !global_scale)
        return MXFP8_ERR_ARG;
    if (!aligned(amax, 4) || !aligned(global_scale, 4))
        return MXFP8_ERR_ALIGN;
    return from_cuda(mx::launch_nvfp4_global_scale(amax, global_scale, reinterpret_cast<cudaStream_t>(stream)));
}

static mxfp8_status nvfp4_quantize_any(const void *X, bool f32, int64_t M, int64_t K, int64_t ldx, const float *g,
                                       void *codes, void *scales, mxfp8_stream_t stream)
{
    if (M < 0 || K <= 0 || ldx < K)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!X || !g || !codes || !scales)
        return MXFP8_ERR_ARG;
    if (K % 16 != 0 || M > kMaxRows || K > kMaxK)
        return MXFP8_ERR_SHAPE;
    if (!aligned(X, 16) || (ldx * (f32 ? 4 : 2)) % 16 != 0 || !aligned(codes, 8) || !aligned(scales, 4) ||
        !aligned(g, 4))
        return MXFP8_ERR_ALIGN;
    return from_cuda(mx::launch_nvfp4_quantize(X, f32, M, K, ldx, g, static_cast<uint8_t *>(codes),
                                               static_cast<uint8_t *>(scales),
                                               reinterpret_cast<cudaStream_t>(stream)));
}

mxfp8_status nvfp4_quantize_bf16(const void *X, int64_t M, int64_t K, int64_t ldx, const float *global_scale,
                                 void *codes, void *scales, mxfp8_stream_t stream)
{
    return nvfp4_quantize_any(X, false, M, K, ldx, global_scale, codes, scales, stream);
}

mxfp8_status nvfp4_quantize_weight_f32(const float *W, int64_t N, int64_t K, const float *global_scale, void *Wq,
                                       void *Wscale, mxfp8_stream_t stream)
{
    return nvfp4_quantize_any(W, true, N, K, K, global_scale, Wq, Wscale, stream);
}

static mxfp8_status nvfp4_gemm_args(const void *Xq, const void *Xscale, int64_t M, int64_t K, const void *Wq,
                                    const void *Wscale, int64_t N, const float *gx, const float *gw,
                                    const void *bias, const void *Y)
{
    if (M < 0 || K <= 0 || N <= 0)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!Xq || !Xscale || !Wq || !Wscale || !Y || !gx || !gw)
        return MXFP8_ERR_ARG;
    if (K % 64 != 0 || N % 8 != 0 || M > kMaxRows || N > kMaxRows || K > kMaxK)
        return MXFP8_ERR_SHAPE;
    if (!aligned(Xq, 16) || !aligned(Xscale, 16) || !aligned(Wq, 16) || !aligned(Wscale, 16) || !aligned(Y, 16) ||
        (bias && !aligned(bias, 16)) || !aligned(gx, 4) || !aligned(gw, 4))
        return MXFP8_ERR_ALIGN;
    return MXFP8_OK;
}

mxfp8_status nvfp4_gemm(const void *Xq, const void *Xscale, int64_t M, int64_t K, const void *Wq,
                        const void *Wscale, int64_t N, const float *x_global_scale, const float *w_global_scale,
                        const void *bias, void *Y, mxfp8_stream_t stream)
{
    mxfp8_status st = nvfp4_gemm_args(Xq, Xscale, M, K, Wq, Wscale, N, x_global_scale, w_global_scale, bias, Y);
    if (st != MXFP8_OK || M == 0)
        return st;
    cudaError_t e;
    /* the block-scaled GEMM in its NVFP4 mode (tcgen05.mma kind::mxf4nvf4) */
    int r = mx::launch_gemm(Xq, Xscale, M, K, Wq, Wscale, N, bias, Y, 4, nullptr,
                            reinterpret_cast<cudaStream_t>(stream), kWaitLimitNs, &e, x_global_scale, w_global_scale);
    if (r == 1)
        return MXFP8_ERR_CUDA;
    return r == 0 ? MXFP8_OK : from_cuda(e);
}

size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K)
{
    if (M < 0 || K <= 0 || K % 16 != 0)
        return 0;
    return round_up((size_t)M * (size_t)(K / 2), 256) + nvfp4_scale_bytes(M, K);
}

mxfp8_status nvfp4_linear(const void *X, int64_t M, int64_t K, const float *x_global_scale, const void *Wq,
                          const void *Wscale, int64_t N, const float *w_global_scale, const void *bias, void *Y,
                          void *workspace, size_t ws_bytes, mxfp8_stream_t stream)
{
    if (M < 0 || K <= 0 || N <= 0)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!X || !workspace || !x_global_scale)
        return MXFP8_ERR_ARG;
    if (K % 64 != 0)
        return MXFP8_ERR_SHAPE;
    if (!aligned(workspace, 256) || !aligned(X, 16))
        return MXFP8_ERR_ALIGN;
    if (ws_bytes < nvfp4_linear_workspace_bytes(M, K))
        return MXFP8_ERR_ARG;
    uint8_t *codes = static_cast<uint8_t *>(workspace);
    uint8_t *scales = codes + round_up((size_t)M * (size_t)(K / 2), 256);
    /* every check of both steps before anything is launched */
    mxfp8_status st =
        nvfp4_gemm_args(codes, scales, M, K, Wq, Wscale, N, x_global_scale, w_global_scale, bias, Y);
    if (st != MXFP8_OK)
        return st;
    st = nvfp4_quantize_bf16(X, M, K, K, x_global_scale, codes, scales, stream);
    if (st != MXFP8_OK)
        return st;
    return nvfp4_gemm(codes, scales, M, K, Wq, Wscale, N, x_global_scale, w_global_scale, bias, Y, stream);
}

mxfp8_status mxfp8_selftest_wait_timeout(int which, uint64_t timeout_ns, mxfp8_stream_t stream)
{
    if (timeout_ns == 0 || timeout_ns > 10000000000ull)
        return MXFP8_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (which) {
    case MXFP8_SELFTEST_GEMM:
        return from_cuda(mx::launch_wait_selftest(timeout_ns, s));
    case MXFP8_SELFTEST_NVFP4_GEMM: /* the same block-scaled GEMM kernel in its NVFP4 mode */
        return from_cuda(mx::launch_wait_selftest(timeout_ns, s));
    case MXFP8_SELFTEST_ROWWISE_QUANT:
        return from_cuda(mx::launch_rw_wait_selftest(timeout_ns, s));
    default:
        return MXFP8_ERR_ARG;
    }
}

mxfp8_status mxfp8_device_status(mxfp8_stream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return MXFP8_ERR_CUDA;
    unsigned int word = 0, rw_word = 0;
    if (mx::read_and_clear_status(&word) != cudaSuccess || mx::read_and_clear_rw_status(&rw_word) != cudaSuccess)
        return MXFP8_ERR_CUDA;
    return (word | rw_word) ? MXFP8_ERR_TIMEOUT : MXFP8_OK;
}

} // extern "C"
