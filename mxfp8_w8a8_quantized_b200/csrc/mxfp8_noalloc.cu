/*
 * mxfp8_noalloc.cu -- mxfp8_linear without a caller-provided workspace.
 *
 * mxfp8_linear needs scratch device memory for the quantized activations
 * (E4M3 codes and E8M0 scales) between its two kernels, and expects the
 * caller to allocate it.  Some callers cannot: code that runs inside another
 * runtime's launch hook (a plugin's enqueue, a callback of a serving engine)
 * where allocating is forbidden, or a process whose memory allocator already
 * holds all of the GPU's memory, so that cudaMalloc -- which also
 * synchronizes the device -- would fail or stall every other stream.  For
 * them this file keeps one fixed scratch array in the library's own device
 * memory and runs the same two kernels on it.
 *
 * The array is a file-scope __device__ variable of MXFP8_NOALLOC_SCRATCH_BYTES
 * (34 MiB): every GPU that loads the library holds it until the process
 * exits.  Host code cannot use the variable's name as a device address, so
 * the first call on each device asks the runtime for its address
 * (cudaGetSymbolAddress, with that device current) and caches it.  The
 * cache entries are atomics, so first calls from several host threads at
 * once are well defined (each stores the same address).  A cudaDeviceReset
 * destroys the context the address belongs to: a process that resets a
 * device must not call mxfp8_linear_noalloc on it afterwards.
 */
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "mxfp8.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[MXFP8_NOALLOC_SCRATCH_BYTES];

namespace {

std::atomic<void *> g_scratch_addr[64];

/* Device address of the scratch array on the current device. */
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    void *p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (!p) {
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_addr[dev].store(p, std::memory_order_relaxed);
    }
    *out = p;
    return cudaSuccess;
}

} // namespace

extern "C" mxfp8_status mxfp8_linear_noalloc(const void *X, int64_t M, int64_t K, const void *Wq,
                                             const void *Wscale, int64_t N, const void *bias, void *Y,
                                             mxfp8_stream_t stream)
{
    if (M < 0 || K <= 0 || N <= 0)
        return MXFP8_ERR_ARG;
    if (M == 0)
        return MXFP8_OK;
    if (!X || !Wq || !Wscale || !Y)
        return MXFP8_ERR_ARG;
    if (K % 128 != 0 || N % 8 != 0)
        return MXFP8_ERR_SHAPE;
    /* the GEMM's checks too, before the quantizer is launched */
    const auto a16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(X) || !a16(Wq) || !a16(Wscale) || !a16(Y) || (bias && !a16(bias)))
        return MXFP8_ERR_ALIGN;
    /* the activation codes and their scales must fit the fixed scratch */
    if (M > MXFP8_NOALLOC_MAX_CODE_BYTES / K ||
        mxfp8_scale_bytes(M, K, MXFP8_SF_TCGEN05) > (size_t)MXFP8_NOALLOC_MAX_SCALE_BYTES)
        return MXFP8_ERR_SHAPE;
    void *base = nullptr;
    if (scratch_address(&base) != cudaSuccess)
        return MXFP8_ERR_CUDA;
    uint8_t *codes = static_cast<uint8_t *>(base);
    uint8_t *scales = codes + MXFP8_NOALLOC_MAX_CODE_BYTES;
    /* Every byte the GEMM reads from the scratch is written by the quantizer
     * in this same call (codes of rows < M, all scale bytes including the
     * padding); rows >= M are never read (the GEMM's loads fill them with
     * zeros), so nothing has to be cleared between calls. */
    mxfp8_status st = mxfp8_quantize(X, M, K, K, codes, scales, MXFP8_SF_TCGEN05, stream);
    if (st != MXFP8_OK)
        return st;
    return mxfp8_gemm_prequant(codes, scales, M, K, Wq, Wscale, N, bias, Y, stream);
}
