/*
 * fp8_rowwise.cu -- per-channel FP8 quantization (sm_100a): one FP32 scale
 * per row, s = amax / 448, codes E4M3(x / s), both binary32 divisions
 * rounded to nearest even ("Model Quantization Techniques", "Quantization
 * Modes": fp8-vllm / fp8-sgl, channel-symmetric FP8 weights and
 * channel-dynamic symmetric FP8 activations; "MiniMax-H3 FP8 with FP16
 * Accumulation": scale = max(abs(x)) / qmax, and qmax = 448 with FP32
 * accumulation, "MiniMax-H3 Video VAE Encoder Conv3D").
 *
 * HBM-bound: 2 (BF16) or 4 (FP32) bytes read + 1 code byte written per
 * element, 4 bytes per row.  One CTA of 256 threads owns a row at a time: the
 * row is loaded once into registers with 16-byte loads (consecutive threads,
 * consecutive chunks), its amax is a block reduction, and the codes are
 * written from the registers -- the row is never read twice.  Rows of up to
 * 16384 elements fit (8 BF16 or 16 FP32 chunks per thread).
 */
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace mx {

constexpr int RW_THREADS = 256;
constexpr int RW_MAX_K = 16384;

template <bool F32_IN>
struct RwCfg {
    static constexpr int EPC = F32_IN ? 4 : 8;                    /* elements per 16-byte chunk */
    static constexpr int CHUNKS = RW_MAX_K / EPC / RW_THREADS;    /* chunks per thread, at most */
};

/* Largest magnitude of a chunk, as the bit pattern of a binary32. */
template <bool F32_IN>
__device__ __forceinline__ uint32_t rw_amax(const uint4 &v)
{
    if constexpr (F32_IN) {
        return max(max(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu), max(v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu));
    } else {
        /* non-negative BF16 bit patterns order like their values */
        const uint32_t k = 0x7FFF7FFFu;
        const uint32_t m = __vmaxu2(__vmaxu2(v.x & k, v.y & k), __vmaxu2(v.z & k, v.w & k));
        return max(m << 16, m & 0xFFFF0000u);
    }
}

/* E4M3 of x / s (binary32 division); a zero scale means x is +-0. */
__device__ __forceinline__ uint32_t rw_code2(float a, float b, float s)
{
    const float qa = s != 0.0f ? __fdiv_rn(a, s) : a;
    const float qb = s != 0.0f ? __fdiv_rn(b, s) : b;
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(qa, qb), __NV_SATFINITE, __NV_E4M3);
}

template <bool F32_IN>
__global__ void __launch_bounds__(RW_THREADS) fp8_rowwise_quantize_kernel(const void *__restrict__ X, int64_t M,
                                                                          int K, int64_t ldx,
                                                                          uint8_t *__restrict__ Q,
                                                                          float *__restrict__ S)
{
    using C = RwCfg<F32_IN>;
    __shared__ uint32_t red[RW_THREADS / 32];
    const int nchunks = K / C::EPC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
        const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(X) +
                                                           r * ldx * (F32_IN ? 4 : 2));
        uint4 v[C::CHUNKS];
        uint32_t amax = 0u;
#pragma unroll
        for (int j = 0; j < C::CHUNKS; ++j) {
            const int c = threadIdx.x + j * RW_THREADS;
            if (c < nchunks) {
                v[j] = __ldcs(row + c);
                amax = max(amax, rw_amax<F32_IN>(v[j]));
            }
        }
        amax = __reduce_max_sync(0xFFFFFFFFu, amax);
        if (lane == 0)
            red[warp] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int w = 1; w < RW_THREADS / 32; ++w)
            amax = max(amax, red[w]);
        __syncthreads(); /* red[] is rewritten for the next row */
        const float s = __fdiv_rn(__uint_as_float(amax), 448.0f);
        if (threadIdx.x == 0)
            S[r] = s;
        uint8_t *qrow = Q + r * (int64_t)K;
#pragma unroll
        for (int j = 0; j < C::CHUNKS; ++j) {
            const int c = threadIdx.x + j * RW_THREADS;
            if (c >= nchunks)
                continue;
            if constexpr (F32_IN) {
                const uint32_t lo = rw_code2(__uint_as_float(v[j].x), __uint_as_float(v[j].y), s);
                const uint32_t hi = rw_code2(__uint_as_float(v[j].z), __uint_as_float(v[j].w), s);
                reinterpret_cast<uint32_t *>(qrow)[c] = lo | (hi << 16);
            } else {
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[i] = rw_code2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u), s);
                reinterpret_cast<uint2 *>(qrow)[c] = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
            }
        }
    }
}

static int rw_num_sms()
{
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        sms[dev] = v;
    }
    return sms[dev];
}

/* X [M, K] (row stride ldx elements) -> Q [M, K], S [M].  K % (8 or 4) == 0,
 * K <= 16384; returns the launch status. */
cudaError_t launch_fp8_rowwise_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, uint8_t *Q,
                                        float *S, cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    int64_t blocks = (int64_t)rw_num_sms() * 8; /* 8 resident CTAs of 256 threads per SM */
    if (blocks > M)
        blocks = M;
    if (f32_in)
        fp8_rowwise_quantize_kernel<true><<<(unsigned)blocks, RW_THREADS, 0, stream>>>(X, M, (int)K, ldx, Q, S);
    else
        fp8_rowwise_quantize_kernel<false><<<(unsigned)blocks, RW_THREADS, 0, stream>>>(X, M, (int)K, ldx, Q, S);
    return cudaGetLastError();
}

} // namespace mx
