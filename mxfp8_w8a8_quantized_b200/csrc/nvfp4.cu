/*
 * nvfp4.cu -- NVFP4 quantization (sm_100a): packed E2M1 codes with one UE4M3
 * scale per 16 elements and an FP32 global scale per tensor (page "Wan2.2
 * I2V A14B, four-step 720p: native LightX2V FP8 and NVFP4", "Conversion and
 * compatibility": packed E2M1 weights with E4M3 block scales, FP32
 * input_global_scale and alpha fields; weights enter the quantizer as BF16).
 *
 * Per 16-element block, all in binary32 (the readings the oracle states):
 *   s = UE4M3(RN(amax * RN(g / 6)))       nearest even, saturating at 448
 *   q = E2M1(RN(x * RN(g / dec(s))))      nearest even, saturating at 6
 * A block whose scale is 0 gets codes +-0.  Codes are packed two per byte,
 * the even element in the low nibble; scales go straight into the
 * tensor-core layout (512-byte atoms of 128 rows x 4 blocks, now 64 K
 * elements per atom).
 *
 * HBM-bound: 2 (BF16) or 4 (FP32) bytes read, 0.5 + 1/16 byte written per
 * element.  One lane owns one block (16 elements, two 16-byte loads), so the
 * block amax needs no shuffle; each warp walks whole rows in segments of 512
 * elements (every address in a row is the row's base plus a multiple of the
 * segment), two segments in flight; four lanes' scale bytes form one 32-bit
 * word of an atom.  The block amax and the scaling run two elements per
 * instruction on the floating-point pipe.  FP32 weights are rounded to BF16
 * (nearest even) on load.
 */
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_element.cuh"

namespace mx {

constexpr int NQ_THREADS = 256;
constexpr int NQ_UNROLL = 2;

/* the 16 elements starting at element k0 of `row`, as 8 words of BF16 pairs */
template <bool F32_IN>
__device__ __forceinline__ void nq_load16(uint32_t (&w)[8], const uint8_t *row, int64_t k0)
{
    if constexpr (F32_IN) {
        const uint4 *p = reinterpret_cast<const uint4 *>(row + k0 * 4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldcs(p + i);
            __nv_bfloat162 a = __floats2bfloat162_rn(__uint_as_float(v.x), __uint_as_float(v.y));
            __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v.z), __uint_as_float(v.w));
            w[2 * i] = *reinterpret_cast<uint32_t *>(&a);
            w[2 * i + 1] = *reinterpret_cast<uint32_t *>(&b);
        }
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(row + k0 * 2);
        const uint4 a = __ldcs(p), b = __ldcs(p + 1);
        w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = b.x, w[5] = b.y, w[6] = b.z, w[7] = b.w;
    }
}

/* max(|a|, |b|) of each BF16 half (sign = xor of the signs; a NaN gives the
 * canonical NaN) */
__device__ __forceinline__ uint32_t nq_absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

/* 8 values -> 4 bytes of E2M1 pairs (even element in the low nibble). */
__device__ __forceinline__ uint32_t nq_e2m1x8(float x0, float x1, float x2, float x3, float x4, float x5, float x6,
                                              float x7)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}\n"
        : "=r"(r)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
    return r;
}

/*
 * X [M, K] (row stride ldx) -> Q [M, K/2] packed codes, S scales (tensor-core
 * layout, kg = ceil(K / 64) atoms per 128 rows).  Each warp walks whole rows
 * (rows warp, warp + nwarps, ...); in segment j lane l owns block 32 j + l.
 * Rows in [M, Mrows) only write zero scale padding.
 */
template <bool F32_IN>
__global__ void __launch_bounds__(NQ_THREADS) nvfp4_quantize_kernel(const void *__restrict__ X, int64_t M, int64_t K,
                                                                    int64_t ldx, const float *__restrict__ gptr,
                                                                    uint8_t *__restrict__ Q,
                                                                    uint8_t *__restrict__ S, int64_t Mrows,
                                                                    int64_t nseg, int64_t kg)
{
    const int lane = threadIdx.x & 31;
    const int warp0 = (int)((blockIdx.x * NQ_THREADS + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * NQ_THREADS) >> 5);
    const int nblocks = (int)(K >> 4);
    const float g = __ldg(gptr);
    const float gs = __fdiv_rn(g, 6.0f);
    const int M32 = (int)M, K32 = (int)K, nseg32 = (int)nseg, Mrows32 = (int)Mrows;
    constexpr int EB = F32_IN ? 4 : 2;

    for (int r = warp0; r < Mrows32; r += nwarps) {
        const bool row_ok = r < M32;
        const uint8_t *xrow = reinterpret_cast<const uint8_t *>(X) + (int64_t)r * ldx * EB;
        uint8_t *qrow = Q + (int64_t)r * (K >> 1);
        uint8_t *srow = S + ((((int64_t)(r >> 7)) * kg) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
        for (int j = 0; j < nseg32; j += NQ_UNROLL) {
            uint32_t w[NQ_UNROLL][8];
            int k0[NQ_UNROLL];
            bool valid[NQ_UNROLL];
#pragma unroll
            for (int i = 0; i < NQ_UNROLL; ++i) {
                k0[i] = (j + i) * 512 + lane * 16;
                valid[i] = row_ok && (j + i < nseg32) && (k0[i] < K32);
                if (valid[i])
                    nq_load16<F32_IN>(w[i], xrow, k0[i]);
            }
#pragma unroll
            for (int i = 0; i < NQ_UNROLL; ++i) {
                if (j + i >= nseg32) /* warp-uniform */
                    break;
                uint32_t sb = 0u;
                if (valid[i]) {
                    const uint32_t a = nq_absmax_bf16x2(w[i][0], w[i][1]);
                    const uint32_t b = nq_absmax_bf16x2(w[i][2], w[i][3]);
                    const uint32_t c = nq_absmax_bf16x2(w[i][4], w[i][5]);
                    const uint32_t d = nq_absmax_bf16x2(w[i][6], w[i][7]);
                    const uint32_t m2 = nq_absmax_bf16x2(nq_absmax_bf16x2(a, b), nq_absmax_bf16x2(c, d)) & 0x7FFF7FFFu;
                    /* non-negative BF16 bit patterns order like their values */
                    const float amax = __uint_as_float(max(m2 << 16, m2 & 0xFFFF0000u));
                    sb = (uint32_t)__nv_cvt_float_to_fp8(amax * gs, __NV_SATFINITE, __NV_E4M3) & 0x7Fu;
                    const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sb, __NV_E4M3);
                    const float ds = __half2float(__half(hr));
                    const float mul = ds > 0.0f ? __fdiv_rn(g, ds) : 0.0f;
                    /* packed binary32 multiplies: each lane rounded like the scalar one */
                    const f32x2 mm = f2_pack(mul, mul);
                    float f[16];
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        f2_unpack(f2_mul(bf16x2_to_f32x2(w[i][k]), mm), f[2 * k], f[2 * k + 1]);
                    const uint32_t lo = nq_e2m1x8(f[0], f[1], f[2], f[3], f[4], f[5], f[6], f[7]);
                    const uint32_t hi = nq_e2m1x8(f[8], f[9], f[10], f[11], f[12], f[13], f[14], f[15]);
                    *reinterpret_cast<uint2 *>(qrow + (k0[i] >> 1)) = make_uint2(lo, hi);
                }
                /* word q (lanes 4q .. 4q+3) = blocks 32 (j+i) + 4q .. 32 (j+i) + 4q + 3 */
                const uint32_t word = sb | (__shfl_down_sync(0xFFFFFFFFu, sb, 1) << 8) |
                                      (__shfl_down_sync(0xFFFFFFFFu, sb, 2) << 16) |
                                      (__shfl_down_sync(0xFFFFFFFFu, sb, 3) << 24);
                const int bk = k0[i] >> 4; /* this lane's block = first block of the word */
                if ((lane & 3) == 0 && bk < nblocks)
                    *reinterpret_cast<uint32_t *>(srow + ((int64_t)(bk >> 2) << 9)) = word;
            }
        }
    }
}

/* Largest magnitude of a tensor (after rounding FP32 input to BF16), as the
 * bit pattern of a binary32, max-combined into *out. */
template <bool F32_IN>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const void *__restrict__ X, int64_t n16,
                                                         unsigned int *__restrict__ out)
{
    uint32_t m2 = 0u;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x) {
        uint32_t w[8];
        nq_load16<F32_IN>(w, reinterpret_cast<const uint8_t *>(X), i * 16);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            m2 = __vmaxu2(m2, w[k] & 0x7FFF7FFFu);
    }
    uint32_t m = max(m2 << 16, m2 & 0xFFFF0000u);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0 && m != 0u)
        atomicMax(out, m);
}

/* The global scale g = RN(448 * 6 / amax) of a tensor whose amax is
 * *amax_bits; 1 when amax is 0 (or not finite) or the quotient overflows,
 * since then no finite scale maps the tensor onto the format's range. */
__global__ void nvfp4_global_scale_kernel(const unsigned int *__restrict__ amax_bits, float *__restrict__ g)
{
    const float amax = __uint_as_float(*amax_bits);
    float v = 1.0f;
    if (amax > 0.0f && amax <= 3.4028235e38f) {
        const float q = __fdiv_rn(448.0f * 6.0f, amax);
        if (q <= 3.4028235e38f)
            v = q;
    }
    *g = v;
}

static int nq_num_sms()
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

cudaError_t launch_nvfp4_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, const float *g,
                                  uint8_t *Q, uint8_t *S, cudaStream_t stream)
{
    const int64_t Mrows = ((M + 127) / 128) * 128;
    const int64_t nseg = (K + 511) / 512;
    const int64_t kg = (K / 16 + 3) / 4;
    const int64_t units = Mrows * nseg;
    if (units == 0)
        return cudaSuccess;
    const int64_t per_block = NQ_THREADS / 32; /* rows per block */
    int64_t blocks = (Mrows + per_block - 1) / per_block;
    const int64_t cap = (int64_t)nq_num_sms() * 8 * 4; /* 8 resident blocks x 4 waves */
    if (blocks > cap)
        blocks = cap;
    if (f32_in)
        nvfp4_quantize_kernel<true><<<(unsigned)blocks, NQ_THREADS, 0, stream>>>(X, M, K, ldx, g, Q, S, Mrows, nseg, kg);
    else
        nvfp4_quantize_kernel<false><<<(unsigned)blocks, NQ_THREADS, 0, stream>>>(X, M, K, ldx, g, Q, S, Mrows, nseg,
                                                                                  kg);
    return cudaGetLastError();
}

/* n % 16 == 0; *out (device) receives the amax bits (cleared first). */
cudaError_t launch_nvfp4_amax(const void *X, bool f32_in, int64_t n, unsigned int *out, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(unsigned int), stream);
    if (e != cudaSuccess || n == 0)
        return e;
    const int64_t n16 = n / 16;
    int64_t blocks = (n16 + 255) / 256;
    const int64_t cap = (int64_t)nq_num_sms() * 8;
    if (blocks > cap)
        blocks = cap;
    if (f32_in)
        nvfp4_amax_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(X, n16, out);
    else
        nvfp4_amax_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(X, n16, out);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_global_scale(const float *amax, float *g, cudaStream_t stream)
{
    nvfp4_global_scale_kernel<<<1, 1, 0, stream>>>(reinterpret_cast<const unsigned int *>(amax), g);
    return cudaGetLastError();
}

} // namespace mx
