/*
 * mxfp8_quant.cu -- MX quantization kernels (sm_100a) and the GELU kernel.
 *
 * Dynamic activation quantization and offline weight quantization to MXFP8
 * (model card "Wan2.2-I2V-A14B-Lightning . MXFP8 (AutoRound OptRTN)",
 * "Quantization Details": group_size / act_group_size 32, symmetric, mx_fp
 * 8-bit; "Coverage per transformer": E4M3 codes with per-32 E8M0 scales,
 * activations quantized dynamically at run time).
 *
 * Per 32-element block: amax = max|x|; scale byte = clamp(E(amax) - 8) where
 * E(amax) is amax's biased binary32 exponent field (so the unbiased scale
 * exponent is floor(log2 amax) - 8 -- the OCP MX rule -- clamped to the E8M0
 * minimum -127 for zero / tiny blocks); codes = cvt.rn.satfinite E4M3 of
 * x * 2^-e (exact: a power-of-two multiply of a BF16/FP32 value).
 *
 * HBM-bound: 2 (BF16) or 4 (FP32) bytes read + 1 code byte + 1/32 scale byte
 * written per element.  Each warp handles row segments of 256 elements: every
 * lane loads 8 consecutive elements with 128-bit loads (fully coalesced 512 B
 * per warp load), 4 lanes form one 32-block and reduce amax with two
 * shuffle-xor steps, each lane packs 8 codes into one 8-byte store (coalesced
 * 256 B per warp), and scales are gathered into 32-bit words written straight
 * into the tensor-core scale layout (see include/mxfp8.h).  Four segments are
 * loaded before any is processed to keep several 16-byte loads in flight per
 * thread.
 */
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace mx {

constexpr int QTHREADS = 256;
constexpr int QUNROLL = 4;

/* Scale byte from the bit pattern of amax as a binary32 (sign cleared). */
__device__ __forceinline__ uint32_t scale_byte_from_amax(uint32_t abits)
{
    uint32_t ef = abits >> 23;
    if (ef >= 255u)
        return 0xFFu;                 /* Inf / NaN in the block */
    return ef > 8u ? ef - 8u : 0u;    /* e = (ef - 127) - 8, clamped at -127 */
}

/* 2^-e as a binary32 for a finite scale byte b (e = b - 127, b <= 246). */
__device__ __forceinline__ float inv_scale(uint32_t b)
{
    return __uint_as_float((254u - b) << 23);
}

__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d)
{
    __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

template <bool F32_IN>
struct Seg8 {
    uint4 v[F32_IN ? 2 : 1];
};

template <bool F32_IN>
__device__ __forceinline__ void load_seg8(Seg8<F32_IN> &s, const void *base, int64_t elem_off)
{
    if constexpr (F32_IN) {
        const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const float *>(base) + elem_off);
        s.v[0] = __ldcs(p);
        s.v[1] = __ldcs(p + 1);
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(base) + elem_off);
        s.v[0] = __ldcs(p);
    }
}

/* The 8 elements as floats, and the max of their magnitudes as binary32 bits. */
template <bool F32_IN>
__device__ __forceinline__ uint32_t unpack_seg8(const Seg8<F32_IN> &s, float (&f)[8])
{
    uint32_t amax = 0;
    if constexpr (F32_IN) {
        const uint32_t w[8] = {s.v[0].x, s.v[0].y, s.v[0].z, s.v[0].w, s.v[1].x, s.v[1].y, s.v[1].z, s.v[1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[i] = __uint_as_float(w[i]);
            amax = max(amax, w[i] & 0x7FFFFFFFu);
        }
    } else {
        const uint32_t w[4] = {s.v[0].x, s.v[0].y, s.v[0].z, s.v[0].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t lo = w[i] << 16, hi = w[i] & 0xFFFF0000u;
            f[2 * i] = __uint_as_float(lo);
            f[2 * i + 1] = __uint_as_float(hi);
            amax = max(amax, max(lo & 0x7FFFFFFFu, hi & 0x7FFFFFFFu));
        }
    }
    return amax;
}

/*
 * X [M, K] (row stride ldx elements) -> Q [M, K] codes, S scales.
 * Work unit = (row r, segment j of 256 elements); rows r in [M, Mrows) only
 * write zero scale padding (tensor-core layout).
 */
template <bool F32_IN, bool SF_TC>
__global__ void __launch_bounds__(QTHREADS) mx_quantize_kernel(const void *__restrict__ X, int64_t M, int64_t K,
                                                               int64_t ldx, uint8_t *__restrict__ Q,
                                                               uint8_t *__restrict__ S, int64_t Mrows,
                                                               int64_t nseg, int64_t kgroups)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * QTHREADS + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * QTHREADS) >> 5;
    const int64_t units = Mrows * nseg;
    const int64_t nblocks = K >> 5;

    for (int64_t u0 = warp0 * QUNROLL; u0 < units; u0 += nwarps * QUNROLL) {
        Seg8<F32_IN> seg[QUNROLL];
        int64_t row[QUNROLL], k0[QUNROLL];
        bool valid[QUNROLL];
#pragma unroll
        for (int i = 0; i < QUNROLL; ++i) {
            const int64_t u = u0 + i;
            row[i] = u / nseg;
            k0[i] = (u - row[i] * nseg) * 256 + lane * 8;
            valid[i] = (u < units) && (row[i] < M) && (k0[i] < K);
            if (valid[i])
                load_seg8<F32_IN>(seg[i], X, row[i] * ldx + k0[i]);
        }
#pragma unroll
        for (int i = 0; i < QUNROLL; ++i) {
            if (u0 + i >= units) /* warp-uniform */
                break;
            float f[8];
            uint32_t amax = 0;
            if (valid[i])
                amax = unpack_seg8<F32_IN>(seg[i], f);
            amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
            amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
            const uint32_t sb = valid[i] ? scale_byte_from_amax(amax) : 0u;
            if (valid[i]) {
                uint2 out;
                if (sb == 0xFFu) {
                    out = make_uint2(0x7F7F7F7Fu, 0x7F7F7F7Fu);
                } else {
                    const float m = inv_scale(sb);
                    out.x = pack4_e4m3(f[0] * m, f[1] * m, f[2] * m, f[3] * m);
                    out.y = pack4_e4m3(f[4] * m, f[5] * m, f[6] * m, f[7] * m);
                }
                *reinterpret_cast<uint2 *>(Q + row[i] * K + k0[i]) = out;
            }
            if constexpr (SF_TC) {
                /* lanes 0,4,8,12 hold blocks 8j..8j+3, lanes 16..28 blocks 8j+4..8j+7 */
                const int base = lane & 16;
                const uint32_t w = __shfl_sync(0xFFFFFFFFu, sb, base) |
                                   (__shfl_sync(0xFFFFFFFFu, sb, base + 4) << 8) |
                                   (__shfl_sync(0xFFFFFFFFu, sb, base + 8) << 16) |
                                   (__shfl_sync(0xFFFFFFFFu, sb, base + 12) << 24);
                if ((lane & 15) == 0) {
                    const int64_t r = row[i];
                    const int64_t kb = ((k0[i] - lane * 8) >> 5) + (lane >> 2); /* first block of this word */
                    if (kb < nblocks) {
                        const int64_t off = (((r >> 7) * kgroups + (kb >> 2)) << 9) + ((r & 31) << 4) +
                                            (((r >> 5) & 3) << 2);
                        *reinterpret_cast<uint32_t *>(S + off) = w;
                    }
                }
            } else {
                if (valid[i] && (lane & 3) == 0)
                    S[row[i] * nblocks + (k0[i] >> 5)] = (uint8_t)sb;
            }
        }
    }
}

/* ------------------------------------------------------------------ GELU */
__device__ __forceinline__ float gelu_tanh_f32(float x)
{
    /* 0.5 x (1 + tanh(u)) == x sigmoid(2u),  u = sqrt(2/pi)(x + 0.044715 x^3);
     * the exponential is taken of -|2u| so that it never overflows: for very
     * negative x the result underflows gradually instead of becoming -0. */
    const float u = 0.7978845608028654f * (x + 0.044715f * x * x * x);
    const float t = expf(-fabsf(2.0f * u));
    return u >= 0.0f ? x / (1.0f + t) : x * t / (1.0f + t);
}

__global__ void __launch_bounds__(256) gelu_tanh_bf16_kernel(const uint4 *__restrict__ X, uint4 *__restrict__ Y,
                                                             int64_t n8)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        uint4 v = X[i];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float lo = gelu_tanh_f32(__uint_as_float(w[j] << 16));
            float hi = gelu_tanh_f32(__uint_as_float(w[j] & 0xFFFF0000u));
            __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
            w[j] = *reinterpret_cast<uint32_t *>(&p);
        }
        Y[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

/* ------------------------------------------------------------ launchers */
static int num_sms_cached()
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

/* Returns the CUDA launch status. */
cudaError_t launch_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, uint8_t *Q, uint8_t *S,
                            bool sf_tc, cudaStream_t stream)
{
    const int64_t Mrows = sf_tc ? ((M + 127) / 128) * 128 : M;
    const int64_t nseg = (K + 255) / 256;
    const int64_t kgroups = (K / 32 + 3) / 4;
    const int64_t units = Mrows * nseg;
    if (units == 0)
        return cudaSuccess;
    const int64_t per_block = (QTHREADS / 32) * QUNROLL;
    int64_t blocks = (units + per_block - 1) / per_block;
    const int64_t cap = (int64_t)num_sms_cached() * 8 * 4; /* 8 resident blocks x 4 waves */
    if (blocks > cap)
        blocks = cap;
    dim3 grid((unsigned)blocks), block(QTHREADS);
    if (f32_in) {
        if (sf_tc)
            mx_quantize_kernel<true, true><<<grid, block, 0, stream>>>(X, M, K, ldx, Q, S, Mrows, nseg, kgroups);
        else
            mx_quantize_kernel<true, false><<<grid, block, 0, stream>>>(X, M, K, ldx, Q, S, Mrows, nseg, kgroups);
    } else {
        if (sf_tc)
            mx_quantize_kernel<false, true><<<grid, block, 0, stream>>>(X, M, K, ldx, Q, S, Mrows, nseg, kgroups);
        else
            mx_quantize_kernel<false, false><<<grid, block, 0, stream>>>(X, M, K, ldx, Q, S, Mrows, nseg, kgroups);
    }
    return cudaGetLastError();
}

cudaError_t launch_gelu(const void *X, void *Y, int64_t n, cudaStream_t stream)
{
    const int64_t n8 = n / 8;
    if (n8 == 0)
        return cudaSuccess;
    int64_t blocks = (n8 + 255) / 256;
    const int64_t cap = (int64_t)num_sms_cached() * 8 * 4;
    if (blocks > cap)
        blocks = cap;
    gelu_tanh_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(X),
                                                                reinterpret_cast<uint4 *>(Y), n8);
    return cudaGetLastError();
}

} // namespace mx
