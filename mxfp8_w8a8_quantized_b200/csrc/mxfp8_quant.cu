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
 * written per element.  Each warp walks whole rows in segments of 512
 * elements: every lane loads 16 consecutive elements with two 128-bit loads
 * (fully coalesced), two lanes form one 32-block and combine their amax with
 * one shuffle, each lane writes its 16 codes with one 16-byte store
 * (coalesced 512 B per warp), and scales are gathered into 32-bit words
 * written straight into the tensor-core scale layout (see include/mxfp8.h).
 * Two segments are loaded before either is processed, keeping four 16-byte
 * loads in flight per thread.  At the SM clocks of a power-capped GPU the
 * kernel is close to bound by its integer instructions, so every address in a
 * row is the row's base plus a multiple of the segment, and the block amax
 * and the scaling run on the floating-point pipe, two elements at a time.
 */
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_element.cuh"

namespace mx {

constexpr int QTHREADS = 256;
constexpr int QUNROLL = 2;              /* row segments in flight per warp */

/* 16 consecutive elements of one row: one lane's share of a row segment. */
template <bool F32_IN>
struct Seg16 {
    uint4 v[F32_IN ? 4 : 2];
};

/* the 16 elements of a row starting at element k0 (streaming loads) */
template <bool F32_IN>
__device__ __forceinline__ void load_seg16(Seg16<F32_IN> &s, const uint8_t *row, int k0)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(row + (int64_t)k0 * (F32_IN ? 4 : 2));
#pragma unroll
    for (int i = 0; i < (F32_IN ? 4 : 2); ++i)
        s.v[i] = __ldcs(p + i);
}

/* max(|a|, |b|) of each BF16 half, two elements per instruction on the
 * floating-point pipe (the integer pipe bounds this kernel at reduced SM
 * clocks); the sign is the xor of the signs, a NaN gives the canonical NaN */
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

/* max |x| of the 16 elements, as the bit pattern of a binary32 (sign cleared) */
template <bool F32_IN>
__device__ __forceinline__ uint32_t amax_seg16(const Seg16<F32_IN> &s)
{
    if constexpr (F32_IN) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m = max(m, s.v[i].x & 0x7FFFFFFFu);
            m = max(m, s.v[i].y & 0x7FFFFFFFu);
            m = max(m, s.v[i].z & 0x7FFFFFFFu);
            m = max(m, s.v[i].w & 0x7FFFFFFFu);
        }
        return m;
    } else {
        /* per half, the largest magnitude (a NaN anywhere gives the canonical
         * NaN, whose exponent field marks the block as non-finite) */
        const uint32_t a = absmax_bf16x2(s.v[0].x, s.v[0].y);
        const uint32_t b = absmax_bf16x2(s.v[0].z, s.v[0].w);
        const uint32_t c = absmax_bf16x2(s.v[1].x, s.v[1].y);
        const uint32_t d = absmax_bf16x2(s.v[1].z, s.v[1].w);
        const uint32_t m = absmax_bf16x2(absmax_bf16x2(a, b), absmax_bf16x2(c, d)) & 0x7FFF7FFFu;
        /* non-negative BF16 bit patterns order like the values */
        return max(m << 16, m & 0xFFFF0000u);
    }
}

/* 16 elements times 2^-e (exact) -> 16 E4M3 codes; `sb` is the block's
 * finite scale byte (e = sb - 127, sb <= 246).  The BF16 path multiplies
 * pairs with one packed binary32 instruction (each lane rounded like the
 * scalar multiply, which is exact here). */
template <bool F32_IN>
__device__ __forceinline__ uint4 codes_seg16(const Seg16<F32_IN> &s, uint32_t sb)
{
    uint32_t out[4];
    if constexpr (F32_IN) {
        const float m = inv_scale(sb);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            out[i] = pack4_e4m3(__uint_as_float(s.v[i].x) * m, __uint_as_float(s.v[i].y) * m,
                                __uint_as_float(s.v[i].z) * m, __uint_as_float(s.v[i].w) * m);
    } else {
        const float m = inv_scale(sb);
        const f32x2 mm = f2_pack(m, m);
        const uint32_t w[8] = {s.v[0].x, s.v[0].y, s.v[0].z, s.v[0].w, s.v[1].x, s.v[1].y, s.v[1].z, s.v[1].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float c0, c1, c2, c3;
            f2_unpack(f2_mul(bf16x2_to_f32x2(w[2 * i]), mm), c0, c1);
            f2_unpack(f2_mul(bf16x2_to_f32x2(w[2 * i + 1]), mm), c2, c3);
            out[i] = pack4_e4m3(c0, c1, c2, c3);
        }
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

/*
 * X [M, K] (row stride ldx elements) -> Q [M, K] codes, S scales.
 * Each warp walks whole rows (rows warp, warp + nwarps, ...), two 512-element
 * segments at a time; lane l covers elements 16l .. 16l+15 of a segment, so
 * lanes 2b and 2b+1 hold block b.  Every address of a row is its base plus a
 * multiple of the segment.  Rows r in [M, Mrows) only write zero scale
 * padding (tensor-core layout).
 */
template <bool F32_IN, bool SF_TC>
__global__ void __launch_bounds__(QTHREADS, 1) mx_quantize_kernel(const void *__restrict__ X, int64_t M,
                                                                              int64_t K, int64_t ldx,
                                                                              uint8_t *__restrict__ Q,
                                                                              uint8_t *__restrict__ S, int64_t Mrows,
                                                                              int64_t nseg, int64_t kgroups)
{
    const int lane = threadIdx.x & 31;
    const int warp0 = (int)((blockIdx.x * QTHREADS + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * QTHREADS) >> 5);
    const int nblocks = (int)(K >> 5);
    const int M32 = (int)M, K32 = (int)K, nseg32 = (int)nseg, Mrows32 = (int)Mrows;
    constexpr int EB = F32_IN ? 4 : 2;

    for (int r = warp0; r < Mrows32; r += nwarps) {
        const bool row_ok = r < M32;
        const uint8_t *xrow = reinterpret_cast<const uint8_t *>(X) + (int64_t)r * ldx * EB;
        uint8_t *qrow = Q + (int64_t)r * K;
        uint8_t *srow = SF_TC ? S + ((((int64_t)(r >> 7)) * kgroups) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2)
                              : S + (int64_t)r * nblocks;
        for (int j = 0; j < nseg32; j += QUNROLL) {
            Seg16<F32_IN> seg[QUNROLL];
            int k0[QUNROLL];
            bool valid[QUNROLL];
#pragma unroll
            for (int i = 0; i < QUNROLL; ++i) {
                k0[i] = (j + i) * 512 + lane * 16;
                valid[i] = row_ok && (j + i < nseg32) && (k0[i] < K32);
                if (valid[i])
                    load_seg16<F32_IN>(seg[i], xrow, k0[i]);
            }
#pragma unroll
            for (int i = 0; i < QUNROLL; ++i) {
                if (j + i >= nseg32) /* warp-uniform */
                    break;
                uint32_t amax = valid[i] ? amax_seg16<F32_IN>(seg[i]) : 0u;
                amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
                const uint32_t sb = valid[i] ? scale_byte_from_amax(amax) : 0u;
                if (valid[i]) {
                    const uint4 out = (sb == 0xFFu) ? make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu)
                                                    : codes_seg16<F32_IN>(seg[i], sb);
                    *reinterpret_cast<uint4 *>(qrow + k0[i]) = out;
                }
                if constexpr (SF_TC) {
                    /* word g (lanes 8g .. 8g+7) = blocks 16(j+i) + 4g .. 16(j+i) + 4g + 3 */
                    const uint32_t w = sb | (__shfl_down_sync(0xFFFFFFFFu, sb, 2) << 8) |
                                       (__shfl_down_sync(0xFFFFFFFFu, sb, 4) << 16) |
                                       (__shfl_down_sync(0xFFFFFFFFu, sb, 6) << 24);
                    const int kb = (j + i) * 16 + (lane >> 1); /* first block of this word */
                    if ((lane & 7) == 0 && kb < nblocks)
                        *reinterpret_cast<uint32_t *>(srow + ((int64_t)(kb >> 2) << 9)) = w;
                } else {
                    if (valid[i] && (lane & 1) == 0)
                        srow[k0[i] >> 5] = (uint8_t)sb;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ GELU */
__global__ void __launch_bounds__(256) gelu_tanh_bf16_kernel(const uint4 *__restrict__ X, uint4 *__restrict__ Y,
                                                             int64_t n8)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = X[i];
        const uint32_t w[4] = {gelu_tanh_bf16x2(v.x), gelu_tanh_bf16x2(v.y), gelu_tanh_bf16x2(v.z),
                               gelu_tanh_bf16x2(v.w)};
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
    const int64_t nseg = (K + 511) / 512;
    const int64_t kgroups = (K / 32 + 3) / 4;
    const int64_t units = Mrows * nseg;
    if (units == 0)
        return cudaSuccess;
    const int64_t per_block = QTHREADS / 32; /* rows per block */
    int64_t blocks = (Mrows + per_block - 1) / per_block;
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
