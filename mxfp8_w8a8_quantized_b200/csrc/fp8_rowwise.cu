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
 * element, 4 bytes per row.  The row's amax is needed before its first code,
 * so a row is read into on-chip memory once and used twice:
 *  - BF16 activations: one warp per row.  Rows arrive in shared memory by
 *    1-D bulk copies (TMA, two row slots per warp, the next row's copy in
 *    flight while the current one is coded), so the loads in flight do not
 *    depend on how many threads are resident; warps never wait for one
 *    another.  Rows up to 14080 elements (8 warps x one or two slots fit).
 *  - FP32 weights (offline) and longer rows: one CTA per row, the row in
 *    registers, a block reduction.
 * The quotient x / s is formed without a division per element (see
 * rw_quot2), bit-identical to the binary32 division.
 */
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mx_element.cuh"
#include "ptx.cuh"

namespace mx {

constexpr int RW_MAX_K = 16384; /* FP8RW_MAX_K of the C-ABI */

template <bool F32_IN, int NT>
struct RwCfg {
    static constexpr int EPC = F32_IN ? 4 : 8;   /* elements per 16-byte chunk */
    static constexpr int CHUNKS = F32_IN ? 16 : 8; /* chunks per thread, at most */
    static constexpr int MAX_K = CHUNKS * NT * EPC;
};
static_assert(RwCfg<false, 256>::MAX_K == RW_MAX_K && RwCfg<true, 256>::MAX_K == RW_MAX_K, "row fits");

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

__device__ unsigned int g_rw_status = 0; /* bit 0: a bounded wait gave up */

/*
 * RN(a / s) for a pair of binary32 values, given r = RN(1 / s), without a
 * division (Markstein's correction step with a fused multiply-add:
 * P. Markstein, "Computation of elementary functions on the IBM RISC
 * System/6000 processor", IBM J. Res. Dev. 34(1), 1990): q0 = RN(a r) is
 * within an ulp of a / s, so the residual a - q0 s is exact in one FMA, and
 * RN(q0 + (a - q0 s) r) is the correctly rounded quotient.  The step fails
 * for divisors whose significand is all ones; rows with such a scale (and
 * rows whose reciprocal overflows, or whose scale is 0) divide instead (see
 * rw_exact_row).  ns2 holds -s.
 */
__device__ __forceinline__ f32x2 rw_quot2(f32x2 a, f32x2 r2, f32x2 ns2)
{
    const f32x2 q0 = f2_mul(a, r2);
    return f2_fma(f2_fma(q0, ns2, a), r2, q0);
}

/* Rows whose codes take the plain division: s = 0 (all +-0), 1/s not finite,
 * or a significand at or near all ones. */
__device__ __forceinline__ bool rw_exact_row(float s, float rcp)
{
    return s == 0.0f || !(rcp < 3.0e38f) || (__float_as_uint(s) & 0x7FFFFFu) >= 0x7FFFF0u;
}

__device__ __forceinline__ uint32_t rw_e4m3x2(float lo, float hi)
{
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

/* Codes of the two BF16 values of a word (low half first), 16 bits. */
__device__ __forceinline__ uint32_t rw_codes_bf16x2(uint32_t w, f32x2 r2, f32x2 ns2)
{
    float lo, hi;
    f2_unpack(rw_quot2(bf16x2_to_f32x2(w), r2, ns2), lo, hi);
    return rw_e4m3x2(lo, hi);
}

/* The same by plain division (rows of rw_exact_row); s = 0 keeps x (+-0). */
__device__ __forceinline__ uint32_t rw_codes2_div(float a, float b, float s)
{
    return s == 0.0f ? rw_e4m3x2(a, b) : rw_e4m3x2(__fdiv_rn(a, s), __fdiv_rn(b, s));
}

/*
 * BF16 rows, one warp each, staged through shared memory: the warp's `ns`
 * slots hold its next rows, filled by bulk copies that lane 0 issues; a slot
 * is refilled as soon as its row is coded.  Every wait is bounded: on
 * timeout the kernel records it in g_rw_status, waits (bounded) for the
 * copies it still has in flight, and stops.
 */
constexpr int RWB_WARPS = 8;
constexpr uint32_t RWB_SMEM = 220u * 1024u; /* row slots of one CTA */

__device__ __forceinline__ bool rw_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity, 100000u))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity, 100000u))
        if (globaltimer_ns() - t0 > limit_ns)
            return false;
    return true;
}

/* Self-test of rw_wait: a wait on an mbarrier that nothing arrives at gives
 * up after limit_ns; the kernel records it as the quantizer does. */
__global__ void rw_wait_selftest_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        if (!rw_wait(smem_u32(&bar), 0u, limit_ns))
            atomicOr(&g_rw_status, 1u);
    }
}

__global__ void __launch_bounds__(RWB_WARPS * 32, 1) fp8_rowwise_quantize_bulk_kernel(
    const uint16_t *__restrict__ X, int64_t M, int K, int64_t ldx, uint8_t *__restrict__ Q, float *__restrict__ S,
    int ns, uint32_t slot_bytes, unsigned long long timeout_ns)
{
    extern __shared__ __align__(128) uint8_t rw_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = K / 8;
    const uint32_t row_bytes = (uint32_t)K * 2u;
    uint8_t *slots = rw_smem + (size_t)warp * ns * slot_bytes;
    const uint32_t slots_u32 = smem_u32(slots);
    const uint32_t bars = smem_u32(rw_smem + (size_t)RWB_WARPS * ns * slot_bytes) + (uint32_t)warp * ns * 8u;
    const int64_t stride = (int64_t)gridDim.x * RWB_WARPS;
    const int64_t first = (int64_t)blockIdx.x * RWB_WARPS + warp;
    if (lane == 0) {
        for (int s = 0; s < ns; ++s)
            mbar_init(bars + 8u * s, 1);
        fence_mbar_init();
        for (int s = 0; s < ns; ++s) {
            const int64_t r = first + s * stride;
            if (r < M) {
                mbar_arrive_expect_tx(bars + 8u * s, row_bytes);
                bulk_load(slots_u32 + s * slot_bytes, X + r * ldx, row_bytes, bars + 8u * s);
            }
        }
    }
    __syncwarp();
    uint32_t it = 0;
    bool ok = true;
    for (int64_t r = first; r < M; r += stride, ++it) {
        const uint32_t s = it % (uint32_t)ns, bar = bars + 8u * s;
        if (!__all_sync(0xFFFFFFFFu, rw_wait(bar, (it / (uint32_t)ns) & 1u, timeout_ns))) {
            ok = false;
            break;
        }
        const uint4 *row = reinterpret_cast<const uint4 *>(slots + s * slot_bytes);
        uint32_t amax = 0u;
#pragma unroll 4
        for (int c = lane; c < nchunks; c += 32)
            amax = max(amax, rw_amax<false>(row[c]));
        amax = __reduce_max_sync(0xFFFFFFFFu, amax);
        const float sc = __fdiv_rn(__uint_as_float(amax), 448.0f);
        const float rcp = __frcp_rn(sc);
        if (lane == 0)
            S[r] = sc;
        uint2 *qrow = reinterpret_cast<uint2 *>(Q + r * (int64_t)K);
        if (!rw_exact_row(sc, rcp)) {
            const f32x2 r2 = f2_pack(rcp, rcp), ns2 = f2_pack(-sc, -sc);
#pragma unroll 4
            for (int c = lane; c < nchunks; c += 32) {
                const uint4 v = row[c];
                qrow[c] = make_uint2(rw_codes_bf16x2(v.x, r2, ns2) | (rw_codes_bf16x2(v.y, r2, ns2) << 16),
                                     rw_codes_bf16x2(v.z, r2, ns2) | (rw_codes_bf16x2(v.w, r2, ns2) << 16));
            }
        } else {
            for (int c = lane; c < nchunks; c += 32) {
                const uint4 v = row[c];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[i] = rw_codes2_div(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u), sc);
                qrow[c] = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
            }
        }
        __syncwarp(); /* every lane has read the slot */
        if (lane == 0) {
            const int64_t rn = r + (int64_t)ns * stride;
            if (rn < M) {
                mbar_arrive_expect_tx(bar, row_bytes);
                bulk_load(slots_u32 + s * slot_bytes, X + rn * ldx, row_bytes, bar);
            }
        }
    }
    if (!ok && lane == 0) {
        atomicOr(&g_rw_status, 1u);
        /* copies still in flight into this warp's slots: wait for them (bounded) */
        for (uint32_t k = 0; k < (uint32_t)ns; ++k) {
            const uint32_t j = it + k;
            const int64_t r = first + (int64_t)j * stride;
            if (r < M)
                (void)rw_wait(bars + 8u * (j % (uint32_t)ns), (j / (uint32_t)ns) & 1u, timeout_ns);
        }
    }
}

/* Longer rows (and FP32 weights): one CTA per row, a block reduction. */
template <bool F32_IN, int NT>
__global__ void __launch_bounds__(NT) fp8_rowwise_quantize_kernel(const void *__restrict__ X, int64_t M, int K,
                                                                  int64_t ldx, uint8_t *__restrict__ Q,
                                                                  float *__restrict__ S)
{
    using C = RwCfg<F32_IN, NT>;
    __shared__ uint32_t red[2][NT / 32];
    const int nchunks = K / C::EPC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int it = 0;
    for (int64_t r = blockIdx.x; r < M; r += gridDim.x, ++it) {
        const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(X) +
                                                           r * ldx * (F32_IN ? 4 : 2));
        uint4 v[C::CHUNKS];
        uint32_t amax = 0u;
#pragma unroll
        for (int j = 0; j < C::CHUNKS; ++j) {
            const int c = threadIdx.x + j * NT;
            if (c < nchunks) {
                v[j] = __ldcs(row + c);
                amax = max(amax, rw_amax<F32_IN>(v[j]));
            }
        }
        amax = __reduce_max_sync(0xFFFFFFFFu, amax);
        uint32_t *rd = red[it & 1]; /* alternate buffers: one barrier per row */
        if (lane == 0)
            rd[warp] = amax;
        __syncthreads();
        amax = rd[0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w)
            amax = max(amax, rd[w]);
        const float s = __fdiv_rn(__uint_as_float(amax), 448.0f);
        const float rcp = __frcp_rn(s);
        const bool exact_row = rw_exact_row(s, rcp);
        const f32x2 r2 = f2_pack(rcp, rcp), ns2 = f2_pack(-s, -s);
        if (threadIdx.x == 0)
            S[r] = s;
        uint8_t *qrow = Q + r * (int64_t)K;
#pragma unroll
        for (int j = 0; j < C::CHUNKS; ++j) {
            const int c = threadIdx.x + j * NT;
            if (c >= nchunks)
                continue;
            if constexpr (F32_IN) {
                uint32_t lo, hi;
                if (!exact_row) {
                    float a, b, d, e;
                    f2_unpack(rw_quot2(f2_pack(__uint_as_float(v[j].x), __uint_as_float(v[j].y)), r2, ns2), a, b);
                    f2_unpack(rw_quot2(f2_pack(__uint_as_float(v[j].z), __uint_as_float(v[j].w)), r2, ns2), d, e);
                    lo = rw_e4m3x2(a, b);
                    hi = rw_e4m3x2(d, e);
                } else {
                    lo = rw_codes2_div(__uint_as_float(v[j].x), __uint_as_float(v[j].y), s);
                    hi = rw_codes2_div(__uint_as_float(v[j].z), __uint_as_float(v[j].w), s);
                }
                reinterpret_cast<uint32_t *>(qrow)[c] = lo | (hi << 16);
            } else {
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[i] = !exact_row ? rw_codes_bf16x2(w[i], r2, ns2)
                                      : rw_codes2_div(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u), s);
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
 * K <= 16384; waits give up after timeout_ns.  Returns the launch status. */
cudaError_t launch_fp8_rowwise_quantize(const void *X, bool f32_in, int64_t M, int64_t K, int64_t ldx, uint8_t *Q,
                                        float *S, cudaStream_t stream, unsigned long long timeout_ns)
{
    if (M == 0)
        return cudaSuccess;
    const uint32_t slot = ((uint32_t)K * 2u + 127u) & ~127u;
    const int ns = (int)(RWB_SMEM / (RWB_WARPS * slot)) >= 2 ? 2 : (int)(RWB_SMEM / (RWB_WARPS * slot));
    if (!f32_in && ns >= 1) {
        const uint32_t smem = (uint32_t)RWB_WARPS * ns * slot + RWB_WARPS * ns * 8u;
        static int attr_set[64] = {0};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess)
            return cudaErrorInvalidDevice;
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            cudaError_t e = cudaFuncSetAttribute(fp8_rowwise_quantize_bulk_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)(RWB_SMEM + RWB_WARPS * 2 * 8));
            if (e != cudaSuccess)
                return e;
            attr_set[dev] = 1;
        }
        int64_t blocks = (M + RWB_WARPS - 1) / RWB_WARPS;
        if (blocks > rw_num_sms())
            blocks = rw_num_sms(); /* one CTA per SM; its warps walk the rows */
        fp8_rowwise_quantize_bulk_kernel<<<(unsigned)blocks, RWB_WARPS * 32, smem, stream>>>(
            static_cast<const uint16_t *>(X), M, (int)K, ldx, Q, S, ns, slot, timeout_ns);
        return cudaGetLastError();
    }
    int64_t blocks = (int64_t)rw_num_sms() * 8;
    if (blocks > M)
        blocks = M;
    if (f32_in)
        fp8_rowwise_quantize_kernel<true, 256><<<(unsigned)blocks, 256, 0, stream>>>(X, M, (int)K, ldx, Q, S);
    else
        fp8_rowwise_quantize_kernel<false, 256><<<(unsigned)blocks, 256, 0, stream>>>(X, M, (int)K, ldx, Q, S);
    return cudaGetLastError();
}

/* Reads and clears the row-wise quantizer's status word (synchronous). */
cudaError_t launch_rw_wait_selftest(unsigned long long limit_ns, cudaStream_t stream)
{
    rw_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t read_and_clear_rw_status(unsigned int *out)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_rw_status, sizeof(unsigned int));
    if (e != cudaSuccess)
        return e;
    return cudaMemcpyToSymbol(g_rw_status, &zero, sizeof(unsigned int));
}

} // namespace mx
