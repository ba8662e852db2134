/*
 * mx_element.cuh -- per-element MX arithmetic shared by the stand-alone
 * quantizer / GELU kernels and the GEMM epilogue that quantizes its own
 * output.  Both call sites must round identically (the fused path is
 * checked bit for bit against GEMM -> GELU -> quantize), so the arithmetic
 * lives here once and is written with explicitly rounded operations where
 * the compiler could otherwise contract a multiply and an add.
 *
 * Scale rule (model card "Wan2.2-I2V-A14B-Lightning . MXFP8 (AutoRound
 * OptRTN)", "Coverage per transformer": E4M3 codes, one E8M0 scale per 32
 * elements; exponent rule of the OCP MX format): e = floor(log2 amax) - 8,
 * clamped to the E8M0 minimum -127; codes = E4M3(x * 2^-e), round to
 * nearest even, saturating at +-448; a block holding Inf/NaN gets scale
 * byte 0xFF and codes 0x7F.
 */
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

namespace mx {

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

/* Pairs of binary32 values in one 64-bit register, operated on by the
 * packed f32x2 instructions of sm_100: each lane is rounded exactly like the
 * scalar operation (round to nearest even, subnormals kept), at half the
 * instruction count. */
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 f2_pack(float lo, float hi)
{
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(f32x2 v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

/* The two BF16 values of a word (low half first) as binary32 (exact). */
__device__ __forceinline__ f32x2 bf16x2_to_f32x2(uint32_t w)
{
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

/* Both lanes rounded to BF16 (nearest even), packed low lane first. */
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(f32x2 v)
{
    float lo, hi;
    f2_unpack(v, lo, hi);
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&b);
}

/* 2^a (a <= 0), the hardware's approximation (relative error about 2^-22);
 * results below 2^-126 flush to zero. */
__device__ __forceinline__ float exp2_approx_ftz(float a)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
    return r;
}

/* 1/a for a in [1, 2], the hardware's approximation (relative error about
 * 2^-23). */
__device__ __forceinline__ float rcp_approx_ftz(float a)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
    return r;
}

/*
 * GELU, tanh form, of the two BF16 values of a word, rounded to BF16:
 *   gelu(x) = 0.5 x (1 + tanh(u)) = x sigmoid(2u),  u = sqrt(2/pi) (x + 0.044715 x^3)
 *           = x / (1 + t)      for u >= 0,
 *           = x t / (1 + t)    for u < 0,        t = e^(-2|u|) = 2^(-2|u| log2 e).
 * -2u log2 e is formed as x (K3 x^2 + K2), and t is taken as
 * 2^(64 - 2|u| log2 e) * 2^-64 so that the hardware exp2 never returns a
 * subnormal: for very negative x the result underflows gradually, in the
 * final products, instead of flushing to -0.  Over all finite BF16 inputs the
 * relative error before the final rounding is below 2^-17 (largest near
 * x = -8, where the rounding of the exponent's argument is magnified), far
 * below a BF16 ulp (2^-8).  Every operation is a single instruction, so all
 * callers get the same bits.
 */
__device__ __forceinline__ uint32_t gelu_tanh_bf16x2(uint32_t w)
{
    const float K2 = -2.302208185195923f;   /* -2 sqrt(2/pi) log2(e) */
    const float K3 = -0.10294324159622192f; /* -2 sqrt(2/pi) 0.044715 log2(e) */
    const f32x2 x = bf16x2_to_f32x2(w);
    const f32x2 ar = f2_mul(x, f2_fma(f2_mul(x, x), f2_pack(K3, K3), f2_pack(K2, K2))); /* -2u log2 e */
    float a0, a1;
    f2_unpack(ar, a0, a1);
    float s0, s1;
    f2_unpack(f2_add(f2_pack(-fabsf(a0), -fabsf(a1)), f2_pack(64.0f, 64.0f)), s0, s1);
    const f32x2 t64 = f2_pack(exp2_approx_ftz(s0), exp2_approx_ftz(s1)); /* t 2^64 */
    const f32x2 m64 = f2_pack(5.421010862427522e-20f, 5.421010862427522e-20f); /* 2^-64 */
    const f32x2 d = f2_fma(t64, m64, f2_pack(1.0f, 1.0f));                   /* 1 + t */
    const f32x2 xt = f2_mul(f2_mul(x, t64), m64);                            /* x t */
    float x0, x1, y0, y1, d0, d1;
    f2_unpack(x, x0, x1);
    f2_unpack(xt, y0, y1);
    f2_unpack(d, d0, d1);
    /* u >= 0 exactly when -2u log2 e carries a sign bit (or is +0 from x = -0,
     * where both forms give -0) */
    const float n0 = (__float_as_uint(a0) >> 31) ? x0 : y0;
    const float n1 = (__float_as_uint(a1) >> 31) ? x1 : y1;
    return f32x2_to_bf16x2(f2_mul(f2_pack(n0, n1), f2_pack(rcp_approx_ftz(d0), rcp_approx_ftz(d1))));
}

} // namespace mx
