/*
 * mxfp8_oracle.c -- CPU oracle for the MXFP8 W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path loads this library:
 * only tests/, the smoke check of __graft_entry__ and the cpu_baseline leg of
 * bench.py call it.  It shares no code, header, table or constant with the
 * CUDA path; every value here is built from the bit-level definitions of the
 * formats, in double precision.
 *
 * What it computes, and the passage each step follows:
 *
 *  [MC] = model card "Wan2.2-I2V-A14B-Lightning . MXFP8 (AutoRound OptRTN)"
 *         (huggingface.co/intel-ai/Wan2.2-I2V-A14B-Lightning-Diffusers-MXFP8-AutoRound)
 *    - SS "Quantization Details", quantization_config.json: bits 8, data_type
 *      mx_fp, group_size 32, sym true; act_bits 8, act_data_type mx_fp,
 *      act_group_size 32, act_sym true, act_dynamic true.
 *    - SS "Coverage per transformer": weights are FP8 E4M3 codes with one
 *      E8M0 scale per 32 elements; activations are quantized to MXFP8
 *      dynamically at run time; the quantized linears keep F16 biases.
 *  [LQ] = "Model Quantization Techniques" (LightX2V quantization.md),
 *         SS "MiniMax-H3 Video VAE Encoder Conv3D": 448 is the E4M3 qmax used
 *         with FP32 accumulation.
 *
 * Readings (the pages name the format but do not spell out its arithmetic):
 *  - E4M3 is the OCP 8-bit float with 4 exponent bits (bias 7), 3 mantissa
 *    bits, no infinities, S.1111.111 = NaN, largest finite 448.
 *  - The shared scale of a 32-element block is 2^e with
 *    e = floor(log2(amax)) - 8 (the OCP Microscaling v1.0 rule; 8 is the
 *    exponent of the largest E4M3 binade), clamped to the E8M0 range
 *    [-127, 127] and stored as the byte e + 127.  amax == 0 gives e = -127.
 *  - Elements are x / 2^e rounded to the nearest E4M3 value, ties to the even
 *    mantissa, magnitudes >= 448 saturating to 448 (never NaN); the sign is
 *    kept, so negative values that round to zero give -0 (0x80).
 *  - A block holding Inf or NaN gets scale byte 0xFF and all codes 0x7F.
 *  - The layer output is Y = Xhat * What^T + bias with the dequantized
 *    operands, summed exactly (FP64 here), bias widened from F16; the BF16
 *    output is that value rounded to nearest-even.
 *  - GELU between the two FFN linears is the tanh form
 *    0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
 *
 * Per-channel FP8 (the "fp8-vllm" / "fp8-sgl" modes of [LQ] SS "Quantization
 * Modes": FP8 channel-symmetric weights, FP8 channel-dynamic symmetric
 * activations; SS "MiniMax-H3 FP8 with FP16 Accumulation": activations use
 * dynamic row-wise quantization with scale = max(abs(x)) / qmax; qmax is 448
 * with FP32 accumulation, SS "MiniMax-H3 Video VAE Encoder Conv3D"; the
 * LightX2V Wan2.2 FP8 checkpoints keep "per-output-channel FP32 scales",
 * page "Wan2.2 I2V A14B, four-step 720p: native LightX2V FP8 and NVFP4",
 * SS "Conversion and compatibility"):
 *  - one FP32 scale per activation row (token) and per weight row (output
 *    channel): s = amax / 448, a binary32 division of the row's largest
 *    magnitude (the pages give the scales as FP32);
 *  - codes are E4M3(x / s) with x / s a binary32 division, rounded to nearest
 *    even and saturating at 448 as above; a row of zeros has s = 0 and codes
 *    of +-0;
 *  - Y = s_x[m] s_w[n] sum_k xq[m,k] wq[n,k] + bias[n], exact (FP64 here).
 *
 * NVFP4 (page "Wan2.2 I2V A14B, four-step 720p: native LightX2V FP8 and
 * NVFP4", SS "Conversion and compatibility": packed E2M1 weights with E4M3
 * block scales, plus FP32 input_global_scale and alpha fields; weights
 * enter the quantizer as BF16).  The pages name the fields, not the
 * arithmetic; readings:
 *  - E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 *    0, 0.5, 1, 1.5, 2, 3, 4, 6; nearest, ties to the even mantissa,
 *    saturating at 6.  Two codes per byte, the lower-index element in the
 *    low nibble.
 *  - blocks of 16 consecutive K elements share one scale byte, an E4M3
 *    value used unsigned (UE4M3); one FP32 global scale g per tensor.
 *  - per block: s = UE4M3(RN(amax * RN(g / 6))) (nearest even, saturating
 *    at 448); elements E2M1(RN(x * RN(g / dec(s)))), all in binary32; a
 *    block whose scale is 0 gets codes +-0.
 *  - dequantized value q dec(s) / g; the layer Y = alpha sum_k qx sx qw sw
 *    + bias with alpha = 1 / (g_x g_w), exact here.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Scalar formats                                                      */
/* ------------------------------------------------------------------ */

/* E4M3: value of one 8-bit code. */
double orc_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int E = (c >> 3) & 0xF;
    int m = c & 0x7;
    double mag;
    if (E == 15 && m == 7)
        return NAN;
    if (E == 0)
        mag = ldexp((double)m, -9); /* subnormal: (m/8) * 2^(1-7) */
    else
        mag = ldexp((double)(8 + m), E - 10); /* (1 + m/8) * 2^(E-7) */
    return s ? -mag : mag;
}

/* The 127 finite non-negative magnitudes, codes 0x00..0x7E, increasing. */
static double e4m3_mag[127];
static int e4m3_mag_ready = 0;

static void e4m3_table_init(void)
{
    if (e4m3_mag_ready)
        return;
    for (int c = 0; c <= 0x7E; ++c)
        e4m3_mag[c] = orc_e4m3_decode((uint8_t)c);
    e4m3_mag_ready = 1;
}

/* E4M3: nearest code to a real v, ties to even mantissa, saturating. */
uint8_t orc_e4m3_encode(double v)
{
    e4m3_table_init();
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= e4m3_mag[0x7E])
        return sign | 0x7E;
    /* binary search: lo = largest code with magnitude <= a */
    int lo = 0, hi = 0x7E;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_mag[mid] <= a)
            lo = mid;
        else
            hi = mid;
    }
    /* now e4m3_mag[lo] <= a < e4m3_mag[lo + 1] */
    double below = a - e4m3_mag[lo];
    double above = e4m3_mag[lo + 1] - a;
    int pick;
    if (below < above)
        pick = lo;
    else if (above < below)
        pick = lo + 1;
    else
        pick = (lo & 1) ? lo + 1 : lo; /* the code's lsb is the mantissa lsb */
    return sign | (uint8_t)pick;
}

/* E8M0 scale byte -> 2^(byte-127); 0xFF is NaN. */
double orc_e8m0_decode(uint8_t b)
{
    if (b == 0xFF)
        return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* BF16 is the upper half of an IEEE binary32. */
double orc_bf16_decode(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
double orc_f16_decode(uint16_t h)
{
    int s = (h >> 15) & 1;
    int E = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double mag;
    if (E == 31)
        mag = m ? NAN : INFINITY;
    else if (E == 0)
        mag = ldexp((double)m, -24);
    else
        mag = ldexp((double)(1024 + m), E - 25);
    return s ? -mag : mag;
}

/* Real -> BF16 bits, round to nearest, ties to even (8 significant bits). */
uint16_t orc_bf16_rne(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return sign | 0x7F80;
    int ex;
    frexp(a, &ex);      /* a in [2^(ex-1), 2^ex) */
    int E = ex - 1;     /* unbiased exponent of a */
    if (E < -126)
        E = -126;       /* subnormal range: fixed quantum 2^-133 */
    double m = rint(ldexp(a, 7 - E)); /* significand in units of 2^(E-7), RNE */
    if (m >= 256.0) {   /* rounded up into the next binade */
        m = 128.0;
        E += 1;
    }
    if (E > 127)
        return sign | 0x7F80;
    uint16_t bits;
    if (m >= 128.0)
        bits = (uint16_t)(((E + 127) << 7) | ((int)m - 128));
    else
        bits = (uint16_t)m; /* subnormal (E == -126) */
    return sign | bits;
}

/* ------------------------------------------------------------------ */
/* MX block quantization                                               */
/* ------------------------------------------------------------------ */

/* One block of n (= 32) values: scale byte and n codes. */
static void quantize_block(const double *x, int n, uint8_t *codes, uint8_t *scale)
{
    double amax = 0.0;
    int nonfinite = 0;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(x[i]))
            nonfinite = 1;
        else if (fabs(x[i]) > amax)
            amax = fabs(x[i]);
    }
    if (nonfinite) {
        *scale = 0xFF;
        for (int i = 0; i < n; ++i)
            codes[i] = 0x7F;
        return;
    }
    int e;
    if (amax == 0.0) {
        e = -127;
    } else {
        int ex;
        frexp(amax, &ex); /* floor(log2(amax)) = ex - 1 */
        e = (ex - 1) - 8;
        if (e < -127)
            e = -127;
        if (e > 127)
            e = 127;
    }
    *scale = (uint8_t)(e + 127);
    for (int i = 0; i < n; ++i)
        codes[i] = orc_e4m3_encode(ldexp(x[i], -e)); /* exact power-of-two scaling */
}

/* Public single-block entry (tests). */
void orc_quantize_block_f64(const double *x, int n, uint8_t *codes, uint8_t *scale)
{
    e4m3_table_init();
    quantize_block(x, n, codes, scale);
}

/*
 * Rows of BF16 activations X[rows, K] (row stride ldx elements) ->
 * codes[rows, K] and scales[rows, K/32] (row-major).  K % 32 == 0.
 */
void orc_quantize_bf16(const uint16_t *x, int64_t rows, int64_t K, int64_t ldx,
                       uint8_t *codes, uint8_t *scales)
{
    e4m3_table_init();
    int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double blk[32];
        for (int64_t b = 0; b < nb; ++b) {
            for (int i = 0; i < 32; ++i)
                blk[i] = orc_bf16_decode(x[r * ldx + b * 32 + i]);
            quantize_block(blk, 32, codes + r * K + b * 32, scales + r * nb + b);
        }
    }
}

/* Same for FP32 weights W[rows, K] (offline RTN quantization). */
void orc_quantize_f32(const float *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales)
{
    e4m3_table_init();
    int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double blk[32];
        for (int64_t b = 0; b < nb; ++b) {
            for (int i = 0; i < 32; ++i)
                blk[i] = (double)w[r * K + b * 32 + i];
            quantize_block(blk, 32, codes + r * K + b * 32, scales + r * nb + b);
        }
    }
}

/* Dequantize codes[rows, K] with row-major scales[rows, K/32] into FP64. */
void orc_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K, double *out)
{
    int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = orc_e4m3_decode(codes[r * K + k]) * orc_e8m0_decode(scales[r * nb + k / 32]);
}

/* ------------------------------------------------------------------ */
/* Linear layer                                                        */
/* ------------------------------------------------------------------ */

/*
 * Y[i, j] = sum_k Xhat[row_i, k] * What[col_j, k] + bias[col_j]   (FP64)
 *
 * Xhat / What are the dequantized operands (codes times their block's
 * scale).  X codes are [M, K] with row-major scales [M, K/32]; W codes are
 * [N, K] (out x in, K contiguous) with row-major scales [N, K/32].  bias is
 * F16 bits [N] or NULL.  rows / cols select which outputs to form (NULL =
 * all); Y is [nr, nc] row-major.
 */
void orc_linear(const uint8_t *xq, const uint8_t *xs, int64_t M, int64_t K,
                const uint8_t *wq, const uint8_t *ws, int64_t N, const uint16_t *bias,
                const int64_t *rows, int64_t nr, const int64_t *cols, int64_t nc, double *Y)
{
    (void)M;
    (void)N;
    int64_t nb = K / 32;
    /* What for the selected output columns, one dequantized row per column */
    double *wd = (double *)malloc((size_t)nc * (size_t)K * sizeof(double));
    if (!wd)
        return;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nc; ++j) {
        int64_t n = cols ? cols[j] : j;
        for (int64_t k = 0; k < K; ++k)
            wd[j * K + k] = orc_e4m3_decode(wq[n * K + k]) * orc_e8m0_decode(ws[n * nb + k / 32]);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nr; ++i) {
        int64_t r = rows ? rows[i] : i;
        double *xd = (double *)malloc((size_t)K * sizeof(double));
        if (!xd)
            continue;
        for (int64_t k = 0; k < K; ++k)
            xd[k] = orc_e4m3_decode(xq[r * K + k]) * orc_e8m0_decode(xs[r * nb + k / 32]);
        for (int64_t j = 0; j < nc; ++j) {
            int64_t n = cols ? cols[j] : j;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += xd[k] * wd[j * K + k];
            if (bias)
                acc += orc_f16_decode(bias[n]);
            Y[i * nc + j] = acc;
        }
        free(xd);
    }
    free(wd);
}

/*
 * The same linear layer with FP32 accumulation in increasing k (one FP32
 * rounding per addition, then the F16 bias added in FP32): one admissible
 * evaluation order of the layer's FP32 accumulation.  Each product of two
 * E4M3 values and two powers of two is exact in FP32 for the scale ranges
 * of real data.  Used to measure how far two valid evaluations of a chain of
 * layers drift apart.
 */
void orc_linear_f32acc(const uint8_t *xq, const uint8_t *xs, int64_t M, int64_t K,
                       const uint8_t *wq, const uint8_t *ws, int64_t N, const uint16_t *bias,
                       const int64_t *rows, int64_t nr, const int64_t *cols, int64_t nc, double *Y)
{
    (void)M;
    (void)N;
    int64_t nb = K / 32;
    double *wd = (double *)malloc((size_t)nc * (size_t)K * sizeof(double));
    if (!wd)
        return;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nc; ++j) {
        int64_t n = cols ? cols[j] : j;
        for (int64_t k = 0; k < K; ++k)
            wd[j * K + k] = orc_e4m3_decode(wq[n * K + k]) * orc_e8m0_decode(ws[n * nb + k / 32]);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nr; ++i) {
        int64_t r = rows ? rows[i] : i;
        double *xd = (double *)malloc((size_t)K * sizeof(double));
        if (!xd)
            continue;
        for (int64_t k = 0; k < K; ++k)
            xd[k] = orc_e4m3_decode(xq[r * K + k]) * orc_e8m0_decode(xs[r * nb + k / 32]);
        for (int64_t j = 0; j < nc; ++j) {
            int64_t n = cols ? cols[j] : j;
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k)
                acc = acc + (float)(xd[k] * wd[j * K + k]);
            if (bias)
                acc = acc + (float)orc_f16_decode(bias[n]);
            Y[i * nc + j] = (double)acc;
        }
        free(xd);
    }
    free(wd);
}

/* FP64 values -> BF16 bits (RNE), elementwise. */
void orc_bf16_rne_array(const double *v, int64_t n, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_bf16_rne(v[i]);
}

/* ------------------------------------------------------------------ */
/* GELU (tanh form) between ffn.net.0.proj and ffn.net.2               */
/* ------------------------------------------------------------------ */

/*
 * 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3), evaluated through
 * the identity 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)): the same function,
 * without the cancellation of 1 + tanh(u) for very negative x.
 */
double orc_gelu_tanh(double x)
{
    const double c = sqrt(2.0 / M_PI);
    double u = c * (x + 0.044715 * x * x * x);
    return x / (1.0 + exp(-2.0 * u));
}

/* BF16 in -> GELU in FP64 -> BF16 out (RNE). */
void orc_gelu_tanh_bf16(const uint16_t *x, int64_t n, uint16_t *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        y[i] = orc_bf16_rne(orc_gelu_tanh(orc_bf16_decode(x[i])));
}

/* ------------------------------------------------------------------ */
/* Per-channel FP8: one FP32 scale per row                             */
/* ------------------------------------------------------------------ */

/*
 * One row of K binary32 values -> E4M3 codes and the row's FP32 scale
 * s = amax / 448.  Both the scale and the quotients x / s are binary32
 * divisions (IEEE, round to nearest even); the quotient then goes to the
 * E4M3 encoder, which rounds it to nearest even and saturates at 448.
 */
static void quantize_row_f32(const float *x, int64_t K, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(x[k]);
        if (a > amax)
            amax = a;
    }
    volatile float s = amax / 448.0f; /* binary32 division */
    *scale = s;
    for (int64_t k = 0; k < K; ++k) {
        if (s == 0.0f) {
            codes[k] = orc_e4m3_encode(x[k]); /* +-0 */
        } else {
            volatile float q = x[k] / s;  /* binary32 division */
            codes[k] = orc_e4m3_encode((double)q);
        }
    }
}

/* BF16 activations [rows, K] (row stride ldx) -> codes [rows, K], FP32 scales [rows]. */
void orc_quantize_rowwise_bf16(const uint16_t *x, int64_t rows, int64_t K, int64_t ldx, uint8_t *codes,
                               float *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float *row = (float *)malloc((size_t)K * sizeof(float));
        if (!row)
            continue;
        for (int64_t k = 0; k < K; ++k)
            row[k] = (float)orc_bf16_decode(x[r * ldx + k]);
        quantize_row_f32(row, K, codes + r * K, scales + r);
        free(row);
    }
}

/* FP32 weights [rows, K] -> codes [rows, K], FP32 scales [rows] (one per output channel). */
void orc_quantize_rowwise_f32(const float *w, int64_t rows, int64_t K, uint8_t *codes, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        quantize_row_f32(w + r * K, K, codes + r * K, scales + r);
}

/*
 * Per-channel FP8 linear: Y[i, j] = sx[m] sw[n] sum_k dec(xq[m,k]) dec(wq[n,k])
 * + bias[n] (m = rows[i], n = cols[j]), exact in FP64.
 */
void orc_linear_rowwise(const uint8_t *xq, const float *sx, int64_t M, int64_t K, const uint8_t *wq,
                        const float *sw, int64_t N, const uint16_t *bias, const int64_t *rows, int64_t nr,
                        const int64_t *cols, int64_t nc, double *Y)
{
    (void)M;
    (void)N;
    double *wd = (double *)malloc((size_t)nc * (size_t)K * sizeof(double));
    if (!wd)
        return;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nc; ++j) {
        int64_t n = cols ? cols[j] : j;
        for (int64_t k = 0; k < K; ++k)
            wd[j * K + k] = orc_e4m3_decode(wq[n * K + k]);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nr; ++i) {
        int64_t r = rows ? rows[i] : i;
        for (int64_t j = 0; j < nc; ++j) {
            int64_t n = cols ? cols[j] : j;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += orc_e4m3_decode(xq[r * K + k]) * wd[j * K + k];
            acc = acc * (double)sx[r] * (double)sw[n];
            if (bias)
                acc += orc_f16_decode(bias[n]);
            Y[i * nc + j] = acc;
        }
    }
    free(wd);
}

/* ------------------------------------------------------------------ */
/* NVFP4: E2M1 elements, UE4M3 scales per 16, FP32 global scale        */
/* ------------------------------------------------------------------ */

/* E2M1: value of one 4-bit code (bit 3 sign, bits 2-1 exponent, bit 0 mantissa). */
double orc_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1;
    int E = (c >> 1) & 3;
    int m = c & 1;
    double mag = E == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, E - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 code, ties to the even mantissa, magnitudes >= 6 -> 6. */
uint8_t orc_e2m1_encode(double v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs(v);
    if (isnan(v))
        return 7; /* out of contract: never produced for finite inputs */
    if (a >= 6.0)
        return sign | 7; /* saturate (far above 6 the distances below would tie) */
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        double dc = fabs(orc_e2m1_decode((uint8_t)c) - a), db = fabs(orc_e2m1_decode((uint8_t)best) - a);
        if (dc < db || (dc == db && (c & 1) == 0))
            best = c;
    }
    return sign | (uint8_t)best;
}

/*
 * One row of K binary32 values -> K/2 packed E2M1 bytes and K/16 UE4M3 scale
 * bytes, global scale g (binary32 arithmetic throughout, as read above).
 */
static void nvfp4_row(const float *x, int64_t K, float g, uint8_t *codes, uint8_t *scales)
{
    volatile float gs = g / 6.0f;
    for (int64_t b = 0; b < K / 16; ++b) {
        float amax = 0.0f;
        for (int j = 0; j < 16; ++j) {
            float a = fabsf(x[16 * b + j]);
            if (a > amax)
                amax = a;
        }
        volatile float sf = amax * gs;
        uint8_t sb = orc_e4m3_encode((double)sf) & 0x7F; /* unsigned use of E4M3 */
        scales[b] = sb;
        double ds = orc_e4m3_decode(sb);
        volatile float mul = ds > 0.0 ? g / (float)ds : 0.0f;
        for (int j = 0; j < 16; j += 2) {
            uint8_t lo, hi;
            if (ds > 0.0) {
                volatile float q0 = x[16 * b + j] * mul, q1 = x[16 * b + j + 1] * mul;
                lo = orc_e2m1_encode((double)q0);
                hi = orc_e2m1_encode((double)q1);
            } else {
                lo = orc_e2m1_encode(x[16 * b + j] * 0.0);
                hi = orc_e2m1_encode(x[16 * b + j + 1] * 0.0);
            }
            codes[(16 * b + j) / 2] = (uint8_t)(lo | (hi << 4));
        }
    }
}

/* BF16 [rows, K] (row stride ldx) -> packed codes [rows, K/2], scales [rows, K/16]. */
void orc_nvfp4_quantize_bf16(const uint16_t *x, int64_t rows, int64_t K, int64_t ldx, float g, uint8_t *codes,
                             uint8_t *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float *row = (float *)malloc((size_t)K * sizeof(float));
        if (!row)
            continue;
        for (int64_t k = 0; k < K; ++k)
            row[k] = (float)orc_bf16_decode(x[r * ldx + k]);
        nvfp4_row(row, K, g, codes + r * (K / 2), scales + r * (K / 16));
        free(row);
    }
}

/* Dequantized values [rows, K]: q dec(s) / g, in FP64. */
void orc_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K, float g,
                          double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + k] = orc_e2m1_decode(c) * orc_e4m3_decode(scales[r * (K / 16) + k / 16]) / (double)g;
        }
}

/*
 * NVFP4 linear: Y[i, j] = sum_k xhat[m, k] what[n, k] + bias[n] with the
 * dequantized operands (m = rows[i], n = cols[j]), exact in FP64.
 */
void orc_nvfp4_linear(const uint8_t *xq, const uint8_t *xs, float gx, int64_t M, int64_t K, const uint8_t *wq,
                      const uint8_t *ws, float gw, int64_t N, const uint16_t *bias, const int64_t *rows, int64_t nr,
                      const int64_t *cols, int64_t nc, double *Y)
{
    (void)M;
    (void)N;
    double *wd = (double *)malloc((size_t)nc * (size_t)K * sizeof(double));
    if (!wd)
        return;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nc; ++j) {
        int64_t n = cols ? cols[j] : j;
        orc_nvfp4_dequantize(wq + n * (K / 2), ws + n * (K / 16), 1, K, gw, wd + j * K);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nr; ++i) {
        int64_t r = rows ? rows[i] : i;
        double *xd = (double *)malloc((size_t)K * sizeof(double));
        if (!xd)
            continue;
        orc_nvfp4_dequantize(xq + r * (K / 2), xs + r * (K / 16), 1, K, gx, xd);
        for (int64_t j = 0; j < nc; ++j) {
            int64_t n = cols ? cols[j] : j;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += xd[k] * wd[j * K + k];
            if (bias)
                acc += orc_f16_decode(bias[n]);
            Y[i * nc + j] = acc;
        }
        free(xd);
    }
    free(wd);
}

/* Threads an OpenMP parallel region uses (1 without OpenMP). */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
