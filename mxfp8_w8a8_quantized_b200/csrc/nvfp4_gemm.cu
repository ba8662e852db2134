/*
 * nvfp4_gemm.cu -- NVFP4 W4A4 GEMM with F16-bias / BF16 epilogue on the
 * sm_100a tensor cores (tcgen05).
 *
 *   Y[m, n] = BF16_RNE( alpha * sum_k xh[m, k] wh[n, k] + F32(bias[n]) )
 *   xh[m, k] = e2m1(qx[m, k]) * ue4m3(sx[m, k / 16]),  wh likewise,
 *   alpha = 1 / (g_x g_w)  (the two tensors' FP32 global scales)
 *
 * (page "Wan2.2 I2V A14B, four-step 720p: native LightX2V FP8 and NVFP4",
 * section "Conversion and compatibility": packed E2M1 values, E4M3 scales
 * per block, FP32 global scale and alpha.)
 *
 * Arithmetic: an E2M1 value (at most 2 significant bits, 0.5 .. 6) times a
 * UE4M3 scale (at most 4 significant bits, 2^-9 .. 448) has at most 6
 * significant bits and lies in [2^-10, 2688], so xh and wh are exact in
 * FP16, and every product xh * wh (at most 12 significant bits) is exact in
 * FP32.  The kernel therefore expands the 4-bit operands to FP16 inside the
 * SM and multiplies them on the FP16 kind of the tensor core
 * (tcgen05.mma kind::f16, FP32 accumulation): the sum is the one a
 * block-scaled 4-bit MMA forms, up to the order of the FP32 additions.  HBM
 * and L2 carry only the 4-bit codes and the scale bytes.
 *
 * Persistent kernel on CTA pairs (cluster of 2, tcgen05.mma.cta_group::2):
 * 256 x 256 output tiles, each CTA holding 128 rows of A and 128 rows of B.
 * Roles (576 threads per CTA):
 *   warp 0       TMA producer: per 128-wide K step ("code stage") the CTA's
 *                128 x 64-byte boxes of A and B codes (64-byte swizzle) and
 *                the two 512-byte scale atoms of its A rows and B rows (one
 *                bulk copy each), into a 3-deep ring.
 *   warp 1       allocates 512 TMEM columns (two 256-column accumulators);
 *                in the leader CTA one thread issues, per 64-wide K step,
 *                four kind::f16 MMAs of K = 16 into the tile's accumulator
 *                and commits the step's release to both CTAs.
 *   warps 2..17  expand and write back.  Two threads per row (A rows, then
 *                B rows), each owning 32 elements of every 64-wide K step:
 *                per code stage a thread turns 2 x 16 code bytes and 2 x 2
 *                scale bytes into 64 FP16 values (cvt.rn.f16x2.e2m1x2, exact
 *                multiply by the scale) stored in the 128-byte-swizzled
 *                K-major layout the MMA reads, into a 4-deep ring; the
 *                generic-proxy stores are fenced to the async proxy and
 *                announced to the leader's barriers (32 arrivals per step,
 *                both CTAs).  Once the next tile's first ring slots are
 *                filled, the same warps drain the previous tile's
 *                accumulator in 32-column pieces (the MMA meanwhile runs the
 *                next tile into the other accumulator) and write Y through
 *                swizzled smem boxes and TMA stores.
 * Every wait is bounded: on timeout the kernel records the timeout in a
 * device status word, drains its own MMAs, lets copies still in flight land
 * (a bounded settle), frees TMEM and returns.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "ptx.cuh"
#include "tmap_host.cuh"

namespace nv {

using namespace mx;

constexpr int XW = 16;                   /* expand / epilogue warps */
constexpr int THREADS = (2 + XW) * 32;
constexpr int FS = 4;                    /* FP16 operand stages */
constexpr int RS = 3;                    /* code / scale stages */
constexpr int KF = 64;                   /* K elements per FP16 stage (128-byte rows) */
constexpr int KR = 128;                  /* K elements per code stage (64 bytes of codes per row) */
constexpr int SUB = KR / KF;             /* FP16 stages per code stage */
constexpr int TILE_M = 256, TILE_N = 256;
constexpr uint32_t TMEM_COLS = 512;      /* two 256-column FP32 accumulators */
constexpr uint32_t TILE_BYTES = 128 * 128; /* FP16 operand slot: 128 rows x 128 bytes */
constexpr uint32_t CODE_BYTES = 128 * 64;  /* code slot: 128 rows x 64 bytes */
constexpr uint32_t SF_BYTES = SUB * 512;   /* two 64-wide scale atoms of 128 rows */
constexpr uint32_t OFF_FA = 0;
constexpr uint32_t OFF_FB = OFF_FA + FS * TILE_BYTES;
constexpr uint32_t OFF_RA = OFF_FB + FS * TILE_BYTES;
constexpr uint32_t OFF_RB = OFF_RA + RS * CODE_BYTES;
constexpr uint32_t OFF_SA = OFF_RB + RS * CODE_BYTES;
constexpr uint32_t OFF_SB = OFF_SA + RS * SF_BYTES;
constexpr uint32_t OFF_EPI = OFF_SB + RS * SF_BYTES;
constexpr uint32_t EPI_BUF = 32 * 32 * 2; /* 32 rows x 32 BF16 */
constexpr uint32_t OFF_BAR = OFF_EPI + XW * EPI_BUF;
/* full[FS], empty[FS], rfull[RS], rempty[RS], tfull[2], tempty[2], drain */
constexpr uint32_t NUM_BARS = 2 * FS + 2 * RS + 5;
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + NUM_BARS * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t SMEM_USED = OFF_TMEMPTR + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024; /* slack to align the base to 1 KiB */
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(SUB == 2 && FS % 2 == 0, "a pass expands the two K steps of one code stage into a ring-slot pair");
static_assert(OFF_RA % 1024 == 0 && OFF_RB % 1024 == 0 && OFF_EPI % 1024 == 0 && CODE_BYTES % 1024 == 0,
              "swizzled buffers must be 1 KiB aligned");
constexpr int RASTER_SMALL_B = 8, RASTER_LARGE_B = 16;
constexpr int64_t RASTER_LARGE_B_BYTES = 48ll << 20; /* weight bytes above which 16 M tiles share a group */
constexpr uint32_t SUSPEND_NS = 1000000u;
/* K steps expanded per pass (1 or 2): two K steps per fence and barrier
 * round measured 1.42 ms against 1.64 ms for one at the Q-projection shape */
constexpr int PASS_STEPS = 2;
static_assert(PASS_STEPS == 1 || PASS_STEPS == 2, "pass of one or two K steps");
constexpr uint32_t ST_TIMEOUT = 1u;
constexpr uint64_t ABORT_SETTLE_NS = 200000; /* after a timeout: time for in-flight copies to land */

__device__ unsigned int g_nv_status = 0;

struct Params {
    const uint8_t *sfa;  /* activation scales, tensor-core layout of 16-element blocks */
    const uint8_t *sfb;  /* weight scales, same layout */
    const __half *bias;  /* [N] or null */
    const float *gx;     /* activation global scale (device) */
    const float *gw;     /* weight global scale (device) */
    int M, N, K;
    int kg;              /* K / 64: scale atoms per 128 rows */
    int num_m, num_n, raster;
    unsigned long long timeout_ns;
};

/* ----------------------------------------------------------- helpers */
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
/* D (+)= A . B^T over the CTA pair, FP16 x FP16 -> FP32, K = 16 per MMA. */
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t tacc, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tacc),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
/*
 * Instruction descriptor of kind::f16: FP32 accumulator (1 at [4,6)), A and
 * B FP16 (0 at [7,10) and [10,13)), both K-major, N >> 3 at [17,23),
 * M >> 4 at [24,29).
 */
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N)
{
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
/* four E2M1 pairs (one 32-bit word, element 2i in the low nibble of byte i)
 * -> four FP16 pairs, each multiplied by the FP16 pair s2 (exact) */
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t s2, uint32_t &h0, uint32_t &h1, uint32_t &h2,
                                            uint32_t &h3)
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        ".reg .b32 t0, t1, t2, t3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 t0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 t1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 t2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 t3, b3;\n\t"
        "mul.rn.f16x2 %0, t0, %5;\n\t"
        "mul.rn.f16x2 %1, t1, %5;\n\t"
        "mul.rn.f16x2 %2, t2, %5;\n\t"
        "mul.rn.f16x2 %3, t3, %5;\n\t}\n"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w), "r"(s2));
}

/* Tile t -> (M tile, N tile): `raster` M tiles are walked together for
 * every N tile so that their A rows stay in L2 while the weights stream. */
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int raster, int &mb, int &nb)
{
    const int per_group = raster * num_n;
    const int g = t / per_group;
    const int first = g * raster;
    const int gm = min(raster, num_m - first);
    const int r = t - g * per_group;
    mb = first + r % gm;
    /* odd groups walk N backwards: a group starts on the weight tiles the
     * previous one ended on, which are still in L2 */
    nb = (g & 1) ? num_n - 1 - r / gm : r / gm;
}

/*
 * Bounded wait: true when the phase of parity `parity` has completed.  On
 * timeout it records ST_TIMEOUT in the device status word and raises the
 * CTA's abort flag, so the other roles stop waiting too.
 */
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                             volatile uint32_t *abort_flag)
{
    if (mbar_try_wait(bar, parity, SUSPEND_NS))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity, SUSPEND_NS))
            return true;
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1u;
            atomicOr(&g_nv_status, ST_TIMEOUT);
            return false;
        }
    }
}
/* every lane waits; the vote makes the outcome warp-uniform */
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                          volatile uint32_t *abort_flag)
{
    const bool ok = wait_bounded(bar, parity, limit_ns, abort_flag);
    return __all_sync(0xFFFFFFFFu, ok);
}

/* scale bytes (b, b, c, c) of a word -> FP16 pairs (dec(b), dec(b)) and
 * (dec(c), dec(c)) */
__device__ __forceinline__ void scale_pairs2(uint32_t d, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}\n"
        : "=r"(lo), "=r"(hi)
        : "r"(d));
}

/*
 * One thread, half a row (32 elements), NS (1 or 2) 64-wide K steps of one
 * code stage, from step j0.  Step j reads the 16-byte code chunk 2 j + h of the row's
 * 64-byte code line (64-byte swizzle: chunk ^ ((row / 2) % 4)) and the
 * scale bytes 2h, 2h + 1 of the row's word in atom j, and writes 32 FP16
 * values as chunks 4h .. 4h + 3 of the row in step j's operand slot
 * (128-byte swizzle: chunk ^ (row % 8)).  All loads are issued first.
 */
template <int NS>
__device__ __forceinline__ void expand_half_row(uint32_t code_row, uint32_t xc, uint32_t sf_word_addr,
                                                bool have_scales, int j0, int h, uint32_t f16_row0,
                                                uint32_t f16_row1, uint32_t xf)
{
    uint4 c[NS];
    uint32_t sw[NS];
#pragma unroll
    for (int j = 0; j < NS; ++j)
        c[j] = ld_shared_v4(code_row + ((((uint32_t)(2 * (j0 + j) + h)) ^ xc) << 4));
#pragma unroll
    for (int j = 0; j < NS; ++j)
        sw[j] = have_scales ? ld_shared_u32(sf_word_addr + (uint32_t)(j0 + j) * 512u) : 0u;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
        uint32_t s_lo, s_hi;
        scale_pairs2(__byte_perm(sw[j], 0u, h ? 0x3322u : 0x1100u), s_lo, s_hi);
        const uint32_t f16_row = j == 0 ? f16_row0 : f16_row1;
        const uint32_t w[4] = {c[j].x, c[j].y, c[j].z, c[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { /* 8 elements; block i / 2 of the half */
            uint32_t h0, h1, h2, h3;
            expand_word(w[i], i < 2 ? s_lo : s_hi, h0, h1, h2, h3);
            st_shared_v4(f16_row + ((((uint32_t)(4 * h + i)) ^ xf) << 4), h0, h1, h2, h3);
        }
    }
}

/* 32 lanes x 32 consecutive 32-bit TMEM columns -> 32 registers, with the
 * wait for the load in the same statement. */
__device__ __forceinline__ void tmem_ld_32x32b_x32_sync(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

/* Y = BF16(alpha acc + bias) for 32 rows x 32 columns, staged through a
 * 64-byte-swizzled smem box and written by one TMA store of the warp. */
__device__ __forceinline__ void epilogue_piece(const uint32_t (&acc)[32], const Params &p, float alpha,
                                               const CUtensorMap *tmap_y, int row0, int colc, int lane,
                                               uint32_t buf, uint32_t rowbase, uint32_t swz)
{
    if (row0 >= p.M || colc >= p.N) /* whole box outside Y */
        return;
    if (lane == 0)
        bulk_wait_group_read0(); /* previous box has left the buffer */
    __syncwarp();
#pragma unroll
    for (int j8 = 0; j8 < 4; ++j8) {
        const int col = colc + 8 * j8;
        float b[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (p.bias && col < p.N) {
            const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(p.bias + col));
            const __half2 *bh = reinterpret_cast<const __half2 *>(&bv);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f2 = __half22float2(bh[j]);
                b[2 * j] = f2.x;
                b[2 * j + 1] = f2.y;
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int a = 8 * j8 + 2 * j;
            __nv_bfloat162 v = __floats2bfloat162_rn(fmaf(alpha, __uint_as_float(acc[a]), b[2 * j]),
                                                     fmaf(alpha, __uint_as_float(acc[a + 1]), b[2 * j + 1]));
            o[j] = *reinterpret_cast<uint32_t *>(&v);
        }
        st_shared_v4(rowbase + ((((uint32_t)j8) ^ swz) << 4), o[0], o[1], o[2], o[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_y, colc, row0, buf);
        bulk_commit_group();
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_y, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank(); /* 0 = leader */
    const int tile0 = (int)cluster_id_x();
    const int tstep = (int)nclusters_x();

    const uint32_t bar_full = sbase + OFF_BAR;        /* + 8 s, s < FS */
    const uint32_t bar_empty = bar_full + FS * 8;     /* + 8 s */
    const uint32_t bar_rfull = bar_empty + FS * 8;    /* + 8 r, r < RS */
    const uint32_t bar_rempty = bar_rfull + RS * 8;   /* + 8 r */
    const uint32_t bar_tfull = bar_rempty + RS * 8;   /* + 8 b, b < 2 */
    const uint32_t bar_tempty = bar_tfull + 2 * 8;    /* + 8 b */
    const uint32_t bar_drain = bar_tempty + 2 * 8;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + OFF_TMEMPTR);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + OFF_ABORT);

    if (threadIdx.x == 0) {
        *abort_flag = 0u;
        for (int s = 0; s < FS; ++s) {
            mbar_init(bar_full + 8 * s, 2 * XW); /* every expand warp of both CTAs */
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int r = 0; r < RS; ++r) {
            mbar_init(bar_rfull + 8 * r, 1);
            mbar_init(bar_rempty + 8 * r, XW);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 2 * XW);
        }
        mbar_init(bar_drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_ptr), TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all(); /* peer barriers initialised before any remote signal */
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    const int KB = p.K / KF;             /* FP16 stages per tile */
    const int KRN = (p.K + KR - 1) / KR; /* code stages per tile */
    const int num_tiles = p.num_m * p.num_n;
    const unsigned long long lim = p.timeout_ns;

    if (warp == 0) {
        /* ------------------------------------------------ TMA producer */
        if (lane == 0) {
            prefetch_tmap(&tmap_a);
            prefetch_tmap(&tmap_b);
            uint32_t ir = 0;
            bool ok = true;
            for (int t = tile0; ok && t < num_tiles; t += tstep) {
                int mb, nb;
                tile_coords(t, p.num_m, p.num_n, p.raster, mb, nb);
                const int rowA = mb * TILE_M + (int)(rank * 128u);
                const int rowB = nb * TILE_N + (int)(rank * 128u);
                const bool a_in = rowA < p.M, b_in = rowB < p.N; /* scale atoms exist for the row block */
                for (int kr = 0; kr < KRN; ++kr, ++ir) {
                    const uint32_t s = ir % RS, ph = (ir / RS) & 1u;
                    if (!wait_bounded(bar_rempty + 8 * s, ph ^ 1u, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int n_at = min(SUB, p.kg - SUB * kr);
                    const uint32_t sf_bytes = (uint32_t)n_at * 512u;
                    const uint32_t full = bar_rfull + 8 * s;
                    mbar_arrive_expect_tx(full, 2u * CODE_BYTES + (a_in ? sf_bytes : 0u) + (b_in ? sf_bytes : 0u));
                    tma_load_2d(sbase + OFF_RA + s * CODE_BYTES, &tmap_a, kr * (KR / 2), rowA, full);
                    tma_load_2d(sbase + OFF_RB + s * CODE_BYTES, &tmap_b, kr * (KR / 2), rowB, full);
                    if (a_in)
                        bulk_load(sbase + OFF_SA + s * SF_BYTES,
                                  p.sfa + ((size_t)(rowA / 128) * p.kg + (size_t)(SUB * kr)) * 512u, sf_bytes, full);
                    if (b_in)
                        bulk_load(sbase + OFF_SB + s * SF_BYTES,
                                  p.sfb + ((size_t)(rowB / 128) * p.kg + (size_t)(SUB * kr)) * 512u, sf_bytes, full);
                }
            }
        }
    } else if (warp == 1) {
        /* ------------------------------------------------ MMA issuer */
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_f16(TILE_M, TILE_N);
            uint32_t it = 0, tl = 0;
            bool ok = true, any = false;
            for (int t = tile0; ok && t < num_tiles; t += tstep, ++tl) {
                const uint32_t ab = tl & 1u; /* accumulator of this tile */
                if (!wait_bounded(bar_tempty + 8 * ab, ((tl >> 1) & 1u) ^ 1u, lim, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tacc = tmem + 256u * ab;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % FS, ph = (it / FS) & 1u;
                    if (!wait_bounded(bar_full + 8 * s, ph, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = desc_kmajor_sw128(sbase + OFF_FA + s * TILE_BYTES);
                    const uint64_t bdesc = desc_kmajor_sw128(sbase + OFF_FB + s * TILE_BYTES);
#pragma unroll
                    for (int k = 0; k < KF / 16; ++k)
                        tc_mma_f16_pair(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                        (kb | k) != 0);
                    tc_commit_pair(bar_empty + 8 * s, (uint16_t)0x3);
                    any = true;
                }
                if (!ok)
                    break;
                tc_commit_pair(bar_tfull + 8 * ab, (uint16_t)0x3);
            }
            if (ok) {
                /* every epilogue (the peer's included) has released the last
                 * accumulators, so no remote arrival is still in flight */
                for (uint32_t u = tl > 2u ? tl - 2u : 0u; u < tl; ++u)
                    (void)wait_bounded(bar_tempty + 8 * (u & 1u), (u >> 1) & 1u, lim, abort_flag);
            }
            if (!ok && any) {
                /* wait for this thread's MMAs before TMEM is freed */
                volatile uint32_t own = 0u;
                tc_commit_pair(bar_drain, (uint16_t)0x1);
                (void)wait_bounded(bar_drain, 0u, lim, &own);
            }
        }
    } else {
        /* ------------------------------------- expand + epilogue warps */
        const int e = (warp - 2) * 32 + lane;
        const int op = e >> 8;        /* 0: A row, 1: B row */
        const int h = (e >> 7) & 1;   /* which 32 elements of each 64-wide K step */
        const int r = e & 127;
        const uint32_t xc = (uint32_t)((r >> 1) & 3); /* 64-byte swizzle of the code line */
        const uint32_t xf = (uint32_t)(r & 7);        /* 128-byte swizzle of the FP16 row */
        const uint32_t sf_off = (uint32_t)((r & 31) * 16 + ((r >> 5) & 3) * 4);
        const uint32_t code_base = sbase + (op ? OFF_RB : OFF_RA) + (uint32_t)r * 64u;
        const uint32_t sf_base = sbase + (op ? OFF_SB : OFF_SA) + sf_off;
        const uint32_t f16_base = sbase + (op ? OFF_FB : OFF_FA) + (uint32_t)r * 128u;
        /* epilogue geometry: TMEM sub-partition and 64-column group */
        const int q = warp & 3;
        const int cg = (warp - 2) >> 2;
        const uint32_t buf = sbase + OFF_EPI + (uint32_t)(warp - 2) * EPI_BUF;
        const uint32_t rowbase = buf + (uint32_t)lane * 64u;
        const uint32_t swz = ((uint32_t)lane >> 1) & 3u;

        /* alpha = 1 / (g_x g_w): the product of two binary32 values is exact
         * in FP64, the quotient is rounded to FP64 and then once to binary32 */
        const float alpha = (float)(1.0 / ((double)__ldg(p.gx) * (double)__ldg(p.gw)));
        uint32_t it = 0, ir = 0, tl = 0;
        bool ok = true;
        bool pending = false;
        int pend_t = 0;
        /* drains the accumulator of tile pend_t in two 32-column pieces and
         * writes its Y; the accumulator is released after the second load */
        auto epilogue = [&]() -> bool {
            int mb, nb;
            tile_coords(pend_t, p.num_m, p.num_n, p.raster, mb, nb);
            const uint32_t ab = tl & 1u;
            const bool got = wait_bounded(bar_tfull + 8 * ab, (tl >> 1) & 1u, lim, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got))
                return false;
            tc_fence_after();
            const int row0 = mb * TILE_M + (int)(rank * 128u) + 32 * q;
            const int col0 = nb * TILE_N + cg * 64;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32_sync(tmem + ((uint32_t)(32 * q) << 16) + 256u * ab + (uint32_t)(cg * 64 + 32 * c),
                                        acc);
                if (c == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive_cluster(mapa_shared(bar_tempty + 8 * ab, 0u));
                }
                epilogue_piece(acc, p, alpha, &tmap_y, row0, col0 + 32 * c, lane, buf, rowbase, swz);
            }
            ++tl;
            return true;
        };

        for (int t = tile0; ok && t < num_tiles; t += tstep) {
            int mb, nb;
            tile_coords(t, p.num_m, p.num_n, p.raster, mb, nb);
            const int row_block = op ? nb * TILE_N + (int)(rank * 128u) : mb * TILE_M + (int)(rank * 128u);
            const bool have_scales = row_block < (op ? p.N : p.M);
            /* PASS_STEPS K steps per pass (one at an odd end) */
            for (int kb = 0; kb < KB;) {
                if (pending && kb == FS) {
                    pending = false;
                    if (!epilogue()) {
                        ok = false;
                        break;
                    }
                }
                const int ns = (PASS_STEPS == 2 && kb + 1 < KB) ? 2 : 1;
                const int j0 = kb % SUB;
                const uint32_t rs = ir % RS;
                const uint32_t s0 = it % FS, s1 = (it + 1) % FS;
                if ((j0 == 0 && !warp_wait(bar_rfull + 8 * rs, (ir / RS) & 1u, lim, abort_flag)) ||
                    !warp_wait(bar_empty + 8 * s0, ((it / FS) & 1u) ^ 1u, lim, abort_flag) ||
                    (ns == 2 && !warp_wait(bar_empty + 8 * s1, (((it + 1) / FS) & 1u) ^ 1u, lim, abort_flag))) {
                    ok = false;
                    break;
                }
                const uint32_t code_row = code_base + rs * CODE_BYTES;
                const uint32_t sf_addr = sf_base + rs * SF_BYTES;
                if (ns == 2)
                    expand_half_row<2>(code_row, xc, sf_addr, have_scales, 0, h, f16_base + s0 * TILE_BYTES,
                                       f16_base + s1 * TILE_BYTES, xf);
                else
                    expand_half_row<1>(code_row, xc, sf_addr, have_scales, j0, h, f16_base + s0 * TILE_BYTES, 0u,
                                       xf);
                fence_proxy_async_smem(); /* generic-proxy stores -> visible to the tensor core */
                __syncwarp();
                if (lane == 0) {
                    /* every thread fenced its stores to the async proxy; one
                     * arrive per warp on the leader's barrier (the peer's
                     * through its shared::cluster address), as the
                     * transform-to-MMA hand-off of the 2-SM UMMA pipelines
                     * does.  A cluster-scope release here costs about 1,400
                     * cycles per arrive and throttled the pair (measured). */
                    mbar_arrive_cluster(mapa_shared(bar_full + 8 * s0, 0u));
                    if (ns == 2)
                        mbar_arrive_cluster(mapa_shared(bar_full + 8 * s1, 0u));
                }
                if (j0 + ns == SUB || kb + ns == KB) { /* code stage consumed */
                    if (lane == 0)
                        mbar_arrive(bar_rempty + 8 * rs);
                    ++ir;
                }
                kb += ns;
                it += (uint32_t)ns;
            }
            if (!ok)
                break;
            if (pending) {
                pending = false;
                if (!epilogue()) {
                    ok = false;
                    break;
                }
            }
            pending = true;
            pend_t = t;
        }
        if (ok && pending)
            (void)epilogue();
        if (lane == 0)
            bulk_wait_group0(); /* stores complete before the CTA exits */
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        /* a wait gave up: copies this CTA issued may still be landing in its
         * shared memory; let them settle (bounded) before the CTA exits */
        if (threadIdx.x == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < ABORT_SETTLE_NS)
                __nanosleep(1000);
        }
        __syncthreads();
    }
    cluster_sync_all(); /* neither CTA leaves while the pair may still touch it */
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

/* Self-test of the bounded wait used by this kernel (as in the MXFP8 GEMM):
 * a wait on an mbarrier that nothing arrives at gives up after limit_ns and
 * records ST_TIMEOUT. */
__global__ void wait_selftest_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0u;
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        (void)wait_bounded(smem_u32(&bar), 0u, limit_ns, &abort_flag);
    }
}

/* ------------------------------------------------------------ host side */
struct DevInfo {
    bool init = false;
    bool attr = false;
    int max_clusters = 0;
};
static DevInfo g_dev[64];

static void cluster_config(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr, unsigned grid, cudaStream_t stream)
{
    cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

static cudaError_t dev_info(DevInfo **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    DevInfo &d = g_dev[dev];
    if (!d.init) {
        e = cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess)
            return e;
        int sms = 148;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaLaunchConfig_t cfg;
        cudaLaunchAttribute attr[1];
        cluster_config(cfg, attr, 2u * (unsigned)sms, nullptr);
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, nvfp4_gemm_kernel, &cfg);
        if (e != cudaSuccess)
            return e;
        if (n <= 0)
            return cudaErrorInvalidConfiguration;
        d.max_clusters = n;
        d.init = true;
    }
    *out = &d;
    return cudaSuccess;
}

} // namespace nv

namespace mx {

/*
 * Xq [M, K/2] / Wq [N, K/2] packed E2M1 codes, Xs / Ws their scales in the
 * tensor-core layout of 16-element blocks, Y BF16 [M, N].  K % 64 == 0.
 * Returns 0 ok, 1 tensor-map failure, 2 CUDA error (in *err).
 */
int launch_nvfp4_gemm(const void *Xq, const void *Xs, int64_t M, int64_t K, const void *Wq, const void *Ws,
                      int64_t N, const float *gx, const float *gw, const void *bias, void *Y,
                      cudaStream_t stream, unsigned long long timeout_ns, cudaError_t *err)
{
    *err = cudaSuccess;
    if (M == 0)
        return 0;
    nv::DevInfo *d = nullptr;
    cudaError_t e = nv::dev_info(&d);
    if (e != cudaSuccess) {
        *err = e;
        return 2;
    }
    CUtensorMap ma, mb, my;
    if (!encode_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, K / 2, M, K / 2, nv::KR / 2, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K / 2, N, K / 2, nv::KR / 2, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return 1;
    nv::Params p;
    p.sfa = static_cast<const uint8_t *>(Xs);
    p.sfb = static_cast<const uint8_t *>(Ws);
    p.bias = static_cast<const __half *>(bias);
    p.gx = gx;
    p.gw = gw;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.kg = (int)(K / 64);
    p.num_m = (int)((M + nv::TILE_M - 1) / nv::TILE_M);
    p.num_n = (int)((N + nv::TILE_N - 1) / nv::TILE_N);
    p.raster = N * K / 2 > nv::RASTER_LARGE_B_BYTES ? nv::RASTER_LARGE_B : nv::RASTER_SMALL_B;
    p.timeout_ns = timeout_ns;
    const int tiles = p.num_m * p.num_n;
    int clusters = d->max_clusters < tiles ? d->max_clusters : tiles;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    nv::cluster_config(cfg, attr, 2u * (unsigned)clusters, stream);
    e = cudaLaunchKernelEx(&cfg, nv::nvfp4_gemm_kernel, ma, mb, my, p);
    if (e != cudaSuccess) {
        *err = e;
        return 2;
    }
    return 0;
}

cudaError_t launch_nv_wait_selftest(unsigned long long limit_ns, cudaStream_t stream)
{
    nv::wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

/* Reads and clears the NVFP4 GEMM's status word (synchronous). */
cudaError_t read_and_clear_nv_status(unsigned int *out)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, nv::g_nv_status, sizeof(unsigned int));
    if (e != cudaSuccess)
        return e;
    return cudaMemcpyToSymbol(nv::g_nv_status, &zero, sizeof(unsigned int));
}

} // namespace mx
