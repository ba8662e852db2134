/*
 * mxfp8_gemm.cu -- block-scaled MXFP8 GEMM with F16-bias / BF16 epilogue on
 * the sm_100a tensor cores (tcgen05).
 *
 *   Y[m, n] = BF16_RNE( sum_b 2^(sx[m,b] + sw[n,b]) sum_{j<32} x[m,32b+j] w[n,32b+j]
 *                       + F32(bias[n]) )
 *
 * (model card "Wan2.2-I2V-A14B-Lightning . MXFP8 (AutoRound OptRTN)":
 * "Performance Profile" -- "linear (MXFP8 W8A8)" is the layer's GEMM;
 * "Coverage per transformer" -- E4M3 codes, per-32 E8M0 scales, F16 biases.)
 *
 * Two variants of one persistent, warp-specialized kernel:
 *
 *  PAIR (default): a cluster of two CTAs on two SMs computes 256 x 256 output
 *   tiles with tcgen05.mma.cta_group::2 (M = 256).  Each CTA stages its own
 *   128 rows of A, its own half (128 rows) of B, the scale atom of its A rows
 *   and both scale atoms of B, so per SM the tensor core is fed 64 bytes per
 *   clock instead of the 96 a single-SM 128 x 256 tile needs -- the L2-to-SM
 *   fabric, not the tensor core, limits the single-SM form on B200.  Loads
 *   use TMA without multicast; their completion is signalled to the leader
 *   CTA's barrier (cta_group::2 form), and the leader's single MMA thread
 *   issues the MMAs for the pair.
 *  SINGLE: one CTA per SM, 128 x 256 tiles, tcgen05.mma.cta_group::1.
 *
 * Roles (352 threads per CTA):
 *   warp 0       TMA producer: per 128-wide K step, A and B tiles (tiled TMA,
 *                128-byte swizzle) and their scale atoms (512 B per 128
 *                rows, 3-D tiled TMA) into a multi-stage smem ring guarded
 *                by mbarriers.
 *   warp 1       allocates 512 TMEM columns; one thread (the leader CTA's in
 *                PAIR) copies the stage's scales to TMEM (tcgen05.cp
 *                32x128b.warpx4) and issues four tcgen05.mma
 *                kind::mxf8f6f4.block_scale of K = 32, the scale byte of each
 *                K step picked by the instruction descriptor's scale-factor
 *                ID; tcgen05.commit frees the stage (in both CTAs) and, after
 *                the tile, signals the epilogues.
 *   warp 10      (leader CTA of a pair) copies each stage's scales to TMEM
 *                with the pair-wide tcgen05.cp and signals the MMA thread
 *                through an mbarrier: that copy stalls the thread issuing it,
 *                which must not be the one that keeps the tensor core fed.
 *   warps 2..9   epilogue: each warp owns one 32-lane TMEM sub-partition and
 *                half the columns; it drains its 32 x 128 FP32 block in one
 *                tcgen05.ld, releases the accumulator to the MMA thread at
 *                once, then adds the bias, rounds to BF16 and writes 32 x 32
 *                boxes through a swizzled smem buffer with TMA stores
 *                (clipped at M and N) while the next tile's MMAs run.
 * The shared-memory data path is the scarce resource: TMA writes each stage
 * and the tensor core reads it (~130 B/clock per SM at full MMA rate), so
 * everything else is kept off it -- waits sleep in mbarrier.try_wait instead
 * of spinning, and the output leaves through bulk TMA stores rather than
 * per-row global stores.  Scale columns in TMEM are per stage, so a scale
 * copy never overwrites scales an earlier, still running MMA reads.  Every wait is bounded: on
 * timeout the kernel records MXFP8_ERR_TIMEOUT in a device status word,
 * drains its own MMAs, lets copies still in flight land (a bounded settle),
 * frees TMEM and returns.  Without block scales (the per-channel FP8 mode)
 * TMEM holds two accumulators and the MMAs of the next tile overlap the
 * epilogue of the last.
 */
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cstdint>
#include <cstdlib>

#include "mx_element.cuh"
#include "ptx.cuh"
#include "tmap_host.cuh"

namespace mx {

constexpr int BK = 128; /* bytes = E4M3 elements per K step */
constexpr int EPI_WARPS = 8;
constexpr int SF_WARP = 2 + EPI_WARPS; /* copies scales to TMEM (CTA-pair variant) */
constexpr int GEMM_THREADS = (3 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0; /* 256 FP32 columns */
/* Tile walk (tile_coords).  Preferred: groups of N tiles whose weight rows
 * (at most RASTER_B_GROUP_BYTES) stay in L2 while the activation rows
 * stream past them once per group -- used when such a group can span at
 * least RASTER_MIN_N_GROUP N tiles; the N tiles are split into the fewest
 * groups of that size, made equal (60 tiles: 20 + 20 + 20, not 24 + 24 + 12).
 * DRAM reads per launch at M = 75348 (81 frames at 832x1104), ncu, cold L2,
 * by N tiles per group:
 *   q/k/v (K 5120, N 15360)          38: 3.40 GB, 24: 2.87, 18: 3.36, all 60: 8.08
 *   ffn.net.0.proj (K 5120, N 13824)  38: 3.36 GB, 27: 2.23, 18: 2.19, all 54: 7.21
 *   ffn.net.2 (K 13824, N 5120)       13: 8.04 GB, 10: 7.26, 7: 7.67, all 20: 9.33
 * (groups of more weight are re-read from DRAM on every wave of tiles; this
 * rule takes 20, 27 and 10).  Otherwise (long K: a weight tile is too large
 * for a useful group) groups of M tiles walk every N tile: 8 when the
 * weights fit in L2 alongside them, 16 when they are re-read from DRAM once
 * per group. */
constexpr int64_t RASTER_B_GROUP_BYTES = 36ll << 20;
constexpr int RASTER_MIN_N_GROUP = 6;
constexpr int RASTER_SMALL_B = 8, RASTER_LARGE_B = 16;
constexpr int64_t RASTER_LARGE_B_BYTES = 48ll << 20;
/* mbarrier.try_wait suspend-time hints (ns): the producer and MMA threads wait
 * briefly and often, the epilogue warps for a whole tile */
constexpr uint32_t SUSPEND_PIPE = 1000000;
constexpr uint32_t SUSPEND_EPI = 1000000;
constexpr uint32_t ST_TIMEOUT = 1u;
constexpr uint64_t ABORT_SETTLE_NS = 200000; /* after a timeout: time for in-flight copies to land */

/* What the epilogue writes. */
enum EpiMode : int {
    EPI_BF16 = 0,       /* Y = BF16(acc + bias) */
    EPI_QUANT = 1,      /* MXFP8 codes + scales of BF16(acc + bias) for the next linear */
    EPI_QUANT_GELU = 2, /* MXFP8 codes + scales of BF16(GELU(BF16(acc + bias))) */
    EPI_ROWWISE = 3,    /* per-channel FP8: no block scales; Y = BF16(acc sx[m] sw[n] + bias) */
    EPI_NVFP4 = 4,      /* NVFP4 operands (E2M1, UE4M3 per 16); Y = BF16(alpha acc + bias) */
};

/* FP4: packed E2M1 operands -- a 128-byte stage row holds 256 elements,
 * four MMAs of K = 64, each with its own scale atom per 128 rows. */
template <bool PAIR, bool FP4 = false>
struct Cfg {
    static constexpr int K_ATOMS = FP4 ? 4 : 1;             /* scale atoms per 128 rows per stage */
    static constexpr int STAGES = FP4 ? (PAIR ? 5 : 3) : (PAIR ? 6 : 4);
    static constexpr int TILE_M = PAIR ? 256 : 128; /* output rows per tile */
    static constexpr int TILE_N = 256;
    static constexpr uint32_t A_ROWS = 128;                 /* A rows staged per CTA */
    static constexpr uint32_t B_ROWS = PAIR ? 128 : 256;    /* B rows staged per CTA */
    static constexpr uint32_t A_BYTES = A_ROWS * BK;
    static constexpr uint32_t B_BYTES = B_ROWS * BK;
    static constexpr uint32_t SFA_BYTES = 512 * K_ATOMS;    /* this CTA's 128 A rows */
    static constexpr uint32_t SFB_BYTES = 1024 * K_ATOMS;   /* all 256 B rows: [row half][atom] */
    static constexpr uint32_t STAGE_TX = (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) * (PAIR ? 2u : 1u);
    static constexpr uint32_t SFA_STEP = 4 * K_ATOMS;       /* TMEM columns per stage */
    static constexpr uint32_t SFB_STEP = 8 * K_ATOMS;
    static constexpr uint32_t SFA_COL = 256;
    static constexpr uint32_t SFB_COL = 256 + SFA_STEP * STAGES;
    static_assert(SFB_COL + SFB_STEP * STAGES <= TMEM_COLS, "TMEM budget");
    static constexpr uint32_t OFF_A = 0;
    static constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr uint32_t OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr uint32_t OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr uint32_t OFF_EPI = OFF_SFB + STAGES * SFB_BYTES; /* 1 KiB aligned */
    static constexpr uint32_t EPI_BUF = 32 * 32 * 2;                    /* 32 rows x 32 BF16 */
    static constexpr uint32_t OFF_BAR = OFF_EPI + EPI_WARPS * EPI_BUF;
    static constexpr uint32_t NUM_BARS = 3 * STAGES + 5; /* full[], empty[], sf_full[], tmem_full[2], tmem_empty[2], drain */
    static constexpr uint32_t OFF_TMEMPTR = OFF_BAR + NUM_BARS * 8;
    static constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
    static constexpr uint32_t SMEM_USED = OFF_TMEMPTR + 16;
    static constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024; /* slack to align the base to 1 KiB */
    static constexpr uint32_t TEMPTY_ARRIVALS = EPI_WARPS * (PAIR ? 2u : 1u);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(OFF_EPI % 1024 == 0, "staging buffers must be swizzle-atom aligned");
};

__device__ unsigned int g_mx_status = 0;

struct GemmParams {
    const __half *bias;   /* [N] or null */
    __nv_bfloat16 *Y;     /* [M, N] (EPI_BF16) */
    uint8_t *S;           /* output scales, tensor-core layout of [M, N] (quantizing modes) */
    const float *sx;      /* [M] row scales (EPI_ROWWISE) */
    const float *sw;      /* [N] column scales (EPI_ROWWISE) */
    const float *gx, *gw; /* the two tensors' FP32 global scales (EPI_NVFP4) */
    int M, N;
    int K;                /* operand row bytes: K elements of E4M3, K / 2 of packed E2M1 */
    int m_pad;            /* M rounded up to 128: rows that own scale bytes */
    int sf_kgroups;       /* N / 128: scale atoms per 128 output rows */
    int num_m, num_n;     /* output tiles */
    int raster;           /* > 0: M tiles per raster group; < 0: N tiles per group */
    unsigned long long timeout_ns;
};

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int raster, int &mb, int &nb)
{
    if (raster > 0) {
        /* groups of `raster` M tiles, each group walked over every N tile */
        const int per_group = raster * num_n;
        const int g = t / per_group;
        const int first = g * raster;
        const int gm = min(raster, num_m - first);
        const int r = t - g * per_group;
        mb = first + r % gm;
        /* odd groups walk N backwards: a group starts on the weight tiles the
         * previous one ended on, which are still in L2 */
        nb = (g & 1) ? num_n - 1 - r / gm : r / gm;
    } else {
        /* groups of -raster N tiles, each group walked over every M tile */
        const int gsz = -raster;
        const int per_group = gsz * num_m;
        const int g = t / per_group;
        const int first = g * gsz;
        const int gn = min(gsz, num_n - first);
        const int r = t - g * per_group;
        nb = first + r % gn;
        mb = (g & 1) ? num_m - 1 - r / gn : r / gn;
    }
}

/*
 * Bounded wait: true when the phase of parity `parity` has completed.  On
 * timeout it records ST_TIMEOUT in the device status word and raises the
 * CTA's abort flag, so the other roles stop waiting too.
 */
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                             volatile uint32_t *abort_flag, uint32_t suspend_ns = SUSPEND_PIPE)
{
    if (mbar_try_wait(bar, parity, suspend_ns))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity, suspend_ns))
            return true;
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1u;
            atomicOr(&g_mx_status, ST_TIMEOUT);
            return false;
        }
    }
}

/* Epilogue writing Y = BF16(acc + bias) (ALPHA: Y = BF16(fma(alpha, acc,
 * bias)), the NVFP4 layer): bias + BF16 rounding, 32 columns at a time,
 * staged through a 64-byte-swizzled smem box and written by one TMA store
 * per warp -- scattered per-row global stores would occupy the L1 /
 * shared-memory data path that feeds the tensor core. */
template <bool ALPHA>
__device__ __forceinline__ void epilogue_bf16(const uint32_t (&acc)[128], const GemmParams &p, float alpha,
                                              const CUtensorMap *tmap_y, int row0, int col0, int lane,
                                              uint32_t buf, uint32_t rowbase, uint32_t swz)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int colc = col0 + 32 * c;
        if (row0 >= p.M || colc >= p.N) /* whole box outside Y: nothing to store */
            continue;
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
                const int a = 32 * c + 8 * j8 + 2 * j;
                __nv_bfloat162 v;
                if constexpr (ALPHA)
                    v = __floats2bfloat162_rn(fmaf(alpha, __uint_as_float(acc[a]), b[2 * j]),
                                              fmaf(alpha, __uint_as_float(acc[a + 1]), b[2 * j + 1]));
                else
                    v = __floats2bfloat162_rn(__uint_as_float(acc[a]) + b[2 * j],
                                              __uint_as_float(acc[a + 1]) + b[2 * j + 1]);
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
}

/* Per-channel FP8 epilogue: Y = BF16(acc sx[row] sw[col] + bias), staged and
 * stored like the BF16 epilogue.  The thread's row scale is one load; the
 * column scales come 8 at a time with the bias. */
__device__ __forceinline__ void epilogue_rowwise(const uint32_t (&acc)[128], const GemmParams &p,
                                                 const CUtensorMap *tmap_y, int row0, int col0, int lane,
                                                 uint32_t buf, uint32_t rowbase, uint32_t swz)
{
    const int row = row0 + lane;
    const float sxr = row < p.M ? __ldg(p.sx + row) : 0.0f;
    const f32x2 sx2 = f2_pack(sxr, sxr);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int colc = col0 + 32 * c;
        if (row0 >= p.M || colc >= p.N) /* whole box outside Y: nothing to store */
            continue;
        if (lane == 0)
            bulk_wait_group_read0(); /* previous box has left the buffer */
        __syncwarp();
#pragma unroll
        for (int j8 = 0; j8 < 4; ++j8) {
            const int col = colc + 8 * j8;
            float b[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (col < p.N) {
                const uint4 w0 = __ldg(reinterpret_cast<const uint4 *>(p.sw + col));
                const uint4 w1 = __ldg(reinterpret_cast<const uint4 *>(p.sw + col + 4));
                w[0] = __uint_as_float(w0.x), w[1] = __uint_as_float(w0.y), w[2] = __uint_as_float(w0.z);
                w[3] = __uint_as_float(w0.w), w[4] = __uint_as_float(w1.x), w[5] = __uint_as_float(w1.y);
                w[6] = __uint_as_float(w1.z), w[7] = __uint_as_float(w1.w);
                if (p.bias) {
                    const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(p.bias + col));
                    const __half2 *bh = reinterpret_cast<const __half2 *>(&bv);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f2 = __half22float2(bh[j]);
                        b[2 * j] = f2.x;
                        b[2 * j + 1] = f2.y;
                    }
                }
            }
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int a = 32 * c + 8 * j8 + 2 * j;
                const f32x2 t = f2_mul(f2_pack(__uint_as_float(acc[a]), __uint_as_float(acc[a + 1])), sx2);
                o[j] = f32x2_to_bf16x2(f2_fma(t, f2_pack(w[2 * j], w[2 * j + 1]), f2_pack(b[2 * j], b[2 * j + 1])));
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
}

/*
 * Epilogue that quantizes the layer's output for the next linear instead of
 * writing it: per row, BF16(acc + bias) (then BF16(GELU(.)) when GELU is
 * set) is exactly what the stand-alone path writes to Y, and the MX
 * quantization of those BF16 values is exactly what the stand-alone
 * quantizer computes from Y.  A thread owns one output row of the warp's
 * 128 columns, i.e. four whole 32-element blocks, so the block maximum is a
 * per-thread reduction.  The accumulator is packed to BF16 pairs first,
 * which halves the registers it holds and leaves room for the GELU's
 * independent chains.  Codes leave as two 32-row x 64-byte boxes through the
 * warp's swizzled staging buffer (TMA store, clipped at M); the four scale
 * bytes of the row form one 32-bit word of the tensor-core scale layout
 * (row r of atom (r / 128, col / 128) at byte (r % 32) * 16 + (r / 32 % 4) *
 * 4), written directly.  Rows in [M, m_pad) get zero scale words, as the
 * stand-alone quantizer writes for its padding rows.
 */
template <bool GELU>
__device__ __forceinline__ void epilogue_quantize(const uint32_t (&acc)[128], const GemmParams &p,
                                                  const CUtensorMap *tmap_q, int row0, int col0, int lane,
                                                  uint32_t buf, uint32_t rowbase, uint32_t swz)
{
    if (col0 >= p.N || row0 >= p.m_pad) /* warp-uniform: N % 128 == 0 */
        return;
    const int row = row0 + lane;
    uint32_t sword = 0u;
    if (row0 < p.M) {
        uint32_t y[64]; /* BF16 pairs: columns 2i, 2i + 1 */
#pragma unroll
        for (int j8 = 0; j8 < 16; ++j8) {
            float b[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (p.bias) {
                const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(p.bias + col0 + 8 * j8));
                const __half2 *bh = reinterpret_cast<const __half2 *>(&bv);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f2 = __half22float2(bh[j]);
                    b[2 * j] = f2.x;
                    b[2 * j + 1] = f2.y;
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int a = 8 * j8 + 2 * j;
                y[4 * j8 + j] = f32x2_to_bf16x2(f2_add(f2_pack(__uint_as_float(acc[a]), __uint_as_float(acc[a + 1])),
                                                       f2_pack(b[2 * j], b[2 * j + 1])));
            }
        }
        /* one 32-column block per iteration, always from y[0 .. 15]; the
         * remaining words move down after each block */
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int g = c & 1; /* position inside the 64-column code box */
            if (g == 0) {
                if (lane == 0)
                    bulk_wait_group_read0(); /* previous box has left the buffer */
                __syncwarp();
            }
            if constexpr (GELU) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    y[i] = gelu_tanh_bf16x2(y[i]);
            }
            /* non-negative BF16 bit patterns order like their values */
            uint32_t m2 = 0u;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                m2 = __vmaxu2(m2, y[i] & 0x7FFF7FFFu);
            const uint32_t sb = scale_byte_from_amax(max(m2 << 16, m2 & 0xFFFF0000u));
            sword |= sb << (8 * c);
            uint32_t o[8];
            if (sb == 0xFFu) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    o[i] = 0x7F7F7F7Fu;
            } else {
                const float m = inv_scale(sb);
                const f32x2 mm = f2_pack(m, m);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float c0, c1, c2, c3;
                    f2_unpack(f2_mul(bf16x2_to_f32x2(y[2 * i]), mm), c0, c1);
                    f2_unpack(f2_mul(bf16x2_to_f32x2(y[2 * i + 1]), mm), c2, c3);
                    o[i] = pack4_e4m3(c0, c1, c2, c3);
                }
            }
            st_shared_v4(rowbase + ((((uint32_t)(2 * g)) ^ swz) << 4), o[0], o[1], o[2], o[3]);
            st_shared_v4(rowbase + ((((uint32_t)(2 * g + 1)) ^ swz) << 4), o[4], o[5], o[6], o[7]);
            if (g == 1) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(tmap_q, col0 + 64 * (c >> 1), row0, buf);
                    bulk_commit_group();
                }
            }
#pragma unroll
            for (int i = 0; i < 48; ++i)
                y[i] = y[i + 16];
        }
    }
    if (row < p.m_pad) {
        const int64_t off = (((int64_t)(row >> 7) * p.sf_kgroups + (col0 >> 7)) << 9) + ((row & 31) << 4) +
                            (((row >> 5) & 3) << 2);
        *reinterpret_cast<uint32_t *>(p.S + off) = row < p.M ? sword : 0u;
    }
}

template <bool PAIR, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    mxfp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmParams p)
{
    constexpr bool FP4 = EPI == EPI_NVFP4;  /* packed E2M1 operands, UE4M3 scales per 16 */
    using C = Cfg<PAIR, FP4>;
    constexpr bool BS = EPI != EPI_ROWWISE; /* block scales (else per-channel FP8) */
    constexpr uint32_t STAGE_TX = BS ? C::STAGE_TX : (C::A_BYTES + C::B_BYTES) * (PAIR ? 2u : 1u);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u; /* 0 = leader */
    const int tile0 = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
    const int tstep = PAIR ? (int)nclusters_x() : (int)gridDim.x;

    const uint32_t bar_full = sbase + C::OFF_BAR;          /* + 8 s */
    const uint32_t bar_empty = bar_full + C::STAGES * 8;   /* + 8 s */
    const uint32_t bar_sffull = bar_empty + C::STAGES * 8; /* + 8 s */
    const uint32_t bar_tfull = bar_sffull + C::STAGES * 8; /* + 8 b, accumulator b */
    const uint32_t bar_tempty = bar_tfull + 2 * 8;        /* + 8 b */
    const uint32_t bar_drain = bar_tempty + 2 * 8;
    /* Accumulators in TMEM: with block scales the scale columns take the
     * upper half, so one; without them (per-channel FP8) two, and the MMA
     * runs the next tile while the epilogue drains the last.  Tile number
     * u uses accumulator acc_buf(u) for the acc_use(u)-th time. */
    constexpr uint32_t NACC = BS ? 1u : 2u;
    auto acc_buf = [](uint32_t u) { return NACC == 2u ? (u & 1u) : 0u; };
    auto acc_use = [](uint32_t u) { return NACC == 2u ? (u >> 1) : u; };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + C::OFF_TMEMPTR);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_ABORT);

    if (threadIdx.x == 0) {
        *abort_flag = 0u;
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
            mbar_init(bar_sffull + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, C::TEMPTY_ARRIVALS);
        }
        mbar_init(bar_drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_ptr), TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_ptr), TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR)
        cluster_sync_all(); /* peer barriers initialised before any remote signal */
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    const int KB = (p.K + BK - 1) / BK; /* a partial last step reads zeros past K */
    const int num_tiles = p.num_m * p.num_n;
    const unsigned long long lim = p.timeout_ns;

    if (warp == 0) {
        /* ------------------------------------------------ TMA producer */
        if (lane == 0) {
            prefetch_tmap(&tmap_a);
            prefetch_tmap(&tmap_b);
            if constexpr (BS) {
                prefetch_tmap(&tmap_sfa);
                prefetch_tmap(&tmap_sfb);
            }
            uint32_t it = 0;
            bool ok = true;
            for (int t = tile0; ok && t < num_tiles; t += tstep) {
                int mb, nb;
                tile_coords(t, p.num_m, p.num_n, p.raster, mb, nb);
                const int rowA = mb * C::TILE_M + (int)(rank * 128u);
                const int rowB = nb * C::TILE_N + (int)(rank * C::B_ROWS);
                const int rbA = rowA / 128;
                const int rbB = nb * 2;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES, ph = (it / C::STAGES) & 1u;
                    if (!wait_bounded(bar_empty + 8 * s, ph ^ 1u, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = bar_full + 8 * s;
                    if (rank == 0)
                        mbar_arrive_expect_tx(full, STAGE_TX);
                    const uint32_t dA = sbase + C::OFF_A + s * C::A_BYTES;
                    const uint32_t dB = sbase + C::OFF_B + s * C::B_BYTES;
                    const uint32_t dSA = sbase + C::OFF_SFA + s * C::SFA_BYTES;
                    const uint32_t dSB = sbase + C::OFF_SFB + s * C::SFB_BYTES;
                    if constexpr (PAIR) {
                        const uint32_t lead = mapa_shared(full, 0u);
                        tma_load_2d_pair(dA, &tmap_a, kb * BK, rowA, lead);
                        tma_load_2d_pair(dB, &tmap_b, kb * BK, rowB, lead);
                        if constexpr (BS) {
                            tma_load_3d_pair(dSA, &tmap_sfa, 0, kb * C::K_ATOMS, rbA, lead);
                            tma_load_3d_pair(dSB, &tmap_sfb, 0, kb * C::K_ATOMS, rbB, lead);
                        }
                    } else {
                        tma_load_2d(dA, &tmap_a, kb * BK, rowA, full);
                        tma_load_2d(dB, &tmap_b, kb * BK, rowB, full);
                        if constexpr (BS) {
                            tma_load_3d(dSA, &tmap_sfa, 0, kb * C::K_ATOMS, rbA, full);
                            tma_load_3d(dSB, &tmap_sfb, 0, kb * C::K_ATOMS, rbB, full);
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        /* ------------------------------------------------ MMA issuer */
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = FP4  ? idesc_nvf4(C::TILE_M, C::TILE_N)
                                   : BS ? idesc_mxf8_e4m3(C::TILE_M, C::TILE_N)
                                        : idesc_f8_e4m3(C::TILE_M, C::TILE_N);
            uint32_t it = 0, tl = 0;
            bool ok = true, any = false;
            for (int t = tile0; ok && t < num_tiles; t += tstep, ++tl) {
                const uint32_t ab = acc_buf(tl);
                const uint32_t tacc = tmem + ACC_COL + 256u * ab;
                if (!wait_bounded(bar_tempty + 8 * ab, (acc_use(tl) & 1u) ^ 1u, lim, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES, ph = (it / C::STAGES) & 1u;
                    if (!wait_bounded(bar_full + 8 * s, ph, lim, abort_flag) ||
                        (PAIR && BS && !wait_bounded(bar_sffull + 8 * s, ph, lim, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tsfa = tmem + C::SFA_COL + C::SFA_STEP * s;
                    const uint32_t tsfb = tmem + C::SFB_COL + C::SFB_STEP * s;
                    const uint32_t sfa_s = sbase + C::OFF_SFA + s * C::SFA_BYTES;
                    const uint32_t sfb_s = sbase + C::OFF_SFB + s * C::SFB_BYTES;
                    const uint64_t adesc = desc_kmajor_sw128(sbase + C::OFF_A + s * C::A_BYTES);
                    const uint64_t bdesc = desc_kmajor_sw128(sbase + C::OFF_B + s * C::B_BYTES);
                    if constexpr (!BS) {
                        (void)tsfa;
                        (void)tsfb;
                        (void)sfa_s;
                        (void)sfb_s;
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k) {
                            if constexpr (PAIR)
                                tc_mma_f8_pair(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k),
                                               idesc, (kb | k) != 0);
                            else
                                tc_mma_f8(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                          (kb | k) != 0);
                        }
                        if constexpr (PAIR)
                            tc_commit_pair(bar_empty + 8 * s, (uint16_t)0x3);
                        else
                            tc_commit(bar_empty + 8 * s);
                    } else if constexpr (PAIR) {
                        /* scales were copied to TMEM by the scale warp */
                        (void)sfa_s;
                        (void)sfb_s;
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k) {
                            if constexpr (FP4) /* K = 64: scale atom k of A, atoms k of both B halves */
                                tc_mma_nvf4_pair(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                                 tsfa + 4u * k, tsfb + 8u * k, (kb | k) != 0);
                            else /* K = 32: byte k of every scale word */
                                tc_mma_mxf8_pair(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k),
                                                 idesc_with_sf_id(idesc, (uint32_t)k), tsfa, tsfb, (kb | k) != 0);
                        }
                        tc_commit_pair(bar_empty + 8 * s, (uint16_t)0x3);
                    } else {
#pragma unroll
                        for (int k = 0; k < C::K_ATOMS; ++k) {
                            tc_cp_32x128b_warpx4(tsfa + 4u * k, desc_sf_32x16(sfa_s + 512u * k));
                            tc_cp_32x128b_warpx4(tsfb + 8u * k, desc_sf_32x16(sfb_s + 512u * k));
                            tc_cp_32x128b_warpx4(tsfb + 8u * k + 4u, desc_sf_32x16(sfb_s + 512u * (C::K_ATOMS + k)));
                        }
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k) {
                            if constexpr (FP4)
                                tc_mma_nvf4(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                            tsfa + 4u * k, tsfb + 8u * k, (kb | k) != 0);
                            else
                                tc_mma_mxf8(tacc, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k),
                                            idesc_with_sf_id(idesc, (uint32_t)k), tsfa, tsfb, (kb | k) != 0);
                        }
                        tc_commit(bar_empty + 8 * s);
                    }
                    any = true;
                }
                if (!ok)
                    break;
                if constexpr (PAIR)
                    tc_commit_pair(bar_tfull + 8 * ab, (uint16_t)0x3);
                else
                    tc_commit(bar_tfull + 8 * ab);
            }
            if (ok) {
                /* every epilogue (the peer's included) has released the last
                 * accumulators, so no remote arrival is still in flight */
                for (uint32_t u = tl > NACC ? tl - NACC : 0u; u < tl; ++u)
                    (void)wait_bounded(bar_tempty + 8 * acc_buf(u), acc_use(u) & 1u, lim, abort_flag);
            }
            if (!ok && any) {
                /* wait for this thread's MMAs and copies before TMEM is freed */
                volatile uint32_t own = 0u;
                if constexpr (PAIR)
                    tc_commit_pair(bar_drain, (uint16_t)0x1);
                else
                    tc_commit(bar_drain);
                (void)wait_bounded(bar_drain, 0u, lim, &own);
            }
        }
    } else if (warp == SF_WARP) {
        /* ------------------------------------------------ scale copies */
        /* The pair-wide tcgen05.cp holds up the thread that issues it, so it
         * is issued here, one stage at a time, and the MMA thread only waits
         * for its completion (sf_full), never for the copy itself. */
        if (PAIR && BS && lane == 0 && rank == 0) {
            uint32_t it = 0;
            for (int t = tile0; t < num_tiles; t += tstep) {
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES, ph = (it / C::STAGES) & 1u;
                    if (!wait_bounded(bar_full + 8 * s, ph, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tsfa = tmem + C::SFA_COL + C::SFA_STEP * s;
                    const uint32_t tsfb = tmem + C::SFB_COL + C::SFB_STEP * s;
                    const uint32_t sfa_s = sbase + C::OFF_SFA + s * C::SFA_BYTES;
                    const uint32_t sfb_s = sbase + C::OFF_SFB + s * C::SFB_BYTES;
                    /* atom k of A to 4 columns; atoms k of the two B row halves to 8 */
#pragma unroll
                    for (int k = 0; k < C::K_ATOMS; ++k) {
                        tc_cp_32x128b_warpx4_pair(tsfa + 4u * k, desc_sf_32x16(sfa_s + 512u * k));
                        tc_cp_32x128b_warpx4_pair(tsfb + 8u * k, desc_sf_32x16(sfb_s + 512u * k));
                        tc_cp_32x128b_warpx4_pair(tsfb + 8u * k + 4u, desc_sf_32x16(sfb_s + 512u * (C::K_ATOMS + k)));
                    }
                    tc_commit_pair(bar_sffull + 8 * s, (uint16_t)0x1);
                }
                if (!ok)
                    break;
            }
        }
    } else {
        /* ------------------------------------------------ epilogue */
        /* NVFP4: alpha = 1 / (g_x g_w); the product of two binary32 values is
         * exact in binary64, the quotient rounded once there, then to binary32 */
        const float alpha = EPI == EPI_NVFP4 ? (float)(1.0 / ((double)__ldg(p.gx) * (double)__ldg(p.gw))) : 1.0f;
        const int q = warp & 3;            /* TMEM sub-partition this warp may read */
        const int h = (warp - 2) >> 2;     /* column half of the 256-wide tile */
        uint32_t tl = 0;
        for (int t = tile0; t < num_tiles; t += tstep, ++tl) {
            int mb, nb;
            tile_coords(t, p.num_m, p.num_n, p.raster, mb, nb);
            /* every lane polls; the vote keeps the warp converged for the
             * .sync.aligned TMEM load and makes the outcome warp-uniform */
            const uint32_t ab = acc_buf(tl);
            const bool got = wait_bounded(bar_tfull + 8 * ab, acc_use(tl) & 1u, lim, abort_flag, SUSPEND_EPI);
            if (!__all_sync(0xFFFFFFFFu, got))
                break;
            tc_fence_after();
            uint32_t acc[128];
            tmem_ld_32x32b_x128_sync(tmem + ((uint32_t)(32 * q) << 16) + ACC_COL + 256u * ab + (uint32_t)(h * 128),
                                     acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR)
                    mbar_arrive_cluster(mapa_shared(bar_tempty + 8 * ab, 0u));
                else
                    mbar_arrive(bar_tempty + 8 * ab);
            }

            const int row0 = mb * C::TILE_M + (int)(rank * 128u) + 32 * q;
            const int col0 = nb * C::TILE_N + h * 128;
            const uint32_t buf = sbase + C::OFF_EPI + (uint32_t)(warp - 2) * C::EPI_BUF;
            const uint32_t rowbase = buf + (uint32_t)lane * 64u;
            const uint32_t swz = ((uint32_t)lane >> 1) & 3u;
            if constexpr (EPI == EPI_BF16)
                epilogue_bf16<false>(acc, p, 1.0f, &tmap_y, row0, col0, lane, buf, rowbase, swz);
            else if constexpr (EPI == EPI_NVFP4)
                epilogue_bf16<true>(acc, p, alpha, &tmap_y, row0, col0, lane, buf, rowbase, swz);
            else if constexpr (EPI == EPI_ROWWISE)
                epilogue_rowwise(acc, p, &tmap_y, row0, col0, lane, buf, rowbase, swz);
            else
                epilogue_quantize<EPI == EPI_QUANT_GELU>(acc, p, &tmap_y, row0, col0, lane, buf, rowbase, swz);
        }
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
    if constexpr (PAIR)
        cluster_sync_all(); /* neither CTA leaves while the pair may still touch it */
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        if constexpr (PAIR)
            tmem_dealloc_pair(tmem, TMEM_COLS);
        else
            tmem_dealloc(tmem, TMEM_COLS);
    }
}

/* Self-test of the GEMM's bounded wait: one thread waits on an mbarrier
 * that nothing arrives at; after limit_ns the wait gives up and records
 * ST_TIMEOUT in the status word, as a stalled pipeline would.  Nothing else
 * is in flight, so the kernel simply returns. */
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
/* K-major E4M3 operand [rows, K]: box 128 (K bytes) x box_rows, 128-byte swizzle. */
static bool make_operand_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K, uint32_t box_rows)
{
    return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, K, rows, K, (uint32_t)BK, box_rows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

/* Scale array in the tensor-core layout viewed as [row blocks][kg][128 u32]
 * (one 512-byte atom per (row block, K group): kg = K / 128 groups of E8M0
 * scales for MXFP8, K / 64 of UE4M3 scales for NVFP4); box = `katoms`
 * consecutive K groups of `atoms` consecutive row blocks (shared-memory order
 * [row block][K group][512 B]).  Atoms past the end read as zero. */
static bool make_scale_map(CUtensorMap *m, const void *base, int64_t rows, int64_t kg, uint32_t katoms,
                           uint32_t atoms)
{
    PFN_encodeTiled enc = get_encode_fn();
    if (!enc)
        return false;
    const int64_t rb = (rows + 127) / 128;
    cuuint64_t dims[3] = {128, (cuuint64_t)kg, (cuuint64_t)rb};
    cuuint64_t strides[2] = {512, (cuuint64_t)(kg * 512)};
    cuuint32_t box[3] = {128, katoms, atoms};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

/* BF16 output Y [M, N]: box 32 columns x 32 rows, 64-byte swizzle (the
 * epilogue's staging layout); stores are clipped at M and N. */
static bool make_output_map(CUtensorMap *m, void *base, int64_t M, int64_t N)
{
    return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

/* MXFP8 codes out [M, N] (quantizing epilogues): box 64 bytes x 32 rows,
 * 64-byte swizzle (same staging layout as the BF16 boxes); clipped at M. */
static bool make_codes_out_map(CUtensorMap *m, void *base, int64_t M, int64_t N)
{
    return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, N, M, N, 64, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

struct DevInfo {
    bool init = false;
    int sms = 148;
    bool pair_checked = false;
    int max_pair_clusters = 0;   /* 0: pairs unavailable */
    bool attr[2][4] = {};        /* [PAIR][EPI]: shared-memory attribute set */
};
static DevInfo g_dev[64];

static DevInfo *dev_info()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    DevInfo &d = g_dev[dev];
    if (!d.init) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            d.sms = v;
        d.init = true;
    }
    return &d;
}

template <bool PAIR, int EPI>
constexpr uint32_t smem_bytes()
{
    return Cfg<PAIR, EPI == EPI_NVFP4>::SMEM_BYTES;
}

template <bool PAIR, int EPI>
static cudaError_t ensure_attr(DevInfo *d)
{
    if (d->attr[PAIR][EPI])
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(mxfp8_gemm_kernel<PAIR, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<PAIR, EPI>());
    if (e == cudaSuccess)
        d->attr[PAIR][EPI] = true;
    return e;
}

static void pair_config(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr, unsigned grid, cudaStream_t stream,
                        uint32_t smem)
{
    cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(GEMM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

/* How many CTA pairs can be resident at once (0: pairs unavailable). */
static void check_pairs(DevInfo *d)
{
    if (d->pair_checked)
        return;
    d->pair_checked = true;
    if (ensure_attr<true, EPI_BF16>(d) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    pair_config(cfg, attr, 2 * (unsigned)d->sms, nullptr, smem_bytes<true, EPI_BF16>());
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, mxfp8_gemm_kernel<true, EPI_BF16>, &cfg) == cudaSuccess)
        d->max_pair_clusters = n;
    else
        cudaGetLastError(); /* clear; fall back to single CTAs */
}

template <bool PAIR, int EPI>
static cudaError_t launch_variant(DevInfo *d, const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &msa,
                                  const CUtensorMap &msb, const CUtensorMap &my, const GemmParams &p, int grid,
                                  cudaStream_t stream)
{
    cudaError_t e = ensure_attr<PAIR, EPI>(d);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    if (PAIR) {
        pair_config(cfg, attr, (unsigned)grid, stream, smem_bytes<PAIR, EPI>());
    } else {
        cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(GEMM_THREADS);
        cfg.dynamicSmemBytes = smem_bytes<PAIR, EPI>();
        cfg.stream = stream;
    }
    return cudaLaunchKernelEx(&cfg, mxfp8_gemm_kernel<PAIR, EPI>, ma, mb, msa, msb, my, p);
}

template <bool PAIR>
static cudaError_t launch_mode(DevInfo *d, int epi, const CUtensorMap &ma, const CUtensorMap &mb,
                               const CUtensorMap &msa, const CUtensorMap &msb, const CUtensorMap &my,
                               const GemmParams &p, int grid, cudaStream_t stream)
{
    switch (epi) {
    case EPI_QUANT:
        return launch_variant<PAIR, EPI_QUANT>(d, ma, mb, msa, msb, my, p, grid, stream);
    case EPI_QUANT_GELU:
        return launch_variant<PAIR, EPI_QUANT_GELU>(d, ma, mb, msa, msb, my, p, grid, stream);
    case EPI_ROWWISE:
        return launch_variant<PAIR, EPI_ROWWISE>(d, ma, mb, msa, msb, my, p, grid, stream);
    case EPI_NVFP4:
        return launch_variant<PAIR, EPI_NVFP4>(d, ma, mb, msa, msb, my, p, grid, stream);
    default:
        return launch_variant<PAIR, EPI_BF16>(d, ma, mb, msa, msb, my, p, grid, stream);
    }
}

/* Whether the CTA-pair variant is used: on unless MXFP8_GEMM_PAIR=0. */
static bool pair_enabled()
{
    static int v = -1;
    if (v < 0) {
        const char *e = getenv("MXFP8_GEMM_PAIR");
        v = (e && e[0] == '0') ? 0 : 1;
    }
    return v == 1;
}

/*
 * epi = 0: Y is BF16 [M, N], S unused.  epi = 1 / 2: Y receives E4M3 codes
 * [M, N] and S the tensor-core scales of [M, N] (2: GELU before the
 * quantization); N % 128 == 0.  epi = 3 (per-channel FP8): Xs / Ws are FP32
 * row scales [M] / [N], Y is BF16 [M, N].  epi = 4 (NVFP4): Xq / Wq are packed
 * E2M1 codes [M, K/2] / [N, K/2], Xs / Ws their UE4M3 scales in the
 * tensor-core layout of 16-element blocks, gx / gw the device global scales,
 * Y is BF16 [M, N]; K % 64 == 0.
 * Returns 0 ok, 1 tensor-map failure, 2 CUDA error (in *err).
 */
int launch_gemm(const void *Xq, const void *Xs, int64_t M, int64_t K, const void *Wq, const void *Ws, int64_t N,
                const void *bias, void *Y, int epi, void *S, cudaStream_t stream, unsigned long long timeout_ns,
                cudaError_t *err, const float *gx, const float *gw)
{
    const bool bs = epi != EPI_ROWWISE;
    const bool fp4 = epi == EPI_NVFP4;
    const int64_t kbytes = fp4 ? K / 2 : K; /* operand row bytes */
    *err = cudaSuccess;
    if (M == 0)
        return 0;
    DevInfo *d = dev_info();
    if (!d) {
        *err = cudaErrorInvalidDevice;
        return 2;
    }
    bool pair = pair_enabled();
    if (pair) {
        check_pairs(d);
        if (d->max_pair_clusters <= 0)
            pair = false;
    }

    const uint32_t b_rows = pair ? Cfg<true>::B_ROWS : Cfg<false>::B_ROWS;
    CUtensorMap ma, mb, msa, msb, my;
    const bool out_ok = (epi == EPI_BF16 || epi == EPI_ROWWISE || fp4) ? make_output_map(&my, Y, M, N)
                                                                         : make_codes_out_map(&my, Y, M, N);
    if (!make_operand_map(&ma, Xq, M, kbytes, 128) || !make_operand_map(&mb, Wq, N, kbytes, b_rows) || !out_ok)
        return 1;
    if (bs) {
        /* K groups of scale atoms: 128 elements (E8M0) or 64 (UE4M3); the
         * GEMM takes one group per 128-byte step, or four */
        const int64_t kg = fp4 ? (K + 63) / 64 : K / 128;
        const uint32_t katoms = fp4 ? 4u : 1u;
        if (!make_scale_map(&msa, Xs, M, kg, katoms, 1) || !make_scale_map(&msb, Ws, N, kg, katoms, 2))
            return 1;
    } else {
        msa = ma; /* not read without block scales */
        msb = mb;
    }
    GemmParams p;
    p.bias = static_cast<const __half *>(bias);
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.S = static_cast<uint8_t *>(S);
    p.sx = bs ? nullptr : static_cast<const float *>(Xs);
    p.sw = bs ? nullptr : static_cast<const float *>(Ws);
    p.gx = gx;
    p.gw = gw;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)kbytes;
    p.m_pad = (int)((M + 127) / 128 * 128);
    p.sf_kgroups = (int)(N / 128);
    const int tile_m = pair ? Cfg<true>::TILE_M : Cfg<false>::TILE_M;
    p.num_m = (int)((M + tile_m - 1) / tile_m);
    p.num_n = (int)((N + 255) / 256);
    const int64_t n_fit =
        std::min<int64_t>(p.num_n, RASTER_B_GROUP_BYTES / ((int64_t)Cfg<true>::TILE_N * kbytes));
    if (n_fit >= RASTER_MIN_N_GROUP) {
        const int64_t groups = (p.num_n + n_fit - 1) / n_fit;
        p.raster = -(int)((p.num_n + groups - 1) / groups);
    } else
        p.raster = (int64_t)N * kbytes > RASTER_LARGE_B_BYTES ? RASTER_LARGE_B : RASTER_SMALL_B;
    p.timeout_ns = timeout_ns;
    const int tiles = p.num_m * p.num_n;
    cudaError_t e;
    if (pair) {
        int clusters = d->max_pair_clusters;
        if (clusters > tiles)
            clusters = tiles;
        e = launch_mode<true>(d, epi, ma, mb, msa, msb, my, p, 2 * clusters, stream);
    } else {
        int grid = d->sms;
        if (grid > tiles)
            grid = tiles;
        e = launch_mode<false>(d, epi, ma, mb, msa, msb, my, p, grid, stream);
    }
    if (e != cudaSuccess) {
        *err = e;
        return 2;
    }
    return 0;
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t stream)
{
    wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

/* Reads and clears the status word of the current device (synchronous). */
cudaError_t read_and_clear_status(unsigned int *out)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_mx_status, sizeof(unsigned int));
    if (e != cudaSuccess)
        return e;
    return cudaMemcpyToSymbol(g_mx_status, &zero, sizeof(unsigned int));
}

} // namespace mx
