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
 * Roles (320 threads per CTA):
 *   warp 0      TMA producer: per 256-wide K step ("raw stage") the CTA's
 *               128 x 128-byte boxes of A and B codes (128-byte swizzle) and
 *               the four 512-byte scale atoms of its A rows and B rows (one
 *               bulk copy each), into a 2-deep ring.
 *   warp 1      allocates 256 TMEM columns; in the leader CTA one thread
 *               issues, per 64-wide K step, four kind::f16 MMAs of K = 16
 *               and commits the step's release to both CTAs.
 *   warps 2..9  expand and write back.  Each thread owns one row (threads
 *               0..127 of A, 128..255 of B) and, per 64-wide K step, turns
 *               its 32 code bytes and 4 scale bytes into 64 FP16 values
 *               (cvt.rn.f16x2.e2m1x2, exact multiply by the scale) stored in
 *               the 128-byte-swizzled K-major layout the MMA reads, into a
 *               4-deep ring; the generic-proxy stores are fenced to the async
 *               proxy and announced to the leader's barrier (16 arrivals per
 *               step, both CTAs).  Between K steps, once the next tile's
 *               first ring slots are filled, the same warps drain the
 *               finished accumulator (one tcgen05.ld of 32 lanes x 128
 *               columns per warp), release it at once, and write Y through
 *               swizzled smem boxes and TMA stores.
 * Every wait is bounded: on timeout the kernel records the timeout in a
 * device status word, drains its own MMAs, frees TMEM and returns.
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

constexpr int XW = 8;                    /* expand / epilogue warps */
constexpr int THREADS = (2 + XW) * 32;
constexpr int FS = 4;                    /* FP16 operand stages */
constexpr int RS = 2;                    /* code / scale stages */
constexpr int KF = 64;                   /* K elements per FP16 stage (128-byte rows) */
constexpr int KR = 256;                  /* K elements per code stage (128 bytes of codes per row) */
constexpr int SUB = KR / KF;             /* FP16 stages per code stage */
constexpr int TILE_M = 256, TILE_N = 256;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TILE_BYTES = 128 * 128; /* 128 rows x 128 bytes */
constexpr uint32_t SF_BYTES = SUB * 512;   /* four 64-wide scale atoms of 128 rows */
constexpr uint32_t OFF_FA = 0;
constexpr uint32_t OFF_FB = OFF_FA + FS * TILE_BYTES;
constexpr uint32_t OFF_RA = OFF_FB + FS * TILE_BYTES;
constexpr uint32_t OFF_RB = OFF_RA + RS * TILE_BYTES;
constexpr uint32_t OFF_SA = OFF_RB + RS * TILE_BYTES;
constexpr uint32_t OFF_SB = OFF_SA + RS * SF_BYTES;
constexpr uint32_t OFF_EPI = OFF_SB + RS * SF_BYTES;
constexpr uint32_t EPI_BUF = 32 * 32 * 2; /* 32 rows x 32 BF16 */
constexpr uint32_t OFF_BAR = OFF_EPI + XW * EPI_BUF;
/* full[FS], empty[FS], rfull[RS], rempty[RS], tfull, tempty, drain */
constexpr uint32_t NUM_BARS = 2 * FS + 2 * RS + 3;
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + NUM_BARS * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t SMEM_USED = OFF_TMEMPTR + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024; /* slack to align the base to 1 KiB */
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_EPI % 1024 == 0 && OFF_RA % 1024 == 0, "swizzled buffers must be 1 KiB aligned");
constexpr int RASTER_SMALL_B = 8, RASTER_LARGE_B = 16;
constexpr int64_t RASTER_LARGE_B_BYTES = 48ll << 20; /* weight bytes above which 16 M tiles share a group */
constexpr uint32_t SUSPEND_NS = 1000000u;
constexpr uint32_t ST_TIMEOUT = 1u;

__device__ unsigned int g_nv_status = 0;

struct Params {
    const uint8_t *sfa;  /* activation scales, tensor-core layout of 16-element blocks */
    const uint8_t *sfb;  /* weight scales, same layout */
    const __half *bias;  /* [N] or null */
    float alpha;
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
/* Wait with acquire at cluster scope: the phase was completed by arrivals
 * (release, cluster scope) of threads in both CTAs of the pair. */
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity, uint32_t suspend_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(suspend_ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
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
/* UE4M3 scale byte -> the FP16 pair (dec(s), dec(s)) */
__device__ __forceinline__ uint32_t scale_pair(uint32_t sbyte)
{
    uint32_t d;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}\n"
        : "=r"(d)
        : "r"(sbyte * 0x101u));
    return d;
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
    nb = r / gm;
}

/*
 * Bounded wait: true when the phase of parity `parity` has completed.  On
 * timeout it records ST_TIMEOUT in the device status word and raises the
 * CTA's abort flag, so the other roles stop waiting too.
 */
template <bool CLUSTER>
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, unsigned long long limit_ns,
                                             volatile uint32_t *abort_flag)
{
    auto probe = [&]() {
        return CLUSTER ? mbar_try_wait_cluster(bar, parity, SUSPEND_NS) : mbar_try_wait(bar, parity, SUSPEND_NS);
    };
    if (probe())
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (probe())
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
    const bool ok = wait_bounded<false>(bar, parity, limit_ns, abort_flag);
    return __all_sync(0xFFFFFFFFu, ok);
}

/*
 * One thread, one row, one 64-wide K step: 32 code bytes (two 16-byte
 * chunks of the row's 128-byte swizzled code line) and the row's 4 scale
 * bytes of the step's atom -> 64 FP16 values, written as 8 chunks of the
 * 128-byte swizzled FP16 row.
 */
__device__ __forceinline__ void expand_row_step(uint32_t code_row, uint32_t sf_word_addr, bool have_scales, int j,
                                                uint32_t f16_row, uint32_t x)
{
    const uint4 c0 = ld_shared_v4(code_row + ((((uint32_t)(2 * j)) ^ x) << 4));
    const uint4 c1 = ld_shared_v4(code_row + ((((uint32_t)(2 * j + 1)) ^ x) << 4));
    const uint32_t sw = have_scales ? ld_shared_u32(sf_word_addr) : 0u;
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t s2 = scale_pair((sw >> (8 * b)) & 0xFFu);
#pragma unroll
        for (int hch = 0; hch < 2; ++hch) {
            const int c = 2 * b + hch; /* FP16 chunk = 8 elements = one code word */
            uint32_t h0, h1, h2, h3;
            expand_word(w[c], s2, h0, h1, h2, h3);
            st_shared_v4(f16_row + ((((uint32_t)c) ^ x) << 4), h0, h1, h2, h3);
        }
    }
}

/* Y = BF16(alpha acc + bias), 32 columns at a time, staged through a
 * 64-byte-swizzled smem box and written by one TMA store per warp. */
__device__ __forceinline__ void epilogue_store(const uint32_t (&acc)[128], const Params &p, const CUtensorMap *tmap_y,
                                               int row0, int col0, int lane, uint32_t buf, uint32_t rowbase,
                                               uint32_t swz)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int colc = col0 + 32 * c;
        if (row0 >= p.M || colc >= p.N)
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
                __nv_bfloat162 v = __floats2bfloat162_rn(fmaf(p.alpha, __uint_as_float(acc[a]), b[2 * j]),
                                                         fmaf(p.alpha, __uint_as_float(acc[a + 1]), b[2 * j + 1]));
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
    const uint32_t bar_tfull = bar_rempty + RS * 8;
    const uint32_t bar_tempty = bar_tfull + 8;
    const uint32_t bar_drain = bar_tempty + 8;
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
        mbar_init(bar_tfull, 1);
        mbar_init(bar_tempty, 2 * XW);
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
                    if (!wait_bounded<false>(bar_rempty + 8 * s, ph ^ 1u, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int n_at = min(SUB, p.kg - SUB * kr);
                    const uint32_t sf_bytes = (uint32_t)n_at * 512u;
                    const uint32_t full = bar_rfull + 8 * s;
                    mbar_arrive_expect_tx(full, 2u * TILE_BYTES + (a_in ? sf_bytes : 0u) + (b_in ? sf_bytes : 0u));
                    tma_load_2d(sbase + OFF_RA + s * TILE_BYTES, &tmap_a, kr * 128, rowA, full);
                    tma_load_2d(sbase + OFF_RB + s * TILE_BYTES, &tmap_b, kr * 128, rowB, full);
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
                if (!wait_bounded<true>(bar_tempty, (tl & 1u) ^ 1u, lim, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % FS, ph = (it / FS) & 1u;
                    if (!wait_bounded<true>(bar_full + 8 * s, ph, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = desc_kmajor_sw128(sbase + OFF_FA + s * TILE_BYTES);
                    const uint64_t bdesc = desc_kmajor_sw128(sbase + OFF_FB + s * TILE_BYTES);
#pragma unroll
                    for (int k = 0; k < KF / 16; ++k)
                        tc_mma_f16_pair(tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                        (kb | k) != 0);
                    tc_commit_pair(bar_empty + 8 * s, (uint16_t)0x3);
                    any = true;
                }
                if (!ok)
                    break;
                tc_commit_pair(bar_tfull, (uint16_t)0x3);
            }
            if (ok && tl > 0) {
                /* every epilogue (the peer's included) has released the last
                 * accumulator, so no remote arrival is still in flight */
                (void)wait_bounded<true>(bar_tempty, (tl & 1u) ^ 1u, lim, abort_flag);
            }
            if (!ok && any) {
                /* wait for this thread's MMAs before TMEM is freed */
                volatile uint32_t own = 0u;
                tc_commit_pair(bar_drain, (uint16_t)0x1);
                (void)wait_bounded<false>(bar_drain, 0u, lim, &own);
            }
        }
    } else {
        /* ------------------------------------- expand + epilogue warps */
        const int e = (warp - 2) * 32 + lane;
        const int op = e >> 7; /* 0: A row, 1: B row */
        const int r = e & 127;
        const uint32_t x = (uint32_t)(r & 7);
        const uint32_t sf_off = (uint32_t)((r & 31) * 16 + ((r >> 5) & 3) * 4);
        const uint32_t code_base = sbase + (op ? OFF_RB : OFF_RA) + (uint32_t)r * 128u;
        const uint32_t sf_base = sbase + (op ? OFF_SB : OFF_SA) + sf_off;
        const uint32_t f16_base = sbase + (op ? OFF_FB : OFF_FA) + (uint32_t)r * 128u;
        const uint32_t tempty_lead = mapa_shared(bar_tempty, 0u);
        /* epilogue geometry: TMEM sub-partition and column half of this warp */
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const uint32_t buf = sbase + OFF_EPI + (uint32_t)(warp - 2) * EPI_BUF;
        const uint32_t rowbase = buf + (uint32_t)lane * 64u;
        const uint32_t swz = ((uint32_t)lane >> 1) & 3u;

        uint32_t it = 0, ir = 0, tl = 0;
        bool ok = true;
        bool pending = false;
        int pend_t = 0;
        /* drains the accumulator of tile pend_t and writes its Y */
        auto epilogue = [&]() -> bool {
            int mb, nb;
            tile_coords(pend_t, p.num_m, p.num_n, p.raster, mb, nb);
            const bool got = wait_bounded<false>(bar_tfull, tl & 1u, lim, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got))
                return false;
            tc_fence_after();
            uint32_t acc[128];
            tmem_ld_32x32b_x128_sync(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * 128), acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(tempty_lead);
            ++tl;
            const int row0 = mb * TILE_M + (int)(rank * 128u) + 32 * q;
            const int col0 = nb * TILE_N + h * 128;
            epilogue_store(acc, p, &tmap_y, row0, col0, lane, buf, rowbase, swz);
            return true;
        };

        for (int t = tile0; ok && t < num_tiles; t += tstep) {
            int mb, nb;
            tile_coords(t, p.num_m, p.num_n, p.raster, mb, nb);
            const int row_block = op ? nb * TILE_N + (int)(rank * 128u) : mb * TILE_M + (int)(rank * 128u);
            const bool have_scales = row_block < (op ? p.N : p.M);
            for (int kb = 0; kb < KB; ++kb, ++it) {
                if (pending && kb == FS) {
                    pending = false;
                    if (!epilogue()) {
                        ok = false;
                        break;
                    }
                }
                const int j = kb % SUB;
                const uint32_t rs = ir % RS;
                if (j == 0 && !warp_wait(bar_rfull + 8 * rs, (ir / RS) & 1u, lim, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t s = it % FS;
                if (!warp_wait(bar_empty + 8 * s, ((it / FS) & 1u) ^ 1u, lim, abort_flag)) {
                    ok = false;
                    break;
                }
                expand_row_step(code_base + rs * TILE_BYTES, sf_base + rs * SF_BYTES + (uint32_t)j * 512u,
                                have_scales, j, f16_base + s * TILE_BYTES, x);
                fence_proxy_async_smem(); /* generic-proxy stores -> visible to the tensor core */
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_release_cluster(mapa_shared(bar_full + 8 * s, 0u));
                if (j == SUB - 1 || kb == KB - 1) {
                    if (lane == 0)
                        mbar_arrive(bar_rempty + 8 * rs);
                    ++ir;
                }
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
    cluster_sync_all(); /* neither CTA leaves while the pair may still touch it */
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem, TMEM_COLS);
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
                      int64_t N, float alpha, const void *bias, void *Y, cudaStream_t stream,
                      unsigned long long timeout_ns, cudaError_t *err)
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
    if (!encode_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, K / 2, M, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K / 2, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return 1;
    nv::Params p;
    p.sfa = static_cast<const uint8_t *>(Xs);
    p.sfb = static_cast<const uint8_t *>(Ws);
    p.bias = static_cast<const __half *>(bias);
    p.alpha = alpha;
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
