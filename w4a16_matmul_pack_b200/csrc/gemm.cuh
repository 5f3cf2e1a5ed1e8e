// gemm.cuh -- prefill W4A16 GEMM on the 5th-generation tensor cores (sm_100a).
//
// y[m][n] = g * sum_k x[m][k] * (e2m1[n][k] * scale[n][k/16])   (NVFP4 weights,
// "EdgeRock-4B-NVFP4" card, intro; BF16 activations).  e2m1 * scale has at most
// 6 significant bits and lies in [2^-10, 2688], so it is exact in BF16 and in
// f16: the dequant warps write it, per 64-k stage, into tensor memory, where it
// is the A operand of tcgen05.mma kind::f16 (A from TMEM, B = x from shared
// memory, FP32 accumulators in TMEM).  The global scale g is applied in the
// epilogue.
//
// Tile: 128 weight rows (MMA M, A) x 192 tokens (MMA N, B = x, K-major with the
// 128-byte swizzle, staged by TMA) x 64 k per stage.  Tensor memory holds four
// A stages (32 columns each) and two 192-column accumulators (512 columns), so
// the epilogue of a tile overlaps the MMAs of the next.  Persistent CTAs, one
// per SM, walk the tiles n-major so that CTAs running together share the same
// packed weight rows in L2.
//
// Warp roles (15 warps):
//   warp 0      TMA producer: x tiles and the packed codes (128-byte swizzle,
//               256 k per codes stage), no multicast.
//   warp 1      allocates / frees the 512 TMEM columns; MMA issuer (one lane):
//               4 x (128x192x16) per stage, commits to the stage barriers and
//               to the accumulator barrier per tile.  It never waits on an
//               mbarrier: a thread with MMAs queued stalls on any shared-memory
//               access until they drain (measured: one wait per four
//               128x256x16 MMAs turns 128 cycles per MMA into 270), so warp 14
//               waits and releases it through named barrier 2 once per stage.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31), times g (and 2^sigma_m, below), float32 / BF16
//               stores.
//   warps 6-13  dequantise: warp w owns TMEM lanes 32*(w%4)..+31 = weight rows;
//               thread (row r, k-half h) turns 32 codes + 2 scales of row r into
//               16 words and stores them with one tcgen05.st, two stages per
//               round (one store wait and one arrival per round).
//   warp 14     waits on the x / A stage barriers and the accumulator barriers
//               for the MMA issuer.
// Every mbarrier wait is bounded (common.cuh: mbar_wait).
//
// Operand precision per tile of 192 tokens.  In f16, e2m1 * scale costs one cvt
// (E2M1 -> f16x2) and one HMUL2 per pair of weights instead of a round trip
// through binary32.  So when the caller provides a workspace, x_to_f16_kernel
// first converts each token row to f16 as x * 2^-sigma_m (sigma_m from the
// row's largest |x|) and flags the rows it cannot convert exactly (a nonzero
// |x * 2^-sigma_m| below 2^-17, or Inf / NaN).  A tile whose rows all converted
// exactly runs kind::f16 with f16 operands and the epilogue multiplies token m
// by 2^sigma_m; any other tile (or every tile, without a workspace) runs on
// BF16 operands (e2m1 -> f16 -> binary32 * scale -> BF16).
#pragma once

#include "common.cuh"

namespace w4 {

namespace gemm {

constexpr int BM = 128;      // weight rows per tile (MMA M)
constexpr int BN = 192;      // tokens per tile (MMA N)
constexpr int BK = 64;       // k per stage (one 128-byte swizzle row of BF16)
constexpr int STAGES = 4;
constexpr int kWarps = 15;
constexpr int kThreads = kWarps * 32;
constexpr int kDequantThreads = 256;
constexpr int kEpiThreads = 128;
constexpr uint32_t X_STAGE_BYTES = BN * BK * 2;   // 24 KB
constexpr uint32_t TMEM_COLS = 512;               // 4 A stages (32 columns each) + two 192-column accumulators
constexpr uint32_t ACC_COL0 = STAGES * (BK / 2);  // accumulators after the A stages
constexpr int WK = 256;                           // k per packed-weight stage (4 k-steps)
constexpr int WSTAGES = 4;
constexpr uint32_t W_STAGE_BYTES = BM * WK / 2;   // 16 KB of codes (128 rows x 128 bytes)

// Instruction descriptor, kind::f16: D = F32 (bit 4), A = BF16 (bits 7-9),
// B = BF16 (bits 10-12), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
// The same with A = B = F16 (format 0).
constexpr uint32_t IDESC_F16 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr int kMaxTilesM = 256;
constexpr int kWaitWarp = 14;     // waits on mbarriers for the MMA issuer (warp 1)   // token tiles whose operand mode is kept in shared memory (M <= 65536)

struct SharedStorage {
    uint8_t x[STAGES][X_STAGE_BYTES];   // 1024-byte aligned (swizzle atoms)
    uint8_t w[WSTAGES][W_STAGE_BYTES];  // packed codes, 128-byte swizzle
    uint64_t w_full[WSTAGES], w_empty[WSTAGES];
    uint64_t x_full[STAGES], x_empty[STAGES];
    uint64_t a_full[STAGES], a_empty[STAGES];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t mma_done;                  // the issuer's last commit: every MMA has finished
    uint32_t tmem_base;
    int abort;
    int f16_tile[kMaxTilesM];   // token tile mt runs with f16 operands (else BF16)
};

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;            // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset
    d |= (uint64_t)1 << 46;            // version
    d |= (uint64_t)2 << 61;            // SWIZZLE_128B
    return d;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mma_f16kind(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// The same with A from tensor memory (K-major: lane = row, 32-bit column = two k).
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}

#define W4_TMEM_LD32(taddr, v)                                                                              \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                  \
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                                   \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                  \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),       \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),   \
                   "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),             \
                   "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),             \
                   "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])              \
                 : "r"(taddr))

// 4 code bytes (8 E2M1 values, element 2i in the low nibble of byte i) times a
// scale -> 4 BF16x2 words.  Exact.
__device__ __forceinline__ uint4 dequant8(uint32_t cw, float s) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t h = e2m1x2_to_f16x2(cw >> (8 * i));
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
        const float2 v = __fmul2_rn(f, make_float2(s, s));
        const __nv_bfloat162 b = __float22bfloat162_rn(v);
        o[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The same 8 weights as f16x2 words: cvt E2M1 -> f16x2, HMUL2 by the scale
// (s2 = the scale in both halves).  Exact (at most 6 significant bits, in
// [2^-10, 2688]).
__device__ __forceinline__ uint4 dequant8_f16(uint32_t cw, uint32_t s2) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t h = e2m1x2_to_f16x2(cw >> (8 * i));
        const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&h), *reinterpret_cast<const __half2 *>(&s2));
        o[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The power of two a BF16-operand tile folds into its weights: the exponent of
// g, clamped so that e2m1 * scale * 2^fold stays an exact BF16 value (e2m1 *
// scale lies in [2^-10, 2688] with at most 6 significant bits).  The products
// x * A then have the size of the true x * w_hat, so the accumulator overflows
// only if the result itself does; the epilogue multiplies by g * 2^-fold.
__device__ __forceinline__ int bf16_fold(float g) {
    const int eg = (int)((__float_as_uint(g) >> 23) & 0xFF) - 127;
    return max(-123, min(116, eg));
}

// Row m of x -> f16 as x * 2^-sigma_m, sigma_m chosen so that the row's largest
// |x * 2^-sigma_m| lies in [2^14, 2^15); bad[m] = 1 when some nonzero value
// lands below 2^-17 (then it may be inexact in f16) or the row holds Inf / NaN.
// One block per row; every launch rewrites sigma and bad of every row.
__global__ void __launch_bounds__(256) x_to_f16_kernel(const uint16_t *x, uint16_t *xh, int *sigma, int *bad, int K) {
    __shared__ uint32_t red[8];
    const int m = blockIdx.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)m * K);
    uint4 *dst = reinterpret_cast<uint4 *>(xh + (size_t)m * K);
    const int nv = K / 8;
    uint32_t mx = 0;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        const uint4 v = __ldg(src + i);
        mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.w & 0x7FFF7FFFu);
    }
    mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    for (int i = 0; i < 8; i++) mx = max(mx, red[i]);
    const int sg = (mx == 0) ? 0 : max((int)(mx >> 7), 1) - 127 - 14;
    const float tiny = 7.62939453125e-06f;   // 2^-17
    bool b = mx >= 0x7F80u;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
        const uint4 v = __ldg(src + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float x0 = __uint_as_float(w[j] << 16), x1 = __uint_as_float(w[j] & 0xFFFF0000u);
            const float a0 = ldexpf(x0, -sg), a1 = ldexpf(x1, -sg);
            b |= (a0 != 0.0f && fabsf(a0) < tiny) | (a1 != 0.0f && fabsf(a1) < tiny);
            const __half2 hv = __floats2half2_rn(a0, a1);
            o[j] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    const int any = __syncthreads_or(b ? 1 : 0);
    if (threadIdx.x == 0) {
        sigma[m] = sg;
        bad[m] = any;
    }
}

struct Params {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *gscale;
    float *y32;
    __nv_bfloat16 *y16;
    const int *bad;      // [M] rows not exact in f16, or null (every tile BF16)
    const int *sigma;    // [M] power of two of each f16 row
    int M, N, K;
    int tiles_m, tiles_n;
};

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                                                            const __grid_constant__ CUtensorMap xmap16,
                                                            const __grid_constant__ CUtensorMap cmap, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    SharedStorage &sh = *reinterpret_cast<SharedStorage *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = p.K / BK;
    const int ntiles = p.tiles_m * p.tiles_n;
    volatile int *abort = &sh.abort;

    if (threadIdx.x == 0) {
        sh.abort = 0;
        for (int i = 0; i < STAGES; i++) {
            mbar_init(&sh.x_full[i], 1);
            mbar_init(&sh.x_empty[i], 1);
            mbar_init(&sh.a_full[i], kDequantThreads / 32);   // one arrival per dequant warp
            mbar_init(&sh.a_empty[i], 1);
        }
        for (int i = 0; i < WSTAGES; i++) {
            mbar_init(&sh.w_full[i], 1);
            mbar_init(&sh.w_empty[i], kDequantThreads / 32);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&sh.acc_full[i], 1);
            mbar_init(&sh.acc_empty[i], kEpiThreads / 32);
        }
        mbar_init(&sh.mma_done, 1);
        fence_mbar_init();
    }
    const bool use_f16 = p.bad != nullptr && p.tiles_m <= kMaxTilesM;
    for (int i = threadIdx.x; i < kMaxTilesM; i += kThreads) sh.f16_tile[i] = use_f16 ? 1 : 0;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&sh.tmem_base)), "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    if (use_f16) {
        // a token tile runs on f16 operands only if all of its rows converted exactly
        for (int i = threadIdx.x; i < p.M; i += kThreads)
            if (__ldg(p.bad + i)) atomicAnd(&sh.f16_tile[i / BN], 0);
        __syncthreads();
    }

    if (warp == 0) {
        // ---------------------------- x producer (TMA) ----------------------------
        if (lane == 0) {
            int it = 0, wit = 0;
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
                const int m0 = (t % p.tiles_m) * BN;
                const int n0 = (t / p.tiles_m) * BM;
                for (int kt = 0; kt < KT; kt++, it++) {
                    if (kt % (WK / BK) == 0) {   // packed codes of the next 256 k
                        const int ws = wit % WSTAGES;
                        if (wit >= WSTAGES) mbar_wait(&sh.w_empty[ws], ((wit / WSTAGES) - 1) & 1, abort);
                        if (*abort) break;
                        mbar_arrive_expect_tx(&sh.w_full[ws], W_STAGE_BYTES);
                        tma_load_2d(sh.w[ws], &cmap, kt * (BK / 2), n0, &sh.w_full[ws]);
                        wit++;
                    }
                    const int s = it % STAGES;
                    if (it >= STAGES) mbar_wait(&sh.x_empty[s], ((it / STAGES) - 1) & 1, abort);
                    if (*abort) break;
                    mbar_arrive_expect_tx(&sh.x_full[s], X_STAGE_BYTES);
                    tma_load_2d(sh.x[s], sh.f16_tile[t % p.tiles_m] ? &xmap16 : &xmap, kt * BK, m0, &sh.x_full[s]);
                }
                if (*abort) break;
            }
            // every issued copy has landed before the CTA can exit (after an abort
            // the loop above stops early, with copies possibly in flight)
            drain_ring(sh.w_full, WSTAGES, wit);
            drain_ring(sh.x_full, STAGES, it);
        }
        __syncwarp();   // the whole warp reaches the final barrier together (it is .aligned)
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -------------------------------
        // A thread that has MMAs queued stalls on any shared-memory access (an
        // mbarrier wait included) until they drain, which would leave the tensor
        // pipe idle between stages.  So this warp never waits on an mbarrier:
        // warp kWaitWarp waits for each stage (and each accumulator) and then
        // meets it at named barrier 2; lane 0 issues.
        int it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int b = ((t - blockIdx.x) / gridDim.x) & 1;
            const uint32_t dtm = tmem + ACC_COL0 + (uint32_t)(b * BN);
            const uint32_t idesc = sh.f16_tile[t % p.tiles_m] ? IDESC_F16 : IDESC;
            for (int kt = 0; kt < KT; kt++, it++) {
                const int s = it % STAGES;
                named_barrier_sync(2, 64);   // stage s (and, at kt == 0, accumulator b) is ready
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t xb = smem_addr(sh.x[s]);
#pragma unroll
                    for (int j = 0; j < BK / 16; j++)   // A (16 k = 8 columns) from tensor memory
                        mma_ts(dtm, tmem + (uint32_t)(s * (BK / 2) + 8 * j), sw128_desc(xb + 32 * j), idesc,
                               (kt | j) ? 1u : 0u);
                    mma_commit(&sh.x_empty[s]);
                    mma_commit(&sh.a_empty[s]);
                    if (kt == KT - 1) mma_commit(&sh.acc_full[b]);
                }
                __syncwarp();
            }
        }
        // tensor memory is released after the final barrier: every MMA this
        // thread issued must have completed by then (also after an abort)
        if (lane == 0) {
            mma_commit(&sh.mma_done);
            mbar_wait_bounded(&sh.mma_done, 0);
        }
        __syncwarp();
    } else if (warp == kWaitWarp) {
        // ------------------------- waits on behalf of the MMA issuer -------------------------
        int it = 0, lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, lt++) {
            const int b = lt & 1;
            if (lt >= 2) mbar_wait(&sh.acc_empty[b], ((lt >> 1) - 1) & 1, abort);
            for (int kt = 0; kt < KT; kt++, it++) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                // on expiry (abort) the stage is garbage, but both warps still meet every barrier
                mbar_wait(&sh.x_full[s], ph, abort);
                mbar_wait(&sh.a_full[s], ph, abort);
                named_barrier_sync(2, 64);
            }
        }
    } else if (warp < 6) {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const float g = __ldg(p.gscale);
        const int fold = bf16_fold(g);
        int lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, lt++) {
            const int b = lt & 1;
            const int m0 = (t % p.tiles_m) * BN, n0 = (t / p.tiles_m) * BM;
            mbar_wait(&sh.acc_full[b], (lt >> 1) & 1, abort);
            tc_fence_after();
            const int n = n0 + q * 32 + lane;
            const bool f16 = sh.f16_tile[t % p.tiles_m] != 0;
            for (int c = 0; c < BN / 32; c++) {
                uint32_t v[32];
                W4_TMEM_LD32(tmem + ((uint32_t)(q * 32) << 16) + ACC_COL0 + (uint32_t)(b * BN + c * 32), v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                // f16 tiles: token m was scaled by 2^-sigma_m (lane j holds sigma of token c*32+j)
                const int mlane = m0 + c * 32 + lane;
                const int sgl = (f16 && mlane < p.M) ? __ldg(p.sigma + mlane) : 0;
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const int sg = __shfl_sync(0xFFFFFFFFu, sgl, j);   // every lane takes part
                    const int m = m0 + c * 32 + j;
                    if (n < p.N) {
                        if (m < p.M) {
                            const float val = scale_out(__uint_as_float(v[j]), g, f16 ? sg : -fold);
                            if (p.y32) p.y32[(size_t)m * p.N + n] = val;
                            if (p.y16) p.y16[(size_t)m * p.N + n] = __float2bfloat16_rn(val);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[b]);
        }
    } else {
        // ------------------------------- dequantise -------------------------------
        // thread (row r, half h): 32 codes of row r per k-step from the swizzled
        // codes stage (conflict-free: 8 consecutive rows read 8 distinct 16-byte
        // chunks), 2 scales from a register ring filled one codes stage ahead.
        // warp w writes TMEM lanes 32*(w%4) .. +31 (the lanes it may access): row r,
        // k-half h of each 64-k stage
        const int r = 32 * (warp & 3) + lane, h = (warp - 6) >> 2;
        const int fold = bf16_fold(__ldg(p.gscale));
        const uint32_t a_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        constexpr int KQ = WK / BK;             // k-steps per codes stage
        int it = 0, wit = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int n = (t / p.tiles_m) * BM + r;
            const bool valid = n < p.N;
            const bool f16 = sh.f16_tile[t % p.tiles_m] != 0;
            const uint8_t *srow = p.scales + (size_t)(valid ? n : 0) * (p.K / 16);
            uint32_t sc[KQ], sn[KQ];
#pragma unroll
            for (int q = 0; q < KQ; q++) sc[q] = (valid && q < KT) ? __ldg(reinterpret_cast<const uint32_t *>(srow) + q) : 0u;
            for (int kw = 0; kw < KT; kw += KQ, wit++) {
                const int ws = wit % WSTAGES;
#pragma unroll
                for (int q = 0; q < KQ; q++)   // prefetch the next stage's scales
                    sn[q] = (valid && kw + KQ + q < KT) ? __ldg(reinterpret_cast<const uint32_t *>(srow) + kw + KQ + q) : 0u;
                mbar_wait(&sh.w_full[ws], (wit / WSTAGES) & 1, abort);
                const uint8_t *wrow = sh.w[ws] + r * 128;
                // two k-steps per round: one proxy fence and one pair of arrivals per two A
                // stages halves the per-stage synchronisation latency of this chain
#pragma unroll
                for (int q = 0; q < KQ; q += 2) {
                    const int nq = min(2, KT - (kw + q));
                    if (nq <= 0) break;
                    // both A stages free first, then both loads, both decodes and both
                    // stores, so that the two k-steps overlap in this warp
#pragma unroll
                    for (int j = 0; j < 2; j++)
                        if (j < nq && it + j >= STAGES)
                            mbar_wait(&sh.a_empty[(it + j) % STAGES], (((it + j) / STAGES) - 1) & 1, abort);
                    tc_fence_after();
                    uint4 cw[2];
#pragma unroll
                    for (int j = 0; j < 2; j++)
                        cw[j] = ld_shared_v4(smem_addr(wrow + ((((q + j) * 2 + h) ^ (r & 7)) * 16)));
                    uint32_t av[2][16];
#pragma unroll
                    for (int j = 0; j < 2; j++) {
                        const uint32_t sw = sc[q + j] >> (16 * h);
                        const uint32_t cws[4] = {cw[j].x, cw[j].y, cw[j].z, cw[j].w};
                        if (f16) {
                            const uint32_t s01 = e4m3x2_to_f16x2(sw & 0xFFFFu);
                            const uint32_t s0 = __byte_perm(s01, 0, 0x1010), s1 = __byte_perm(s01, 0, 0x3232);
#pragma unroll
                            for (int cc = 0; cc < 4; cc++) {
                                const uint4 o = valid ? dequant8_f16(cws[cc], cc < 2 ? s0 : s1) : make_uint4(0, 0, 0, 0);
                                av[j][4 * cc] = o.x, av[j][4 * cc + 1] = o.y, av[j][4 * cc + 2] = o.z, av[j][4 * cc + 3] = o.w;
                            }
                        } else {
                            const float s0 = mul_pow2(e4m3_to_f32(sw & 0xFFu), fold),
                                        s1 = mul_pow2(e4m3_to_f32((sw >> 8) & 0xFFu), fold);
#pragma unroll
                            for (int cc = 0; cc < 4; cc++) {
                                const uint4 o = valid ? dequant8(cws[cc], cc < 2 ? s0 : s1) : make_uint4(0, 0, 0, 0);
                                av[j][4 * cc] = o.x, av[j][4 * cc + 1] = o.y, av[j][4 * cc + 2] = o.z, av[j][4 * cc + 3] = o.w;
                            }
                        }
                    }
                    // 32 k of row r: columns 16h .. 16h+15 of A stage s
#pragma unroll
                    for (int j = 0; j < 2; j++)
                        if (j < nq) tmem_st16(a_lane + (uint32_t)(((it + j) % STAGES) * (BK / 2) + 16 * h), av[j]);
                    // the stores complete, then one arrival per warp and stage
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        for (int j = 0; j < nq; j++) mbar_arrive(&sh.a_full[(it + j) % STAGES]);
                    it += nq;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.w_empty[ws]);
#pragma unroll
                for (int q = 0; q < KQ; q++) sc[q] = sn[q];
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

}  // namespace gemm

// ---------------------------------------------------------------- host side --

// Workspace of the GEMM: x in f16 [M][K] (16-byte aligned), then sigma [M] and
// bad [M] (int32).  Without it every tile runs on BF16 operands.
inline size_t gemm_workspace_bytes(const w4_weights *w, int M) {
    if (!w || M < 1) return 0;
    return (((size_t)M * w->K * 2 + 15) & ~(size_t)15) + (((size_t)M * 8 + 15) & ~(size_t)15);
}

inline size_t gemm_smem_bytes() { return sizeof(gemm::SharedStorage) + 1024; }

inline w4_status gemm_launch(const w4_weights *w, const void *x, int M, float *y32, void *y16, void *ws,
                             size_t ws_bytes, cudaStream_t st) {
    using namespace gemm;
    if (w->fmt != W4_FMT_NVFP4) return W4_ERR_UNSUPPORTED;
    const int K = w->K, N = w->N;
    if (K % BK) return W4_ERR_UNSUPPORTED;
    PFN_encodeTiled enc = get_encode_tiled();
    if (!enc) return W4_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, BN};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return W4_ERR_CUDA;
    // f16 copy of x in the workspace (when there is room for it)
    const bool f16 = ws && ws_bytes >= gemm_workspace_bytes(w, M);
    uint16_t *xh = reinterpret_cast<uint16_t *>(ws);
    int *sigma = f16 ? reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(ws) +
                                               (((size_t)M * K * 2 + 15) & ~(size_t)15))
                     : nullptr;
    int *bad = f16 ? sigma + M : nullptr;
    CUtensorMap map16 = map;
    if (f16 && enc(&map16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xh, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return W4_ERR_CUDA;
    CUtensorMap cmap;
    const cuuint64_t cdims[2] = {(cuuint64_t)K / 2, (cuuint64_t)N};
    const cuuint64_t cstrides[1] = {(cuuint64_t)K / 2};
    const cuuint32_t cbox[2] = {WK / 2, BM};
    if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w->codes), cdims, cstrides, cbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return W4_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))
        return W4_ERR_CUDA;
    const size_t smem = gemm_smem_bytes();
    if (!set_smem_limit(reinterpret_cast<const void *>(gemm_kernel), smem)) return W4_ERR_CUDA;
    Params p;
    p.codes = w->codes;
    p.scales = w->scales;
    p.gscale = w->global_scale;
    p.y32 = y32;
    p.y16 = reinterpret_cast<__nv_bfloat16 *>(y16);
    p.M = M;
    p.N = N;
    p.K = K;
    p.tiles_m = (M + BN - 1) / BN;
    p.tiles_n = (N + BM - 1) / BM;
    p.bad = bad;
    p.sigma = sigma;
    if (f16) x_to_f16_kernel<<<M, 256, 0, st>>>(reinterpret_cast<const uint16_t *>(x), xh, sigma, bad, K);
    const int ntiles = p.tiles_m * p.tiles_n;
    gemm_kernel<<<std::min(ntiles, sms), kThreads, smem, st>>>(map, map16, cmap, p);
    return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

}  // namespace w4
