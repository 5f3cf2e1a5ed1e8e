// gemm.cuh -- prefill W4A16 GEMM on the 5th-generation tensor cores (sm_100a).
//
// NVFP4: y[m][n] = g * sum_k x[m][k] * (e2m1[n][k] * scale[n][k/16])
// ("EdgeRock-4B-NVFP4" card, intro).  ROCmFP4 Dual / FAST: y[m][n] = sum_k
// x[m][k] * level[n][k] * dec(u) ("rocmwhy" page, format table and sections
// 01-02; no global scale).  x is BF16.  The decoded weight (e2m1 * scale, at
// most 6 significant bits in [2^-10, 2688]; level * dec(u), at most 7 bits in
// [2^-9, 4480]) is exact in BF16 and in f16, so the dequantised tile is an
// exact operand of tcgen05.mma kind::f16: the dequant warps write it, per 64-k
// stage, into tensor memory (A), B = x is staged by TMA in shared memory, and
// the accumulators are FP32 in tensor memory.  g (NVFP4) is applied in the
// epilogue.
//
// Tile: 128 weight rows (MMA M) x 192 tokens (MMA N) x 64 k per stage.  Tensor
// memory holds four A stages (32 columns each) and two 192-column accumulators
// (512 columns), so the epilogue of a tile overlaps the MMAs of the next.
// Persistent CTAs, one per SM, walk the tiles n-major so that CTAs running
// together share the same packed weight rows in L2.
//
// The dequantisation is what limits a tile of this shape if it runs as one
// chain per stage (decode, store to tensor memory, wait for the store, signal
// the MMA): the chain takes several times the 4 x 96 cycles of MMA per stage.
// So it runs in four groups of four warps, group g owning A stage g (the k-steps
// i = g mod 4): a group decodes its next k-step into registers while the MMAs
// of the previous use of its stage run, and only the store and its signal wait
// for the stage to be free.  Each thread writes one weight row (one TMEM lane)
// of 64 k with one tcgen05.st.
//
// Warp roles (24 warps):
//   warp 0       TMA producer of x: three stages of 128 k, each two 192 x 64
//                BF16 / f16 boxes with the 128-byte swizzle, no multicast.
//   warp 1       allocates / frees the 512 TMEM columns; MMA issuer (one lane):
//                4 x (128x192x16) per stage, commits to the stage barriers and
//                to the accumulator barrier per tile.  It never waits on an
//                mbarrier: a thread with MMAs queued stalls on any shared-memory
//                access until they drain, so warp 22 waits and releases it
//                through named barrier 2 once per stage.
//   warps 2-5    epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//                32*(w%4)..+31), times g (and 2^sigma_m, below), FP32 / BF16
//                stores.
//   warps 6-21   dequantise, four groups of four (warp w owns TMEM lanes
//                32*(w%4)..+31 = weight rows).
//   warp 22      waits on the x / A stage barriers and the accumulator barriers
//                for the MMA issuer.
//   warp 23      TMA producer of the packed weights (NVFP4: codes with the
//                128-byte swizzle plus the E4M3 scales, 256 k per stage; ROCmFP4:
//                the 18- / 17-byte blocks of 128 rows, 256 / 512 k per stage).
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
// BF16 operands (decoded in binary32, times 2^fold for NVFP4, rounded to BF16).
#pragma once

#include "gemv_tc.cuh"

namespace w4 {

namespace gemm {

constexpr int BM = 128;      // weight rows per tile (MMA M)
constexpr int BN = 192;      // tokens per tile (MMA N)
constexpr int BK = 64;       // k per stage (one 128-byte swizzle row of BF16)
constexpr int STAGES = 4;    // A stages in tensor memory (32 columns each), one per dequant group
constexpr int XK = 2;        // k-steps per x stage (one 192 x 64 swizzled box each)
constexpr int XSTAGES = 3;   // x stages in shared memory (48 KB each)
constexpr int kGroups = STAGES;
constexpr int kDqWarp0 = 6;
constexpr int kDqWarps = 4 * kGroups;
constexpr int kWaitWarp = kDqWarp0 + kDqWarps;   // 22
constexpr int kWProdWarp = kWaitWarp + 1;        // 23
constexpr int kWarps = kWProdWarp + 1;           // 24
constexpr int kThreads = kWarps * 32;
constexpr int kEpiThreads = 128;
constexpr uint32_t X_BOX_BYTES = BN * BK * 2;    // 24 KB: one k-step of x
constexpr uint32_t X_STAGE_BYTES = XK * X_BOX_BYTES;
constexpr uint32_t TMEM_COLS = 512;               // 4 A stages (32 columns each) + two 192-column accumulators
constexpr uint32_t ACC_COL0 = STAGES * (BK / 2);  // accumulators after the A stages
constexpr int kMaxTilesM = 256;   // token tiles whose operand mode is kept in shared memory (M <= 49152)

// Packed-weight stages per format: k per stage (WK), bytes per row of a stage,
// block bytes, scale bytes per row, stages in the ring.
//   NVFP4: 256 k = 128 code bytes per row (128-byte swizzle) + 16 scale bytes.
//   ROCmFP4 Dual: 256 k = 8 blocks of 18 bytes = 144 bytes per row; FAST: 512 k =
//          16 blocks of 17 bytes = 272 bytes (a TMA box row must be a multiple of
//          16 bytes).  Scales travel inside the blocks.  No swizzle.
template <int FMT> struct WFormat;
template <> struct WFormat<W4_FMT_NVFP4> {
    static constexpr int WK = 256, ROW_BYTES = 128, BB = 0, SCALE_BYTES = 16, WSTAGES = 4;
};
template <> struct WFormat<W4_FMT_ROCMFP4_DUAL> {
    static constexpr int WK = 256, ROW_BYTES = 144, BB = 18, SCALE_BYTES = 0, WSTAGES = 4;
};
template <> struct WFormat<W4_FMT_ROCMFP4_FAST> {
    static constexpr int WK = 512, ROW_BYTES = 272, BB = 17, SCALE_BYTES = 0, WSTAGES = 2;
};

// Instruction descriptor, kind::f16: D = F32 (bit 4), A = BF16 (bits 7-9),
// B = BF16 (bits 10-12), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
// The same with A = B = F16 (format 0).
constexpr uint32_t IDESC_F16 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

template <int FMT>
struct SharedStorage {
    using F = WFormat<FMT>;
    static constexpr uint32_t W_CODE_BYTES = BM * F::ROW_BYTES;
    static constexpr uint32_t W_STAGE_BYTES = W_CODE_BYTES + BM * F::SCALE_BYTES;
    uint8_t x[XSTAGES][X_STAGE_BYTES];          // 1024-byte aligned (swizzle atoms)
    uint8_t w[F::WSTAGES][W_STAGE_BYTES];       // packed weights of 128 rows (each stage 1024-byte aligned)
    uint64_t w_full[F::WSTAGES], w_empty[F::WSTAGES];
    uint64_t x_full[XSTAGES], x_empty[XSTAGES];
    uint64_t a_full[STAGES], a_empty[STAGES];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t mma_done;                          // the issuer's last commit: every MMA has finished
    uint32_t tmem_base;
    int abort;
    int f16_tile[kMaxTilesM];                   // token tile mt runs with f16 operands (else BF16)
    float fac[BN];                              // epilogue: g * 2^e of each token of the tile (NaN: not exact)
    int fac_exact;                              // every factor of the tile is exact
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

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// D (TMEM) += A (TMEM; K-major: lane = row, 32-bit column = two k) * B (shared memory).
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// 32 consecutive 32-bit columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}

#define W4_TMEM_LD16(taddr, v)                                                                              \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "                                                  \
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"                           \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),       \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),   \
                   "=r"(v[14]), "=r"(v[15])                                                                  \
                 : "r"(taddr))

// 4 code bytes (8 E2M1 values, element 2i in the low nibble of byte i) times a
// scale -> 4 BF16x2 words at o[0..3].  Exact.
__device__ __forceinline__ void dequant8_bf16(uint32_t cw, float s, uint32_t *o) {
    uint32_t hh[4];
    e2m1x8_to_f16x2(cw, hh);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t h = hh[i];
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
        const float2 v = __fmul2_rn(f, make_float2(s, s));
        const __nv_bfloat162 b = __float22bfloat162_rn(v);
        o[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
}

// The same 8 weights as f16x2 words: cvt E2M1 -> f16x2, HMUL2 by the scale
// (s2 = the scale in both halves).  Exact.
__device__ __forceinline__ void dequant8_f16(uint32_t cw, uint32_t s2, uint32_t *o) {
    e2m1x8_to_f16x2(cw, o);
#pragma unroll
    for (int i = 0; i < 4; i++) o[i] = hmul2_u32(o[i], s2);
}

// One ROCmFP4 block (32 weights at shared-memory byte address A: Dual = two
// UE4M3 half scales + 16 code bytes, FAST = one scale + 16 code bytes; code byte
// j holds elements j (low nibble) and j + 16) -> 16 words in k order at o[0..15],
// word c = elements 2c, 2c+1, each level * dec(u) ("rocmwhy" page, format table
// and sections 01-02), as f16x2 (f16) or BF16x2.  Codebook10 level / 2 is the
// E2M1 value of the same nibble with index 7 (6) lowered to 5, so a level is the
// E2M1 conversion clamped to [-5, 5] times 2; level * dec(u) has at most 7
// significant bits and lies in [2^-9, 4480], exact in f16 and in BF16.  The
// block may start on any byte: six aligned words are read and realigned with
// funnel shifts (up to 6 bytes past the block, still inside shared memory).
template <bool DUAL>
__device__ __forceinline__ void dequant_rocm_block(uint32_t A, bool f16, uint32_t *o) {
    const uint32_t base = A & ~3u, sh = (A & 3u) * 8u;
    uint32_t W[6], S[5];
#pragma unroll
    for (int i = 0; i < 6; i++) W[i] = ld_shared_u32(base + 4u * i);
#pragma unroll
    for (int i = 0; i < 5; i++) S[i] = __funnelshift_r(W[i], W[i + 1], sh);   // bytes A + 4i .. + 3
    const uint32_t u0 = S[0] & 0xFFu, u1 = DUAL ? (S[0] >> 8) & 0xFFu : u0;
    uint32_t C[4];
#pragma unroll
    for (int j = 0; j < 4; j++) C[j] = __funnelshift_r(S[j], S[j + 1], DUAL ? 16 : 8);
    const __half2 lim = __floats2half2_rn(5.0f, 5.0f), nlim = __floats2half2_rn(-5.0f, -5.0f);
    const uint32_t sc = e4m3x2_to_f16x2(u0 | (u1 << 8));           // (dec u0, dec u1), exact
    const __half2 sc2 = __hadd2(*reinterpret_cast<const __half2 *>(&sc), *reinterpret_cast<const __half2 *>(&sc));
    const __half2 s0 = __low2half2(sc2), s1 = __high2half2(sc2);    // 2 dec(u): elements 0..15 / 16..31
    const float2 f2 = __half22float2(sc2);
#pragma unroll
    for (int q = 0; q < 4; q++) {
        // low nibbles: elements 4q .. 4q+3; high nibbles: 4q+16 .. 4q+19; pair them as (k, k+1)
        const uint32_t lo = C[q] & 0x0F0F0F0Fu, hi = (C[q] >> 4) & 0x0F0F0F0Fu;
        const uint32_t plo = (lo | (lo >> 4)) & 0x00FF00FFu, phi = (hi | (hi >> 4)) & 0x00FF00FFu;
        const uint32_t pb[4] = {plo, plo >> 16, phi, phi >> 16};
        const int col[4] = {2 * q, 2 * q + 1, 8 + 2 * q, 9 + 2 * q};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const uint32_t h = e2m1x2_to_f16x2(pb[e]);
            const __half2 v = __hmin2(__hmax2(*reinterpret_cast<const __half2 *>(&h), nlim), lim);
            uint32_t w;
            if (f16) {
                const __half2 r = __hmul2(v, e < 2 ? s0 : s1);
                w = *reinterpret_cast<const uint32_t *>(&r);
            } else {
                const float sv = e < 2 ? f2.x : f2.y;
                const float2 fv = __fmul2_rn(__half22float2(v), make_float2(sv, sv));
                const __nv_bfloat162 b = __float22bfloat162_rn(fv);
                w = *reinterpret_cast<const uint32_t *>(&b);
            }
            o[col[e]] = w;
        }
    }
}

// The power of two a BF16-operand NVFP4 tile folds into its weights: the
// exponent of g, clamped so that e2m1 * scale * 2^fold stays an exact BF16 value
// (e2m1 * scale lies in [2^-10, 2688] with at most 6 significant bits).  The
// products x * A then have the size of the true x * w_hat, so the accumulator
// overflows only if the result itself does; the epilogue multiplies by
// g * 2^-fold.
__device__ __forceinline__ int bf16_fold(float g) {
    const int eg = (int)((__float_as_uint(g) >> 23) & 0xFF) - 127;
    return max(-123, min(116, eg));
}

// g * 2^e as binary32 when it is exactly a normal binary32 value or zero, else
// NaN (the caller then forms the product in binary64).
__device__ __forceinline__ float epilogue_factor(float g, int e) {
    const double gd = (double)g * __longlong_as_double((long long)(1023 + e) << 52);
    const double a = fabs(gd);
    return (gd == 0.0 || (a >= 0x1p-126 && a < 0x1p128)) ? (float)gd : __int_as_float(0x7FC00000);
}

// Row m of x -> f16 as x * 2^-sigma_m, sigma_m chosen so that the row's largest
// |x * 2^-sigma_m| lies in [2^14, 2^15); bad[m] = 1 when some nonzero value
// lies below 2^(sigma_m - 17) (then x * 2^-sigma_m may be inexact in f16) or
// the row holds Inf / NaN.  One CTA of four warps per row, so that enough rows
// are in flight to hide the load latency; every launch rewrites sigma and bad
// of every row.  Rows of up to kXcVec * kXcThreads * 8 values are read once
// (kept in registers); longer rows are read twice.
constexpr int kXcThreads = 128;
constexpr int kXcWarps = kXcThreads / 32;
constexpr int kXcVec = 8;

// Per 16-bit lane: the largest magnitude, and the smallest of (|x| - 1) over
// |x| != 0 (0 -> 0xFFFF), of eight BF16 values.
__device__ __forceinline__ void x_stats8(uint4 v, uint32_t &mx2, uint32_t &mn2) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint32_t mag = w[j] & 0x7FFF7FFFu;
        mx2 = __vmaxu2(mx2, mag);
        mn2 = __vminu2(mn2, (mag + 0x7FFF7FFFu) ^ 0x80008000u);
    }
}

__device__ __forceinline__ uint4 x_row_to_f16(uint4 v, const XScale &xs) {
    if (xs.one)
        return make_uint4(x_pair_f16_scaled(v.x, xs.p), x_pair_f16_scaled(v.y, xs.p), x_pair_f16_scaled(v.z, xs.p),
                          x_pair_f16_scaled(v.w, xs.p));
    bool unused = false;
    return make_uint4(x_pair_f16(v.x, xs, unused), x_pair_f16(v.y, xs, unused), x_pair_f16(v.z, xs, unused),
                      x_pair_f16(v.w, xs, unused));
}

__global__ void __launch_bounds__(kXcThreads) x_to_f16_kernel(const uint16_t *x, uint16_t *xh, int *sigma, int *bad,
                                                              int M, int K) {
    __shared__ uint32_t red[2][kXcWarps];
    pdl_allow_dependents();   // the GEMM may start its prologue; it waits for this grid before reading x
    const int m = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)m * K);
    uint4 *dst = reinterpret_cast<uint4 *>(xh + (size_t)m * K);
    const int nv = K / 8;
    const bool in_regs = nv <= kXcVec * kXcThreads;
    uint4 keep[kXcVec];
    uint32_t mx2 = 0u, mn2 = 0xFFFFFFFFu;
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kXcVec; r++) {
            const int i = threadIdx.x + r * kXcThreads;
            if (i < nv) keep[r] = __ldg(src + i);
        }
#pragma unroll
        for (int r = 0; r < kXcVec; r++)
            if (threadIdx.x + r * kXcThreads < nv) x_stats8(keep[r], mx2, mn2);
    } else {
        for (int i = threadIdx.x; i < nv; i += kXcThreads) x_stats8(__ldg(src + i), mx2, mn2);
    }
    uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, max(mx2 & 0xFFFFu, mx2 >> 16));
    uint32_t mn = __reduce_min_sync(0xFFFFFFFFu, min(mn2 & 0xFFFFu, mn2 >> 16));
    if (lane == 0) red[0][warp] = mx, red[1][warp] = mn;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kXcWarps; w++) mx = max(mx, red[0][w]), mn = min(mn, red[1][w]);
    const int sg = (mx == 0) ? 0 : max((int)(mx >> 7), 1) - 127 - 14;
    const XScale xs = make_xscale(sg);
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kXcVec; r++) {
            const int i = threadIdx.x + r * kXcThreads;
            if (i < nv) dst[i] = x_row_to_f16(keep[r], xs);
        }
    } else {
        for (int i = threadIdx.x; i < nv; i += kXcThreads) dst[i] = x_row_to_f16(__ldg(src + i), xs);
    }
    if (threadIdx.x == 0) {
        sigma[m] = sg;
        // Inf / NaN, or a nonzero |x| below 2^(sigma - 17) (mn + 1: the smallest nonzero magnitude)
        bad[m] = (mx >= 0x7F80u || mn + 1u < xs.thr) ? 1 : 0;
    }
}

struct Params {
    const uint8_t *scales;   // NVFP4 scales [N][K/16], read directly when scales_tma == 0
    const float *gscale;
    float *y32;
    __nv_bfloat16 *y16;
    const int *bad;      // [M] rows not exact in f16, or null (every tile BF16)
    const int *sigma;    // [M] power of two of each f16 row
    int M, N, K;
    int tiles_m, tiles_n;
    int scales_tma;      // NVFP4 scales staged by TMA with the codes (K % 256 == 0: 16-byte rows)
};

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                                                            const __grid_constant__ CUtensorMap xmap16,
                                                            const __grid_constant__ CUtensorMap cmap,
                                                            const __grid_constant__ CUtensorMap smap, const Params p) {
    using SS = SharedStorage<FMT>;
    using F = WFormat<FMT>;
    constexpr int WK = F::WK, ROW_BYTES = F::ROW_BYTES, BB = F::BB, WSTAGES = F::WSTAGES;
    constexpr int KQ = WK / BK;             // k-steps per packed-weight stage
    constexpr bool NV = FMT == W4_FMT_NVFP4;
    extern __shared__ uint8_t smem_raw[];
    SS &sh = *reinterpret_cast<SS *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = p.K / BK;
    const int ntiles = p.tiles_m * p.tiles_n;
    volatile int *abort = &sh.abort;

    if (threadIdx.x == 0) {
        sh.abort = 0;
        for (int i = 0; i < XSTAGES; i++) {
            mbar_init(&sh.x_full[i], 1);
            mbar_init(&sh.x_empty[i], 1);
        }
        for (int i = 0; i < STAGES; i++) {
            mbar_init(&sh.a_full[i], 4);   // the four warps of group i
            mbar_init(&sh.a_empty[i], 1);
        }
        for (int i = 0; i < WSTAGES; i++) {
            mbar_init(&sh.w_full[i], 1);
            mbar_init(&sh.w_empty[i], kDqWarps);
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
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&sh.tmem_base)), "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    // with the f16 pass launched just before (programmatic dependent launch),
    // everything above overlapped its tail; x, sigma and bad are its output
    pdl_wait_prior_grid();
    if (use_f16) {
        // a token tile runs on f16 operands only if all of its rows converted exactly
        for (int i = threadIdx.x; i < p.M; i += kThreads)
            if (__ldg(p.bad + i)) atomicAnd(&sh.f16_tile[i / BN], 0);
        __syncthreads();
    }

    if (warp == 0) {
        // ---------------------------- x producer (TMA) ----------------------------
        if (lane == 0) {
            // x stages of XK k-steps: fewer, larger copies stream faster than
            // one stage per k-step
            int it = 0;   // x stages issued
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
                const int m0 = (t % p.tiles_m) * BN;
                const CUtensorMap *xm = sh.f16_tile[t % p.tiles_m] ? &xmap16 : &xmap;
                for (int kt = 0; kt < KT; kt += XK, it++) {
                    const int s = it % XSTAGES, nk = min(XK, KT - kt);
                    if (it >= XSTAGES) mbar_wait(&sh.x_empty[s], ((it / XSTAGES) - 1) & 1, abort);
                    if (*abort) break;
                    mbar_arrive_expect_tx(&sh.x_full[s], (uint32_t)nk * X_BOX_BYTES);
                    for (int j = 0; j < nk; j++)
                        tma_load_2d(sh.x[s] + j * X_BOX_BYTES, xm, (kt + j) * BK, m0, &sh.x_full[s]);
                }
            }
            // every issued copy has landed before the CTA can exit (after an abort
            // the loop above stops early, with copies possibly in flight)
            drain_ring(sh.x_full, XSTAGES, it);
        }
        __syncwarp();   // the whole warp reaches the final barrier together (it is .aligned)
    } else if (warp == kWProdWarp) {
        // ------------------------ packed-weight producer (TMA) ------------------------
        if (lane == 0) {
            int wit = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
                const int n0 = (t / p.tiles_m) * BM;
                for (int kw = 0; kw < KT; kw += KQ, wit++) {
                    const int ws = wit % WSTAGES;
                    if (wit >= WSTAGES) mbar_wait(&sh.w_empty[ws], ((wit / WSTAGES) - 1) & 1, abort);
                    if (*abort) break;
                    if constexpr (NV) {
                        mbar_arrive_expect_tx(&sh.w_full[ws], p.scales_tma ? SS::W_STAGE_BYTES : SS::W_CODE_BYTES);
                        tma_load_2d(sh.w[ws], &cmap, (kw / KQ) * ROW_BYTES, n0, &sh.w_full[ws]);
                        if (p.scales_tma)
                            tma_load_2d(sh.w[ws] + SS::W_CODE_BYTES, &smap, (kw / KQ) * F::SCALE_BYTES, n0,
                                        &sh.w_full[ws]);
                    } else {
                        mbar_arrive_expect_tx(&sh.w_full[ws], SS::W_STAGE_BYTES);
                        // 2-byte elements: a FAST row of 272 bytes is one 136-element box row
                        tma_load_2d(sh.w[ws], &cmap, (kw / KQ) * (ROW_BYTES / 2), n0, &sh.w_full[ws]);
                    }
                }
            }
            drain_ring(sh.w_full, WSTAGES, wit);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -------------------------------
        // A thread that has MMAs queued stalls on any shared-memory access (an
        // mbarrier wait included) until they drain, which would leave the tensor
        // pipe idle between stages.  So this warp never waits on an mbarrier:
        // warp kWaitWarp waits for each stage (and each accumulator) and then
        // meets it at named barrier 2; lane 0 issues.
        int it = 0, xi = 0;   // k-steps, x stages
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int b = ((t - blockIdx.x) / gridDim.x) & 1;
            const uint32_t dtm = tmem + ACC_COL0 + (uint32_t)(b * BN);
            const uint32_t idesc = sh.f16_tile[t % p.tiles_m] ? IDESC_F16 : IDESC;
            for (int kt = 0; kt < KT; kt++, it++) {
                const int s = it % STAGES, xs = xi % XSTAGES, sub = kt % XK;
                named_barrier_sync(2, 64);   // k-step it (and, at kt == 0, accumulator b) is ready
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t xb = smem_addr(sh.x[xs]) + (uint32_t)(sub * X_BOX_BYTES);
#pragma unroll
                    for (int j = 0; j < BK / 16; j++)   // A (16 k = 8 columns) from tensor memory
                        mma_ts(dtm, tmem + (uint32_t)(s * (BK / 2) + 8 * j), sw128_desc(xb + 32 * j), idesc,
                               (kt | j) ? 1u : 0u);
                    mma_commit(&sh.a_empty[s]);
                    if (sub == XK - 1 || kt == KT - 1) mma_commit(&sh.x_empty[xs]);
                    if (kt == KT - 1) mma_commit(&sh.acc_full[b]);
                }
                __syncwarp();
                if (sub == XK - 1 || kt == KT - 1) xi++;
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
        int it = 0, lt = 0, xi = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, lt++) {
            const int b = lt & 1;
            if (lt >= 2) mbar_wait(&sh.acc_empty[b], ((lt >> 1) - 1) & 1, abort);
            for (int kt = 0; kt < KT; kt++, it++) {
                // on expiry (abort) the stage is garbage, but both warps still meet every barrier
                if (kt % XK == 0) mbar_wait(&sh.x_full[xi % XSTAGES], (xi / XSTAGES) & 1, abort);
                mbar_wait(&sh.a_full[it % STAGES], (it / STAGES) & 1, abort);
                named_barrier_sync(2, 64);
                if (kt % XK == XK - 1 || kt == KT - 1) xi++;
            }
        }
    } else if (warp < kDqWarp0) {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const float g = NV ? __ldg(p.gscale) : 1.0f;   // ROCmFP4: no global scale
        const int fold = NV ? bf16_fold(g) : 0;
        int lt = 0;
        const int et = threadIdx.x - 2 * 32;   // 0..127 over the four epilogue warps
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, lt++) {
            const int b = lt & 1;
            const int m0 = (t % p.tiles_m) * BN, n0 = (t / p.tiles_m) * BM;
            const bool f16 = sh.f16_tile[t % p.tiles_m] != 0;
            // the tile's per-token factors g * 2^e (f16 tiles: token m was scaled by
            // 2^-sigma_m), exact in binary32 when a normal number or zero: then acc *
            // factor rounded once is the binary64 product of scale_out rounded once,
            // bit for bit; otherwise NaN, and that token goes through scale_out
            named_barrier_sync(3, kEpiThreads);   // the previous tile's factors are no longer read
            if (et == 0) sh.fac_exact = 1;
            named_barrier_sync(3, kEpiThreads);
            for (int i = et; i < BN; i += kEpiThreads) {
                const int m = m0 + i;
                const int e = f16 ? (m < p.M ? __ldg(p.sigma + m) : 0) : -fold;
                const float f = epilogue_factor(g, e);
                sh.fac[i] = f;
                if (isnan(f)) sh.fac_exact = 0;
            }
            named_barrier_sync(3, kEpiThreads);
            const bool exact = sh.fac_exact != 0;
            mbar_wait(&sh.acc_full[b], (lt >> 1) & 1, abort);
            tc_fence_after();
            const int n = n0 + q * 32 + lane;
            const bool nok = n < p.N;
            for (int c = 0; c < BN / 16; c++) {
                uint32_t v[16];
                W4_TMEM_LD16(tmem + ((uint32_t)(q * 32) << 16) + ACC_COL0 + (uint32_t)(b * BN + c * 16), v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                const int mc = m0 + c * 16;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const int m = mc + j;
                    if (!nok || m >= p.M) continue;
                    const float acc = __uint_as_float(v[j]);
                    const float gj = sh.fac[c * 16 + j];   // the same address in every lane
                    float val;
                    if (exact) {
                        val = acc * gj;
                    } else {
                        const int e = f16 ? __ldg(p.sigma + m) : -fold;
                        val = isnan(gj) ? scale_out(acc, g, e) : acc * gj;
                    }
                    if (p.y32) p.y32[(size_t)m * p.N + n] = val;
                    if (p.y16) p.y16[(size_t)m * p.N + n] = __float2bfloat16_rn(val);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[b]);
        }
    } else {
        // ------------------------------- dequantise -------------------------------
        // group gi = (warp - 6) / 4 takes the k-steps i == gi (mod 4) into A stage gi;
        // thread = weight row r (TMEM lane r) and all 64 k of the k-step.  Rows past
        // N arrive as zero bytes (TMA fill), which decode to zero weights.
        const int gi = (warp - kDqWarp0) >> 2;
        const int r = 32 * (warp & 3) + lane;
        const int fold = NV ? bf16_fold(__ldg(p.gscale)) : 0;
        const uint32_t a_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(gi * (BK / 2));
        int it = 0, wit = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, it += KT) {
            const bool f16 = sh.f16_tile[t % p.tiles_m] != 0;
            const int n = (t / p.tiles_m) * BM + r;
            const uint32_t *srow =
                NV ? reinterpret_cast<const uint32_t *>(p.scales) + (size_t)(n < p.N ? n : 0) * (p.K / 64) : nullptr;
            for (int kw = 0; kw < KT; kw += KQ, wit++) {
                const int ws = wit % WSTAGES;
                // every dequant warp takes every packed stage (and arrives on its
                // empty barrier), whether or not one of its k-steps lies in it
                mbar_wait(&sh.w_full[ws], (wit / WSTAGES) & 1, abort);
                const uint32_t wst = smem_addr(sh.w[ws]);
                const uint32_t wrow = wst + (uint32_t)(r * ROW_BYTES);
#pragma unroll 1
                for (int q = (gi - (it + kw)) & 3; q < KQ && kw + q < KT; q += 4) {
                    const int i = it + kw + q;   // this group's k-step: i % 4 == gi
                    uint32_t av[32];
                    if constexpr (NV) {
                        // 64 k of row r: chunks 2q, 2q+1 of the swizzled 128-byte row;
                        // 4 block scales at byte 4q of the row's 16 scale bytes (or the
                        // row's scale word kw + q in global memory)
                        const uint4 c0 = ld_shared_v4(wrow + (uint32_t)(((2 * q) ^ (r & 7)) * 16));
                        const uint4 c1 = ld_shared_v4(wrow + (uint32_t)(((2 * q + 1) ^ (r & 7)) * 16));
                        const uint32_t sw =
                            p.scales_tma ? ld_shared_u32(wst + SS::W_CODE_BYTES + (uint32_t)(r * F::SCALE_BYTES + 4 * q))
                                         : (n < p.N ? __ldg(srow + kw + q) : 0u);
                        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                        if (f16) {
                            const uint32_t s01 = e4m3x2_to_f16x2(sw & 0xFFFFu), s23 = e4m3x2_to_f16x2(sw >> 16);
                            const uint32_t sd[4] = {__byte_perm(s01, 0, 0x1010), __byte_perm(s01, 0, 0x3232),
                                                    __byte_perm(s23, 0, 0x1010), __byte_perm(s23, 0, 0x3232)};
#pragma unroll
                            for (int c = 0; c < 8; c++) dequant8_f16(cw[c], sd[c >> 1], av + 4 * c);
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; c++)
                                dequant8_bf16(cw[c], mul_pow2(e4m3_to_f32((sw >> (8 * (c >> 1))) & 0xFFu), fold),
                                              av + 4 * c);
                        }
                    } else {
                        // blocks 2q, 2q+1 of row r
                        dequant_rocm_block<FMT == W4_FMT_ROCMFP4_DUAL>(wrow + (uint32_t)(2 * q * BB), f16, av);
                        dequant_rocm_block<FMT == W4_FMT_ROCMFP4_DUAL>(wrow + (uint32_t)((2 * q + 1) * BB), f16,
                                                                        av + 16);
                    }
                    // the stage is free once the MMAs of its previous use have completed
                    if (i >= STAGES) mbar_wait(&sh.a_empty[gi], ((i / STAGES) - 1) & 1, abort);
                    tc_fence_after();
                    tmem_st32(a_addr, av);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.a_full[gi]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.w_empty[ws]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
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

template <int FMT>
inline size_t gemm_smem_bytes() { return sizeof(gemm::SharedStorage<FMT>) + 1024; }

template <int FMT>
inline w4_status gemm_launch_fmt(const w4_weights *w, const void *x, int M, float *y32, void *y16, void *ws,
                                 size_t ws_bytes, cudaStream_t st) {
    using namespace gemm;
    using F = WFormat<FMT>;
    static_assert(sizeof(SharedStorage<FMT>) + 1024 <= 227 * 1024, "shared memory of the GEMM");
    static_assert(SharedStorage<FMT>::W_STAGE_BYTES % 1024 == 0 && (XSTAGES * X_STAGE_BYTES) % 1024 == 0,
                  "stages on 1024-byte boundaries");
    const int K = w->K, N = w->N;
    // NVFP4: 64-k steps (a last partial packed stage reads zeros past K);
    // ROCmFP4: whole packed stages, whose row pieces are 16-byte multiples
    if (K % (FMT == W4_FMT_NVFP4 ? BK : F::WK)) return W4_ERR_UNSUPPORTED;
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
    // packed weights: NVFP4 codes [N][K/2] bytes with the 128-byte swizzle and
    // scales [N][K/16] bytes; ROCmFP4 blocks [N][K/32 * 18|17] bytes as 2-byte
    // elements (the FAST box row of 272 bytes exceeds 256 one-byte elements)
    CUtensorMap cmap, smap;
    // the scales map needs 16-byte rows (K % 256 == 0); otherwise the dequant
    // warps read the scale words directly
    const bool scales_tma = FMT == W4_FMT_NVFP4 && K % 256 == 0;
    if (FMT == W4_FMT_NVFP4) {
        const cuuint64_t cdims[2] = {(cuuint64_t)K / 2, (cuuint64_t)N};
        const cuuint64_t cstr[1] = {(cuuint64_t)K / 2};
        const cuuint32_t cbox[2] = {(cuuint32_t)F::ROW_BYTES, BM};
        const cuuint64_t sdims[2] = {(cuuint64_t)K / 16, (cuuint64_t)N};
        const cuuint64_t sstr[1] = {(cuuint64_t)K / 16};
        const cuuint32_t sbox[2] = {(cuuint32_t)F::SCALE_BYTES, BM};
        if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w->codes), cdims, cstr, cbox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            (scales_tma &&
             enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w->scales), sdims, sstr, sbox, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS))
            return W4_ERR_CUDA;
        if (!scales_tma) smap = cmap;   // not read
    } else {
        const cuuint64_t row_bytes = (cuuint64_t)(K / F::WK) * F::ROW_BYTES;
        const cuuint64_t cdims[2] = {row_bytes / 2, (cuuint64_t)N};
        const cuuint64_t cstr[1] = {row_bytes};
        const cuuint32_t cbox[2] = {(cuuint32_t)F::ROW_BYTES / 2, BM};
        if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint8_t *>(w->codes), cdims, cstr, cbox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
        smap = cmap;   // not read
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))
        return W4_ERR_CUDA;
    const size_t smem = gemm_smem_bytes<FMT>();
    if (!set_smem_limit(reinterpret_cast<const void *>(gemm_kernel<FMT>), smem)) return W4_ERR_CUDA;
    Params p;
    p.scales = w->scales;
    p.scales_tma = scales_tma ? 1 : 0;
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
    if (f16)
        x_to_f16_kernel<<<M, kXcThreads, 0, st>>>(reinterpret_cast<const uint16_t *>(x), xh, sigma, bad, M, K);
    const int ntiles = p.tiles_m * p.tiles_n;
    const int grid = std::max(1, std::min(ntiles, sms));   // persistent, one CTA per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = f16 ? 1 : 0;   // overlap the prologue with the f16 pass just launched
    if (cudaLaunchKernelEx(&cfg, gemm_kernel<FMT>, map, map16, cmap, smap, p) != cudaSuccess) return W4_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

inline w4_status gemm_launch(const w4_weights *w, const void *x, int M, float *y32, void *y16, void *ws,
                             size_t ws_bytes, cudaStream_t st) {
    switch (w->fmt) {
    case W4_FMT_NVFP4: return gemm_launch_fmt<W4_FMT_NVFP4>(w, x, M, y32, y16, ws, ws_bytes, st);
    case W4_FMT_ROCMFP4_DUAL: return gemm_launch_fmt<W4_FMT_ROCMFP4_DUAL>(w, x, M, y32, y16, ws, ws_bytes, st);
    case W4_FMT_ROCMFP4_FAST: return gemm_launch_fmt<W4_FMT_ROCMFP4_FAST>(w, x, M, y32, y16, ws, ws_bytes, st);
    }
    return W4_ERR_UNSUPPORTED;
}

}  // namespace w4
