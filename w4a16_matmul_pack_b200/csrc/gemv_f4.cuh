// gemv_f4.cuh -- one-token NVFP4 GEMV with the packed E2M1 codes fed to the
// tensor cores as they are stored (tcgen05.mma kind::f8f6f4, sm_100a).
//
// y[n] = g * sum_b s[n][b] * sum_{k in block b} e2m1[n][k] * x[k]
// ("EdgeRock-4B-NVFP4" card, intro: E2M1 values, one E4M3 scale per 16 along K,
// one FP32 global scale; the fused W4A16 decode GEMV of the
// "Nanbeige4.2-3B-NVFP4A16" card, Serving).
//
// A = codes.  The TMA data type 16U4_ALIGN16B unpacks every 8 bytes (16 codes)
// of a row into a 16-byte shared-memory unit (the codes, then 8 bytes of
// padding), the layout in which kind::f8f6f4 reads a 4-bit operand; with the
// 128-byte swizzle a 128-k box of 128 rows is one K-major SW128 tile.  No
// instruction decodes a weight.
//
// B = x.  Block b (16 k) is scaled by 2^-sigma_b (its largest |x'| in
// [2^14, 2^15)) and split into three E5M2 parts, x' = h + m + l with
// h = RN(x'), m = RN(x' - h), l = x' - h - m.  A bf16 value has 8 significant
// bits and E5M2 3, so the split is exact whenever every x' of the block is a
// multiple of 2^-16 (E5M2's smallest subnormal): for every block whose values
// lie within 2^23 of its largest.  The three parts of block b are three
// columns of B that are nonzero only in the k of block b, so each D column of
// the MMA holds the unscaled partial sum of one (block, part); e2m1 x E5M2
// products are exact.  The per-row E4M3 block scale is applied afterwards in
// binary32 by the epilogue: acc += (D_h + D_m + D_l) * s[n][b] * 2^(sigma_b - rho),
// rho = the largest sigma_b of x, y = (g * acc) * 2^rho.  A block that cannot be
// split exactly (values spread over more than 2^23, Inf / NaN, or a factor
// 2^(sigma_b - rho) that would leave binary32's normal range) gets zero parts
// and the epilogue adds its 16 products (exact in binary64) from the codes in
// shared memory and x in global memory.
//
// One MMA step is 128 rows x 32 k (two blocks, N = 16 columns): step j of a
// 256-k stage uses rows 6(j%2) .. 6(j%2)+5 of its B (block 2j: parts at 0..2,
// block 2j+1: parts at 3..5, shifted by 6 for odd j) and writes D columns
// 16(j/2) .. +15 of the stage's 64-column TMEM slot: the even step initialises
// the 16 columns, the odd one accumulates into its own six.  A 128 x 16 x 32
// MMA takes 46 cycles (measured), i.e. about 89 weights per cycle per SM, twice
// what an SM's share of HBM delivers.
//
// Work split: CTA c of a problem owns rows [r0, r1) (multiples of 8, balanced)
// and all of K; it walks 128-row tiles (the last one partial: the box rows past
// r1 belong to the next CTA, which reads them at about the same time, so they
// come from L2; rows past N are zero-filled and not read) in 256-k stages.
//
// Warp roles (11 warps):
//   0      TMA producer: per stage two 128 x 128 code boxes + the 128 x 16 scales.
//   1      TMEM allocation (512 columns) and the MMA issuer (one lane), released
//          per stage by warp 2 through named barrier 2: a thread with MMAs queued
//          stalls on any shared-memory access, so it never waits on an mbarrier.
//   2      waits for the stage's codes and x parts, then releases warp 1.
//   3-6    x builders: x into shared memory and rho, then per stage the 16
//          blocks' parts, factors and fallback mask (thread = one pair of k).
//   7-10   epilogue: warp w reads TMEM lanes 32*(w%4)..+31 = rows of the tile,
//          applies scales and factors, writes y at the end of each tile.
// Every mbarrier wait is bounded (common.cuh: mbar_wait).
#pragma once

#include "gemv_m1.cuh"
#include "gemv_umma.cuh"

namespace w4 {
namespace f4 {

constexpr int kRows = 128;                       // MMA M, rows per tile
constexpr int kStageK = 256;                     // k per stage
constexpr int kSteps = kStageK / 32;             // MMAs per stage
constexpr uint32_t kABytes = kRows * kStageK;    // unpacked codes in shared memory (1 byte per code)
constexpr uint32_t kSBytes = kRows * (kStageK / 16);
constexpr uint32_t kBBytes = kSteps * 512;       // 16 rows x 32 bytes per step
constexpr uint32_t kFBytes = 128;                // 16 factors + the fallback mask
constexpr uint32_t kStageBytes = (kABytes + kSBytes + kBBytes + kFBytes + 1023) & ~1023u;
// bytes the TMA reports per stage: the packed codes (half a byte each) + scales
constexpr uint32_t kTxBytes = kRows * kStageK / 2 + kSBytes;
constexpr int kMaxStages = 8;                    // 64 TMEM columns per stage
constexpr uint32_t kTmemCols = 512;
constexpr int kWarps = 11;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp = 1, kWaitWarp = 2, kBuild0 = 3, kEpi0 = 7;

// kind::f8f6f4: D = F32 (bit 4), A = E2M1 (5, bits 7-9), B = E5M2 (1, bits
// 10-12), both K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (5u << 7) | (1u << 10) | ((uint32_t)(16 >> 3) << 17) |
                            ((uint32_t)(kRows >> 4) << 24);

struct Args {
    const uint16_t *x;   // [K] bf16
    float *y;            // [N]
    const float *gscale;
    int K, N, NS;
};

// Shared memory: NS stages, x (bf16, K), barriers and flags.
__host__ __device__ __forceinline__ size_t x_bytes(int K) { return ((size_t)K * 2 + 127) & ~(size_t)127; }
__host__ __device__ __forceinline__ size_t smem_bytes(int NS, int K) {
    return 1024 + (size_t)NS * kStageBytes + x_bytes(K) + (size_t)(4 * NS + 1) * 8 + 16;
}

// K-major, 128-byte swizzle, 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void mma_f8f6f4(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %4, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(acc), "r"(kIdesc));
}

// f16x2 -> E5M2x2, round to nearest even (low half -> low byte).
__device__ __forceinline__ uint32_t f16x2_to_e5m2x2(uint32_t h) {
    uint16_t r;
    asm("cvt.rn.satfinite.e5m2x2.f16x2 %0, %1;" : "=h"(r) : "r"(h));
    return r;
}
// E5M2x2 -> f16x2: an E5M2 byte is the high byte of the f16 of the same value.
__device__ __forceinline__ uint32_t e5m2x2_to_f16x2(uint32_t e) { return __byte_perm(e, 0, 0x1404); }
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) { um::tmem_ld32(taddr, v); }

// The kernel body for CTA `cta` of `ncta` working on one problem.
__device__ __forceinline__ void body(const CUtensorMap &amap, const CUtensorMap &smap, const Args &a, int cta,
                                     int ncta) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
    const int K = a.K, N = a.N, NS = a.NS;
    uint16_t *xs = reinterpret_cast<uint16_t *>(sm + (size_t)NS * kStageBytes);
    uint64_t *full_w = reinterpret_cast<uint64_t *>(sm + (size_t)NS * kStageBytes + x_bytes(K));
    uint64_t *full_b = full_w + NS;
    uint64_t *done = full_b + NS;
    uint64_t *freeb = done + NS;
    uint64_t *fin = freeb + NS;
    uint32_t *tbase = reinterpret_cast<uint32_t *>(fin + 1);
    int *rho_s = reinterpret_cast<int *>(tbase + 1);
    volatile int *abort = rho_s + 1;
    auto A = [&](int s) { return sm + (size_t)s * kStageBytes; };
    auto S = [&](int s) { return sm + (size_t)s * kStageBytes + kABytes; };
    auto B = [&](int s) { return sm + (size_t)s * kStageBytes + kABytes + kSBytes; };
    auto F = [&](int s) { return reinterpret_cast<float *>(sm + (size_t)s * kStageBytes + kABytes + kSBytes + kBBytes); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = (int)((long long)cta * (N / 8) / ncta) * 8;
    const int r1 = (int)((long long)(cta + 1) * (N / 8) / ncta) * 8;
    const int ntiles = (r1 - r0 + kRows - 1) / kRows;
    const int SK = K / kStageK;
    const int total = ntiles * SK;

    // B rows that no step writes stay zero for the whole kernel
    for (int i = threadIdx.x; i < NS * (int)(kBBytes / 16); i += kThreads) {
        const int s = i / (kBBytes / 16), o = i % (kBBytes / 16);
        *reinterpret_cast<uint4 *>(B(s) + 16 * o) = make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; i++) {
            mbar_init(full_w + i, 1);
            mbar_init(full_b + i, 4);
            mbar_init(done + i, 1);
            mbar_init(freeb + i, 4);
        }
        mbar_init(fin, 1);
        *rho_s = 0;
        *const_cast<int *>(abort) = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tbase)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    um::fence_async_smem();
    um::fence_before();
    __syncthreads();
    um::fence_after();
    const uint32_t tmem = *tbase;
    pdl_allow_dependents();

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int i = 0; i < total; i++) {
                const int s = i % NS;
                if (i >= NS) mbar_wait(freeb + s, ((i / NS) - 1) & 1, abort);
                const int row = r0 + (i / SK) * kRows, k0 = (i % SK) * kStageK;
                mbar_arrive_expect_tx(full_w + s, kTxBytes);
                tma_load_2d(A(s), &amap, k0, row, full_w + s);
                tma_load_2d(A(s) + kABytes / 2, &amap, k0 + 128, row, full_w + s);
                tma_load_2d(S(s), &smap, k0 / 16, row, full_w + s);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------- MMA issuer
        for (int i = 0; i < total; i++) {
            named_barrier_sync(2, 64);
            if (lane == 0) {
                const int s = i % NS;
                um::fence_after();
                const uint32_t a0 = smem_addr(A(s)), b0 = smem_addr(B(s));
                const uint32_t d0 = tmem + 64u * (uint32_t)s;
#pragma unroll
                for (int j = 0; j < kSteps; j++)
                    mma_f8f6f4(d0 + 16u * (uint32_t)(j >> 1),
                               sw128_desc(a0 + (uint32_t)(j >> 2) * (kABytes / 2) + 32u * (uint32_t)(j & 3)),
                               um::b_desc(b0 + 512u * (uint32_t)j), (uint32_t)(j & 1));
                um::mma_commit(done + s);
            }
            __syncwarp();
        }
        if (lane == 0) {   // every MMA has completed before TMEM is freed
            um::mma_commit(fin);
            mbar_wait_bounded(fin, 0);
        }
        __syncwarp();
    } else if (warp == kWaitWarp) {
        // ------------------------------------------- waits for the MMA issuer
        for (int i = 0; i < total; i++) {
            const int s = i % NS;
            const uint32_t ph = (i / NS) & 1;
            mbar_wait(full_w + s, ph, abort);
            mbar_wait(full_b + s, ph, abort);
            named_barrier_sync(2, 64);
        }
    } else if (warp < kEpi0) {
        // ------------------------------------------------------ x builders
        const int bt = threadIdx.x - 32 * kBuild0;   // 0..127
        const uint32_t *x32 = reinterpret_cast<const uint32_t *>(xs);
        pdl_wait_prior_grid();   // x may come from the previous kernel
        // x -> shared memory (all loads in flight at once), and rho = the largest
        // sigma_b of x (sigma of the largest |x|)
        uint32_t mx = 0;
        {
            const uint4 *xg = reinterpret_cast<const uint4 *>(a.x);
            uint4 *xd = reinterpret_cast<uint4 *>(xs);
            for (int i = bt; i < K / 8; i += 128) {
                const uint4 v = __ldg(xg + i);
                xd[i] = v;
                mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                           __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
            }
        }
        mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if (lane == 0 && mx != 0) atomicMax(rho_s, max((int)(mx >> 7), 1) - 127 - 14 + 1000);
        named_barrier_sync(3, 128);
        const int rho = *rho_s == 0 ? 0 : *rho_s - 1000;

        const int blk = bt >> 3, q = bt & 7;       // block of the stage, pair within it
        const int j = blk >> 1, kg = blk & 1, p = j & 1;
        const uint32_t boff = 512u * j + 128u * kg + 2u * q;   // + row (n/8)*256 + (n%8)*16
        for (int i = 0; i < total; i++) {
            const int s = i % NS;
            if (i >= NS) mbar_wait(freeb + s, ((i / NS) - 1) & 1, abort);
            const int k = (i % SK) * kStageK + 16 * blk + 2 * q;
            const uint32_t w = x32[k >> 1];
            uint32_t am = max(w & 0x7FFFu, (w >> 16) & 0x7FFFu);
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 4));
            bool bad = am >= 0x7F80u;   // Inf / NaN in the block
            uint32_t hb = 0, mb = 0, lb = 0;
            float fac = 0.0f;
            if (am != 0 && !bad) {
                const int sg = max((int)(am >> 7), 1) - 127 - 14;   // largest |x'| in [2^14, 2^15)
                const float x0 = mul_pow2(bf16_lo(w), -sg), x1 = mul_pow2(bf16_hi(w), -sg);
                const float tiny = 1.52587890625e-05f;                // 2^-16
                bad |= (x0 != 0.0f && fabsf(x0) < tiny) | (x1 != 0.0f && fabsf(x1) < tiny);
                const __half2 xh2 = __floats2half2_rn(x0, x1);        // exact: 8 bits, in f16 range
                const uint32_t xh = *reinterpret_cast<const uint32_t *>(&xh2);
                hb = f16x2_to_e5m2x2(xh);
                const uint32_t r = hsub2_u32(xh, e5m2x2_to_f16x2(hb));
                mb = f16x2_to_e5m2x2(r);
                const uint32_t t = hsub2_u32(r, e5m2x2_to_f16x2(mb));
                lb = f16x2_to_e5m2x2(t);
                bad |= e5m2x2_to_f16x2(lb) != t;
                const int fe = 120 + sg - rho;   // factor 2^fe, times the scale's 2^-120
                bad |= fe < 3;
                fac = __int_as_float((127 + max(fe, 3)) << 23);
            }
            // a block falls back as a whole
            const uint32_t bm = __ballot_sync(0xFFFFFFFFu, bad);
            const bool bbad = ((bm >> (8 * ((blk & 3)))) & 0xFFu) != 0;
            if (bbad) hb = mb = lb = 0;
            uint8_t *bs = B(s);
            const uint32_t n0 = 6u * p + 3u * kg;
            const uint32_t parts[3] = {hb, mb, lb};
#pragma unroll
            for (int part = 0; part < 3; part++) {
                const uint32_t n = n0 + part;
                *reinterpret_cast<uint16_t *>(bs + boff + (n >> 3) * 256u + (n & 7) * 16u) = (uint16_t)parts[part];
            }
            if (q == 0) F(s)[blk] = fac;
            if (lane == 0) {
                uint32_t mask = 0;
#pragma unroll
                for (int b = 0; b < 4; b++) mask |= (((bm >> (8 * b)) & 0xFFu) != 0 ? 1u : 0u) << b;
                reinterpret_cast<uint8_t *>(F(s) + 16)[warp - kBuild0] = (uint8_t)mask;
            }
            um::fence_async_smem();   // the parts are read by the tensor core (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(full_b + s);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int ew = warp & 3;
        const int rt = 32 * ew + lane;   // row within the tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(32 * ew) << 16);
        const float gs = __ldg(a.gscale);
        pdl_wait_prior_grid();   // y may be read by the previous kernel
        float acc = 0.0f;     // sum of s * partial sums * 2^(sigma_b - rho)
        double accb = 0.0;    // blocks summed directly (binary64: x up to 2^128 times s cannot overflow)
        for (int i = 0; i < total; i++) {
            const int s = i % NS;
            const uint32_t ph = (i / NS) & 1;
            mbar_wait(full_w + s, ph, abort);   // scales (and codes of fallback blocks) visible
            mbar_wait(full_b + s, ph, abort);   // factors and mask visible
            mbar_wait(done + s, ph, abort);
            um::fence_after();
            uint32_t d0[32], d1[32];
            tmem_ld32(lane_base + 64u * (uint32_t)s, d0);
            tmem_ld32(lane_base + 64u * (uint32_t)s + 32u, d1);
            um::tmem_wait_ld();
            const uint4 sc = um::lds128(smem_addr(S(s)) + 16u * (uint32_t)rt);
            const float *f = F(s);
            const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int col = 16 * ((b >> 2) & 1) + 3 * (b & 3);
                const uint32_t *d = (b < 8) ? d0 : d1;
                const float t = __uint_as_float(d[col]) + __uint_as_float(d[col + 1]) + __uint_as_float(d[col + 2]);
                const float ssc = __uint_as_float(((scw[b >> 2] >> (8 * (b & 3))) << 20) & 0x07F00000u);
                acc = __fmaf_rn(t, ssc * f[b], acc);
            }
            const uint32_t mask = *reinterpret_cast<const uint32_t *>(f + 16);
            if (mask != 0) {
                // blocks that could not be split: their 16 products in binary32
                const int k0 = (i % SK) * kStageK;
#pragma unroll 1
                for (int b = 0; b < 16; b++) {
                    if (!((mask >> (8 * (b >> 2) + (b & 3))) & 1u)) continue;
                    const uint8_t *rowp = A(s) + (b >> 3) * (kABytes / 2) + rt * 128;
                    const uint2 c = *reinterpret_cast<const uint2 *>(rowp + (((b & 7) ^ (rt & 7)) << 4));
                    float2 wv[8];
                    decode_nvfp4(c, wv);
                    const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + k0 + 16 * b);
                    const uint4 u0 = __ldg(xg), u1 = __ldg(xg + 1);
                    const uint32_t xw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                    double part = 0.0;   // exact: 16 products of 2 x 8 significant bits
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        part = fma((double)wv[e].x, (double)bf16_lo(xw[e]), part);
                        part = fma((double)wv[e].y, (double)bf16_hi(xw[e]), part);
                    }
                    accb = fma(part, (double)e4m3_to_f32((scw[b >> 2] >> (8 * (b & 3))) & 0xFFu), accb);
                }
            }
            um::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(freeb + s);
            if (i % SK == SK - 1) {
                const int rho = *rho_s == 0 ? 0 : *rho_s - 1000;
                const int n = r0 + (i / SK) * kRows + rt;
                // g before 2^rho: the product stays finite whenever y does
                if (n < r1) a.y[n] = (float)((double)mul_pow2(gs * acc, rho) + (double)gs * accb);
                acc = 0.0f;
                accb = 0.0;
            }
        }
    }

    __syncwarp();
    um::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        um::fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemv_nvfp4_f4_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap smap,
                         const Args a) {
    body(amap, smap, a, blockIdx.x, gridDim.x);
}

constexpr int kMaxGroup = 8;

struct GroupArgs {
    CUtensorMap amap[kMaxGroup];
    CUtensorMap smap[kMaxGroup];
    Args a[kMaxGroup];
    int cta0[kMaxGroup + 1];
    int G;
};

// Several one-token problems in one launch: CTAs [cta0[p], cta0[p+1]) work on
// problem p exactly as the CTAs of a single-problem launch do.
__global__ void __launch_bounds__(kThreads, 1) gemv_nvfp4_f4_grouped_kernel(const __grid_constant__ GroupArgs g) {
    int p = 0;
    while (p + 1 < g.G && (int)blockIdx.x >= g.cta0[p + 1]) p++;
    body(g.amap[p], g.smap[p], g.a[p], (int)blockIdx.x - g.cta0[p], g.cta0[p + 1] - g.cta0[p]);
}

}  // namespace f4
}  // namespace w4
