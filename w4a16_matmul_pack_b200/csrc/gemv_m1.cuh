// gemv_m1.cuh -- NVFP4 decode GEMV for one token (M = 1): the E2M1 x x products
// on the tensor cores, the per-16 E4M3 block scales applied afterwards in
// binary32.
//
// y[n] = g * sum_b s[n][b] * sum_{k in block b} e2m1[n][k] * x[k]
// ("EdgeRock-4B-NVFP4" card, intro: E2M1 values, one E4M3 scale per 16 along K,
// one FP32 global scale; the fused W4A16 decode kernel of the
// "Nanbeige4.2-3B-NVFP4A16" card, Serving).
//
// Why a separate kernel for M = 1.  In the general tensor-core GEMV a lane
// turns two codes into f16 with one cvt and multiplies them by their block
// scale with one HMUL2 before the MMA; with one token only one of the MMA's
// eight B columns carries data, and the conversion pipe (cvt + HMUL2) is what
// limits the kernel.  Here the eight columns are the eight 16-k scale blocks of
// a 128-k super-chunk: B[k][c] = x[k] when k lies in block c, else 0.  The MMA
// then yields, for each of its 16 rows, the eight unscaled block partial sums
// D[row][b]; a lane owns two of them per row (the blocks of its own codes) and
// adds s * D with one FFMA each.  No HMUL2, no scale duplication, and every
// MMA column is used.
//
// x is converted to f16 once per CTA, as x * 2^-sigma with one power of two
// for the whole slice (its largest |x'| in [2^14, 2^15)), exact whenever every
// nonzero |x'| >= 2^-17; all consumer warps convert together and permute each
// 128-k super-chunk to the MMA operand order.  A CTA whose x does not convert
// exactly (range above 2^31, Inf/NaN) computes in binary32 on the CUDA cores
// from the bf16 x in global memory.  The output is acc * g * 2^sigma, formed
// in binary64 (scale_out).
//
// Codes stages (16 rows x KP k) arrive as one 3-D TMA box of 128-byte lines
// with the 128-byte swizzle; each warp quarter reads two rows whose lines differ
// by 4 mod 8 (a fixed remap of MMA rows to physical rows), so the 16-byte code
// loads are free of bank conflicts.  A short tail tile (fewer than 4 rows)
// comes as row copies in the dense layout.  The super-chunks of a stage are
// shared out among the 8 consumer warps with an offset that rotates by tile.
//
// Shared memory: x' [kc + 32] f16, the NS weight stages (1024-byte aligned),
// the per-warp partial sums, mbarriers and flags.
#pragma once

#include "gemv_tc.cuh"

namespace w4 {

// Offsets (bytes) of the M = 1 kernel's shared-memory regions.
struct M1Layout {
    size_t stages, red, bars, total;
};

__host__ __device__ __forceinline__ M1Layout m1_layout(int xstride, int kc, int NS, int tile_bytes, int red_tiles) {
    M1Layout L;
    L.stages = ((size_t)xstride * 2 + 127) & ~(size_t)127;
    L.red = L.stages + 1024 + (size_t)NS * tile_bytes;   // + room to align the stages to 1024 bytes
    L.bars = L.red + (size_t)red_tiles * kTcParts * kTcRows * 4;
    L.total = L.bars + (size_t)(2 * NS + 1) * 8 + 4 * (2 + kTcWarps);   // barriers, flags
    return L;
}

// 16 code bytes of one row (32 k) -> 16 f16x2 (h[i] = elements 2i, 2i+1), exact.
__device__ __forceinline__ void decode_codes32(uint4 c, uint32_t (&h)[16]) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 16; i++) h[i] = e2m1x2_to_f16x2(w[i >> 2] >> (8 * (i & 3)));
}

// E4M3 byte (bits 0..7 of v after the shift) -> its value * 2^-120 as binary32
// bits: exponent and mantissa fields moved into place; an E4M3 subnormal becomes
// a binary32 subnormal of the same scaled value.
__device__ __forceinline__ float e4m3_lo_scaled(uint32_t v) { return __uint_as_float((v << 20) & 0x07F00000u); }
__device__ __forceinline__ float e4m3_hi_scaled(uint32_t v) { return __uint_as_float((v << 12) & 0x07F00000u); }

// The kernel body for one CTA: CTA `cta` of `ncta` working on rows of one
// problem, K-slice `slice` of `nslices` (split-K partials when nslices > 1).
__device__ __forceinline__ void m1_body(const CUtensorMap &cmap, const CUtensorMap &smap, const GemvTcArgs &a,
                                        int cta, int ncta, int slice, int nslices) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int K = a.K, N = a.N, kc = a.kc, KP = a.KP, NS = a.NS;
    const int k0 = slice * kc, kcs = min(kc, K - k0);
    const int npieces = (kcs + KP - 1) / KP;
    const int CS = KP / 2, SS = KP / 16;
    const M1Layout L = m1_layout(a.xstride, kc, NS, a.tile_bytes, a.red_tiles);

    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    // stages on 1024 bytes (the codes box's swizzle atom), whatever the base alignment
    uint8_t *stages = smem + ((smem_addr(smem) + L.stages + 1023) & ~1023u) - smem_addr(smem);
    float *red = reinterpret_cast<float *>(smem + L.red);  // [red_tiles][kTcParts][16]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + NS;
    uint64_t *xfull = empty + NS;
    int *flags = reinterpret_cast<int *>(xfull + 1);
    volatile int *abort = flags;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long r0, r1;
    if (a.rows_mode == 0) {
        r0 = (long long)cta * N / ncta;
        r1 = (long long)(cta + 1) * N / ncta;
    } else {
        r0 = (long long)cta * a.tiles_per_cta * kTcRows;
        r1 = min((long long)N, r0 + (long long)a.tiles_per_cta * kTcRows);
    }
    const int ntiles = (int)((r1 - r0 + kTcRows - 1) / kTcRows);
    const int nstages = ntiles * npieces;

    if (threadIdx.x == 0) {
        flags[0] = 0;   // abort
        flags[1] = 0;   // x not exact in f16
        for (int i = 0; i < NS; i++) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, kTcWarps);
        }
        mbar_init(xfull, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_allow_dependents();

    if (warp == kTcWarps) {
        if (lane == 0)
            tc_produce(cmap, smap, a, 1, xs, stages, full, empty, xfull, abort, r0, r1, k0, kcs, npieces, nstages);
        return;
    }

    // -------------------------------- consumers --------------------------------
    const float gs = __ldg(a.gscale);
    pdl_wait_prior_grid();   // y may be read by the previous kernel
    mbar_wait(xfull, 0, abort);

    // x -> f16 with one power of two for the whole slice, permuted per 128-k
    // super-chunk (convert_x_f16, all consumer warps); a CTA whose x does not
    // convert exactly computes in binary32 on the CUDA cores from the BF16 x in
    // global memory.
    int sigma;
    uint32_t mx;
    convert_x_f16<false>(xs, a.xstride, 1, kcs, warp, lane, flags, sigma, mx);
    named_barrier_sync(1, kTcWarps * 32);
    const bool fast = flags[1] == 0;
    // binary32 path: partial sums in units of x * 2^fold
    const int fold = fast ? 0 : fallback_fold(gs, mx >= ((127u + 100u) << 7));   // largest |x| >= 2^100
    const int sref = fast ? sigma : -fold;
    const float p120 = __int_as_float((127 + 120) << 23);   // e4m3_*_scaled(s) * 2^120 = s

    // MMA operands.  Lane (g, t) holds rows g, g+8 of the codes of k = 32t .. 32t+31
    // (blocks 2t, 2t+1) and B column g.  Column g is block g: it is nonzero only for
    // the k of lanes t = g/2, and only in the MMAs of block g (the first four MMAs
    // for even g, the last four for odd g).  So the 8 lanes with g/2 == t load x,
    // two 16-byte pieces each, and the rest feed zeros.
    const int g = lane >> 2, t4 = lane & 3;
    const bool xact = (g >> 1) == t4;
    const bool odd = (g & 1) != 0;
    // pieces j = 2*odd + {0, 1}; the order (odd lanes j = 3 first) keeps the 8
    // active lanes of each load on distinct banks
    const int xoffA = 32 * (odd ? 3 : 0) + 8 * t4, xoffB = 32 * (odd ? 2 : 1) + 8 * t4;

    const int lines = KP / 256;                    // 128-byte lines per row of a swizzled stage
    const int rdist = swz_row_distance(lines);
    int st_idx = 0;
    for (int tile = 0; tile < ntiles; tile++) {
        float accA = 0.0f, accB = 0.0f;   // rows pr0, pr0+8 (fast) / row lane/2 (binary32)
        // this tile's stages: swizzled box, or (a short tail) row copies in the dense layout
        const int trows = (int)min((long long)kTcRows, r1 - (r0 + (long long)tile * kTcRows));
        const bool dense = !a.swz || trows < a.box_min_rows;
        const int pr0 = dense ? g : swz_phys_row(g, rdist);   // physical row of MMA row g
        for (int piece = 0; piece < npieces; piece++, st_idx++) {
            const int st = st_idx % NS;
            // on expiry the tile is garbage, but the warp still reaches every barrier
            mbar_wait(full + st, (st_idx / NS) & 1, abort);
            const uint8_t *tp = stages + (size_t)st * a.tile_bytes;
            const int kbase = piece * KP;
            const int kps = min(KP, kcs - kbase);
            const int SC = kps / 128;
            // super-chunks [sb, se) of this stage; the shares rotate by tile so that a
            // stage whose count does not divide by 8 does not load one warp alone
            const int wr = (warp + tile) % kTcWarps;
            const int sb = wr * SC / kTcWarps, se = (wr + 1) * SC / kTcWarps;
            if (fast) {
                const uint8_t *c0p = tp + pr0 * CS + 16 * t4;
                const uint8_t *c1p = c0p + 8 * CS;
                const uint8_t *s0p = tp + kTcRows * CS + pr0 * SS + 2 * t4;
                const uint8_t *s1p = s0p + 8 * SS;
                const uint16_t *xp = xs + kbase;
#pragma unroll 2
                for (int s = sb; s < se; s++) {
                    uint4 c0, c1;
                    if (dense) {
                        c0 = *reinterpret_cast<const uint4 *>(c0p + s * 64);
                        c1 = *reinterpret_cast<const uint4 *>(c1p + s * 64);
                    } else {
                        c0 = *reinterpret_cast<const uint4 *>(tp + swz_chunk(pr0, s, t4, lines));
                        c1 = *reinterpret_cast<const uint4 *>(tp + swz_chunk(pr0 + 8, s, t4, lines));
                    }
                    const uint32_t sc0 = *reinterpret_cast<const uint16_t *>(s0p + s * 8);
                    const uint32_t sc1 = *reinterpret_cast<const uint16_t *>(s1p + s * 8);
                    uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
                    if (xact) {
                        xa = *reinterpret_cast<const uint4 *>(xp + s * 128 + xoffA);
                        xb = *reinterpret_cast<const uint4 *>(xp + s * 128 + xoffB);
                    }
                    // B pieces of MMA pairs j = 0..3 (x of k = 32t + 8j .. +7, or zero)
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    const uint4 b0 = odd ? z : xa, b1 = odd ? z : xb, b2 = odd ? xb : z, b3 = odd ? xa : z;
                    uint32_t h0[16], h1[16];
                    decode_codes32(c0, h0);
                    decode_codes32(c1, h1);
                    // four independent chains of two MMAs (the MMA latency, not
                    // its rate, is what a chain of eight would cost)
                    float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    float e0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, e1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    mma_f16_16816(d0, h0[0], h1[0], h0[1], h1[1], b0.x, b0.y);
                    mma_f16_16816(e0, h0[2], h1[2], h0[3], h1[3], b0.z, b0.w);
                    mma_f16_16816(d1, h0[8], h1[8], h0[9], h1[9], b2.x, b2.y);
                    mma_f16_16816(e1, h0[10], h1[10], h0[11], h1[11], b2.z, b2.w);
                    mma_f16_16816(d0, h0[4], h1[4], h0[5], h1[5], b1.x, b1.y);
                    mma_f16_16816(e0, h0[6], h1[6], h0[7], h1[7], b1.z, b1.w);
                    mma_f16_16816(d1, h0[12], h1[12], h0[13], h1[13], b3.x, b3.y);
                    mma_f16_16816(e1, h0[14], h1[14], h0[15], h1[15], b3.z, b3.w);
                    // d0 + e0 holds block 2t in column 2t, d1 + e1 block 2t+1 in column 2t+1
                    accA = __fmaf_rn(e4m3_lo_scaled(sc0) * p120, d0[0] + e0[0], accA);
                    accA = __fmaf_rn(e4m3_hi_scaled(sc0) * p120, d1[1] + e1[1], accA);
                    accB = __fmaf_rn(e4m3_lo_scaled(sc1) * p120, d0[2] + e0[2], accB);
                    accB = __fmaf_rn(e4m3_hi_scaled(sc1) * p120, d1[3] + e1[3], accB);
                }
            } else {
                // binary32 on the CUDA cores: lane l takes row l/2, 64 k of each super-chunk
                const int row = lane >> 1, half = lane & 1;
                for (int s = sb; s < se; s++) {
                    const uint8_t *cp = tp + row * CS + s * 64 + 32 * half;
                    const uint8_t *sp = tp + kTcRows * CS + row * SS + s * 8 + 4 * half;
                    const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + k0 + kbase + s * 128 + 64 * half);
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const uint8_t *cq = dense ? cp + 8 * q
                                                  : tp + swz_chunk(row, s, 2 * half + (q >> 1), lines) + 8 * (q & 1);
                        const uint2 c = *reinterpret_cast<const uint2 *>(cq);
                        float2 w[8], xv[8];
                        decode_nvfp4(c, w);
                        scale_pairs(w, fold);
                        const uint4 u0 = __ldg(xg + 2 * q), u1 = __ldg(xg + 2 * q + 1);
                        const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                        for (int i = 0; i < 8; i++) xv[i] = make_float2(bf16_lo(wv[i]), bf16_hi(wv[i]));
                        accA = dot_group<8>(w, xv, e4m3_to_f32(sp[q]), accA);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + st);
        }

        // ---- this warp's partial sums of the tile -> shared memory ----
        const bool all_at_end = a.red_tiles >= ntiles;
        float *rb = red + (size_t)(all_at_end ? tile : (tile & 1)) * kTcParts * kTcRows;
        if (fast) {
            accA += __shfl_xor_sync(0xFFFFFFFFu, accA, 1);
            accA += __shfl_xor_sync(0xFFFFFFFFu, accA, 2);
            accB += __shfl_xor_sync(0xFFFFFFFFu, accB, 1);
            accB += __shfl_xor_sync(0xFFFFFFFFu, accB, 2);
            if (t4 == 0) {
                rb[warp * kTcRows + pr0] = scale_out(accA, gs, sref);
                rb[warp * kTcRows + pr0 + 8] = scale_out(accB, gs, sref);
            }
        } else {
            accA += __shfl_xor_sync(0xFFFFFFFFu, accA, 1);
            if ((lane & 1) == 0) rb[warp * kTcRows + (lane >> 1)] = scale_out(accA, gs, sref);
        }
        if (!all_at_end) {
            named_barrier_sync(1, kTcWarps * 32);
            const long long rt = r0 + (long long)tile * kTcRows;
            const int rows = (int)min((long long)kTcRows, r1 - rt);
            if (threadIdx.x < rows) {
                float s = 0.0f;
                for (int q = 0; q < kTcParts; q++) s += rb[q * kTcRows + threadIdx.x];
                const long long n = rt + threadIdx.x;
                if (nslices == 1)
                    a.y[n] = s;
                else
                    a.partial[(size_t)slice * N + n] = s;
            }
            // the buffer of tile+2 is written only after every warp passed tile+1's barrier
        }
    }
    if (a.red_tiles >= ntiles) {
        named_barrier_sync(1, kTcWarps * 32);
        for (int i = threadIdx.x; i < ntiles * kTcRows; i += kTcWarps * 32) {
            const long long n = r0 + i;
            if (n >= r1) continue;
            const float *rb = red + (size_t)(i / kTcRows) * kTcParts * kTcRows + (i % kTcRows);
            float s = 0.0f;
            for (int q = 0; q < kTcParts; q++) s += rb[q * kTcRows];
            if (nslices == 1)
                a.y[n] = s;
            else
                a.partial[(size_t)slice * N + n] = s;
        }
    }
}

__global__ void __launch_bounds__(kTcThreads, 1)
    gemv_nvfp4_m1_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap smap,
                         const GemvTcArgs a) {
    m1_body(cmap, smap, a, blockIdx.x, gridDim.x, blockIdx.y, gridDim.y);
}

// Several independent one-token problems in one launch (e.g. the q, k and v
// projections of a layer, or any set of GEMVs that are ready at the same time):
// CTAs [cta0[p], cta0[p+1]) work on problem p, each on its own balanced range
// of rows, exactly as a CTA of the single-problem kernel does.
constexpr int kMaxGroup = 8;

struct GroupArgs {
    CUtensorMap cmap[kMaxGroup];
    CUtensorMap smap[kMaxGroup];
    GemvTcArgs a[kMaxGroup];
    int cta0[kMaxGroup + 1];
    int G;
};

__global__ void __launch_bounds__(kTcThreads, 1) gemv_nvfp4_m1_grouped_kernel(const __grid_constant__ GroupArgs g) {
    int p = 0;
    while (p + 1 < g.G && (int)blockIdx.x >= g.cta0[p + 1]) p++;
    m1_body(g.cmap[p], g.smap[p], g.a[p], (int)blockIdx.x - g.cta0[p], g.cta0[p + 1] - g.cta0[p], 0, 1);
}

}  // namespace w4
