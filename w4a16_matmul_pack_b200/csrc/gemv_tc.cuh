// gemv_tc.cuh -- NVFP4 decode GEMV (M = 1..16) with the products on the tensor
// cores (sm_100a, mma.sync.m16n8k16, f16 inputs, binary32 accumulation).
//
// y[m][n] = g * sum_k x[m][k] * e2m1[n][k] * scale[n][k/16]   ("EdgeRock-4B-NVFP4"
// card, intro; the fused W4A16 decode kernel of the "Nanbeige4.2-3B-NVFP4A16"
// card, Serving).  The kernel is bound by HBM: every packed byte is read once.
//
// Decode on the CUDA cores would cost ~6 lane instructions per weight, above the
// ~4 the SMs can issue per weight at 75% of HBM bandwidth.  Here a lane decodes
// two E2M1 codes with one cvt (E2M1 -> f16x2, exact) and applies the block scale
// with one HMUL2 (e2m1 * E4M3 has at most 6 significant bits and lies in
// [2^-10, 2688]: exact in f16); the MMA does the multiply-add.  x is converted
// once per CTA to f16 as x * 2^-sigma (sigma from the largest |x|), exact when
// every x fits f16's range; a CTA that finds an x it cannot convert exactly runs
// a binary32 CUDA-core loop on the same staged tiles instead.
//
// Data movement: bulk copies only reach full HBM bandwidth when each copy is
// large (>= 16 KB; small copies are limited by a per-copy cost), so a stage is
// one 2-D TMA box of codes (16 rows x KP/2 bytes, the codes viewed as 8-byte
// elements) and one box of scales (16 rows x KP/16 bytes), in an NS-deep
// mbarrier ring filled by one producer thread.  Rows are contiguous in shared
// memory.
//
// MMA operand mapping.  In an m16n8k16 a lane (g = lane/4, t = lane%4) holds A
// rows g and g+8 at two k-pairs and B column g at the same k-pairs.  Any
// permutation of k applied to both operands leaves the product unchanged, so
// within a 128-k super-chunk lane t owns k = 32t..32t+31: one 16-byte load per
// row gives the codes of 8 MMAs (two scale groups: 2t and 2t+1), and x is
// stored permuted (the 8 x of MMAs 2j, 2j+1 of lane t at offset 32j + 8t) so
// that the B loads of the four lanes of a row are one contiguous 64-byte run.
// Consumer warp w takes a contiguous 1/8 of each stage's super-chunks; the MMA
// accumulators persist over the k-pieces of a row tile and the 8 warps' partial
// sums are added in a fixed order at its end.
#pragma once

#include "gemv.cuh"

namespace w4 {

struct GemvTcArgs {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *gscale;
    const uint16_t *x;   // [M][K] bf16
    float *y;            // [M][N]
    float *partial;      // [S][M][N] when gridDim.y > 1
    int K, N;
    int kc;              // slice length (split-K over blockIdx.y)
    int KP;              // k per stage (multiple of 256, <= 4096)
    int NS;              // stages
    int xstride;         // halves per x row in shared memory (kc + 32)
    int tile_bytes;      // bytes of one stage: 16 * (KP/2 + KP/16), rounded up
    int rows_mode;       // 0: balanced rows per CTA; 1: whole 16-row tiles per CTA
    int tiles_per_cta;   // rows_mode 1
    int box_min_rows;    // a partial tile with at least this many rows uses the TMA box
    int red_tiles;       // tiles whose partial sums fit the reduction buffer at once (>= ntiles:
                         // one barrier per CTA; else 2 and a barrier per tile)
    int pdl;             // launched with programmatic dependent launch: prefetch weights before x
    int fmt;             // w4_format
    int bb;              // ROCmFP4 block bytes (18 Dual, 17 FAST)
};

// Bytes of one row of a stage of KP k: NVFP4 codes (scales follow all 16 rows'
// codes), or ROCmFP4 blocks.
__host__ __device__ __forceinline__ int stage_row_bytes(int fmt, int bb, int kp) {
    return fmt == W4_FMT_NVFP4 ? kp / 2 : (kp / 32) * bb;
}

// v * 2^e for |e| <= 252 as two exact multiplies (each factor a normal power of two).
__device__ __forceinline__ float mul_pow2(float v, int e) {
    const int h = e / 2, h2 = e - h;
    return (v * __int_as_float((127 + h) << 23)) * __int_as_float((127 + h2) << 23);
}

// v * g * 2^e rounded once to binary32.  The kernels accumulate in units of
// x * 2^-e (x rescaled into f16's range) with the weights' global scale g left
// out; the output is the product of all three.  In binary64 the product v * g of
// two binary32 values is exact and 2^e (|e| <= 400 here) is in range, so no
// intermediate overflows or underflows: the result is finite whenever the true
// product is below binary32's largest value.
__device__ __forceinline__ float scale_out(float v, float g, int e) {
    const double p2 = __longlong_as_double((long long)(1023 + e) << 52);
    return (float)((double)v * (double)g * p2);
}

// g * 2^e in binary64 (exact for |e| <= 400).  (double)v times it, rounded once
// (scale_by), is the exact v * g * 2^e rounded once: scale_out bit for bit, with
// the factor computed once per CTA.
__device__ __forceinline__ double out_factor(float g, int e) {
    return (double)g * __longlong_as_double((long long)(1023 + e) << 52);
}
__device__ __forceinline__ float scale_by(float v, double f) { return (float)((double)v * f); }

// Power of two folded into the decoded weights of the binary32 fallback paths:
// the exponent of g, clamped to [-100, 0], when x reaches 2^100 (else 0).  Sums
// of x * e2m1 * 2^fold (and their products with the block scale) then stay near
// the size of the true x * w_hat, so a finite result cannot overflow inside the
// accumulator.
__device__ __forceinline__ int fallback_fold(float g, bool x_huge) {
    if (!x_huge) return 0;
    const int eg = (int)((__float_as_uint(g) >> 23) & 0xFF) - 127;
    return max(-100, min(0, eg));
}

// w[p] *= 2^e (exact for the E2M1 values of a fallback block, e in [-100, 0]).
template <int NP>
__device__ __forceinline__ void scale_pairs(float2 (&w)[NP], int e) {
    const float f = __int_as_float((127 + e) << 23);
#pragma unroll
    for (int p = 0; p < NP; p++) w[p] = __fmul2_rn(w[p], make_float2(f, f));
}

// x * 2^-sigma for the one-power-of-two f16 staging of x: sigma puts the
// largest |x'| in [2^14, 2^15), so x' never overflows f16, and a BF16 value
// (8 significant bits) converts exactly unless it is nonzero and below 2^-17
// after scaling (then its last bit may fall under the f16 subnormal spacing).
// thr = the BF16 magnitude bits of 2^(sigma - 17): a nonzero |x| whose bits are
// below thr is flagged (conservative: some such values would convert exactly).
struct XScale {
    float p;       // 2^-sigma when that is a normal binary32 value
    bool one;      // one multiply suffices
    int sigma;
    uint32_t thr;
};

__device__ __forceinline__ XScale make_xscale(int sigma) {
    XScale x;
    x.sigma = sigma;
    x.one = sigma >= -126 && sigma <= 126;
    x.p = x.one ? __int_as_float((127 - sigma) << 23) : 0.0f;
    const int e = sigma - 17 + 127;   // BF16 biased exponent of 2^(sigma - 17)
    x.thr = e >= 1 ? (uint32_t)e << 7 : (e + 6 >= 0 ? 1u << (e + 6) : 0u);
    return x;
}

// Two BF16 values (one 32-bit word) -> f16x2 of x * 2^-sigma; bad |= not exact.
__device__ __forceinline__ uint32_t x_pair_f16(uint32_t w, const XScale &xs, bool &bad) {
    const float x0 = bf16_lo(w), x1 = bf16_hi(w);
    const float a0 = xs.one ? x0 * xs.p : mul_pow2(x0, -xs.sigma);
    const float a1 = xs.one ? x1 * xs.p : mul_pow2(x1, -xs.sigma);
    const __half2 h = __floats2half2_rn(a0, a1);
    const uint32_t m0 = w & 0x7FFFu, m1 = (w >> 16) & 0x7FFFu;
    bad |= (m0 != 0u && m0 < xs.thr) | (m1 != 0u && m1 < xs.thr);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Two BF16 values -> f16x2 of x * p (p = 2^-sigma, x known to convert exactly).
__device__ __forceinline__ uint32_t x_pair_f16_scaled(uint32_t w, float p) {
    const __half2 h = __floats2half2_rn(bf16_lo(w) * p, bf16_hi(w) * p);
    return *reinterpret_cast<const uint32_t *>(&h);
}

constexpr int kTcRows = 16;                    // rows per tile (one MMA M)
constexpr int kTcWarps = 8;                    // consumer warps, each a contiguous share of a tile's k
constexpr int kTcParts = kTcWarps;
constexpr int kTcThreads = (kTcWarps + 1) * 32; // + one producer warp
constexpr int kTcFbRows = kTcRows / kTcWarps;  // rows per warp on the binary32 path

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two E4M3 bytes (low 16 bits) -> f16x2 (low byte -> low half).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t r;
    const uint16_t b = (uint16_t)(two & 0xFFFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(b));
    return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// 16 code bytes of one row (32 k) times their two group scales -> 16 f16x2
// values (h[i] = elements 2i, 2i+1 of the lane's 32 k).
__device__ __forceinline__ void decode_row32(uint4 c, uint32_t s2, uint32_t (&h)[16]) {
    const uint32_t sc = e4m3x2_to_f16x2(s2);        // (s_lo, s_hi)
    const uint32_t slo = __byte_perm(sc, 0, 0x1010); // (s_lo, s_lo)
    const uint32_t shi = __byte_perm(sc, 0, 0x3232); // (s_hi, s_hi)
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; q++) e2m1x8_to_f16x2(w[q], h + 4 * q);
#pragma unroll
    for (int i = 0; i < 16; i++) h[i] = hmul2_u32(h[i], i < 8 ? slo : shi);
}

// One ROCmFP4 block (32 weights at shared-memory byte address A, any byte
// alignment: Dual = two UE4M3 half scales + 16 code bytes, FAST = one scale +
// 16 code bytes; code byte j holds elements j and j + 16) -> 16 f16x2 words,
// h[j] = (element j * 2 dec(s0), element j+16 * 2 dec(s1)) with the Codebook10
// level / 2 taken as the E2M1 value clamped to [-5, 5] ("rocmwhy" page, format
// table and sections 01-02: level * dec(u), at most 7 significant bits, exact
// in f16).  Six aligned words are read and realigned with funnel shifts.
template <bool DUAL>
__device__ __forceinline__ void decode_rocm_pairs(uint32_t A, uint32_t (&h)[16]) {
    const uint32_t base = A & ~3u, sh = (A & 3u) * 8u;
    uint32_t W[6], S[5];
#pragma unroll
    for (int i = 0; i < 6; i++) W[i] = ld_shared_u32(base + 4u * i);
#pragma unroll
    for (int i = 0; i < 5; i++) S[i] = __funnelshift_r(W[i], W[i + 1], sh);
    const uint32_t u0 = S[0] & 0xFFu, u1 = DUAL ? (S[0] >> 8) & 0xFFu : u0;
    uint32_t C[4];
#pragma unroll
    for (int j = 0; j < 4; j++) C[j] = __funnelshift_r(S[j], S[j + 1], DUAL ? 16 : 8);
    const uint32_t sc = e4m3x2_to_f16x2(u0 | (u1 << 8));
    const __half2 s2 = __hadd2(*reinterpret_cast<const __half2 *>(&sc), *reinterpret_cast<const __half2 *>(&sc));
    const __half2 lim = __floats2half2_rn(5.0f, 5.0f), nlim = __floats2half2_rn(-5.0f, -5.0f);
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const uint32_t e = e2m1x2_to_f16x2(C[i >> 2] >> (8 * (i & 3)));
        const __half2 v = __hmul2(__hmin2(__hmax2(*reinterpret_cast<const __half2 *>(&e), nlim), lim), s2);
        h[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
}

// Sum a tile's parts in a fixed order and store (per-tile reduction mode).
__device__ __forceinline__ void reduce_tile(const GemvTcArgs &a, const float *rb, long long rt, int rows, int nparts,
                                            float gs, int yexp, int slice, int M) {
    for (int i = threadIdx.x; i < rows * M; i += kTcWarps * 32) {
        const int row = i / M, m = i % M;
        float s = 0.0f;
        for (int q = 0; q < nparts; q++) s += rb[(q * kTcRows + row) * M + m];
        const long long n = rt + row;
        const float v = scale_out(s, gs, yexp);
        if (gridDim.y == 1)
            a.y[(size_t)m * a.N + n] = v;
        else
            a.partial[((size_t)slice * M + m) * a.N + n] = v;
    }
}

// The producer lane: x (after the dependency wait) and the weight stages of a
// CTA's row range, in order, into the NS-deep ring.  Under programmatic launch
// the first NS weight stages go out before the wait (weights do not depend on
// earlier kernels); otherwise x goes first.
__device__ __forceinline__ void tc_produce(const CUtensorMap &cmap, const CUtensorMap &smap, const GemvTcArgs &a,
                                           int M, uint16_t *xs, uint8_t *stages, uint64_t *full, uint64_t *empty,
                                           uint64_t *xfull, volatile int *abort, long long r0, long long r1, int k0,
                                           int kcs, int npieces, int nstages) {
    const int K = a.K, KP = a.KP, NS = a.NS, XS = a.xstride;
    const bool nv = a.fmt == W4_FMT_NVFP4;
    const int CS = stage_row_bytes(a.fmt, a.bb, KP), SS = nv ? KP / 16 : 0;
    const int RB = stage_row_bytes(a.fmt, a.bb, K);   // ROCmFP4: bytes of a whole row in memory
    const uint64_t pol = policy_evict_first();
    const int before = a.pdl ? min(NS, nstages) : 0;
    int issued = 0;        // weight stages issued
    bool x_issued = false;
    for (int t = 0; t < nstages + 1; t++) {
        if (t == before) {
            pdl_wait_prior_grid();
            mbar_arrive_expect_tx(xfull, (uint32_t)(M * kcs * 2));
            for (int m = 0; m < M; m++)
                bulk_g2s(xs + (size_t)m * XS, a.x + (size_t)m * K + k0, (uint32_t)(kcs * 2), xfull, pol);
            x_issued = true;
            continue;
        }
        const int tt = t > before ? t - 1 : t;   // weight stage index
        const int st = tt % NS;
        if (tt >= NS && !mbar_wait(empty + st, ((tt / NS) - 1) & 1, abort)) break;
        issued++;
        const long long rt = r0 + (long long)(tt / npieces) * kTcRows;
        const int rows = (int)min((long long)kTcRows, r1 - rt);
        const int kpos = k0 + (tt % npieces) * KP;
        const int kps = min(KP, k0 + kcs - kpos);
        uint8_t *dst = stages + (size_t)st * a.tile_bytes;
        uint8_t *dsts = dst + kTcRows * CS;
        if (!nv) {
            // ROCmFP4: one box of 16 rows x KP/32 blocks (8-byte elements; blocks
            // beyond K and rows beyond N are zero-filled), or row pieces for a short tail
            if (rows == kTcRows || rows >= a.box_min_rows) {
                mbar_arrive_expect_tx(full + st, (uint32_t)(kTcRows * CS));
                tma_load_2d(dst, &cmap, stage_row_bytes(a.fmt, a.bb, kpos) / 8, (int)rt, full + st);
            } else {
                const int pb = stage_row_bytes(a.fmt, a.bb, kps);
                mbar_arrive_expect_tx(full + st, (uint32_t)(rows * pb));
                for (int i = 0; i < rows; i++)
                    bulk_g2s(dst + i * CS, a.codes + (rt + i) * RB + stage_row_bytes(a.fmt, a.bb, kpos), (uint32_t)pb,
                             full + st, pol);
            }
        } else if (rows == kTcRows || rows >= a.box_min_rows) {
            // two boxes of 16 rows x KP (k beyond K and rows beyond N are zero-filled)
            mbar_arrive_expect_tx(full + st, (uint32_t)(kTcRows * (CS + SS)));
            tma_load_2d(dst, &cmap, kpos / 16, (int)rt, full + st);
            tma_load_2d(dsts, &smap, kpos / 16, (int)rt, full + st);
        } else {
            // a short tail: row-piece copies of exactly the bytes needed
            mbar_arrive_expect_tx(full + st, (uint32_t)(rows * (kps / 2 + kps / 16)));
            for (int i = 0; i < rows; i++) {
                bulk_g2s(dst + i * CS, a.codes + (rt + i) * (K / 2) + kpos / 2, (uint32_t)(kps / 2), full + st, pol);
                bulk_g2s(dsts + i * SS, a.scales + (rt + i) * (K / 16) + kpos / 16, (uint32_t)(kps / 16), full + st,
                         pol);
            }
        }
    }
    // no copy may still be landing in shared memory when the CTA exits
    drain_ring(full, NS, issued);
    if (x_issued) mbar_wait_bounded(xfull, 0);
}

// x[M][kcs] (BF16 in shared memory, row stride XS halves) -> f16 x * 2^-sigma,
// in place, each 128-k super-chunk permuted to the MMA operand order: the 8
// values k = 32t + 8j .. +7 go to offset 32j + 8t (VIRT, for ROCmFP4 blocks:
// first put x[j], x[j+16] side by side within each 32-k block).  sigma puts the
// largest |x| in [2^14, 2^15); flags[1] is set when some x does not convert
// exactly (a nonzero |x'| below 2^-17 scaled back differs, Inf / NaN), and the
// caller then takes the binary32 path.  All NW consumer warps take part (named
// barrier 1); flags[2 .. 2 + NW) is scratch.  mx: the largest |x| (BF16 bits).
template <bool VIRT, int NW = kTcWarps>
__device__ __forceinline__ void convert_x_f16(uint16_t *xs, int XS, int M, int kcs, int warp, int lane, int *flags,
                                              int &sigma, uint32_t &mx) {
    mx = 0;
    {
        const int nvec = kcs / 8;
        for (int i = threadIdx.x; i < M * nvec; i += NW * 32) {
            const int m = i / nvec, v = i % nvec;
            const uint4 val = *reinterpret_cast<const uint4 *>(xs + (size_t)m * XS + v * 8);
            const uint32_t w4v[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
            for (int j = 0; j < 4; j++) mx = max(mx, max(w4v[j] & 0x7FFFu, (w4v[j] >> 16) & 0x7FFFu));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 0) flags[2 + warp] = (int)mx;
    named_barrier_sync(1, NW * 32);
    for (int i = 0; i < NW; i++) mx = max(mx, (uint32_t)flags[2 + i]);
    const int emax = (int)((mx >> 7) & 0xFFu);
    sigma = (mx == 0) ? 0 : max(emax, 1) - 127 - 14;
    // A warp owns whole super-chunks (lane l converts vector l % 16 of super-chunk
    // 2i + l / 16), so __syncwarp orders its loads before its stores.
    const int nsc = kcs / 128, total = M * nsc;
    bool bad = mx >= 0x7F80u;   // NaN / Inf: binary32 path
    for (int base = 2 * warp; base < total; base += 2 * NW) {
        const int sc = base + (lane >> 4), q = lane & 15;
        uint4 out = make_uint4(0, 0, 0, 0);
        uint16_t *row = nullptr;
        if (sc < total) {
            row = xs + (size_t)(sc / nsc) * XS + (sc % nsc) * 128;
            uint4 val;
            if (!VIRT) {
                val = *reinterpret_cast<const uint4 *>(row + q * 8);
            } else {
                // virtual vector q of block q/4: x[j], x[j+16] for j = 4(q%4) .. +3
                const uint16_t *blk = row + (q >> 2) * 32 + 4 * (q & 3);
                const uint2 lo = *reinterpret_cast<const uint2 *>(blk);
                const uint2 hi = *reinterpret_cast<const uint2 *>(blk + 16);
                val = make_uint4(__byte_perm(lo.x, hi.x, 0x5410), __byte_perm(lo.x, hi.x, 0x7632),
                                 __byte_perm(lo.y, hi.y, 0x5410), __byte_perm(lo.y, hi.y, 0x7632));
            }
            const uint32_t in[4] = {val.x, val.y, val.z, val.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float x0 = bf16_lo(in[j]), x1 = bf16_hi(in[j]);
                const __half2 h = __floats2half2_rn(mul_pow2(x0, -sigma), mul_pow2(x1, -sigma));
                const float2 back = __half22float2(h);
                bad |= (mul_pow2(back.x, sigma) != x0) | (mul_pow2(back.y, sigma) != x1);
                o[j] = *reinterpret_cast<const uint32_t *>(&h);
            }
            out = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncwarp();
        if (sc < total) *reinterpret_cast<uint4 *>(row + ((q & 3) * 4 + (q >> 2)) * 8) = out;
        __syncwarp();
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(&flags[1], 1);
}

// The binary32 CUDA-core path of one stage (x that could not be rescaled
// exactly into f16): warp w takes rows kTcFbRows*w .. +kTcFbRows-1, lanes
// stride over the scale groups; facc[j][m] accumulates row j, token m.  Kept out
// of line so that its registers do not constrain the tensor-core loop.
template <int FMT, int M>
__device__ __noinline__ void fallback_piece(const uint8_t *tp, const uint16_t *xs, int XS, int kbase, int kps, int CS,
                                            int SS, int rows, int warp, int lane, int fold,
                                            float (&facc)[kTcFbRows][M]) {
    constexpr bool NV = FMT == W4_FMT_NVFP4;
    constexpr int BB = FMT == W4_FMT_ROCMFP4_DUAL ? 18 : 17;
    const int ngr = kps / (NV ? 16 : 32);
#pragma unroll
    for (int j = 0; j < kTcFbRows; j++) {
        const int row = kTcFbRows * warp + j;
        if (row >= rows) continue;
        for (int q = lane; q < ngr; q += 32) {
            if constexpr (!NV) {
                // ROCmFP4 block q: pairs (element j, element j + 16), two half scales
                float s0, s1;
                float2 w[16];
                decode_rocm<FMT == W4_FMT_ROCMFP4_DUAL>(tp + row * CS + q * BB, w, s0, s1);
                scale_pairs(w, fold);
                for (int m = 0; m < M; m++) {
                    float2 xv[16];
                    load_x32_split(xs + (size_t)m * XS + kbase + q * 32, xv);
                    facc[j][m] = dot_group2(w, xv, s0, s1, facc[j][m]);
                }
            } else {
                const uint2 c = *reinterpret_cast<const uint2 *>(tp + row * CS + q * 8);
                const float sv = e4m3_to_f32(tp[kTcRows * CS + row * SS + q]);
                float2 w[8];
                decode_nvfp4(c, w);
                scale_pairs(w, fold);
                for (int m = 0; m < M; m++) {
                    float2 xv[8];
                    load_x16(xs + (size_t)m * XS + kbase + q * 16, xv);
                    facc[j][m] = dot_group<8>(w, xv, sv, facc[j][m]);
                }
            }
        }
    }
}

// FMT: NVFP4, or ROCmFP4 Dual / FAST.  For ROCmFP4 a lane's 32 k of a 128-k
// super-chunk are one 32-weight block: decode_rocm_pairs gives the pairs
// (element j, element j + 16), and x is staged in the same "virtual" order
// (x[j], x[j+16] adjacent within each block), so the MMA operand mapping below
// is the NVFP4 one unchanged.
template <int FMT, int M>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap smap,
                   const GemvTcArgs a) {
    constexpr int NT = (M + 7) / 8;   // n-tiles of 8 tokens
    constexpr bool NV = FMT == W4_FMT_NVFP4;
    constexpr int BB = FMT == W4_FMT_ROCMFP4_DUAL ? 18 : 17;
    extern __shared__ __align__(128) uint8_t smem[];
    const int K = a.K, N = a.N, kc = a.kc, KP = a.KP, NS = a.NS, XS = a.xstride;
    const int slice = blockIdx.y, k0 = slice * kc, kcs = min(kc, K - k0);
    const int npieces = (kcs + KP - 1) / KP;
    const int CS = stage_row_bytes(FMT, BB, KP), SS = NV ? KP / 16 : 0;   // row strides of a stage (bytes)

    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);                              // [M][XS]
    uint8_t *stages = smem + (((size_t)M * XS * 2 + 127) & ~(size_t)127);          // NS x tile_bytes
    float *red = reinterpret_cast<float *>(stages + (size_t)NS * a.tile_bytes);    // [red_tiles][P][16][M]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + (size_t)a.red_tiles * kTcParts * kTcRows * M);
    uint64_t *empty = full + NS;
    uint64_t *xfull = empty + NS;
    int *flags = reinterpret_cast<int *>(xfull + 1);   // [0] abort, [1] inexact x, [2..] per-warp max
    volatile int *abort = flags;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long r0, r1;
    if (a.rows_mode == 0) {
        r0 = (long long)blockIdx.x * N / gridDim.x;
        r1 = (long long)(blockIdx.x + 1) * N / gridDim.x;
    } else {
        r0 = (long long)blockIdx.x * a.tiles_per_cta * kTcRows;
        r1 = min((long long)N, r0 + (long long)a.tiles_per_cta * kTcRows);
    }
    const int ntiles = (int)((r1 - r0 + kTcRows - 1) / kTcRows);
    const int nstages = ntiles * npieces;

    if (threadIdx.x == 0) {
        flags[0] = 0;
        flags[1] = 0;
        for (int i = 0; i < NS; i++) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, kTcWarps);
        }
        mbar_init(xfull, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_allow_dependents();
    const float gs = NV ? __ldg(a.gscale) : 1.0f;   // weights do not depend on earlier kernels; ROCmFP4: no g

    if (warp == kTcWarps) {
        if (lane == 0)
            tc_produce(cmap, smap, a, M, xs, stages, full, empty, xfull, abort, r0, r1, k0, kcs, npieces, nstages);
        return;
    }

    // -------------------------------- consumers --------------------------------
    pdl_wait_prior_grid();   // y may be read by the previous kernel
    mbar_wait(xfull, 0, abort);
    int sigma;
    uint32_t mx;
    convert_x_f16<!NV>(xs, XS, M, kcs, warp, lane, flags, sigma, mx);
    named_barrier_sync(1, kTcWarps * 32);
    const bool fast = flags[1] == 0;
    if (!fast) {
        // an x could not be converted exactly: restage the bf16 values in natural order
        const int nvec = kcs / 8;
        for (int i = threadIdx.x; i < M * nvec; i += kTcWarps * 32) {
            const int m = i / nvec, v = i % nvec;
            *reinterpret_cast<uint4 *>(xs + (size_t)m * XS + v * 8) =
                __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)m * K + k0) + v);
        }
        named_barrier_sync(1, kTcWarps * 32);
    }
    // undo the x scaling (f16 path); the binary32 path folds a power of two into
    // the decoded weights instead when x is huge (fallback_fold)
    const int fold = fast ? 0 : fallback_fold(gs, mx >= ((127u + 100u) << 7));   // largest |x| >= 2^100
    const int yexp = fast ? sigma : -fold;

    const int g = lane >> 2, t4 = lane & 3;
    int st_idx = 0;
    for (int tile = 0; tile < ntiles; tile++) {
        const long long rt = r0 + (long long)tile * kTcRows;
        const int rows = (int)min((long long)kTcRows, r1 - rt);
        // independent accumulator chains: one per MMA of a super-chunk (8) for one
        // 8-token tile; 4 per tile for two tiles (register room: 9 warps put 3 on
        // one SM sub-partition, 168 registers per thread at most)
        constexpr int CH = NT == 1 ? 8 : 4;
        float acc[NT][CH][4];
        float facc[kTcFbRows][M];
#pragma unroll
        for (int n = 0; n < NT; n++)
#pragma unroll
            for (int q = 0; q < CH; q++)
#pragma unroll
                for (int i = 0; i < 4; i++) acc[n][q][i] = 0.0f;
#pragma unroll
        for (int j = 0; j < kTcFbRows; j++)
#pragma unroll
            for (int m = 0; m < M; m++) facc[j][m] = 0.0f;

        for (int piece = 0; piece < npieces; piece++, st_idx++) {
            const int st = st_idx % NS;
            // on expiry the tile is garbage, but the warp still reaches every barrier
            mbar_wait(full + st, (st_idx / NS) & 1, abort);
            const uint8_t *tp = stages + (size_t)st * a.tile_bytes;
            const int kbase = piece * KP;                 // offset inside the slice
            const int kps = min(KP, kcs - kbase);
            if (fast) {
                const int SC = kps / 128;
                const int sb = warp * SC / kTcParts, se = (warp + 1) * SC / kTcParts;
                const uint8_t *c0p = tp + g * CS + 16 * t4;
                const uint8_t *c1p = c0p + 8 * CS;
                const uint8_t *s0p = tp + kTcRows * CS + g * SS + 2 * t4;
                const uint8_t *s1p = s0p + 8 * SS;
                const uint32_t r0a = smem_addr(tp) + (uint32_t)(g * CS + t4 * BB);   // ROCmFP4: block t4 of row g
#pragma unroll 2
                for (int s = sb; s < se; s++) {
                    uint32_t h0[16], h1[16];
                    if constexpr (NV) {
                        decode_row32(*reinterpret_cast<const uint4 *>(c0p + s * 64),
                                     *reinterpret_cast<const uint16_t *>(s0p + s * 8), h0);
                        decode_row32(*reinterpret_cast<const uint4 *>(c1p + s * 64),
                                     *reinterpret_cast<const uint16_t *>(s1p + s * 8), h1);
                    } else {
                        decode_rocm_pairs<FMT == W4_FMT_ROCMFP4_DUAL>(r0a + (uint32_t)(4 * s * BB), h0);
                        decode_rocm_pairs<FMT == W4_FMT_ROCMFP4_DUAL>(r0a + (uint32_t)(8 * CS + 4 * s * BB), h1);
                    }
#pragma unroll
                    for (int n = 0; n < NT; n++) {
                        const int m = n * 8 + g;
#pragma unroll
                        for (int j = 0; j < 4; j++) {   // MMAs 2j, 2j+1: k = 32t + 8j .. +7
                            uint4 xb = make_uint4(0, 0, 0, 0);
                            if (m < M)
                                xb = *reinterpret_cast<const uint4 *>(xs + (size_t)m * XS + kbase + s * 128 + j * 32 +
                                                                      t4 * 8);
                            mma_f16_16816(acc[n][(2 * j) % CH], h0[4 * j], h1[4 * j], h0[4 * j + 1], h1[4 * j + 1],
                                          xb.x, xb.y);
                            mma_f16_16816(acc[n][(2 * j + 1) % CH], h0[4 * j + 2], h1[4 * j + 2], h0[4 * j + 3],
                                          h1[4 * j + 3], xb.z, xb.w);
                        }
                    }
                }
            } else {
                // binary32 CUDA-core path: warp w handles rows kTcFbRows*w ..
                fallback_piece<FMT, M>(tp, xs, XS, kbase, kps, CS, SS, rows, warp, lane, fold, facc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + st);
        }

        // ---- this tile's partial sums -> shared memory ----
        const bool all_at_end = a.red_tiles >= ntiles;
        float *rb = red + (size_t)(all_at_end ? tile : (tile & 1)) * kTcParts * kTcRows * M;
        if (fast) {
#pragma unroll
            for (int n = 0; n < NT; n++) {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int row = g + ((i & 2) ? 8 : 0);
                    const int m = n * 8 + 2 * t4 + (i & 1);
                    float v = 0.0f;
#pragma unroll
                    for (int q = 0; q < CH; q++) v += acc[n][q][i];
                    if (m < M) rb[(warp * kTcRows + row) * M + m] = v;
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < kTcFbRows; j++)
#pragma unroll
                for (int m = 0; m < M; m++) {
                    float v = facc[j][m];
#pragma unroll
                    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                    if (lane == 0) rb[(kTcFbRows * warp + j) * M + m] = v;
                }
        }
        if (!all_at_end) {
            named_barrier_sync(1, kTcWarps * 32);
            reduce_tile(a, rb, rt, rows, fast ? kTcParts : 1, gs, yexp, slice, M);
        }
    }
    if (a.red_tiles >= ntiles) {
        // every tile's parts are in shared memory: one barrier, then all threads sum
        named_barrier_sync(1, kTcWarps * 32);
        const int nparts = fast ? kTcParts : 1;
        const int per_tile = kTcRows * M;
        for (int i = threadIdx.x; i < ntiles * per_tile; i += kTcWarps * 32) {
            const int tile = i / per_tile, row = (i % per_tile) / M, m = i % M;
            const long long n = r0 + (long long)tile * kTcRows + row;
            if (n >= r1) continue;
            const float *rb = red + (size_t)tile * kTcParts * kTcRows * M;
            float s = 0.0f;
            for (int q = 0; q < nparts; q++) s += rb[(q * kTcRows + row) * M + m];
            const float v = scale_out(s, gs, yexp);
            if (gridDim.y == 1)
                a.y[(size_t)m * N + n] = v;
            else
                a.partial[((size_t)slice * M + m) * N + n] = v;
        }
    }
}

}  // namespace w4
