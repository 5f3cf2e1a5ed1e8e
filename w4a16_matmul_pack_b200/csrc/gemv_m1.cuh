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
// Data movement.  The packed weights are read once, so they are not staged in
// shared memory: each lane loads its own MMA operands with 16-byte streaming
// loads straight into registers (lane (g, t) takes 16 code bytes of rows g and
// g+8 and their two scale bytes, per 128-k super-chunk), kM1Depth super-chunks
// at a time, and sixteen warps per SM keep enough of them in flight to stream
// at HBM speed -- on B200 a ring of shared-memory stages fed by bulk copies
// delivered less per SM than direct loads for this access pattern.
//
// Work split.  A CTA owns whole 16-row tiles [t0, t1) of one K slice.  Its
// (tile, super-chunk) items, tile by tile, are cut into sixteen contiguous runs,
// one per warp, so that a warp changes tile (and flushes its partial sums to
// shared memory) only a few times; the CTA adds the partials of a row in warp
// order: the result does not depend on timing.
//
// x is converted to f16 once per CTA, as x itself when every nonzero |x| lies
// in [2^-17, 65280] (decided with one barrier), else as x * 2^-sigma with one
// power of two for the whole slice (its largest |x'| in [2^14, 2^15)), exact
// whenever every nonzero |x'| >= 2^-17; either way permuted per 128-k
// super-chunk to the MMA operand order.  A CTA whose x does not convert exactly (range above 2^31, Inf/NaN)
// computes in binary32 on the CUDA cores from the bf16 x in global memory.  A
// warp's partial sum is scaled to acc * g * 2^sigma in binary64 (the factor
// g * 2^sigma is exact there; one rounding to binary32) before the partials are
// added.
//
// The kernel waits on nothing but its own loads and CTA barriers.
#pragma once

#include "gemv_tc.cuh"

namespace w4 {

constexpr int kM1Warps = 16;
constexpr int kM1Threads = kM1Warps * 32;
constexpr int kM1Depth = 2;   // super-chunks per batch (two batches in flight)

// Shared memory of the one-token kernel: x' [xstride] f16, the partial sums
// [red_tiles][kM1Warps][16] float, flags [2 + 2 * kM1Warps] int (the per-warp
// largest and smallest magnitudes of x).
struct M1Layout {
    size_t red, flags, total;
};

__host__ __device__ __forceinline__ M1Layout m1_layout(int xstride, int red_tiles) {
    M1Layout L;
    L.red = ((size_t)xstride * 2 + 127) & ~(size_t)127;
    L.flags = L.red + (size_t)red_tiles * kM1Warps * kTcRows * 4;
    L.total = L.flags + 4 * (2 + 2 * kM1Warps);
    return L;
}

// 16 code bytes of one row (32 k) -> 16 f16x2 (h[i] = elements 2i, 2i+1), exact.
__device__ __forceinline__ void decode_codes32(uint4 c, uint32_t (&h)[16]) {
    e2m1x8_to_f16x2(c.x, h);
    e2m1x8_to_f16x2(c.y, h + 4);
    e2m1x8_to_f16x2(c.z, h + 8);
    e2m1x8_to_f16x2(c.w, h + 12);
}

// x' in shared memory: per 128-k super-chunk the 128 values in MMA operand
// order (the 8 values k = 32t + 8j .. +7 at offset 32j + 8t) followed by 8
// zeros, so that every lane loads its four B pieces (or zeros) by address.
constexpr int kM1ScStride = 136;   // halves per super-chunk

// x slice (BF16, global) -> x' (f16, x * 2^-sigma) in the zero-padded B
// layout, ending with a CTA barrier whenever x' is used (a CTA whose x does not
// convert exactly returns without one: its binary32 path reads no x').  x is
// first written with sigma = 0 and kept when every value converts exactly (one
// barrier decides).  Otherwise each thread keeps its pieces in registers
// between two more passes: the largest magnitude and the smallest nonzero one
// (two 16-bit lanes at a time) decide sigma and whether the f16 copy is exact,
// and only an exact copy is written (otherwise the CTA computes in binary32
// from global memory).
constexpr int kM1MaxSlice = 32768;   // longest K slice of one CTA
constexpr int kM1XPieces = kM1MaxSlice / 8 / kM1Threads;
constexpr int kM1XRegs = 3;   // pieces a thread keeps in registers (slices up to 12288 k); later ones are read twice

__device__ __forceinline__ void m1_convert_x(const uint16_t *xg, uint16_t *xs, int kcs, int warp, int lane,
                                             int *flags, int &sigma, bool &exact, uint32_t &mx) {
    const uint4 *src = reinterpret_cast<const uint4 *>(xg);
    const int nvec = kcs / 8;
    uint4 val[kM1XRegs];
    uint32_t mx2 = 0u, mn2 = 0xFFFFFFFFu;   // per 16-bit lane: max |x|, min (|x| - 1) over |x| != 0
#pragma unroll
    for (int u = 0; u < kM1XRegs; u++) {
        const int i = threadIdx.x + u * kM1Threads;
        if (i < nvec) val[u] = __ldg(src + i);
    }
    // First try sigma = 0 (x as it is), decided with a single barrier: every
    // nonzero |x| in [2^-17, 65280] (BF16 bits 0x3700 .. 0x477F) converts
    // exactly.  The partial sums do not depend on sigma (powers of two scale
    // every product and sum exactly), so this only saves the statistics pass
    // when x is in that range -- as activations normally are.
    bool ok = true;
#pragma unroll
    for (int u = 0; u < kM1XPieces; u++) {
        const int i = threadIdx.x + u * kM1Threads;
        if (i < nvec) {
            const uint4 v = u < kM1XRegs ? val[u] : __ldg(src + i);
            const uint32_t w4v[4] = {v.x, v.y, v.z, v.w};
            uint32_t hi2 = 0u, lo2 = 0xFFFFFFFFu;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t mag = w4v[j] & 0x7FFF7FFFu;
                hi2 = __vmaxu2(hi2, mag);
                lo2 = __vminu2(lo2, (mag + 0x7FFF7FFFu) ^ 0x80008000u);   // 0 -> 0xFFFF, else |x| - 1
            }
            ok &= max(hi2 & 0xFFFFu, hi2 >> 16) <= 0x477Fu && min(lo2 & 0xFFFFu, lo2 >> 16) + 1u >= 0x3700u;
            const int sc = i >> 4, q = i & 15;
            uint16_t *row = xs + (size_t)sc * kM1ScStride;
            *reinterpret_cast<uint4 *>(row + ((q & 3) * 4 + (q >> 2)) * 8) =
                make_uint4(x_pair_f16_scaled(v.x, 1.0f), x_pair_f16_scaled(v.y, 1.0f), x_pair_f16_scaled(v.z, 1.0f),
                           x_pair_f16_scaled(v.w, 1.0f));
            if (q == 0) *reinterpret_cast<uint4 *>(row + 128) = make_uint4(0, 0, 0, 0);
        }
    }
    if (__syncthreads_and(ok)) {   // also the barrier after the x' writes
        sigma = 0;
        exact = true;
        mx = 0u;
        return;
    }
#pragma unroll
    for (int u = 0; u < kM1XPieces; u++) {
        const int i = threadIdx.x + u * kM1Threads;
        if (i < nvec) {
            const uint4 v = u < kM1XRegs ? val[u] : __ldg(src + i);
            const uint32_t w4v[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t mag = w4v[j] & 0x7FFF7FFFu;
                mx2 = __vmaxu2(mx2, mag);
                mn2 = __vminu2(mn2, (mag + 0x7FFF7FFFu) ^ 0x80008000u);   // 0 -> 0xFFFF, else |x| - 1
            }
        }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, max(mx2 & 0xFFFFu, mx2 >> 16));
    uint32_t mn = __reduce_min_sync(0xFFFFFFFFu, min(mn2 & 0xFFFFu, mn2 >> 16));
    if (lane == 0) flags[2 + warp] = (int)mx, flags[2 + kM1Warps + warp] = (int)mn;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kM1Warps; i++) {
        mx = max(mx, (uint32_t)flags[2 + i]);
        mn = min(mn, (uint32_t)flags[2 + kM1Warps + i]);
    }
    const int emax = (int)((mx >> 7) & 0xFFu);
    sigma = (mx == 0) ? 0 : max(emax, 1) - 127 - 14;
    const XScale xsc = make_xscale(sigma);
    // exact: no NaN / Inf, and every nonzero |x| >= 2^(sigma - 17)
    exact = mx < 0x7F80u && mn + 1u >= xsc.thr;
    if (!exact) return;   // (uniform: the caller's binary32 path reads no x')
    bool unused = false;
#pragma unroll
    for (int u = 0; u < kM1XPieces; u++) {
        const int i = threadIdx.x + u * kM1Threads;
        if (i < nvec) {
            const int sc = i >> 4, q = i & 15;
            const uint4 v = u < kM1XRegs ? val[u] : __ldg(src + i);
            uint4 out;
            if (xsc.one) {
                out = make_uint4(x_pair_f16_scaled(v.x, xsc.p), x_pair_f16_scaled(v.y, xsc.p),
                                 x_pair_f16_scaled(v.z, xsc.p), x_pair_f16_scaled(v.w, xsc.p));
            } else {
                out = make_uint4(x_pair_f16(v.x, xsc, unused), x_pair_f16(v.y, xsc, unused),
                                 x_pair_f16(v.z, xsc, unused), x_pair_f16(v.w, xsc, unused));
            }
            uint16_t *row = xs + (size_t)sc * kM1ScStride;
            *reinterpret_cast<uint4 *>(row + ((q & 3) * 4 + (q >> 2)) * 8) = out;
            if (q == 0) *reinterpret_cast<uint4 *>(row + 128) = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
}

// The CTA's items in order: item i is super-chunk i % SC of tile i / SC.  Warp
// w takes the contiguous run [w n / 16, (w + 1) n / 16) of the n = nt * SC
// items, so it crosses few tile boundaries (each one costs a flush of its
// partial sums).
__device__ __forceinline__ void m1_range(int w, int nt, int SC, int &lo, int &hi) {
    const int n = nt * SC;
    lo = w * n / kM1Warps;
    hi = (w + 1) * n / kM1Warps;
}

// Whether warp w has items of tile j (and so partial sums of it).
__device__ __forceinline__ bool m1_has(int w, int j, int nt, int SC) {
    int lo, hi;
    m1_range(w, nt, SC, lo, hi);
    return lo < hi && lo < (j + 1) * SC && hi > j * SC;
}

// Walks warp w's items: tile j (nt once done), super-chunk s.
struct M1Items {
    int j, s, left;
    __device__ __forceinline__ void first(int w, int nt, int SC) {
        int lo, hi;
        m1_range(w, nt, SC, lo, hi);
        left = hi - lo;
        j = left > 0 ? lo / SC : nt;
        s = lo - (lo / SC) * SC;
    }
    __device__ __forceinline__ void next(int, int nt, int SC) {
        if (--left == 0) {
            j = nt;
        } else if (++s == SC) {
            s = 0;
            j++;
        }
    }
};

// D items of one warp in registers: tile (-1: none), super-chunk, the lane's
// code bytes of rows g and g+8, their scale bytes.
template <int D = kM1Depth>
struct M1Batch {
    int jt[D], st[D];
    uint4 c0[D], c1[D];
    uint32_t s0[D], s1[D];
};

// A lane's view of the CTA's weight rows: the codes and scales of row g of the
// CTA's first tile at the lane's k offset in the K slice, and the last row of
// the matrix relative to that tile.  Rows past it are read as that row (their
// sums land in rows that are never written out), so the loads need no test.
struct M1Rows {
    const uint8_t *c, *s;
    uint32_t RB, SB;   // row strides of codes and scales (bytes)
    int rmax;          // N - 1 - first row of the CTA
};

__device__ __forceinline__ M1Rows m1_rows(const GemvTcArgs &a, int t0, int k0, int t4) {
    M1Rows w;
    const size_t RB = (size_t)a.K / 2, SB = (size_t)a.K / 16, row0 = (size_t)t0 * kTcRows;
    w.c = a.codes + row0 * RB + (size_t)k0 / 2 + 16 * t4;
    w.s = a.scales + row0 * SB + (size_t)k0 / 16 + 2 * t4;
    w.RB = (uint32_t)RB;
    w.SB = (uint32_t)SB;
    w.rmax = (int)((long long)a.N - 1 - (long long)row0);
    return w;
}

// 16 code bytes, read once (evict-first).  The 256-byte L2 fetch size brings
// the row's next three super-chunks into L2 with this one: a warp's run walks
// a tile's super-chunks in order, so its later loads of the row hit L2.
__device__ __forceinline__ uint4 ld_codes16(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.cs.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Issue the loads of the warp's next item into slot d of a batch (streaming:
// read once); the slot's tile becomes -1 once the warp's items run out.
template <int D>
__device__ __forceinline__ void m1_load_one(M1Batch<D> &b, int d, M1Items &it, const M1Rows &w, int warp, int nt,
                                            int SC, int g) {
    b.jt[d] = it.j < nt ? it.j : -1;
    b.st[d] = it.s;
    if (b.jt[d] >= 0) {
        const uint32_t r0 = (uint32_t)min(b.jt[d] * kTcRows + g, w.rmax);
        const uint32_t r1 = (uint32_t)min(b.jt[d] * kTcRows + g + 8, w.rmax);
        const uint32_t kc = (uint32_t)b.st[d] * 64u, ks = (uint32_t)b.st[d] * 8u;
        b.c0[d] = ld_codes16(w.c + ((uint64_t)r0 * w.RB + kc));
        b.c1[d] = ld_codes16(w.c + ((uint64_t)r1 * w.RB + kc));
        b.s0[d] = __ldcs(reinterpret_cast<const unsigned short *>(w.s + ((uint64_t)r0 * w.SB + ks)));
        b.s1[d] = __ldcs(reinterpret_cast<const unsigned short *>(w.s + ((uint64_t)r1 * w.SB + ks)));
        it.next(warp, nt, SC);
    }
}

// Issue the loads of the warp's next D items.
template <int D>
__device__ __forceinline__ void m1_load(M1Batch<D> &b, M1Items &it, const M1Rows &w, int warp, int nt, int SC,
                                        int g) {
#pragma unroll
    for (int d = 0; d < D; d++) m1_load_one(b, d, it, w, warp, nt, SC, g);
}

// The kernel body for one CTA: CTA `cta` of `ncta` working on tiles of one
// problem, K-slice `slice` of `nslices` (split-K partials when nslices > 1).
//
// REFILL: each item's registers get the warp's next item as soon as the item is
// decoded (loads in flight earlier; the grouped launch, measured faster there),
// else a batch's slots are refilled after the whole batch (fewer registers: the
// single-problem kernel, whose split-K bookkeeping leaves no room for REFILL).
template <bool REFILL>
__device__ __forceinline__ void m1_body(const GemvTcArgs &a, int cta, int ncta, int slice, int nslices) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int K = a.K, N = a.N, kc = a.kc;
    const int k0 = slice * kc, kcs = min(kc, K - k0);
    const int SC = kcs / 128;
    const M1Layout L = m1_layout(a.xstride, a.red_tiles);
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    float *red = reinterpret_cast<float *>(smem + L.red);   // [tile][warp][16]
    int *flags = reinterpret_cast<int *>(smem + L.flags);   // [2..] per-warp statistics of x

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = (N + kTcRows - 1) / kTcRows;
    const int t0 = (int)((long long)cta * T / ncta), t1 = (int)((long long)(cta + 1) * T / ncta);
    const int nt = t1 - t0;
    const size_t RB = (size_t)K / 2, SB = (size_t)K / 16;   // row strides of codes and scales
    const int g = lane >> 2, t4 = lane & 3;

    pdl_allow_dependents();
    // The weights do not depend on the previous kernel: the first two batches of
    // this warp's items are loaded before waiting for it (and before x is ready).
    M1Items it;
    it.first(warp, nt, SC);
    M1Batch<> bA, bB;
    const M1Rows wrows = m1_rows(a, t0, k0, t4);
    m1_load(bA, it, wrows, warp, nt, SC, g);
    m1_load(bB, it, wrows, warp, nt, SC, g);
    const float gs = __ldg(a.gscale);
    pdl_wait_prior_grid();   // x (and y, which the previous kernel may read) belong to it

    // x slice -> f16 with one power of two, in the B-operand layout
    int sigma;
    uint32_t mx;
    bool fast;
    m1_convert_x(a.x + k0, xs, kcs, warp, lane, flags, sigma, fast, mx);   // barrier when x' is used
    // binary32 path: partial sums in units of x * 2^fold
    const int fold = fast ? 0 : fallback_fold(gs, mx >= ((127u + 100u) << 7));   // largest |x| >= 2^100
    const int sref = fast ? sigma : -fold;
    const double osc = out_factor(gs, sref);   // partial sums -> units of y

    // MMA operands.  Lane (g, t) holds rows g, g+8 of the codes of k = 32t .. 32t+31
    // (blocks 2t, 2t+1) and B column g.  Column g is block g: it is nonzero only for
    // the k of lanes t = g/2, and only in the MMAs of block g (the four over the
    // first 16 of those k for even g, over the last 16 for odd g).  So lane (g, t) takes its B pieces
    // j = 0..3 (x of k = 32t + 8j .. +7) from x' when g/2 == t and j/2 == g%2,
    // and from the super-chunk's eight zeros otherwise: four loads by address.
    const bool xact = (g >> 1) == t4;
    const bool odd = (g & 1) != 0;
    int xoff[4];
#pragma unroll
    for (int j = 0; j < 4; j++) xoff[j] = (xact && (j >> 1) == (odd ? 1 : 0)) ? 32 * j + 8 * t4 : 128;

    int cur = -1;                      // tile being accumulated
    float accA = 0.0f, accB = 0.0f;    // rows g, g+8 (fast) / row lane/2 (binary32)
    // this warp's partial sums of tile cur -> shared memory
    auto flush = [&]() {
        float* rb = red + ((size_t)cur * kM1Warps + warp) * kTcRows;
        if (fast) {
            accA += __shfl_xor_sync(0xFFFFFFFFu, accA, 1);
            accA += __shfl_xor_sync(0xFFFFFFFFu, accA, 2);
            accB += __shfl_xor_sync(0xFFFFFFFFu, accB, 1);
            accB += __shfl_xor_sync(0xFFFFFFFFu, accB, 2);
            if (t4 == 0) {
                rb[g] = scale_by(accA, osc);
                rb[g + 8] = scale_by(accB, osc);
            }
        } else {
            accA += __shfl_xor_sync(0xFFFFFFFFu, accA, 1);
            if ((lane & 1) == 0) rb[lane >> 1] = scale_by(accA, osc);
        }
        accA = 0.0f;
        accB = 0.0f;
    };
    // the math of one batch (fast path); with REFILL each item's slot takes the
    // warp's next item as soon as its codes and scales are decoded, so that
    // load is in flight while the item's MMAs and the rest of the batch run
    auto compute = [&](M1Batch<> &b) {
#pragma unroll
        for (int d = 0; d < kM1Depth; d++) {
            if (b.jt[d] < 0) break;
            if (b.jt[d] != cur) {
                if (cur >= 0) flush();
                cur = b.jt[d];
            }
            // B pieces of MMA pairs j = 0..3 (x of k = 32t + 8j .. +7, or zero)
            const uint16_t *xp = xs + b.st[d] * kM1ScStride;
            const uint4 b0 = *reinterpret_cast<const uint4 *>(xp + xoff[0]);
            const uint4 b1 = *reinterpret_cast<const uint4 *>(xp + xoff[1]);
            const uint4 b2 = *reinterpret_cast<const uint4 *>(xp + xoff[2]);
            const uint4 b3 = *reinterpret_cast<const uint4 *>(xp + xoff[3]);
            uint32_t h0[16], h1[16];
            decode_codes32(b.c0[d], h0);
            decode_codes32(b.c1[d], h1);
            // the two scales of each row, exact in f16 and then in binary32
            const uint32_t sa = e4m3x2_to_f16x2(b.s0[d]), sb = e4m3x2_to_f16x2(b.s1[d]);
            if constexpr (REFILL) m1_load_one(b, d, it, wrows, warp, nt, SC, g);
            // two chains of four MMAs: block 2t in column 2t of d0, block 2t+1 in column 2t+1 of d1
            float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            mma_f16_16816(d0, h0[0], h1[0], h0[1], h1[1], b0.x, b0.y);
            mma_f16_16816(d1, h0[8], h1[8], h0[9], h1[9], b2.x, b2.y);
            mma_f16_16816(d0, h0[2], h1[2], h0[3], h1[3], b0.z, b0.w);
            mma_f16_16816(d1, h0[10], h1[10], h0[11], h1[11], b2.z, b2.w);
            mma_f16_16816(d0, h0[4], h1[4], h0[5], h1[5], b1.x, b1.y);
            mma_f16_16816(d1, h0[12], h1[12], h0[13], h1[13], b3.x, b3.y);
            mma_f16_16816(d0, h0[6], h1[6], h0[7], h1[7], b1.z, b1.w);
            mma_f16_16816(d1, h0[14], h1[14], h0[15], h1[15], b3.z, b3.w);
            const float2 fa = __half22float2(*reinterpret_cast<const __half2 *>(&sa));
            const float2 fb = __half22float2(*reinterpret_cast<const __half2 *>(&sb));
            accA = __fmaf_rn(fa.x, d0[0], accA);
            accA = __fmaf_rn(fa.y, d1[1], accA);
            accB = __fmaf_rn(fb.x, d0[2], accB);
            accB = __fmaf_rn(fb.y, d1[3], accB);
        }
    };
    if (fast) {
        // software pipeline: one batch's loads are in flight while the other is
        // multiplied (both were issued before the wait for the previous kernel)
        for (;;) {
            if (bA.jt[0] < 0) break;
            compute(bA);
            if constexpr (!REFILL) m1_load(bA, it, wrows, warp, nt, SC, g);
            if (bB.jt[0] < 0) break;
            compute(bB);
            if constexpr (!REFILL) m1_load(bB, it, wrows, warp, nt, SC, g);
        }
    } else {
        // binary32 on the CUDA cores: lane l takes row l/2 of the tile, 64 k of each super-chunk
        // (the loads already issued for the fast path are not used)
        const int row = lane >> 1, half = lane & 1;
        for (it.first(warp, nt, SC); it.j < nt; it.next(warp, nt, SC)) {
            if (it.j != cur) {
                if (cur >= 0) flush();
                cur = it.j;
            }
            const long long r = (long long)(t0 + it.j) * kTcRows + row;
            if (r >= N) continue;
            const int kb = k0 + it.s * 128 + 64 * half;
            const uint8_t *cp = a.codes + r * RB + kb / 2;
            const uint8_t *sp = a.scales + r * SB + kb / 16;
            const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + kb);
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint2 c = __ldg(reinterpret_cast<const uint2 *>(cp + 8 * q));
                float2 w[8], xv[8];
                decode_nvfp4(c, w);
                scale_pairs(w, fold);
                const uint4 u0 = __ldg(xg + 2 * q), u1 = __ldg(xg + 2 * q + 1);
                const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int i = 0; i < 8; i++) xv[i] = make_float2(bf16_lo(wv[i]), bf16_hi(wv[i]));
                accA = dot_group<8>(w, xv, e4m3_to_f32(__ldg(sp + q)), accA);
            }
        }
    }
    if (cur >= 0) flush();
    __syncthreads();

    // rows of the CTA's tiles: the partials of the warps with a share of the tile,
    // in warp order (all sixteen loads issued first; the entries of a warp
    // without a share are never written and not added)
    for (int i = threadIdx.x; i < nt * kTcRows; i += kM1Threads) {
        const int j = i / kTcRows, r = i % kTcRows;
        const long long n = (long long)(t0 + j) * kTcRows + r;
        if (n >= N) continue;
        float v[kM1Warps];
#pragma unroll
        for (int w = 0; w < kM1Warps; w++) v[w] = red[((size_t)j * kM1Warps + w) * kTcRows + r];
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kM1Warps; w++)
            if (m1_has(w, j, nt, SC)) s += v[w];
        if (nslices == 1)
            a.y[n] = s;
        else
            a.partial[(size_t)slice * N + n] = s;
    }
}

__global__ void __launch_bounds__(kM1Threads, 1) gemv_nvfp4_m1_kernel(const GemvTcArgs a) {
    m1_body<false>(a, blockIdx.x, gridDim.x, blockIdx.y, gridDim.y);
}

// Several independent one-token problems in one launch (e.g. the q, k and v
// projections of a layer, or any set of GEMVs that are ready at the same time):
// CTAs [cta0[p], cta0[p+1]) work on problem p, each on its own range of tiles,
// exactly as a CTA of the single-problem kernel does.
constexpr int kMaxGroup = 8;

struct GroupArgs {
    GemvTcArgs a[kMaxGroup];
    int cta0[kMaxGroup + 1];
    int G;
};

__global__ void __launch_bounds__(kM1Threads, 1) gemv_nvfp4_m1_grouped_kernel(const __grid_constant__ GroupArgs g) {
    int p = 0;
    while (p + 1 < g.G && (int)blockIdx.x >= g.cta0[p + 1]) p++;
    m1_body<true>(g.a[p], (int)blockIdx.x - g.cta0[p], g.cta0[p + 1] - g.cta0[p], 0, 1);
}

}  // namespace w4
