// gemv_skinny.cuh -- NVFP4 GEMV for M = 2..16 tokens (skinny GEMM: decode of a
// small batch, the speculative-verify step): y[m][n] = g * sum_k x[m][k] *
// e2m1[n][k] * scale[n][k/16] ("EdgeRock-4B-NVFP4" card, intro; the batched
// decode and n-gram verification of the "Nanbeige4.2-3B-NVFP4A16" card,
// Serving).
//
// The structure of the one-token kernel (gemv_m1.cuh): sixteen warps, whole
// 16-row tiles per CTA, every warp a rotating share of each tile's 128-k
// super-chunks, its MMA operands loaded straight from HBM into registers.
// With several tokens the B columns are the tokens, so the block scale is
// applied to the decoded codes first (E2M1 * E4M3 has at most 6 significant
// bits: exact in f16, one HMUL2 per pair), and the MMAs accumulate a tile's
// super-chunks directly in their C operand.  x of the K slice is staged once
// per CTA as f16 rows (one power of two for all of x, exact whenever every
// nonzero |x'| >= 2^-17; otherwise the CTA computes in binary32 from global
// memory); within a super-chunk the 16-byte pieces of the four lanes of a row
// are interleaved and the rows lie 64 bytes apart modulo 128, so that the
// loads of a warp fall on distinct banks.  Per-warp partial sums of the CTA's
// tiles are added in warp order (no atomics).  A K too long for the
// x slice runs in slices whose partials gemv_finalize_kernel adds.
#pragma once

#include "gemv_m1.cuh"

namespace w4 {

// x' of the slice: NT*8 token rows of xstride halves (slice length + 32).
// Partial sums: [red_tiles][kM1Warps][16][MP] float (MP = M rounded up to 4).
// Flags: [2 + 2 * kM1Warps] int (the per-warp largest and smallest magnitudes of x).
constexpr size_t kSkinnyXBytes = 96 * 1024;

__host__ __device__ constexpr int skinny_pad(int M) { return (M + 3) / 4 * 4; }

// Longest K slice whose x' fits kSkinnyXBytes (rows padded to 8 tokens).
__host__ __device__ constexpr int skinny_kmax(int M) {
    return (int)((kSkinnyXBytes / (2 * (size_t)((M + 7) / 8 * 8)) - 32) / 256 * 256);
}

// 16-byte pieces of an x slice that one thread converts, at most.
__host__ __device__ constexpr int skinny_pieces(int M) {
    return (M * (skinny_kmax(M) / 8) + kM1Threads - 1) / kM1Threads;
}

__host__ __device__ __forceinline__ M1Layout skinny_layout(int M, int xstride, int red_tiles) {
    const int R = (M + 7) / 8 * 8;
    M1Layout L;
    L.red = ((size_t)R * xstride * 2 + 127) & ~(size_t)127;
    L.flags = L.red + (size_t)red_tiles * kM1Warps * kTcRows * skinny_pad(M) * 4;
    L.total = L.flags + 4 * (2 + 2 * kM1Warps);
    return L;
}

// x[M][K] slice (BF16, global; SC super-chunks of 128 k from k0) -> x' rows
// (f16, x * 2^-sigma), ending with a CTA barrier whenever x' is used (the
// binary32 path of an inexact x reads no x').  x is first written with
// sigma = 0 and kept when every value converts exactly (one barrier decides).
// Otherwise each thread holds its pieces in registers between two more
// passes: the largest magnitude and the smallest nonzero one (two 16-bit lanes
// at a time) decide sigma and whether the f16 copy is exact; only then is it
// written.  Token rows M .. 8*NT-1 are left as they are: they only feed
// MMA columns whose sums are never read.
template <int M>
__device__ __forceinline__ void skinny_convert_x(const uint16_t *x, int K, int k0, int SC, uint16_t *xs, int XS,
                                                 int warp, int lane, int *flags, int &sigma, bool &exact,
                                                 uint32_t &mx) {
    constexpr int V = skinny_pieces(M);
    const int total = M * 16 * SC;
    uint4 val[V];
    uint32_t mx2 = 0u, mn2 = 0xFFFFFFFFu;   // per 16-bit lane: max |x|, min (|x| - 1) over |x| != 0
#pragma unroll
    for (int u = 0; u < V; u++) {
        const int i = threadIdx.x + u * kM1Threads;
        if (i < total) {
            const int q = i & 15, r = i >> 4, m = r % M, sc = r / M;
            val[u] = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)m * K + k0 + sc * 128) + q);
        }
    }
    // First try sigma = 0 (x as it is), decided with one barrier: every nonzero
    // |x| in [2^-17, 65280] (BF16 bits 0x3700 .. 0x477F) converts exactly, and
    // the partial sums do not depend on sigma (powers of two scale every product
    // and sum exactly).  Up to 8 tokens only: above that the extra pass costs
    // the fast path registers (measured slower at 16 tokens).
    if constexpr (M <= 8) {
        bool ok = true;
#pragma unroll
        for (int u = 0; u < V; u++) {
            const int i = threadIdx.x + u * kM1Threads;
            if (i < total) {
                const int q = i & 15, r = i >> 4, m = r % M, sc = r / M;
                const uint32_t w4v[4] = {val[u].x, val[u].y, val[u].z, val[u].w};
                uint32_t hi2 = 0u, lo2 = 0xFFFFFFFFu;
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const uint32_t mag = w4v[j] & 0x7FFF7FFFu;
                    hi2 = __vmaxu2(hi2, mag);
                    lo2 = __vminu2(lo2, (mag + 0x7FFF7FFFu) ^ 0x80008000u);
                }
                ok &= max(hi2 & 0xFFFFu, hi2 >> 16) <= 0x477Fu && min(lo2 & 0xFFFFu, lo2 >> 16) + 1u >= 0x3700u;
                *reinterpret_cast<uint4 *>(xs + (size_t)m * XS + sc * 128 + ((q & 3) * 4 + (q >> 2)) * 8) =
                    make_uint4(x_pair_f16_scaled(val[u].x, 1.0f), x_pair_f16_scaled(val[u].y, 1.0f),
                               x_pair_f16_scaled(val[u].z, 1.0f), x_pair_f16_scaled(val[u].w, 1.0f));
            }
        }
        if (__syncthreads_and(ok)) {   // also the barrier after the x' writes
            sigma = 0;
            exact = true;
            mx = 0u;
            return;
        }
    }
#pragma unroll
    for (int u = 0; u < V; u++) {
        if (threadIdx.x + u * kM1Threads < total) {
            const uint32_t w4v[4] = {val[u].x, val[u].y, val[u].z, val[u].w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t mag = w4v[j] & 0x7FFF7FFFu;
                mx2 = __vmaxu2(mx2, mag);
                // |x| = 0 -> 0xFFFF, else |x| - 1 (no carry between the lanes: mag <= 0x7FFF)
                mn2 = __vminu2(mn2, (mag + 0x7FFF7FFFu) ^ 0x80008000u);
            }
        }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, max(mx2 & 0xFFFFu, mx2 >> 16));
    uint32_t mn = __reduce_min_sync(0xFFFFFFFFu, min(mn2 & 0xFFFFu, mn2 >> 16));
    if (lane == 0) flags[2 + warp] = (int)mx, flags[2 + kM1Warps + warp] = (int)mn;
    __syncthreads();
    for (int i = 0; i < kM1Warps; i++) {
        mx = max(mx, (uint32_t)flags[2 + i]);
        mn = min(mn, (uint32_t)flags[2 + kM1Warps + i]);
    }
    const int emax = (int)((mx >> 7) & 0xFFu);
    sigma = (mx == 0) ? 0 : max(emax, 1) - 127 - 14;
    const XScale xsc = make_xscale(sigma);
    // exact: no NaN / Inf, and every nonzero |x| >= 2^(sigma - 17)
    exact = mx < 0x7F80u && mn + 1u >= xsc.thr;
    if (!exact) return;
    bool unused = false;
#pragma unroll
    for (int u = 0; u < V; u++) {
        const int i = threadIdx.x + u * kM1Threads;
        if (i < total) {
            const int q = i & 15, r = i >> 4, m = r % M, sc = r / M;
            uint4 out;
            if (xsc.one) {
                out = make_uint4(x_pair_f16_scaled(val[u].x, xsc.p), x_pair_f16_scaled(val[u].y, xsc.p),
                                 x_pair_f16_scaled(val[u].z, xsc.p), x_pair_f16_scaled(val[u].w, xsc.p));
            } else {
                out = make_uint4(x_pair_f16(val[u].x, xsc, unused), x_pair_f16(val[u].y, xsc, unused),
                                 x_pair_f16(val[u].z, xsc, unused), x_pair_f16(val[u].w, xsc, unused));
            }
            // 16-byte piece j of lane t's 32 k of a super-chunk at piece 4j + t
            *reinterpret_cast<uint4 *>(xs + (size_t)m * XS + sc * 128 + ((q & 3) * 4 + (q >> 2)) * 8) = out;
        }
    }
    __syncthreads();
}

// The binary32 path of one CTA (x that could not be rescaled exactly into
// f16): lane l takes row l/2 of each tile and 64 k of each of the warp's
// super-chunks, every token; writes the warp's partial sums of each tile to
// red.  Kept out of line so that its registers do not constrain the fast path.
template <int M>
__device__ __noinline__ void skinny_fallback(const GemvTcArgs &a, float *red, int warp, int lane, int nt, int SC,
                                             int t0, int k0, float gs, int fold, int sref) {
    const int K = a.K, N = a.N;
    const double osc = out_factor(gs, sref);
    const size_t RB = (size_t)K / 2, SB = (size_t)K / 16;
    const int row = lane >> 1, half = lane & 1;
    float facc[M];
#pragma unroll
    for (int m = 0; m < M; m++) facc[m] = 0.0f;
    int cur = -1;
    auto flush = [&]() {
        float *rb = red + ((size_t)cur * kM1Warps + warp) * kTcRows * skinny_pad(M);
#pragma unroll
        for (int m = 0; m < M; m++) {
            facc[m] += __shfl_xor_sync(0xFFFFFFFFu, facc[m], 1);
            if ((lane & 1) == 0) rb[(lane >> 1) * skinny_pad(M) + m] = scale_by(facc[m], osc);
            facc[m] = 0.0f;
        }
    };
    M1Items it;
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
        for (int q = 0; q < 4; q++) {
            const uint2 c = __ldg(reinterpret_cast<const uint2 *>(cp + 8 * q));
            float2 w[8];
            decode_nvfp4(c, w);
            scale_pairs(w, fold);
            const float sv = e4m3_to_f32(__ldg(sp + q));
#pragma unroll
            for (int m = 0; m < M; m++) {
                float2 xv[8];
                load_x16(a.x + (size_t)m * K + kb + 16 * q, xv);
                facc[m] = dot_group<8>(w, xv, sv, facc[m]);
            }
        }
    }
    if (cur >= 0) flush();
}

template <int M>
__global__ void __launch_bounds__(kM1Threads, 1) gemv_nvfp4_skinny_kernel(const GemvTcArgs a) {
    constexpr int NT = (M + 7) / 8;   // n-tiles of 8 tokens
    constexpr int D = M <= 8 ? 2 : 1; // super-chunks per batch (two batches in flight)
    constexpr int MP = skinny_pad(M), M4 = MP / 4;
    extern __shared__ __align__(128) uint8_t smem[];
    const int K = a.K, N = a.N, kc = a.kc, XS = a.xstride;
    const int slice = blockIdx.y, nslices = gridDim.y;
    const int k0 = slice * kc, kcs = min(kc, K - k0);
    const int SC = kcs / 128;
    const M1Layout L = skinny_layout(M, XS, a.red_tiles);
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    float *red = reinterpret_cast<float *>(smem + L.red);   // [tile][warp][16][M]
    int *flags = reinterpret_cast<int *>(smem + L.flags);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = (N + kTcRows - 1) / kTcRows;
    const int cta = blockIdx.x, ncta = gridDim.x;
    const int t0 = (int)((long long)cta * T / ncta), t1 = (int)((long long)(cta + 1) * T / ncta);
    const int nt = t1 - t0;
    const int g = lane >> 2, t4 = lane & 3;

    pdl_allow_dependents();
    // the first batch of this warp's weights is loaded before waiting for the
    // previous kernel (and before x is ready)
    M1Items it;
    it.first(warp, nt, SC);
    M1Batch<D> bA, bB;
    const M1Rows wrows = m1_rows(a, t0, k0, t4);
    m1_load(bA, it, wrows, warp, nt, SC, g);
    const float gs = __ldg(a.gscale);
    pdl_wait_prior_grid();
    int sigma;
    uint32_t mx;
    bool fast;
    skinny_convert_x<M>(a.x, K, k0, SC, xs, XS, warp, lane, flags, sigma, fast, mx);   // barrier when x' is used
    const int fold = fast ? 0 : fallback_fold(gs, mx >= ((127u + 100u) << 7));   // largest |x| >= 2^100
    const int sref = fast ? sigma : -fold;
    const double osc = out_factor(gs, sref);   // partial sums -> units of y

    int cur = -1;                       // tile being accumulated
    float acc[NT][4];                   // MMA C fragments (rows g, g+8 x tokens 8nt + 2t, +1)
#pragma unroll
    for (int q = 0; q < NT; q++) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
    // this warp's partial sums of tile cur -> shared memory
    auto flush = [&]() {
        float *rb = red + ((size_t)cur * kM1Warps + warp) * kTcRows * MP;
#pragma unroll
        for (int q = 0; q < NT; q++) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int row = g + 8 * (e >> 1), m = 8 * q + 2 * t4 + (e & 1);
                if (m < M) rb[row * MP + m] = scale_by(acc[q][e], osc);
                acc[q][e] = 0.0f;
            }
        }
    };
    // the math of one batch (fast path)
    auto compute = [&](const M1Batch<D> &b) {
#pragma unroll
        for (int d = 0; d < D; d++) {
            if (b.jt[d] < 0) break;
            if (b.jt[d] != cur) {
                if (cur >= 0) flush();
                cur = b.jt[d];
            }
            uint32_t h0[16], h1[16];
            decode_row32(b.c0[d], b.s0[d], h0);   // e2m1 * scale, f16, exact
            decode_row32(b.c1[d], b.s1[d], h1);
#pragma unroll
            for (int q = 0; q < NT; q++) {
                // x of token 8q + g, k = 32t .. 32t+31 of the super-chunk (pieces 4v + t)
                const uint4 *xp = reinterpret_cast<const uint4 *>(xs + (size_t)(8 * q + g) * XS + b.st[d] * 128) + t4;
                uint32_t xv[16];
#pragma unroll
                for (int v = 0; v < 4; v++) {
                    const uint4 u = xp[4 * v];
                    xv[4 * v] = u.x, xv[4 * v + 1] = u.y, xv[4 * v + 2] = u.z, xv[4 * v + 3] = u.w;
                }
#pragma unroll
                for (int j = 0; j < 8; j++)
                    mma_f16_16816(acc[q], h0[2 * j], h1[2 * j], h0[2 * j + 1], h1[2 * j + 1], xv[2 * j], xv[2 * j + 1]);
            }
        }
    };
    if (fast) {
        // software pipeline: the next batch's loads are in flight while this one is multiplied
        for (;;) {
            if (bA.jt[0] < 0) break;
            m1_load(bB, it, wrows, warp, nt, SC, g);
            compute(bA);
            if (bB.jt[0] < 0) break;
            m1_load(bA, it, wrows, warp, nt, SC, g);
            compute(bB);
        }
        if (cur >= 0) flush();
    } else {
        skinny_fallback<M>(a, red, warp, lane, nt, SC, t0, k0, gs, fold, sref);
    }
    __syncthreads();

    // rows of the CTA's tiles, four tokens at a time: the partials of the warps
    // with a share of the tile, in warp order (all sixteen loads issued first;
    // the entries of a warp without a share are never written and not added)
    for (int i = threadIdx.x; i < nt * kTcRows * M4; i += kM1Threads) {
        const int c = i % M4, r = (i / M4) % kTcRows, j = i / (M4 * kTcRows);
        const long long n = (long long)(t0 + j) * kTcRows + r;
        if (n >= N) continue;
        const float4 *src = reinterpret_cast<const float4 *>(red + ((size_t)j * kM1Warps * kTcRows + r) * MP) + c;
        float4 v[kM1Warps];
#pragma unroll
        for (int w = 0; w < kM1Warps; w++) v[w] = src[(size_t)w * kTcRows * M4];
        float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
        for (int w = 0; w < kM1Warps; w++)
            if (m1_has(w, j, nt, SC)) s0 += v[w].x, s1 += v[w].y, s2 += v[w].z, s3 += v[w].w;
        const float o[4] = {s0, s1, s2, s3};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int m = 4 * c + e;
            if (m >= M) break;
            if (nslices == 1)
                a.y[(size_t)m * N + n] = o[e];
            else
                a.partial[((size_t)slice * M + m) * N + n] = o[e];
        }
    }
}

}  // namespace w4
