// gemv.cuh -- fused dequantise x multiply for decode-sized M (1..16), sm_100a.
//
// y[m][n] = sum_k x[m][k] * w_hat[n][k] over packed NVFP4 or ROCmFP4 rows
// ("Nanbeige4.2-3B-NVFP4A16" card, Serving: the fused W4A16 kernel a decode
// step spends its weight bandwidth on).  HBM-bound: every packed byte is read
// once, at 4.5 / 4.25 bits per weight.
//
// Structure (persistent CTAs, one per SM by default):
//   - CTA c owns a contiguous range of output rows and, for split-K, one
//     slice [k0, k0 + kc) of the reduction (blockIdx.y).
//   - Warp 8 is the producer: one lane streams tiles of TR rows x kc columns
//     (the packed bytes of those row pieces) into an NS-stage shared-memory
//     ring with cp.async.bulk, completion counted on per-stage mbarriers.
//     Weights do not depend on earlier kernels, so it starts before the
//     programmatic-dependent-launch wait.
//   - Warps 0..7 consume: after the PDL wait they stage x[M][k0 .. k0+kc) in
//     shared memory (BF16), then for each tile warp w takes rows
//     {R*(w % NG) .. +R-1} (NG = TR / R row groups) and k-part w / NG of P
//     parts.  A lane owns whole scale groups: it decodes codes in registers
//     (cvt e2m1x2 -> f16x2 -> f32), accumulates the group's partial dot product
//     with packed binary32 FMAs and adds scale * partial to its accumulator.
//   - Per tile the lanes are reduced with xor shuffles, parts are summed in a
//     fixed order, and the row result (times the NVFP4 global scale) is stored
//     -- or, for split-K, written as a slice partial that gemv_finalize sums.
#pragma once

#include "common.cuh"

namespace w4 {

constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvThreads = (kGemvConsumerWarps + 1) * 32;

struct GemvArgs {
    const uint8_t *codes;   // NVFP4 codes [N][K/2] or ROCmFP4 blocks [N][K/32][BB]
    const uint8_t *scales;  // NVFP4 scales [N][K/16]; unused for ROCmFP4
    const float *gscale;    // NVFP4 global scale; unused for ROCmFP4
    const uint16_t *x;      // [M][K] bf16 bits
    float *y;               // [M][N]
    float *partial;         // [S][M][N] when S > 1
    int K, N;
    int kc;                 // slice length (K when S == 1)
    int TR;                 // rows per tile
    int P;                  // k-parts per tile row group
    int NS;                 // pipeline stages
    int tile_bytes;         // bytes of one stage buffer (TR rows)
};

// Bytes of one row piece of kc columns.
template <int FMT>
__host__ __device__ __forceinline__ int row_piece_bytes(int kc) {
    if (FMT == W4_FMT_NVFP4) return kc / 2 + kc / 16;
    return (kc / 32) * (FMT == W4_FMT_ROCMFP4_DUAL ? 18 : 17);
}

// ---- per scale group compute ------------------------------------------------

// 16 bf16 x values (elements 2p, 2p+1 -> pair p) from shared memory.
__device__ __forceinline__ void load_x16(const uint16_t *p, float2 (&xv)[8]) {
    const uint4 u0 = reinterpret_cast<const uint4 *>(p)[0], u1 = reinterpret_cast<const uint4 *>(p)[1];
    const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int q = 0; q < 8; q++) xv[q] = make_float2(bf16_lo(wv[q]), bf16_hi(wv[q]));
}

// 32 bf16 x values paired as (x[j], x[j+16]) -> pair j, matching the ROCmFP4
// code byte j that holds elements j and j+16.
__device__ __forceinline__ void load_x32_split(const uint16_t *p, float2 (&xv)[16]) {
    const uint4 *q4 = reinterpret_cast<const uint4 *>(p);
    const uint4 u0 = q4[0], u1 = q4[1], u2 = q4[2], u3 = q4[3];
    const uint32_t lo[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    const uint32_t hi[8] = {u2.x, u2.y, u2.z, u2.w, u3.x, u3.y, u3.z, u3.w};
#pragma unroll
    for (int q = 0; q < 8; q++) {
        xv[2 * q] = make_float2(bf16_lo(lo[q]), bf16_lo(hi[q]));
        xv[2 * q + 1] = make_float2(bf16_hi(lo[q]), bf16_hi(hi[q]));
    }
}

// NVFP4 16-weight group: 8 code bytes -> 8 (even, odd) E2M1 value pairs.
__device__ __forceinline__ void decode_nvfp4(uint2 c, float2 (&w)[8]) {
    const uint32_t cw[2] = {c.x, c.y};
#pragma unroll
    for (int p = 0; p < 8; p++) {
        const uint32_t h = e2m1x2_to_f16x2(cw[p >> 2] >> (8 * (p & 3)));
        w[p] = __half22float2(*reinterpret_cast<const __half2 *>(&h));
    }
}

// ROCmFP4 32-weight block: pair j = (element j, element j+16) as Codebook10
// level / 2 (the E2M1 value of the same nibble, except index 7 -> 5 instead
// of 6: clamp to [-5, 5]); s0 / s1 = 2 * scale of elements 0..15 / 16..31.
template <bool DUAL>
__device__ __forceinline__ void decode_rocm(const uint8_t *blk, float2 (&w)[16], float &s0, float &s1) {
    constexpr int hdr = DUAL ? 2 : 1;
    s0 = 2.0f * e4m3_to_f32(blk[0]);
    s1 = DUAL ? 2.0f * e4m3_to_f32(blk[1]) : s0;
    const __half2 lim = __floats2half2_rn(5.0f, 5.0f);
    const __half2 nlim = __floats2half2_rn(-5.0f, -5.0f);
#pragma unroll
    for (int j = 0; j < 16; j++) {
        const uint32_t h = e2m1x2_to_f16x2(blk[hdr + j]);
        __half2 v = *reinterpret_cast<const __half2 *>(&h);
        v = __hmin2(__hmax2(v, nlim), lim);
        w[j] = __half22float2(v);
    }
}

// acc + s * sum(w . x) over one scale group (packed binary32 FMAs).
template <int NP>
__device__ __forceinline__ float dot_group(const float2 (&w)[NP], const float2 (&xv)[NP], float s, float acc) {
    float2 part = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int p = 0; p < NP; p++) part = __ffma2_rn(w[p], xv[p], part);
    return __fmaf_rn(s, part.x + part.y, acc);
}

// As dot_group, with the two lanes of each pair scaled separately (Dual halves).
__device__ __forceinline__ float dot_group2(const float2 (&w)[16], const float2 (&xv)[16], float s0, float s1,
                                            float acc) {
    float2 part = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int p = 0; p < 16; p++) part = __ffma2_rn(w[p], xv[p], part);
    return __fmaf_rn(s1, part.y, __fmaf_rn(s0, part.x, acc));
}

// ---- kernel -----------------------------------------------------------------

template <int FMT, int M, int R>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int K = a.K, N = a.N, kc = a.kc, TR = a.TR, P = a.P, NS = a.NS;
    const int NG = TR / R;
    const int slice = blockIdx.y;
    const int k0 = slice * kc;
    const int kcs = min(kc, K - k0);                 // this slice's length (last may be shorter)
    const int rowB = row_piece_bytes<FMT>(kc);       // smem stride of a row piece
    const int rowBs = row_piece_bytes<FMT>(kcs);     // bytes copied per row piece
    const int fullRowB = row_piece_bytes<FMT>(K);
    const int codeB = (FMT == W4_FMT_NVFP4) ? kc / 2 : rowB;  // code bytes per row piece

    // shared memory carve-up
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);                         // [M][kc] bf16
    uint8_t *stages = smem + (((size_t)M * kc * 2 + 127) & ~(size_t)127);      // NS x tile_bytes
    float *red = reinterpret_cast<float *>(stages + (size_t)NS * a.tile_bytes); // [2][TR][P][M]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * TR * P * M);
    uint64_t *empty = full + NS;
    volatile int *abort = reinterpret_cast<volatile int *>(empty + NS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long r0 = (long long)blockIdx.x * N / gridDim.x;
    const long long r1 = (long long)(blockIdx.x + 1) * N / gridDim.x;
    const int nrows = (int)(r1 - r0);
    const int ntiles = (nrows + TR - 1) / TR;

    if (threadIdx.x == 0) {
        *abort = 0;
        for (int i = 0; i < NS; i++) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, kGemvConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_allow_dependents();

    if (warp == kGemvConsumerWarps) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int issued = 0;
            for (int t = 0; t < ntiles; t++) {
                const int st = t % NS;
                if (t >= NS && !mbar_wait(empty + st, ((t / NS) - 1) & 1, abort)) break;
                issued++;
                const long long rt = r0 + (long long)t * TR;
                const int rows = (int)min((long long)TR, r1 - rt);
                uint8_t *dst = stages + (size_t)st * a.tile_bytes;
                mbar_arrive_expect_tx(full + st, (uint32_t)(rows * rowBs));
                if (FMT == W4_FMT_NVFP4) {
                    uint8_t *dsts = dst + (size_t)TR * codeB;
                    if (kcs == K) {
                        bulk_g2s(dst, a.codes + rt * (K / 2), (uint32_t)(rows * (K / 2)), full + st, pol);
                        bulk_g2s(dsts, a.scales + rt * (K / 16), (uint32_t)(rows * (K / 16)), full + st, pol);
                    } else {
                        for (int i = 0; i < rows; i++) {
                            bulk_g2s(dst + i * (kc / 2), a.codes + (rt + i) * (K / 2) + k0 / 2,
                                     (uint32_t)(kcs / 2), full + st, pol);
                            bulk_g2s(dsts + i * (kc / 16), a.scales + (rt + i) * (K / 16) + k0 / 16,
                                     (uint32_t)(kcs / 16), full + st, pol);
                        }
                    }
                } else {
                    const int off = row_piece_bytes<FMT>(k0);
                    if (kcs == K) {
                        bulk_g2s(dst, a.codes + rt * fullRowB, (uint32_t)(rows * rowB), full + st, pol);
                    } else {
                        for (int i = 0; i < rows; i++)
                            bulk_g2s(dst + i * rowB, a.codes + (rt + i) * fullRowB + off, (uint32_t)rowBs,
                                     full + st, pol);
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            drain_ring(full, NS, issued);
        }
        return;
    }

    // -------------------------------- consumers --------------------------------
    pdl_wait_prior_grid();  // x (and y) belong to the previous kernel on the stream
    {
        const int nvec = kcs / 8;  // uint4 = 8 bf16
        for (int i = threadIdx.x; i < M * nvec; i += kGemvConsumerWarps * 32) {
            const int m = i / nvec, v = i % nvec;
            const uint4 val = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)m * K + k0) + v);
            reinterpret_cast<uint4 *>(xs + (size_t)m * kc)[v] = val;
        }
    }
    named_barrier_sync(1, kGemvConsumerWarps * 32);

    const float g = (FMT == W4_FMT_NVFP4) ? __ldg(a.gscale) : 1.0f;
    const int gi = warp % NG, pi = warp / NG;
    constexpr int GW = (FMT == W4_FMT_NVFP4) ? 16 : 32;  // weights per scale group of a lane
    const int ngroups = kcs / GW;
    const int gbeg = pi * ngroups / P, gend = (pi + 1) * ngroups / P;

    for (int t = 0; t < ntiles; t++) {
        const int st = t % NS;
        // On expiry the tile is garbage but the warp still takes part in the
        // barriers below, so the CTA ends; the error word reports the failure.
        mbar_wait(full + st, (t / NS) & 1, abort);
        const long long rt = r0 + (long long)t * TR;
        const int rows = (int)min((long long)TR, r1 - rt);
        const uint8_t *tile = stages + (size_t)st * a.tile_bytes;

        float acc[R][M];
#pragma unroll
        for (int j = 0; j < R; j++)
#pragma unroll
            for (int m = 0; m < M; m++) acc[j][m] = 0.0f;

        for (int gq = gbeg + lane; gq < gend; gq += 32) {
            if constexpr (FMT == W4_FMT_NVFP4) {
                const uint8_t *sbase = tile + (size_t)TR * codeB;
                if constexpr (M <= 4) {
                    // x of this group in registers, reused by the R rows
                    float2 xv[M][8];
#pragma unroll
                    for (int m = 0; m < M; m++) load_x16(xs + (size_t)m * kc + gq * 16, xv[m]);
#pragma unroll
                    for (int j = 0; j < R; j++) {
                        const int row = gi * R + j;
                        if (row < rows) {
                            const uint2 c = *reinterpret_cast<const uint2 *>(tile + (size_t)row * codeB + gq * 8);
                            const float s = e4m3_to_f32(sbase[(size_t)row * (kc / 16) + gq]);
                            float2 w[8];
                            decode_nvfp4(c, w);
#pragma unroll
                            for (int m = 0; m < M; m++) acc[j][m] = dot_group<8>(w, xv[m], s, acc[j][m]);
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < R; j++) {
                        const int row = gi * R + j;
                        if (row < rows) {
                            const uint2 c = *reinterpret_cast<const uint2 *>(tile + (size_t)row * codeB + gq * 8);
                            const float s = e4m3_to_f32(sbase[(size_t)row * (kc / 16) + gq]);
                            float2 w[8];
                            decode_nvfp4(c, w);
#pragma unroll
                            for (int m = 0; m < M; m++) {
                                float2 xv[8];
                                load_x16(xs + (size_t)m * kc + gq * 16, xv);
                                acc[j][m] = dot_group<8>(w, xv, s, acc[j][m]);
                            }
                        }
                    }
                }
            } else {
                constexpr bool DUAL = (FMT == W4_FMT_ROCMFP4_DUAL);
                constexpr int BB = DUAL ? 18 : 17;
                if constexpr (M <= 4) {
                    float2 xv[M][16];
#pragma unroll
                    for (int m = 0; m < M; m++) load_x32_split(xs + (size_t)m * kc + gq * 32, xv[m]);
#pragma unroll
                    for (int j = 0; j < R; j++) {
                        const int row = gi * R + j;
                        if (row < rows) {
                            const uint8_t *blk = tile + (size_t)row * rowB + gq * BB;
                            float s0, s1;
                            float2 w[16];
                            decode_rocm<DUAL>(blk, w, s0, s1);
#pragma unroll
                            for (int m = 0; m < M; m++) acc[j][m] = dot_group2(w, xv[m], s0, s1, acc[j][m]);
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < R; j++) {
                        const int row = gi * R + j;
                        if (row < rows) {
                            const uint8_t *blk = tile + (size_t)row * rowB + gq * BB;
                            float s0, s1;
                            float2 w[16];
                            decode_rocm<DUAL>(blk, w, s0, s1);
#pragma unroll
                            for (int m = 0; m < M; m++) {
                                float2 xv[16];
                                load_x32_split(xs + (size_t)m * kc + gq * 32, xv);
                                acc[j][m] = dot_group2(w, xv, s0, s1, acc[j][m]);
                            }
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + st);

        // lane reduction, fixed xor order
#pragma unroll
        for (int j = 0; j < R; j++)
#pragma unroll
            for (int m = 0; m < M; m++) {
                float v = acc[j][m];
#pragma unroll
                for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                acc[j][m] = v;
            }
        float *rb = red + (size_t)(t & 1) * TR * P * M;
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < R; j++)
#pragma unroll
                for (int m = 0; m < M; m++) rb[((gi * R + j) * P + pi) * M + m] = acc[j][m];
        }
        named_barrier_sync(1, kGemvConsumerWarps * 32);
        for (int i = threadIdx.x; i < rows * M; i += kGemvConsumerWarps * 32) {
            const int row = i / M, m = i % M;
            float s = 0.0f;
            for (int q = 0; q < P; q++) s += rb[(row * P + q) * M + m];
            const long long n = rt + row;
            if (gridDim.y == 1)
                a.y[(size_t)m * N + n] = g * s;
            else
                a.partial[((size_t)slice * M + m) * N + n] = s;
        }
    }
}

// y[m][n] = g * sum_s partial[s][m][n], slices in order.
__global__ void gemv_finalize_kernel(const float *__restrict__ partial, int S, int MN,
                                     const float *__restrict__ gscale, float *__restrict__ y) {
    const float g = gscale ? __ldg(gscale) : 1.0f;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < MN; i += gridDim.x * blockDim.x) {
        float s = 0.0f;
        for (int q = 0; q < S; q++) s += partial[(size_t)q * MN + i];
        y[i] = g * s;
    }
}

}  // namespace w4
