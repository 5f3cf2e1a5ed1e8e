// gemv.cuh -- per-group decode and dot-product helpers of the decode GEMVs
// binary32 CUDA-core paths (used when x cannot be rescaled exactly into f16),
// and the fixed-order sum of split-K partials.
//
// y[m][n] = sum_k x[m][k] * w_hat[n][k] over packed NVFP4 or ROCmFP4 rows
// ("Nanbeige4.2-3B-NVFP4A16" card, Serving: the fused W4A16 kernel a decode
// step spends its weight bandwidth on).  The tensor-core kernels live in
// gemv_tc.cuh (M = 1..16, both formats) and gemv_m1.cuh (one NVFP4 token).
#pragma once

#include "common.cuh"

namespace w4 {

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

// Decode GEMV for any K the packers accept (K % 16 == 0 for NVFP4, K % 32 for
// ROCmFP4), used when K is not a multiple of the fast kernels' 256 / 512: one
// warp per weight row, lanes stride over the scale groups reading the packed
// bytes and x straight from global memory, products and sums in binary64 (the
// products of E2M1 or Codebook10 values with BF16 x are exact there), then one
// rounding of g * sum to binary32 and a fixed xor-shuffle order across lanes.
template <int FMT, int M>
__global__ void __launch_bounds__(256) gemv_any_kernel(const uint8_t *__restrict__ codes,
                                                       const uint8_t *__restrict__ scales,
                                                       const float *__restrict__ gscale,
                                                       const uint16_t *__restrict__ x, float *__restrict__ y, int K,
                                                       int N) {
    constexpr bool NV = FMT == W4_FMT_NVFP4;
    constexpr int BB = FMT == W4_FMT_ROCMFP4_DUAL ? 18 : 17;
    const int lane = threadIdx.x & 31;
    const long long n = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    pdl_wait_prior_grid();
    if (n >= N) return;
    double acc[M];
#pragma unroll
    for (int m = 0; m < M; m++) acc[m] = 0.0;
    const int ngr = K / (NV ? 16 : 32);
    for (int q = lane; q < ngr; q += 32) {
        if constexpr (NV) {
            const uint8_t *c = codes + (size_t)n * (K / 2) + (size_t)q * 8;
            const double s = (double)e4m3_to_f32(scales[(size_t)n * (K / 16) + q]);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const uint32_t h = e2m1x2_to_f16x2(c[i]);
                const float2 w = __half22float2(*reinterpret_cast<const __half2 *>(&h));
#pragma unroll
                for (int m = 0; m < M; m++) {
                    const uint16_t *xr = x + (size_t)m * K + (size_t)q * 16 + 2 * i;
                    acc[m] += s * ((double)w.x * (double)bf16_lo(xr[0]) + (double)w.y * (double)bf16_lo(xr[1]));
                }
            }
        } else {
            const uint8_t *blk = codes + (size_t)n * (K / 32) * BB + (size_t)q * BB;
            float s0, s1;
            float2 w[16];
            decode_rocm<FMT == W4_FMT_ROCMFP4_DUAL>(blk, w, s0, s1);
#pragma unroll
            for (int m = 0; m < M; m++) {
                const uint16_t *xr = x + (size_t)m * K + (size_t)q * 32;
                double a0 = 0.0, a1 = 0.0;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    a0 += (double)w[j].x * (double)bf16_lo(xr[j]);
                    a1 += (double)w[j].y * (double)bf16_lo(xr[j + 16]);
                }
                acc[m] += (double)s0 * a0 + (double)s1 * a1;
            }
        }
    }
    const double g = NV ? (double)__ldg(gscale) : 1.0;
#pragma unroll
    for (int m = 0; m < M; m++) {
        double v = acc[m];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) y[(size_t)m * N + n] = (float)(g * v);
    }
}

// y[m][n] = g * sum_s partial[s][m][n], slices in order.
__global__ void gemv_finalize_kernel(const float *__restrict__ partial, int S, int MN,
                                     const float *__restrict__ gscale, float *__restrict__ y) {
    pdl_allow_dependents();
    pdl_wait_prior_grid();   // the slices' partials (a no-op without programmatic dependent launch)
    const float g = gscale ? __ldg(gscale) : 1.0f;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < MN; i += gridDim.x * blockDim.x) {
        float s = 0.0f;
        for (int q = 0; q < S; q++) s += partial[(size_t)q * MN + i];
        y[i] = g * s;
    }
}

}  // namespace w4
