// pack.cuh -- NVFP4 and ROCmFP4 packers (sm_100a, CUDA cores).
//
// NVFP4 ("EdgeRock-4B-NVFP4" card, intro; round-to-nearest recipe of the
// "Nanbeige4.2-3B-NVFP4A16" card, Creation):
//   global g = absmax / (6 * 448); block scale s = E4M3(absmax_block / 6 / g);
//   code = E2M1(x / (s * g)).  Two launches: an abs-max reduction into the
//   workspace, then one thread per 16-element block.
// ROCmFP4 ("rocmwhy" page, sections 01-03): for each scale group every finite
//   UE4M3 code is scored by its binary32 reconstruction error with nearest
//   Codebook10 levels; one warp per 32-weight block, lanes split the 127
//   candidates, a lexicographic (error, code) shuffle reduction picks the
//   winner (ties to the smaller code).
// Importance weighting (the same page, section 03: "optional importance
//   weighting"): one weight w_k >= 0 per input channel, E = sum fma(w_k d, d, E).
// NVFP4 block scale by search: the same warp-per-block search over the finite
//   E4M3 codes with the global scale fixed by the abs-max rule; under each
//   candidate the codes are the abs-max packer's E2M1(x / (scale * g)).
#pragma once

#include "common.cuh"

namespace w4 {

// ---------------------------------------------------------------- NVFP4 ----

// ws[0]: max over |W| as bf16 magnitude bits (monotone in the value for finite
// inputs); ws[1]: non-zero if any element is NaN or Inf.
__global__ void __launch_bounds__(256) nvfp4_absmax_kernel(const uint4 *__restrict__ W, long long n8,
                                                           unsigned *__restrict__ ws) {
    unsigned m = 0, bad = 0;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8;
         i += (long long)gridDim.x * blockDim.x) {
        uint4 v = __ldg(W + i);
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            unsigned lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
            bad |= (lo >= 0x7F80u) | (hi >= 0x7F80u);
            m = max(m, max(lo, hi));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        bad |= __shfl_xor_sync(0xFFFFFFFFu, bad, o);
    }
    __shared__ unsigned sm[8], sb[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        sm[warp] = m;
        sb[warp] = bad;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < (int)(blockDim.x >> 5); i++) {
            m = max(m, sm[i]);
            bad |= sb[i];
        }
        if (m) atomicMax(ws, m);
        if (bad) atomicOr(ws + 1, 1u);
    }
}

// One thread per 16-element block; block b covers W[16b .. 16b+15] (rows are
// K-contiguous and K % 16 == 0, so blocks never straddle rows).
__global__ void __launch_bounds__(256) nvfp4_encode_kernel(const uint4 *__restrict__ W, long long nblocks,
                                                           const unsigned *__restrict__ ws,
                                                           uint2 *__restrict__ codes,
                                                           uint8_t *__restrict__ scales,
                                                           float *__restrict__ global_scale,
                                                           int *__restrict__ d_status) {
    const float amax = __uint_as_float(ws[0] << 16);
    const float g = __fdiv_rn(amax, 2688.0f);  // absmax / (6 * 448)
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *global_scale = g;
        if (ws[1]) {
            if (d_status) *d_status = W4_ERR_NONFINITE;
            record_error(W4_ERR_NONFINITE);
        }
    }
    for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < nblocks;
         b += (long long)gridDim.x * blockDim.x) {
        const uint4 v0 = __ldg(W + 2 * b), v1 = __ldg(W + 2 * b + 1);
        const unsigned w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float x[16];
        float bamax = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            x[2 * j] = bf16_lo(w[j]);
            x[2 * j + 1] = bf16_hi(w[j]);
            bamax = fmaxf(bamax, fmaxf(fabsf(x[2 * j]), fabsf(x[2 * j + 1])));
        }
        uint32_t s = 0;
        if (g != 0.0f) s = f32_to_e4m3(__fdiv_rn(__fdiv_rn(bamax, 6.0f), g));
        const float d = __fmul_rn(e4m3_to_f32(s), g);
        uint32_t c[2] = {0u, 0u};
        if (d != 0.0f) {
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint32_t byte = f32x2_to_e2m1x2(__fdiv_rn(x[2 * j], d), __fdiv_rn(x[2 * j + 1], d));
                c[j >> 2] |= byte << (8 * (j & 3));
            }
        }
        codes[b] = make_uint2(c[0], c[1]);
        scales[b] = (uint8_t)s;
    }
}

// -------------------------------------------------------------- ROCmFP4 ----

// Binary32 reconstruction error of n weights (xs, in k order) at scale s with
// nearest Codebook10 levels.  Level = nearest of s*{0,1,2,3,4,6,8,10}; the
// midpoints s*{.5,1.5,2.5,3.5,5,7,9} are exact in binary32, and a tie goes to
// the even level index, i.e. ">=" at the midpoints that lead to an even index
// (1.5, 3.5, 7) and ">" at the others.
template <int n, bool WT = false>
__device__ __forceinline__ float rocm_error(const float (&xs)[n], float s, const float (&wv)[n]) {
    const float t0 = s * 0.5f, t1 = s * 1.5f, t2 = s * 2.5f, t3 = s * 3.5f;
    const float t4 = s * 5.0f, t5 = s * 7.0f, t6 = s * 9.0f;
    float E = 0.0f;
#pragma unroll
    for (int i = 0; i < n; i++) {
        const float a = fabsf(xs[i]);
        float L = (a > t0 ? 1.0f : 0.0f) + (a >= t1 ? 1.0f : 0.0f) + (a > t2 ? 1.0f : 0.0f) +
                  (a >= t3 ? 1.0f : 0.0f);
        L += 2.0f * ((a > t4 ? 1.0f : 0.0f) + (a >= t5 ? 1.0f : 0.0f) + (a > t6 ? 1.0f : 0.0f));
        const float d = __fsub_rn(a, __fmul_rn(s, L));
        E = __fmaf_rn(WT ? __fmul_rn(wv[i], d) : d, d, E);
    }
    return E;
}

// Codebook10 code (bit 3 sign, bits 2..0 level index) of x at scale s.
__device__ __forceinline__ uint32_t rocm_code(float x, float s) {
    if (s == 0.0f) return 0u;
    const float a = fabsf(x);
    const uint32_t idx = (a > s * 0.5f) + (a >= s * 1.5f) + (a > s * 2.5f) + (a >= s * 3.5f) +
                         (a > s * 5.0f) + (a >= s * 7.0f) + (a > s * 9.0f);
    if (idx == 0) return 0u;
    return idx | ((__float_as_uint(x) >> 28) & 8u);
}

// Lexicographic (error, code) minimum across `width` lanes (xor shuffles).
__device__ __forceinline__ void argmin_lanes(float &E, uint32_t &u, int width) {
    for (int o = width >> 1; o; o >>= 1) {
        const float Eo = __shfl_xor_sync(0xFFFFFFFFu, E, o);
        const uint32_t uo = __shfl_xor_sync(0xFFFFFFFFu, u, o);
        if (Eo < E || (Eo == E && uo < u)) {
            E = Eo;
            u = uo;
        }
    }
}

// DUAL: lanes 0..15 search the scale of elements 0..15 (8 candidates each),
// lanes 16..31 the scale of 16..31.  FAST: all 32 lanes search one scale (4
// candidates each).  Lane l ends holding the winning scale of element l.
template <bool DUAL, bool WT>
__global__ void __launch_bounds__(256) rocm_pack_kernel(const uint16_t *__restrict__ W, long long nblk, int K,
                                                        const float *__restrict__ imp,
                                                        uint8_t *__restrict__ out,
                                                        int *__restrict__ d_status) {
    constexpr int BB = DUAL ? 18 : 17;
    constexpr int NG = DUAL ? 16 : 32;  // weights per scale group
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long blk = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; blk < nblk; blk += warps) {
        const uint32_t bits = __ldg(W + blk * 32 + lane);
        const float xl = __uint_as_float(bits << 16);
        if ((bits & 0x7F80u) == 0x7F80u) {
            if (d_status) atomicExch(d_status, W4_ERR_NONFINITE);
            record_error(W4_ERR_NONFINITE);
        }
        float wl = 1.0f;   // this lane's channel weight
        if (WT) {
            wl = __ldg(imp + (blk % (K / 32)) * 32 + lane);
            if (!(wl >= 0.0f && wl <= 3.402823466e38f)) {
                if (d_status) atomicExch(d_status, W4_ERR_NONFINITE);
                record_error(W4_ERR_NONFINITE);
            }
        }
        const int base = DUAL ? (lane & 16) : 0;
        float xs[NG], wv[NG];
#pragma unroll
        for (int i = 0; i < NG; i++) {
            xs[i] = __shfl_sync(0xFFFFFFFFu, xl, base + i);
            wv[i] = WT ? __shfl_sync(0xFFFFFFFFu, wl, base + i) : 1.0f;
        }

        float bestE = 0.0f;
        uint32_t bestU = 0xFFu;
        const int sub = DUAL ? (lane & 15) : lane;
#pragma unroll 1
        for (int t = 0; t < (DUAL ? 8 : 4); t++) {
            const uint32_t u = (uint32_t)(sub + t * NG);
            if (u > 0x7Eu) break;
            const float E = rocm_error<NG, WT>(xs, e4m3_to_f32(u), wv);
            if (bestU == 0xFFu || E < bestE) {
                bestE = E;
                bestU = u;
            }
        }
        argmin_lanes(bestE, bestU, NG);

        const uint32_t code = rocm_code(xl, e4m3_to_f32(bestU));
        const uint32_t hi = __shfl_down_sync(0xFFFFFFFFu, code, 16);
        uint8_t *o = out + blk * BB;
        if (DUAL) {
            const uint32_t u1 = __shfl_sync(0xFFFFFFFFu, bestU, 16);
            if (lane == 0) {
                o[0] = (uint8_t)bestU;
                o[1] = (uint8_t)u1;
            }
        } else if (lane == 0) {
            o[0] = (uint8_t)bestU;
        }
        if (lane < 16) o[(DUAL ? 2 : 1) + lane] = (uint8_t)(code | (hi << 4));
    }
}

// NVFP4 block scale by search.  One warp per 16-element block: lane l scores
// the E4M3 codes l, l+32, l+64, l+96 (up to 0x7E): d = E4M3(u) * g, each code
// E2M1(x / d), r = e2m1 * d, E = sum over k in order of fma(w * (x - r), x - r, E)
// (w = 1 without weights) in binary32; the lexicographic (E, u) minimum wins.
// Lane 0 then encodes the block under the winner, as nvfp4_encode_kernel does.
template <bool WT>
__global__ void __launch_bounds__(256) nvfp4_search_kernel(const uint16_t *__restrict__ W, long long nblocks, int K,
                                                           const unsigned *__restrict__ ws,
                                                           const float *__restrict__ imp,
                                                           uint2 *__restrict__ codes, uint8_t *__restrict__ scales,
                                                           float *__restrict__ global_scale,
                                                           int *__restrict__ d_status) {
    const float amax = __uint_as_float(ws[0] << 16);
    const float g = __fdiv_rn(amax, 2688.0f);  // absmax / (6 * 448)
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *global_scale = g;
        if (ws[1]) {
            if (d_status) *d_status = W4_ERR_NONFINITE;
            record_error(W4_ERR_NONFINITE);
        }
    }
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const int kb = K / 16;
    for (long long blk = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; blk < nblocks; blk += warps) {
        const float xe = __uint_as_float((uint32_t)__ldg(W + blk * 16 + (lane & 15)) << 16);
        float we = 1.0f;
        if (WT) {
            we = __ldg(imp + (blk % kb) * 16 + (lane & 15));
            if (lane < 16 && !(we >= 0.0f && we <= 3.402823466e38f)) {
                if (d_status) atomicExch(d_status, W4_ERR_NONFINITE);
                record_error(W4_ERR_NONFINITE);
            }
        }
        float xs[16], wv[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            xs[i] = __shfl_sync(0xFFFFFFFFu, xe, i);
            wv[i] = WT ? __shfl_sync(0xFFFFFFFFu, we, i) : 1.0f;
        }
        float bestE = 0.0f;
        uint32_t bestU = 0xFFu;
#pragma unroll 1
        for (int t = 0; t < 4; t++) {
            const uint32_t u = (uint32_t)(lane + 32 * t);
            if (u > 0x7Eu) break;
            const float d = __fmul_rn(e4m3_to_f32(u), g);
            float E = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                float2 r = make_float2(0.0f, 0.0f);
                if (d != 0.0f) {
                    const uint32_t byte = f32x2_to_e2m1x2(__fdiv_rn(xs[2 * j], d), __fdiv_rn(xs[2 * j + 1], d));
                    const uint32_t h = e2m1x2_to_f16x2(byte);
                    const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&h));
                    r = make_float2(__fmul_rn(v.x, d), __fmul_rn(v.y, d));
                }
                const float e0 = __fsub_rn(xs[2 * j], r.x), e1 = __fsub_rn(xs[2 * j + 1], r.y);
                E = __fmaf_rn(WT ? __fmul_rn(wv[2 * j], e0) : e0, e0, E);
                E = __fmaf_rn(WT ? __fmul_rn(wv[2 * j + 1], e1) : e1, e1, E);
            }
            if (bestU == 0xFFu || E < bestE) {
                bestE = E;
                bestU = u;
            }
        }
        argmin_lanes(bestE, bestU, 32);
        if (lane == 0) {
            const float d = __fmul_rn(e4m3_to_f32(bestU), g);
            uint32_t c[2] = {0u, 0u};
            if (d != 0.0f) {
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const uint32_t byte = f32x2_to_e2m1x2(__fdiv_rn(xs[2 * j], d), __fdiv_rn(xs[2 * j + 1], d));
                    c[j >> 2] |= byte << (8 * (j & 3));
                }
            }
            codes[blk] = make_uint2(c[0], c[1]);
            scales[blk] = (uint8_t)bestU;
        }
    }
}

// ---------------------------------------------------------------- Q4_0 ----
// Stock Q4_0, the pages' comparison format ("rocmwhy" format table and section
// 02): one thread per 32-weight block; m = the first weight of largest
// magnitude, d = FP16(m / -8) saturating at 65504, code = clamp(RNE(x / d),
// -8, 7) + 8 in binary32, d == 0 -> codes 8.  Block = [d lo, d hi, 16 code
// bytes], code byte j = code[j] | code[j+16] << 4.
__global__ void __launch_bounds__(256) q4_0_pack_kernel(const uint4 *__restrict__ W, long long nblk,
                                                        uint8_t *__restrict__ out, int *__restrict__ d_status) {
    for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < nblk;
         b += (long long)gridDim.x * blockDim.x) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const uint4 v = __ldg(W + 4 * b + i);
            w[4 * i] = v.x, w[4 * i + 1] = v.y, w[4 * i + 2] = v.z, w[4 * i + 3] = v.w;
        }
        float x[32];
        int jm = 0;
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 32; j++) {
            x[j] = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
            bad |= !isfinite(x[j]);
        }
        if (bad) {
            if (d_status) atomicExch(d_status, W4_ERR_NONFINITE);
            record_error(W4_ERR_NONFINITE);
        }
        float am = fabsf(x[0]);
#pragma unroll
        for (int j = 1; j < 32; j++)
            if (fabsf(x[j]) > am) {
                am = fabsf(x[j]);
                jm = j;
            }
        const float dq = fminf(fmaxf(__fdiv_rn(x[jm], -8.0f), -65504.0f), 65504.0f);
        const __half h = __float2half_rn(dq);
        const float d = __half2float(h);
        uint32_t code[32];
#pragma unroll
        for (int j = 0; j < 32; j++) {
            float q = 0.0f;
            if (d != 0.0f) q = fminf(fmaxf(rintf(__fdiv_rn(x[j], d)), -8.0f), 7.0f);
            code[j] = (uint32_t)((int)q + 8);
        }
        uint8_t *o = out + b * 18;
        const uint16_t hb = __half_as_ushort(h);
        o[0] = (uint8_t)(hb & 0xFF);
        o[1] = (uint8_t)(hb >> 8);
#pragma unroll
        for (int j = 0; j < 16; j++) o[2 + j] = (uint8_t)(code[j] | (code[j + 16] << 4));
    }
}

// ------------------------------------------------------ reconstruction error ----
// Sum over a packed matrix of (W - w_hat)^2 and W^2 in binary64: one 32-weight
// block per thread step, a fixed-order block reduction to one partial per
// CTA, then one thread adds the partials in order.
constexpr int kReconMaxGrid = 1024;

__device__ __forceinline__ double e2m1_value(uint32_t c) {
    const double m[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    return (c & 8u) ? -m[c & 7u] : m[c & 7u];
}
__device__ __forceinline__ double cb10_value(uint32_t c) {
    const double m[8] = {0.0, 1.0, 2.0, 3.0, 4.0, 6.0, 8.0, 10.0};
    return (c & 8u) ? -m[c & 7u] : m[c & 7u];
}

__global__ void __launch_bounds__(256) recon_partial_kernel(int fmt, int K, long long nblk,
                                                            const uint8_t *__restrict__ codes,
                                                            const uint8_t *__restrict__ scales,
                                                            const float *__restrict__ gscale,
                                                            const uint16_t *__restrict__ W,
                                                            double2 *__restrict__ partial) {
    const int nb = K / 32;
    const double g = fmt == W4_FMT_NVFP4 ? (double)__ldg(gscale) : 1.0;
    double se = 0.0, sq = 0.0;
    for (long long blk = blockIdx.x * (long long)blockDim.x + threadIdx.x; blk < nblk;
         blk += (long long)gridDim.x * blockDim.x) {
        const long long n = blk / nb;
        const int b = (int)(blk % nb);
        for (int j = 0; j < 32; j++) {
            const long long k = 32LL * b + j;
            const double x = (double)__uint_as_float((uint32_t)__ldg(W + n * K + k) << 16);
            double wh;
            if (fmt == W4_FMT_NVFP4) {
                const uint32_t byte = __ldg(codes + n * (K / 2) + k / 2);
                const uint32_t c = (k & 1) ? (byte >> 4) : (byte & 15u);
                wh = e2m1_value(c) * (double)e4m3_to_f32(__ldg(scales + n * (K / 16) + k / 16)) * g;
            } else {
                const int bb = fmt == W4_FMT_ROCMFP4_FAST ? 17 : 18;
                const uint8_t *p = codes + blk * bb;
                const int c0 = fmt == W4_FMT_ROCMFP4_FAST ? 1 : 2;
                const uint32_t byte = __ldg(p + c0 + (j & 15));
                const uint32_t c = j < 16 ? (byte & 15u) : (byte >> 4);
                if (fmt == W4_FMT_Q4_0) {
                    const uint16_t hb = (uint16_t)(__ldg(p) | (__ldg(p + 1) << 8));
                    wh = (double)__half2float(__ushort_as_half(hb)) * (double)((int)c - 8);
                } else {
                    const uint32_t sb = (fmt == W4_FMT_ROCMFP4_DUAL && j >= 16) ? __ldg(p + 1) : __ldg(p);
                    wh = cb10_value(c) * (double)e4m3_to_f32(sb);
                }
            }
            const double e = x - wh;
            se += e * e;
            sq += x * x;
        }
    }
    __shared__ double2 red[256];
    red[threadIdx.x] = make_double2(se, sq);
    __syncthreads();
    for (int o = 128; o; o >>= 1) {
        if ((int)threadIdx.x < o) {
            red[threadIdx.x].x += red[threadIdx.x + o].x;
            red[threadIdx.x].y += red[threadIdx.x + o].y;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

__global__ void recon_final_kernel(const double2 *__restrict__ partial, int n, double *__restrict__ out) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        double se = 0.0, sq = 0.0;
        for (int i = 0; i < n; i++) {
            se += partial[i].x;
            sq += partial[i].y;
        }
        out[0] = se;
        out[1] = sq;
    }
}

// Elementwise conversion check kernel (the packers' encoders on raw floats).
__global__ void encode_scalars_kernel(const float *__restrict__ v, long long n, uint8_t *__restrict__ e4,
                                      uint8_t *__restrict__ e2) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const float x = v[i];
        if (e4) e4[i] = (uint8_t)f32_to_e4m3(x);
        if (e2) e2[i] = (uint8_t)(f32x2_to_e2m1x2(x, 0.0f) & 0xFu);
    }
}

}  // namespace w4
