// gemm.cuh -- prefill W4A16 GEMM on the 5th-generation tensor cores (sm_100a).
//
// y[m][n] = g * sum_k x[m][k] * (e2m1[n][k] * scale[n][k/16])   (NVFP4 weights,
// "EdgeRock-4B-NVFP4" card, intro; BF16 activations).  e2m1 * scale has at most
// 6 significant bits and lies in [2^-10, 2688], so it is exact in BF16: the
// weights are dequantised once per tile into shared memory and multiplied with
// tcgen05.mma kind::f16 (BF16 x BF16 -> FP32 in tensor memory).  The global
// scale g is applied in the epilogue.
//
// Tile: 128 weight rows (MMA M, operand A = dequantised W) x 256 tokens (MMA N,
// operand B = x) x 64 k per stage; both operands K-major with the 128-byte
// swizzle.  Persistent CTAs, one per SM, walk the tiles n-major so that CTAs
// running together share the same packed weight rows in L2.
//
// Warp roles (14 warps):
//   warp 0      TMA producer of x tiles (cp.async.bulk.tensor, no multicast);
//               allocates / frees the 512 TMEM columns.
//   warp 1      MMA issuer (one thread): 4 x (128x256x16) per stage, commits to
//               the stage barriers, and to the accumulator barrier per tile.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31), times g, float32 / BF16 stores.
//   warps 6-13  dequantise: thread (row r, half h) turns 32 codes + 2 scales of
//               row r into BF16 in the swizzled A stage.
// Two accumulators of 256 columns let the epilogue of a tile overlap the MMAs
// of the next.  Every mbarrier wait is bounded (common.cuh: mbar_wait).
#pragma once

#include "common.cuh"

namespace w4 {

namespace gemm {

constexpr int BM = 128;      // weight rows per tile (MMA M)
constexpr int BN = 256;      // tokens per tile (MMA N)
constexpr int BK = 64;       // k per stage (one 128-byte swizzle row of BF16)
constexpr int STAGES = 4;
constexpr int kWarps = 14;
constexpr int kThreads = kWarps * 32;
constexpr int kDequantThreads = 256;
constexpr int kEpiThreads = 128;
constexpr uint32_t X_STAGE_BYTES = BN * BK * 2;   // 32 KB
constexpr uint32_t A_STAGE_BYTES = BM * BK * 2;   // 16 KB
constexpr uint32_t TMEM_COLS = 512;               // two 256-column fp32 accumulators
constexpr int WK = 256;                           // k per packed-weight stage (4 k-steps)
constexpr int WSTAGES = 2;
constexpr uint32_t W_STAGE_BYTES = BM * WK / 2;   // 16 KB of codes (128 rows x 128 bytes)

// Instruction descriptor, kind::f16: D = F32 (bit 4), A = BF16 (bits 7-9),
// B = BF16 (bits 10-12), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

struct SharedStorage {
    uint8_t x[STAGES][X_STAGE_BYTES];   // 1024-byte aligned (swizzle atoms)
    uint8_t a[STAGES][A_STAGE_BYTES];
    uint8_t w[WSTAGES][W_STAGE_BYTES];  // packed codes, 128-byte swizzle
    uint64_t w_full[WSTAGES], w_empty[WSTAGES];
    uint64_t x_full[STAGES], x_empty[STAGES];
    uint64_t a_full[STAGES], a_empty[STAGES];
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort;
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

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate));
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

struct Params {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *gscale;
    float *y32;
    __nv_bfloat16 *y16;
    int M, N, K;
    int tiles_m, tiles_n;
};

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap xmap,
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
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&sh.tmem_base)), "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

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
                    tma_load_2d(sh.x[s], &xmap, kt * BK, m0, &sh.x_full[s]);
                }
                if (*abort) break;
            }
        }
        __syncwarp();   // the whole warp reaches the final barrier together (it is .aligned)
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -------------------------------
        if (lane == 0) {
            int it = 0, lt = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, lt++) {
                const int b = lt & 1;
                if (lt >= 2) mbar_wait(&sh.acc_empty[b], ((lt >> 1) - 1) & 1, abort);
                tc_fence_after();
                const uint32_t dtm = tmem + (uint32_t)(b * BN);
                for (int kt = 0; kt < KT; kt++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    mbar_wait(&sh.x_full[s], ph, abort);
                    mbar_wait(&sh.a_full[s], ph, abort);
                    if (*abort) break;
                    tc_fence_after();
                    const uint32_t ab = smem_addr(sh.a[s]), xb = smem_addr(sh.x[s]);
#pragma unroll
                    for (int j = 0; j < BK / 16; j++)
                        mma_bf16(dtm, sw128_desc(ab + 32 * j), sw128_desc(xb + 32 * j), (kt | j) ? 1u : 0u);
                    mma_commit(&sh.x_empty[s]);
                    mma_commit(&sh.a_empty[s]);
                }
                mma_commit(&sh.acc_full[b]);
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const float g = __ldg(p.gscale);
        int lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, lt++) {
            const int b = lt & 1;
            const int m0 = (t % p.tiles_m) * BN, n0 = (t / p.tiles_m) * BM;
            mbar_wait(&sh.acc_full[b], (lt >> 1) & 1, abort);
            tc_fence_after();
            const int n = n0 + q * 32 + lane;
            for (int c = 0; c < BN / 32; c++) {
                uint32_t v[32];
                W4_TMEM_LD32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN + c * 32), v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (n < p.N) {
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int m = m0 + c * 32 + j;
                        if (m < p.M) {
                            const float val = g * __uint_as_float(v[j]);
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
        const int dt = threadIdx.x - 6 * 32;    // 0..255
        const int r = dt & (BM - 1), h = dt >> 7;
        constexpr int KQ = WK / BK;             // k-steps per codes stage
        int it = 0, wit = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int n = (t / p.tiles_m) * BM + r;
            const bool valid = n < p.N;
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
#pragma unroll
                for (int q = 0; q < KQ; q++) {
                    if (kw + q < KT) {
                        const int s = it % STAGES;
                        if (it >= STAGES) mbar_wait(&sh.a_empty[s], ((it / STAGES) - 1) & 1, abort);
                        const uint4 cw = *reinterpret_cast<const uint4 *>(wrow + (((q * 2 + h) ^ (r & 7)) * 16));
                        const uint32_t sw = sc[q] >> (16 * h);
                        const float s0 = e4m3_to_f32(sw & 0xFFu), s1 = e4m3_to_f32((sw >> 8) & 0xFFu);
                        uint8_t *arow = sh.a[s] + r * 128;
                        const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                        for (int cc = 0; cc < 4; cc++) {
                            const uint4 o = valid ? dequant8(cws[cc], cc < 2 ? s0 : s1) : make_uint4(0, 0, 0, 0);
                            const int chunk = (h * 4 + cc) ^ (r & 7);
                            *reinterpret_cast<uint4 *>(arow + chunk * 16) = o;
                        }
                        // each thread makes its stores visible to the tensor core's
                        // (async) proxy; the warp then arrives once
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sh.a_full[s]);
                        it++;
                    }
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

inline size_t gemm_workspace_bytes(const w4_weights *, int) { return 0; }

inline size_t gemm_smem_bytes() { return sizeof(gemm::SharedStorage) + 1024; }

inline w4_status gemm_launch(const w4_weights *w, const void *x, int M, float *y32, void *y16, void *, size_t,
                             cudaStream_t st) {
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
    static bool configured = false;
    const size_t smem = gemm_smem_bytes();
    if (!configured) {
        if (cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return W4_ERR_CUDA;
        configured = true;
    }
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
    const int ntiles = p.tiles_m * p.tiles_n;
    gemm_kernel<<<std::min(ntiles, sms), kThreads, smem, st>>>(map, cmap, p);
    return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

}  // namespace w4
