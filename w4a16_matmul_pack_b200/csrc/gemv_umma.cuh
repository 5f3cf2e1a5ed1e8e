// gemv_umma.cuh -- NVFP4 decode GEMV for one token (M = 1) on the 5th-generation
// tensor cores: weights decoded by the CUDA cores into tensor memory, the
// products issued by one thread with tcgen05.mma (A from TMEM, B from shared
// memory, f32 accumulators in TMEM).
//
// y[n] = g * sum_k x[k] * e2m1[n][k] * scale[n][k/16]   ("EdgeRock-4B-NVFP4"
// card, intro; the fused W4A16 decode kernel of the "Nanbeige4.2-3B-NVFP4A16"
// card, Serving).  e2m1 * E4M3 scale has at most 6 significant bits and lies in
// [2^-10, 2688]: exact in f16, so A = that product in f16.  x is converted to
// f16 as x * 2^-sigma (sigma from the largest |x|), exact whenever every
// nonzero |x * 2^-sigma| >= 2^-17; otherwise the CTA computes in binary32 on the
// CUDA cores from the same staged tiles.
//
// Layout of one MMA (M = 128, N = 32, K = 16).  A tile is 4 weight rows.  TMEM
// lane 32r + j holds row r, "phase" j: the 16-k blocks j, j + 32, j + 64, ...
// of that row, one block per MMA step (8 TMEM columns of f16 pairs).  B row n of
// step s is x block 32s + n.  The MMA therefore forms D[32r + j][n] = sum over
// steps of (row r, block 32s + j) . (x block 32s + n); the diagonal n = j is the
// row's partial sum over its phase-j blocks, and a warp-shuffle sum over the 32
// lanes of row r gives y.  The off-diagonal columns are discarded: the tensor
// core has far more throughput than the decode needs.  With this layout a warp's
// 32 lanes read 256 contiguous code bytes per step (one 8-byte load each) and
// 32 contiguous scale bytes.
//
// Roles (15 warps):
//   warps 0-7   decode: the CTA's tiles form one sequence of MMA steps, grouped
//               four to an A slot; warp w writes row w%4, steps {2h, 2h+1}
//               (h = w/4) of each slot: LDS.64 codes -> cvt e2m1x2 -> HMUL2 by
//               the block scale -> tcgen05.st, software-pipelined so that the
//               next slot is decoded while the previous store completes.  They
//               also convert x, once the A ring is full (so decoding of the
//               prefetched weights overlaps the wait for x).
//   warp 8      allocates TMEM; lane 0 issues the MMAs and commits.  It never
//               waits on an mbarrier (a thread with MMAs queued stalls on any
//               shared-memory access until they drain): warp 14 waits and
//               releases it through a named barrier once per A slot.
//   warp 9      lane 0: TMA producer (x after the dependency wait, weight
//               stages of TB tiles, prefetched before the wait under PDL).
//   warps 10-13 epilogue: row w%4 of each tile (tcgen05.ld of D, diagonal,
//               shuffle sum, store); the binary32 path when x is not exact.
// TMEM (256 columns, so that two CTAs can be resident under programmatic
// launch): six 32-column A slots and two 32-column accumulators.
#pragma once

#include "gemv_m1.cuh"

namespace w4 {
namespace um {

constexpr int kPhases = 32;            // TMEM lanes per row = MMA N
constexpr int kTileRows = 4;           // 128 lanes / 32 phases
constexpr int kStepK = 16 * kPhases;   // k per MMA step (512)
constexpr int kDecWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kProdWarp = 9;
constexpr int kEpiWarp0 = 10;
constexpr int kWaitWarp = 14;   // waits on mbarriers for the MMA issuer
constexpr int kThreads = 15 * 32;
constexpr int kSlots = 6;              // A ring slots of 4 steps (32 columns)
constexpr int kSlotSteps = 4;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kDCol0 = kSlots * 32;   // accumulators at columns 192, 224
// kind::f16, D = F32, A = B = F16, both K-major, N = 32, M = 128
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kPhases >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

struct Args {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *gscale;
    const uint16_t *x;   // [K] bf16
    float *y;            // [N]
    int K, N;
    int TB;              // tiles per full stage
    int NS;              // stages
    int pdl;
};

// Shared-memory layout (bytes); host and device agree through this function.
struct Layout {
    size_t xnat, xb, stages, stage_bytes, codes_bytes, bars, flags, fb, total;
};

__host__ __device__ __forceinline__ Layout layout(int K, int TB, int NS) {
    Layout L;
    L.xnat = 0;
    L.xb = ((size_t)K * 2 + 127) & ~(size_t)127;
    L.stages = (L.xb + (size_t)K * 2 + 1023) & ~(size_t)1023;
    L.codes_bytes = (size_t)kTileRows * TB * (K / 2);
    L.stage_bytes = (L.codes_bytes + (size_t)kTileRows * TB * (K / 16) + 127) & ~(size_t)127;
    L.bars = L.stages + (size_t)NS * L.stage_bytes;
    // stage full/empty, slot full/empty, acc full/empty, xfull, xb ready
    L.flags = L.bars + (size_t)(2 * NS + 2 * kSlots + 4 + 2) * 8;
    L.fb = L.flags + 64;   // abort, binary32 path, TMEM base, sigma, per-warp max
    L.total = L.fb;
    return L;
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
          "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// MMA with A from tensor memory, B from a shared-memory descriptor.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// B operand of one step: 32 rows (x blocks) x 16 k, K-major without swizzle.
// The 8x8 core matrix of rows n..n+7 and k 8h..8h+7 sits at (n/8)*256 + h*128
// bytes, its row n%8 at +16*(n%8): leading byte offset 128 (the next 8 k),
// stride byte offset 256 (the next 8 rows).
__device__ __forceinline__ uint64_t b_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128 >> 4) << 16;
    d |= (uint64_t)(256 >> 4) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version
    return d;                 // layout type 0: no swizzle
}

// Byte offset of x element k in the B layout (step k/512, row (k/16)%32, k%16).
__device__ __forceinline__ uint32_t xb_offset(int k) {
    const int s = k >> 9, n = (k >> 4) & 31, kk = k & 15;
    return (uint32_t)(s * 1024 + (n >> 3) * 256 + (kk >> 3) * 128 + (n & 7) * 16 + (kk & 7) * 2);
}

// 8 code bytes (one 16-k block) times the block scale (f16x2 holding the scale
// twice) -> 8 f16x2, element 2i in the low half of h[i].  Exact.
__device__ __forceinline__ void decode_step(uint2 c, uint32_t s2, uint32_t *h) {
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 8; i++) h[i] = hmul2_u32(e2m1x2_to_f16x2(w[i >> 2] >> (8 * (i & 3))), s2);
}

// v[lane] of 32 per-thread registers (a select network).
__device__ __forceinline__ float pick_lane(uint32_t (&v)[32], int lane) {
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = (lane & 16) ? v[i + 16] : v[i];
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = (lane & 8) ? v[i + 8] : v[i];
#pragma unroll
    for (int i = 0; i < 4; i++) v[i] = (lane & 4) ? v[i + 4] : v[i];
#pragma unroll
    for (int i = 0; i < 2; i++) v[i] = (lane & 2) ? v[i + 2] : v[i];
    return __uint_as_float((lane & 1) ? v[1] : v[0]);
}

// A decode warp's position in its CTA's sequence of MMA steps, and the stage
// bookkeeping: the warp waits for every stage in order and releases each one
// after its last read (each warp arrives exactly once per stage).
struct DecodeCursor {
    int steps, TB, NS, total, h, q, lane, CSB, SSB;
    uint32_t stage_bytes, codes_bytes, st_sa;
    uint64_t *st_full, *st_empty;
    volatile int *abort;
    int cur;          // stage waited for and not yet released (-1: none)
    int s, i, ti;     // step within the tile, stage, tile within the stage of this warp's next step

    __device__ __forceinline__ void wrap() {
        while (s >= steps) {
            s -= steps;
            if (++ti == TB) ti = 0, i++;
        }
    }
    __device__ __forceinline__ void advance_to(int stage) {
        while (cur < stage) {
            if (cur >= 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(st_empty + cur % NS);
            }
            cur++;
            mbar_wait(st_full + cur % NS, (cur / NS) & 1, abort);
        }
    }
};

// Steps {4g + 2h, 4g + 2h + 1} of slot g (the cursor points at the first) -> out[16];
// moves the cursor to the next slot.  Returns how many of the two steps exist.
__device__ __forceinline__ int load_slot(DecodeCursor &c, int g, uint32_t *out) {
    const int G0 = g * kSlotSteps + 2 * c.h;
    const int cnt = max(0, min(2, c.total - G0));
    uint2 cw[2] = {make_uint2(0, 0), make_uint2(0, 0)};
    uint32_t b[2] = {0, 0};
    int s = c.s, i = c.i, ti = c.ti;
#pragma unroll
    for (int k = 0; k < 2; k++) {
        if (k < cnt) {
            c.advance_to(i);
            const uint32_t base = c.st_sa + (uint32_t)(i % c.NS) * c.stage_bytes;
            const int r = ti * kTileRows + c.q;
            cw[k] = lds64(base + (uint32_t)(r * c.CSB + s * 256 + 8 * c.lane));
            b[k] = lds8(base + c.codes_bytes + (uint32_t)(r * c.SSB + s * 32 + c.lane));
        }
        if (++s == c.steps) {
            s = 0;
            if (++ti == c.TB) ti = 0, i++;
        }
    }
    if (cnt > 0) {
        const uint32_t sc = e4m3x2_to_f16x2(b[0] | (b[1] << 8));
        decode_step(cw[0], __byte_perm(sc, 0, 0x1010), out);
        decode_step(cw[1], __byte_perm(sc, 0, 0x3232), out + 8);
    }
    c.s += kSlotSteps;
    c.wrap();
    return cnt;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemv_umma_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap smap,
                     const __grid_constant__ CUtensorMap cmap1, const __grid_constant__ CUtensorMap smap1,
                     const Args a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int K = a.K, N = a.N, TB = a.TB, NS = a.NS;
    const Layout L = layout(K, TB, NS);
    uint16_t *xnat = reinterpret_cast<uint16_t *>(smem + L.xnat);
    uint8_t *xb = smem + L.xb;
    uint8_t *stages = smem + L.stages;
    uint64_t *st_full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *st_empty = st_full + NS;
    uint64_t *a_full = st_empty + NS;
    uint64_t *a_empty = a_full + kSlots;
    uint64_t *d_full = a_empty + kSlots;
    uint64_t *d_empty = d_full + 2;
    uint64_t *xfull = d_empty + 2;
    uint64_t *xready = xfull + 1;
    // [0] abort [1] binary32 path [2] TMEM base [3] sigma [4..11] per-warp max
    int *flags = reinterpret_cast<int *>(smem + L.flags);
    volatile int *abort = flags;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = (N + kTileRows - 1) / kTileRows;
    const int t0 = (int)((long long)blockIdx.x * T / gridDim.x);
    const int t1 = (int)((long long)(blockIdx.x + 1) * T / gridDim.x);
    const int ntiles = t1 - t0;
    const int nstages = (ntiles + TB - 1) / TB;
    const int steps = K / kStepK;                          // MMA steps per tile
    const int total = ntiles * steps;                      // MMA steps of the CTA
    const int nslots = (total + kSlotSteps - 1) / kSlotSteps;
    const int CSB = K / 2, SSB = K / 16;                   // row bytes of codes / scales

    if (threadIdx.x == 0) {
        flags[0] = 0;
        flags[1] = 0;
        flags[3] = 0;
        for (int i = 0; i < NS; i++) {
            mbar_init(st_full + i, 1);
            mbar_init(st_empty + i, kDecWarps);
        }
        for (int i = 0; i < kSlots; i++) {
            mbar_init(a_full + i, kDecWarps);
            mbar_init(a_empty + i, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(d_full + i, 1);
            mbar_init(d_empty + i, 4);
        }
        mbar_init(xfull, 1);
        mbar_init(xready, kDecWarps);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(flags + 2)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    pdl_allow_dependents();
    const uint32_t tmem = (uint32_t)flags[2];

    if (warp == kProdWarp) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            const int before = a.pdl ? min(NS, nstages) : 0;
            for (int t = 0; t < nstages + 1; t++) {
                if (t == before) {
                    pdl_wait_prior_grid();
                    mbar_arrive_expect_tx(xfull, (uint32_t)(K * 2));
                    bulk_g2s(xnat, a.x, (uint32_t)(K * 2), xfull, pol);
                    continue;
                }
                const int i = t > before ? t - 1 : t;   // stage index
                const int st = i % NS;
                if (i >= NS && !mbar_wait(st_empty + st, ((i / NS) - 1) & 1, abort)) break;
                const int ta = t0 + i * TB, nt = min(TB, t1 - ta);
                uint8_t *dc = stages + (size_t)st * L.stage_bytes;
                uint8_t *ds = dc + L.codes_bytes;
                if (nt == TB) {
                    mbar_arrive_expect_tx(st_full + st, (uint32_t)(kTileRows * TB * (CSB + SSB)));
                    tma_load_3d(dc, &cmap, 0, 0, ta * kTileRows, st_full + st);
                    tma_load_3d(ds, &smap, 0, 0, ta * kTileRows, st_full + st);
                } else {
                    mbar_arrive_expect_tx(st_full + st, (uint32_t)(kTileRows * nt * (CSB + SSB)));
                    for (int q = 0; q < nt; q++) {
                        tma_load_3d(dc + (size_t)q * kTileRows * CSB, &cmap1, 0, 0, (ta + q) * kTileRows, st_full + st);
                        tma_load_3d(ds + (size_t)q * kTileRows * SSB, &smap1, 0, 0, (ta + q) * kTileRows, st_full + st);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------ MMA issuer ------------------------------
        // A thread with MMAs queued stalls on any shared-memory access (an mbarrier
        // wait included) until they drain.  So this warp never waits on an
        // mbarrier: warp kWaitWarp does, and meets it at named barrier 2 once per
        // A slot (after x is converted, and before each slot).
        named_barrier_sync(2, 64);
        const bool run = flags[1] == 0 && total > 0;   // read before any MMA is queued
        if (run) {
            const uint32_t xb_addr = smem_addr(xb);
            for (int g = 0; g < nslots; g++) {
                const int slot = g % kSlots;
                named_barrier_sync(2, 64);   // slot g written; the accumulators it starts are free
                fence_after();
                if (lane == 0) {
                    const int G1 = min(total, (g + 1) * kSlotSteps);
                    for (int G = g * kSlotSteps; G < G1; G++) {
                        const int t = G / steps, s = G - t * steps, db = t & 1;
                        mma_ts(tmem + kDCol0 + 32u * db, tmem + 32u * slot + 8u * (G - g * kSlotSteps),
                               b_desc(xb_addr + 1024u * s), s > 0 ? 1u : 0u);
                        if (s == steps - 1) mma_commit(d_full + db);
                    }
                    mma_commit(a_empty + slot);
                }
                __syncwarp();
            }
            // the last products must be complete before tensor memory is released
            mbar_wait_bounded(d_full + ((ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1);
        }
    } else if (warp == kWaitWarp) {
        // ---------------------- waits on behalf of the MMA issuer ----------------------
        mbar_wait(xready, 0, abort);
        named_barrier_sync(2, 64);
        if (flags[1] == 0 && total > 0) {
            for (int g = 0; g < nslots; g++) {
                const int slot = g % kSlots;
                mbar_wait(a_full + slot, (g / kSlots) & 1, abort);
                const int G1 = min(total, (g + 1) * kSlotSteps);
                for (int G = g * kSlotSteps; G < G1; G++) {
                    const int t = G / steps, s = G - t * steps;
                    if (s == 0 && t >= 2) mbar_wait(d_empty + (t & 1), ((t >> 1) - 1) & 1, abort);
                }
                named_barrier_sync(2, 64);
            }
        }
    } else if (warp < kDecWarps) {
        // ------------------------------ decode warps ------------------------------
        const int q = warp & 3, h = warp >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const uint32_t st_sa = smem_addr(stages), xn_sa = smem_addr(xnat), xb_sa = smem_addr(xb);
        bool x_done = false, fast = true;
        DecodeCursor dc;
        dc.steps = steps; dc.TB = TB; dc.NS = NS; dc.total = total; dc.h = h; dc.q = q; dc.lane = lane;
        dc.CSB = CSB; dc.SSB = SSB; dc.stage_bytes = (uint32_t)L.stage_bytes; dc.codes_bytes = (uint32_t)L.codes_bytes;
        dc.st_sa = st_sa; dc.st_full = st_full; dc.st_empty = st_empty; dc.abort = abort;
        dc.cur = -1;
        dc.s = 2 * h;
        dc.i = dc.ti = 0;
        dc.wrap();
        uint32_t hv[16], hn[16];
        int ns = 0, nn = 0;

        for (int g = 0; g < nslots; g++) {
            const int slot = g % kSlots;
            if (g == 0) ns = load_slot(dc, 0, hv);
            if (g >= kSlots) {
                if (!x_done) {
                    // the ring is full: the MMAs need x now.  x -> f16 in the B layout (all 8
                    // decode warps, named barrier 1)
                    mbar_wait(xfull, 0, abort);
                    uint32_t mx = 0;
                    for (int i = threadIdx.x; i < K / 8; i += kDecWarps * 32) {
                        const uint4 v = lds128(xn_sa + 16u * i);
                        mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
                        mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
                        mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
                        mx = __vmaxu2(mx, v.w & 0x7FFF7FFFu);
                    }
                    mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
                    for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                    if (lane == 0) flags[4 + warp] = (int)mx;
                    named_barrier_sync(1, kDecWarps * 32);
                    for (int i = 0; i < kDecWarps; i++) mx = max(mx, (uint32_t)flags[4 + i]);
                    // largest |x * 2^-sigma| in [2^14, 2^15)
                    const int sigma = (mx == 0) ? 0 : max((int)(mx >> 7), 1) - 127 - 14;
                    bool bad = mx >= 0x7F80u;   // Inf / NaN
                    for (int i = threadIdx.x; i < K / 8; i += kDecWarps * 32) {
                        const uint4 v = lds128(xn_sa + 16u * i);
                        const uint4 o = make_uint4(bf16x2_to_f16x2_scaled(v.x, -sigma, bad),
                                                   bf16x2_to_f16x2_scaled(v.y, -sigma, bad),
                                                   bf16x2_to_f16x2_scaled(v.z, -sigma, bad),
                                                   bf16x2_to_f16x2_scaled(v.w, -sigma, bad));
                        sts128(xb_sa + xb_offset(8 * i), o);
                    }
                    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags + 1, 1);
                    if (threadIdx.x == 0) flags[3] = sigma;
                    fence_async_smem();   // generic-proxy writes of xb -> visible to the tensor core
                    named_barrier_sync(1, kDecWarps * 32);
                    fast = flags[1] == 0;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(xready);
                    x_done = true;
                }
                if (!fast) break;
                mbar_wait(a_empty + slot, ((g / kSlots) - 1) & 1, abort);
                fence_after();
            }
            const uint32_t col = lane_base + 32u * slot + 16u * h;
            if (ns == 2)
                tmem_st16(col, hv);
            else if (ns == 1)
                tmem_st8(col, hv);
            nn = 0;
            if (g + 1 < nslots) nn = load_slot(dc, g + 1, hn);   // overlaps the store
            tmem_wait_st();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(a_full + slot);
#pragma unroll
            for (int i = 0; i < 16; i++) hv[i] = hn[i];
            ns = nn;
        }
        // stages this warp had no step of (or skipped after a switch to binary32)
        dc.advance_to(nstages - 1);
        __syncwarp();
        if (lane == 0) mbar_arrive(st_empty + dc.cur % NS);
        if (!x_done) {
            // fewer slots than the ring holds: convert x here (same code as above)
            mbar_wait(xfull, 0, abort);
            uint32_t mx = 0;
            for (int i = threadIdx.x; i < K / 8; i += kDecWarps * 32) {
                const uint4 v = lds128(xn_sa + 16u * i);
                mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, v.w & 0x7FFF7FFFu);
            }
            mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            if (lane == 0) flags[4 + warp] = (int)mx;
            named_barrier_sync(1, kDecWarps * 32);
            for (int i = 0; i < kDecWarps; i++) mx = max(mx, (uint32_t)flags[4 + i]);
            const int sigma = (mx == 0) ? 0 : max((int)(mx >> 7), 1) - 127 - 14;
            bool bad = mx >= 0x7F80u;
            for (int i = threadIdx.x; i < K / 8; i += kDecWarps * 32) {
                const uint4 v = lds128(xn_sa + 16u * i);
                const uint4 o = make_uint4(bf16x2_to_f16x2_scaled(v.x, -sigma, bad),
                                           bf16x2_to_f16x2_scaled(v.y, -sigma, bad),
                                           bf16x2_to_f16x2_scaled(v.z, -sigma, bad),
                                           bf16x2_to_f16x2_scaled(v.w, -sigma, bad));
                sts128(xb_sa + xb_offset(8 * i), o);
            }
            if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags + 1, 1);
            if (threadIdx.x == 0) flags[3] = sigma;
            fence_async_smem();
            named_barrier_sync(1, kDecWarps * 32);
            __syncwarp();
            if (lane == 0) mbar_arrive(xready);
        }
    } else {
        // ------------------------------ epilogue warps ------------------------------
        const int q = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const float gs = __ldg(a.gscale);
        mbar_wait(xready, 0, abort);
        const bool fast = flags[1] == 0;
        const int sigma = flags[3];
        for (int t = 0; t < ntiles; t++) {
            const int row = (t0 + t) * kTileRows + q;
            float sum = 0.0f;
            if (fast) {
                const int db = t & 1;
                mbar_wait(d_full + db, (t >> 1) & 1, abort);
                fence_after();
                uint32_t v[32];
                tmem_ld32(lane_base + kDCol0 + 32u * db, v);
                tmem_wait_ld();
                fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(d_empty + db);
                sum = pick_lane(v, lane);
            } else if (row < N) {
                // binary32 on the CUDA cores from global memory: lane j takes blocks j, j+32, ...
                const uint8_t *cg = a.codes + (size_t)row * CSB;
                const uint8_t *sg = a.scales + (size_t)row * SSB;
                for (int s = 0; s < steps; s++) {
                    const uint2 c = __ldg(reinterpret_cast<const uint2 *>(cg + (size_t)s * 256 + 8 * lane));
                    float2 w[8], xv[8];
                    decode_nvfp4(c, w);
                    const uint4 *xp = reinterpret_cast<const uint4 *>(xnat + s * kStepK + 16 * lane);
                    const uint4 u0 = xp[0], u1 = xp[1];
                    const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                    for (int k = 0; k < 8; k++) xv[k] = make_float2(bf16_lo(wv[k]), bf16_hi(wv[k]));
                    sum = dot_group<8>(w, xv, e4m3_to_f32(__ldg(sg + s * 32 + lane)), sum);
                }
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
            pdl_wait_prior_grid();   // y may be read by the previous kernel
            if (lane == 0 && row < N) a.y[row] = fast ? gs * mul_pow2(sum, sigma) : gs * sum;
        }
    }
    fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace um
}  // namespace w4
