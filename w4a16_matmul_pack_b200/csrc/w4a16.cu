// w4a16.cu -- the C ABI of libw4a16.so (declared in include/w4a16.h): host-side
// validation, launch configuration and launches of the sm_100a kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "pack.cuh"
#include "gemv.cuh"
#include "gemv_tc.cuh"
#include "gemv_m1.cuh"
#include "gemv_skinny.cuh"
#include "gemm.cuh"

using namespace w4;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

w4_status device_info(DeviceInfo &out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (d.sms == 0) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
            d.sms = 0;
            return W4_ERR_CUDA;
        }
    }
    out = d;
    return W4_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline w4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// ------------------------------------------------------------------ GEMV ----

constexpr size_t kXBudget = 64 * 1024;      // shared bytes for the x slice

// Alignment unit of K for the GEMV stages: row pieces must start on 16 bytes.
inline int k_unit(int fmt) { return fmt == W4_FMT_ROCMFP4_FAST ? 512 : 256; }

// NVFP4 decode GEMV on the tensor cores (gemv_tc.cuh).
struct GemvTcPlan {
    int M = 1, S = 1, kc = 0, KP = 0, NS = 0, xstride = 0, tile_bytes = 0, grid = 0;
    int rows_mode = 0, tiles_per_cta = 0, box_min_rows = 4, red_tiles = 2;
    size_t smem = 0, ws_bytes = 0;
};

constexpr int kTcPieceMax = 4096;      // k per stage (TMA box: 256 8-byte elements of codes)
constexpr double kSmBytesPerUs = 48e3;  // bytes per us one SM streams with a deep copy ring
constexpr double kHbmBytesPerUs = 7e6;  // whole-device streaming rate
constexpr double kCopyUs = 0.2;         // cost of one bulk / tensor copy on an SM

// force_grid > 0: exactly that many CTAs, each on a balanced range of rows (the
// grouped launch gives every problem its own share of the SMs).
inline int block_bytes(int fmt) { return fmt == W4_FMT_ROCMFP4_DUAL ? 18 : 17; }

// One NVFP4 token (gemv_m1.cuh): K slices of at most kM1MaxSlice (x' of a slice
// in shared memory as f16); a problem with fewer 16-row tiles than half the SMs
// is also split along K (slices of at least 2048 k) so that the launch still
// fills the GPU; at most kM1MaxTiles tiles per CTA (its partial-sum buffer).
constexpr int kM1MaxTiles = 32;

w4_status plan_gemv_m1(int K, int N, GemvTcPlan &p, int force_grid, const DeviceInfo &d) {
    p.M = 1;
    const int T = (N + kTcRows - 1) / kTcRows;
    int S = (K + kM1MaxSlice - 1) / kM1MaxSlice;
    if (force_grid <= 0 && T < d.sms / 2) S = std::max(S, std::min(d.sms / T, K / 2048));
    S = std::max(S, 1);
    p.kc = ((K + S - 1) / S + 255) / 256 * 256;
    p.S = (K + p.kc - 1) / p.kc;
    if (force_grid > 0) {
        if (p.S != 1) return W4_ERR_UNSUPPORTED;
        p.grid = std::min(force_grid, T);
    } else {
        p.grid = std::min(T, std::max(1, d.sms / p.S));
        p.grid = std::max(p.grid, (T + kM1MaxTiles - 1) / kM1MaxTiles);
    }
    p.red_tiles = (T + p.grid - 1) / p.grid;
    p.xstride = (p.kc / 128) * kM1ScStride;
    p.KP = p.kc;
    p.NS = 0;
    p.tile_bytes = 0;
    p.rows_mode = 1;
    p.tiles_per_cta = p.red_tiles;
    p.smem = m1_layout(p.xstride, p.red_tiles).total;
    if (p.smem > (size_t)d.smem_optin) return W4_ERR_UNSUPPORTED;
    p.ws_bytes = p.S > 1 ? (size_t)p.S * N * sizeof(float) : 0;
    return W4_OK;
}

// NVFP4, M = 2..16 (gemv_skinny.cuh): K slices whose x' (rows padded to 8
// tokens) fits kSkinnyXBytes; short problems are also split along K as for one
// token; tiles per CTA as many as the partial-sum buffer holds.

w4_status plan_gemv_skinny(int K, int N, int M, GemvTcPlan &p, const DeviceInfo &d) {
    p.M = M;
    const int R = (M + 7) / 8 * 8;
    const int T = (N + kTcRows - 1) / kTcRows;
    const int kmax = skinny_kmax(M);
    int S = (K + kmax - 1) / kmax;
    if (T < d.sms / 2) S = std::max(S, std::min(d.sms / T, K / 2048));
    S = std::max(S, 1);
    p.kc = ((K + S - 1) / S + 255) / 256 * 256;
    p.S = (K + p.kc - 1) / p.kc;
    p.xstride = p.kc + 32;   // rows 64 bytes apart modulo 128
    const size_t xbytes = ((size_t)R * p.xstride * 2 + 127) & ~(size_t)127;
    const size_t per_tile = (size_t)kM1Warps * kTcRows * skinny_pad(M) * 4;
    const size_t fbytes = 4 * (2 + 2 * kM1Warps);
    const size_t room = (size_t)d.smem_optin > xbytes + fbytes ? (size_t)d.smem_optin - xbytes - fbytes : 0;
    const int red_max = (int)(room / per_tile);
    if (red_max < 1) return W4_ERR_UNSUPPORTED;
    p.grid = std::min(T, std::max(1, d.sms / p.S));
    p.grid = std::max(p.grid, (T + red_max - 1) / red_max);
    p.red_tiles = (T + p.grid - 1) / p.grid;
    p.KP = p.kc;
    p.NS = 0;
    p.tile_bytes = 0;
    p.rows_mode = 1;
    p.tiles_per_cta = p.red_tiles;
    p.smem = skinny_layout(M, p.xstride, p.red_tiles).total;
    if (p.smem > (size_t)d.smem_optin) return W4_ERR_UNSUPPORTED;
    p.ws_bytes = p.S > 1 ? (size_t)p.S * M * N * sizeof(float) : 0;
    return W4_OK;
}

w4_status plan_gemv_tc(int fmt, int K, int N, int M, bool pdl, GemvTcPlan &p, int force_grid = 0) {
    DeviceInfo d;
    if (device_info(d) != W4_OK) return W4_ERR_CUDA;
    if (fmt == W4_FMT_NVFP4 && M == 1) return plan_gemv_m1(K, N, p, force_grid, d);
    if (fmt == W4_FMT_NVFP4 && force_grid <= 0) return plan_gemv_skinny(K, N, M, p, d);
    p.M = M;
    const bool nv = fmt == W4_FMT_NVFP4;
    const int unit = k_unit(fmt);
    const int units = K / unit;
    int per = (int)std::max<size_t>(1, kXBudget / ((size_t)2 * M * unit));
    per = std::min(per, units);
    p.kc = per * unit;
    p.S = (units + per - 1) / per;
    // ROCmFP4 stages: a box row of KP/32 blocks is at most 256 8-byte elements
    const int piece_max = nv ? kTcPieceMax : 3584;
    int npieces = (p.kc + piece_max - 1) / piece_max;
    p.KP = ((p.kc + npieces - 1) / npieces + unit - 1) / unit * unit;
    p.xstride = p.kc + 32;
    p.tile_bytes = nv ? (kTcRows * (p.KP / 2 + p.KP / 16) + 127) & ~127
                      : (kTcRows * stage_row_bytes(fmt, block_bytes(fmt), p.KP) + 127) & ~127;
    const size_t xs = ((size_t)M * p.xstride * 2 + 127) & ~(size_t)127;
    const size_t tail = 16 + 4 * kTcWarps;   // flags
    const size_t budget = std::min<size_t>(200 * 1024, (size_t)d.smem_optin);

    // rows per CTA: balanced ranges (a partial last tile per CTA) or whole tiles.
    // With split-K the S slices of a row range run side by side, so the row
    // grid takes SMs / S: the launch stays one wave of resident CTAs.
    const int row_sms = std::max(1, d.sms / p.S);
    const double rowB = nv ? (double)K / 2 + K / 16 : (double)stage_row_bytes(fmt, block_bytes(fmt), K);
    const int T = (N + kTcRows - 1) / kTcRows;
    const int gA = std::min(row_sms, N);
    const int rowsA = (N + gA - 1) / gA, tailA = rowsA % kTcRows, fullA = rowsA / kTcRows;
    const int readA = fullA * kTcRows + (tailA >= p.box_min_rows ? kTcRows : tailA);
    const int copiesA = 2 * fullA + (tailA == 0 ? 0 : (tailA >= p.box_min_rows ? 2 : 2 * tailA));
    const double costA = std::max(readA * rowB / kSmBytesPerUs, (double)N * rowB / kHbmBytesPerUs) +
                         copiesA * p.S * kCopyUs;
    const int q = (T + row_sms - 1) / row_sms, gB = (T + q - 1) / q;
    const double costB = std::max(q * kTcRows * rowB / kSmBytesPerUs, (double)T * kTcRows * rowB / kHbmBytesPerUs) +
                         2 * q * p.S * kCopyUs;
    int tiles_max;
    if (force_grid > 0) {
        p.rows_mode = 0;
        p.tiles_per_cta = 0;
        p.grid = std::min(force_grid, N);
        const int rows = (N + p.grid - 1) / p.grid;
        tiles_max = (rows + kTcRows - 1) / kTcRows + 1;
    } else if (costB <= costA) {
        p.rows_mode = 1;
        p.tiles_per_cta = q;
        p.grid = gB;
        tiles_max = q;
    } else {
        p.rows_mode = 0;
        p.tiles_per_cta = 0;
        p.grid = gA;
        tiles_max = (rowsA + kTcRows - 1) / kTcRows;
    }
    // partial sums of all of a CTA's tiles at once when they fit (one barrier per CTA)
    const size_t part_bytes = (size_t)kTcParts * kTcRows * M * 4;
    p.red_tiles = (tiles_max * part_bytes <= 24 * 1024) ? std::max(tiles_max, 2) : 2;
    const size_t red = (size_t)p.red_tiles * part_bytes;

    auto total = [&](int ns) -> size_t { return xs + (size_t)ns * p.tile_bytes + red + 16 * ns + tail; };
    int NS = 8;
    while (NS > 2 && total(NS) > budget) NS--;
    p.NS = NS;
    p.smem = total(NS);
    if (p.smem > (size_t)d.smem_optin) return W4_ERR_UNSUPPORTED;
    p.ws_bytes = p.S > 1 ? (size_t)p.S * M * N * sizeof(float) : 0;
    return W4_OK;
}

// Tensor maps of one NVFP4 matrix for the GEMV stages (16-row x KP-k boxes) and
// the kernel arguments.
w4_status gemv_tc_setup(const w4_weights *w, const void *x, float *y, void *ws, const GemvTcPlan &p, bool pdl,
                        CUtensorMap &cmap, CUtensorMap &smap, GemvTcArgs &a) {
    PFN_encodeTiled enc = get_encode_tiled();
    if (!enc) return W4_ERR_CUDA;
    const int K = w->K, N = w->N;
    const cuuint64_t cdims[2] = {(cuuint64_t)K / 16, (cuuint64_t)N};   // codes as 8-byte elements
    const cuuint64_t cstr[1] = {(cuuint64_t)K / 2};
    const cuuint32_t cbox[2] = {(cuuint32_t)p.KP / 16, (cuuint32_t)kTcRows};
    // one token: codes as [N][K/256][16 x 8 bytes], 3-D box of 16 rows x KP/256
    // lines of 128 bytes, 128-byte swizzle (the consumers' chunk XOR)
    const bool nv = w->fmt == W4_FMT_NVFP4;
    const bool direct = nv;   // the NVFP4 kernels load their operands directly
    // ROCmFP4: blocks as 8-byte elements, a box of 16 rows x KP/32 blocks, no scales map
    const int bb = nv ? 0 : block_bytes(w->fmt);
    const cuuint64_t rdims[2] = {(cuuint64_t)stage_row_bytes(w->fmt, bb, K) / 8, (cuuint64_t)N};
    const cuuint64_t rstr[1] = {(cuuint64_t)stage_row_bytes(w->fmt, bb, K)};
    const cuuint32_t rbox[2] = {(cuuint32_t)stage_row_bytes(w->fmt, bb, p.KP) / 8, (cuuint32_t)kTcRows};
    const cuuint64_t sdims[2] = {(cuuint64_t)K / 16, (cuuint64_t)N};
    const cuuint64_t sstr[1] = {(cuuint64_t)K / 16};
    const cuuint32_t sbox[2] = {(cuuint32_t)p.KP / 16, (cuuint32_t)kTcRows};
    const cuuint32_t estr[2] = {1, 1};
    if (!nv) {
        if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t *>(w->codes), rdims, rstr, rbox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
        smap = cmap;
    }
    if (nv && !direct &&
        (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t *>(w->codes), cdims, cstr, cbox, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
         enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w->scales), sdims, sstr, sbox, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS))
        return W4_ERR_CUDA;
    a.codes = w->codes;
    a.scales = w->scales;
    a.gscale = w->global_scale;
    a.x = reinterpret_cast<const uint16_t *>(x);
    a.y = y;
    a.partial = reinterpret_cast<float *>(ws);
    a.K = K;
    a.N = N;
    a.kc = p.kc;
    a.KP = p.KP;
    a.NS = p.NS;
    a.xstride = p.xstride;
    a.tile_bytes = p.tile_bytes;
    a.rows_mode = p.rows_mode;
    a.tiles_per_cta = p.tiles_per_cta;
    a.box_min_rows = p.box_min_rows;
    a.red_tiles = p.red_tiles;
    a.pdl = pdl ? 1 : 0;
    a.fmt = w->fmt;
    a.bb = bb;
    return W4_OK;
}

template <int FMT, int M>
w4_status launch_gemv_tc_m(const w4_weights *w, const void *x, float *y, void *ws, const GemvTcPlan &p, bool pdl,
                           cudaStream_t st) {
    // one NVFP4 token: block scales applied after the MMA, operands loaded
    // directly (gemv_m1.cuh); otherwise TMA-staged tiles (gemv_tc.cuh)
    constexpr bool direct = FMT == W4_FMT_NVFP4;
    const void *kern = !direct ? reinterpret_cast<const void *>(gemv_tc_kernel<FMT, M>)
                               : (M == 1 ? reinterpret_cast<const void *>(gemv_nvfp4_m1_kernel)
                                         : reinterpret_cast<const void *>(gemv_nvfp4_skinny_kernel<M>));
    if (!set_smem_limit(kern, p.smem)) return W4_ERR_CUDA;
    const int N = w->N;
    CUtensorMap cmap, smap;
    GemvTcArgs a;
    const w4_status s0 = gemv_tc_setup(w, x, y, ws, p, pdl, cmap, smap, a);
    if (s0 != W4_OK) return s0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, p.S, 1);
    cfg.blockDim = dim3(direct ? kM1Threads : kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e;
    if constexpr (direct && M == 1)
        e = cudaLaunchKernelEx(&cfg, gemv_nvfp4_m1_kernel, a);
    else if constexpr (direct)
        e = cudaLaunchKernelEx(&cfg, gemv_nvfp4_skinny_kernel<M>, a);
    else
        e = cudaLaunchKernelEx(&cfg, gemv_tc_kernel<FMT, M>, cmap, smap, a);
    if (e != cudaSuccess) return W4_ERR_CUDA;
    if (p.S > 1) {
        const int MN = M * N;
        // the slice partials already carry the global scale (scale_out); with
        // PDL the adds launch early and wait for the slices in the kernel
        cudaLaunchConfig_t fc = {};
        fc.gridDim = dim3(std::min((MN + 255) / 256, 1024), 1, 1);
        fc.blockDim = dim3(256, 1, 1);
        fc.stream = st;
        fc.attrs = attr;
        fc.numAttrs = pdl ? 1 : 0;
        if (cudaLaunchKernelEx(&fc, gemv_finalize_kernel, (const float *)a.partial, p.S, MN, (const float *)nullptr,
                               y) != cudaSuccess)
            return W4_ERR_CUDA;
    }
    return launch_status();
}

// SMs shared out among G problems so that the heaviest CTA carries as few
// bytes as whole 16-row tiles allow: with a load L, problem p needs
// ceil(T_p / floor(L / b_p)) CTAs (T_p = max_cta[p] tiles of b_p bytes each),
// and the smallest L whose CTAs fit in the SMs is found by bisection.  SMs
// left over go one at a time to the problem whose CTAs carry the most bytes
// on average (never more CTAs than tiles).  Every problem gets at least one
// CTA, even when there are more problems than SMs.
void share_sms(const w4_weights *w, int G, int sms, const int *max_cta, int *alloc) {
    long long tb[kMaxGroup], lo = 1, hi = 1;
    for (int p = 0; p < G; p++) {
        tb[p] = (long long)kTcRows * (w[p].K / 2 + w[p].K / 16);
        lo = std::max(lo, tb[p]);
        hi = std::max(hi, tb[p] * max_cta[p]);
    }
    auto ctas_for = [&](long long L, int *a) {
        long long sum = 0;
        for (int p = 0; p < G; p++) {
            const long long k = std::max<long long>(1, L / tb[p]);   // tiles per CTA
            a[p] = (int)((max_cta[p] + k - 1) / k);
            sum += a[p];
        }
        return sum;
    };
    if (ctas_for(hi, alloc) > sms) return;   // one CTA per problem
    while (lo < hi) {
        const long long mid = lo + (hi - lo) / 2;
        if (ctas_for(mid, alloc) <= sms)
            hi = mid;
        else
            lo = mid + 1;
    }
    long long sum = ctas_for(lo, alloc);
    while (sum < sms) {
        int best = -1;
        for (int p = 0; p < G; p++)
            if (alloc[p] < max_cta[p] &&
                (best < 0 || (double)tb[p] * max_cta[p] / alloc[p] > (double)tb[best] * max_cta[best] / alloc[best]))
                best = p;
        if (best < 0) break;
        alloc[best]++;
        sum++;
    }
}

// Most CTAs a grouped launch gives problem p: one per 16-row tile, at least one.
void grouped_max_cta(const w4_weights *w, int G, int *max_cta) {
    for (int p = 0; p < G; p++) max_cta[p] = (w[p].N + kTcRows - 1) / kTcRows;
}

// Several one-token NVFP4 problems in one launch (gemv_m1.cuh): the SMs are
// shared out so that the heaviest CTA carries as few whole tiles' bytes as
// possible (share_sms), and every CTA runs the single-problem kernel body on a
// balanced range of its problem's tiles.
w4_status launch_gemv_grouped(const w4_weights *w, const void *const *x, float *const *y, int G, bool pdl,
                              cudaStream_t st) {
    DeviceInfo d;
    if (device_info(d) != W4_OK) return W4_ERR_CUDA;
    int tiles[kMaxGroup], alloc[kMaxGroup];
    grouped_max_cta(w, G, tiles);
    share_sms(w, G, d.sms, tiles, alloc);
    static GroupArgs g;   // host staging of the kernel parameter (copied at launch)
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    g.G = G;
    g.cta0[0] = 0;
    size_t smem = 0;
    for (int p = 0; p < G; p++) {
        GemvTcPlan plan;
        w4_status s = plan_gemv_tc(W4_FMT_NVFP4, w[p].K, w[p].N, 1, pdl, plan, alloc[p]);
        if (s != W4_OK) return s;
        if (plan.S != 1) return W4_ERR_UNSUPPORTED;
        CUtensorMap unused_c, unused_s;
        s = gemv_tc_setup(&w[p], x[p], y[p], nullptr, plan, pdl, unused_c, unused_s, g.a[p]);
        if (s != W4_OK) return s;
        g.cta0[p + 1] = g.cta0[p] + plan.grid;
        smem = std::max(smem, plan.smem);
    }
    if (!set_smem_limit(reinterpret_cast<const void *>(gemv_nvfp4_m1_grouped_kernel), smem)) return W4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.cta0[G], 1, 1);
    cfg.blockDim = dim3(kM1Threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, gemv_nvfp4_m1_grouped_kernel, g) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

template <int FMT>
w4_status launch_gemv_tc_fmt(const w4_weights *w, const void *x, int M, float *y, void *ws, const GemvTcPlan &p,
                             bool pdl, cudaStream_t st) {
    switch (M) {
#define W4_CASE(m) \
    case m: return launch_gemv_tc_m<FMT, m>(w, x, y, ws, p, pdl, st);
        W4_CASE(1) W4_CASE(2) W4_CASE(3) W4_CASE(4) W4_CASE(5) W4_CASE(6) W4_CASE(7) W4_CASE(8)
        W4_CASE(9) W4_CASE(10) W4_CASE(11) W4_CASE(12) W4_CASE(13) W4_CASE(14) W4_CASE(15) W4_CASE(16)
#undef W4_CASE
    }
    return W4_ERR_ARG;
}

w4_status launch_gemv_tc(const w4_weights *w, const void *x, int M, float *y, void *ws, const GemvTcPlan &p, bool pdl,
                         cudaStream_t st) {
    switch (w->fmt) {
    case W4_FMT_NVFP4: return launch_gemv_tc_fmt<W4_FMT_NVFP4>(w, x, M, y, ws, p, pdl, st);
    case W4_FMT_ROCMFP4_DUAL: return launch_gemv_tc_fmt<W4_FMT_ROCMFP4_DUAL>(w, x, M, y, ws, p, pdl, st);
    case W4_FMT_ROCMFP4_FAST: return launch_gemv_tc_fmt<W4_FMT_ROCMFP4_FAST>(w, x, M, y, ws, p, pdl, st);
    }
    return W4_ERR_ARG;
}

// Any K the packers accept (gemv_any_kernel): one warp per weight row.
template <int FMT>
w4_status launch_gemv_any(const w4_weights *w, const void *x, int M, float *y, cudaStream_t st) {
    const int grid = (w->N + 7) / 8;
    const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
    switch (M) {
#define W4_CASE(m) \
    case m: gemv_any_kernel<FMT, m><<<grid, 256, 0, st>>>(w->codes, w->scales, w->global_scale, xb, y, w->K, w->N); break;
        W4_CASE(1) W4_CASE(2) W4_CASE(3) W4_CASE(4) W4_CASE(5) W4_CASE(6) W4_CASE(7) W4_CASE(8)
        W4_CASE(9) W4_CASE(10) W4_CASE(11) W4_CASE(12) W4_CASE(13) W4_CASE(14) W4_CASE(15) W4_CASE(16)
#undef W4_CASE
    default: return W4_ERR_ARG;
    }
    return launch_status();
}

w4_status check_weights(const w4_weights *w) {
    if (!w || !w->codes || w->K <= 0 || w->N <= 0) return W4_ERR_ARG;
    if (w->fmt == W4_FMT_NVFP4) {
        if (!w->scales || !w->global_scale || w->K % 16) return W4_ERR_ARG;
        if (!aligned16(w->codes) || !aligned16(w->scales) || (reinterpret_cast<uintptr_t>(w->global_scale) & 3))
            return W4_ERR_ALIGN;
    } else if (w->fmt == W4_FMT_ROCMFP4_DUAL || w->fmt == W4_FMT_ROCMFP4_FAST) {
        if (w->K % 32) return W4_ERR_ARG;
        if (!aligned16(w->codes)) return W4_ERR_ALIGN;
    } else if (w->fmt == W4_FMT_Q4_0) {
        return W4_ERR_UNSUPPORTED;   // a comparison format: packed and scored, not multiplied
    } else {
        return W4_ERR_ARG;
    }
    return W4_OK;
}

// As check_weights, for entry points that accept every format (Q4_0 included).
w4_status check_weights_any(const w4_weights *w) {
    if (w && w->fmt == W4_FMT_Q4_0) {
        if (!w->codes || w->K <= 0 || w->N <= 0 || w->K % 32) return W4_ERR_ARG;
        if (!aligned16(w->codes)) return W4_ERR_ALIGN;
        return W4_OK;
    }
    return check_weights(w);
}

}  // namespace

// ======================================================================== ABI

extern "C" {

size_t pack_nvfp4_workspace_bytes(void) { return 16; }

w4_status pack_nvfp4_ex(const void *W, int K, int N, int block, int scale_search, const float *importance,
                        uint8_t *codes, uint8_t *scales, float *global_scale, void *workspace, size_t workspace_bytes,
                        int *d_status, void *stream) {
    if (!W || !codes || !scales || !global_scale || K < 16 || N < 1 || K % 16 || block != 16) return W4_ERR_ARG;
    if (scale_search != W4_SCALE_ABSMAX && scale_search != W4_SCALE_MSE) return W4_ERR_ARG;
    if (importance && scale_search != W4_SCALE_MSE) return W4_ERR_ARG;
    if (!workspace || workspace_bytes < pack_nvfp4_workspace_bytes()) return W4_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || !aligned16(workspace) ||
        (importance && !aligned16(importance)) || (reinterpret_cast<uintptr_t>(global_scale) & 3) ||
        (reinterpret_cast<uintptr_t>(d_status) & 3))
        return W4_ERR_ALIGN;
    DeviceInfo d;
    if (device_info(d) != W4_OK) return W4_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    const long long total = (long long)K * N;
    if (cudaMemsetAsync(workspace, 0, 8, st) != cudaSuccess) return W4_ERR_CUDA;
    if (d_status && cudaMemsetAsync(d_status, 0, sizeof(int), st) != cudaSuccess) return W4_ERR_CUDA;
    const long long n8 = total / 8;
    const int g1 = (int)std::min<long long>((n8 + 255) / 256, (long long)d.sms * 8);
    nvfp4_absmax_kernel<<<g1, 256, 0, st>>>(reinterpret_cast<const uint4 *>(W), n8,
                                             reinterpret_cast<unsigned *>(workspace));
    const long long nb = total / 16;
    if (scale_search == W4_SCALE_MSE) {
        const int g3 = (int)std::min<long long>((nb + 7) / 8, (long long)d.sms * 16);
        if (importance)
            nvfp4_search_kernel<true><<<g3, 256, 0, st>>>(
                reinterpret_cast<const uint16_t *>(W), nb, K, reinterpret_cast<const unsigned *>(workspace), importance,
                reinterpret_cast<uint2 *>(codes), scales, global_scale, d_status);
        else
            nvfp4_search_kernel<false><<<g3, 256, 0, st>>>(
                reinterpret_cast<const uint16_t *>(W), nb, K, reinterpret_cast<const unsigned *>(workspace), nullptr,
                reinterpret_cast<uint2 *>(codes), scales, global_scale, d_status);
        return launch_status();
    }
    const int g2 = (int)std::min<long long>((nb + 255) / 256, (long long)d.sms * 16);
    nvfp4_encode_kernel<<<g2, 256, 0, st>>>(reinterpret_cast<const uint4 *>(W), nb,
                                             reinterpret_cast<const unsigned *>(workspace),
                                             reinterpret_cast<uint2 *>(codes), scales, global_scale, d_status);
    return launch_status();
}

w4_status pack_nvfp4(const void *W, int K, int N, int block, int scale_search, uint8_t *codes, uint8_t *scales,
                     float *global_scale, void *workspace, size_t workspace_bytes, int *d_status, void *stream) {
    return pack_nvfp4_ex(W, K, N, block, scale_search, nullptr, codes, scales, global_scale, workspace,
                         workspace_bytes, d_status, stream);
}

w4_status pack_rocmfp4(const void *W, int K, int N, int block, int fmt, const float *importance, uint8_t *blocks,
                       int *d_status, void *stream) {
    if (!W || !blocks || K < 32 || N < 1 || K % 32 || block != 32) return W4_ERR_ARG;
    if (fmt != W4_FMT_ROCMFP4_DUAL && fmt != W4_FMT_ROCMFP4_FAST) return W4_ERR_ARG;
    if (!aligned16(W) || !aligned16(blocks) || (importance && !aligned16(importance)) ||
        (reinterpret_cast<uintptr_t>(d_status) & 3))
        return W4_ERR_ALIGN;
    DeviceInfo d;
    if (device_info(d) != W4_OK) return W4_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (d_status && cudaMemsetAsync(d_status, 0, sizeof(int), st) != cudaSuccess) return W4_ERR_CUDA;
    const long long nblk = (long long)K * N / 32;
    const int grid = (int)std::min<long long>((nblk + 7) / 8, (long long)d.sms * 16);
    const uint16_t *w16 = reinterpret_cast<const uint16_t *>(W);
    if (fmt == W4_FMT_ROCMFP4_DUAL) {
        if (importance)
            rocm_pack_kernel<true, true><<<grid, 256, 0, st>>>(w16, nblk, K, importance, blocks, d_status);
        else
            rocm_pack_kernel<true, false><<<grid, 256, 0, st>>>(w16, nblk, K, nullptr, blocks, d_status);
    } else {
        if (importance)
            rocm_pack_kernel<false, true><<<grid, 256, 0, st>>>(w16, nblk, K, importance, blocks, d_status);
        else
            rocm_pack_kernel<false, false><<<grid, 256, 0, st>>>(w16, nblk, K, nullptr, blocks, d_status);
    }
    return launch_status();
}

w4_status pack_q4_0(const void *W, int K, int N, int block, uint8_t *blocks, int *d_status, void *stream) {
    if (!W || !blocks || K < 32 || N < 1 || K % 32 || block != 32) return W4_ERR_ARG;
    if (!aligned16(W) || !aligned16(blocks) || (reinterpret_cast<uintptr_t>(d_status) & 3)) return W4_ERR_ALIGN;
    DeviceInfo d;
    if (device_info(d) != W4_OK) return W4_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (d_status && cudaMemsetAsync(d_status, 0, sizeof(int), st) != cudaSuccess) return W4_ERR_CUDA;
    const long long nblk = (long long)K * N / 32;
    const int grid = (int)std::min<long long>((nblk + 255) / 256, (long long)d.sms * 16);
    q4_0_pack_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4 *>(W), nblk, blocks, d_status);
    return launch_status();
}

size_t w4_reconstruction_workspace_bytes(void) { return (size_t)kReconMaxGrid * sizeof(double2); }

w4_status w4_reconstruction_error(const w4_weights *w, const void *W, double *out, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    w4_status s = check_weights_any(w);
    if (s != W4_OK) return s;
    if (!W || !out) return W4_ERR_ARG;
    if (w->K % 32) return W4_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < w4_reconstruction_workspace_bytes()) return W4_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(out) || !aligned16(workspace)) return W4_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    const long long nblk = (long long)w->K * w->N / 32;
    const int grid = (int)std::min<long long>((nblk + 255) / 256, kReconMaxGrid);
    recon_partial_kernel<<<grid, 256, 0, st>>>(w->fmt, w->K, nblk, w->codes, w->scales, w->global_scale,
                                               reinterpret_cast<const uint16_t *>(W),
                                               reinterpret_cast<double2 *>(workspace));
    recon_final_kernel<<<1, 32, 0, st>>>(reinterpret_cast<const double2 *>(workspace), grid, out);
    return launch_status();
}

size_t w4a16_workspace_bytes(const w4_weights *w, int M) {
    if (check_weights(w) != W4_OK || M < 1) return 0;
    if (M <= 16) {
        if (w->K % k_unit(w->fmt)) return 0;
        GemvTcPlan p, q;
        if (plan_gemv_tc(w->fmt, w->K, w->N, M, false, p) != W4_OK) return 0;
        if (plan_gemv_tc(w->fmt, w->K, w->N, M, true, q) != W4_OK) return p.ws_bytes;
        return std::max(p.ws_bytes, q.ws_bytes);
    }
    return gemm_workspace_bytes(w, M);
}

w4_status w4a16_gemv_ex(const w4_weights *w, const void *x, int M, float *y, void *workspace,
                        size_t workspace_bytes, unsigned flags, void *stream) {
    w4_status s = check_weights(w);
    if (s != W4_OK) return s;
    if (!x || !y || M < 1 || M > 16 || (flags & ~W4_LAUNCH_PDL)) return W4_ERR_ARG;
    if (!aligned16(x) || !aligned16(y) || (workspace && !aligned16(workspace))) return W4_ERR_ALIGN;
    const bool pdl = (flags & W4_LAUNCH_PDL) != 0;
    cudaStream_t st = as_stream(stream);
    if (w->K % k_unit(w->fmt)) {
        // K the fast kernels' 16-byte row pieces do not fit: the general path
        switch (w->fmt) {
        case W4_FMT_NVFP4: return launch_gemv_any<W4_FMT_NVFP4>(w, x, M, y, st);
        case W4_FMT_ROCMFP4_DUAL: return launch_gemv_any<W4_FMT_ROCMFP4_DUAL>(w, x, M, y, st);
        case W4_FMT_ROCMFP4_FAST: return launch_gemv_any<W4_FMT_ROCMFP4_FAST>(w, x, M, y, st);
        }
        return W4_ERR_ARG;
    }
    GemvTcPlan p;
    if ((s = plan_gemv_tc(w->fmt, w->K, w->N, M, pdl, p)) != W4_OK) return s;
    if (p.ws_bytes && (!workspace || workspace_bytes < p.ws_bytes)) return W4_ERR_WORKSPACE;
    return launch_gemv_tc(w, x, M, y, workspace, p, pdl, st);
}

w4_status w4_plan_grouped(const w4_weights *w, int G, int sms, unsigned flags, int *ctas) {
    if (!w || !ctas || G < 1 || G > kMaxGroup || sms < 1 || (flags & ~W4_LAUNCH_PDL)) return W4_ERR_ARG;
    for (int p = 0; p < G; p++) {
        const w4_status s = check_weights(&w[p]);
        if (s != W4_OK) return s;
        if (w[p].fmt != W4_FMT_NVFP4) return W4_ERR_UNSUPPORTED;
    }
    int max_cta[kMaxGroup];
    grouped_max_cta(w, G, max_cta);
    share_sms(w, G, sms, max_cta, ctas);
    return W4_OK;
}

w4_status w4a16_gemv_grouped(const w4_weights *w, const void *const *x, float *const *y, int G, unsigned flags,
                             void *stream) {
    if (!w || !x || !y || G < 1 || G > kMaxGroup || (flags & ~W4_LAUNCH_PDL)) return W4_ERR_ARG;
    for (int p = 0; p < G; p++) {
        const w4_status s = check_weights(&w[p]);
        if (s != W4_OK) return s;
        if (w[p].fmt != W4_FMT_NVFP4) return W4_ERR_UNSUPPORTED;
        if (!x[p] || !y[p]) return W4_ERR_ARG;
        if (!aligned16(x[p]) || !aligned16(y[p])) return W4_ERR_ALIGN;
        if (w[p].K % 256) return W4_ERR_UNSUPPORTED;
    }
    return launch_gemv_grouped(w, x, y, G, (flags & W4_LAUNCH_PDL) != 0, as_stream(stream));
}

w4_status w4a16_gemv(const w4_weights *w, const void *x, int M, float *y, void *workspace, size_t workspace_bytes,
                     void *stream) {
    return w4a16_gemv_ex(w, x, M, y, workspace, workspace_bytes, 0u, stream);
}

w4_status w4a16_gemm(const w4_weights *w, const void *x, int M, float *y_f32, void *y_bf16, void *workspace,
                     size_t workspace_bytes, void *stream) {
    w4_status s = check_weights(w);
    if (s != W4_OK) return s;
    if (!x || M < 1 || (!y_f32 && !y_bf16)) return W4_ERR_ARG;
    if (!aligned16(x) || (y_f32 && !aligned16(y_f32)) || (y_bf16 && !aligned16(y_bf16))) return W4_ERR_ALIGN;
    return gemm_launch(w, x, M, y_f32, y_bf16, workspace, workspace_bytes, as_stream(stream));
}

w4_status w4_encode_scalars(const float *v, size_t n, uint8_t *e4m3, uint8_t *e2m1, void *stream) {
    if (!v || (!e4m3 && !e2m1)) return W4_ERR_ARG;
    if (n == 0) return W4_OK;
    DeviceInfo d;
    if (device_info(d) != W4_OK) return W4_ERR_CUDA;
    const int grid = (int)std::min<long long>(((long long)n + 255) / 256, (long long)d.sms * 16);
    encode_scalars_kernel<<<grid, 256, 0, as_stream(stream)>>>(v, (long long)n, e4m3, e2m1);
    return launch_status();
}

w4_status w4_device_error(int *out, int clear) {
    if (!out) return W4_ERR_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return W4_ERR_CUDA;
    if (cudaMemcpyFromSymbol(out, g_device_error, sizeof(int)) != cudaSuccess) return W4_ERR_CUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return W4_ERR_CUDA;
    }
    return W4_OK;
}

const char *w4_status_string(int status) {
    switch (status) {
    case W4_OK: return "W4_OK";
    case W4_ERR_ARG: return "W4_ERR_ARG: invalid argument";
    case W4_ERR_ALIGN: return "W4_ERR_ALIGN: pointer not 16-byte aligned";
    case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED: shape or option not supported";
    case W4_ERR_CUDA: return "W4_ERR_CUDA: CUDA call or launch failed";
    case W4_ERR_NONFINITE: return "W4_ERR_NONFINITE: NaN or Inf in the input matrix";
    case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT: device-side wait expired";
    case W4_ERR_WORKSPACE: return "W4_ERR_WORKSPACE: workspace missing or too small";
    }
    return "unknown w4_status";
}

w4_status w4_set_wait_limit(unsigned long long ns) {
    const unsigned long long v = ns ? ns : kWaitLimitNs;
    if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return W4_ERR_CUDA;
    return W4_OK;
}

const char *w4_version(void) { return "w4a16 0.2.0 (sm_100a)"; }

}  // extern "C"
