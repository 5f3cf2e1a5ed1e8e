// common.cuh -- device helpers for the sm_100a kernels: format conversions,
// mbarrier / bulk-copy PTX wrappers, bounded waits, programmatic dependent
// launch.  Single translation unit: included once from w4a16.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#include "../../include/w4a16.h"

namespace w4 {

// Sticky device error word (w4_status of the first device-side failure).
__device__ int g_device_error;

// A wait on an mbarrier that takes longer than this is treated as a failure:
// the kernel records W4_ERR_TIMEOUT and returns instead of spinning forever.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Limit of the waits that gate progress (mbar_wait), per device; settable from
// the host (w4_set_wait_limit) so that failure detection can be exercised.  The
// waits that drain a CTA's own copies and MMAs before it exits (mbar_wait_bounded)
// keep the fixed kWaitLimitNs.
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ void record_error(int status) {
    atomicCAS(&g_device_error, 0, status);
}

// ------------------------------------------------------------------ formats --

// Two E2M1 codes in the low byte of `byte` (element 0 in the low nibble) ->
// f16x2 with element 0 in the low half.  Exact (E2M1 values are f16 values).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(r) : "r"(byte));
    return r;
}

// 4 code bytes (8 E2M1 values, element 2i in the low nibble of byte i) -> 4
// f16x2 (h[i] = elements 2i, 2i+1), exact.  The word is split into its bytes
// as a vector move, so the conversions read their bytes in place instead of
// after a shift and a truncation each.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t *h) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
}

// E4M3FN byte (low 8 bits) -> float.  Exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    uint32_t r;
    uint16_t b = (uint16_t)(byte & 0xFF);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(b));
    return __half2float(__ushort_as_half((unsigned short)(r & 0xFFFF)));
}

// float -> E4M3FN byte: round to nearest even, saturate to +-448, NaN -> 0x7F.
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFF;
}

// Two floats -> byte of two E2M1 codes (v0 in the low nibble): round to nearest
// even, saturate to +-6.  The sign bit of each code is the sign bit of its input
// (so -0 and negatives that round to zero give 0x8).
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float v0, float v1) {
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
        : "=h"(r) : "f"(v1), "f"(v0));
    uint32_t s = ((__float_as_uint(v0) >> 28) & 0x8u) | ((__float_as_uint(v1) >> 24) & 0x80u);
    return ((uint32_t)r & 0x77u) | s;
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ------------------------------------------------------------ async copies --

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Non-blocking test of phase `parity`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Test of phase `parity` that may suspend the thread for up to about
// kSuspendNs while the phase is incomplete.
constexpr uint32_t kSuspendNs = 128;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity), "n"(kSuspendNs) : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of an mbarrier, for at most g_wait_limit_ns.  `abort`
// is a CTA-shared flag: once any wait of the CTA has expired every later wait
// returns false at once, so all threads run to the end of the kernel (and
// through its barriers) instead of spinning.  Returns false on expiry/abort and
// records W4_ERR_TIMEOUT.  The limit is checked after every suspension that
// ended with the phase still incomplete; a limit shorter than one suspension
// (kSuspendNs) allows none, so the first wait that cannot pass at once expires.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long limit = g_wait_limit_ns;
    if (limit >= kSuspendNs) {
        const unsigned long long t0 = global_ns();
        for (;;) {
            if (mbar_try_wait(bar, parity)) return true;
            if (*abort) return false;
            if (global_ns() - t0 > limit) break;
        }
    } else if (*abort) {
        return false;
    }
    *abort = 1;
    record_error(W4_ERR_TIMEOUT);
    return false;
}

// Waits on barriers that another CTA of the cluster arrives on (a remote
// arrival, a multicast commit) take the same form as local ones: the arrival
// orders the arriving CTA's prior work, the wait acquires at CTA scope.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return mbar_wait(bar, parity, abort);
}

// Global -> shared bulk copy (no multicast), completion counted in bytes on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// L2 policy: streamed-once data (packed weights) is evicted first.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Programmatic dependent launch.  Both are no-ops when the kernel was not
// launched with the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_wait_prior_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// 2-D tiled TMA load (no multicast) of the box at (c0, c1) into shared memory,
// completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

// Wait as mbar_wait, but ignoring the CTA's abort flag and the settable limit
// (still bounded, by kWaitLimitNs): for the completions a CTA must see before it
// releases tensor memory or exits -- its own bulk copies and MMAs in flight.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) {
            record_error(W4_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// mbar_wait_bounded for barriers that another CTA of the cluster arrives on.
__device__ __forceinline__ bool mbar_wait_bounded_cluster(uint64_t *bar, uint32_t parity) {
    return mbar_wait_bounded(bar, parity);
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device.  The attribute belongs to the device's context, so the sizes
// already set are kept per (kernel, device), under a lock shared by all host
// threads.
inline bool set_smem_limit(const void *kernel, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lk(mu);
    size_t &cur = done[{kernel, dev}];
    if (bytes <= cur) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    cur = bytes;
    return true;
}

// Before a producer lane returns: wait for the copies it issued into a ring of
// `ns` stages whose fill count is `issued` (stage i went to slot i % ns with
// phase (i / ns) & 1), so that no copy is still writing shared memory when the
// CTA exits -- on the normal path these phases have long completed; after an
// aborted run the copies issued before the abort still land.
__device__ __forceinline__ void drain_ring(uint64_t *full, int ns, int issued) {
    for (int i = max(0, issued - ns); i < issued; i++) mbar_wait_bounded(full + (i % ns), (uint32_t)((i / ns) & 1));
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                    CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

inline PFN_encodeTiled get_encode_tiled() {
    static PFN_encodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
    }
    return fn;
}

}  // namespace w4
