/*
 * w4a16.h -- C ABI of the W4A16 pack + matmul library (libw4a16.so, sm_100a).
 *
 * Block-scaled 4-bit weight-only linear layers: pack BF16 weight matrices to
 * NVFP4 or ROCmFP4, then multiply BF16 activations by the packed weights.
 *
 * Sources (web pages on the subject):
 *   [EdgeRock]  "EdgeRock-4B-NVFP4" model card, intro: the W4A16 NVFP4 format --
 *               E2M1 4-bit weights, one FP8 E4M3 scale per 16 values and one
 *               FP32 global scale per matrix; activations stay BF16.
 *   [Nanbeige]  "Nanbeige4.2-3B-NVFP4A16" card, Creation: data-free
 *               round-to-nearest quantisation, group 16; Serving: the fused
 *               W4A16 kernel is the batch-1 decode path.
 *   [rocmwhy]   "rocmwhy" ROCmFP4 research page, sections 01-03 and the format
 *               table: Codebook10 levels 0,+-1,+-2,+-3,+-4,+-6,+-8,+-10; Dual
 *               blocks (32 weights, two unsigned E4M3 half scales, 18 bytes,
 *               4.50 bits/weight) and FAST blocks (one scale, 17 bytes, 4.25
 *               bits/weight); scales chosen by exhaustive search over the
 *               finite UE4M3 candidates scored by reconstruction error.
 *
 * Conventions shared by every entry point
 *   - Matrices are "K-major": logical weight W is K x N (y = x . W) and is
 *     stored as rows n = 0..N-1 of K contiguous elements, like the weight of a
 *     torch Linear layer.  x is M x K row-major BF16, y is M x N row-major.
 *   - Every pointer argument is caller-owned DEVICE memory (cudaMalloc or
 *     equivalent) unless stated otherwise.  The library never allocates; the
 *     scratch an operation needs is passed in as `workspace` (size from the
 *     matching *_workspace_bytes query).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it: arguments are validated on the host first and an
 *     error is returned before anything is launched; a launch failure returns
 *     W4_ERR_CUDA.  Device-side conditions (non-finite input, a bounded wait
 *     that expired) are reported through `d_status` where the call has one,
 *     and always through the sticky word read by w4_device_error().
 *   - Device pointers must be 16-byte aligned (W4_ERR_ALIGN otherwise).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4_OK = 0,
    W4_ERR_ARG = 1,          /* bad size, null pointer, bad enum */
    W4_ERR_ALIGN = 2,        /* a pointer is not 16-byte aligned */
    W4_ERR_UNSUPPORTED = 3,  /* valid request this build does not implement */
    W4_ERR_CUDA = 4,         /* a CUDA call or launch failed */
    W4_ERR_NONFINITE = 5,    /* NaN or Inf in a matrix given to a packer */
    W4_ERR_TIMEOUT = 6,      /* a bounded device-side wait expired */
    W4_ERR_WORKSPACE = 7     /* workspace missing or smaller than required */
} w4_status;

typedef enum {
    W4_FMT_NVFP4 = 1,         /* [EdgeRock] E2M1 + E4M3 per 16 + FP32 global */
    W4_FMT_ROCMFP4_DUAL = 2,  /* [rocmwhy] 18-byte blocks, two half scales   */
    W4_FMT_ROCMFP4_FAST = 3,  /* [rocmwhy] 17-byte blocks, one scale         */
    W4_FMT_Q4_0 = 4           /* [rocmwhy] table: stock Q4_0, for comparison  */
} w4_format;

typedef enum {
    W4_SCALE_ABSMAX = 0,  /* NVFP4 round-to-nearest abs-max recipe */
    W4_SCALE_MSE = 1      /* exhaustive finite-scale error search */
} w4_scale_search;

/*
 * A packed weight matrix (all pointers device memory, owned by the caller).
 *   NVFP4:   codes  = [N][K/2] bytes; element k of row n sits in byte k/2, the
 *                     even element in the low nibble.  Nibble = E2M1 code (bit 3
 *                     sign, bits 2..1 exponent with bias 1, bit 0 mantissa).
 *            scales = [N][K/16] E4M3FN bytes (one per 16 consecutive k).
 *            global_scale = one float.  w_hat = e2m1 * scale * global.
 *   ROCmFP4: codes  = [N][K/32] blocks of 18 (Dual) or 17 (FAST) bytes, blocks
 *                     contiguous along K.  Dual block: byte 0 = scale of
 *                     elements 0..15, byte 1 = scale of 16..31; FAST block:
 *                     byte 0 = scale of all 32.  Then 16 code bytes, byte j =
 *                     code[j] | code[j+16] << 4.  Code = Codebook10 nibble (bit
 *                     3 sign, bits 2..0 index into 0,1,2,3,4,6,8,10).  Scale =
 *                     unsigned E4M3 byte 0x00..0x7E.  w_hat = level * scale.
 *            scales = NULL, global_scale = NULL.
 *   Q4_0:    codes  = [N][K/32] blocks of 18 bytes: the FP16 scale d (little
 *                     endian), then 16 code bytes, byte j = code[j] |
 *                     code[j+16] << 4; w_hat = d * (code - 8).  A comparison
 *                     format: packed and scored (w4_reconstruction_error), not
 *                     accepted by the matmuls (W4_ERR_UNSUPPORTED).
 *            scales = NULL, global_scale = NULL.
 */
typedef struct {
    int fmt;                     /* w4_format */
    int K;                       /* reduction length (input features) */
    int N;                       /* output features */
    const uint8_t *codes;
    const uint8_t *scales;
    const float *global_scale;
} w4_weights;

/* ---------------------------------------------------------------- packers -- */

/*
 * pack_nvfp4 -- quantise a BF16 matrix to NVFP4 ([EdgeRock] intro; the
 * round-to-nearest recipe of [Nanbeige] Creation):
 *   global g = absmax(W) / (6 * 448)                      (binary32)
 *   block scale s = E4M3(absmax(block) / 6 / g)           (two binary32 divisions,
 *                                                          round to nearest even,
 *                                                          saturate at 448)
 *   code = E2M1(x / (s * g))                              (binary32, nearest even,
 *                                                          saturate at 6, sign kept)
 * g == 0, or a block whose s * g is 0, gives all-zero scales and codes.
 *   W            [N][K] BF16, K % 16 == 0, K >= 16, N >= 1.
 *   block        must be 16.
 *   scale_search W4_SCALE_ABSMAX as above, or W4_SCALE_MSE: g as above, and
 *                each block scale chosen by search over the E4M3 codes
 *                u = 0x00..0x7E (the [rocmwhy] section 03 recipe applied to
 *                NVFP4 blocks): under u, d = dec(u) * g, each code is
 *                E2M1(x / d) as above, r = e2m1 * d, and the block error
 *                E(u) = sum fma(x - r, x - r, E) over k in order, binary32;
 *                the smallest E wins, ties to the smaller code.  The abs-max
 *                scale is one of the candidates, so the error never grows.
 *   codes        out [N][K/2];  scales out [N][K/16];  global_scale out float.
 *   workspace    >= pack_nvfp4_workspace_bytes() bytes of device scratch.
 *   d_status     optional device int: set to W4_OK at the start of the call,
 *                W4_ERR_NONFINITE if W holds NaN/Inf (outputs then undefined).
 */
w4_status pack_nvfp4(const void *W, int K, int N, int block, int scale_search,
                     uint8_t *codes, uint8_t *scales, float *global_scale,
                     void *workspace, size_t workspace_bytes, int *d_status,
                     void *stream);

/*
 * pack_nvfp4_ex -- pack_nvfp4 with importance weights for the scale search
 * ([rocmwhy] section 03: candidates scored by reconstruction error "with
 * optional importance weighting").
 *   importance  NULL, or device float[K]: one weight w_k per input channel,
 *               finite and >= 0 (otherwise d_status = W4_ERR_NONFINITE and the
 *               outputs are undefined); requires scale_search = W4_SCALE_MSE
 *               (W4_ERR_ARG otherwise).  The block error becomes
 *               E(u) = sum fma(w_k * (x - r), x - r, E); w = 1 gives exactly
 *               the unweighted bytes.
 */
w4_status pack_nvfp4_ex(const void *W, int K, int N, int block, int scale_search,
                        const float *importance, uint8_t *codes, uint8_t *scales,
                        float *global_scale, void *workspace, size_t workspace_bytes,
                        int *d_status, void *stream);
size_t pack_nvfp4_workspace_bytes(void);

/*
 * pack_rocmfp4 -- quantise a BF16 matrix to ROCmFP4 Dual or FAST ([rocmwhy]
 * sections 01-03).  For each scale group (16-weight half for Dual, the whole
 * 32-weight block for FAST) every finite UE4M3 code u = 0x00..0x7E is tried:
 * each weight takes the nearest Codebook10 level at scale dec(u) (ties to the
 * even level index), and the group error E(u) = sum fma(d, d, E) over the
 * weights in k order, d = x - level * dec(u), binary32.  The smallest E wins,
 * ties to the smaller code.
 *   W        [N][K] BF16, K % 32 == 0.
 *   block    must be 32.  fmt = W4_FMT_ROCMFP4_DUAL or W4_FMT_ROCMFP4_FAST.
 *   importance NULL, or device float[K]: one weight w_k per input channel
 *            ([rocmwhy] section 03, "optional importance weighting"), finite
 *            and >= 0 (otherwise d_status = W4_ERR_NONFINITE, outputs
 *            undefined); the error becomes E(u) = sum fma(w_k * d, d, E), and
 *            w = 1 gives exactly the unweighted bytes.
 *   blocks   out [N][K/32][18 | 17] (layout as in w4_weights).
 *   d_status optional, as for pack_nvfp4.
 */
w4_status pack_rocmfp4(const void *W, int K, int N, int block, int fmt,
                       const float *importance, uint8_t *blocks, int *d_status,
                       void *stream);

/*
 * pack_q4_0 -- stock Q4_0, the pages' comparison format ([rocmwhy] format
 * table: 32 weights, evenly spaced integers, one FP16 scale, 18-byte blocks,
 * "signed abs-max" reference scale; section 02's lab: the outlier 8.2 gives the
 * shared scale 1.025 = 8.2 / 8).  Per 32-weight block: m = the weight of
 * largest magnitude (the first in k order on ties), d = FP16(m / -8) (binary32
 * division, then nearest even, saturating at 65504), code = the nearest
 * integer (ties to even) of x / d in binary32, clamped to [-8, 7], plus 8;
 * d == 0 gives codes 8.
 *   W        [N][K] BF16, K % 32 == 0.  block must be 32.
 *   blocks   out [N][K/32][18] (layout as in w4_weights).
 *   d_status optional, as for pack_nvfp4.
 */
w4_status pack_q4_0(const void *W, int K, int N, int block, uint8_t *blocks, int *d_status,
                    void *stream);

/*
 * w4_reconstruction_error -- how well a packed matrix reproduces its source:
 * out[0] = sum over all weights of (W - w_hat)^2, out[1] = sum of W^2, both in
 * binary64 (w_hat exact in binary64 for every format), summed in a fixed order
 * (the same bits on every call).  Any w4_format, including W4_FMT_Q4_0.
 *   W          [N][K] BF16, the matrix w was packed from.
 *   out        device double[2].
 *   workspace  >= w4_reconstruction_workspace_bytes() bytes of device scratch.
 */
w4_status w4_reconstruction_error(const w4_weights *w, const void *W, double *out, void *workspace,
                                  size_t workspace_bytes, void *stream);
size_t w4_reconstruction_workspace_bytes(void);

/* ---------------------------------------------------------------- matmul --- */

/*
 * w4a16_gemv -- y[M][N] = x[M][K] . w_hat, fused dequantise-and-multiply for
 * decode-sized M ([Nanbeige] Serving: the W4A16 kernel a decode step spends its
 * weight bandwidth on).  NVFP4: products on the tensor cores from f16 operands
 * (e2m1 * scale is exact in f16; x is rescaled by powers of two into f16's range,
 * with a binary32 CUDA-core path for x that does not convert exactly), binary32
 * accumulation; the global scale and the power of two are applied together at
 * the end in binary64, so the output is finite whenever the exact result is.
 * ROCmFP4: level * scale products in binary32.  The result is deterministic (a
 * fixed summation order for a given shape and M).
 *   w        packed NVFP4 or ROCmFP4 weights (Q4_0: W4_ERR_UNSUPPORTED), any K
 *            the packers accept.  K % 256 == 0 (NVFP4, ROCmFP4 Dual) or
 *            K % 512 == 0 (ROCmFP4 FAST) takes the tensor-core kernels (every
 *            row piece they copy starts on 16 bytes); other K take a general
 *            CUDA-core path (one warp per row, binary64 sums, no workspace).
 *   x        [M][K] BF16, 1 <= M <= 16.
 *   y        out [M][N] float.
 *   workspace>= w4a16_workspace_bytes(w, M) bytes (0 for most shapes: NULL
 *            allowed then); the split-K partial sums of long K at large M.
 */
w4_status w4a16_gemv(const w4_weights *w, const void *x, int M, float *y,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4a16_gemv_ex -- w4a16_gemv with launch flags.  W4_LAUNCH_PDL launches the
 * kernel with programmatic dependent launch: it may start streaming weights
 * while the previous kernel on the stream is still running, and reads x only
 * after that kernel has completed.  Use inside a captured CUDA graph of
 * back-to-back layers.  Any other bit returns W4_ERR_ARG.
 */
#define W4_LAUNCH_PDL 1u
w4_status w4a16_gemv_ex(const w4_weights *w, const void *x, int M, float *y,
                        void *workspace, size_t workspace_bytes, unsigned flags,
                        void *stream);

/*
 * w4a16_gemv_grouped -- G independent one-token NVFP4 GEMVs in one launch:
 * y[p][N_p] = x[p][K_p] . w_hat[p] for p < G (the decode GEMV of the
 * "Nanbeige4.2-3B-NVFP4A16" card, Serving, applied to several weight matrices
 * that are ready together: the q, k and v projections of a layer read the same
 * x, as do gate and up).  The SMs are shared out among the problems so
 * that the most heavily loaded CTA (a CTA works on whole 16-row tiles) carries
 * as few bytes as possible, and small matrices do not each pay a launch and a
 * pipeline fill.
 *   w      array of G NVFP4 weights (K_p % 256 == 0, K_p <= 32768).
 *   x      array of G device pointers to [K_p] BF16 (may repeat).
 *   y      array of G device pointers to [N_p] float (must not overlap).
 *   G      1..8.
 *   flags  0 or W4_LAUNCH_PDL.
 * The arrays are read on the host before the call returns; no workspace.
 * Errors: W4_ERR_ARG (null pointers, G out of range, unknown flags),
 * W4_ERR_ALIGN, W4_ERR_UNSUPPORTED (format or K), W4_ERR_CUDA.
 */
w4_status w4a16_gemv_grouped(const w4_weights *w, const void *const *x, float *const *y, int G,
                             unsigned flags, void *stream);

/*
 * w4_plan_grouped -- host only (no CUDA call): the CTAs w4a16_gemv_grouped
 * gives each problem on a GPU with `sms` SMs.  With T_p 16-row tiles of b_p
 * packed bytes, ctas[p] = ceil(T_p / floor(L / b_p)) for the smallest load L
 * (bytes of the heaviest CTA) whose total fits in `sms`; the SMs left over go
 * one at a time to the problem with the most bytes per CTA.  At least 1 and at
 * most T_p each; the total is min(sms, sum of T_p) unless G forces more.
 *   w, G, flags  as for w4a16_gemv_grouped.  ctas  out int[G].
 */
w4_status w4_plan_grouped(const w4_weights *w, int G, int sms, unsigned flags, int *ctas);

/*
 * w4a16_gemm -- y = x . w_hat for prefill-sized M on the 5th-generation tensor
 * cores (tcgen05.mma kind::f16, binary32 accumulators in tensor memory).  The
 * packed NVFP4 tiles are dequantised (e2m1 * scale, exact in f16 and in BF16)
 * by CUDA-core warps straight into tensor memory, where they are the MMA's A
 * operand; x tiles (the B operand) are staged in shared memory by TMA.  The
 * epilogue applies the global scale (and the per-row power of two below) in
 * binary64 and writes binary32 and/or BF16 (round to nearest even).
 * Operands per 192-token tile: with a workspace, x_to_f16 first writes each
 * token row as f16 x * 2^-sigma_m (exact for rows whose range fits f16); tiles
 * whose rows all converted exactly run on f16 operands, any other tile (and
 * every tile without a workspace) on BF16 operands, with g's power of two
 * folded into the weights.
 *   w        NVFP4 weights, K % 64 == 0 (W4_ERR_UNSUPPORTED otherwise; ROCmFP4
 *            and Q4_0 are W4_ERR_UNSUPPORTED too).
 *   x        [M][K] BF16, M >= 1.
 *   y_f32    out [M][N] float, or NULL;  y_bf16 out [M][N] BF16, or NULL
 *            (at least one of the two).
 *   workspace NULL, or >= w4a16_workspace_bytes(w, M) bytes: the f16 copy of x
 *            and two ints per row (smaller or NULL: BF16 operands throughout).
 */
w4_status w4a16_gemm(const w4_weights *w, const void *x, int M, float *y_f32,
                     void *y_bf16, void *workspace, size_t workspace_bytes,
                     void *stream);

/* Scratch bytes w4a16_gemv / w4a16_gemm need for this shape (0 if none). */
size_t w4a16_workspace_bytes(const w4_weights *w, int M);

/*
 * w4a16_gemv_noalloc -- w4a16_gemv for callers that cannot allocate device
 * memory (for example a plugin whose host framework owns every device
 * allocation, or an embedded runtime with a fixed memory budget): the same
 * computation, but the split-K scratch comes from a device array built into
 * the library instead of a caller-provided workspace.  The pages have no
 * counterpart to this entry point; it only changes where scratch lives.
 *   w, x, M, y, stream  as for w4a16_gemv (x, y and the packed weights are still
 *                       caller-owned device memory).
 *   Returns W4_ERR_WORKSPACE, before launching anything, when the shape needs
 *   more than W4_NOALLOC_SCRATCH_BYTES of scratch (w4a16_workspace_bytes).
 * The array (W4_NOALLOC_SCRATCH_BYTES) is held by every GPU that loads the
 * library until the process exits.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current) and
 * caches it; make that first call before any stream capture.  All calls on a
 * device share the array: calls whose work overlaps on the GPU race and must
 * be serialised by the caller.  Every scratch value a call reads is written
 * earlier in the same call, so no clearing is needed between calls.  The cached
 * address belongs to the device's current context: after cudaDeviceReset (or
 * with another primary context on that device) it is stale, so the library must
 * not be used across a reset in one process.
 */
#define W4_NOALLOC_SCRATCH_BYTES (8u << 20)
w4_status w4a16_gemv_noalloc(const w4_weights *w, const void *x, int M, float *y, void *stream);

/* ------------------------------------------------------------- utilities --- */

/*
 * w4_encode_scalars -- the binary32 -> E4M3 (saturating, nearest even) and
 * binary32 -> E2M1 (saturating, nearest even, sign kept) conversions the packers
 * use, applied elementwise: e4m3[i] = E4M3(v[i]), e2m1[i] = E2M1(v[i]) (low
 * nibble).  For checking conversions; v, e4m3, e2m1 are device arrays of n.
 */
w4_status w4_encode_scalars(const float *v, size_t n, uint8_t *e4m3, uint8_t *e2m1,
                            void *stream);

/*
 * w4_device_error -- read (and, if clear != 0, reset) the library's sticky
 * device error word on the current device: 0, or the w4_status of the first
 * device-side failure (W4_ERR_TIMEOUT, W4_ERR_NONFINITE) since the last reset.
 * Synchronises the device.
 */
w4_status w4_device_error(int *out, int clear);

/*
 * w4_set_wait_limit -- limit, in nanoseconds, of the device-side waits that
 * gate a kernel's progress (a consumer waiting for its data, a producer for a
 * free buffer), on the current device; 0 restores the default of 2 s.  When
 * such a wait expires the kernel records W4_ERR_TIMEOUT in the sticky word
 * (w4_device_error), every other wait of its CTA returns at once, and the CTA
 * runs to its end: before exiting it still waits (up to 2 s, whatever this
 * limit) for the copies and MMAs it has already issued, so no asynchronous
 * write outlives it.  The outputs of a call whose wait expired are undefined.
 * A wait that cannot pass at once suspends the thread in steps of about
 * 128 ns; a limit below that step expires the first such wait.  Meant for
 * exercising that failure path (a short limit makes the first waits expire);
 * it applies to kernels launched after it returns.  Synchronous.
 */
w4_status w4_set_wait_limit(unsigned long long ns);

/* Human-readable name of a status code. */
const char *w4_status_string(int status);

/* Library version string. */
const char *w4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
