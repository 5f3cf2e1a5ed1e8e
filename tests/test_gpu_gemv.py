"""CUDA GEMV vs the oracle's binary64 matmul: |y - y_ref| <= 1e-3 * sum|x w_hat|.

The packed weights given to the GPU are the oracle's own packing, so these
tests check the matmul alone."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4
from gpu_util import assert_within_tolerance, np_of

pytestmark = pytest.mark.gpu


def nvfp4_packed(W):
    c, s, g = O.pack_nvfp4(W)
    pw = W4.PackedWeights(W4.FMT_NVFP4, W.shape[1], W.shape[0], torch.from_numpy(c).cuda(),
                          torch.from_numpy(s).cuda(), torch.tensor([g], dtype=torch.float32).cuda())
    return pw, O.dequant_nvfp4(c, s, g)


def rocm_packed(W, fmt):
    b = O.pack_rocmfp4(W, fmt)
    return W4.PackedWeights(fmt, W.shape[1], W.shape[0], torch.from_numpy(b).cuda()), O.dequant_rocmfp4(b, fmt)


def run_and_check(pw, w_hat, x, flags=0):
    y = W4.w4a16_gemv(pw, x.cuda(), flags=flags)
    yr, ar = O.matmul(x, w_hat)
    assert_within_tolerance(np_of(y), yr, ar)
    return y


def test_nvfp4_small_case():
    W, x = I.nvfp4_small()
    pw, wh = nvfp4_packed(W)
    run_and_check(pw, wh, x)


@pytest.mark.parametrize("idx", range(5))
@pytest.mark.parametrize("M", [1, 4, 16])
def test_nvfp4_sweep(idx, M):
    K, N = I.SWEEP_SHAPES[idx]
    pw, wh = nvfp4_packed(I.sweep_weights(K, N, idx))
    run_and_check(pw, wh, I.sweep_x(M, K, idx))


@pytest.mark.parametrize("M", [2, 3, 5, 7, 8, 9, 12])
def test_nvfp4_other_m(M):
    pw, wh = nvfp4_packed(I.sweep_weights(9728, 2560, 4))
    run_and_check(pw, wh, I.sweep_x(M, 9728, 4))


@pytest.mark.parametrize("N,K", [(1, 256), (7, 512), (333, 2560), (149, 1024), (2, 9728), (1000, 256)])
@pytest.mark.parametrize("M", [1, 3, 16])
def test_nvfp4_ragged(N, K, M):
    pw, wh = nvfp4_packed(I.matrix("student_t4", N, K, N + K, 0.02, 1e-3))
    run_and_check(pw, wh, I.activations(M, K, 9 + M))


@pytest.mark.parametrize("fmt", [W4.FMT_ROCMFP4_DUAL, W4.FMT_ROCMFP4_FAST])
@pytest.mark.parametrize("M", [1, 8])
def test_rocm_laplace(fmt, M):
    W = I.rocm_weights()[:1536].contiguous()
    pw, wh = rocm_packed(W, fmt)
    run_and_check(pw, wh, I.rocm_x(M))


@pytest.mark.parametrize("fmt", [W4.FMT_ROCMFP4_DUAL, W4.FMT_ROCMFP4_FAST])
@pytest.mark.parametrize("N,K,M", [(1, 512, 1), (77, 1024, 2), (5, 9728, 16), (300, 2560, 4)])
def test_rocm_ragged(fmt, N, K, M):
    pw, wh = rocm_packed(I.matrix("laplace", N, K, N * 3 + K, 0.015, 1e-3), fmt)
    run_and_check(pw, wh, I.activations(M, K, 40 + M))


def test_outlier_activations_and_zero_weights():
    K, N = 2560, 512
    W = I.sweep_weights(K, N, 1)[:N].clone()
    W[:5] = 0
    pw, wh = nvfp4_packed(W.contiguous())
    x = I.activations(4, K, 3, outlier_cols=16, outlier_mult=30.0)
    y = run_and_check(pw, wh, x)
    assert torch.all(y[:, :5] == 0)


def test_deterministic_and_pdl_flag_and_graph():
    pw, wh = nvfp4_packed(I.sweep_weights(2560, 9728, 3))
    x = I.sweep_x(1, 2560, 3).cuda()
    y1 = W4.w4a16_gemv(pw, x)
    y2 = W4.w4a16_gemv(pw, x)
    y3 = W4.w4a16_gemv(pw, x, flags=W4.LAUNCH_PDL)
    assert torch.equal(y1, y2) and torch.equal(y1, y3)
    out = torch.empty_like(y1)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        W4.w4a16_gemv(pw, x, out=out, flags=W4.LAUNCH_PDL)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(3):
            W4.w4a16_gemv(pw, x, out=out, flags=W4.LAUNCH_PDL)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, y1)
    assert W4.w4_device_error(clear=True) == 0


@pytest.mark.parametrize("K", [16, 272, 288, 2576])
@pytest.mark.parametrize("M", [1, 5, 16])
def test_nvfp4_any_k(K, M):
    """K that is not a multiple of 256 takes the general path (binary64 sums)."""
    pw, wh = nvfp4_packed(I.matrix("student_t4", 37, K, K + M, 0.02, 1e-3))
    run_and_check(pw, wh, I.activations(M, K, 60 + M))


@pytest.mark.parametrize("fmt,K", [(W4.FMT_ROCMFP4_DUAL, 32), (W4.FMT_ROCMFP4_DUAL, 288),
                                   (W4.FMT_ROCMFP4_FAST, 256), (W4.FMT_ROCMFP4_FAST, 2592)])
@pytest.mark.parametrize("M", [1, 8])
def test_rocm_any_k(fmt, K, M):
    pw, wh = rocm_packed(I.matrix("laplace", 41, K, K + M, 0.015, 1e-3), fmt)
    run_and_check(pw, wh, I.activations(M, K, 70 + M))


def test_save_reload_in_fresh_process(tmp_path):
    """Pack on the GPU, write the bytes, reload them in a new process: the GEMV
    output there is bit-identical (fresh-process reload check)."""
    W = I.sweep_weights(2560, 1024, 1)
    x = I.sweep_x(1, 2560, 1)
    pw = W4.pack_nvfp4(W.cuda())
    y = W4.w4a16_gemv(pw, x.cuda())
    path = tmp_path / "packed.w4"
    W4.save_packed(pw, path)                     # versioned header + the packed bytes
    torch.save({"x": x, "y": y.cpu()}, tmp_path / "xy.pt")
    code = (
        "import torch, w4a16_matmul_pack_b200 as W4\n"
        f"pw = W4.load_packed({str(path)!r})\n"
        f"d = torch.load({str(tmp_path / 'xy.pt')!r})\n"
        "y = W4.w4a16_gemv(pw, d['x'].cuda()).cpu()\n"
        "assert torch.equal(y, d['y']), (y - d['y']).abs().max()\n"
    )
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    subprocess.run([sys.executable, "-c", code], check=True, cwd=root,
                   env={**os.environ, "PYTHONPATH": root})


@pytest.mark.parametrize("case", ["scaled_up", "scaled_down", "wide_range", "subnormal"])
@pytest.mark.parametrize("M", [1, 3, 12])
def test_activation_range_cases(case, M):
    """x far from 1 (the tensor-core path rescales x by a power of two) and x whose
    dynamic range no single power of two maps into f16 (the binary32 path)."""
    K, N = 2560, 512
    pw, wh = nvfp4_packed(I.sweep_weights(K, N, 1)[:N].contiguous())
    x = I.activations(M, K, 17 + M).double()
    if case == "scaled_up":
        x *= 2.0 ** 100
    elif case == "scaled_down":
        x *= 2.0 ** -100
    elif case == "wide_range":
        x[:, :8] *= 2.0 ** 40
        x[:, 8:16] *= 2.0 ** -40
    else:
        x[:, ::3] = 2.0 ** -130
    run_and_check(pw, wh, I.bf16_rne(x))


@pytest.mark.parametrize("case", ["zeros", "one_block", "range_2p30", "far_blocks", "inf"])
@pytest.mark.parametrize("K,N", [(2560, 300), (9728, 160)])
def test_single_token_block_exponents(case, K, N):
    """One token: x is converted per 16-k block with its own power of two, and a
    warp whose blocks it cannot all convert exactly falls back to binary32."""
    pw, wh = nvfp4_packed(I.sweep_weights(K, N, 3)[:N].contiguous())
    x = I.activations(1, K, 5).double()
    if case == "zeros":
        x[:] = 0.0
    elif case == "one_block":
        x[:] = 0.0
        x[:, 4 * 16:5 * 16] = I.activations(1, 16, 6).double()
    elif case == "range_2p30":          # inside one block: still exact in f16 after scaling
        x[:, 16:24] *= 2.0 ** 15
        x[:, 24:32] *= 2.0 ** -15
    elif case == "far_blocks":          # blocks of one warp 2^120 apart
        x[:, :16] *= 2.0 ** 60
        x[:, 16:32] *= 2.0 ** -60
    else:
        x[:, 100] = float("inf")
    x = I.bf16_rne(x)
    y = np_of(W4.w4a16_gemv(pw, x.cuda()))
    yr, ar = O.matmul(x, wh)
    if case == "inf":
        # every row with a nonzero weight at k = 100 is +-inf or nan on both sides
        assert np.array_equal(np.isfinite(y), np.isfinite(yr))
        fin = np.isfinite(yr)
        assert_within_tolerance(y[fin], yr[fin], ar[fin])
    else:
        assert_within_tolerance(y, yr, ar)


def check_group(pws, whs, xs, flags=0):
    ys = W4.w4a16_gemv_grouped(pws, [x.cuda() for x in xs], flags=flags)
    for y, wh, x in zip(ys, whs, xs):
        yr, ar = O.matmul(x, wh)
        assert_within_tolerance(np_of(y), yr, ar)
    return ys


def test_grouped_sweep():
    """The five sweep matrices, each with its own x, in one launch."""
    pws, whs, xs = [], [], []
    for idx, (K, N) in enumerate(I.SWEEP_SHAPES):
        pw, wh = nvfp4_packed(I.sweep_weights(K, N, idx))
        pws.append(pw); whs.append(wh); xs.append(I.sweep_x(1, K, idx))
    check_group(pws, whs, xs)
    check_group(pws, whs, xs, flags=W4.LAUNCH_PDL)


def test_grouped_shared_x_and_ragged():
    """q, k, v reading one x; then ragged shapes (1 row, fewer rows than CTAs, K = 256)."""
    K = 2560
    mats = [nvfp4_packed(I.sweep_weights(K, N, 30 + i)[:N].contiguous()) for i, N in enumerate((4096, 1024, 1024))]
    x = I.activations(1, K, 31)
    check_group([m[0] for m in mats], [m[1] for m in mats], [x, x, x])
    shapes = [(256, 7), (1024, 149), (2560, 333), (9728, 2), (512, 1), (4096, 4096)]
    pws, whs, xs = [], [], []
    for i, (K, N) in enumerate(shapes):
        pw, wh = nvfp4_packed(I.sweep_weights(K, N, 40 + i)[:N].contiguous())
        pws.append(pw); whs.append(wh); xs.append(I.activations(1, K, 50 + i))
    check_group(pws, whs, xs)


def test_grouped_eight_and_graph():
    """The largest group; replayed in a CUDA graph with PDL it gives the same bits."""
    shapes = [(2560, 1024)] * 4 + [(4096, 512)] * 2 + [(1024, 2048), (9728, 256)]
    pws, whs, xs = [], [], []
    for i, (K, N) in enumerate(shapes):
        pw, wh = nvfp4_packed(I.sweep_weights(K, N, 60 + i)[:N].contiguous())
        pws.append(pw); whs.append(wh); xs.append(I.activations(1, K, 70 + i))
    ref = [y.clone() for y in check_group(pws, whs, xs)]
    xd = [x.cuda() for x in xs]
    outs = [torch.empty(1, w.N, device="cuda") for w in pws]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        W4.w4a16_gemv_grouped(pws, xd, outs=outs, flags=W4.LAUNCH_PDL)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        W4.w4a16_gemv_grouped(pws, xd, outs=outs, flags=W4.LAUNCH_PDL)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(ref, outs):
        assert torch.equal(a, b)


def test_grouped_argument_errors():
    pw, _ = nvfp4_packed(I.sweep_weights(256, 16, 80)[:16].contiguous())
    x = I.activations(1, 256, 81).cuda()
    with pytest.raises(W4.W4Error):
        W4.w4a16_gemv_grouped([pw] * 9, [x] * 9)
    with pytest.raises(W4.W4Error):
        W4.w4a16_gemv_grouped([pw], [x], flags=2)
    pr = W4.pack_rocmfp4(I.matrix("laplace", 16, 256, 82, 0.015, 0.0, device="cuda"), "dual")
    with pytest.raises(W4.W4Error):
        W4.w4a16_gemv_grouped([pr], [x])


def huge_range_case(case, M, K, seed):
    """x (and W) scaled so that the binary64 y is finite in binary32 while the
    kernels' internal sums, taken without the global scale g, would not be:
    rows of x at 2^110..2^125, or weights near 2^100 against x near 2^-110."""
    W = I.sweep_weights(K, 512, 1)[:512].double()
    x = I.activations(M, K, seed).double()
    if case == "x_2p110":
        x *= 2.0 ** 110
    elif case == "x_2p118":
        x *= 2.0 ** 118
    elif case == "x_2p125_sparse":          # few nonzero x so that y stays below 2^128
        keep = torch.zeros(K, dtype=torch.bool)
        keep[::160] = True
        x[:, ~keep] = 0.0
        x *= 2.0 ** 125
    elif case == "w_2p100_x_2pm110":
        W *= 2.0 ** 100
        x *= 2.0 ** -110
    return I.bf16_rne(W), I.bf16_rne(x)


HUGE_CASES = ["x_2p110", "x_2p118", "x_2p125_sparse", "w_2p100_x_2pm110"]


@pytest.mark.parametrize("case", HUGE_CASES)
@pytest.mark.parametrize("M", [1, 4, 16])
def test_huge_range_outputs(case, M):
    """The global scale is applied together with the power of two that undoes x's
    rescaling, so outputs near the top (and bottom) of binary32's range are finite
    and within the bound (M = 1, the skinny kernel, and split-K at M = 16)."""
    for K in (2560, 9728):
        W, x = huge_range_case(case, M, K, 300 + M)
        pw, wh = nvfp4_packed(W.contiguous())
        yr, ar = O.matmul(x, wh)
        assert np.all(np.abs(yr) < 3.0e38) and np.all(np.isfinite(ar))
        if case == "x_2p118":
            # without g the sums reach y / g: above binary32's range here
            assert float(np.max(np.abs(yr))) / float(pw.global_scale.item()) > 3.5e38
        run_and_check(pw, wh, x)


@pytest.mark.parametrize("case", HUGE_CASES)
def test_huge_range_grouped(case):
    pws, whs, xs = [], [], []
    for i, K in enumerate((2560, 4096, 9728)):
        W, x = huge_range_case(case, 1, K, 320 + i)
        pw, wh = nvfp4_packed(W.contiguous())
        pws.append(pw); whs.append(wh); xs.append(x)
    check_group(pws, whs, xs)


@pytest.mark.parametrize("M", [1, 4, 9])
def test_x_conversion_paths_agree(M):
    """x whose every value converts to f16 as it is takes the one-barrier
    conversion with no power of two (up to 8 tokens); the same x times 2^20
    exceeds f16 and takes the conversion with a power of two.  A power of two
    scales every product and partial sum exactly, so the two outputs must differ
    by exactly 2^20, and both meet the oracle's bound.  x holding the edges of
    the unscaled range (2^-17, 65280), or values just outside it (2^-18, 65536),
    must meet it too."""
    K, N = 2560, 512
    pw, wh = nvfp4_packed(I.sweep_weights(K, N, 4)[:N].contiguous())
    x = I.activations(M, K, 41 + M)
    y = run_and_check(pw, wh, x)
    y_big = run_and_check(pw, wh, I.bf16_rne(x.double() * 2.0 ** 20))
    assert torch.equal(y_big, y * 2.0 ** 20)
    for lo, hi in ((2.0 ** -17, 65280.0), (2.0 ** -18, 65536.0)):
        xe = x.double().clone()
        xe[:, 7], xe[:, 8], xe[:, 9], xe[:, 10] = lo, -lo, hi, -hi
        run_and_check(pw, wh, I.bf16_rne(xe))


def test_grouped_x_conversion_paths_agree():
    """The grouped one-token launch: the same two conversions, the same exact 2^20."""
    K, N = 2560, 512
    pw, wh = nvfp4_packed(I.sweep_weights(K, N, 5)[:N].contiguous())
    x = I.activations(1, K, 43)
    xb = I.bf16_rne(x.double() * 2.0 ** 20)
    y, y_big = W4.w4a16_gemv_grouped([pw, pw], [x.cuda(), xb.cuda()])
    yr, ar = O.matmul(x, wh)
    assert_within_tolerance(np_of(y), yr, ar)
    assert torch.equal(y_big, y * 2.0 ** 20)
