"""CUDA tcgen05 GEMM vs the oracle's binary64 matmul.

float32 output: |y - y_ref| <= 1e-3 * sum|x w_hat|.  BF16 output: the same
bound plus half a BF16 unit in the last place of y_ref (the rounding of the
result itself)."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4
from gpu_util import assert_within_tolerance, np_of

pytestmark = pytest.mark.gpu


def packed(W):
    c, s, g = O.pack_nvfp4(W)
    pw = W4.PackedWeights(W4.FMT_NVFP4, W.shape[1], W.shape[0], torch.from_numpy(c).cuda(),
                          torch.from_numpy(s).cuda(), torch.tensor([g], dtype=torch.float32).cuda())
    return pw, (c, s, g)


def half_ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -133)))
    return np.where(a > 0, 2.0 ** (e - 8), 2.0 ** -134)


def check(pw, cs, x, rows=None, workspace=None):
    c, s, g = cs
    y32, y16 = W4.w4a16_gemm(pw, x.cuda(), workspace=workspace)
    torch.cuda.synchronize()
    y32, y16 = np_of(y32), np_of(y16.float())
    N = pw.N
    rows = np.arange(N) if rows is None else np.asarray(rows)
    wh = np.concatenate([O.dequant_nvfp4(c, s, g, int(r), 1) for r in rows])
    yr, ar = O.matmul(x, wh)
    assert_within_tolerance(y32[:, rows], yr, ar)
    err16 = np.abs(y16[:, rows] - yr)
    bound16 = 1e-3 * ar + half_ulp_bf16(yr)
    assert np.all(err16 <= bound16), float((err16 - bound16).max())


def test_prefill_full_size_sampled_rows():
    W, x = I.prefill()
    pw, cs = packed(W)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([np.arange(0, 130), np.arange(9600, 9728), rng.integers(0, 9728, 64)]))
    check(pw, cs, x, rows)


@pytest.mark.parametrize("M,N,K", [(256, 128, 64), (300, 200, 128), (1, 77, 640), (16, 1000, 2560),
                                   (513, 384, 1024), (2048, 256, 256)])
def test_ragged_shapes(M, N, K):
    W = I.matrix("student_t4", N, K, M + N + K, 0.02, 1e-3)
    x = I.activations(M, K, 7, outlier_cols=min(16, K // 8))
    pw, cs = packed(W)
    check(pw, cs, x)


def test_repeatable():
    W = I.matrix("student_t4", 512, 1024, 3, 0.02, 1e-3)
    x = I.activations(512, 1024, 4).cuda()
    pw, _ = packed(W)
    a = W4.w4a16_gemm(pw, x)[0].clone()
    b = W4.w4a16_gemm(pw, x)[0]
    assert torch.equal(a, b)
    assert W4.w4_device_error(clear=True) == 0


def test_unsupported_inputs():
    W = I.matrix("normal", 64, 96, 1, 0.02)
    pw, _ = packed(W)
    with pytest.raises(W4.W4Error) as e:
        W4.w4a16_gemm(pw, I.activations(4, 96, 1).cuda())
    assert e.value.status == 3
    # ROCmFP4 rows must be whole 16-byte pieces: K % 256 (Dual), K % 512 (FAST)
    for fmt, K in ((O.FMT_DUAL, 128), (O.FMT_FAST, 256)):
        b = O.pack_rocmfp4(I.matrix("laplace", 64, K, 2, 0.015), fmt)
        pr = W4.PackedWeights(fmt, K, 64, torch.from_numpy(b).cuda())
        with pytest.raises(W4.W4Error) as e:
            W4.w4a16_gemm(pr, I.activations(4, K, 1).cuda())
        assert e.value.status == 3


def rocm_check(fmt, W, x, rows=None, workspace=None):
    b = O.pack_rocmfp4(W, fmt)
    pr = W4.PackedWeights(fmt, W.shape[1], W.shape[0], torch.from_numpy(b).cuda())
    y32, y16 = W4.w4a16_gemm(pr, x.cuda(), workspace=workspace)
    torch.cuda.synchronize()
    y32, y16 = np_of(y32), np_of(y16.float())
    rows = np.arange(W.shape[0]) if rows is None else np.asarray(rows)
    wh = np.concatenate([O.dequant_rocmfp4(b, fmt, int(r), 1) for r in rows])
    yr, ar = O.matmul(x, wh)
    assert_within_tolerance(y32[:, rows], yr, ar)
    err16 = np.abs(y16[:, rows] - yr)
    assert np.all(err16 <= 1e-3 * ar + half_ulp_bf16(yr)), float((err16 - 1e-3 * ar - half_ulp_bf16(yr)).max())


@pytest.mark.parametrize("fmt", [O.FMT_DUAL, O.FMT_FAST])
@pytest.mark.parametrize("with_workspace", [True, False])
def test_rocm_prefill_full_size_sampled_rows(fmt, with_workspace):
    """ROCmFP4 prefill GEMM on the 2560 x 9728 Laplace matrix, 2048 tokens with 16
    outlier channels: f16 operands (x rescaled per row, with the workspace) and
    BF16 operands (without); every token, sampled weight rows incl. both edges."""
    W = I.rocm_weights()
    _, x = I.prefill()
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([np.arange(0, 130), np.arange(9600, 9728), rng.integers(0, 9728, 48)]))
    ws = None if with_workspace else torch.empty(0, dtype=torch.uint8, device="cuda")
    rocm_check(fmt, W, x, rows, ws)


@pytest.mark.parametrize("fmt", [O.FMT_DUAL, O.FMT_FAST])
@pytest.mark.parametrize("M,N,K", [(1, 77, 512), (300, 200, 1024), (513, 384, 2048), (2048, 136, 512)])
def test_rocm_ragged_shapes(fmt, M, N, K):
    W = I.matrix("laplace", N, K, M + N + K, 0.015, 1e-3)
    x = I.activations(M, K, 8, outlier_cols=min(16, K // 8))
    rocm_check(fmt, W, x)


def test_rocm_operand_modes_per_token_tile():
    M, N, K = 600, 256, 1024
    W = I.matrix("laplace", N, K, 21, 0.015, 1e-3)
    x = I.activations(M, K, 22, outlier_cols=16).double()
    x[300, :8] *= 2.0 ** 40            # token tile 1: BF16 operands
    x[300, 8:16] *= 2.0 ** -40
    x[520:530] *= 2.0 ** 100           # token tile 2: large, exact after scaling
    rocm_check(O.FMT_DUAL, W, I.bf16_rne(x))
    rocm_check(O.FMT_FAST, W, I.bf16_rne(x))


def test_operand_modes_per_token_tile():
    """Token tiles whose rows convert exactly to f16 (after a power-of-two scale per
    row) run on f16 operands; a tile holding a row with a wider range than f16 can
    represent runs on BF16 operands.  Both meet the bound, in one call."""
    M, N, K = 600, 256, 1024
    W = I.matrix("student_t4", N, K, 11, 0.02, 1e-3)
    x = I.activations(M, K, 12, outlier_cols=16).double()
    x[300, :8] *= 2.0 ** 40            # token tile 1: not exact in f16 -> BF16 operands
    x[300, 8:16] *= 2.0 ** -40
    x[520:530] *= 2.0 ** 100           # token tile 2: large but exact after scaling
    x[540:545] *= 2.0 ** -100
    x[560] = 0.0
    pw, cs = packed(W)
    check(pw, cs, I.bf16_rne(x))


def test_bf16_operands_without_workspace():
    """Without a workspace every tile runs on BF16 operands."""
    M, N, K = 300, 200, 512
    W = I.matrix("student_t4", N, K, 13, 0.02, 1e-3)
    x = I.activations(M, K, 14, outlier_cols=16)
    pw, cs = packed(W)
    check(pw, cs, x, workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("case", ["x_2p110", "x_2p118", "x_2p125_sparse", "w_2p100_x_2pm110"])
@pytest.mark.parametrize("with_workspace", [True, False])
def test_huge_range_outputs(case, with_workspace):
    """Outputs near the top and bottom of binary32's range: the epilogue applies g
    and 2^sigma in one binary64 product, and BF16-operand tiles fold g's exponent
    into the weights, so nothing overflows before the result does."""
    M, N, K = 256, 384, 2560
    W = I.matrix("student_t4", N, K, 401, 0.02, 1e-3).double()
    x = I.activations(M, K, 402).double()
    if case == "x_2p110":
        x *= 2.0 ** 110
    elif case == "x_2p118":
        x *= 2.0 ** 118
    elif case == "x_2p125_sparse":
        x[:, [k for k in range(K) if k % 160]] = 0.0
        x *= 2.0 ** 125
    else:
        W *= 2.0 ** 100
        x *= 2.0 ** -110
    W, x = I.bf16_rne(W).contiguous(), I.bf16_rne(x).contiguous()
    pw, cs = packed(W)
    wh = O.dequant_nvfp4(*cs)
    yr, ar = O.matmul(x, wh)
    assert np.all(np.abs(yr) < 3.0e38)
    ws = None if with_workspace else torch.empty(0, dtype=torch.uint8, device="cuda")
    check(pw, cs, x, workspace=ws)
