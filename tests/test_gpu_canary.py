"""Out-of-bounds writes, checked without a sanitizer: every output buffer of
every entry point is followed by canary bytes (a fixed pattern) that must be
unchanged after the call, on ragged shapes where tiles, boxes and warps only
partly cover the output."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4

pytestmark = pytest.mark.gpu

CANARY = 256          # bytes after each buffer
PATTERN = 0xA5


def canaried(shape, dtype):
    """A tensor of `shape` whose storage is followed by CANARY bytes of PATTERN."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((n + CANARY,), PATTERN, dtype=torch.uint8, device="cuda")
    return raw[:n].view(dtype).view(shape), raw


def intact(raw):
    torch.cuda.synchronize()
    tail = raw[-CANARY:].cpu().numpy()
    return bool(np.all(tail == PATTERN))


@pytest.mark.parametrize("N,K", [(77, 256), (333, 2560), (1, 512), (1000, 4096)])
def test_packers(N, K):
    W = I.matrix("student_t4", N, K, N + K, 0.02, 1e-3, device="cuda")
    codes, rc = canaried((N, K // 2), torch.uint8)
    scales, rs = canaried((N, K // 16), torch.uint8)
    g, rg = canaried((1,), torch.float32)
    W4.pack_nvfp4(W, out=W4.PackedWeights(W4.FMT_NVFP4, K, N, codes, scales, g))
    assert intact(rc) and intact(rs) and intact(rg)
    W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE, out=W4.PackedWeights(W4.FMT_NVFP4, K, N, codes, scales, g))
    assert intact(rc) and intact(rs) and intact(rg)
    for fmt, bb in (("dual", 18), ("fast", 17)):
        blocks, rb = canaried((N, K // 32, bb), torch.uint8)
        W4.pack_rocmfp4(W, fmt, out=blocks)
        assert intact(rb)
    blocks, rb = canaried((N, K // 32, 18), torch.uint8)
    W4.pack_q4_0(W, out=blocks)
    assert intact(rb)


@pytest.mark.parametrize("fmt", [W4.FMT_NVFP4, W4.FMT_ROCMFP4_DUAL, W4.FMT_ROCMFP4_FAST])
@pytest.mark.parametrize("M,N,K", [(1, 77, 512), (3, 333, 2560), (9, 1000, 1024), (16, 5, 9728), (1, 2, 4096)])
def test_gemv_outputs(fmt, M, N, K):
    W = I.matrix("student_t4", N, K, M + N + K, 0.02, 1e-3, device="cuda")
    pw = W4.pack_nvfp4(W) if fmt == W4.FMT_NVFP4 else W4.pack_rocmfp4(W, {2: "dual", 3: "fast"}[fmt])
    x = I.activations(M, K, 3, device="cuda")
    y, ry = canaried((M, N), torch.float32)
    need = W4.w4a16_workspace_bytes(pw, M)
    ws, rw = canaried((max(need, 16),), torch.uint8)
    W4.w4a16_gemv(pw, x, out=y, workspace=ws)
    assert intact(ry) and intact(rw)
    assert W4.w4_device_error(clear=True) == 0


def test_grouped_outputs():
    shapes = [(256, 7), (1024, 149), (2560, 333), (9728, 2), (512, 1)]
    pws = [W4.pack_nvfp4(I.matrix("student_t4", N, K, 7 + i, 0.02, 1e-3, device="cuda"))
           for i, (K, N) in enumerate(shapes)]
    xs = [I.activations(1, K, 9 + i, device="cuda") for i, (K, _) in enumerate(shapes)]
    outs = [canaried((1, N), torch.float32) for _, N in shapes]
    W4.w4a16_gemv_grouped(pws, xs, outs=[o[0] for o in outs])
    assert all(intact(o[1]) for o in outs)


@pytest.mark.parametrize("fmt", [W4.FMT_NVFP4, W4.FMT_ROCMFP4_DUAL, W4.FMT_ROCMFP4_FAST])
@pytest.mark.parametrize("M,N,K", [(1, 77, 512), (300, 200, 1024), (197, 300, 2048)])
def test_gemm_outputs(fmt, M, N, K):
    W = I.matrix("student_t4", N, K, M + N, 0.02, 1e-3, device="cuda")
    pw = W4.pack_nvfp4(W) if fmt == W4.FMT_NVFP4 else W4.pack_rocmfp4(W, {2: "dual", 3: "fast"}[fmt])
    x = I.activations(M, K, 5, device="cuda")
    y32, r32 = canaried((M, N), torch.float32)
    y16, r16 = canaried((M, N), torch.bfloat16)
    ws, rw = canaried((W4.w4a16_workspace_bytes(pw, M),), torch.uint8)
    W4.w4a16_gemm(pw, x, out_f32=y32, out_bf16=y16, workspace=ws)
    assert intact(r32) and intact(r16) and intact(rw)
    assert W4.w4_device_error(clear=True) == 0


def test_reconstruction_error_outputs():
    W = I.matrix("laplace", 333, 512, 4, 0.015, 1e-3, device="cuda")
    pw = W4.pack_rocmfp4(W, "dual")
    ws, rw = canaried((W4.lib().w4_reconstruction_workspace_bytes(),), torch.uint8)
    W4.reconstruction_error(pw, W, workspace=ws)
    assert intact(rw)
