"""CUDA packers vs the oracle: packed bytes, scales and global scale bit-exact."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4
from gpu_util import np_of

pytestmark = pytest.mark.gpu


def check_nvfp4(W):
    pw = W4.pack_nvfp4(W.cuda())
    c, s, g = O.pack_nvfp4(W)
    torch.cuda.synchronize()
    assert np.float32(pw.global_scale.item()).tobytes() == np.float32(g).tobytes()
    assert np.array_equal(np_of(pw.scales), s)
    gc = np_of(pw.codes)
    bad = np.argwhere(gc != c)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:4].tolist()}"


def test_nvfp4_small_case():
    W, _ = I.nvfp4_small()
    check_nvfp4(W)


@pytest.mark.parametrize("idx", range(5))
def test_nvfp4_sweep_shapes(idx):
    K, N = I.SWEEP_SHAPES[idx]
    check_nvfp4(I.sweep_weights(K, N, idx))


@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (7, 272), (1, 2560), (333, 160)])
def test_nvfp4_ragged_and_minimum(N, K):
    check_nvfp4(I.matrix("student_t4", N, K, 77 + N, 0.02, 1e-2))


def test_nvfp4_zero_and_tiny():
    check_nvfp4(torch.zeros(5, 64, dtype=torch.bfloat16))
    W = torch.zeros(4, 64, dtype=torch.float64)
    W[0, :16] = 2.0 ** -130          # bf16 subnormals
    W[1, 3] = -(2.0 ** -133)
    W[2, 20] = 1.0
    W[3, 40:56] = torch.linspace(-1e-3, 1e-3, 16, dtype=torch.float64)
    check_nvfp4(I.bf16_rne(W))
    check_nvfp4(I.bf16_rne(W * 2.0 ** -100))   # global scale underflows to subnormal / zero


def test_nvfp4_nonfinite_sets_status():
    W = I.matrix("normal", 4, 64, 5, 0.02).cuda()
    W[2, 7] = float("nan")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    W4.w4_device_error(clear=True)
    W4.pack_nvfp4(W, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 5
    assert W4.w4_device_error(clear=True) == 5
    st.fill_(-1)
    W4.pack_nvfp4(I.matrix("normal", 4, 64, 5, 0.02).cuda(), d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0


def check_rocm(W, fmt):
    code = W4.FMT_ROCMFP4_DUAL if fmt == "dual" else W4.FMT_ROCMFP4_FAST
    pw = W4.pack_rocmfp4(W.cuda(), fmt)
    ref = O.pack_rocmfp4(W, code)
    got = np_of(pw.codes)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("fmt", ["dual", "fast"])
def test_rocm_laplace_matrix(fmt):
    W = I.rocm_weights()
    rows = torch.cat([torch.arange(0, 192), torch.arange(4800, 4864), torch.arange(9728 - 64, 9728)])
    check_rocm(W[rows].contiguous(), fmt)


@pytest.mark.parametrize("fmt", ["dual", "fast"])
@pytest.mark.parametrize("N,K", [(1, 32), (5, 96), (3, 2560)])
def test_rocm_ragged(fmt, N, K):
    check_rocm(I.matrix("laplace", N, K, 11 * N + K, 0.015, 1e-2), fmt)


@pytest.mark.parametrize("fmt", ["dual", "fast"])
def test_rocm_degenerate(fmt):
    W = torch.zeros(3, 64, dtype=torch.float64)
    W[1, 5] = 10.6
    W[1, 6:21] = 1.0
    W[2, :] = 2.0 ** -130
    check_rocm(I.bf16_rne(W), fmt)
    check_rocm(torch.zeros(2, 64, dtype=torch.bfloat16), fmt)


def test_full_laplace_matrix_dual():
    check_rocm(I.rocm_weights(), "dual")


# ---- scale search for NVFP4 blocks and importance weighting (both formats) ----
def importance_vector(K, seed, zeros=True):
    g = torch.Generator().manual_seed(seed)
    w = torch.rand(K, generator=g, dtype=torch.float32) * 2.0
    if zeros:
        w[::7] = 0.0
    return w


def check_nvfp4_search(W, imp=None):
    pw = W4.pack_nvfp4(W.cuda(), scale_search=W4.SCALE_MSE, importance=None if imp is None else imp.cuda())
    c, s, g = O.pack_nvfp4(W, mse=True, importance=None if imp is None else imp.numpy())
    torch.cuda.synchronize()
    assert np.float32(pw.global_scale.item()).tobytes() == np.float32(g).tobytes()
    bad = np.argwhere(np_of(pw.scales) != s)
    assert bad.size == 0, f"{len(bad)} scales differ, first {bad[:4].tolist()}"
    bad = np.argwhere(np_of(pw.codes) != c)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("idx", [0, 1, 4])
def test_nvfp4_scale_search_sweep_rows(idx):
    K, N = I.SWEEP_SHAPES[idx]
    check_nvfp4_search(I.sweep_weights(K, N, idx)[:96].contiguous())


@pytest.mark.parametrize("N,K", [(1, 16), (7, 272), (333, 160)])
def test_nvfp4_scale_search_ragged_and_weighted(N, K):
    W = I.matrix("student_t4", N, K, 99 + N, 0.02, 1e-2)
    check_nvfp4_search(W)
    check_nvfp4_search(W, importance_vector(K, N))


def test_nvfp4_scale_search_degenerate():
    check_nvfp4_search(torch.zeros(3, 64, dtype=torch.bfloat16))
    W = torch.zeros(4, 64, dtype=torch.float64)
    W[0, :16] = 2.0 ** -130
    W[2, 20] = 1.0
    W[3, 40:56] = torch.linspace(-1e-3, 1e-3, 16, dtype=torch.float64)
    check_nvfp4_search(I.bf16_rne(W))
    check_nvfp4_search(I.bf16_rne(W), importance_vector(64, 3))


@pytest.mark.parametrize("fmt", ["dual", "fast"])
def test_rocm_importance_weighted(fmt):
    W = I.rocm_weights()[:64].contiguous()
    imp = importance_vector(2560, 11)
    pw = W4.pack_rocmfp4(W.cuda(), fmt, importance=imp.cuda())
    ref = O.pack_rocmfp4(W, O.FMT_DUAL if fmt == "dual" else O.FMT_FAST, importance=imp.numpy())
    torch.cuda.synchronize()
    bad = np.argwhere(np_of(pw.codes) != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first {bad[:4].tolist()}"
    # unit weights give the unweighted bytes
    ones = W4.pack_rocmfp4(W.cuda(), fmt, importance=torch.ones(2560, device="cuda"))
    plain = W4.pack_rocmfp4(W.cuda(), fmt)
    assert torch.equal(ones.codes, plain.codes)


def test_bad_importance_sets_status():
    W = I.matrix("normal", 4, 64, 5, 0.02).cuda()
    imp = torch.ones(64, device="cuda")
    imp[9] = -1.0
    for run in (lambda st: W4.pack_rocmfp4(W, "dual", importance=imp, d_status=st),
                lambda st: W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE, importance=imp, d_status=st)):
        st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        W4.w4_device_error(clear=True)
        run(st)
        torch.cuda.synchronize()
        assert st.item() == 5
        assert W4.w4_device_error(clear=True) == 5
    with pytest.raises(W4.W4Error):   # weights only with the scale search
        W4.pack_nvfp4(W, importance=torch.ones(64, device="cuda"))
