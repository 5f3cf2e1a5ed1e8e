"""Stock Q4_0 comparison packer and the reconstruction-error report on the GPU
against the oracle: Q4_0 bytes bit-exact, binary64 error sums equal up to
summation order, for every format."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4
from gpu_util import np_of

pytestmark = pytest.mark.gpu


def check_q4_0(W):
    pw = W4.pack_q4_0(W.cuda())
    ref = O.pack_q4_0(W)
    torch.cuda.synchronize()
    bad = np.argwhere(np_of(pw.codes) != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first {bad[:4].tolist()}"
    return pw


def test_q4_0_laplace_and_student_t():
    check_q4_0(I.rocm_weights()[:256].contiguous())
    check_q4_0(I.sweep_weights(2560, 9728, 3)[:128].contiguous())


@pytest.mark.parametrize("N,K", [(1, 32), (5, 96), (3, 2560), (77, 64)])
def test_q4_0_ragged(N, K):
    check_q4_0(I.matrix("laplace", N, K, 200 + N, 0.015, 1e-2, 20.0))


def test_q4_0_extremes():
    W = torch.zeros(6, 64, dtype=torch.float64)
    W[1, :32] = torch.linspace(-1e6, 3e5, 32, dtype=torch.float64)   # scale saturates at 65504
    W[2, 5] = 2.0 ** -20                                               # FP16-subnormal scale
    W[2, 40] = -(2.0 ** -30)                                           # scale underflows to 0
    W[3, :] = 1.0                                                      # ties on the largest magnitude
    W[4, 32:] = torch.tensor([(-1) ** j * (j % 9) * 0.5 for j in range(32)], dtype=torch.float64)
    W[5, :32] = 2.0 ** -130                                            # bf16 subnormals
    check_q4_0(I.bf16_rne(W))
    check_q4_0(I.bf16_rne(-W))


def test_q4_0_nonfinite_sets_status_and_matmul_refuses():
    W = I.matrix("normal", 4, 64, 5, 0.02).cuda()
    W[1, 3] = float("inf")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    W4.w4_device_error(clear=True)
    W4.pack_q4_0(W, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 5
    assert W4.w4_device_error(clear=True) == 5
    pw = W4.pack_q4_0(I.matrix("normal", 4, 64, 5, 0.02).cuda())
    with pytest.raises(W4.W4Error):
        W4.w4a16_gemv(pw, I.activations(1, 64, 1).cuda())


def oracle_hat(fmt, W, pw_cpu):
    if fmt == "nvfp4" or fmt == "nvfp4_search":
        return O.dequant_nvfp4(*pw_cpu)
    if fmt == "q4_0":
        return O.dequant_q4_0(pw_cpu)
    return O.dequant_rocmfp4(pw_cpu, O.FMT_DUAL if fmt == "dual" else O.FMT_FAST)


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_search", "dual", "fast", "q4_0"])
def test_reconstruction_error_matches_oracle(fmt):
    W = I.rocm_weights()[:96].contiguous()
    Wd = W.cuda()
    if fmt == "nvfp4":
        pw, ref = W4.pack_nvfp4(Wd), O.pack_nvfp4(W)
    elif fmt == "nvfp4_search":
        pw, ref = W4.pack_nvfp4(Wd, scale_search=W4.SCALE_MSE), O.pack_nvfp4(W, mse=True)
    elif fmt == "q4_0":
        pw, ref = W4.pack_q4_0(Wd), O.pack_q4_0(W)
    else:
        pw, ref = W4.pack_rocmfp4(Wd, fmt), O.pack_rocmfp4(W, O.FMT_DUAL if fmt == "dual" else O.FMT_FAST)
    e, q = W4.reconstruction_error(pw, Wd)
    e2, q2 = W4.reconstruction_error(pw, Wd)
    assert (e, q) == (e2, q2)                       # fixed summation order
    re, rq = O.reconstruction_sse(W, oracle_hat(fmt, W, ref))
    assert abs(e - re) <= 1e-12 * re and abs(q - rq) <= 1e-12 * rq
    assert 0.0 < e < q
