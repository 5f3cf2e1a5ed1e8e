"""w4a16_gemv_noalloc: the decode GEMV for callers that cannot allocate device
memory (for example a plugin whose host framework owns every allocation).

It is called through the C ABI and must agree with w4a16_gemv -- the entry point
that takes a caller-provided workspace -- within the tolerance the GEMV tests
use, on two calls in a row (the second call finds the first call's leftovers in
the shared scratch array).  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4

pytestmark = pytest.mark.gpu

W4_ERR_WORKSPACE = 7


def noalloc_fn():
    f = W4.lib().w4a16_gemv_noalloc
    f.argtypes = [ctypes.POINTER(W4._Weights), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def call_noalloc(pw, x, y):
    s = pw.struct()
    return noalloc_fn()(ctypes.byref(s), ctypes.c_void_p(x.data_ptr()), x.shape[0],
                        ctypes.c_void_p(y.data_ptr()),
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("K,N,M", [(9728, 2560, 16), (2560, 1024, 1), (2560, 333, 8)])
def test_matches_workspace_entry_point(K, N, M):
    W = I.matrix("student_t4", N, K, K + N + M, 0.02, 1e-4, 20.0)
    c, s, g = O.pack_nvfp4(W)
    pw = W4.PackedWeights(W4.FMT_NVFP4, K, N, torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(),
                          torch.tensor([g], dtype=torch.float32).cuda())
    x = I.activations(M, K, 31 + M).cuda()
    y_ref = W4.w4a16_gemv(pw, x)            # caller-provided workspace
    torch.cuda.synchronize()
    _, a = O.matmul(x.cpu(), O.dequant_nvfp4(c, s, g))
    bound = 1e-3 * a
    for _ in range(2):                      # two calls in a row
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert call_noalloc(pw, x, y) == 0
        torch.cuda.synchronize()
        err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref.cpu().numpy())
        assert np.all(err <= bound)
    assert W4.w4_device_error(clear=True) == 0


def test_rejects_shapes_beyond_the_scratch_limit():
    # M=16, K=9728 splits K into 5 slices: 5*16*N*4 bytes of scratch exceed 8 MiB for N=40000
    dummy = torch.empty(64, dtype=torch.uint8, device="cuda")
    pw = W4.PackedWeights(W4.FMT_NVFP4, 9728, 40000, dummy, dummy, dummy.view(torch.float32))
    assert W4.w4a16_workspace_bytes(pw, 16) > 8 << 20
    x = torch.empty(16, 9728, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(16, dtype=torch.float32, device="cuda")
    assert call_noalloc(pw, x, y) == W4_ERR_WORKSPACE
