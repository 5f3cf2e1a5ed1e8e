"""w4a16_gemv_noalloc: the decode GEMV for callers that cannot allocate device
memory (for example a plugin whose host framework owns every allocation, or an
embedded runtime with a fixed memory budget), so they cannot hand the GEMV the
split-K scratch that w4a16_gemv takes as a workspace.

Called through the C ABI, it must give exactly the bits of w4a16_gemv (the same
kernels, with the scratch taken from the library's device array instead of a
caller-provided workspace) and meet the oracle's bound, on two calls in a row
(the second finds the first call's leftovers in the shared array).  The shapes
are chosen so that the GEMV really splits K and uses the scratch.  This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4
from gpu_util import assert_within_tolerance

pytestmark = pytest.mark.gpu

W4_ERR_WORKSPACE = 7
NOALLOC_SCRATCH_BYTES = 8 << 20


def noalloc_fn():
    f = W4.lib().w4a16_gemv_noalloc
    f.argtypes = [ctypes.POINTER(W4._Weights), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def call_noalloc(pw, x, y, stream=None):
    s = pw.struct()
    st = torch.cuda.current_stream() if stream is None else stream
    return noalloc_fn()(ctypes.byref(s), ctypes.c_void_p(x.data_ptr()), x.shape[0],
                        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(st.cuda_stream))


@pytest.mark.parametrize("K,N,M", [(9728, 2560, 16), (9728, 1024, 4), (9728, 333, 8), (4096, 2560, 16)])
def test_matches_workspace_entry_point(K, N, M):
    W = I.matrix("student_t4", N, K, K + N + M, 0.02, 1e-4, 20.0)
    c, s, g = O.pack_nvfp4(W)
    pw = W4.PackedWeights(W4.FMT_NVFP4, K, N, torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(),
                          torch.tensor([g], dtype=torch.float32).cuda())
    need = W4.w4a16_workspace_bytes(pw, M)
    assert 0 < need <= NOALLOC_SCRATCH_BYTES          # this shape splits K: the scratch is used
    x = I.activations(M, K, 31 + M)
    xd = x.cuda()
    y_ws = W4.w4a16_gemv(pw, xd)                     # caller-provided workspace
    torch.cuda.synchronize()
    yr, ar = O.matmul(x, O.dequant_nvfp4(c, s, g))
    for _ in range(2):                               # two calls in a row
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert call_noalloc(pw, xd, y) == 0
        torch.cuda.synchronize()
        assert torch.equal(y, y_ws)
        assert_within_tolerance(y.cpu().numpy(), yr, ar)
    assert W4.w4_device_error(clear=True) == 0


def test_on_a_side_stream():
    K, N, M = 9728, 2560, 16
    W = I.matrix("student_t4", N, K, 77, 0.02, 1e-4, 20.0)
    c, s, g = O.pack_nvfp4(W)
    pw = W4.PackedWeights(W4.FMT_NVFP4, K, N, torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(),
                          torch.tensor([g], dtype=torch.float32).cuda())
    xd = I.activations(M, K, 78).cuda()
    y_ws = W4.w4a16_gemv(pw, xd)
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    with torch.cuda.stream(st):
        assert call_noalloc(pw, xd, y, st) == 0
    st.synchronize()
    assert torch.equal(y, y_ws)


def test_rejects_shapes_beyond_the_scratch_limit():
    # M=16, K=9728 splits K into 5 slices: 5 * 16 * N * 4 bytes of scratch exceed 8 MiB for N = 40000.
    # The buffers have the real sizes, so even a wrongly accepted call would stay inside them.
    K, N, M = 9728, 40000, 16
    codes = torch.zeros(N, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(N, K // 16, dtype=torch.uint8, device="cuda")
    gs = torch.ones(1, dtype=torch.float32, device="cuda")
    pw = W4.PackedWeights(W4.FMT_NVFP4, K, N, codes, scales, gs)
    assert W4.w4a16_workspace_bytes(pw, M) > NOALLOC_SCRATCH_BYTES
    x = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    assert call_noalloc(pw, x, y) == W4_ERR_WORKSPACE
