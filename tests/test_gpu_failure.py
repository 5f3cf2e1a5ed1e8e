"""Failure detection on the GPU, without a fault: with a wait limit short enough
that the kernels' first waits expire, every call of a kernel that waits on
mbarriers (the TMA-staged ROCmFP4 GEMV, the prefill GEMM) records
W4_ERR_TIMEOUT in the sticky device word and returns (each CTA still waits for
the copies and MMAs it had issued before it exits).  With the default limit
restored, the next calls on the same context are correct against the oracle and
record nothing.  The NVFP4 GEMVs wait on no mbarrier and must finish, correct,
under the same limit.

Also here: the library called from two host threads at once on one device (the
per-device launch state is shared under a lock) gives the single-thread bits."""
import threading

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4
from gpu_util import assert_within_tolerance, np_of

pytestmark = pytest.mark.gpu

W4_ERR_TIMEOUT = 6


@pytest.fixture
def default_limit_after():
    W4.w4_device_error(clear=True)
    yield
    W4.set_wait_limit(0)
    W4.w4_device_error(clear=True)


def nvfp4(K, N, seed):
    W = I.matrix("student_t4", N, K, seed, 0.02, 1e-4, 20.0)
    c, s, g = O.pack_nvfp4(W)
    pw = W4.PackedWeights(W4.FMT_NVFP4, K, N, torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(),
                          torch.tensor([g], dtype=torch.float32).cuda())
    return pw, O.dequant_nvfp4(c, s, g)


def expire_then_recover(run, check):
    W4.set_wait_limit(1)                      # 1 ns: the first wait that does not pass at once expires
    run()
    torch.cuda.synchronize()
    assert W4.w4_device_error(clear=True) == W4_ERR_TIMEOUT
    W4.set_wait_limit(0)                      # back to 2 s
    out = run()
    torch.cuda.synchronize()
    assert W4.w4_device_error(clear=True) == 0
    check(out)


@pytest.mark.parametrize("M", [4, 9, 16])
def test_nvfp4_gemv_kernels_do_not_wait(default_limit_after, M):
    """The NVFP4 GEMVs for several tokens load their operands directly as the
    one-token kernels do and wait on no mbarrier: with a 1 ns limit they still
    finish, correct, and record nothing (K = 9728 also exercises the split-K
    partials and their finalize)."""
    K, N = 9728, 1024
    pw, wh = nvfp4(K, N, 500 + M)
    x = I.activations(M, K, 501)
    yr, ar = O.matmul(x, wh)
    W4.set_wait_limit(1)
    y = W4.w4a16_gemv(pw, x.cuda())
    torch.cuda.synchronize()
    assert W4.w4_device_error(clear=True) == 0
    assert_within_tolerance(np_of(y), yr, ar)


def test_one_token_kernels_do_not_wait(default_limit_after):
    """The one-token kernels (single and grouped) load their operands directly and
    wait on no mbarrier: with a 1 ns limit they still finish, correct, and record
    nothing."""
    mats = [nvfp4(K, N, 510 + i) for i, (K, N) in enumerate(I.SWEEP_SHAPES)]
    xs = [I.activations(1, K, 520 + i) for i, (K, _) in enumerate(I.SWEEP_SHAPES)]
    xd = [x.cuda() for x in xs]
    W4.set_wait_limit(1)
    ys = W4.w4a16_gemv_grouped([m[0] for m in mats], xd)
    y1 = [W4.w4a16_gemv(m[0], x) for m, x in zip(mats, xd)]
    torch.cuda.synchronize()
    assert W4.w4_device_error(clear=True) == 0
    for y, yb, (_, wh), x in zip(ys, y1, mats, xs):
        yr, ar = O.matmul(x, wh)
        assert_within_tolerance(np_of(y), yr, ar)
        assert_within_tolerance(np_of(yb), yr, ar)


@pytest.mark.parametrize("fmt", [W4.FMT_ROCMFP4_DUAL, W4.FMT_ROCMFP4_FAST])
def test_rocm_gemv_wait_expiry(default_limit_after, fmt):
    K, N = 2560, 1536
    W = I.matrix("laplace", N, K, 530, 0.015, 1e-4, 20.0)
    b = O.pack_rocmfp4(W, fmt)
    pw = W4.PackedWeights(fmt, K, N, torch.from_numpy(b).cuda())
    x = I.activations(8, K, 531)
    yr, ar = O.matmul(x, O.dequant_rocmfp4(b, fmt))
    xd = x.cuda()
    expire_then_recover(lambda: W4.w4a16_gemv(pw, xd), lambda y: assert_within_tolerance(np_of(y), yr, ar))


@pytest.mark.parametrize("with_workspace", [True, False])
def test_gemm_wait_expiry(default_limit_after, with_workspace):
    M, K, N = 512, 2560, 768
    pw, wh = nvfp4(K, N, 540)
    x = I.activations(M, K, 541, outlier_cols=16)
    yr, ar = O.matmul(x, wh)
    xd = x.cuda()
    ws = None if with_workspace else torch.empty(0, dtype=torch.uint8, device="cuda")
    expire_then_recover(lambda: W4.w4a16_gemm(pw, xd, want_bf16=False, workspace=ws)[0],
                        lambda y: assert_within_tolerance(np_of(y), yr, ar))


def test_two_host_threads_one_device():
    """Two threads, each on its own stream, alternate GEMVs (M = 1 and 9) and
    GEMMs on one device: every result equals the one-thread result bit for bit."""
    pw, _ = nvfp4(2560, 2048, 550)
    xs = {M: I.activations(M, 2560, 551 + M).cuda() for M in (1, 9, 300)}
    ref = {M: (W4.w4a16_gemv(pw, xs[M]) if M <= 16 else W4.w4a16_gemm(pw, xs[M], want_bf16=False)[0]).clone()
           for M in xs}
    torch.cuda.synchronize()
    errors = []

    def work(seed):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for i in range(30):
                    M = (1, 9, 300)[(i + seed) % 3]
                    y = W4.w4a16_gemv(pw, xs[M]) if M <= 16 else W4.w4a16_gemm(pw, xs[M], want_bf16=False)[0]
                    s.synchronize()
                    if not torch.equal(y, ref[M]):
                        errors.append((seed, i, M))
        except Exception as e:  # noqa: BLE001
            errors.append(repr(e))

    ts = [threading.Thread(target=work, args=(k,)) for k in range(2)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors[:5]
    assert W4.w4_device_error(clear=True) == 0
