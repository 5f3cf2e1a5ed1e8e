"""Pins for the oracle's matmul (y = x . w_hat, binary64) and for the seeded inputs."""
from fractions import Fraction

import numpy as np
import torch

import oracle as O
import w4a16_inputs as I


def test_matmul_exact_rationals_tiny():
    x = I.activations(3, 32, 1)
    W = I.matrix("normal", 5, 32, 9, 0.02)
    c, s, g = O.pack_nvfp4(W)
    wh = O.dequant_nvfp4(c, s, g)
    y, a = O.matmul(x, wh)
    xs = x.double().numpy()
    for m in range(3):
        for r in range(5):
            exact = sum(Fraction(xs[m, k]) * Fraction(wh[r, k]) for k in range(32))
            mag = sum(abs(Fraction(xs[m, k]) * Fraction(wh[r, k])) for k in range(32))
            assert abs(Fraction(y[m, r]) - exact) <= mag * Fraction(32, 2 ** 52)
            assert abs(Fraction(a[m, r]) - mag) <= mag * Fraction(32, 2 ** 52)


def test_matmul_vs_numpy():
    x = I.activations(4, 2560, 3)
    W = I.sweep_weights(2560, 1024, 1)[:64]
    c, s, g = O.pack_nvfp4(W)
    wh = O.dequant_nvfp4(c, s, g)
    y, a = O.matmul(x, wh)
    ref = x.double().numpy() @ wh.T
    assert np.all(np.abs(y - ref) <= 1e-12 * a)
    assert np.allclose(a, np.abs(x.double().numpy()) @ np.abs(wh).T, rtol=1e-12)


def test_matmul_one_hot_picks_a_column():
    K = 64
    x = torch.zeros(1, K, dtype=torch.bfloat16)
    x[0, 17] = 1.0
    W = I.matrix("laplace", 8, K, 4, 0.015)
    blk = O.pack_rocmfp4(W, O.FMT_DUAL)
    wh = O.dequant_rocmfp4(blk, O.FMT_DUAL)
    y, a = O.matmul(x, wh)
    assert np.array_equal(y[0], wh[:, 17]) and np.array_equal(a[0], np.abs(wh[:, 17]))


# ---------------------------------------------------------------- inputs -----
def test_bf16_rounding_is_single_nearest_even():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(2000) * 10.0 ** rng.uniform(-5, 5, 2000)
    got = I.bf16_rne(torch.tensor(v)).double().numpy()
    for x, r in zip(v, got):
        fx = Fraction(x)
        m, e = np.frexp(abs(x))
        step = Fraction(2) ** (int(e) - 8)
        lo = (abs(fx) // step) * step
        hi = lo + step
        d_lo, d_hi = abs(fx) - lo, hi - abs(fx)
        want = lo if d_lo < d_hi else hi if d_hi < d_lo else (lo if (lo / step) % 2 == 0 else hi)
        assert Fraction(abs(r)) == want and np.sign(r) == np.sign(x)


def test_generators_are_deterministic_and_chunk_free():
    a = I.matrix("student_t4", 3, 1000, 42, 0.02, 1e-3)
    b = I.matrix("student_t4", 3, 1000, 42, 0.02, 1e-3)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    u_all = I.uniform(I.stream_key(9), 0, 1000)
    u_part = torch.cat([I.uniform(I.stream_key(9), 0, 400), I.uniform(I.stream_key(9), 400, 600)])
    assert torch.equal(u_all, u_part)


def test_distribution_parameters():
    W = I.sweep_weights(2560, 1024, 1).double()
    n_out = int(round(1e-4 * W.numel()))
    assert abs(W.std().item() - 0.02 * (1 + 19 ** 2 * 1e-4) ** 0.5) < 0.0015
    L = I.rocm_weights().double()
    assert abs(L.abs().median().item() - 0.015 * np.log(2)) < 3e-4    # Laplace median |x| = b ln 2
    x = I.activations(16, 4096, 5).double()
    assert abs(x.mean().item()) < 0.02 and abs(x.std().item() - 1) < 0.02
    pos = I.distinct_positions(I.stream_key(2001, 1), n_out, W.numel())
    assert pos.unique().numel() == n_out


def test_small_case_has_eight_half_outliers():
    W, x = I.nvfp4_small()
    assert W.shape == (1024, 1024) and x.shape == (1, 1024)
    assert int((W.double().abs() == 0.5).sum()) == 8
