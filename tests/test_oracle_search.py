"""Pins for the oracle's scale searches with importance weighting (ROCmFP4,
Dual and FAST) and for the NVFP4 block scale chosen by search.

Method ("rocmwhy" ROCmFP4 page, section 03: finite scale candidates scored by
reconstruction error, with optional importance weighting; its interactive
example gives a synthetic outlier low importance so that the search may prefer
the rest of the half-block).  The same search over the finite E4M3 codes
chooses NVFP4 block scales ("EdgeRock-4B-NVFP4" card, intro: E2M1 values, one
E4M3 scale per 16, one FP32 global scale), with the global scale fixed by the
abs-max rule.

Pins: the chosen NVFP4 scale attains the exact optimum (rational arithmetic,
separable per element) up to binary32 rounding; it is never worse than the
abs-max scale; the packed codes are the RNE encoding under the chosen scale;
unit weights reproduce the unweighted bytes; a zero weight is the same as
removing the element; scaling all weights by a power of two changes nothing;
the page's low-importance-outlier example; invalid weights are refused.
"""
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
SIGNED = sorted({s * v for v in E2M1 for s in (1, -1)})


def bf16_list(vals):
    t = torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(torch.bfloat16)
    return [float(v) for v in t.float()]


def exact_nvfp4_error(x, u, g, w=None):
    """Exact weighted error at scale code u: every element takes its nearest
    E2M1 level times d = binary32(E4M3(u) * g) (the per-scale optimum)."""
    d = Fraction(float(np.float32(O.e4m3_decode(u)) * np.float32(g)))
    tot = Fraction(0)
    for i, xi in enumerate(x):
        best = min((Fraction(xi) - Fraction(l) * d) ** 2 for l in SIGNED)
        tot += (Fraction(float(w[i])) if w is not None else 1) * best
    return tot


@pytest.mark.parametrize("seed", range(6))
def test_nvfp4_search_attains_exact_optimum(seed):
    rnd = random.Random(seed)
    x = bf16_list([rnd.gauss(0, 0.02) * (20 if rnd.random() < 0.1 else 1) for _ in range(16)])
    g = np.float32(max(abs(v) for v in x) * rnd.uniform(0.8, 3.0) / 2688.0)
    w = None if seed % 2 == 0 else np.array([rnd.uniform(0, 2) for _ in range(16)], np.float32)
    u_star, _ = O.nvfp4_search(np.array(x, np.float32), g, w)
    errs = [exact_nvfp4_error(x, u, g, w) for u in range(127)]
    emin = min(errs)
    # binary32 rounding of 16 quotients, products and sums: well inside 2^-17 relative
    assert errs[u_star] - emin <= emin * Fraction(1, 2 ** 17) + Fraction(1, 2 ** 140)
    strict = [u for u in range(127) if errs[u] - emin <= emin * Fraction(1, 2 ** 17)]
    assert u_star == strict[0]


def test_nvfp4_search_never_worse_than_absmax_and_codes_follow_scale():
    W = I.sweep_weights(512, 48, 2)
    ca, sa, g = O.pack_nvfp4(W)
    cm, sm, gm = O.pack_nvfp4(W, mse=True)
    assert gm == g
    X = W.float().numpy()
    worse = 0
    for n in range(48):
        for b in range(512 // 16):
            x = X[n, 16 * b:16 * b + 16]
            ea = O.nvfp4_error(x, int(sa[n, b]), g)
            em = O.nvfp4_error(x, int(sm[n, b]), g)
            worse += em > ea
            # codes are the RNE E2M1 encoding of x / (scale * g) in binary32
            d = np.float32(O.e4m3_decode(int(sm[n, b]))) * np.float32(g)
            q = (x / d).astype(np.float32) if d != 0 else np.zeros(16, np.float32)
            c = O.e2m1_encode_array(q) if d != 0 else np.zeros(16, np.uint8)
            packed = (c[0::2] | (c[1::2] << 4)).astype(np.uint8)
            assert np.array_equal(packed, cm[n, 8 * b:8 * b + 8])
    assert worse == 0
    # the search changes a good share of the abs-max choices on Student-t weights
    assert (sm != sa).mean() > 0.2


def test_nvfp4_search_zero_and_exact_blocks():
    g = np.float32(0.001)
    u, e = O.nvfp4_search(np.zeros(16, np.float32), g)
    assert (u, e) == (0, 0.0)
    # one value that some (level, scale) pair reproduces exactly: error 0
    v = np.float32(3.0 * O.e4m3_decode(40)) * g
    x = np.zeros(16, np.float32)
    x[5] = v
    u, e = O.nvfp4_search(x, g)
    assert e == 0.0
    assert O.nvfp4_error(x, u, g) == 0.0
    assert all(O.nvfp4_error(x, v2, g) > 0.0 for v2 in range(u))


@pytest.mark.parametrize("fmt", [O.FMT_DUAL, O.FMT_FAST])
def test_unit_weights_reproduce_unweighted_bytes(fmt):
    W = I.rocm_weights()[:24, :256].contiguous()
    ones = np.ones(256, np.float32)
    assert np.array_equal(O.pack_rocmfp4(W, fmt), O.pack_rocmfp4(W, fmt, importance=ones))
    Wn = I.sweep_weights(256, 24, 3)
    a = O.pack_nvfp4(Wn, mse=True)
    b = O.pack_nvfp4(Wn, mse=True, importance=ones)
    assert all(np.array_equal(p, q) for p, q in zip(a, b))


@pytest.mark.parametrize("seed", range(4))
def test_zero_weight_is_element_removed_and_power_of_two_invariance(seed):
    rnd = random.Random(100 + seed)
    for n in (16, 32):
        x = np.array(bf16_list([rnd.gauss(0, 0.015) for _ in range(n)]), np.float32)
        w = np.array([rnd.uniform(0.1, 3) for _ in range(n)], np.float32)
        j = rnd.randrange(n)
        w0 = w.copy(); w0[j] = 0.0
        x0 = x.copy(); x0[j] = 0.0
        assert O.rocm_search(x, w0) == O.rocm_search(x0, w)
        u, e = O.rocm_search(x, w)
        u4, e4 = O.rocm_search(x, w * np.float32(4))
        assert u4 == u and e4 == 4 * e
        if n == 16:
            g = np.float32(float(np.abs(x).max()) / 2688.0)
            assert O.nvfp4_search(x, g, w0) == O.nvfp4_search(x0, g, w)
            u, e = O.nvfp4_search(x, g, w)
            u4, e4 = O.nvfp4_search(x, g, w * np.float32(0.25))
            assert u4 == u and e4 == e / 4


def test_low_importance_outlier_lets_the_rest_win():
    """The page's example: with the outlier's importance lowered, the search
    fits the other fifteen weights of the half-block better."""
    rnd = random.Random(7)
    x = np.array(bf16_list([rnd.gauss(0, 0.01) for _ in range(16)]), np.float32)
    x[3] = np.float32(bf16_list([0.4])[0])
    u_plain, _ = O.rocm_search(x)
    w = np.ones(16, np.float32); w[3] = 0.0
    u_w, _ = O.rocm_search(x, w)
    assert u_w < u_plain
    rest = np.ones(16, np.float32); rest[3] = 0.0
    assert O.rocm_error(x, u_w, rest) < O.rocm_error(x, u_plain, rest)


def test_invalid_weights_are_refused():
    W = I.rocm_weights()[:2, :64].contiguous()
    for bad in (-1.0, float("nan"), float("inf")):
        w = np.ones(64, np.float32); w[7] = bad
        with pytest.raises(O.OracleError):
            O.pack_rocmfp4(W, O.FMT_DUAL, importance=w)
        with pytest.raises(O.OracleError):
            O.pack_nvfp4(W, mse=True, importance=w)
    with pytest.raises(O.OracleError):   # weights only go with the search
        O.pack_nvfp4(W, importance=np.ones(64, np.float32))
