"""Pins for the oracle's ROCmFP4 packer (Dual and FAST).

Method ("rocmwhy" ROCmFP4 page, sections 01-03 and the format table):
Codebook10 levels, one unsigned E4M3 scale per 16-weight half (Dual, 18-byte
blocks) or per 32 weights (FAST, 17 bytes), the scale chosen by exhaustive
search over the finite UE4M3 candidates, scored by reconstruction error.

Pins: exact brute force over scales x level vectors on tiny blocks, exact
per-element nearest levels, exact round trips of on-grid blocks, the page's
outlier-clipping example, byte-count facts, and sign symmetry.
"""
import itertools
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CB = [0, 1, 2, 3, 4, 6, 8, 10]
SCALES = [Fraction(O.e4m3_decode(u)) for u in range(127)]


def bf16_vals(vals):
    return torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(torch.bfloat16)


def exact_error(x, u, levels):
    s = SCALES[u]
    return sum((Fraction(float(xi)) - s * l) ** 2 for xi, l in zip(x, levels))


def brute_min_error(x, u):
    """Minimum exact error at scale u over every signed level vector."""
    signed = [l for v in CB for l in ({v, -v})]
    best = None
    for lv in itertools.product(signed, repeat=len(x)):
        e = exact_error(x, u, lv)
        best = e if best is None or e < best else best
    return best


@pytest.mark.parametrize("n,seed", [(1, 0), (1, 1), (2, 2), (2, 3)])
def test_search_matches_full_brute_force_tiny(n, seed):
    """n = 1, 2 elements: enumerate all 127 scales x all 15^n signed level vectors."""
    rnd = random.Random(seed)
    x = [float(bf16_vals([rnd.uniform(-3, 3)])[0]) for _ in range(n)]
    u_star, _ = O.rocm_search(x)
    errs = [brute_min_error(x, u) for u in range(127)]
    emin = min(errs)
    # the chosen scale attains the exact global minimum up to binary32 rounding of the sum
    assert errs[u_star] - emin <= emin * Fraction(1, 2 ** 20) + Fraction(1, 2 ** 140)
    # and it is the smallest code that does so when the minimum is well separated
    strict = [u for u in range(127) if errs[u] - emin <= emin * Fraction(1, 2 ** 20)]
    assert u_star == strict[0]


@pytest.mark.parametrize("n,seed", [(3, 4), (4, 5), (16, 6), (32, 7)])
def test_search_matches_separable_brute_force(n, seed):
    """For each scale the exact optimum is separable: each element independently
    takes its nearest signed level (brute force over the 15 levels)."""
    rnd = random.Random(seed)
    x = [float(v) for v in bf16_vals([rnd.gauss(0, 0.02) for _ in range(n)])]
    u_star, e_star = O.rocm_search(x)
    signed = sorted({l for v in CB for l in (v, -v)})
    errs = []
    for u in range(127):
        s = SCALES[u]
        errs.append(sum(min((Fraction(xi) - s * l) ** 2 for l in signed) for xi in x))
    emin = min(errs)
    assert errs[u_star] - emin <= emin * Fraction(n, 2 ** 20)
    # the oracle's own per-scale error equals that optimum up to binary32 rounding
    for u in (u_star, max(u_star - 3, 0), min(u_star + 3, 126)):
        assert abs(Fraction(O.rocm_error(np.array(x, np.float32), u)) - errs[u]) <= errs[u] * Fraction(n, 2 ** 21) + Fraction(1, 2 ** 149)


def test_levels_are_exact_nearest_per_element():
    W = I.rocm_weights()[:2, :256]
    for fmt in (O.FMT_DUAL, O.FMT_FAST):
        blk = O.pack_rocmfp4(W, fmt)
        wh = O.dequant_rocmfp4(blk, fmt)
        x = W.double().numpy()
        for r in range(2):
            for b in range(blk.shape[1]):
                for j in range(32):
                    u = blk[r, b, (j // 16) if fmt == O.FMT_DUAL else 0]
                    s = SCALES[u]
                    xv = Fraction(x[r, 32 * b + j])
                    if s == 0:
                        assert wh[r, 32 * b + j] == 0
                        continue
                    cand = sorted(((abs(xv - s * l * (1 if xv >= 0 else -1)), i % 2, i)
                                   for i, l in enumerate(CB)))
                    want = Fraction(CB[cand[0][2]]) * s * (1 if xv >= 0 else -1)
                    assert Fraction(wh[r, 32 * b + j]) == want


def test_on_grid_blocks_round_trip_exactly():
    """Halves built as level * s with levels 1, 3 and 10 present have exactly one
    zero-error candidate, which the search must find."""
    rnd = np.random.default_rng(3)
    rows = []
    for _ in range(4):
        row = []
        for _h in range(4):                         # 4 halves = 2 Dual blocks
            u = int(rnd.integers(0x18, 0x60))
            lv = rnd.choice(CB, size=16) * rnd.choice([-1, 1], size=16)
            lv[:3] = [1, -3, 10]
            row.extend(float(l) * O.e4m3_decode(u) for l in lv)
        rows.append(row)
    W = np.array(rows)
    Wb = bf16_vals(W)
    assert np.array_equal(Wb.double().numpy(), W)
    blk = O.pack_rocmfp4(Wb, O.FMT_DUAL)
    assert np.array_equal(O.dequant_rocmfp4(blk, O.FMT_DUAL), W)


def test_outlier_clipping_can_win():
    """rocmwhy 03 ("one imperfect value can buy 15 better ones"): with 15 values
    near 1 and an outlier of 10.6, the chosen scale clips the outlier and its
    error is below that of the smallest scale that still reaches 10.6."""
    rnd = random.Random(5)
    x = [float(v) for v in bf16_vals([rnd.uniform(0.8, 1.2) for _ in range(15)] + [10.6])]
    u, e = O.rocm_search(x)
    s = O.e4m3_decode(u)
    assert 10 * s < x[-1]
    u_keep = min(v for v in range(127) if 10 * O.e4m3_decode(v) >= x[-1])
    assert e < O.rocm_error(np.array(x, np.float32), u_keep)


def test_all_zero_half_takes_code_zero():
    W = torch.zeros(2, 64, dtype=torch.bfloat16)
    W[1, 20] = 0.5
    blk = O.pack_rocmfp4(W, O.FMT_DUAL)
    assert not blk[0].any()
    assert blk[1, 0, 0] == 0 and blk[1, 0, 1] != 0 and not blk[1, 1].any()


def test_format_table_facts():
    table = {}
    for line in open(os.path.join(GOLDEN, "rocmwhy_format_table.txt")):
        if line.strip() and not line.startswith("#"):
            f = line.split()
            table[f[0]] = (int(f[1]), int(f[3]), float(f[4]))
    K, N = 2560, 3
    W = I.rocm_weights()[:N]
    for fmt, name in ((O.FMT_DUAL, "rocmfp4_dual"), (O.FMT_FAST, "rocmfp4_fast")):
        blk = O.pack_rocmfp4(W, fmt)
        per, nbytes, bpw = table[name]
        assert blk.shape == (N, K // per, nbytes)
        assert 8 * blk.nbytes / (K * N) == bpw


def test_sign_symmetry():
    W = I.rocm_weights()[:4, :512]
    for fmt in (O.FMT_DUAL, O.FMT_FAST):
        a = O.pack_rocmfp4(W, fmt)
        b = O.pack_rocmfp4(-W, fmt)
        hdr = 2 if fmt == O.FMT_DUAL else 1
        assert np.array_equal(a[..., :hdr], b[..., :hdr])
        lo = lambda c: c & 15
        hi = lambda c: c >> 4
        for f in (lo, hi):
            ca, cb = f(a[..., hdr:]), f(b[..., hdr:])
            nz = (ca & 7) != 0
            assert np.array_equal(cb[nz], ca[nz] ^ 8) and np.all(cb[~nz] == 0)


def test_dual_never_worse_than_fast():
    """Each Dual half may pick the FAST block's scale, so the Dual error is never larger."""
    W = I.rocm_weights()[:8]
    x = W.double().numpy()
    ed = ((O.dequant_rocmfp4(O.pack_rocmfp4(W, O.FMT_DUAL), O.FMT_DUAL) - x) ** 2).reshape(-1, 32).sum(1)
    ef = ((O.dequant_rocmfp4(O.pack_rocmfp4(W, O.FMT_FAST), O.FMT_FAST) - x) ** 2).reshape(-1, 32).sum(1)
    assert np.all(ed <= ef * (1 + 1e-5))


def test_nonfinite_rejected():
    W = torch.zeros(1, 32, dtype=torch.bfloat16)
    W[0, 0] = float("inf")
    with pytest.raises(O.OracleError):
        O.pack_rocmfp4(W, O.FMT_DUAL)
