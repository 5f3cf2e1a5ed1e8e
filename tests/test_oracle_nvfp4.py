"""Pins for the oracle's NVFP4 packer and dequantiser.

Recipe (EdgeRock-4B-NVFP4 card, intro; Nanbeige4.2-3B-NVFP4A16 card,
Creation: data-free RTN, group 16): global = absmax / (6 * 448), block scale
= E4M3(block absmax / 6 / global), code = E2M1(x / (scale * global)).

Pins: exact round trips of on-grid matrices, power-of-two scaling and sign
symmetry, brute-force nearest checks of every code and scale against exact
rationals, a hand-worked 16-element block, and the byte-count fact.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, np.float64)).to(torch.float32).to(torch.bfloat16)


def nib(codes: np.ndarray) -> np.ndarray:
    """[N][K/2] bytes -> [N][K] nibbles, element 2i in the low nibble (reading C8)."""
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = codes & 15
    out[:, 1::2] = codes >> 4
    return out


E2M1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def on_grid_matrix(N, K, g_exp, seed):
    """W = e2m1 * E4M3(s) * 2^g_exp with a +-6 in every block and one block at scale 448."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, size=(N, K))
    codes[:, ::16] = np.where(rng.integers(0, 2, size=(N, K // 16)) == 1, 15, 7)  # +-6 per block
    scl = rng.integers(0x20, 0x7E, size=(N, K // 16))        # normal E4M3 scales
    scl[0, 0] = 0x7E                                          # 448 -> sets absmax = 6*448*g
    val = np.array([O.e2m1_decode(c) for c in range(16)])[codes]
    sv = np.array([O.e4m3_decode(s) for s in range(256)])[np.repeat(scl, 16, axis=1)]
    W = val * sv * 2.0 ** g_exp
    return W, codes, scl


@pytest.mark.parametrize("g_exp,seed", [(-12, 1), (-20, 2), (0, 3)])
def test_on_grid_round_trip_is_exact(g_exp, seed):
    W, codes, scl = on_grid_matrix(8, 64, g_exp, seed)
    Wb = bf16(W)
    assert np.array_equal(Wb.double().numpy(), W)            # on grid -> exact in bf16
    c, s, g = O.pack_nvfp4(Wb)
    assert g == np.float32(2.0 ** g_exp)
    assert np.array_equal(s, scl)
    # codes equal except that the two encodings of zero are not distinguished by value
    n = nib(c)
    z = (codes & 7) == 0
    assert np.array_equal(n[~z], codes[~z])
    assert np.all((n[z] & 7) == 0)
    assert np.array_equal(O.dequant_nvfp4(c, s, g), W)


def test_global_scale_is_absmax_over_2688_in_binary32():
    W, _ = I.nvfp4_small()
    _, _, g = O.pack_nvfp4(W)
    amax = np.float32(W.float().abs().max().item())
    assert g == np.float32(amax / np.float32(2688.0))
    assert amax == np.float32(0.5)                            # the planted +-0.5 outliers


def _check_rtn(Wb, c, s, g):
    """Every scale is the nearest E4M3 value to (bamax/6)/g and every code the
    nearest E2M1 point to x/d -- brute force over the grids in exact rationals,
    from the binary32 quotients."""
    W = Wb.float().numpy()
    N, K = W.shape
    n = nib(c)
    e4 = [Fraction(O.e4m3_decode(b)) for b in range(127)]
    e2 = [Fraction(v) for v in E2M1]
    for r in range(N):
        for b in range(K // 16):
            x = W[r, 16 * b:16 * b + 16]
            bamax = np.float32(np.abs(x).max())
            sf = (bamax / np.float32(6.0)) / np.float32(g)
            a = Fraction(float(sf))
            best = 126 if a >= 448 else min(range(127), key=lambda i: (abs(a - e4[i]), i % 2))
            assert s[r, b] == best, (r, b, float(sf))
            d = np.float32(O.e4m3_decode(int(s[r, b]))) * np.float32(g)
            for j in range(16):
                q = x[j] / d if d != 0 else np.float32(0)
                qa = Fraction(float(abs(q)))
                want = 7 if qa >= 6 else min(range(8), key=lambda i: (abs(qa - e2[i]), i % 2))
                code = int(n[r, 16 * b + j])
                assert code & 7 == want, (r, b, j, float(q))
                if d != 0:
                    assert (code >> 3) == int(np.signbit(q)), (r, b, j)


def test_random_rows_are_round_to_nearest():
    W = I.sweep_weights(2560, 9728, 3)[:3]                    # 3 rows of a t(4) matrix
    c, s, g = O.pack_nvfp4(W)
    _check_rtn(W, c, s, g)


def test_small_case_rows_are_round_to_nearest():
    W, _ = I.nvfp4_small()
    c, s, g = O.pack_nvfp4(W)
    rows = [0, 511, 1023]
    _check_rtn(W[rows], c[rows], s[rows], g)


def test_power_of_two_scaling_and_sign_symmetry():
    W = I.sweep_weights(2560, 1024, 1)[:16]
    c, s, g = O.pack_nvfp4(W)
    c2, s2, g2 = O.pack_nvfp4((W.double() * 8).to(torch.bfloat16))
    assert np.array_equal(c, c2) and np.array_equal(s, s2) and g2 == g * 8
    cn, sn, gn = O.pack_nvfp4(-W)
    assert np.array_equal(s, sn) and gn == g
    assert np.array_equal(nib(cn), nib(c) ^ 8)               # every code flips its sign bit


def test_dequant_error_bound():
    """RTN bound: |x - w_hat| <= half the local E2M1 gap times d (gap <= 2, so <= d),
    except saturated elements, which sit at most one E4M3 rounding above 6*d."""
    W = I.sweep_weights(4096, 2560, 2)[:32]
    c, s, g = O.pack_nvfp4(W)
    wh = O.dequant_nvfp4(c, s, g)
    d = np.repeat(np.array([O.e4m3_decode(int(v)) for v in s.ravel()]).reshape(s.shape), 16, axis=1) * g
    err = np.abs(W.double().numpy() - wh)
    assert np.all(err <= d * (1.0 + 6 / 16) + 1e-30)


def test_degenerate_zero_matrix_and_zero_blocks():
    c, s, g = O.pack_nvfp4(torch.zeros(4, 64, dtype=torch.bfloat16))
    assert g == 0 and not s.any() and not c.any()
    W = torch.zeros(2, 64, dtype=torch.float64)
    W[0, :16] = 1.0
    W[1, 40] = -3.0
    c, s, g = O.pack_nvfp4(W.to(torch.bfloat16))
    assert np.all(s[0, 1:] == 0) and np.all(s[1, [0, 1, 3]] == 0)
    assert np.all(c[0, 8:] == 0)


def test_nonfinite_input_is_rejected():
    W = torch.zeros(2, 32, dtype=torch.bfloat16)
    W[1, 3] = float("nan")
    with pytest.raises(O.OracleError):
        O.pack_nvfp4(W)
    W[1, 3] = float("inf")
    with pytest.raises(O.OracleError):
        O.pack_nvfp4(W)


def test_hand_worked_block():
    """A 16-element block worked by hand (the tensor has one block).
    absmax = 3, g = 3/2688 (binary32), (3/6)/g = 448 exactly -> scale 0x7E,
    d = 448 * g = 0.5 (binary32: 448 * fl(3/2688) rounds to 0.5), so code = E2M1(2x)."""
    x = [3.0, -3.0, 0.25, -0.25, 0.375, 0.625, 1.0, -1.5, 2.0, 2.5, 1.75, 0.0, -0.0, 0.125, 0.875, 1.25]
    c, s, g = O.pack_nvfp4(bf16([x]))
    assert s[0, 0] == 0x7E
    assert np.float32(448.0) * g == np.float32(0.5)
    # 2x = 6,-6,.5,-.5,.75,1.25,2,-3,4,5,3.5,0,-0,.25,1.75,2.5
    # -> E2M1 index: 7, 7|8, 1, 1|8, 2 (0.75 tie -> even index 2), 2 (1.25 tie -> 2),
    #    4, 5|8, 6, 6 (5 tie between 4 and 6 -> even index 6), 6 (3.5 tie -> 6),
    #    0, 8 (-0 keeps its sign), 0 (0.25 tie -> 0), 4 (1.75 tie -> 4), 4 (2.5 tie -> 4)
    want = [7, 15, 1, 9, 2, 2, 4, 13, 6, 6, 6, 0, 8, 0, 4, 4]
    assert list(nib(c)[0]) == want
    assert list(c[0]) == [want[i] | (want[i + 1] << 4) for i in range(0, 16, 2)]


def test_byte_count_fact():
    """EdgeRock card: 4-bit codes plus one 8-bit scale per 16 weights = 4.5 bits
    per weight (plus one 4-byte global scale per matrix)."""
    fact = [l.split() for l in open(os.path.join(GOLDEN, "rocmwhy_format_table.txt"))
            if l.startswith("nvfp4")][0]
    K, N = 2560, 8
    c, s, g = O.pack_nvfp4(torch.zeros(N, K, dtype=torch.bfloat16))
    bits = 8 * (c.nbytes + s.nbytes) / (K * N)
    assert bits == float(fact[4]) == 4.5
