"""Property checks of the oracle's scale searches on random blocks (hypothesis):
the chosen code's error is the minimum over all 127 candidates, ties go to the
smallest code, the abs-max NVFP4 scale is never better, and uniform weights
change nothing ("rocmwhy" page, section 03: finite scale candidates scored by
reconstruction error with optional importance weighting)."""
import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle as O

finite_bf16 = st.floats(min_value=-50.0, max_value=50.0, allow_nan=False, width=32).map(
    lambda v: float(torch.tensor(v).to(torch.bfloat16).float()))
weights = st.floats(min_value=0.0, max_value=4.0, allow_nan=False, width=32)


@settings(max_examples=60, deadline=None)
@given(x=st.lists(finite_bf16, min_size=16, max_size=16), w=st.lists(weights, min_size=16, max_size=16),
       gexp=st.integers(min_value=-14, max_value=-2))
def test_nvfp4_search_is_the_minimum(x, w, gexp):
    x = np.array(x, np.float32)
    w = np.array(w, np.float32)
    g = np.float32(max(float(np.abs(x).max()), 1e-3) / 2688.0 * 2.0 ** (gexp + 8))
    for imp in (None, w):
        u, e = O.nvfp4_search(x, g, imp)
        errs = [O.nvfp4_error(x, v, g, imp) for v in range(127)]
        assert e == errs[u] == min(errs)
        assert u == errs.index(min(errs))
    # the abs-max rule's code is one of the candidates
    s_abs = O.e4m3_encode(float(np.float32(np.float32(np.abs(x).max()) / np.float32(6.0)) / g)) if g != 0 else 0
    if s_abs <= 126:
        assert O.nvfp4_search(x, g)[1] <= O.nvfp4_error(x, s_abs, g)


@settings(max_examples=60, deadline=None)
@given(x=st.lists(finite_bf16, min_size=16, max_size=32), c=st.floats(min_value=0.25, max_value=4.0, width=32))
def test_rocm_search_is_the_minimum_and_uniform_weights_change_nothing(x, c):
    x = np.array(x, np.float32)
    u, e = O.rocm_search(x)
    errs = [O.rocm_error(x, v) for v in range(127)]
    assert e == errs[u] == min(errs) and u == errs.index(min(errs))
    # a uniform weight c multiplies every candidate's error terms alike
    cw = np.full(x.size, np.float32(2.0) ** int(np.round(np.log2(c))), np.float32)   # a power of two: exact
    uw, ew = O.rocm_search(x, cw)
    assert uw == u and ew == e * float(cw[0])


@settings(max_examples=60, deadline=None)
@given(x=st.lists(finite_bf16, min_size=32, max_size=32))
def test_q4_0_block_properties(x):
    """Stock Q4_0 ("rocmwhy" format table; signed abs-max scale, integer steps):
    the largest weight sits at -8, every code is the nearest integer step to its
    weight within the clamp, and the block reconstructs within half a step."""
    W = torch.tensor([x], dtype=torch.float32).to(torch.bfloat16)
    blk = O.pack_q4_0(W)[0, 0]
    d = O.fp16_decode(int(blk[0]) | int(blk[1]) << 8)
    codes = [int(blk[2 + (j & 15)] >> (4 * (j >> 4))) & 15 for j in range(32)]
    xs = W.float().numpy()[0]
    jm = int(np.argmax(np.abs(xs)))
    if d == 0.0:
        assert all(c == 8 for c in codes)
        return
    assert codes[jm] == 0
    wh = O.dequant_q4_0(O.pack_q4_0(W))[0]
    for j in range(32):
        q = float(xs[j]) / d
        if -8.0 <= q <= 7.0:
            assert abs(float(xs[j]) - wh[j]) <= abs(d) * (0.5 + 1e-6)
