"""The CUDA packers' binary32 -> E4M3 / E2M1 conversions agree with the
oracle's encoders (round to nearest even, saturating, sign kept)."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a16_matmul_pack_b200 as W4

pytestmark = pytest.mark.gpu


def _values():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=1 << 21, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    # dense coverage of the ranges that matter: |v| in [2^-12, 2^10]
    e = rng.uniform(-12, 10, size=1 << 21)
    w = (np.exp2(e) * rng.choice([-1, 1], size=e.size)).astype(np.float32)
    grid4 = np.array([O.e4m3_decode(i) for i in range(127)])
    mids4 = ((grid4[1:] + grid4[:-1]) / 2).astype(np.float32)
    grid2 = np.array([O.e2m1_decode(i) for i in range(8)])
    mids2 = ((grid2[1:] + grid2[:-1]) / 2).astype(np.float32)
    edges = np.concatenate([mids4, grid4.astype(np.float32), mids2, grid2.astype(np.float32),
                            np.float32([0.0, -0.0, 448, 464, 1e30, -1e30, np.inf, -np.inf])])
    around = np.concatenate([np.nextafter(edges, np.float32(np.inf)), np.nextafter(edges, np.float32(-np.inf))])
    allv = np.concatenate([v, w, edges, -edges, around, -around]).astype(np.float32)
    return allv


def test_encoders_match_oracle():
    v = _values()
    e4, e2 = W4.w4_encode_scalars(torch.from_numpy(v).cuda())
    e4, e2 = e4.cpu().numpy(), e2.cpu().numpy()
    r4, r2 = O.e4m3_encode_array(v), O.e2m1_encode_array(v)
    bad4 = np.nonzero(e4 != r4)[0]
    bad2 = np.nonzero(e2 != r2)[0]
    assert bad4.size == 0, [(float(v[i]), int(e4[i]), int(r4[i])) for i in bad4[:8]]
    assert bad2.size == 0, [(float(v[i]), int(e2[i]), int(r2[i])) for i in bad2[:8]]
