"""Host logic without a GPU: how w4a16_gemv_grouped shares the SMs out among
its problems (w4_plan_grouped runs the same host code as the launch, with the
SM count given instead of queried)."""
import math

import pytest

import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4


class FakeNvfp4:
    """Weights descriptor with aligned dummy addresses: planning never touches memory."""

    def __init__(self, K, N, fmt=W4.FMT_NVFP4):
        self.K, self.N, self.fmt = K, N, fmt

    def struct(self):
        return W4._Weights(self.fmt, self.K, self.N, 1 << 12, 1 << 13, 1 << 14)


def packed_bytes(w):
    return w.N * (w.K // 2 + w.K // 16)


def tile_bytes(w):
    return 16 * (w.K // 2 + w.K // 16)


def heaviest_cta(ws, ctas):
    """Bytes of the most loaded CTA: CTAs take balanced ranges of whole tiles."""
    return max(math.ceil(math.ceil(w.N / 16) / c) * tile_bytes(w) for w, c in zip(ws, ctas))


def best_load(ws, sms):
    """Brute force over every possible load (a whole number of one problem's tiles)."""
    best = None
    for w in ws:
        for k in range(1, math.ceil(w.N / 16) + 1):
            L = k * tile_bytes(w)
            need = sum(math.ceil(math.ceil(v.N / 16) / max(1, L // tile_bytes(v))) for v in ws)
            if need <= sms and (best is None or L < best):
                best = L
    return best


@pytest.mark.parametrize("sms", [148, 132, 100, 37])
def test_sweep_minimises_the_heaviest_cta(sms):
    ws = [FakeNvfp4(K, N) for K, N in I.SWEEP_SHAPES]
    ctas = W4.plan_grouped(ws, sms)
    assert sum(ctas) == sms
    for w, c in zip(ws, ctas):
        assert 1 <= c <= math.ceil(w.N / 16)
    assert heaviest_cta(ws, ctas) == best_load(ws, sms)
    # close to an even share of the bytes
    assert heaviest_cta(ws, ctas) <= 1.25 * sum(packed_bytes(w) for w in ws) / sms


def test_mixed_shapes_minimise_the_heaviest_cta():
    ws = [FakeNvfp4(4096, 4096), FakeNvfp4(4096, 1024), FakeNvfp4(16384, 4096), FakeNvfp4(1024, 14336)]
    ctas = W4.plan_grouped(ws, 148)
    assert heaviest_cta(ws, ctas) == best_load(ws, 148)


def test_caps_and_small_problems():
    ws = [FakeNvfp4(2560, 16), FakeNvfp4(256, 8), FakeNvfp4(9728, 2560)]
    ctas = W4.plan_grouped(ws, 148)
    assert ctas[0] == 1 and ctas[1] == 1                 # one 16-row tile each
    assert ctas[2] == 146                                # the rest, under its 160-tile cap
    assert sum(W4.plan_grouped([FakeNvfp4(512, 32)] * 3, 148)) == 3 * 2   # total capped by the tiles


def test_more_problems_than_sms():
    ws = [FakeNvfp4(1024, 1024)] * 8
    assert W4.plan_grouped(ws, 4) == [1] * 8             # every problem still gets a CTA


def test_plan_argument_errors():
    w = FakeNvfp4(512, 64)
    with pytest.raises(W4.W4Error):
        W4.plan_grouped([w] * 9, 148)
    with pytest.raises(W4.W4Error):
        W4.plan_grouped([w], 0)
    with pytest.raises(W4.W4Error):
        W4.plan_grouped([w], 148, 2)                     # unknown flag
    with pytest.raises(W4.W4Error):
        W4.plan_grouped([FakeNvfp4(512, 64, W4.FMT_ROCMFP4_DUAL)], 148)
