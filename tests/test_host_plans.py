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


def test_sweep_shares_by_bytes():
    ws = [FakeNvfp4(K, N) for K, N in I.SWEEP_SHAPES]
    ctas = W4.plan_grouped(ws, 148)
    assert sum(ctas) == 148
    for w, c in zip(ws, ctas):
        assert 1 <= c <= math.ceil(w.N / 16)
    ideal = sum(packed_bytes(w) for w in ws) / 148
    per_cta = [packed_bytes(w) / c for w, c in zip(ws, ctas)]
    assert max(per_cta) <= 1.1 * ideal          # the heaviest CTA stays close to an even share
    # one more CTA for the heaviest problem would have to come from a problem
    # whose CTAs would then carry more than the heaviest does now
    p = max(range(len(ws)), key=lambda i: per_cta[i])
    for q in range(len(ws)):
        if q != p and ctas[q] > 1:
            assert packed_bytes(ws[q]) / (ctas[q] - 1) >= per_cta[p] * 0.999


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
