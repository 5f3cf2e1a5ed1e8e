"""The measurement contract of bench.py, checked without a GPU: the headline's
algorithmic bytes follow from the packed layout (0.5 B of codes + 1/16 B of
E4M3 scale per weight, 4 B of global scale per matrix), every rotation reads
more than 4x the L2, and the measured DRAM traffic is reported only for the
kernel sources it was measured on."""
import importlib.util
import os

import pytest

import w4a16_inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_headline_bytes_are_the_packed_layout(bench):
    weights = sum(K * N for K, N in I.SWEEP_SHAPES)
    assert bench.sweep_step_bytes() == weights * 9 // 16 + 4 * len(I.SWEEP_SHAPES) == 41_287_700
    cfg = bench.headline_config(1)
    assert cfg["bytes_per_step"] == 41_287_700 and cfg["M"] == 1


@pytest.mark.parametrize("nbytes", [1, 1_474_564, 14_008_324, 41_287_700, 213_000_000, 10 ** 9])
def test_rotation_reads_more_than_four_l2(bench, nbytes):
    r = bench.n_copies(nbytes)
    assert r >= 2 and r * nbytes > 4 * 126 * 1024 * 1024
    if r > 2:   # no more copies than needed
        assert (r - 1) * nbytes <= 4 * 126 * 1024 * 1024


def test_traffic_only_for_the_measured_sources(bench, monkeypatch):
    sha = bench.kernel_source_sha256()
    monkeypatch.setattr(bench, "TRAFFIC", {"bytes": 123, "source_sha256": sha})
    assert bench.measured_traffic()[0] == 123
    monkeypatch.setattr(bench, "TRAFFIC", {"bytes": 123, "source_sha256": "0" * 64})
    value, note = bench.measured_traffic()
    assert value is None and "null" in note
