"""The versioned on-disk format of packed weights (host only): round trips are
byte-exact for every format, and corrupt or foreign headers are refused."""
import struct

import numpy as np
import pytest
import torch

import oracle as O
import w4a16_inputs as I
import w4a16_matmul_pack_b200 as W4


def cpu_packed(fmt, N=5, K=64):
    W = I.matrix("student_t4", N, K, 3, 0.02, 1e-3)
    if fmt == W4.FMT_NVFP4:
        c, s, g = O.pack_nvfp4(W)
        return W4.PackedWeights(fmt, K, N, torch.from_numpy(c), torch.from_numpy(s),
                                torch.tensor([g], dtype=torch.float32))
    if fmt == W4.FMT_Q4_0:
        return W4.PackedWeights(fmt, K, N, torch.from_numpy(O.pack_q4_0(W)))
    return W4.PackedWeights(fmt, K, N, torch.from_numpy(O.pack_rocmfp4(W, fmt)))


@pytest.mark.parametrize("fmt", [W4.FMT_NVFP4, W4.FMT_ROCMFP4_DUAL, W4.FMT_ROCMFP4_FAST, W4.FMT_Q4_0])
def test_round_trip(tmp_path, fmt):
    pw = cpu_packed(fmt)
    p = tmp_path / "w.bin"
    W4.save_packed(pw, p)
    back = W4.load_packed(p, device="cpu")
    assert (back.fmt, back.K, back.N) == (pw.fmt, pw.K, pw.N)
    for a, b in ((pw.codes, back.codes), (pw.scales, back.scales), (pw.global_scale, back.global_scale)):
        assert (a is None and b is None) or torch.equal(a, b)


def test_refuses_corrupt_files(tmp_path):
    pw = cpu_packed(W4.FMT_NVFP4)
    p = tmp_path / "w.bin"
    W4.save_packed(pw, p)
    raw = bytearray(p.read_bytes())
    for patch in ((0, b"X"), (7, bytes([2])), (12, struct.pack("<i", 63)), (24, struct.pack("<q", 1))):
        bad = bytearray(raw)
        bad[patch[0]:patch[0] + len(patch[1])] = patch[1]
        q = tmp_path / "bad.bin"
        q.write_bytes(bytes(bad))
        with pytest.raises(ValueError):
            W4.load_packed(q, device="cpu")
    (tmp_path / "short.bin").write_bytes(bytes(raw[:-1]))
    with pytest.raises(ValueError):
        W4.load_packed(tmp_path / "short.bin", device="cpu")
    with pytest.raises(ValueError):
        W4.save_packed(W4.PackedWeights(W4.FMT_NVFP4, 64, 5, pw.codes[:4], pw.scales, pw.global_scale),
                       tmp_path / "x.bin")
