"""Helpers for the GPU parity tests (CUDA library vs CPU oracle)."""
import numpy as np
import torch

import oracle as O
import w4a16_matmul_pack_b200 as W4


def np_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def oracle_packed(pw: "W4.PackedWeights"):
    """Packed bytes the GPU produced, as numpy, for the oracle's dequantiser."""
    if pw.fmt == W4.FMT_NVFP4:
        return np_of(pw.codes), np_of(pw.scales), np.float32(pw.global_scale.item())
    return np_of(pw.codes)


def oracle_w_hat(pw, n0=0, rows=None):
    if pw.fmt == W4.FMT_NVFP4:
        c, s, g = oracle_packed(pw)
        return O.dequant_nvfp4(c, s, g, n0, rows)
    return O.dequant_rocmfp4(np_of(pw.codes), pw.fmt, n0, rows)


def assert_within_tolerance(y_gpu: np.ndarray, y_ref: np.ndarray, a_ref: np.ndarray, rel=1e-3):
    """|y_gpu - y_ref| <= rel * sum_k |x_k w_hat_k|, elementwise."""
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bound = rel * a_ref
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (f"{len(bad)} outputs out of tolerance; first {bad[:3].tolist()}: "
                           f"err {err[tuple(bad[0])]:.3e} bound {bound[tuple(bad[0])]:.3e}")
    assert np.all(np.isfinite(y_gpu))
