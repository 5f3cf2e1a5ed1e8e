"""CPU oracle for the W4A16 pack + matmul path (TEST INFRASTRUCTURE).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It wraps the plain C oracle in ``w4a16_oracle.c`` (built on
first use with gcc, ``-O2 -fopenmp -ffp-contract=off``) and shares no code with
the CUDA library.  Inputs and outputs are numpy arrays; bfloat16 tensors are
passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4a16_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FMT_NVFP4, FMT_DUAL, FMT_FAST, FMT_Q4_0 = 1, 2, 3, 4
BLOCK_BYTES = {FMT_DUAL: 18, FMT_FAST: 17, FMT_Q4_0: 18}


def build(force: bool = False) -> str:
    """Compile liboracle.so next to the source if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_decode.argtypes = [I]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [I]
        L.orc_cb10_decode.restype = ctypes.c_double
        L.orc_cb10_decode.argtypes = [I]
        L.orc_e2m1_encode.argtypes = [F]
        L.orc_e4m3_encode.argtypes = [F]
        L.orc_cb10_index.argtypes = [F, F]
        L.orc_pack_nvfp4.argtypes = [P, I, I, P, P, P]
        L.orc_pack_nvfp4_ex.argtypes = [P, I, I, I, P, P, P, P]
        L.orc_nvfp4_error.restype = F
        L.orc_nvfp4_error.argtypes = [P, P, I, F]
        L.orc_nvfp4_search.argtypes = [P, P, F, P]
        L.orc_rocm_error_w.restype = F
        L.orc_rocm_error_w.argtypes = [P, P, I, I]
        L.orc_rocm_search_w.argtypes = [P, P, I, P]
        L.orc_pack_rocmfp4_w.argtypes = [P, I, I, I, P, P]
        L.orc_fp16_decode.restype = ctypes.c_double
        L.orc_fp16_decode.argtypes = [I]
        L.orc_fp16_encode.argtypes = [F]
        L.orc_pack_q4_0.argtypes = [P, I, I, P]
        L.orc_dequant_q4_0.argtypes = [P, I, I, I, P]
        L.orc_reconstruction_sse.argtypes = [P, P, ctypes.c_longlong, P]
        L.orc_dequant_nvfp4.argtypes = [P, P, F, I, I, I, P]
        L.orc_rocm_error.restype = F
        L.orc_rocm_error.argtypes = [P, I, I]
        L.orc_rocm_search.argtypes = [P, I, P]
        L.orc_pack_rocmfp4.argtypes = [P, I, I, I, P]
        L.orc_dequant_rocmfp4.argtypes = [P, I, I, I, I, P]
        L.orc_matmul.argtypes = [P, I, I, P, I, P, P]
        L.orc_set_threads.argtypes = [I]
        L.orc_e4m3_encode_array.argtypes = [P, ctypes.c_longlong, P]
        L.orc_e2m1_encode_array.argtypes = [P, ctypes.c_longlong, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(W) -> np.ndarray:
    """bfloat16 tensor/array -> contiguous uint16 bit patterns."""
    if hasattr(W, "view") and hasattr(W, "dtype") and str(W.dtype) == "torch.bfloat16":
        import torch
        return W.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(W)
    assert a.dtype == np.uint16
    return a


class OracleError(RuntimeError):
    pass


def _check(rc: int):
    if rc != 0:
        raise OracleError({1: "bad argument", 5: "non-finite input"}.get(rc, f"status {rc}"))


# --- scalar formats ---------------------------------------------------------
def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def cb10_decode(code: int) -> float:
    return lib().orc_cb10_decode(code)


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(v)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(v)


def cb10_index(a: float, s: float) -> int:
    return lib().orc_cb10_index(a, s)


def e4m3_encode_array(v) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e2m1_encode_array(v) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().orc_e2m1_encode_array(_p(v), v.size, _p(out))
    return out


# --- packers ------------------------------------------------------------------
def _weights(imp, n):
    if imp is None:
        return None
    w = np.ascontiguousarray(imp, np.float32)
    assert w.size == n
    return w


def pack_nvfp4(W, mse: bool = False, importance=None):
    """W: bf16 [N][K] -> (codes u8 [N][K/2], scales u8 [N][K/16], global scale float32).
    mse: block scales by the error search (importance: K channel weights or None)."""
    b = _bits(W)
    N, K = b.shape
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 16), np.uint8)
    g = np.zeros(1, np.float32)
    w = _weights(importance, K)
    _check(lib().orc_pack_nvfp4_ex(_p(b), K, N, 1 if mse else 0, None if w is None else _p(w),
                                   _p(codes), _p(scales), _p(g)))
    return codes, scales, np.float32(g[0])


def nvfp4_error(x, u: int, g, importance=None) -> float:
    """Binary32 reconstruction error of 16 weights under E4M3 code u and global scale g."""
    x = np.ascontiguousarray(x, np.float32)
    assert x.size == 16
    w = _weights(importance, 16)
    return lib().orc_nvfp4_error(_p(x), None if w is None else _p(w), u, float(np.float32(g)))


def nvfp4_search(x, g, importance=None):
    """-> (best E4M3 code, its binary32 error) for 16 weights at global scale g."""
    x = np.ascontiguousarray(x, np.float32)
    assert x.size == 16
    w = _weights(importance, 16)
    e = np.zeros(1, np.float32)
    u = lib().orc_nvfp4_search(_p(x), None if w is None else _p(w), float(np.float32(g)), _p(e))
    return u, float(e[0])


def dequant_nvfp4(codes, scales, g, n0: int = 0, rows: int | None = None) -> np.ndarray:
    N, K = codes.shape[0], codes.shape[1] * 2
    rows = N - n0 if rows is None else rows
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequant_nvfp4(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                            float(g), K, n0, rows, _p(out))
    return out


def rocm_error(x, u: int, importance=None) -> float:
    x = np.ascontiguousarray(x, np.float32)
    w = _weights(importance, x.size)
    return lib().orc_rocm_error_w(_p(x), None if w is None else _p(w), x.size, u)


def rocm_search(x, importance=None):
    """-> (best UE4M3 code, its binary32 error)."""
    x = np.ascontiguousarray(x, np.float32)
    w = _weights(importance, x.size)
    e = np.zeros(1, np.float32)
    u = lib().orc_rocm_search_w(_p(x), None if w is None else _p(w), x.size, _p(e))
    return u, float(e[0])


def pack_rocmfp4(W, fmt: int, importance=None) -> np.ndarray:
    """W: bf16 [N][K] -> blocks u8 [N][K/32][18 (Dual) | 17 (FAST)]; importance:
    K channel weights (finite, >= 0) or None."""
    b = _bits(W)
    N, K = b.shape
    out = np.zeros((N, K // 32, BLOCK_BYTES[fmt]), np.uint8)
    w = _weights(importance, K)
    _check(lib().orc_pack_rocmfp4_w(_p(b), K, N, fmt, None if w is None else _p(w), _p(out)))
    return out


def dequant_rocmfp4(blocks, fmt: int, n0: int = 0, rows: int | None = None) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks)
    N, nb = blocks.shape[0], blocks.shape[1]
    K = nb * 32
    rows = N - n0 if rows is None else rows
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequant_rocmfp4(_p(blocks), fmt, K, n0, rows, _p(out))
    return out


def fp16_decode(h: int) -> float:
    return lib().orc_fp16_decode(h)


def fp16_encode(v: float) -> int:
    return lib().orc_fp16_encode(float(np.float32(v)))


def pack_q4_0(W) -> np.ndarray:
    """Stock Q4_0 (comparison format): W bf16 [N][K] -> blocks u8 [N][K/32][18]."""
    b = _bits(W)
    N, K = b.shape
    out = np.zeros((N, K // 32, 18), np.uint8)
    _check(lib().orc_pack_q4_0(_p(b), K, N, _p(out)))
    return out


def dequant_q4_0(blocks, n0: int = 0, rows: int | None = None) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks)
    N, nb = blocks.shape[0], blocks.shape[1]
    K = nb * 32
    rows = N - n0 if rows is None else rows
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequant_q4_0(_p(blocks), K, n0, rows, _p(out))
    return out


def reconstruction_sse(W, w_hat: np.ndarray):
    """-> (sum (W - w_hat)^2, sum W^2) in float64 over the whole matrix."""
    b = _bits(W)
    w = np.ascontiguousarray(w_hat, np.float64)
    assert w.shape == b.shape
    out = np.zeros(2, np.float64)
    lib().orc_reconstruction_sse(_p(b), _p(w), b.size, _p(out))
    return float(out[0]), float(out[1])


# --- matmul ---------------------------------------------------------------------
def matmul(x, w_hat: np.ndarray):
    """x: bf16 [M][K]; w_hat: float64 [R][K] -> (y [M][R], a [M][R]) in float64,
    with a = sum_k |x * w_hat| (the tolerance scale)."""
    xb = _bits(x)
    M, K = xb.shape
    w = np.ascontiguousarray(w_hat, np.float64)
    R = w.shape[0]
    y = np.zeros((M, R), np.float64)
    a = np.zeros((M, R), np.float64)
    lib().orc_matmul(_p(xb), M, K, _p(w), R, _p(y), _p(a))
    return y, a


def max_threads() -> int:
    return lib().orc_max_threads()


def set_threads(n: int) -> None:
    lib().orc_set_threads(n)
