"""The C-ABI library loads without a GPU and exports every entry point that
include/w4a16.h declares; host-side argument checks answer before any launch."""
import ctypes
import os
import re

import pytest
import torch

import w4a16_matmul_pack_b200 as W4
from w4a16_matmul_pack_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return W4.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "w4a16.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"pack_nvfp4", "pack_rocmfp4", "w4a16_gemv", "w4a16_gemm"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(8):
        assert lib.w4_status_string(s).decode().startswith("W4_")
    assert b"sm_100a" in lib.w4_version()


def test_host_validation_without_gpu(lib):
    P = ctypes.c_void_p
    # null matrix / bad block size / bad format: rejected before any CUDA call
    assert lib.pack_nvfp4(None, 64, 4, 16, 0, P(16), P(16), P(16), P(16), 16, None, None) == 1
    assert lib.pack_nvfp4(P(16), 64, 4, 32, 0, P(16), P(16), P(16), P(16), 16, None, None) == 1
    assert lib.pack_nvfp4(P(16), 64, 4, 16, 2, P(16), P(16), P(16), P(16), 16, None, None) == 1
    # importance weights only with the scale search, and 16-byte aligned
    assert lib.pack_nvfp4_ex(P(16), 64, 4, 16, 0, P(16), P(16), P(16), P(16), P(16), 16, None, None) == 1
    assert lib.pack_nvfp4_ex(P(16), 64, 4, 16, 1, P(20), P(16), P(16), P(16), P(16), 16, None, None) == 2
    assert lib.pack_nvfp4(P(16), 64, 4, 16, 0, P(16), P(16), P(16), P(16), 4, None, None) == 7
    assert lib.pack_nvfp4(P(17), 64, 4, 16, 0, P(16), P(16), P(16), P(16), 16, None, None) == 2
    assert lib.pack_rocmfp4(P(16), 48, 4, 32, 2, None, P(16), None, None) == 1
    assert lib.pack_rocmfp4(P(16), 64, 4, 32, 9, None, P(16), None, None) == 1
    assert lib.pack_rocmfp4(P(16), 64, 4, 32, 2, P(20), P(16), None, None) == 2
    # the Q4_0 packer and the reconstruction report
    assert lib.pack_q4_0(P(16), 64, 4, 16, P(16), None, None) == 1          # block must be 32
    assert lib.pack_q4_0(P(16), 48, 4, 32, P(16), None, None) == 1          # K % 32
    assert lib.pack_q4_0(P(16), 64, 4, 32, P(24), None, None) == 2          # alignment
    q = W4._Weights(4, 64, 4, 16, None, None)
    ws = lib.w4_reconstruction_workspace_bytes()
    assert ws >= 16
    assert lib.w4_reconstruction_error(ctypes.byref(q), None, P(16), P(16), ws, None) == 1
    assert lib.w4_reconstruction_error(ctypes.byref(q), P(16), P(16), P(16), ws - 1, None) == 7
    assert lib.w4_reconstruction_error(ctypes.byref(q), P(16), P(24), P(16), ws, None) == 2
    bad_k = W4._Weights(4, 48, 4, 16, None, None)
    assert lib.w4_reconstruction_error(ctypes.byref(bad_k), P(16), P(16), P(16), ws, None) == 1
    # Q4_0 is scored, not multiplied
    assert lib.w4a16_gemv(ctypes.byref(q), P(16), 1, P(16), None, 0, None) == 3
    assert lib.w4a16_gemm(ctypes.byref(q), P(16), 64, P(16), None, None, 0, None) == 3
    w = W4._Weights(1, 256, 8, 16, 16, 16)
    assert lib.w4a16_gemv(ctypes.byref(w), P(16), 17, P(16), None, 0, None) == 1
    assert lib.w4a16_gemv(ctypes.byref(w), P(16), 0, P(16), None, 0, None) == 1
    assert lib.w4a16_gemv(ctypes.byref(w), P(24), 1, P(16), None, 0, None) == 2
    bad = W4._Weights(7, 256, 8, 16, 16, 16)
    assert lib.w4a16_gemv(ctypes.byref(bad), P(16), 1, P(16), None, 0, None) == 1
    assert lib.w4a16_gemm(ctypes.byref(w), P(16), 4, None, None, None, 0, None) == 1


def test_python_binding_refuses_cpu_tensors():
    with pytest.raises(ValueError):
        W4.pack_nvfp4(torch.zeros(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        W4.pack_rocmfp4(torch.zeros(4, 64, dtype=torch.bfloat16), "dual")


def declared_parameter_counts():
    """name -> number of parameters, from the prototypes in include/w4a16.h."""
    text = open(os.path.join(ROOT, "include", "w4a16.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(([^)]*)\)\s*;", text, re.M):
        params = " ".join(m.group(2).split())
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(lib):
    """Every function the Python binding declares to ctypes takes as many
    arguments as its prototype in the header."""
    counts = declared_parameter_counts()
    bound = [n for n in counts if getattr(lib, n).argtypes is not None]
    assert {"pack_nvfp4_ex", "pack_q4_0", "w4a16_gemv_grouped", "w4_plan_grouped",
            "w4_reconstruction_error"} <= set(bound)
    for name in bound:
        assert len(getattr(lib, name).argtypes) == counts[name], name
