"""Python binding of libw4a16.so -- block-scaled 4-bit weight-only (W4A16) linear
layers on B200 (sm_100a).

Argument marshalling only: every step runs in the CUDA kernels behind the C ABI
declared in ``include/w4a16.h``.  PyTorch supplies device memory and streams.
The functions keep the C names:

    pack_nvfp4(W)            -> PackedWeights   (NVFP4: E2M1 + E4M3/16 + FP32 global)
    pack_rocmfp4(W, fmt)     -> PackedWeights   (ROCmFP4 Dual / FAST, Codebook10)
    w4a16_gemv(w, x)         -> y float32 [M][N]  (decode, M <= 16)
    w4a16_gemm(w, x)         -> (y float32, y bf16) (prefill)

There is no CPU fallback: if the library is missing the import of a function
raises, and every call requires CUDA tensors.
"""
from __future__ import annotations

import ctypes
import os
import struct
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "W4Error", "PackedWeights", "FMT_NVFP4", "FMT_ROCMFP4_DUAL", "FMT_ROCMFP4_FAST", "FMT_Q4_0",
    "pack_q4_0", "reconstruction_error", "plan_grouped",
    "LAUNCH_PDL", "set_wait_limit", "pack_nvfp4", "pack_rocmfp4", "w4a16_gemv", "w4a16_gemv_grouped", "w4a16_gemm",
    "w4a16_workspace_bytes", "pack_nvfp4_workspace_bytes", "w4_encode_scalars", "save_packed", "load_packed",
    "w4_device_error", "lib", "library_path",
]

FMT_NVFP4, FMT_ROCMFP4_DUAL, FMT_ROCMFP4_FAST, FMT_Q4_0 = 1, 2, 3, 4
SCALE_ABSMAX, SCALE_MSE = 0, 1
LAUNCH_PDL = 1
BLOCK_BYTES = {FMT_ROCMFP4_DUAL: 18, FMT_ROCMFP4_FAST: 17}
_FMT_NAMES = {"nvfp4": FMT_NVFP4, "dual": FMT_ROCMFP4_DUAL, "fast": FMT_ROCMFP4_FAST}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libw4a16.so")


def library_path() -> str:
    return _LIB_PATH


class W4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().w4_status_string(status).decode()}")


class _Weights(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("K", ctypes.c_int), ("N", ctypes.c_int),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("global_scale", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m w4a16_matmul_pack_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, U, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
        WP = ctypes.POINTER(_Weights)
        sig = {
            "pack_nvfp4": ([P, I, I, I, I, P, P, P, P, S, P, P], I),
            "pack_nvfp4_ex": ([P, I, I, I, I, P, P, P, P, P, S, P, P], I),
            "pack_q4_0": ([P, I, I, I, P, P, P], I),
            "w4_plan_grouped": ([P, I, I, U, P], I),
            "w4_reconstruction_error": ([WP, P, P, P, S, P], I),
            "w4_reconstruction_workspace_bytes": ([], S),
            "pack_nvfp4_workspace_bytes": ([], S),
            "pack_rocmfp4": ([P, I, I, I, I, P, P, P, P], I),
            "w4a16_gemv": ([WP, P, I, P, P, S, P], I),
            "w4a16_gemv_ex": ([WP, P, I, P, P, S, U, P], I),
            "w4a16_gemv_grouped": ([WP, P, P, I, U, P], I),
            "w4a16_gemm": ([WP, P, I, P, P, P, S, P], I),
            "w4a16_workspace_bytes": ([WP, I], S),
            "w4_encode_scalars": ([P, S, P, P, P], I),
            "w4_device_error": ([ctypes.POINTER(ctypes.c_int), I], I),
            "w4_set_wait_limit": ([ctypes.c_ulonglong], I),
            "w4_status_string": ([I], ctypes.c_char_p),
            "w4_version": ([], ctypes.c_char_p),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != 0:
        raise W4Error(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class PackedWeights:
    """A packed K x N weight matrix (layout in include/w4a16.h)."""
    fmt: int
    K: int
    N: int
    codes: torch.Tensor                   # uint8: NVFP4 [N][K/2]; ROCmFP4 [N][K/32][18|17]
    scales: Optional[torch.Tensor] = None  # uint8 [N][K/16] (NVFP4)
    global_scale: Optional[torch.Tensor] = None  # float32 [1] (NVFP4)

    def struct(self) -> _Weights:
        return _Weights(self.fmt, self.K, self.N, self.codes.data_ptr(),
                        None if self.scales is None else self.scales.data_ptr(),
                        None if self.global_scale is None else self.global_scale.data_ptr())

    @property
    def nbytes(self) -> int:
        n = self.codes.numel()
        if self.scales is not None:
            n += self.scales.numel()
        return n


# Packed weights on disk: a 64-byte little-endian header, then the codes, the
# scales and the global scale as stored in memory.  Header: magic "W4A16PK",
# layout version (1), then int32 fmt, K, N, block, and int64 byte counts of
# codes, scales and global scale.
_MAGIC = b"W4A16PK"
_LAYOUT_VERSION = 1
_HEADER = struct.Struct("<7sB4i3q")


def _expected_bytes(fmt: int, K: int, N: int):
    if fmt == FMT_NVFP4:
        return N * K // 2, N * K // 16, 4
    if fmt in BLOCK_BYTES or fmt == FMT_Q4_0:
        return N * (K // 32) * (18 if fmt in (FMT_ROCMFP4_DUAL, FMT_Q4_0) else 17), 0, 0
    raise ValueError(f"unknown format {fmt}")


def save_packed(w: "PackedWeights", path) -> None:
    """Write packed weights with a versioned header (format, K, N, block, sizes)."""
    parts = [w.codes, w.scales, w.global_scale]
    raw = [b"" if t is None else t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes() for t in parts]
    if tuple(len(r) for r in raw) != _expected_bytes(w.fmt, w.K, w.N):
        raise ValueError("packed tensors do not match their format and shape")
    block = 16 if w.fmt == FMT_NVFP4 else 32
    with open(path, "wb") as f:
        f.write(_HEADER.pack(_MAGIC, _LAYOUT_VERSION, w.fmt, w.K, w.N, block, *(len(r) for r in raw)))
        f.write(b"\0" * (64 - _HEADER.size))
        for r in raw:
            f.write(r)


def load_packed(path, device="cuda") -> "PackedWeights":
    """Read packed weights written by save_packed; refuses unknown versions and
    headers whose sizes do not match the format and shape."""
    with open(path, "rb") as f:
        head = f.read(64)
        if len(head) != 64:
            raise ValueError("truncated header")
        magic, ver, fmt, K, N, block, nc, ns, ng = _HEADER.unpack(head[:_HEADER.size])
        if magic != _MAGIC or ver != _LAYOUT_VERSION:
            raise ValueError(f"not a packed-weights file of layout version {_LAYOUT_VERSION}")
        if K <= 0 or N <= 0 or block != (16 if fmt == FMT_NVFP4 else 32) or K % block:
            raise ValueError("bad shape in header")
        if (nc, ns, ng) != _expected_bytes(fmt, K, N):
            raise ValueError("byte counts do not match the format and shape")
        data = [f.read(n) for n in (nc, ns, ng)]
        if [len(d) for d in data] != [nc, ns, ng] or f.read(1):
            raise ValueError("truncated or oversized payload")
    def t(b, shape, dtype):
        return torch.frombuffer(bytearray(b), dtype=torch.uint8).view(dtype).reshape(shape).to(device)
    if fmt == FMT_NVFP4:
        return PackedWeights(fmt, K, N, t(data[0], (N, K // 2), torch.uint8), t(data[1], (N, K // 16), torch.uint8),
                             t(data[2], (1,), torch.float32))
    bb = nc // (N * (K // 32))
    return PackedWeights(fmt, K, N, t(data[0], (N, K // 32, bb), torch.uint8))


def pack_nvfp4_workspace_bytes() -> int:
    return lib().pack_nvfp4_workspace_bytes()


def pack_nvfp4(W: torch.Tensor, *, scale_search: int = SCALE_ABSMAX, importance: Optional[torch.Tensor] = None,
               out: Optional[PackedWeights] = None, workspace: Optional[torch.Tensor] = None,
               d_status: Optional[torch.Tensor] = None, stream=None) -> PackedWeights:
    """Quantise bf16 W[N][K] to NVFP4 (see pack_nvfp4 / pack_nvfp4_ex in include/w4a16.h);
    importance: float32 [K] channel weights for the W4_SCALE_MSE search."""
    _cuda(W, "W", torch.bfloat16)
    if importance is not None:
        _cuda(importance, "importance", torch.float32)
    N, K = W.shape
    dev = W.device
    if out is None:
        out = PackedWeights(FMT_NVFP4, K, N,
                            torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
                            torch.empty(N, K // 16, dtype=torch.uint8, device=dev),
                            torch.empty(1, dtype=torch.float32, device=dev))
    if workspace is None:
        workspace = torch.empty(pack_nvfp4_workspace_bytes(), dtype=torch.uint8, device=dev)
    _check(lib().pack_nvfp4_ex(_ptr(W), K, N, 16, scale_search, _ptr(importance), _ptr(out.codes),
                               _ptr(out.scales), _ptr(out.global_scale), _ptr(workspace), workspace.numel(),
                               _ptr(d_status), _stream(stream)), "pack_nvfp4_ex")
    return out


def pack_rocmfp4(W: torch.Tensor, fmt="dual", *, importance: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, d_status: Optional[torch.Tensor] = None,
                 stream=None) -> PackedWeights:
    """Quantise bf16 W[N][K] to ROCmFP4 Dual ("dual") or FAST ("fast"); importance:
    float32 [K] channel weights for the error search, or None."""
    fmt = _FMT_NAMES.get(fmt, fmt)
    _cuda(W, "W", torch.bfloat16)
    if importance is not None:
        _cuda(importance, "importance", torch.float32)
    N, K = W.shape
    if fmt not in BLOCK_BYTES:
        raise ValueError("fmt must be 'dual' or 'fast'")
    if out is None:
        out = torch.empty(N, K // 32, BLOCK_BYTES[fmt], dtype=torch.uint8, device=W.device)
    _check(lib().pack_rocmfp4(_ptr(W), K, N, 32, fmt, _ptr(importance), _ptr(out), _ptr(d_status),
                              _stream(stream)),
           "pack_rocmfp4")
    return PackedWeights(fmt, K, N, out)


def pack_q4_0(W: torch.Tensor, *, out: Optional[torch.Tensor] = None, d_status: Optional[torch.Tensor] = None,
              stream=None) -> PackedWeights:
    """Stock Q4_0, the comparison format (see pack_q4_0 in include/w4a16.h)."""
    _cuda(W, "W", torch.bfloat16)
    N, K = W.shape
    if out is None:
        out = torch.empty(N, K // 32, 18, dtype=torch.uint8, device=W.device)
    _check(lib().pack_q4_0(_ptr(W), K, N, 32, _ptr(out), _ptr(d_status), _stream(stream)), "pack_q4_0")
    return PackedWeights(FMT_Q4_0, K, N, out)


def reconstruction_error(w: PackedWeights, W: torch.Tensor, *, workspace: Optional[torch.Tensor] = None,
                         stream=None):
    """(sum (W - w_hat)^2, sum W^2) in binary64 for a packed matrix and its bf16
    source (see w4_reconstruction_error); reads the two numbers back to the host."""
    _cuda(W, "W", torch.bfloat16)
    out = torch.empty(2, dtype=torch.float64, device=W.device)
    if workspace is None:
        workspace = torch.empty(lib().w4_reconstruction_workspace_bytes(), dtype=torch.uint8, device=W.device)
    s = w.struct()
    _check(lib().w4_reconstruction_error(ctypes.byref(s), _ptr(W), _ptr(out), _ptr(workspace), workspace.numel(),
                                         _stream(stream)), "w4_reconstruction_error")
    e, q = out.tolist()
    return e, q


def w4a16_workspace_bytes(w: PackedWeights, M: int) -> int:
    s = w.struct()
    return lib().w4a16_workspace_bytes(ctypes.byref(s), M)


def w4a16_gemv(w: PackedWeights, x: torch.Tensor, *, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, flags: int = 0, stream=None) -> torch.Tensor:
    """y[M][N] = x[M][K] . w_hat for M <= 16 (float32 output)."""
    _cuda(x, "x", torch.bfloat16)
    M = x.shape[0]
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.float32, device=x.device)
    need = w4a16_workspace_bytes(w, M)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    s = w.struct()
    _check(lib().w4a16_gemv_ex(ctypes.byref(s), _ptr(x), M, _ptr(out), _ptr(workspace),
                               0 if workspace is None else workspace.numel(), flags, _stream(stream)),
           "w4a16_gemv")
    return out


def plan_grouped(ws, sms: int, flags: int = 0):
    """Host only: the CTAs w4a16_gemv_grouped gives each problem on `sms` SMs."""
    G = len(ws)
    structs = (_Weights * G)(*[w.struct() for w in ws])
    out = (ctypes.c_int * G)()
    _check(lib().w4_plan_grouped(ctypes.cast(structs, ctypes.c_void_p), G, sms, flags,
                                 ctypes.cast(out, ctypes.c_void_p)), "w4_plan_grouped")
    return list(out)


def w4a16_gemv_grouped(ws, xs, *, outs=None, flags: int = 0, stream=None):
    """Several one-token NVFP4 GEMVs in one launch: returns [y_p[1][N_p] float32]."""
    G = len(ws)
    if len(xs) != G or (outs is not None and len(outs) != G):
        raise W4Error(-1, "w4a16_gemv_grouped: ws, xs and outs must have the same length")
    for x in xs:
        _cuda(x, "x", torch.bfloat16)
    if outs is None:
        outs = [torch.empty(1, w.N, dtype=torch.float32, device=xs[0].device) for w in ws]
    structs = (_Weights * G)(*[w.struct() for w in ws])
    xp = (ctypes.c_void_p * G)(*[_ptr(x) for x in xs])
    yp = (ctypes.c_void_p * G)(*[_ptr(y) for y in outs])
    _check(lib().w4a16_gemv_grouped(structs, ctypes.cast(xp, ctypes.c_void_p), ctypes.cast(yp, ctypes.c_void_p), G,
                                    flags, _stream(stream)), "w4a16_gemv_grouped")
    return outs


def w4a16_gemm(w: PackedWeights, x: torch.Tensor, *, want_f32: bool = True, want_bf16: bool = True,
               out_f32: Optional[torch.Tensor] = None, out_bf16: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None):
    """Prefill GEMM: returns (y float32 or None, y bf16 or None)."""
    _cuda(x, "x", torch.bfloat16)
    M = x.shape[0]
    if want_f32 and out_f32 is None:
        out_f32 = torch.empty(M, w.N, dtype=torch.float32, device=x.device)
    if want_bf16 and out_bf16 is None:
        out_bf16 = torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    need = w4a16_workspace_bytes(w, M)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    s = w.struct()
    _check(lib().w4a16_gemm(ctypes.byref(s), _ptr(x), M, _ptr(out_f32), _ptr(out_bf16), _ptr(workspace),
                            0 if workspace is None else workspace.numel(), _stream(stream)), "w4a16_gemm")
    return out_f32, out_bf16


def w4_encode_scalars(v: torch.Tensor, stream=None):
    """Elementwise float32 -> (E4M3 byte, E2M1 nibble) with the packers' rounding."""
    _cuda(v, "v", torch.float32)
    e4 = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    e2 = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(lib().w4_encode_scalars(_ptr(v), v.numel(), _ptr(e4), _ptr(e2), _stream(stream)),
           "w4_encode_scalars")
    return e4, e2


def set_wait_limit(ns: int = 0):
    """Limit (ns) of the device-side waits that gate progress, on the current
    device; 0 restores the default (2 s).  For exercising failure detection."""
    _check(lib().w4_set_wait_limit(ns), "w4_set_wait_limit")


def w4_device_error(clear: bool = True) -> int:
    """Sticky device error word of the current device (0 = none)."""
    out = ctypes.c_int(0)
    _check(lib().w4_device_error(ctypes.byref(out), 1 if clear else 0), "w4_device_error")
    return out.value
