"""Seeded synthetic inputs shared by the CPU oracle tests, the CUDA parity tests
and the benchmark.

This module holds no quantisation or matmul arithmetic: it only draws numbers.
Every value is a pure function of (seed, index), so the same tensor comes out on
the CPU and on a CUDA device, chunk by chunk, in any order.

Random source: the SplitMix64 output function (Steele, Lea & Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014) applied to a Weyl
sequence, used as a counter-based generator: word i of stream `key` is
mix(key + (i + 1) * 0x9E3779B97F4A7C15).  Distributions are drawn in float64
and rounded once, round-to-nearest-even, to bfloat16.

Workload shapes follow the 4B-class decoder of the EdgeRock-4B / Qwen3.5-4B
pages (hidden 2560, 16 query heads and 4 KV heads of width 256) with the
9728-wide MLP and 36 layers fixed for this library's benchmark.
"""
from __future__ import annotations

import math

import torch

_M64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_CHUNK = 1 << 22


def _s64(v: int) -> int:
    """Two's-complement view of a 64-bit unsigned constant (torch has no uint64 math)."""
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 words holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(_C1)
    z = (z ^ _srl(z, 27)) * _s64(_C2)
    return z ^ _srl(z, 31)


def _mix_int(v: int) -> int:
    v &= _M64
    v = ((v ^ (v >> 30)) * _C1) & _M64
    v = ((v ^ (v >> 27)) * _C2) & _M64
    return v ^ (v >> 31)


def stream_key(seed: int, purpose: int = 0) -> int:
    """Key of an independent stream for (seed, purpose)."""
    return _mix_int((seed * 64 + purpose) * _GOLDEN + 0x632BE59BD9B4E019)


def words(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """uint64 words start..start+count-1 of stream `key`, as int64 bit patterns."""
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _mix(i * _s64(_GOLDEN) + _s64(key))


def uniform(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """float64 uniforms in the open interval (0, 1): (top 53 bits + 0.5) / 2^53."""
    w = _srl(words(key, start, count, device), 11)
    return (w.to(torch.float64) + 0.5) * (2.0 ** -53)


def _normal(key, start, count, device):
    u = uniform(key, 2 * start, 2 * count, device).view(count, 2)
    return torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(2.0 * math.pi * u[:, 1])


def _student_t4(key, start, count, device):
    """Student-t with 4 degrees of freedom: Z / sqrt(V/4), V = -2 ln(U3 U4) ~ chi^2_4."""
    u = uniform(key, 4 * start, 4 * count, device).view(count, 4)
    z = torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(2.0 * math.pi * u[:, 1])
    v = -2.0 * torch.log(u[:, 2] * u[:, 3])
    return z / torch.sqrt(v / 4.0)


def _laplace(key, start, count, device):
    """Laplace(0, 1) by inversion."""
    v = uniform(key, start, count, device) - 0.5
    return -torch.sign(v) * torch.log1p(-2.0 * v.abs())


def bf16_rne(x: torch.Tensor) -> torch.Tensor:
    """Round float64 to bfloat16 once, to nearest, ties to even (no double rounding)."""
    m, e = torch.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    r = torch.ldexp(torch.round(m * 256.0), (e - 8).to(torch.float64))
    tiny = x.abs() < 2.0 ** -126                # bfloat16 subnormal range: fixed step 2^-133
    r = torch.where(tiny, torch.round(x * 2.0 ** 133) * 2.0 ** -133, r)
    return r.to(torch.float32).to(torch.bfloat16)


def distinct_positions(key: int, count: int, numel: int) -> torch.Tensor:
    """`count` distinct indices in [0, numel), first-drawn order (drawn on the CPU)."""
    out: list[int] = []
    seen: set[int] = set()
    start = 0
    while len(out) < count:
        w = words(key, start, 4 * count + 64)
        start += 4 * count + 64
        for v in (_srl(w, 1) % numel).tolist():
            if v not in seen:
                seen.add(v)
                out.append(v)
                if len(out) == count:
                    break
    return torch.tensor(out, dtype=torch.int64)


_DISTS = {"normal": _normal, "student_t4": _student_t4, "laplace": _laplace}


def matrix(dist: str, N: int, K: int, seed: int, scale: float, outlier_frac: float = 0.0,
           outlier_mult: float = 20.0, device="cpu") -> torch.Tensor:
    """bfloat16 weight matrix W[N][K] (row n holds output n; K contiguous).

    dist: "normal" (scale = std), "student_t4" (scale = std; t_4 has std sqrt(2)),
    "laplace" (scale = b).  outlier_frac of the entries (rounded to an integer
    count, distinct positions) are multiplied by outlier_mult in float64 before
    the single rounding to bfloat16.
    """
    gen = _DISTS[dist]
    mult = scale / math.sqrt(2.0) if dist == "student_t4" else scale
    key = stream_key(seed, 0)
    numel = N * K
    flat = torch.empty(numel, dtype=torch.float64, device=device)
    for s in range(0, numel, _CHUNK):
        c = min(_CHUNK, numel - s)
        flat[s:s + c] = gen(key, s, c, device) * mult
    n_out = int(round(outlier_frac * numel))
    if n_out:
        pos = distinct_positions(stream_key(seed, 1), n_out, numel).to(device)
        flat[pos] *= outlier_mult
    return bf16_rne(flat).view(N, K)


def activations(M: int, K: int, seed: int, outlier_cols: int = 0, outlier_mult: float = 30.0,
                device="cpu") -> torch.Tensor:
    """bfloat16 activations x[M][K] ~ N(0, 1); `outlier_cols` random columns scaled in float64."""
    key = stream_key(seed, 2)
    flat = _normal(key, 0, M * K, device).view(M, K)
    if outlier_cols:
        cols = distinct_positions(stream_key(seed, 3), outlier_cols, K).to(device)
        flat[:, cols] *= outlier_mult
    return bf16_rne(flat)


# ----------------------------------------------------------------------------
# Named workloads
# ----------------------------------------------------------------------------

#: Decode GEMV shapes (K, N) of the 4B-class decoder.
SWEEP_SHAPES = [(2560, 4096), (2560, 1024), (4096, 2560), (2560, 9728), (9728, 2560)]
SWEEP_M = (1, 4, 16)

#: One decoder layer in execution order: name, K (input width), N (output width).
LAYER = [("q", 2560, 4096), ("k", 2560, 1024), ("v", 2560, 1024), ("o", 4096, 2560),
         ("gate", 2560, 9728), ("up", 2560, 9728), ("down", 9728, 2560)]
N_LAYERS = 36


def nvfp4_small(device="cpu"):
    """1024x1024 N(0, 0.02) weights with 8 entries set to +-0.5, and x[1][1024] ~ N(0, 1)."""
    seed = 1000
    W = matrix("normal", 1024, 1024, seed, 0.02, device="cpu").to(torch.float64)
    pos = distinct_positions(stream_key(seed, 4), 8, 1024 * 1024)
    sign = torch.where(words(stream_key(seed, 5), 0, 8) < 0, -0.5, 0.5).to(torch.float64)
    W.view(-1)[pos] = sign
    x = activations(1, 1024, seed + 1)
    return bf16_rne(W).to(device), x.to(device)


def sweep_weights(K: int, N: int, index: int, device="cpu") -> torch.Tensor:
    """Student-t(4) weights of std 0.02 with 0.01% of entries x20."""
    return matrix("student_t4", N, K, 2000 + index, 0.02, 1e-4, 20.0, device=device)


def sweep_x(M: int, K: int, index: int, device="cpu") -> torch.Tensor:
    return activations(M, K, 2500 + 16 * index + M, device=device)


def rocm_weights(device="cpu") -> torch.Tensor:
    """2560x9728 (K x N) Laplace(0, b=0.015) weights with 0.01% of entries x20."""
    return matrix("laplace", 9728, 2560, 3000, 0.015, 1e-4, 20.0, device=device)


def rocm_x(M: int, device="cpu") -> torch.Tensor:
    return activations(M, 2560, 3500 + M, device=device)


def prefill(device="cpu"):
    """Prefill GEMM inputs: W[9728][2560] Student-t, x[2048][2560] with 16 columns x30."""
    W = matrix("student_t4", 9728, 2560, 4000, 0.02, 1e-4, 20.0, device=device)
    x = activations(2048, 2560, 4001, outlier_cols=16, outlier_mult=30.0, device=device)
    return W, x


def stream_weights(layer: int, j: int, device="cpu") -> torch.Tensor:
    """Weights of matrix j of decoder layer `layer` (own seed per matrix)."""
    _, K, N = LAYER[j]
    return matrix("student_t4", N, K, 5000 + 8 * layer + j, 0.02, 1e-4, 20.0, device=device)
