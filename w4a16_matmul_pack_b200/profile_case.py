"""Run one operation of the library on one shape a few times (for profilers).

    python -m w4a16_matmul_pack_b200.profile_case gemv --fmt nvfp4 --K 2560 --N 9728 --M 1 --reps 3
    python -m w4a16_matmul_pack_b200.profile_case gemm --M 2048 --K 2560 --N 9728 --reps 2
    python -m w4a16_matmul_pack_b200.profile_case pack --fmt dual --K 2560 --N 9728
    python -m w4a16_matmul_pack_b200.profile_case pack --fmt nvfp4 --search [--importance]
    python -m w4a16_matmul_pack_b200.profile_case q4_0 --K 9728 --N 9728
    python -m w4a16_matmul_pack_b200.profile_case recon --fmt nvfp4 --K 9728 --N 9728
    python -m w4a16_matmul_pack_b200.profile_case grouped --reps 3

`grouped` runs the five decode-sweep matrices (K,N) = (2560,4096), (2560,1024),
(4096,2560), (2560,9728), (9728,2560) at one token as one grouped launch.

Inputs are the seeded synthetic matrices (Student-t weights, N(0,1) x; Laplace
weights for ROCmFP4 and Q4_0).  Exits non-zero on any library or CUDA error.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import w4a16_inputs as I  # noqa: E402
import w4a16_matmul_pack_b200 as W4  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["gemv", "gemm", "pack", "grouped", "q4_0", "recon"])
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "dual", "fast"])
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--K", type=int, default=2560)
    ap.add_argument("--N", type=int, default=9728)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--search", action="store_true", help="pack: NVFP4 block scales by error search")
    ap.add_argument("--importance", action="store_true", help="pack: importance-weighted search")
    ap.add_argument("--flags", type=int, default=0, help="launch flags of the GEMV (1 = W4_LAUNCH_PDL)")
    a = ap.parse_args()
    torch.cuda.set_device(0)
    if a.op == "grouped":
        ws = [W4.pack_nvfp4(I.sweep_weights(K, N, i, device="cuda")) for i, (K, N) in enumerate(I.SWEEP_SHAPES)]
        xs = [I.sweep_x(1, K, i, device="cuda") for i, (K, _) in enumerate(I.SWEEP_SHAPES)]
        torch.cuda.synchronize()
        for _ in range(a.reps):
            W4.w4a16_gemv_grouped(ws, xs, flags=a.flags)
        finish()
        return
    if a.fmt == "nvfp4" and a.op != "q4_0":
        W = I.matrix("student_t4", a.N, a.K, 7, 0.02, 1e-4, 20.0, device="cuda")
    else:
        W = I.matrix("laplace", a.N, a.K, 7, 0.015, 1e-4, 20.0, device="cuda")
    imp = None
    if a.importance:
        imp = torch.rand(a.K, generator=torch.Generator().manual_seed(5)).cuda() * 2.0
    if a.op == "pack":
        for _ in range(a.reps):
            if a.fmt == "nvfp4":
                W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE if a.search else W4.SCALE_ABSMAX, importance=imp)
            else:
                W4.pack_rocmfp4(W, a.fmt, importance=imp)
    elif a.op == "q4_0":
        for _ in range(a.reps):
            W4.pack_q4_0(W)
    elif a.op == "recon":
        pw = W4.pack_nvfp4(W) if a.fmt == "nvfp4" else W4.pack_rocmfp4(W, a.fmt)
        for _ in range(a.reps):
            W4.reconstruction_error(pw, W)
    else:
        x = I.activations(a.M, a.K, 8, device="cuda")
        pw = W4.pack_nvfp4(W) if a.fmt == "nvfp4" else W4.pack_rocmfp4(W, a.fmt)
        torch.cuda.synchronize()
        for _ in range(a.reps):
            if a.op == "gemv":
                W4.w4a16_gemv(pw, x, flags=a.flags)
            else:
                W4.w4a16_gemm(pw, x)
    finish()


def finish():
    torch.cuda.synchronize()
    err = W4.w4_device_error(clear=True)
    if err:
        print(f"device error word: {err}")
        sys.exit(1)
    print("ok")


if __name__ == "__main__":
    main()
