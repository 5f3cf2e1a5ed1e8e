#!/usr/bin/env python
"""Benchmark of the W4A16 pack + matmul path on B200.

Headline (one JSON line from rank 0): W4A16 GEMV HBM GB/s at M=1 on the decode
GEMV sweep -- NVFP4 weights of the 4B-class decoder shapes (K, N) = (2560,4096),
(2560,1024), (4096,2560), (2560,9728), (9728,2560), Student-t(4) weights of std
0.02 with 0.01% of entries x20, BF16 activations N(0,1).  One step = one GEMV
over each of the five matrices, issued as one grouped launch
(w4a16_gemv_grouped); the steps of one rotation over the packed copies are
captured in one CUDA graph.  GB/s counts the packed bytes read (codes + scales
+ global scale, 4.5 bits per weight).  Every weight matrix has enough packed
copies that one rotation reads more than four times the 126 MB L2, so no step
finds its weights in L2.

The same line carries the other rows of the path, each measured in this run
with the same rotation rule and reported as the median of at least 50 timed
repeats with their min and max: the sweep as separate launches, each sweep
shape alone, the sweep at M = 4, 9 (speculative verify) and 16, the prefill
GEMM (M=2048, K=2560, N=9728, TFLOP/s), the 36-layer weight stream (tokens/s at
M=1, M=16 and looped; at M=1 also with q/k/v and gate/up grouped), the ROCmFP4
GEMV, the packers (NVFP4 abs-max and scale search, ROCmFP4 Dual / FAST,
importance-weighted, Q4_0), and the reconstruction-error quality report of
every format.  `--impl reference` times the CPU oracle on the same workload.

Multi-GPU: the path has no exchange step; `--gpus N` under torchrun runs N
independent replicas (weak scaling) and reports the summed bytes over the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMV HBM GB/s (M=1), GEMM TFLOP/s (M=2048), % of roofline"
WORKLOAD = ("decode GEMV sweep, NVFP4 W4A16, M=1, (K,N) in {(2560,4096),(2560,1024),(4096,2560),"
            "(2560,9728),(9728,2560)}, Student-t(4) std 0.02 weights with 0.01% x20, BF16 x ~ N(0,1)")
L2_BYTES = 126 * 1024 * 1024
ROTATE_BYTES = 4 * L2_BYTES + 1     # one rotation over the copies reads more than 4x L2
REPEATS = 60                        # individually timed repeats behind every median


def n_copies(nbytes: int) -> int:
    """Packed copies of an operand so that one rotation reads more than 4x L2."""
    return max(2, -(-ROTATE_BYTES // int(nbytes)))


def sweep_step_bytes() -> int:
    import w4a16_inputs as I
    return sum(N * (K // 2 + K // 16) + 4 for K, N in I.SWEEP_SHAPES)


def headline_config(world: int) -> dict:
    """The config both arms report (the same keys and values)."""
    nb = sweep_step_bytes()
    return {"workload": WORKLOAD, "M": 1,
            "step": "5 GEMVs in one grouped launch (programmatic dependent launch between steps); one rotation "
                    "of steps per CUDA graph",
            "l2": f"{n_copies(nb)} rotating packed copies per matrix ({n_copies(nb) * nb / 1e6:.0f} MB > 4x the "
                  f"126 MB L2)",
            "bytes_per_step": nb, "parallelism": f"replicas x{world}"}


# ----------------------------------------------------------------------------- util
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="headline only (skip GEMM/stream/packers)")
    ap.add_argument("--cpu-seconds", type=float, default=8.0, help="CPU oracle sample length")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class Clocks:
    """nvidia-smi sampling in the background (SM clock, max clock, throttle reasons)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = [l.split(", ") for l in open(self.f.name).read().strip().splitlines() if l.strip()]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) >= 9:
                for n, v in zip(names, r[5:9]):
                    if v.strip() == "Active":
                        reasons.add(n)
        busy = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)]
        return {"sm_mhz": statistics.median(busy or sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "note": "sampled every 100 ms over warm-up and timed steps"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    elif args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float, device="cuda") -> float:
    """The largest of each rank's v (device timings are combined as the slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, step_bytes: float, ms_total: float, steps: int) -> float:
    """Whole-job GB/s of `world` replicas that each process step_bytes per step,
    over the slowest rank's time for `steps` steps."""
    return world * step_bytes / (ms_total / steps) / 1e6


# ------------------------------------------------------------------ workloads (GPU)
def clone_packed(W4, base):
    return W4.PackedWeights(base.fmt, base.K, base.N, base.codes.clone(),
                            None if base.scales is None else base.scales.clone(),
                            None if base.global_scale is None else base.global_scale.clone())


def sweep_setup(W4, I, M=1):
    """The five sweep matrices, each with enough packed copies that one rotation
    over them reads more than 4x L2."""
    R = n_copies(sweep_step_bytes())
    mats = []
    for idx, (K, N) in enumerate(I.SWEEP_SHAPES):
        W = I.sweep_weights(K, N, idx, device="cuda")
        base = W4.pack_nvfp4(W)
        del W
        copies = [base] + [clone_packed(W4, base) for _ in range(R - 1)]
        x = I.sweep_x(M, K, idx, device="cuda")
        y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        mats.append({"K": K, "N": N, "copies": copies, "x": x, "y": y, "bytes": base.nbytes + 4})
    torch.cuda.synchronize()
    return mats


def capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm (sets kernel attributes outside capture)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_replays(graph, reps=REPEATS, warmup=3):
    """Milliseconds of each of `reps` replays, timed one by one with CUDA events
    on the replaying stream (after `warmup` untimed replays)."""
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record()
    for i in range(reps):
        graph.replay()
        ev[i + 1].record()
    torch.cuda.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]


def summary(ms_list, per: int = 1):
    """Median / min / max of repeat times, in us per unit (`per` units per repeat)."""
    v = sorted(m * 1e3 / per for m in ms_list)
    return {"median_us": round(statistics.median(v), 3), "min_us": round(v[0], 3), "max_us": round(v[-1], 3),
            "repeats": len(v)}


def rate(nbytes: float, st: dict, peak: float):
    gbs = nbytes / st["median_us"] / 1e3
    return {"GB/s": round(gbs, 1), "frac": round(gbs / peak, 4)}


def separate_sweep(W4, mats, pk):
    """The sweep as five w4a16_gemv launches per step (PDL-chained), one rotation per graph."""
    R = len(mats[0]["copies"])

    def run():
        for r in range(R):
            for m in mats:
                W4.w4a16_gemv(m["copies"][r], m["x"], out=m["y"], flags=W4.LAUNCH_PDL)
    g = capture(run)
    st = summary(time_replays(g, REPEATS), R)
    step_bytes = sum(m["bytes"] for m in mats)
    return {**st, **rate(step_bytes, st, pk["hbm_gbs"]), "launches_per_step": 5}


def per_shape(W4, mats, pk):
    """Each sweep shape alone: back-to-back launches over enough copies of that
    matrix to read more than 4x L2 per rotation."""
    out = {}
    for m in mats:
        R = n_copies(m["bytes"])
        copies = [m["copies"][i] if i < len(m["copies"]) else clone_packed(W4, m["copies"][0]) for i in range(R)]

        def run(copies=copies, m=m):
            for c in copies:
                W4.w4a16_gemv(c, m["x"], out=m["y"])
        g = capture(run)
        st = summary(time_replays(g, REPEATS), R)
        out[f"{m['K']}x{m['N']}"] = {**st, **rate(m["bytes"], st, pk["hbm_gbs"]), "copies": R}
        del g, copies
        torch.cuda.empty_cache()
    return out


def sweep_m_bench(W4, I, mats, pk):
    """The decode sweep at M = 4, 9 (a speculative-verify step: one token plus
    eight drafted ones) and 16 (same packed copies, PDL graph per rotation)."""
    out = {}
    R = len(mats[0]["copies"])
    for M in (4, 9, 16):
        xs = [I.sweep_x(M, m["K"], idx, device="cuda") for idx, m in enumerate(mats)]
        ys = [torch.empty(M, m["N"], dtype=torch.float32, device="cuda") for m in mats]
        ws = torch.empty(max(W4.w4a16_workspace_bytes(m["copies"][0], M) for m in mats) + 16,
                         dtype=torch.uint8, device="cuda")

        def run():
            for r in range(R):
                for m, x, y in zip(mats, xs, ys):
                    W4.w4a16_gemv(m["copies"][r], x, out=y, workspace=ws, flags=W4.LAUNCH_PDL)
        g = capture(run)
        st = summary(time_replays(g, REPEATS), R)
        nb = sum(m["bytes"] for m in mats)
        out[f"M{M}"] = {**st, **rate(nb, st, pk["hbm_gbs"])}
        del g
    return out


def rocm_gemv_bench(W4, I, pk):
    """ROCmFP4 GEMV on the 2560x9728 Laplace matrix, Dual and FAST, M = 1 and 8."""
    out = {}
    L = I.rocm_weights(device="cuda")
    for fmt in ("dual", "fast"):
        base = W4.pack_rocmfp4(L, fmt)
        nb = base.nbytes
        R = n_copies(nb)
        copies = [base] + [clone_packed(W4, base) for _ in range(R - 1)]
        for M in (1, 8):
            x = I.rocm_x(M, device="cuda")
            y = torch.empty(M, base.N, dtype=torch.float32, device="cuda")
            ws = torch.empty(W4.w4a16_workspace_bytes(base, M) + 16, dtype=torch.uint8, device="cuda")

            def run():
                for c in copies:
                    W4.w4a16_gemv(c, x, out=y, workspace=ws)
            g = capture(run)
            st = summary(time_replays(g, REPEATS), R)
            out[f"{fmt}_M{M}"] = {**st, **rate(nb, st, pk["hbm_gbs"]), "bytes": nb, "copies": R}
            del g
        del copies
        torch.cuda.empty_cache()
    return out


def gemm_bench(W4, I, pk):
    W, x = I.prefill(device="cuda")
    pw = W4.pack_nvfp4(W)
    del W
    M, K, N = 2048, 2560, 9728
    R = n_copies(pw.nbytes + x.numel() * 2)
    ws = [pw] + [clone_packed(W4, pw) for _ in range(R - 1)]
    xs = [x] + [x.clone() for _ in range(R - 1)]
    y16 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp = torch.empty(W4.w4a16_workspace_bytes(pw, M), dtype=torch.uint8, device="cuda")

    def run():
        for w_, x_ in zip(ws, xs):
            W4.w4a16_gemm(w_, x_, want_f32=False, out_bf16=y16, workspace=wsp)
    g = capture(run)
    st = summary(time_replays(g, REPEATS, warmup=2), R)
    flops = 2.0 * M * N * K
    tf = flops / st["median_us"] / 1e6
    out = {"config": f"M=2048 K=2560 N=9728, NVFP4 Student-t weights, x N(0,1) with 16 columns x30, out bf16 (the prefill activation), "
                     f"{R} rotating weight+x copies (> 4x L2); time per GEMM includes its x -> f16 pass",
           **st, "TFLOP/s": round(tf, 1), "frac": round(tf / pk["bf16_tflops"], 4), "peak": pk["bf16_tflops"],
           "peak_unit": f"TFLOP/s ({pk['source']} cuBLAS bf16 burst)"}
    del g, ws, xs
    return out


def rocm_gemm_bench(W4, I, pk):
    """ROCmFP4 prefill GEMM (Dual, FAST) on the 2560x9728 Laplace matrix, 2048 tokens, BF16 out."""
    L = I.rocm_weights(device="cuda")
    _, x = I.prefill(device="cuda")
    M, K, N = 2048, 2560, 9728
    out = {}
    for fmt in ("dual", "fast"):
        base = W4.pack_rocmfp4(L, fmt)
        R = n_copies(base.nbytes + x.numel() * 2)
        ws = [base] + [clone_packed(W4, base) for _ in range(R - 1)]
        xs = [x] + [x.clone() for _ in range(R - 1)]
        y16 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        wsp = torch.empty(W4.w4a16_workspace_bytes(base, M), dtype=torch.uint8, device="cuda")

        def run(ws=ws, xs=xs, y16=y16, wsp=wsp):
            for w_, x_ in zip(ws, xs):
                W4.w4a16_gemm(w_, x_, want_f32=False, out_bf16=y16, workspace=wsp)
        g = capture(run)
        st = summary(time_replays(g, REPEATS, warmup=2), R)
        tf = 2.0 * M * N * K / st["median_us"] / 1e6
        out[fmt] = {**st, "TFLOP/s": round(tf, 1), "frac": round(tf / pk["bf16_tflops"], 4)}
        del g, ws, xs
    out["config"] = ("M=2048 K=2560 N=9728, ROCmFP4 Laplace weights, out bf16, rotating weight+x copies (> 4x L2), "
                     "time per GEMM includes its x -> f16 pass")
    out["peak"] = pk["bf16_tflops"]
    return out


def stream_bench(W4, I):
    layers = []
    for L in range(I.N_LAYERS):
        row = []
        for j in range(len(I.LAYER)):
            W = I.stream_weights(L, j, device="cuda")
            row.append(W4.pack_nvfp4(W))
            del W
        layers.append(row)
    torch.cuda.synchronize()
    nbytes = sum(p.nbytes + 4 for row in layers for p in row)
    res = {}
    for M in (1, 16):
        xs = {K: I.activations(M, K, 6000 + K, device="cuda") for K in (2560, 4096, 9728)}
        ys = {N: torch.empty(M, N, dtype=torch.float32, device="cuda") for N in (1024, 2560, 4096, 9728)}
        ws = torch.empty(max(W4.w4a16_workspace_bytes(p, M) for p in layers[0]) + 16,
                         dtype=torch.uint8, device="cuda")
        for loops in (1, 2):
            def run():
                for row in layers:
                    for _ in range(loops):
                        for p in row:
                            W4.w4a16_gemv(p, xs[p.K], out=ys[p.N], workspace=ws, flags=W4.LAUNCH_PDL)
            g = capture(run)
            st = summary(time_replays(g, 20, warmup=2))
            key = f"M{M}" + ("_looped" if loops == 2 else "")
            ms = st["median_us"] / 1e3
            res[key] = {"tokens/s": round(M * 1e3 / ms, 1), "ms_per_token_pass": round(ms, 4),
                        "GB/s": round(loops * nbytes / ms / 1e6, 1), **st}
            del g
    # one token with the projections that share an input issued together:
    # {q,k,v} and {gate,up} as grouped launches, o and down alone (4 launches per layer)
    x1 = {K: I.activations(1, K, 6000 + K, device="cuda") for K in (2560, 4096, 9728)}
    y1 = [torch.empty(1, N, dtype=torch.float32, device="cuda") for (_, _, N) in I.LAYER]
    groups = [(0, 1, 2), (3,), (4, 5), (6,)]
    for loops in (1, 2):
        def run():
            for row in layers:
                for _ in range(loops):
                    for grp in groups:
                        if len(grp) == 1:
                            p = row[grp[0]]
                            W4.w4a16_gemv(p, x1[p.K], out=y1[grp[0]], flags=W4.LAUNCH_PDL)
                        else:
                            W4.w4a16_gemv_grouped([row[j] for j in grp], [x1[row[j].K] for j in grp],
                                                  outs=[y1[j] for j in grp], flags=W4.LAUNCH_PDL)
        g = capture(run)
        st = summary(time_replays(g, 20, warmup=2))
        ms = st["median_us"] / 1e3
        key = "M1_grouped" + ("_looped" if loops == 2 else "")
        res[key] = {"tokens/s": round(1e3 / ms, 1), "ms_per_token_pass": round(ms, 4),
                    "GB/s": round(loops * nbytes / ms / 1e6, 1), **st}
        del g
    res["packed_bytes_per_pass"] = nbytes
    res["config"] = ("36 layers x {q,k,v,o,gate,up,down}, NVFP4, one CUDA graph per token pass (2.04 GB > L2), "
                     "median of 20 passes; M1/M16: 7 launches per layer with PDL; M1_grouped: {q,k,v} and "
                     "{gate,up} grouped, 4 launches per layer")
    return res


def quality_report(W4, I):
    """Relative reconstruction error sum (W - w_hat)^2 / sum W^2 of every format
    on the 2560x9728 Student-t sweep matrix and the 2560x9728 Laplace matrix
    (the pages' quality-per-byte comparison, computed on the GPU in binary64)."""
    out = {}
    for name, W in (("student_t4_2560x9728", I.sweep_weights(2560, 9728, 3, device="cuda")),
                    ("laplace_2560x9728", I.rocm_weights(device="cuda"))):
        row = {}
        for fmt, bpw, pack in (("nvfp4_absmax", 4.5, lambda w: W4.pack_nvfp4(w)),
                               ("nvfp4_scale_search", 4.5, lambda w: W4.pack_nvfp4(w, scale_search=W4.SCALE_MSE)),
                               ("rocmfp4_dual", 4.5, lambda w: W4.pack_rocmfp4(w, "dual")),
                               ("rocmfp4_fast", 4.25, lambda w: W4.pack_rocmfp4(w, "fast")),
                               ("q4_0", 4.5, lambda w: W4.pack_q4_0(w))):
            e, q = W4.reconstruction_error(pack(W), W)
            row[fmt] = {"rel_sq_error": float(f"{e / q:.6g}"), "bits_per_weight": bpw}
        out[name] = row
        del W
    return out


def time_calls(fn, reps=11, warmup=2):
    """Milliseconds of each of `reps` calls of fn (CUDA events around each)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record()
    for i in range(reps):
        fn()
        ev[i + 1].record()
    torch.cuda.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]


def pack_bench(W4, I):
    """Each packer on a 2560 x 9728 matrix (the sweep's Student-t matrix for
    NVFP4, the Laplace matrix for ROCmFP4 and Q4_0); median of 11 calls.  For
    the HBM-bound packers GB/s counts bf16 read + packed bytes written."""
    out = {}
    W = I.sweep_weights(2560, 9728, 3, device="cuda")
    L = I.rocm_weights(device="cuda")
    n = W.numel()
    imp = torch.rand(L.shape[1], generator=torch.Generator().manual_seed(5)).cuda() * 2.0
    # preallocated outputs: the timed calls launch only the packer kernels
    cd = torch.empty(9728, 1280, dtype=torch.uint8, device="cuda")
    sc = torch.empty(9728, 160, dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    wsp = torch.empty(W4.pack_nvfp4_workspace_bytes(), dtype=torch.uint8, device="cuda")
    nv = W4.PackedWeights(W4.FMT_NVFP4, 2560, 9728, cd, sc, gs)
    blk18 = torch.empty(9728, 80, 18, dtype=torch.uint8, device="cuda")
    blk17 = torch.empty(9728, 80, 17, dtype=torch.uint8, device="cuda")
    legs = [
        ("pack_nvfp4", lambda: W4.pack_nvfp4(W, out=nv, workspace=wsp), "hbm", 2 + 0.5625),
        ("pack_q4_0", lambda: W4.pack_q4_0(L, out=blk18), "hbm", 2 + 0.5625),
        ("pack_rocmfp4_dual", lambda: W4.pack_rocmfp4(L, "dual", out=blk18), "search", None),
        ("pack_rocmfp4_fast", lambda: W4.pack_rocmfp4(L, "fast", out=blk17), "search", None),
        ("pack_rocmfp4_dual_weighted", lambda: W4.pack_rocmfp4(L, "dual", importance=imp, out=blk18), "search", None),
        ("pack_nvfp4_scale_search", lambda: W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE, out=nv, workspace=wsp),
         "search", None),
        ("pack_nvfp4_scale_search_weighted",
         lambda: W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE, importance=imp, out=nv, workspace=wsp), "search", None),
    ]
    for name, fn, kind, bpw in legs:
        st = summary(time_calls(fn))
        row = {"shape": "K=2560 N=9728", **st}
        if kind == "hbm":
            row["GB/s"] = round(n * bpw / st["median_us"] / 1e3, 1)
        else:
            row["candidate_evals/s"] = round(127 * n / st["median_us"] * 1e6, 1)
        out[name] = row
    return out


# ----------------------------------------------------------------------- CPU oracle
def oracle_sweep_setup(I):
    """The sweep matrices packed by the oracle itself (its inputs never come from the GPU)."""
    import oracle as O
    mats = []
    for idx, (K, N) in enumerate(I.SWEEP_SHAPES):
        c, s, g = O.pack_nvfp4(I.sweep_weights(K, N, idx))
        mats.append((c, s, g, I.sweep_x(1, K, idx), c.nbytes + s.nbytes + 4))
    return mats


def oracle_gemv_sample(mats, seconds: float):
    """Time the oracle's GEMV (dequantise + binary64 dot products) at M=1, whole
    sweep matrices in rotation, until `seconds` have passed (at least one pass)."""
    import oracle as O
    done_bytes, t0, n = 0, time.perf_counter(), 0
    while True:
        c, s, g, x, nb = mats[n % len(mats)]
        O.matmul(x, O.dequant_nvfp4(c, s, g))
        done_bytes += nb
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds and n >= len(mats):
            break
    return done_bytes / el / 1e9, n, el, O.max_threads()


def oracle_legs(I, seconds: float, mats):
    """The oracle's other CPU legs, each a bounded sample (about `seconds` of work)
    of the same workloads: the GEMV on one thread, the NVFP4 abs-max packer, the
    ROCmFP4 Dual packer (exhaustive 127-candidate search) and the binary64 GEMM
    of the prefill shape on a subsample of weight rows (time extrapolated
    linearly to all 9728 rows)."""
    import oracle as O
    cores = O.max_threads()
    legs = {}
    O.set_threads(1)
    try:
        gbs, n, el, _ = oracle_gemv_sample(mats, seconds)
    finally:
        O.set_threads(cores)
    legs["gemv_m1_1thread"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1,
                               "sample": f"{n} whole-matrix GEMVs over the 5 sweep matrices in {el:.1f} s"}

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    W = I.sweep_weights(2560, 9728, 3)
    rows = 4096
    el = timed(lambda: O.pack_nvfp4(W[:rows].contiguous()))
    legs["pack_nvfp4"] = {"value": round(rows * 2560 / el / 1e6, 2), "unit": "Mweights/s", "cores": cores,
                          "sample": f"abs-max pack of {rows} of the 9728 rows of the 2560-wide Student-t matrix "
                                    f"in {el:.2f} s"}
    L = I.rocm_weights()
    rows = 1024
    el = timed(lambda: O.pack_rocmfp4(L[:rows].contiguous(), O.FMT_DUAL))
    legs["pack_rocmfp4_dual"] = {"value": round(rows * 2560 / el / 1e6, 3), "unit": "Mweights/s", "cores": cores,
                                 "sample": f"Dual pack (127 candidates per half) of {rows} of the 9728 rows of the "
                                           f"2560-wide Laplace matrix in {el:.2f} s"}
    Wp, x = I.prefill()
    rows = 256
    c, s_, g = O.pack_nvfp4(Wp[:rows].contiguous())
    wh = O.dequant_nvfp4(c, s_, g)
    el = timed(lambda: O.matmul(x, wh))
    full_s = el * 9728 / rows
    legs["gemm_prefill"] = {"value": round(2.0 * 2048 * 2560 * rows / el / 1e9, 3), "unit": "GFLOP/s",
                            "cores": cores,
                            "sample": f"binary64 GEMM M=2048 K=2560 over {rows} of the 9728 weight rows in {el:.2f} s; "
                                      f"all rows extrapolated linearly: {full_s:.0f} s"}
    return legs


# ------------------------------------------------------------------------------ main
def run_ours(args, world, rank, local):
    import w4a16_inputs as I
    import w4a16_matmul_pack_b200 as W4
    from w4a16_matmul_pack_b200 import build as B
    if B.stale():
        B.build()
    pk = peaks()
    mats = sweep_setup(W4, I, M=1)
    R = len(mats[0]["copies"])
    step_bytes = sum(m["bytes"] for m in mats)
    assert step_bytes == sweep_step_bytes()

    xs, ys = [m["x"] for m in mats], [m["y"] for m in mats]

    def step_fn(r):
        def run():
            # programmatic dependent launch: a step streams its first weight
            # stages while the previous step drains, and reads x only after it
            W4.w4a16_gemv_grouped([m["copies"][r] for m in mats], xs, outs=ys, flags=W4.LAUNCH_PDL)
        return run
    graphs = [capture(step_fn(r)) for r in range(R)]
    # the R steps of one rotation in a single graph (one graph launch per R
    # steps); single-step graphs cover a remainder
    graph_rot = capture(lambda: [step_fn(r)() for r in range(R)])

    def run_steps(n):
        for _ in range(n // R):
            graph_rot.replay()
        for i in range(n % R):
            graphs[i].replay()

    clocks = Clocks(local)
    clocks.start()
    # untimed pre-heat (~1 s) so the timed steps run at load clocks, then W warm-up steps
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        run_steps(4 * R)
        torch.cuda.synchronize()
    run_steps(args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    run_steps(args.steps)
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ck = clocks.stop()
    ms_total = max_over_ranks(world, a.elapsed_time(b))
    ms_step = ms_total / args.steps
    value = replica_value(world, step_bytes, ms_total, args.steps)  # GB/s over all ranks
    launches = args.steps
    # distribution of the step time: REPEATS rotations timed one by one
    dist = summary(time_replays(graph_rot, REPEATS, warmup=2), R)

    # the step is one launch of the dominant kernel (the grouped M=1 GEMV)
    achieved = step_bytes / ms_step / 1e6
    traffic, traffic_note = measured_traffic()
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
            "kernel": "w4::gemv_nvfp4_m1_grouped_kernel",
            "note": f"one launch per step: algorithmic bytes of the 5 sweep matrices ({step_bytes} B) / "
                    f"average step duration over the timed steps (CUDA events on the launching stream); "
                    f"peak = {pk['source']} copy bandwidth ({'of measured' if pk['source'] == 'measured' else 'of fallback'}); "
                    f"{traffic_note}"}

    # end-to-end through the public API with pinned host buffers: the five x
    # (and the five y) lie back to back in one buffer on each side (every
    # piece starts on a 16-byte boundary), so a step moves one host -> device
    # copy of all x and one device -> host copy of all y
    kx = [m["K"] for m in mats]
    ny = [m["N"] for m in mats]
    xh_all = torch.cat([m["x"].reshape(-1).cpu() for m in mats]).pin_memory()
    yh_all = torch.empty(sum(ny), dtype=torch.float32).pin_memory()
    xd_all = torch.empty_like(xh_all, device="cuda")
    yd_all = torch.empty(sum(ny), dtype=torch.float32, device="cuda")
    xd = list(xd_all.split(kx))
    xd = [t.view(1, k) for t, k in zip(xd, kx)]
    yd = [t.view(1, n) for t, n in zip(yd_all.split(ny), ny)]
    xh, yh = [xh_all], [yh_all]
    e2e_steps = max(20, min(args.steps, 200))

    def e2e_step(r):
        xd_all.copy_(xh_all, non_blocking=True)
        W4.w4a16_gemv_grouped([m["copies"][r] for m in mats], xd, outs=yd)
        yh_all.copy_(yd_all, non_blocking=True)
        torch.cuda.synchronize()  # the step's result is read on the host
    for r in range(2):
        e2e_step(r)
    barrier(world)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record()
    for s_ in range(e2e_steps):
        e2e_step(s_ % R)
    eb.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, ea.elapsed_time(eb)) / e2e_steps
    e2e = {"value": round(world * step_bytes / e2e_ms / 1e6, 1), "unit": "GB/s",
           "h2d_bytes_per_step": sum(t.numel() * 2 for t in xh),
           "d2h_bytes_per_step": sum(t.numel() * 4 for t in yh),
           "note": "per step: the 5 x (one pinned buffer) -> device in one copy, one w4a16_gemv_grouped via the "
                   "Python binding of the C ABI (no graph), the 5 y -> one pinned host buffer in one copy, "
                   "synchronize; packed weights resident"}

    extras = {}

    def extra(name, fn):
        # one failing side measurement is recorded, not allowed to lose the headline line
        try:
            extras[name] = fn()
        except Exception as e:  # noqa: BLE001
            extras[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
        torch.cuda.empty_cache()

    if not args.no_extras:
        extra("sweep_separate_launches", lambda: separate_sweep(W4, mats, pk))
        extra("sweep_skinny", lambda: sweep_m_bench(W4, I, mats, pk))
        extra("per_shape_isolated", lambda: per_shape(W4, mats, pk))
        del graphs, graph_rot, mats
        torch.cuda.empty_cache()
        extra("gemm", lambda: gemm_bench(W4, I, pk))
        extra("gemm_rocmfp4", lambda: rocm_gemm_bench(W4, I, pk))
        extra("rocm_gemv", lambda: rocm_gemv_bench(W4, I, pk))
        extra("packers", lambda: pack_bench(W4, I))
        extra("quality", lambda: quality_report(W4, I))
        extra("stream", lambda: stream_bench(W4, I))
    err = W4.w4_device_error(clear=True)

    cpu = None
    if rank == 0 and world == 1:
        secs = max(2.0, args.cpu_seconds)
        omats = oracle_sweep_setup(I)
        gbs, n, el, cores = oracle_gemv_sample(omats, secs)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} whole-matrix oracle GEMVs (dequantise + fp64 dot) over the 5 sweep "
                         f"matrices at M=1 in {el:.1f} s"}
        if not args.no_extras:
            try:
                cpu["legs"] = oracle_legs(I, secs / 3, omats)
            except Exception as e:  # noqa: BLE001
                cpu["legs"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4-w/bf16-x/f32-acc",
                "data": "synthetic (seeded Student-t(4) weights, N(0,1) activations)",
                "config": headline_config(world), "step_time": dist,
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": ck, "device_error": err, **extras}
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    """The oracle as the reference arm: same metric, workload and config on the host cores."""
    if rank != 0:
        return
    import w4a16_inputs as I
    import oracle as O
    mats = oracle_sweep_setup(I)
    per_step = max(1.0, args.cpu_seconds / max(args.steps, 1))
    for _ in range(args.warmup):
        oracle_gemv_sample(mats, 0.0)
    vals, total_el = [], 0.0
    for _ in range(args.steps):
        gbs, n, el, cores = oracle_gemv_sample(mats, per_step)
        vals.append(gbs)
        total_el += el
    gbs = statistics.median(vals)
    sample = (f"per step: whole-matrix oracle GEMVs (dequantise + fp64 dot) over the 5 sweep matrices "
              f"at M=1 for >= {per_step:.1f} s; value = median over steps")
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_el / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(world),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": O.max_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# DRAM bytes (read + write, ncu dram__bytes_read.sum + dram__bytes_write.sum) of
# one launch of the dominant kernel, w4::gemv_nvfp4_m1_grouped_kernel, on the
# five sweep matrices, with the SHA-256 of the kernel sources it was measured
# on.  The bench reports it only while those sources are unchanged.
TRAFFIC = {"bytes": 41407488, "source_sha256": "3069d169f809520928beaa43fc45705d26d85d62d20ae0692f00e798c204e9db"}
TRAFFIC_SOURCES = ("common.cuh", "gemv_tc.cuh", "gemv_m1.cuh", "w4a16.cu")


def kernel_source_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "w4a16_matmul_pack_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic():
    sha = kernel_source_sha256()
    if TRAFFIC["bytes"] is not None and TRAFFIC["source_sha256"] == sha:
        return TRAFFIC["bytes"], "traffic = ncu DRAM bytes (read + write) of one launch, measured on these sources"
    return None, f"traffic = null: no ncu capture of the current kernel sources (sha256 {sha[:16]})"


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
