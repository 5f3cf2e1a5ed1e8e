#!/usr/bin/env python
"""Benchmark of the W4A16 pack + matmul path on B200.

Headline (one JSON line from rank 0): W4A16 GEMV HBM GB/s at M=1 on the decode
GEMV sweep -- NVFP4 weights of the 4B-class decoder shapes (K, N) = (2560,4096),
(2560,1024), (4096,2560), (2560,9728), (9728,2560), Student-t(4) weights of std
0.02 with 0.01% of entries x20, BF16 activations N(0,1).  One step = one GEMV
over each of the five matrices, issued as one grouped launch
(w4a16_gemv_grouped), six steps (one per rotating weight copy) captured in one
CUDA graph; the same sweep as five separate launches chained with programmatic
dependent launch is reported beside it.  GB/s counts the packed bytes read
(codes + scales + global scale, 4.5 bits per weight).  Six packed copies of
every matrix rotate across steps (248 MB > the 126 MB L2), so no step finds its
weights in L2.

The same line carries the other rows of the path, each measured in this run:
the sweep at M = 4, 9 (speculative verify) and 16, the prefill GEMM (M=2048,
K=2560, N=9728, TFLOP/s), the 36-layer weight stream (tokens/s at M=1, M=16
and looped; at M=1 also with q/k/v and gate/up grouped), each sweep shape timed
alone, the ROCmFP4 GEMV, the packers (NVFP4 abs-max and scale search, ROCmFP4
Dual / FAST, importance-weighted, Q4_0), and the reconstruction-error quality
report of every format.  `--impl reference` times the CPU oracle on the same
workload instead.

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
ROTATE = 6


# ----------------------------------------------------------------------------- util
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="headline only (skip GEMM/stream/packers)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample length")
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
def sweep_setup(W4, I, M=1):
    mats = []
    for idx, (K, N) in enumerate(I.SWEEP_SHAPES):
        W = I.sweep_weights(K, N, idx, device="cuda")
        base = W4.pack_nvfp4(W)
        del W
        copies = [base] + [W4.PackedWeights(base.fmt, K, N, base.codes.clone(), base.scales.clone(),
                                            base.global_scale.clone()) for _ in range(ROTATE - 1)]
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


def time_graphs(graphs, steps, warmup):
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(steps):
        graphs[i % len(graphs)].replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps  # ms per replay


def separate_sweep(W4, mats, reps=120):
    """The sweep as five w4a16_gemv launches per step (CUDA graph, PDL-chained)."""
    def step_fn(r):
        def run():
            for m in mats:
                W4.w4a16_gemv(m["copies"][r], m["x"], out=m["y"], flags=W4.LAUNCH_PDL)
        return run
    graphs = [capture(step_fn(r)) for r in range(ROTATE)]
    ms = time_graphs(graphs, reps, 2 * ROTATE)
    step_bytes = sum(m["bytes"] for m in mats)
    return {"us_per_step": round(ms * 1e3, 2), "GB/s": round(step_bytes / ms / 1e6, 1), "launches_per_step": 5}


def per_shape(W4, mats, reps=40):
    out = {}
    for m in mats:
        def run(m=m):
            for c in m["copies"]:
                W4.w4a16_gemv(c, m["x"], out=m["y"])
        g = capture(run)
        ms = time_graphs([g], reps, 5) / ROTATE
        out[f"{m['K']}x{m['N']}"] = {"us": round(ms * 1e3, 3), "GB/s": round(m["bytes"] / ms / 1e6, 1)}
    return out


def sweep_m_bench(W4, I, mats, pk):
    """The decode sweep at M = 4, 9 (a speculative-verify step: one token plus
    eight drafted ones) and 16 (same packed copies, PDL graph per step)."""
    out = {}
    for M in (4, 9, 16):
        xs = [I.sweep_x(M, m["K"], idx, device="cuda") for idx, m in enumerate(mats)]
        ys = [torch.empty(M, m["N"], dtype=torch.float32, device="cuda") for m in mats]
        ws = torch.empty(max(W4.w4a16_workspace_bytes(m["copies"][0], M) for m in mats) + 16,
                         dtype=torch.uint8, device="cuda")

        def step(r):
            def run():
                for m, x, y in zip(mats, xs, ys):
                    W4.w4a16_gemv(m["copies"][r], x, out=y, workspace=ws, flags=W4.LAUNCH_PDL)
            return run
        graphs = [capture(step(r)) for r in range(ROTATE)]
        ms = time_graphs(graphs, 60, 6)
        nb = sum(m["bytes"] for m in mats)
        out[f"M{M}"] = {"GB/s": round(nb / ms / 1e6, 1), "frac": round(nb / ms / 1e6 / pk["hbm_gbs"], 4),
                        "us_per_step": round(ms * 1e3, 2)}
        del graphs
    return out


def rocm_gemv_bench(W4, I, pk):
    """ROCmFP4 GEMV on the 2560x9728 Laplace matrix, Dual and FAST, M = 1 and 8."""
    out = {}
    L = I.rocm_weights(device="cuda")
    for fmt in ("dual", "fast"):
        base = W4.pack_rocmfp4(L, fmt)
        copies = [base] + [W4.PackedWeights(base.fmt, base.K, base.N, base.codes.clone()) for _ in range(ROTATE - 1)]
        nb = base.nbytes
        for M in (1, 8):
            x = I.rocm_x(M, device="cuda")
            y = torch.empty(M, base.N, dtype=torch.float32, device="cuda")
            ws = torch.empty(W4.w4a16_workspace_bytes(base, M) + 16, dtype=torch.uint8, device="cuda")

            def run():
                for c in copies:
                    W4.w4a16_gemv(c, x, out=y, workspace=ws)
            g = capture(run)
            ms = time_graphs([g], 20, 3) / ROTATE
            out[f"{fmt}_M{M}"] = {"us": round(ms * 1e3, 2), "GB/s": round(nb / ms / 1e6, 1),
                                  "frac": round(nb / ms / 1e6 / pk["hbm_gbs"], 4), "bytes": nb}
        del copies
    return out


def gemm_bench(W4, I, pk):
    W, x = I.prefill(device="cuda")
    pw = W4.pack_nvfp4(W)
    del W
    ws = [pw] + [W4.PackedWeights(pw.fmt, pw.K, pw.N, pw.codes.clone(), pw.scales.clone(),
                                  pw.global_scale.clone()) for _ in range(ROTATE - 1)]
    xs = [x] + [x.clone() for _ in range(ROTATE - 1)]
    M, K, N = 2048, 2560, 9728
    y32 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    y16 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")

    def run():
        for w_, x_ in zip(ws, xs):
            W4.w4a16_gemm(w_, x_, out_f32=y32, out_bf16=y16)
    g = capture(run)
    ms = time_graphs([g], 10, 2) / ROTATE
    flops = 2.0 * M * N * K
    tf = flops / ms / 1e9
    return {"config": "M=2048 K=2560 N=9728, NVFP4 Student-t weights, x N(0,1) with 16 columns x30, "
                      "out fp32+bf16, 6 rotating input copies",
            "us": round(ms * 1e3, 2), "TFLOP/s": round(tf, 1),
            "frac": round(tf / pk["bf16_tflops"], 4), "peak": pk["bf16_tflops"],
            "peak_unit": "TFLOP/s (measured cuBLAS bf16 burst)"}


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
            ms = time_graphs([g], 5, 2)
            key = f"M{M}" + ("_looped" if loops == 2 else "")
            res[key] = {"tokens/s": round(M * 1e3 / ms, 1), "ms_per_token_pass": round(ms, 4),
                        "GB/s": round(loops * nbytes / ms / 1e6, 1)}
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
                                                  outs=[y1[j] for j in grp])
        g = capture(run)
        ms = time_graphs([g], 5, 2)
        key = "M1_grouped" + ("_looped" if loops == 2 else "")
        res[key] = {"tokens/s": round(1e3 / ms, 1), "ms_per_token_pass": round(ms, 4),
                    "GB/s": round(loops * nbytes / ms / 1e6, 1)}
        del g
    res["packed_bytes_per_pass"] = nbytes
    res["config"] = ("36 layers x {q,k,v,o,gate,up,down}, NVFP4, one CUDA graph per token; M1/M16: 7 launches "
                     "per layer with PDL; M1_grouped: {q,k,v} and {gate,up} grouped, 4 launches per layer")
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


def pack_bench(W4, I):
    out = {}
    W = I.sweep_weights(2560, 9728, 3, device="cuda")
    Ws = [W] + [W.clone() for _ in range(2)]
    g = capture(lambda: [W4.pack_nvfp4(w) for w in Ws])
    ms = time_graphs([g], 10, 2) / len(Ws)
    out["pack_nvfp4"] = {"shape": "K=2560 N=9728", "us": round(ms * 1e3, 2),
                         "GB/s": round((W.numel() * 2 + W.numel() * 0.5625) / ms / 1e6, 1)}
    L = I.rocm_weights(device="cuda")
    for fmt in ("dual", "fast"):
        W4.pack_rocmfp4(L, fmt)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        W4.pack_rocmfp4(L, fmt)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        out[f"pack_rocmfp4_{fmt}"] = {"shape": "K=2560 N=9728 Laplace", "ms": round(ms, 3),
                                      "candidate_evals/s": round(127 * L.numel() / ms / 1e3, 1)}
    W4.pack_q4_0(L)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    W4.pack_q4_0(L)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    out["pack_q4_0"] = {"shape": "K=2560 N=9728 Laplace", "us": round(ms * 1e3, 2),
                        "GB/s": round((L.numel() * 2 + L.numel() * 0.5625) / ms / 1e6, 1)}
    imp = torch.rand(L.shape[1], generator=torch.Generator().manual_seed(5)).cuda() * 2.0
    W4.pack_rocmfp4(L, "dual", importance=imp)
    W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE)
    W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE, importance=imp)
    torch.cuda.synchronize()
    for name, fn in (("pack_rocmfp4_dual_weighted", lambda: W4.pack_rocmfp4(L, "dual", importance=imp)),
                     ("pack_nvfp4_scale_search", lambda: W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE)),
                     ("pack_nvfp4_scale_search_weighted",
                      lambda: W4.pack_nvfp4(W, scale_search=W4.SCALE_MSE, importance=imp))):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        out[name] = {"shape": "K=2560 N=9728", "ms": round(ms, 3),
                     "candidate_evals/s": round(127 * W.numel() / ms / 1e3, 1)}
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


# ------------------------------------------------------------------------------ main
def run_ours(args, world, rank, local):
    import w4a16_inputs as I
    import w4a16_matmul_pack_b200 as W4
    from w4a16_matmul_pack_b200 import build as B
    if B.stale():
        B.build()
    pk = peaks()
    mats = sweep_setup(W4, I, M=1)
    step_bytes = sum(m["bytes"] for m in mats)

    xs, ys = [m["x"] for m in mats], [m["y"] for m in mats]

    def step_fn(r):
        def run():
            W4.w4a16_gemv_grouped([m["copies"][r] for m in mats], xs, outs=ys)
        return run
    graphs = [capture(step_fn(r)) for r in range(ROTATE)]
    # the ROTATE steps of one rotation in a single graph (one graph launch per
    # ROTATE steps); single-step graphs cover a remainder
    graph_rot = capture(lambda: [step_fn(r)() for r in range(ROTATE)])

    def run_steps(n):
        for _ in range(n // ROTATE):
            graph_rot.replay()
        for i in range(n % ROTATE):
            graphs[i].replay()

    clocks = Clocks(local)
    clocks.start()
    # untimed pre-heat (~1 s) so the timed steps run at load clocks, then W warm-up steps
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        run_steps(60)
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

    # the step is one launch of the dominant kernel (the grouped M=1 GEMV)
    achieved = step_bytes / ms_step / 1e6
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": TRAFFIC_PER_LAUNCH,
            "kernel": "w4::gemv_nvfp4_m1_grouped_kernel",
            "note": f"one launch per step: algorithmic bytes of the 5 sweep matrices ({step_bytes} B) / "
                    f"average step duration in the timed graphs (CUDA events on the launching stream); "
                    f"peak = {pk['source']} copy bandwidth; traffic = ncu DRAM bytes of one launch"}

    # end-to-end through the public API with pinned host buffers
    xh = [m["x"].cpu().pin_memory() for m in mats]
    yh = [torch.empty_like(m["y"], device="cpu").pin_memory() for m in mats]
    xd = [torch.empty_like(m["x"]) for m in mats]
    e2e_steps = max(20, min(args.steps, 200))
    def e2e_step(r):
        for i in range(len(mats)):
            xd[i].copy_(xh[i], non_blocking=True)
        W4.w4a16_gemv_grouped([m["copies"][r] for m in mats], xd, outs=ys)
        for i in range(len(mats)):
            yh[i].copy_(ys[i], non_blocking=True)
        torch.cuda.synchronize()  # the step's result is read on the host
    for r in range(2):
        e2e_step(r)
    barrier(world)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record()
    for s in range(e2e_steps):
        e2e_step(s % ROTATE)
    eb.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, ea.elapsed_time(eb)) / e2e_steps
    e2e = {"value": round(world * step_bytes / e2e_ms / 1e6, 1), "unit": "GB/s",
           "h2d_bytes_per_step": sum(t.numel() * 2 for t in xh),
           "d2h_bytes_per_step": sum(t.numel() * 4 for t in yh),
           "note": "per step: 5 pinned x -> device, one w4a16_gemv_grouped via the Python binding of the "
                   "C ABI (no graph), 5 y -> pinned host, synchronize; packed weights resident"}

    extras = {}

    def extra(name, fn):
        # one failing side measurement is recorded, not allowed to lose the headline line
        try:
            extras[name] = fn()
        except Exception as e:  # noqa: BLE001
            extras[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
        torch.cuda.empty_cache()

    if not args.no_extras:
        extra("sweep_separate_launches", lambda: separate_sweep(W4, mats))
        extra("per_shape_isolated", lambda: per_shape(W4, mats))
        extra("sweep_skinny", lambda: sweep_m_bench(W4, I, mats, pk))
        del graphs, graph_rot, mats
        torch.cuda.empty_cache()
        extra("gemm", lambda: gemm_bench(W4, I, pk))
        extra("packers", lambda: pack_bench(W4, I))
        extra("quality", lambda: quality_report(W4, I))
        extra("rocm_gemv", lambda: rocm_gemv_bench(W4, I, pk))
        extra("stream", lambda: stream_bench(W4, I))
    err = W4.w4_device_error(clear=True)

    cpu = None
    if rank == 0 and world == 1:
        gbs, n, el, cores = oracle_gemv_sample(oracle_sweep_setup(I), args.cpu_seconds)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} whole-matrix oracle GEMVs (dequantise + fp64 dot) over the 5 sweep "
                         f"matrices at M=1 in {el:.1f} s"}
    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4-w/bf16-x/f32-acc",
                "data": "synthetic (seeded Student-t(4) weights, N(0,1) activations)",
                "config": {"workload": WORKLOAD, "M": 1,
                           "step": f"5 GEMVs in one grouped launch; {ROTATE} steps per CUDA graph",
                           "l2": f"{ROTATE} rotating packed copies per matrix (248 MB > L2)",
                           "bytes_per_step": step_bytes, "parallelism": f"replicas x{world}"},
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": ck, "device_error": err, **extras}
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    """The oracle as the reference arm: same metric and workload on the host cores."""
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
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_el / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": 1},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": O.max_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ncu-measured DRAM bytes (read + write) of one launch of the dominant kernel,
# w4::gemv_nvfp4_m1_grouped_kernel, on the five sweep matrices
# (profiles/gemv_nvfp4_m1_grouped_sweep.md).
# Set to None when that kernel changes until it is measured again.
TRAFFIC_PER_LAUNCH = 41381888


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
