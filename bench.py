#!/usr/bin/env python
"""Benchmark of the block-sparse linear layer on B200.

Default workload: the large LLM-MLP forward (X[8192,4096] bf16, W[14336,4096]
in 64x64 blocks at density 0.1 with Zipf(1.1)-skewed block rows).  One step
is one forward pass Y = X W^T of one batch through the C ABI (bsl_forward);
the weight is packed once before timing, as the pages' layer fixes its
sparsity pattern at initialisation (pytorch_block_sparse release note,
"Future Development Roadmap": patterns are fixed at initialisation), and the
pack is timed separately (``config.pack_ms``).

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun): every rank runs an
independent replica of the workload (the layer is not sharded: replicas
only), ``value`` is the sum over ranks of the work divided by the slowest
rank's time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # fp64 CPU oracle on a bounded sample
  python bench.py --kernel-only fwd|dx|dw --workload NAME --reps R
      # runs one contraction R times on one input copy (for ncu captures)

``--workload semi24_fwd`` measures the 2:4 semi-structured layer instead
(X[8192,4096], W[14336,4096] with two of every four weights kept, compressed
once before timing; one step is one forward through bsl_semi24_forward), and
``--workload bsr24_fwd`` the block-sparse layer with 2:4 inside its kept
blocks (the large workload's shape and mask kind; bsl_bsr24_forward).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "block-sparse GEMM effective TFLOP/s, % roofline, speedup vs dense at 75/90% sparse"
UNIT = "TFLOP/s"
METRIC_SEMI24 = "2:4 semi-structured GEMM TFLOP/s of kept products, % roofline, speedup vs dense"
METRIC_BSR24 = "block-sparse GEMM with 2:4 blocks, TFLOP/s of kept products, % roofline, speedup vs dense"
L2_BYTES_DEFAULT = 126 * 2 ** 20

# DRAM traffic per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by workload.  The
# entry is only used while the kernel source still hashes to `src_sha`.
TRAFFIC = {
    ("large_fwd", "fwd"): {"bytes": 289312768, "src_sha": "77cfcf7e0f6eadf7",
                           "files": ["spmm_tc.cu", "common.cuh"]},
    ("decode_fwd", "fwd"): {"bytes": 22775552, "src_sha": "3f8c2a55a00991df",
                            "files": ["stream_fwd.cu", "common.cuh"]},
    ("enc_train_d1.0", "dx"): {"bytes": 29967872, "src_sha": "77cfcf7e0f6eadf7",
                               "files": ["spmm_tc.cu", "common.cuh"]},
    ("enc_train_d1.0", "dw"): {"bytes": 31494912, "src_sha": "3b6be507a67442e5",
                               "files": ["sddmm_tc.cu", "common.cuh"]},
    ("semi24_fwd", "fwd"): {"bytes": 501997568, "src_sha": "8af7749e74284a89",
                            "files": ["semi24.cu", "common.cuh"]},
    ("bsr24_fwd", "fwd"): {"bytes": 296606208, "src_sha": "14e6d2faba6afb35",
                           "files": ["bsr24.cu", "common.cuh"]},
}
# the kernel source files each contraction's traffic figure depends on
TRAFFIC_FILES = {"fwd": ["spmm_tc.cu", "common.cuh"], "fwd_small": ["stream_fwd.cu", "common.cuh"],
                 "dx": ["spmm_tc.cu", "common.cuh"], "dw": ["sddmm_tc.cu", "common.cuh"]}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def src_sha(*names):
    """Hash of the kernel sources with comments and blank lines removed, so a
    traffic figure stays tied to the code it was measured on, not its prose."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sparse_gemm_b200", "csrc", n), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ----------------------------------------------------------------------------- workload

def algorithmic(w: synth.Workload, nnz: int):
    """Flops and HBM bytes per launch of each contraction (minimum traffic:
    every operand read once, every output written once)."""
    b, M, N, K = w.b, w.M, w.N, w.K
    R, C = N // b, K // b
    flops = 2 * M * b * b * nnz
    wbytes = nnz * b * b * 2 + (R + 1 + nnz) * 4           # values + BSR index
    wbytes_t = nnz * b * b * 2 + (C + 1 + 2 * nnz) * 4     # values + CSC index + map
    return {
        "fwd": {"flops": flops, "bytes": M * K * 2 + wbytes + M * N * 2},
        "dx": {"flops": flops, "bytes": M * N * 2 + wbytes_t + M * K * 2},
        "dw": {"flops": flops, "bytes": M * N * 2 + M * K * 2 + nnz * b * b * 2 + (C + 1 + 2 * nnz) * 4},
    }


def roofline_entry(kind: str, alg: dict, dur_ms: float, pk: dict, burst: bool = True):
    tc_peak = pk["bf16_tflops"] if burst else pk["bf16_tflops_sustained"]
    t_tc = alg["flops"] / (tc_peak * 1e12)
    t_hbm = alg["bytes"] / (pk["hbm_gbs"] * 1e9)
    s = dur_ms * 1e-3
    if t_tc >= t_hbm:
        achieved = alg["flops"] / s / 1e12
        return {"bound": "tensor", "achieved": round(achieved, 2), "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4)}
    achieved = alg["bytes"] / s / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4)}


def cpu_sample(w: synth.Workload, inp: dict, budget_s: float, kinds: list[str]):
    """Time the fp64 oracle, as it is, on a bounded sample of the workload.

    Forward / dX: a sample of token rows (all N or K outputs of each);
    dW: a sample of stored blocks (each reduced over all M rows).  The
    operands are widened and the dense-with-zeros weight is built once,
    outside the timed calls.  Returns (flops_done, seconds, description).
    """
    import oracle
    oracle.build()
    b = w.b
    Xd = oracle.widen(inp["X"])
    Wt = oracle.dense_weight(inp["W"], inp["mask"], b)
    dYd = oracle.widen(inp["dY"]) if "dY" in inp else None
    nthreads = oracle.num_threads()
    per_row = 2 * w.N * w.K                       # dense-with-zeros flops per token row
    eff_ratio = w.nnz / (w.R * w.C)
    done_eff, secs, desc = 0.0, 0.0, []
    share = budget_s / len(kinds)
    for kind in kinds:
        if kind in ("fwd", "dx"):
            def call(rows):
                if kind == "fwd":
                    oracle.forward(None, None, None, b, rows=rows, Xd=Xd, Wt=Wt)
                else:
                    oracle.backward_input(None, None, None, b, rows=rows, dYd=dYd, Wt=Wt)
            t0 = time.perf_counter()
            call(np.arange(min(nthreads, w.M)))
            t1 = time.perf_counter() - t0
            n = int(min(w.M, max(1, share / max(t1, 1e-6)) * min(nthreads, w.M)))
            n = max(1, min(n, w.M))
            rows = np.random.default_rng(0).choice(w.M, size=n, replace=False)
            t0 = time.perf_counter()
            call(rows)
            dt = time.perf_counter() - t0
            done_eff += 2 * n * w.N * w.K * eff_ratio
            secs += dt
            desc.append(f"{kind}: {n} of {w.M} token rows")
        else:
            rr, cc = np.nonzero(inp["mask"])
            t0 = time.perf_counter()
            oracle.backward_weight(None, None, inp["mask"], b, blocks=[(int(rr[0]), int(cc[0]))],
                                   dYd=dYd, Xd=Xd)
            t1 = time.perf_counter() - t0
            n = int(max(1, min(len(rr), share / max(t1, 1e-6))))
            pick = np.random.default_rng(0).choice(len(rr), size=n, replace=False)
            t0 = time.perf_counter()
            oracle.backward_weight(None, None, inp["mask"], b,
                                   blocks=[(int(rr[i]), int(cc[i])) for i in pick], dYd=dYd, Xd=Xd)
            dt = time.perf_counter() - t0
            done_eff += 2 * n * b * b * w.M
            secs += dt
            desc.append(f"dw: {n} of {len(rr)} blocks")
    del per_row
    return done_eff, secs, "; ".join(desc), nthreads


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_sample_blockskip(w: synth.Workload, inp: dict, budget_s: float):
    """Time the oracle's block-skipping forward (only the stored blocks'
    work) on a bounded sample of token rows; flops counted are the effective
    2*b*b per stored block and token.  Returns (flops, seconds, description)."""
    import oracle
    oracle.build()
    Xd = oracle.widen(inp["X"])
    Wt = oracle.dense_weight(inp["W"], inp["mask"], w.b)
    nthreads = oracle.num_threads()
    probe = np.arange(min(nthreads, w.M))
    t0 = time.perf_counter()
    oracle.forward_blockskip(None, None, inp["mask"], w.b, rows=probe, Xd=Xd, Wt=Wt)
    t1 = time.perf_counter() - t0
    n = int(min(w.M, max(1, budget_s / max(t1, 1e-6)) * len(probe)))
    n = max(1, min(n, w.M))
    rows = np.random.default_rng(1).choice(w.M, size=n, replace=False)
    t0 = time.perf_counter()
    oracle.forward_blockskip(None, None, inp["mask"], w.b, rows=rows, Xd=Xd, Wt=Wt)
    dt = time.perf_counter() - t0
    return 2.0 * n * w.b * w.b * w.nnz, dt, f"fwd: {n} of {w.M} token rows"


# ----------------------------------------------------------------------------- ranks
# The layer is not sharded: under torchrun every rank runs the whole workload
# on its own GPU (replicas) and the job's throughput is all ranks' work over
# the slowest rank's time.  Every rank calls these in the same order.

def max_over_ranks(x, world, device=None):
    """The largest value of `x` over all ranks (the slowest rank's time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, flops_per_step, steps, total_ms):
    """Weak scaling: TFLOP/s of all ranks' steps over the slowest rank's time."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args):
    import torch
    import torch.distributed as dist

    import sparse_gemm_b200 as sg

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    from sparse_gemm_b200 import build as _b
    _b.build()

    w = synth.WORKLOADS[args.workload]
    train = w.with_dy
    inp = synth.make_inputs(w)
    pk = peaks()
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", L2_BYTES_DEFAULT) or L2_BYTES_DEFAULT

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    Wd = dev_bf16(inp["W"])
    mask = torch.from_numpy(inp["mask"]).to(dev)
    X0 = dev_bf16(inp["X"])
    dY0 = dev_bf16(inp["dY"]) if train else None

    # pack (timed separately: once per weight)
    stream = torch.cuda.current_stream(dev)
    Wp = sg.pack(Wd, mask, w.b, nnz=w.nnz)
    torch.cuda.synchronize()
    pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pack_ms = []
    for _ in range(5):
        pe0.record(stream)
        sg.pack(Wd, mask, w.b, nnz=w.nnz)
        pe1.record(stream)
        torch.cuda.synchronize()
        pack_ms.append(pe0.elapsed_time(pe1))
    if sg.device_status(Wp) != 0:
        raise RuntimeError("pack reported a device error")

    # L2-cold protocol: rotate through copies of every input so that one
    # rotation touches more than 2x L2 before an input is reused
    in_bytes = X0.numel() * 2 + (dY0.numel() * 2 if train else 0) + w.nnz * w.b * w.b * 2
    ncopy = int(min(16, max(2, math.ceil(2 * l2 / in_bytes) + 1)))
    Xs = [X0] + [X0.clone() for _ in range(ncopy - 1)]
    dYs = ([dY0] + [dY0.clone() for _ in range(ncopy - 1)]) if train else None
    Wps = [Wp] + [sg.pack(Wd, mask, w.b, nnz=w.nnz) for _ in range(ncopy - 1)]
    Y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((w.M, w.K), dtype=torch.bfloat16, device=dev) if train else None
    dWv = torch.empty((w.nnz, w.b, w.b), dtype=torch.bfloat16, device=dev) if train else None
    ws = torch.zeros(max(16, sg.forward_workspace_bytes(w.M, Wp)), dtype=torch.uint8, device=dev)
    small = w.M <= sg.small_m_max()

    kinds = ["fwd", "dx", "dw"] if train else ["fwd"]
    launches_per_step = 1 + (2 if train else 0)  # kernels per step (each also has a small memset)

    def step(i):
        j = i % ncopy
        sg.forward(Xs[j], Wps[j], out=Y, workspace=ws)
        if train:
            sg.backward_input(dYs[j], Wps[j], out=dX)
            sg.backward_weight(dYs[j], Xs[j], Wps[j], out=dWv)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if sg.device_status(Wp) != 0:
        raise RuntimeError("kernels reported a device error")

    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def capture(fn):
        """CUDA graph of K consecutive steps (rotating input copies)."""
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(stream)
        with torch.cuda.graph(g, stream=cs):
            for i in range(K):
                fn(i)
        stream.wait_stream(cs)
        torch.cuda.synchronize()
        return g

    def replay_times(g, reps):
        """`reps` timed replays of a K-step graph, each bracketed by a
        synchronize (and a barrier across ranks) on both sides."""
        g.replay()                      # untimed: first replay uploads the graph
        torch.cuda.synchronize()
        out = []
        for _ in range(reps):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            ev0.record(stream)
            g.replay()
            ev1.record(stream)
            torch.cuda.synchronize()
            out.append(ev0.elapsed_time(ev1))
        return out

    def replay_ms(g, reps=None):
        return statistics.median(replay_times(g, reps or args.replays))

    timing = "cuda-graph"
    try:
        g_step = capture(step)
        # the same K steps on one input copy: operands stay in L2 between steps
        g_warm = capture(lambda i: step(0))
        kernel_graphs = {}
        if train:
            kernel_graphs["fwd"] = capture(lambda i: sg.forward(Xs[i % ncopy], Wps[i % ncopy], out=Y, workspace=ws))
            kernel_graphs["dx"] = capture(lambda i: sg.backward_input(dYs[i % ncopy], Wps[i % ncopy], out=dX))
            kernel_graphs["dw"] = capture(lambda i: sg.backward_weight(dYs[i % ncopy], Xs[i % ncopy],
                                                                       Wps[i % ncopy], out=dWv))
    except Exception as e:  # noqa: BLE001 - fall back to eager launches, said so in the output
        log("graph capture failed, timing eager launches:", repr(e))
        timing = "eager"

    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_times = None
    if timing == "cuda-graph":
        step_times = replay_times(g_step, args.replays)
        total_ms = statistics.median(step_times)
    else:
        ev0.record(stream)
        for i in range(K):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        total_ms = ev0.elapsed_time(ev1)
    if world > 1:
        dist.barrier()
    warm_ms = statistics.median(replay_times(g_warm, args.replays)) if timing == "cuda-graph" else None
    # keep the GPU busy inside the clock window for at least ~0.5 s
    t_end = time.time() + 0.5
    while timing == "cuda-graph" and time.time() < t_end:
        g_step.replay()
        torch.cuda.synchronize()
    clk = clocks.stop()
    if timing == "cuda-graph":
        if train:
            per_kernel = {k: replay_ms(g) / K for k, g in kernel_graphs.items()}
        else:
            per_kernel = {"fwd": total_ms / K}
    else:
        per_kernel = {k: total_ms / K / len(kinds) for k in kinds}
    total_ms = max_over_ranks(total_ms, world, dev)
    spread = None
    if step_times:
        spread = {"replays": len(step_times), "min_ms_per_step": round(min(step_times) / K, 5),
                  "max_ms_per_step": round(max(step_times) / K, 5),
                  "median_ms_per_step": round(statistics.median(step_times) / K, 5)}

    alg = algorithmic(w, w.nnz)
    flops_step = sum(alg[k]["flops"] for k in kinds)
    value = whole_job_value(world, flops_step, K, total_ms)
    ms_per_step = total_ms / K

    # dominant kernel + its roofline
    dom = max(per_kernel, key=per_kernel.get)
    roof = roofline_entry(dom, alg[dom], per_kernel[dom], pk)
    roof["kernel"] = {"fwd": "k_stream_fwd" if small else "k_spmm_tc (forward)",
                      "dx": "k_spmm_tc (input gradient)", "dw": "k_sddmm_tc"}[dom]
    roof["peak_source"] = pk["source"] + (" burst bf16" if roof["unit"] == "TFLOP/s" else " HBM copy")
    tr = TRAFFIC.get((w.name, dom))
    files = TRAFFIC_FILES["fwd_small" if (dom == "fwd" and small) else dom]
    roof["traffic"] = tr["bytes"] if tr and tr.get("src_sha") == src_sha(*files) else None
    roof["algorithmic_bytes"] = alg[dom]["bytes"]
    roof["algorithmic_flops"] = alg[dom]["flops"]
    roof["tensor_frac_of_sustained"] = round(alg[dom]["flops"] / (per_kernel[dom] * 1e-3) / 1e12
                                             / pk["bf16_tflops_sustained"], 4)

    # cuBLAS dense of the same shapes (zeros in place), same rotation
    Wdz = Wd * torch.repeat_interleave(torch.repeat_interleave(mask.to(torch.bfloat16), w.b, 0), w.b, 1)
    Wdzs = [Wdz] + [Wdz.clone() for _ in range(min(ncopy, 4) - 1)]

    def dense_step(i):
        j = i % len(Wdzs)
        x = Xs[i % ncopy]
        torch.matmul(x, Wdzs[j].t(), out=Y)
        if train:
            torch.matmul(dYs[i % ncopy], Wdzs[j], out=dX)
            torch.matmul(dYs[i % ncopy].t(), x)

    for i in range(max(3, args.warmup)):
        dense_step(i)
    torch.cuda.synchronize()
    if timing == "cuda-graph":
        dense_ms = replay_ms(capture(dense_step)) / K
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            dense_step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / K

    # end to end through the public API: pinned host X (+dY) in, Y (+dX, dW) out,
    # every step.  When a step moves enough data for PCIe to dominate (8 MB or
    # more), steps are pipelined the way a serving loop would run them: uploads
    # on one stream, the layer on another, downloads on a third, with two sets
    # of device buffers, so step i's download overlaps step i+1's upload and
    # compute (PCIe moves data both ways at once).  Smaller steps are bound by
    # launch latency and run back to back on one stream.
    hX = torch.empty(X0.shape, dtype=torch.bfloat16, pin_memory=True).copy_(X0.cpu())
    hdY = torch.empty(dY0.shape, dtype=torch.bfloat16, pin_memory=True).copy_(dY0.cpu()) if train else None
    hY = torch.empty(Y.shape, dtype=torch.bfloat16, pin_memory=True)
    hdX = torch.empty(dX.shape, dtype=torch.bfloat16, pin_memory=True) if train else None
    hdW = torch.empty(dWv.shape, dtype=torch.bfloat16, pin_memory=True) if train else None
    bufs = []
    for _ in range(2):
        bufs.append({"X": torch.empty_like(X0), "dY": torch.empty_like(dY0) if train else None,
                     "Y": torch.empty_like(Y), "dX": torch.empty_like(dX) if train else None,
                     "dW": torch.empty_like(dWv) if train else None})
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]    # upload of buffer set j done
    ev_comp = [torch.cuda.Event() for _ in range(2)]  # layer done with buffer set j
    ev_out = [torch.cuda.Event() for _ in range(2)]   # download of buffer set j done
    for j in range(2):  # nothing pending on either buffer set yet
        ev_comp[j].record(s_comp)
        ev_out[j].record(s_out)

    def e2e_step(i):
        j = i % 2
        b = bufs[j]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[j])           # the layer finished reading this set
            b["X"].copy_(hX, non_blocking=True)
            if train:
                b["dY"].copy_(hdY, non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[j])
            s_comp.wait_event(ev_out[j])          # the previous result of this set is downloaded
            sg.forward(b["X"], Wp, out=b["Y"], workspace=ws)
            if train:
                sg.backward_input(b["dY"], Wp, out=b["dX"])
                sg.backward_weight(b["dY"], b["X"], Wp, out=b["dW"])
            ev_comp[j].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[j])
            hY.copy_(b["Y"], non_blocking=True)
            if train:
                hdX.copy_(b["dX"], non_blocking=True)
                hdW.copy_(b["dW"], non_blocking=True)
            ev_out[j].record(s_out)

    def e2e_step_serial(i):
        b = bufs[0]
        b["X"].copy_(hX, non_blocking=True)
        if train:
            b["dY"].copy_(hdY, non_blocking=True)
        sg.forward(b["X"], Wp, out=b["Y"], workspace=ws)
        hY.copy_(b["Y"], non_blocking=True)
        if train:
            sg.backward_input(b["dY"], Wp, out=b["dX"])
            sg.backward_weight(b["dY"], b["X"], Wp, out=b["dW"])
            hdX.copy_(b["dX"], non_blocking=True)
            hdW.copy_(b["dW"], non_blocking=True)

    xfer = hX.numel() * 2 + hY.numel() * 2 + ((hdY.numel() + hdX.numel() + hdW.numel()) * 2 if train else 0)
    pipelined = xfer >= 8 * 2 ** 20
    run_step = e2e_step if pipelined else e2e_step_serial
    for i in range(2):
        run_step(i)
    torch.cuda.synchronize()
    ke = max(3, min(K, 50))
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pipelined:
        t0.record(s_in)
        s_comp.wait_event(t0)
        s_out.wait_event(t0)
    else:
        t0.record(stream)
    for i in range(ke):
        run_step(i)
    t1.record(s_out if pipelined else stream)  # the last download ends after everything else
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1) / ke
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    h2d = X0.numel() * 2 + (dY0.numel() * 2 if train else 0)
    d2h = Y.numel() * 2 + ((dX.numel() + dWv.numel()) * 2 if train else 0)

    if sg.device_status(Wp) != 0:
        raise RuntimeError("kernels reported a device error")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, secs, desc, nthr = cpu_sample(w, inp, args.cpu_budget * 2 / 3, kinds)
        cpu = {"value": round(done / secs / 1e12, 8), "unit": UNIT, "cores": nthr, "kind": "oracle",
               "sample": desc + f" ({secs:.1f} s, fp64 dense-with-zeros loops)",
               "cpu_model": cpu_model()}
        bdone, bsecs, bdesc = cpu_sample_blockskip(w, inp, args.cpu_budget / 3)
        cpu["block_skipping"] = {"value": round(bdone / bsecs / 1e12, 8), "unit": UNIT,
                                 "sample": bdesc + f" ({bsecs:.1f} s, fp64 loops over the stored blocks only)"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": w.name, "M": w.M, "N": w.N, "K": w.K, "b": w.b, "nnz": w.nnz,
            "density": round(w.nnz / (w.R * w.C), 5), "mask": w.mask_kind, "seed": w.seed,
            "contractions_per_step": kinds, "global_batch": w.M * world,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"rotating {ncopy} copies of every input ({ncopy * in_bytes / 2**20:.0f} MiB > 2x L2)",
            "pack_ms": round(statistics.median(pack_ms), 4),
            "timing": timing,
        },
        "timing_spread": spread,
        "warm_l2": ({"ms_per_step": round(warm_ms / K, 5),
                     "value": round(whole_job_value(1, flops_step, K, warm_ms), 3),
                     "note": "same K steps on one input copy (operands stay in L2); not the headline"}
                    if warm_ms else None),
        "kernels_ms": {k: round(v, 5) for k, v in per_kernel.items()},
        "roofline": roof,
        "dense_cublas_ms_per_step": round(dense_ms, 5),
        "speedup_vs_dense": round(dense_ms / ms_per_step, 3),
        "e2e": {"value": round(whole_job_value(world, flops_step, 1, e2e_ms), 3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "timing": ("public API calls, uploads / layer / downloads pipelined on three streams"
                           if pipelined else "public API calls, one stream")},
        "gpu_launches": K * launches_per_step,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    return out


# ----------------------------------------------------------------------------- 2:4 semi-structured

def algorithmic_semi24(w: synth.Semi24Workload):
    """Flops (products with the kept half of the weight) and minimum HBM bytes
    (X, compressed values, 2-bit positions and Y each moved once)."""
    M, N, K = w.M, w.N, w.K
    return {"flops": w.flops(), "bytes": M * K * 2 + N * (K // 2) * 2 + N * (K // 16) * 2 + M * N * 2}


def cpu_sample_semi24(w: synth.Semi24Workload, inp: dict, budget_s: float):
    """Time the oracle's 2:4 forward on a bounded sample of token rows (the
    compressed form and the widened operands are prepared outside the timed
    call).  Flops counted: the kept products, N*K per row.  Returns (flops,
    seconds, description, threads)."""
    import oracle
    oracle.build()
    v, m = oracle.compress24(inp["W"])
    Xd = oracle.widen(inp["X"])
    Wt = oracle.widen(oracle.decompress24(v, m))
    nthreads = oracle.num_threads()
    probe = np.arange(min(nthreads, w.M))
    t0 = time.perf_counter()
    oracle.forward(None, None, None, None, rows=probe, Xd=Xd, Wt=Wt)
    t1 = time.perf_counter() - t0
    n = int(min(w.M, max(1, budget_s / max(t1, 1e-6)) * len(probe)))
    n = max(1, min(n, w.M))
    rows = np.random.default_rng(2).choice(w.M, size=n, replace=False)
    t0 = time.perf_counter()
    oracle.forward(None, None, None, None, rows=rows, Xd=Xd, Wt=Wt)
    dt = time.perf_counter() - t0
    return float(n) * w.N * w.K, dt, f"fwd: {n} of {w.M} token rows", nthreads


def algorithmic_bsr24(w: synth.Workload, nnz: int):
    """Block-sparse weight with 2:4 blocks: flops of the kept products
    (2*M*b*b*nnz / 2); bytes X + compressed blocks + their position words +
    the BSR index + Y."""
    b, M, N, K = w.b, w.M, w.N, w.K
    R = N // b
    return {"flops": M * b * b * nnz,
            "bytes": M * K * 2 + nnz * b * (b // 2) * 2 + nnz * b * (b // 16) * 2 + (R + 1 + nnz) * 4 + M * N * 2}


def cpu_sample_bsr24(w: synth.Workload, inp: dict, budget_s: float):
    """The oracle's block-skipping forward on a bounded sample of token rows
    of the 2:4-block workload; flops counted are the kept products
    (b*b per stored block and token)."""
    f, secs, desc = cpu_sample_blockskip(w, inp, budget_s)
    import oracle
    return f / 2, secs, desc, oracle.num_threads()


def run_gpu_2of4(args):
    """The 2:4 workloads (plain 2:4, and 2:4 inside the blocks of a
    block-sparse weight): compress once, then K forwards per step graph,
    timed like the block-sparse workloads (rotating input copies, CUDA-graph
    replays, median over replays, max over ranks)."""
    import torch
    import torch.distributed as dist

    import sparse_gemm_b200 as sg

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from sparse_gemm_b200 import build as _b
    _b.build()

    pk = peaks()
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", L2_BYTES_DEFAULT) or L2_BYTES_DEFAULT

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    stream = torch.cuda.current_stream(dev)
    if args.workload in synth.SEMI24_WORKLOADS:
        w = synth.SEMI24_WORKLOADS[args.workload]
        inp = synth.make_semi24_inputs(w)
        Wd, X0 = dev_bf16(inp["W"]), dev_bf16(inp["X"])
        compress = lambda out=None: sg.compress24(Wd, out=out)  # noqa: E731
        forward = lambda x, ww, out=None: sg.forward24(x, ww, out=out)  # noqa: E731
        status = sg.semi24_status
        Wdense = Wd
        alg = algorithmic_semi24(w)
        wbytes = w.N * (w.K // 2) * 2 + w.N * (w.K // 16) * 2
        kernel, metric = "k_semi24_fwd", METRIC_SEMI24
        extra = {"pattern": "2:4 along K"}
        cpu_fn = cpu_sample_semi24
        cpu_what = "fp64 loops over the dense weight with zeros in place"
    else:
        w = synth.BSR24_WORKLOADS[args.workload]
        inp = synth.make_bsr24_inputs(w)
        Wd, X0 = dev_bf16(inp["W"]), dev_bf16(inp["X"])
        mask = torch.from_numpy(inp["mask"]).to(dev)
        Wp = sg.pack(Wd, mask, w.b, nnz=w.nnz)
        compress = lambda out=None: sg.compress_bsr24(Wp, out=out)  # noqa: E731
        forward = lambda x, ww, out=None: sg.forward_bsr24(x, ww, out=out)  # noqa: E731
        status = lambda ww: sg.device_status(ww.packed)  # noqa: E731
        Wdense = Wd * torch.repeat_interleave(torch.repeat_interleave(mask.to(torch.bfloat16), w.b, 0), w.b, 1)
        alg = algorithmic_bsr24(w, w.nnz)
        wbytes = w.nnz * w.b * (w.b // 2) * 2 + w.nnz * w.b * (w.b // 16) * 2
        kernel, metric = "k_bsr24_fwd", METRIC_BSR24
        extra = {"b": w.b, "nnz": w.nnz, "density": round(w.nnz / (w.R * w.C), 5), "mask": w.mask_kind,
                 "pattern": "2:4 along K inside the kept blocks"}
        cpu_fn = cpu_sample_bsr24
        cpu_what = "fp64 loops over the stored blocks only"
    w0 = compress()
    torch.cuda.synchronize()
    ce0, ce1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    comp_ms = []
    for _ in range(5):
        ce0.record(stream)
        compress(out=w0)
        ce1.record(stream)
        torch.cuda.synchronize()
        comp_ms.append(ce0.elapsed_time(ce1))
    if status(w0) != 0:
        raise RuntimeError("compress reported a device error")

    in_bytes = X0.numel() * 2 + wbytes
    ncopy = int(min(16, max(2, math.ceil(2 * l2 / in_bytes) + 1)))
    Xs = [X0] + [X0.clone() for _ in range(ncopy - 1)]
    ws = [w0] + [compress() for _ in range(ncopy - 1)]
    Y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)

    def step(i):
        forward(Xs[i % ncopy], ws[i % ncopy], out=Y)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(stream)
        with torch.cuda.graph(g, stream=cs):
            for i in range(K):
                fn(i)
        stream.wait_stream(cs)
        torch.cuda.synchronize()
        return g

    def replay_times(g, reps):
        g.replay()
        torch.cuda.synchronize()
        out = []
        for _ in range(reps):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            ev0.record(stream)
            g.replay()
            ev1.record(stream)
            torch.cuda.synchronize()
            out.append(ev0.elapsed_time(ev1))
        return out

    g_step = capture(step)
    g_warm = capture(lambda i: step(0))
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_times = replay_times(g_step, args.replays)
    total_ms = statistics.median(step_times)
    warm_ms = statistics.median(replay_times(g_warm, args.replays))
    t_end = time.time() + 0.5
    while time.time() < t_end:
        g_step.replay()
        torch.cuda.synchronize()
    clk = clocks.stop()
    fwd_ms = total_ms / K
    total_ms = max_over_ranks(total_ms, world, dev)
    value = whole_job_value(world, alg["flops"], K, total_ms)
    ms_per_step = total_ms / K

    # the kept products run at twice the dense rate on the sparse MMA, so the
    # useful-flop peak of the 2:4 kernel is the dense bf16 peak
    roof = roofline_entry("fwd", alg, fwd_ms, pk)
    roof["kernel"] = kernel
    roof["peak_source"] = pk["source"] + (" burst bf16 (useful flops of the 2:4 MMA)"
                                          if roof["unit"] == "TFLOP/s" else " HBM copy")
    tr = TRAFFIC.get((w.name, "fwd"))
    roof["traffic"] = tr["bytes"] if tr and tr.get("src_sha") == src_sha(*tr["files"]) else None
    roof["algorithmic_bytes"] = alg["bytes"]
    roof["algorithmic_flops"] = alg["flops"]
    roof["dense_equivalent_tflops"] = round(2 * alg["flops"] / (fwd_ms * 1e-3) / 1e12, 2)
    roof["tensor_frac_of_sustained"] = round(alg["flops"] / (fwd_ms * 1e-3) / 1e12
                                             / pk["bf16_tflops_sustained"], 4)

    # cuBLAS dense on the same weight (zeros in place), same rotation
    Wds = [Wdense] + [Wdense.clone() for _ in range(min(ncopy, 3) - 1)]

    def dense_step(i):
        torch.matmul(Xs[i % ncopy], Wds[i % len(Wds)].t(), out=Y)

    for i in range(max(3, args.warmup)):
        dense_step(i)
    torch.cuda.synchronize()
    dense_ms = statistics.median(replay_times(capture(dense_step), args.replays)) / K

    # end to end through the public API: pinned host X in, Y out, every step;
    # uploads, layer and downloads pipelined on three streams with two buffer sets
    hX = torch.empty(X0.shape, dtype=torch.bfloat16, pin_memory=True).copy_(X0.cpu())
    hY = torch.empty(Y.shape, dtype=torch.bfloat16, pin_memory=True)
    bufs = [{"X": torch.empty_like(X0), "Y": torch.empty_like(Y)} for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for j in range(2):
        ev_comp[j].record(s_comp)
        ev_out[j].record(s_out)

    def e2e_step(i):
        j = i % 2
        b = bufs[j]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[j])
            b["X"].copy_(hX, non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[j])
            s_comp.wait_event(ev_out[j])
            forward(b["X"], w0, out=b["Y"])
            ev_comp[j].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[j])
            hY.copy_(b["Y"], non_blocking=True)
            ev_out[j].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    ke = max(3, min(K, 50))
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_comp.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(ke):
        e2e_step(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / ke, world, dev)
    for ww in ws:
        if status(ww) != 0:
            raise RuntimeError("kernels reported a device error")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, secs, desc, nthr = cpu_fn(w, inp, args.cpu_budget)
        cpu = {"value": round(done / secs / 1e12, 8), "unit": UNIT, "cores": nthr, "kind": "oracle",
               "sample": desc + f" ({secs:.1f} s, {cpu_what})", "cpu_model": cpu_model()}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None
    return {
        "metric": metric, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": w.name, "M": w.M, "N": w.N, "K": w.K, **extra, "seed": w.seed,
            "contractions_per_step": ["fwd"], "global_batch": w.M * world,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"rotating {ncopy} copies of every input ({ncopy * in_bytes / 2**20:.0f} MiB > 2x L2)",
            "compress_ms": round(statistics.median(comp_ms), 4),
            "timing": "cuda-graph",
        },
        "timing_spread": {"replays": len(step_times), "min_ms_per_step": round(min(step_times) / K, 5),
                          "max_ms_per_step": round(max(step_times) / K, 5),
                          "median_ms_per_step": round(statistics.median(step_times) / K, 5)},
        "warm_l2": {"ms_per_step": round(warm_ms / K, 5),
                    "value": round(whole_job_value(1, alg["flops"], K, warm_ms), 3),
                    "note": "same K steps on one input copy (operands stay in L2); not the headline"},
        "kernels_ms": {"fwd": round(fwd_ms, 5)},
        "roofline": roof,
        "dense_cublas_ms_per_step": round(dense_ms, 5),
        "speedup_vs_dense": round(dense_ms / ms_per_step, 3),
        "e2e": {"value": round(whole_job_value(world, alg["flops"], 1, e2e_ms), 3), "unit": UNIT,
                "h2d_bytes_per_step": X0.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2,
                "ms_per_step": round(e2e_ms, 4),
                "timing": "public API calls, uploads / layer / downloads pipelined on three streams"},
        "gpu_launches": K,
        "clocks": clk,
        "cpu_baseline": cpu,
    }


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample of the workload; value is effective TFLOP/s over the sample."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    per_step = max(0.5, min(20.0, args.reference_budget / max(1, args.steps + args.warmup)))
    if args.workload in synth.SEMI24_WORKLOADS or args.workload in synth.BSR24_WORKLOADS:
        return run_reference_2of4(args, world, per_step)
    w = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(w)
    kinds = ["fwd", "dx", "dw"] if w.with_dy else ["fwd"]
    for _ in range(args.warmup):
        cpu_sample(w, inp, per_step, kinds)
    done, secs, descs = 0.0, 0.0, []
    nthr = 1
    for _ in range(args.steps):
        d, s, desc, nthr = cpu_sample(w, inp, per_step, kinds)
        done += d
        secs += s
        descs.append(desc)
    value = done / secs / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 8), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "b": w.b, "nnz": w.nnz,
                   "density": round(w.nnz / (w.R * w.C), 5), "mask": w.mask_kind, "seed": w.seed},
        "cpu_baseline": {"value": round(value, 8), "unit": UNIT, "cores": nthr, "kind": "oracle",
                         "sample": descs[0] + " per step (fp64 dense-with-zeros loops)",
                         "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 8), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_2of4(args, world, per_step):
    """The oracle's forward of a 2:4 workload on the host cores, a bounded
    sample of token rows per step; value is TFLOP/s of kept products."""
    if args.workload in synth.SEMI24_WORKLOADS:
        w = synth.SEMI24_WORKLOADS[args.workload]
        inp = synth.make_semi24_inputs(w)
        fn, metric, what = cpu_sample_semi24, METRIC_SEMI24, "fp64 loops over the dense weight with zeros in place"
        cfg = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "pattern": "2:4 along K", "seed": w.seed}
    else:
        w = synth.BSR24_WORKLOADS[args.workload]
        inp = synth.make_bsr24_inputs(w)
        fn, metric, what = cpu_sample_bsr24, METRIC_BSR24, "fp64 loops over the stored blocks only"
        cfg = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "b": w.b, "nnz": w.nnz,
               "density": round(w.nnz / (w.R * w.C), 5), "mask": w.mask_kind,
               "pattern": "2:4 along K inside the kept blocks", "seed": w.seed}
    for _ in range(args.warmup):
        fn(w, inp, per_step)
    done, secs, descs, nthr = 0.0, 0.0, [], 1
    for _ in range(args.steps):
        d, s_, desc, nthr = fn(w, inp, per_step)
        done += d
        secs += s_
        descs.append(desc)
    value = done / secs / 1e12
    return {
        "impl": "reference", "metric": metric, "value": round(value, 8), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": round(value, 8), "unit": UNIT, "cores": nthr, "kind": "oracle",
                         "sample": descs[0] + f" per step ({what})", "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 8), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_kernel_only(args):
    """One contraction of a workload, `--reps` times, on a single input copy
    (no rotation, no comparison runs): the command the ncu captures use."""
    import torch

    import sparse_gemm_b200 as sg
    from sparse_gemm_b200 import build as _b
    _b.build()
    dev = torch.device("cuda", 0)
    if args.workload in synth.SEMI24_WORKLOADS:
        if args.kernel_only != "fwd":
            raise SystemExit("the 2:4 workload has a forward only")
        w = synth.SEMI24_WORKLOADS[args.workload]
        inp = synth.make_semi24_inputs(w)
        bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        w24 = sg.compress24(bits(inp["W"]))
        X = bits(inp["X"])
        for _ in range(args.reps):
            sg.forward24(X, w24)
        torch.cuda.synchronize()
        st = sg.semi24_status(w24)
        if st != 0:
            raise RuntimeError(f"device status {st}")
        print(json.dumps({"kernel_only": "fwd", "workload": w.name, "reps": args.reps}))
        return
    if args.workload in synth.BSR24_WORKLOADS:
        if args.kernel_only != "fwd":
            raise SystemExit("the 2:4-block workload has a forward only")
        w = synth.BSR24_WORKLOADS[args.workload]
        inp = synth.make_bsr24_inputs(w)
        bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        Wp = sg.pack(bits(inp["W"]), torch.from_numpy(inp["mask"]).to(dev), w.b, nnz=w.nnz)
        w24 = sg.compress_bsr24(Wp)
        X = bits(inp["X"])
        for _ in range(args.reps):
            sg.forward_bsr24(X, w24)
        torch.cuda.synchronize()
        st = sg.device_status(Wp)
        if st != 0:
            raise RuntimeError(f"device status {st}")
        print(json.dumps({"kernel_only": "fwd", "workload": w.name, "reps": args.reps}))
        return
    w = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(w, with_dy=args.kernel_only != "fwd")

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    Wp = sg.pack(to_dev(inp["W"]), torch.from_numpy(inp["mask"]).to(dev), w.b, nnz=w.nnz)
    X = to_dev(inp["X"])
    dY = to_dev(inp["dY"]) if args.kernel_only != "fwd" else None
    torch.cuda.synchronize()
    for _ in range(args.reps):
        if args.kernel_only == "fwd":
            sg.forward(X, Wp)
        elif args.kernel_only == "dx":
            sg.backward_input(dY, Wp)
        else:
            sg.backward_weight(dY, X, Wp)
    torch.cuda.synchronize()
    st = sg.device_status(Wp)
    if st != 0:
        raise RuntimeError(f"device status {st}")
    print(json.dumps({"kernel_only": args.kernel_only, "workload": w.name, "reps": args.reps}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_fwd",
                    choices=sorted(synth.WORKLOADS) + sorted(synth.SEMI24_WORKLOADS)
                    + sorted(synth.BSR24_WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of CPU oracle work")
    ap.add_argument("--reference-budget", type=float, default=120.0)
    ap.add_argument("--kernel-only", choices=["fwd", "dx", "dw"], default=None)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--replays", type=int, default=15,
                    help="timed replays of the K-step graph; the median is reported")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.kernel_only:
        run_kernel_only(args)
        return
    if args.impl == "reference":
        out = run_reference(args)
    elif args.workload in synth.SEMI24_WORKLOADS or args.workload in synth.BSR24_WORKLOADS:
        out = run_gpu_2of4(args)
    else:
        out = run_gpu(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
