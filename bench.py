#!/usr/bin/env python
"""Benchmark of the MixLLM mixed-precision quantized linear layer on B200.

One step = the run-time hot path over one batch of synthetic tokens:
quantize the activations (per-token 8-bit symmetric) and run the mixed W8/W4
GEMM with two-step dequantization and scatter into Y.  Weight packing is the
method's offline step (weights are pre-packed once, MixLLM section 3.3) and is
done before timing; its own throughput is reported under "pack".

Timing: inputs live in HBM before the timed region; each step uses the next of R
rotated copies of the packed weights, activations and outputs, with R chosen so
that the bytes touched between two uses of one copy exceed 4x the L2 size.  The
K timed steps are replayed from CUDA graphs, bracketed by a barrier and device
synchronisation, timed with CUDA events and max-reduced over ranks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
       python bench.py --impl reference ...   (the CPU oracle on the same workload)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mixed W4.4A8 GEMM TOPS and GB/s, % of INT8 TC peak / HBM roofline"

WORKLOADS = {
    # name: (M, K, N) -- Llama 3 layer shapes, 10% 8-bit rows, group 128
    "llama3-8b-qo-m1": (1, 4096, 4096),
    "llama3-8b-qo-m16": (16, 4096, 4096),
    "llama3-8b-up-m256": (256, 4096, 14336),
    "llama3-8b-up-m2048": (2048, 4096, 14336),
    "llama3-8b-down-m2048": (2048, 14336, 4096),
    "llama3-70b-up-m1": (1, 8192, 28672),
    "llama3-70b-down-m1": (1, 28672, 8192),
    "llama3-70b-up-m16": (16, 8192, 28672),
    "llama3-70b-down-m16": (16, 28672, 8192),
    "llama3-70b-up-m4096": (4096, 8192, 28672),
    "llama3-70b-down-m4096": (4096, 28672, 8192),
}
DEFAULT_WORKLOAD = "llama3-70b-up-m4096"
# lines measured after the named workload in the same run: the same weights at another M
SECONDARY = {"llama3-70b-up-m4096": ("llama3-70b-up-m1", "llama3-70b-up-m16"),
             "llama3-70b-down-m4096": ("llama3-70b-down-m1", "llama3-70b-down-m16")}
HBM_BOUND_MAX_M = 128        # below the ~150-token ridge the step is bound by HBM


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=0, help="timed steps (0: about one second of work)")
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--frac8", type=float, default=0.10)
    p.add_argument("--group", type=int, default=128)
    p.add_argument("--path", type=int, default=0,
                   help="0 auto, 1 split-K CUDA cores, 2 tensor cores, 3 whole rows per CTA, "
                        "4 tensor cores on CTA pairs, 5 the same with 256-token tiles, "
                        "6 tensor cores for decode-sized M (one CTA per row tile)")
    p.add_argument("--act-group", type=int, default=0,
                   help="activation scales: 0 one per token; the weight group: one per token and group")
    p.add_argument("--impl", default="mx", choices=["mx", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true",
                   help="only the named workload (not the decode line measured after it)")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--sweep", action="store_true",
                   help="the K = N = 8192 sweep over 8-bit row fraction, M and group size: one JSON "
                        "line per (fraction, group, M, path) and the GEMV / tensor-core crossover")
    p.add_argument("--search", action="store_true",
                   help="the global precision search: channel saliency of one Llama-3-8B decoder "
                        "layer's seven linears, then the top-10%% choice over all 32 layers' rows")
    p.add_argument("--blockwise", action="store_true",
                   help="block-wise bit widths: the decode GEMM on Llama-3-8B up (K 4096, N 14336) "
                        "at M 1, 4, 16 against HBM, widths {2, 3, 4, 8}")
    a = p.parse_args()
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


KERNEL_SOURCES = {1: "gemm_decode.cu", 2: "gemm_tc.cu", 3: "gemm_rows.cu", 4: "gemm_tc2.cu", 5: "gemm_tc3.cu",
                  6: "gemm_tcd.cu"}
KERNEL_NAMES = {1: "gemm_decode_kernel (cluster split-K, CUDA cores)",
                2: "gemm_tc_kernel (tcgen05)",
                3: "gemm_rows_kernel (whole rows per CTA, CUDA cores)",
                4: "gemm_tc2_kernel (tcgen05 on CTA pairs)",
                5: "gemm_tc3_kernel (tcgen05 on CTA pairs, 256-token tiles)",
                6: "gemm_tcd_kernel (tcgen05 on one CTA per row tile, decode-sized token tile)"}


def src_digest(path: int) -> str:
    """Digest of one GEMM path's kernel source and the headers every kernel includes:
    a traffic record stays valid while these are unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixed_precision_quantized_mx_b200", "csrc")
    for f in (KERNEL_SOURCES[path], "mx_internal.cuh", "sm100.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ clocks (NVML)
class ClockSampler:
    """Samples SM clock and clock-event reasons of one GPU every few ms."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = str(e)
        self.samples = []
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.ok:
            self._stop.clear()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self, t0=None, t1=None):
        if not self.ok:
            return {"error": self.err}
        s = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not s:
            return None
        mhz = [x[1] for x in s]
        bits = 0
        for x in s:
            bits |= x[2]
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(s)}


# ------------------------------------------------------------------ reference arm
def oracle_step_sample(lay, budget_s: float = 0.5):
    """A bounded sample of one step for the CPU oracle: which (m, n) outputs to compute."""
    M, N, K = lay.M, lay.N, lay.K
    per_pair = K * 12e-9                     # ~12 ns per MAC pair on one core (both forms)
    budget = max(64, int(budget_s / per_pair))
    if M * N <= budget:
        m = np.repeat(np.arange(M, dtype=np.int32), N)
        n = np.tile(np.arange(N, dtype=np.int32), M)
        return m, n, f"all {M}x{N} outputs"
    rng = np.random.default_rng(1)
    m = rng.integers(0, M, budget).astype(np.int32)
    n = rng.integers(0, N, budget).astype(np.int32)
    return m, n, f"{budget} random (token, row) outputs of {M}x{N}"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_oracle(lay, canonical, steps: int, min_seconds: float = 0.0, act_group: int = 0,
                threads: int = 1):
    """Run the oracle's quantize + sampled GEMM; return (seconds per step, sample, fraction,
    steps done).  With threads > 1 the sampled outputs are cut into `threads` disjoint
    slices computed at the same time (the oracle's C routine runs with the interpreter
    lock released), the quantizer once per step; the oracle's arithmetic is unchanged."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    m, n, desc = oracle_step_sample(lay, budget_s=0.5 * threads)
    frac = len(m) / (lay.M * lay.N)
    X = lay.X.astype(np.float32)
    cuts = np.linspace(0, len(m), threads + 1).astype(int)
    pool = ThreadPoolExecutor(threads) if threads > 1 else None
    done, t0 = 0, time.perf_counter()
    while done < steps or time.perf_counter() - t0 < min_seconds:
        Aq, sa = oracle.quant_act(X, act_group=act_group)
        if pool is None:
            oracle.gemm(Aq, sa, canonical, act_group=act_group, pairs=(m, n))
        else:
            futs = [pool.submit(oracle.gemm, Aq, sa, canonical, act_group, (m[cuts[i]:cuts[i + 1]],
                                                                            n[cuts[i]:cuts[i + 1]]))
                    for i in range(threads)]
            for f in futs:
                f.result()
        done += 1
    sec = (time.perf_counter() - t0) / done
    if pool is not None:
        pool.shutdown()
    return sec, desc, frac, done


def cpu_baseline(lay, canonical, unit: str, act_group: int, seconds: float = 10.0) -> dict:
    """The oracle timed on this host's cores on a bounded sample of one step: all cores
    (the reported value) and one core."""
    units = step_units(lay.M, lay.K, lay.N, lay.group, lay.n8, unit)
    cores = host_cores()
    sec, desc, frac, done = time_oracle(lay, canonical, 1, min_seconds=seconds, act_group=act_group,
                                        threads=cores)
    sec1, desc1, frac1, done1 = time_oracle(lay, canonical, 1, min_seconds=seconds / 2, act_group=act_group)
    return {"value": units * frac / sec, "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{done} steps on {cores} threads, each: quantize {lay.M}x{lay.K} activations + "
                      f"{desc}, cut into {cores} slices",
            "single_thread": {"value": units * frac1 / sec1, "unit": unit, "cores": 1,
                              "sample": f"{done1} steps, each: quantize + {desc1}"}}


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
            else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch and layer (weak scaling: fixed work per GPU)."""
    return seed + 1000003 * rank


def step_units(M, K, N, g, n8, unit):
    from mixed_precision_quantized_mx_b200 import model
    if unit == "GB/s":
        return model.linear_bytes(M, N, K, g, n8, 2) / 1e9
    return model.gemm_ops(M, N, K) / 1e12


def run_reference(a):
    """The oracle on this host's cores, on the same workload, metric and unit as the main
    arm: each step quantizes the step's activations and computes a bounded sample of its
    outputs, the sample cut into one slice per core."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mixed_precision_quantized_mx_b200 import inputs
    import oracle
    M, K, N = WORKLOADS[a.workload]
    lay = inputs.llama_layer(M, K, N, a.frac8, a.group, seed=a.seed)
    can = oracle.pack(lay.W, lay.is8, lay.group)
    unit = "GB/s" if M <= HBM_BOUND_MAX_M else "TOPS"
    cores = host_cores()
    time_oracle(lay, can, a.warmup, act_group=a.act_group, threads=cores)
    sec, desc, frac, done = time_oracle(lay, can, a.steps or 5, act_group=a.act_group, threads=cores)
    value = step_units(M, K, N, a.group, lay.n8, unit) * frac / sec
    sample = (f"each step: quantize {M}x{K} activations + {desc} (fraction {frac:.3g} of the step), "
              f"cut into {cores} slices on {cores} threads")
    line = {
        "metric": METRIC, "value": value, "unit": unit, "impl": "reference",
        "n_gpus": a.gpus, "steps": done, "warmup": a.warmup, "ms_per_step": sec * 1e3 / frac,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": a.workload, "M": M, "K": K, "N": N, "group": a.group,
                   "frac8": a.frac8, "n8": lay.n8, "act_group": a.act_group},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ sweep
SWEEP_FRACS = (0.0, 0.05, 0.10, 0.25, 0.50)
SWEEP_M = (1, 8, 64, 512, 8192)
SWEEP_GROUPS = (64, 128)


def run_sweep(a):
    """K = N = 8192: 8-bit row fraction x M x group size.  Every step is one mx_linear call
    (quantizer + GEMM) replayed from a CUDA graph over rotated copies (>= 4x L2), timed with
    events on its stream after warm-up replays.  Each (fraction, group, M) is timed on the
    decode path (split-K, 1) where it serves and on the tensor cores (4, on CTA pairs); the
    crossover is the smallest M at which the tensor cores win."""
    import torch
    from mixed_precision_quantized_mx_b200 import binding as mx
    from mixed_precision_quantized_mx_b200 import build as mxbuild
    from mixed_precision_quantized_mx_b200 import inputs, model

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    mxbuild.build()
    peaks = load_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    K = N = 8192
    s = torch.cuda.Stream(dev)
    rows = []
    for g in SWEEP_GROUPS:
        for frac in SWEEP_FRACS:
            base = inputs.llama_layer(1, K, N, frac, g, seed=a.seed)
            n8 = base.n8
            L = mx.mx_layout_init(N, K, g, n8)
            blob0 = torch.empty(L.total_bytes, dtype=torch.uint8, device=dev)
            mx.mx_pack_weights(L, torch.from_numpy(base.W).to(dev), torch.from_numpy(base.is8).to(dev), blob0)
            rng = np.random.default_rng(a.seed + 17)
            for M in SWEEP_M:
                X = torch.from_numpy(inputs.activations(rng, M, K, int(round(0.01 * K)), dtype=np.float16)).to(dev)
                per_step = L.total_bytes + X.nbytes + 2 * M * N
                R = int(min(16, max(2, math.ceil(4 * l2 / per_step))))
                blobs = [blob0] + [blob0.clone() for _ in range(R - 1)]
                Xs = [X] + [X.clone() for _ in range(R - 1)] if M <= 64 else [X] * R
                Ys = [torch.empty((M, N), dtype=torch.float16, device=dev) for _ in range(min(R, 2))]
                auto = mx.mx_gemm_select_path(L, M)
                for path in (1, 4):
                    if path == 1 and M > 64:
                        continue                       # decode-sized M only
                    try:
                        ws_n = mx.mx_linear_workspace_size(L, M, torch.float16, path=path)
                    except mx.MXError:
                        continue
                    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)

                    def step(i):
                        mx.mx_linear(L, blobs[i], Xs[i], Ys[i % len(Ys)], workspace=ws, path=path)
                    try:
                        with torch.cuda.stream(s):
                            for i in range(R):
                                step(i)
                        torch.cuda.synchronize()
                    except mx.MXError:
                        continue                       # the path does not serve this shape
                    gr = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gr, stream=s):
                        for i in range(R):
                            step(i)
                    for _ in range(3):                 # uploads the graph and warms up
                        gr.replay()
                    torch.cuda.synchronize()
                    t0 = time.perf_counter()
                    gr.replay()
                    torch.cuda.synchronize()
                    reps = int(min(200, max(3, 0.15 / max(time.perf_counter() - t0, 1e-6))))
                    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    ev0.record(s)
                    with torch.cuda.stream(s):
                        for _ in range(reps):
                            gr.replay()
                    ev1.record(s)
                    torch.cuda.synchronize()
                    us = ev0.elapsed_time(ev1) * 1e3 / (reps * R)
                    ops = model.gemm_ops(M, N, K)
                    byts = model.linear_bytes(M, N, K, g, n8, 2)
                    row = {"sweep": "K=N=8192", "frac8": frac, "group": g, "n8": n8, "M": M, "path": path,
                           "auto_path": auto, "us_per_step": round(us, 3),
                           "tops": round(ops / us / 1e6, 2), "gbs": round(byts / us / 1e3, 1),
                           "frac_hbm": round(byts / us / 1e3 / peaks["hbm_gbs"], 4),
                           "frac_int8": round(ops / us / 1e6 / (2 * peaks["bf16_tflops"]), 4)}
                    rows.append(row)
                    print(json.dumps(row), flush=True)
                    del gr
                del blobs, Xs, Ys
                torch.cuda.empty_cache()
    # the crossover: smallest M at which the tensor cores beat the decode path
    summary = []
    for g in SWEEP_GROUPS:
        for frac in SWEEP_FRACS:
            cross = None
            for M in SWEEP_M:
                t = {r["path"]: r["us_per_step"] for r in rows if r["group"] == g and r["frac8"] == frac and r["M"] == M}
                if 4 in t and (1 not in t or t[4] < t[1]):
                    cross = M
                    break
            summary.append({"frac8": frac, "group": g, "tensor_cores_from_M": cross})
    print(json.dumps({"sweep_crossover": summary}), flush=True)


# ------------------------------------------------------------------ precision search
SEARCH_LINEARS = {"q": (4096, 4096), "k": (4096, 1024), "v": (4096, 1024), "o": (4096, 4096),
                  "gate": (4096, 14336), "up": (4096, 14336), "down": (14336, 4096)}   # (K, N)
SEARCH_LAYERS = 32


def run_search(a):
    """Times the two steps of the precision search on Llama-3-8B shapes.  Saliency: one
    decoder layer's seven linears, W and G fp16 on the device (W ~ N(0, 0.02), G ~ N(0, 1e-3)
    times a log-normal row scale, from a seeded device generator), 872 MB per pass, so
    larger than L2; HBM-bound: its algorithmic bytes are N K (2 + 2) + 4 N per linear.
    Selection: the 10% largest of all 32 layers' 1,376,256 row scores (fp32).  The oracle's
    saliency is timed beside it on a bounded sample of rows of the gate projection."""
    import torch
    from mixed_precision_quantized_mx_b200 import binding as mx
    from mixed_precision_quantized_mx_b200 import build as mxbuild
    from mixed_precision_quantized_mx_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    mxbuild.build()
    peaks = load_peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(a.seed)
    s = torch.cuda.Stream(dev)
    lin = []
    for name, (K, N) in SEARCH_LINEARS.items():
        W = (torch.randn((N, K), generator=gen, device=dev) * 0.02).half()
        rs = torch.exp(torch.randn((N, 1), generator=gen, device=dev))
        G = (torch.randn((N, K), generator=gen, device=dev) * 1e-3 * rs).half()
        lin.append((name, W, G, torch.empty(N, dtype=torch.float32, device=dev)))
    nbytes = sum(W.numel() * 2 + G.numel() * 2 + 4 * S.numel() for _, W, G, S in lin)

    def sal_pass():
        for _, W, G, S in lin:
            mx.mx_saliency(W, G, a.group, S, stream=s)

    with torch.cuda.stream(s):
        for _ in range(a.warmup):
            sal_pass()
    torch.cuda.synchronize()
    steps = a.steps or 20
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(s)
    for _ in range(steps):
        sal_pass()
    ev[1].record(s)
    torch.cuda.synchronize()
    us_sal = ev[0].elapsed_time(ev[1]) * 1e3 / steps
    gbs = nbytes / us_sal / 1e3
    # the global choice over all layers' scores (the layer's own scores, perturbed per layer)
    S_one = torch.cat([S for *_, S in lin])
    S_all = torch.cat([S_one * (1 + 1e-3 * torch.rand(S_one.shape, generator=gen, device=dev))
                       for _ in range(SEARCH_LAYERS)])
    n = S_all.numel()
    n_top = inputs.n8_for(n, 0.10)
    is8 = torch.empty(n, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(s):
        for _ in range(a.warmup):
            mx.mx_select_top(S_all, n_top, is8, stream=s)
    torch.cuda.synchronize()
    ev[0].record(s)
    for _ in range(steps):
        mx.mx_select_top(S_all, n_top, is8, stream=s)
    ev[1].record(s)
    torch.cuda.synchronize()
    us_sel = ev[0].elapsed_time(ev[1]) * 1e3 / steps
    assert int(is8.sum().item()) == n_top
    line = {"metric": "saliency_bandwidth", "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1,
            "steps": steps, "warmup": a.warmup, "us_per_layer_saliency": round(us_sal, 2),
            "select_rows": n, "select_top": n_top, "us_select": round(us_sel, 2),
            "dtype": "f16 in, f64 sums", "data": "synthetic",
            "config": {"workload": "llama3-8b decoder layer, 7 linears, group %d" % a.group,
                       "bytes_per_pass": nbytes, "l2": "inputs 872 MB > L2"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None}}
    if not a.no_cpu_baseline:
        import oracle
        rng = np.random.default_rng(a.seed)
        rows = 256
        Wc = inputs.weights(rng, rows, 4096)
        Gc = inputs.gradients(rng, rows, 4096)
        t0 = time.perf_counter()
        oracle.saliency(Wc, Gc, a.group)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(rows * 4096 * 4 / dt / 1e9, 3), "unit": "GB/s", "cores": 1,
                                "kind": "oracle", "sample": "%d rows of the gate projection (K=4096), bytes counted "
                                                           "as fp16 W and G like the GPU line" % rows}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ block-wise bit widths
BW_TABLE = (2, 3, 4, 8)
BW_PROBS = (0.25, 0.25, 0.40, 0.10)       # about 3.6 bits per weight


def run_blockwise(a):
    """Times mx_bw_gemm on the Llama-3-8B up projection with seed-drawn block widths
    (table {2, 3, 4, 8}, probabilities 0.25 / 0.25 / 0.40 / 0.10), M = 1, 4 and 16, over
    rotated copies of the blob (at least 4x L2, the multiple is in the line), with events
    on the launching stream after warm-up.  Before timing, each M's Y is checked against
    the oracle on 512 sampled outputs.  Algorithmic bytes: model.bw_gemm_bytes."""
    import torch
    import oracle
    from mixed_precision_quantized_mx_b200 import binding as mx
    from mixed_precision_quantized_mx_b200 import build as mxbuild
    from mixed_precision_quantized_mx_b200 import inputs, model

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    mxbuild.build()
    peaks = load_peaks()
    K, N = inputs.SHAPES["llama3-8b-up"]
    rng = np.random.default_rng(a.seed)
    codes = inputs.block_codes(rng, N, K, BW_PROBS)
    meta = oracle.pack_block_codes(codes)
    L = mx.mx_bw_layout_init(N, K, BW_TABLE, meta)
    Wh = inputs.weights(rng, N, K, outlier_frac=0.001)
    W = torch.from_numpy(Wh).to(dev)
    blob0 = torch.empty(L.total_bytes, dtype=torch.uint8, device=dev)
    mx.mx_bw_pack(L, meta, W, blob0)
    torch.cuda.synchronize()
    del W
    bref = oracle.pack_blockwise(Wh, codes, BW_TABLE)
    del Wh
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = int(max(2, math.ceil(4 * l2 / L.total_bytes)))
    blobs = [blob0] + [blob0.clone() for _ in range(R - 1)]
    s = torch.cuda.Stream(dev)
    cpu = None
    if not a.no_cpu_baseline:
        # the oracle's pack + GEMM of M = 1 on the first 256 rows, scaled to GB/s like the GPU line
        rows = 256
        Wc = inputs.weights(rng, rows, K)
        bc = oracle.pack_blockwise(Wc, codes[:rows // 64], BW_TABLE)
        Ac, sc = oracle.quant_act(inputs.activations(rng, 1, K, 4, dtype=np.float32))
        reps, t0 = 0, time.perf_counter()
        while reps == 0 or time.perf_counter() - t0 < 3.0:
            oracle.gemm_blockwise(Ac, sc, bc)
            reps += 1
        dt = (time.perf_counter() - t0) / reps
        cb = mx.mx_bw_layout_init(rows, K, BW_TABLE, oracle.pack_block_codes(codes[:rows // 64])).code_bytes
        cpu = {"value": round(model.bw_gemm_bytes(1, rows, K, cb) / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
               "kind": "oracle", "sample": "M=1 GEMM over the first %d rows, %d calls in 3 s" % (rows, reps)}
    for M in (1, 4, 16):
        X = torch.from_numpy(inputs.activations(rng, M, K, int(round(0.01 * K)))).to(dev)
        Aq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sa = torch.empty(M, dtype=torch.float16, device=dev)
        mx.mx_quant_act(X, Aq, sa)
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        # the result is checked against the oracle on sampled outputs before anything is timed
        mx.mx_bw_gemm(L, blob0, Aq, sa, Y, stream=s)
        torch.cuda.synchronize()
        Ao, so = oracle.quant_act(X.cpu().numpy().astype(np.float32))
        pm = rng.integers(0, M, 512).astype(np.int32)
        pn = rng.integers(0, N, 512).astype(np.int32)
        _, yt, _, _ = oracle.gemm_blockwise(Ao, so, bref, pairs=(pm, pn))
        yg = Y.cpu().numpy()[pm, pn].astype(np.float64)
        rms = float(np.sqrt(np.mean(yt ** 2)))
        if not (np.all(np.abs(yg - yt) <= 2e-3 * np.abs(yt) + 2e-3 * rms)
                and np.linalg.norm(yg - yt) <= 2e-3 * np.linalg.norm(yt)):
            raise SystemExit(f"blockwise GEMM at M={M} differs from the oracle on sampled outputs")
        steps = a.steps or 200
        with torch.cuda.stream(s):
            for i in range(max(a.warmup, R)):
                mx.mx_bw_gemm(L, blobs[i % R], Aq, sa, Y, stream=s)
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(s)
        with torch.cuda.stream(s):
            for i in range(steps):
                mx.mx_bw_gemm(L, blobs[i % R], Aq, sa, Y, stream=s)
        ev1.record(s)
        torch.cuda.synchronize()
        us = ev0.elapsed_time(ev1) * 1e3 / steps
        byts = model.bw_gemm_bytes(M, N, K, L.code_bytes)
        gbs = byts / us / 1e3
        print(json.dumps({
            "metric": "blockwise_gemm_bandwidth", "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1,
            "steps": steps, "warmup": a.warmup, "us_per_call": round(us, 3), "M": M,
            "bits_per_weight": round(L.code_bytes * 8 / (N * K), 3), "dtype": "int8 (dp4a)", "data": "synthetic",
            "config": {"workload": "llama3-8b up K=4096 N=14336, widths %s" % (BW_TABLE,), "rotated_copies": R,
                       "l2": "blob rotates over %d copies (%.0f MB, %.1fx the %.0f MB L2)" % (
                           R, R * L.total_bytes / 1e6, R * L.total_bytes / l2, l2 / 1e6),
                       "checked": "Y within 2e-3 of the oracle on 512 sampled outputs before timing"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None},
            "cpu_baseline": cpu}), flush=True)


# ------------------------------------------------------------------ main arm
TIMED_REPEATS = 5            # the K-step timed region is repeated; the median is reported


def measure_layer(a, lay, workload: str, dev, rank: int, world: int, l2: int, peaks: dict) -> dict:
    """One workload through mx_linear: pack (offline, timed on its own), then W warm-up
    steps and TIMED_REPEATS timed regions of K steps replayed from CUDA graphs over rotated
    copies (>= 4x L2); the dominant kernel timed live on its stream for the roofline; and
    the end-to-end pass through MixedPrecisionLinear.graphed (pinned host X in, Y out)."""
    import torch
    import torch.distributed as dist
    from mixed_precision_quantized_mx_b200 import binding as mx
    from mixed_precision_quantized_mx_b200 import model
    from mixed_precision_quantized_mx_b200.layer import MixedPrecisionLinear

    M, K, N = lay.M, lay.K, lay.N
    g = lay.group
    ag = a.act_group
    n8 = lay.n8
    L = mx.mx_layout_init(N, K, g, n8)
    unit = "GB/s" if M <= HBM_BOUND_MAX_M else "TOPS"
    bound = "hbm" if unit == "GB/s" else "tensor"

    # ---- pack once (offline step), timed on its own
    Wd = torch.from_numpy(lay.W).to(dev)
    is8d = torch.from_numpy(lay.is8).to(dev)
    blob0 = torch.empty(L.total_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mx.mx_pack_weights(L, Wd, is8d, blob0, status=status)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise SystemExit("packer reported an error")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        mx.mx_pack_weights(L, Wd, is8d, blob0)
    e1.record()
    torch.cuda.synchronize()
    pack_ms = e0.elapsed_time(e1) / 3
    del Wd

    # ---- rotated copies beyond L2
    per_step = model.linear_bytes(M, N, K, g, n8, 2)
    R = int(min(64, max(2, math.ceil(4 * l2 / per_step))))
    R = max(2, min(R, int(20e9 // max(per_step, 1))))
    Xh = torch.from_numpy(lay.X)
    Xs = [Xh.to(dev) for _ in range(R)]
    blobs = [blob0] + [blob0.clone() for _ in range(R - 1)]
    Aqs = [torch.empty((M, K), dtype=torch.int8, device=dev) for _ in range(R)]
    sas = [torch.empty((M, K // ag) if ag else (M,), dtype=torch.float16, device=dev) for _ in range(R)]
    Ys = [torch.empty((M, N), dtype=torch.float16, device=dev) for _ in range(R)]
    ws_bytes = mx.mx_linear_workspace_size(L, M, torch.float16, path=a.path, act_group=ag)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    fused = ws_bytes == 0                      # one kernel quantizes X and multiplies
    path_used = mx.mx_gemm_select_path(L, M, path=a.path)

    def step(i):
        mx.mx_linear(L, blobs[i], Xs[i], Ys[i], workspace=ws, path=a.path, act_group=ag)

    gws_bytes = mx.mx_gemm_workspace_size(L, M, path=a.path)     # split sums of a K split, if any
    gws = torch.empty(max(gws_bytes, 16), dtype=torch.uint8, device=dev)

    def gemm_only(i):
        mx.mx_gemm(L, blobs[i], Aqs[i], sas[i], Ys[i], workspace=gws, path=a.path, act_group=ag)

    dominant = step if fused else gemm_only
    for i in range(R):                          # codes the GEMM-only timing reads
        mx.mx_quant_act_grouped(Xs[i], Aqs[i], sas[i], ag)

    s = torch.cuda.Stream(dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for i in range(R):          # eager pass: configures kernels before capture
            step(i)
    torch.cuda.synchronize()

    def capture(fn, count, start=0):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            for j in range(count):
                fn((start + j) % R)
        return gr

    g_full = capture(step, R)
    # estimate step time to size the default K (about one second of timed work)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(3):
        g_full.replay()
    torch.cuda.synchronize()
    est = (time.perf_counter() - t0) / (3 * R)
    K_steps = a.steps or int(min(200000, max(50, 1.0 / max(est, 1e-7))))
    q, rem = divmod(K_steps, R)
    g_rem = capture(step, rem) if rem else None
    qw, rw = divmod(a.warmup, R)
    g_wrem = capture(step, rw) if rw else None

    def replay_steps(nfull, grem):
        for _ in range(nfull):
            g_full.replay()
        if grem is not None:
            grem.replay()

    # the first replay of a graph uploads it: do that for every graph of the timed
    # region before timing (these replays are extra, untimed steps)
    for gr in (g_rem, g_wrem):
        if gr is not None:
            gr.replay()
    torch.cuda.synchronize()

    lead = torch.empty(int(2 * l2) // 4, dtype=torch.int32, device=dev)
    sampler = ClockSampler(dev.index)
    # sustained run of the same step graph (clock reference even for short timed regions)
    sampler.start()
    t_load0 = time.perf_counter()
    while time.perf_counter() - t_load0 < 0.6:
        g_full.replay()
    torch.cuda.synchronize()
    t_load1 = time.perf_counter()

    replay_steps(qw, g_wrem)                       # W warm-up steps
    torch.cuda.synchronize()
    times = []
    t_time0 = time.perf_counter()
    for _ in range(TIMED_REPEATS):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # an L2-sized fill ahead of the start event keeps the device busy while the host
        # submits the step graphs, so the timed region holds the steps and not the
        # submission gap; it also leaves L2 holding none of the step's inputs
        with torch.cuda.stream(s):
            lead.fill_(1)
        ev0.record(s)
        with torch.cuda.stream(s):
            replay_steps(q, g_rem)
        ev1.record(s)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        times.append(max_over_ranks(ev0.elapsed_time(ev1), dev))
    t_time1 = time.perf_counter()
    sampler.stop()
    ms = float(np.median(times))
    units_per_step = step_units(M, K, N, g, n8, unit)
    value = units_per_step * K_steps * world / (ms / 1e3)

    # ---- dominant kernel: the fused kernel (the whole step) or the GEMM call alone,
    # timed live on its stream
    nd = max(R, min(4 * R, 400))
    g_gemm = capture(dominant, nd)
    g_gemm.replay()
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(s)
    with torch.cuda.stream(s):
        for _ in range(3):
            g_gemm.replay()
    d1.record(s)
    torch.cuda.synchronize()
    gemm_ms = d0.elapsed_time(d1) / (3 * nd)
    if bound == "hbm":
        algo = model.linear_bytes(M, N, K, g, n8, 2) if fused else model.gemm_bytes(M, N, K, g, n8)
        achieved = algo / (gemm_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        r_unit = "GB/s"
    else:
        algo = model.gemm_ops(M, N, K)
        achieved = algo / (gemm_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"] * 2.0    # dense int8 = 2x dense bf16 (nominal 4.5 / 2.25 PF)
        r_unit = "TOPS"
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if os.path.exists(tfile):
        rec = json.load(open(tfile)).get(workload)
        if (rec and rec.get("src_digest") == src_digest(path_used) and rec.get("path") == path_used
                and rec.get("fused", False) == fused):
            traffic = rec["dram_bytes_per_launch"]
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": r_unit,
                "frac": achieved / peak, "traffic": traffic,
                "kernel": KERNEL_NAMES[path_used] + (", activation quantizer fused" if fused else ""),
                "algorithmic_per_launch": algo, "launch_ms": gemm_ms,
                "peak_source": (f"{peaks['source']} HBM copy" if bound == "hbm" else
                                f"{peaks['source']} bf16 cuBLAS burst x 2 (nominal int8/bf16 ratio)")}

    # ---- end to end through the public API: pinned host X in, host Y out, every step
    layer = MixedPrecisionLinear.from_blob(blob0)
    Xpin = Xh.pin_memory()
    Ypin = torch.empty((M, N), dtype=torch.float16).pin_memory()
    runner = layer.graphed(Xpin, Ypin, path=a.path, act_group=ag)   # H2D, mx_linear, D2H: one graph
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(3):
        runner.replay()
    torch.cuda.synchronize()
    est_e2e = (time.perf_counter() - t0) / 3
    Ke = max(20, min(K_steps, 5000, int(2.0 / max(est_e2e, 1e-7))))
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(runner.stream)
    for _ in range(Ke):
        runner.replay()
    f1.record(runner.stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / Ke, dev)
    e2e = {"value": units_per_step * world / (e2e_ms / 1e3), "unit": unit,
           "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
           "ms_per_step": e2e_ms,
           "api": "MixedPrecisionLinear.graphed: pinned X read in by a copy kernel, mx_linear, Y written "
                  "to pinned host memory by a copy kernel, one graph per step"}

    clocks = sampler.summary(t_time0, t_time1) or sampler.summary(t_load0, t_load1)
    if clocks is not None and "error" not in clocks:
        clocks["window"] = ("timed regions" if sampler.summary(t_time0, t_time1)
                            else "sustained replay of the same step graph just before the timed regions")
    # fused kernel, or activation quantizer + GEMM (+ the reduction of a K split)
    kernels_per_step = 1 if fused else 2 + (1 if gws_bytes > 0 else 0)
    out = {
        "value": value, "unit": unit, "ms_per_step": ms / K_steps, "steps": K_steps,
        "repeats_ms": [round(t, 4) for t in times],
        "config": {"workload": workload, "M": M, "K": K, "N": N, "group": g, "frac8": a.frac8,
                   "act_group": ag, "n8": n8, "path": path_used, "fused_quantizer": fused,
                   "l2": f"inputs rotate over {R} copies ({R * per_step / 1e6:.0f} MB >= 4x the "
                         f"{l2 / 1e6:.0f} MB L2); no flush",
                   "graphs": "timed steps replayed from CUDA graphs",
                   "timing": f"median of {TIMED_REPEATS} timed regions of K steps"},
        "roofline": roofline, "e2e": e2e,
        "gpu_launches": kernels_per_step * K_steps, "clocks": clocks,
        "tops": model.gemm_ops(M, N, K) * K_steps * world / (ms / 1e3) / 1e12,
        "gbs": model.linear_bytes(M, N, K, g, n8, 2) * K_steps * world / (ms / 1e3) / 1e9,
        "pack": {"ms": pack_ms, "weights_gb_per_s": (N * K * 4) / (pack_ms / 1e3) / 1e9},
    }
    del g_full, g_rem, g_wrem, g_gemm, runner
    del blobs, Xs, Aqs, sas, Ys, ws, gws, lead
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def main():
    a = parse()
    if a.impl == "reference":
        return run_reference(a)
    if a.sweep:
        return run_sweep(a)
    if a.search:
        return run_search(a)
    if a.blockwise:
        return run_blockwise(a)

    import torch
    import torch.distributed as dist
    from mixed_precision_quantized_mx_b200 import binding as mx
    from mixed_precision_quantized_mx_b200 import build as mxbuild
    from mixed_precision_quantized_mx_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    mxbuild.build()
    mx.lib()
    peaks = load_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    M, K, N = WORKLOADS[a.workload]
    lay = inputs.llama_layer(M, K, N, a.frac8, a.group, seed=rank_seed(a.seed, rank))
    primary = measure_layer(a, lay, a.workload, dev, rank, world, l2, peaks)
    secondary = []
    if not a.no_secondary:
        for name in SECONDARY.get(a.workload, ()):
            M2, K2, N2 = WORKLOADS[name]
            assert (K2, N2) == (K, N)
            # the same weights and 8-bit rows, a batch of M2 tokens of the same distribution
            rng = np.random.default_rng(rank_seed(a.seed, rank) + 7)
            lay2 = inputs.Layer(inputs.activations(rng, M2, K, int(round(0.01 * K))), lay.W, lay.is8,
                                lay.group, name)
            sec = measure_layer(a, lay2, name, dev, rank, world, l2, peaks)
            secondary.append((lay2, sec))

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        import oracle
        can = oracle.pack(lay.W, lay.is8, lay.group)
        cpu = cpu_baseline(lay, can, primary["unit"], a.act_group)
        for lay2, sec in secondary:
            sec["cpu_baseline"] = cpu_baseline(lay2, can, sec["unit"], a.act_group, seconds=6.0)

    line = {
        "metric": METRIC, "value": primary["value"], "unit": primary["unit"], "n_gpus": world,
        "steps": primary["steps"], "warmup": a.warmup, "ms_per_step": primary["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic", "config": primary["config"], "roofline": primary["roofline"],
        "cpu_baseline": cpu, "e2e": primary["e2e"], "gpu_launches": primary["gpu_launches"],
        "clocks": primary["clocks"], "tops": primary["tops"], "gbs": primary["gbs"],
        "repeats_ms": primary["repeats_ms"], "pack": primary["pack"],
        "secondary": [dict(sec, metric=METRIC, n_gpus=world, warmup=a.warmup) for _, sec in secondary],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
