#!/usr/bin/env python
"""Throughput of the QLoRA linear layer hot path on B200.

One step = the whole hot path over one batch, for each linear of the
workload (default: the large MLP pair k=8192 -> d=22016 and 22016 -> 8192,
r = 64, alpha = 16, 16384 tokens per GPU):
    nf4_quantize(W0) -> qlora_fwd -> qlora_bwd -> lora_merge -> lora_unmerge
and, with more than one GPU, the data-parallel sum of dA and dB over ranks.

Metric: algorithmic fwd+bwd TFLOP/s, F = 4Tdk + 6Tr(d+k) per linear (no
weight gradient), summed over linears and ranks, divided by the step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s and tokens/s at 1 B200; % of bf16 tensor peak"
L2_BYTES = 126 * 1024 * 1024


def algorithmic_flops(T, d, k, r):
    return 4 * T * d * k + 6 * T * r * (d + k)


def nf4_bytes(d, k):
    """Stored bytes of one NF4 weight: codes, E4M3 constants, group scales, mean."""
    n_b = d * k // 64
    return d * k // 2 + n_b + 4 * ((n_b + 255) // 256) + 4


def algorithmic_bytes(T, d, k, r):
    """Least HBM traffic of one forward plus one backward call: the NF4 weight
    is read by each; A and B are read by each; the forward reads X and writes
    Y and U (fp32); the backward reads X, U and dY and writes dX, dA and dB
    (fp32)."""
    weights = 2 * nf4_bytes(d, k)
    adapters = 2 * 2 * (r * k + d * r) + 4 * (r * k + d * r)
    acts = (2 * T * k + 2 * T * d + 4 * T * r) + (2 * T * k + 4 * T * r + 2 * T * d + 2 * T * k)
    return weights + adapters + acts


def workload(config_index: int, tokens=None):
    cfg = synthetic.config(config_index)
    T = cfg.tokens[0] if tokens is None else tokens
    return cfg, T


def workload_name(cfg, T):
    lin = ", ".join(f"{l.name} k={l.k}->d={l.d}" for l in cfg.linears)
    return f"QLoRA linear layer: {lin}; r={cfg.r}, alpha={cfg.alpha:g}, T={T} tokens per GPU"


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self, wait_first=5.0):
        """Start sampling every 100 ms; returns once the first sample arrived
        (nvidia-smi takes a moment to start) or after `wait_first` seconds."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
            return
        t_end = time.time() + wait_first
        while not self.lines and time.time() < t_end:
            time.sleep(0.02)

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0 = getattr(self, "t_begin", None)
        t1 = getattr(self, "t_end", None)
        window = [(t, ln) for t, ln in self.lines
                  if t0 is None or t1 is None or t0 <= t <= t1]
        for _, ln in window:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle sample
def oracle_sample_step(cfg, rows_d=512, tokens=1024):
    """The oracle on a bounded slice of the first linear: W0 cut to `rows_d`
    output rows, `tokens` tokens; quantise, fwd, bwd, merge, unmerge.
    Returns (algorithmic fwd+bwd flops of the slice, seconds)."""
    from oracle import lora, nf4
    lin = cfg.linears[0]
    lay = synthetic.make_layer(cfg, 0, shape_override=(rows_d, lin.k, tokens))
    t0 = time.perf_counter()
    qt = nf4.quantize(lay.W0)
    Wp = nf4.bf16_to_f64(nf4.dequantize(qt))
    X, A, B, dY = (nf4.bf16_to_f64(a) for a in (lay.X, lay.A, lay.B, lay.dY))
    fw = lora.forward(X, Wp, A, B, cfg.s)
    lora.backward(X, Wp, A, B, cfg.s, dY, fw["U"])
    Wm = lora.merge(Wp, A, B, cfg.s)
    lora.unmerge(nf4.bf16_to_f64(Wm), A, B, cfg.s)
    dt = time.perf_counter() - t0
    return algorithmic_flops(tokens, rows_d, lin.k, cfg.r), dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(cfg, budget_s=15.0):
    flops, dt = oracle_sample_step(cfg)
    reps = 1
    total_f, total_t = flops, dt
    while total_t < budget_s and reps < 8:
        f, t = oracle_sample_step(cfg)
        total_f += f
        total_t += t
        reps += 1
    lin = cfg.linears[0]
    return {"value": total_f / total_t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": (f"{reps} x oracle quantise+fwd+bwd+merge+unmerge of linear '{lin.name}' cut to "
                       f"d=512 rows (k={lin.k}), r={cfg.r}, 1024 tokens; float64 numpy, "
                       f"{total_t:.1f} s")}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg, T = workload(args.config, args.tokens)
    flops_step = 0.0
    times = []
    for i in range(args.warmup + args.steps):
        f, t = oracle_sample_step(cfg)
        if i >= args.warmup:
            times.append(t)
            flops_step = f
    ms = 1e3 * statistics.mean(times)
    value = flops_step / (ms / 1e3) / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_name(cfg, T) + " (oracle: bounded slice per step)",
                   "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "one step = oracle quantise+fwd+bwd+merge+unmerge of the first "
                                   "linear cut to d=512 rows and 1024 tokens"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm
# The files the roofline kernel (gemm_nf4_kernel) is built from: its header,
# the headers that one includes, the C ABI header, and the host file that sets
# its launch parameters.  Its recorded DRAM traffic stays valid while these
# are unchanged (other kernels of the library live in other headers).
GEMM_SOURCES = ("parameter_efficient_fine_nf4_b200/csrc/nf4_gemm.cuh",
                "parameter_efficient_fine_nf4_b200/csrc/gemm_tc.cuh",
                "parameter_efficient_fine_nf4_b200/csrc/ptx.cuh",
                "parameter_efficient_fine_nf4_b200/csrc/nf4_kernels.cuh",
                "parameter_efficient_fine_nf4_b200/csrc/libqlora.cu",
                "include/qlora.h")


def _code_only(text: str) -> str:
    """Source text without comments and blank space, so that edits to comments
    do not invalidate a recorded capture."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash():
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, f), "r", encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def read_traffic(kernel: str):
    """ncu DRAM bytes per launch for `kernel`, if captured on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            t = json.load(f)
        if t.get("source_hash") != kernel_source_hash():
            return None
        return t.get("kernels", {}).get(kernel)
    except Exception:
        return None


FWD_BWD_KERNELS = ("gemm_lora_down", "gemm_fwd_main", "gemm_nf4_fwd", "gemm_nf4_small_fwd", "pad_cols_bf16",
                   "scale_f32_to_bf16_hilo", "gemm_lora_g", "gemm_lora_dB", "splitk_reduce_f32", "gemm_lora_dA",
                   "gemm_bwd_dx", "gemm_nf4_dx", "gemm_nf4_small_dx", "memset")


def measure_write_ceiling(torch, dev, stream, nbytes=512 << 20, reps=5):
    """A plain fill of a buffer larger than L2 (a torch kernel): the rate at
    which this GPU writes HBM, the ceiling of write-dominated kernels."""
    buf = torch.empty(nbytes // 4, dtype=torch.float32, device=dev)
    buf.fill_(1.0)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        buf.fill_(0.5)
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / reps
    del buf
    return {"gbs": nbytes / 1e9 / (ms / 1e3), "how": f"torch fill_ of {nbytes >> 20} MiB, {reps} calls"}


def make_device_layers(torch, q4, cfg, T, dev, rank=0):
    """Device tensors of every linear of `cfg` with T tokens: the frozen W0 drawn
    from the config's distribution (quantised once here), A and B from the
    seeded host recipe, X and dY ~ N(0, 1) drawn on the device."""
    out = []

    def bf16_host(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    for li, lin in enumerate(cfg.linears):
        gen = torch.Generator(device=dev)
        gen.manual_seed(synthetic.seed_for(cfg.index, "W0", li))
        W0 = torch.randn(lin.d, lin.k, generator=gen, device=dev, dtype=torch.float32) * cfg.sigma_w
        A = bf16_host(synthetic.normal_bf16(synthetic.seed_for(cfg.index, "A", li), (cfg.r, lin.k), cfg.sigma_a))
        B = bf16_host(synthetic.normal_bf16(synthetic.seed_for(cfg.index, "B", li), (lin.d, cfg.r), cfg.sigma_b))
        gen.manual_seed(synthetic.seed_for(cfg.index, "X", li) + 1000 * rank)
        X = torch.randn(T, lin.k, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        dY = torch.randn(T, lin.d, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        qw = q4.qlora_nf4_quantize(W0)
        del W0
        nbytes = max(q4.qlora_fwd_workspace_bytes(lin.d, lin.k, cfg.r, T),
                     q4.qlora_bwd_workspace_bytes(lin.d, lin.k, cfg.r, T),
                     q4.lora_merge_workspace_bytes(lin.d, lin.k, cfg.r))
        out.append({"lin": lin, "qw": qw, "A": A, "B": B, "X": X, "dY": dY,
                    "Y": torch.empty(T, lin.d, dtype=torch.bfloat16, device=dev),
                    "U": torch.empty(T, cfg.r, dtype=torch.float32, device=dev),
                    "dX": torch.empty(T, lin.k, dtype=torch.bfloat16, device=dev),
                    "dA": torch.empty(cfg.r, lin.k, dtype=torch.float32, device=dev),
                    "dB": torch.empty(lin.d, cfg.r, dtype=torch.float32, device=dev),
                    "ws": q4.workspace(nbytes, dev)})
    return out


def config_block(torch, q4, dev, stream, flush, peaks, write_ceiling, steps=10, warmup=3):
    """fwd+bwd of every linear of configs 1, 2, 3 and 5 (T = 4096 and T = 16),
    timed like the headline (CUDA events per step on the launch stream, L2
    flushed between steps outside the events), plus merge and unmerge of
    config 3 alone.  Returns the per-config entries of the JSON line."""
    hbm = float(peaks.get("hbm_gbs"))
    burst = float(peaks.get("bf16_tflops"))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    out = {}
    cases = [(1, 16), (2, 4096), (3, 8192), (5, 4096), (5, 16)]
    for ci, T in cases:
        cfg = synthetic.config(ci)
        layers = make_device_layers(torch, q4, cfg, T, dev)

        def step():
            for L in layers:
                q4.qlora_fwd(L["qw"], L["A"], L["B"], cfg.alpha, L["X"], Y=L["Y"], U_save=L["U"], ws=L["ws"])
                q4.qlora_bwd(L["qw"], L["A"], L["B"], cfg.alpha, L["X"], L["U"], L["dY"], dX=L["dX"],
                             dA=L["dA"], dB=L["dB"], ws=L["ws"])

        for _ in range(warmup):
            step()
        torch.cuda.synchronize(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        n0 = q4.qlora_launch_count()
        for i in range(steps):
            flush.zero_()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        launches = (q4.qlora_launch_count() - n0) / steps
        assert q4.qlora_get_device_status() == 0
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        flops = sum(algorithmic_flops(T, L["lin"].d, L["lin"].k, cfg.r) for L in layers)
        nbytes = sum(algorithmic_bytes(T, L["lin"].d, L["lin"].k, cfg.r) for L in layers)
        key = f"config{ci}_T{T}"
        e = {"linears": [f"{L['lin'].name} {L['lin'].k}->{L['lin'].d}" for L in layers], "r": cfg.r,
             "tokens": T, "ms_fwd_bwd": ms, "us_fwd_bwd": 1e3 * ms, "tflops": flops / (ms / 1e3) / 1e12,
             "frac_of_dense_burst": flops / (ms / 1e3) / 1e12 / burst,
             "frac_of_sustained": flops / (ms / 1e3) / 1e12 / sustained,
             "tokens_per_s": T / (ms / 1e3), "launches_per_step": launches,
             "algorithmic_bytes": nbytes, "gbs": nbytes / 1e9 / (ms / 1e3),
             "frac_of_hbm": nbytes / 1e9 / (ms / 1e3) / hbm}
        e["bound"] = "hbm" if T <= 64 else "tensor"
        if T <= 64:
            # a decode-like step is launch-bound on the host: replay it as one
            # CUDA graph (the library's launches are stream-ordered and
            # capturable; tensor maps are baked into the kernel parameters)
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step()
            stream.wait_stream(side)
            torch.cuda.synchronize(dev)
            with torch.cuda.graph(g):
                step()
            for _ in range(warmup):
                g.replay()
            torch.cuda.synchronize(dev)
            gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for i in range(steps):
                flush.zero_()
                gev[i][0].record(stream)
                g.replay()
                gev[i][1].record(stream)
            torch.cuda.synchronize(dev)
            assert q4.qlora_get_device_status() == 0
            gms = statistics.median(a.elapsed_time(b) for a, b in gev)
            e["graph"] = {"us_fwd_bwd": 1e3 * gms, "tflops": flops / (gms / 1e3) / 1e12,
                          "gbs": nbytes / 1e9 / (gms / 1e3), "frac_of_hbm": nbytes / 1e9 / (gms / 1e3) / hbm,
                          "how": "the fwd+bwd step of every linear captured once as a CUDA graph, replayed"}
            del g
        # per-kernel device time of one more step (library profiler: events on
        # the launch stream around every launch)
        flush.zero_()
        torch.cuda.synchronize(dev)
        q4.qlora_profile_begin()
        step()
        st = q4.qlora_profile_end()
        e["kernels_us"] = {x["name"]: round(1e3 * x["total_ms"], 2) for x in st}
        out[key] = e
        if cfg.merge:
            L = layers[0]
            lin = L["lin"]
            Wm = torch.empty(lin.d, lin.k, dtype=torch.bfloat16, device=dev)
            W0u = torch.empty_like(Wm)
            for name, fn, bpw, kern in (
                    ("merge", lambda: q4.lora_merge(L["qw"], L["A"], L["B"], cfg.alpha, W_out=Wm, ws=L["ws"]),
                     2.5 + 1 / 64, "lora_merge"),
                    ("unmerge", lambda: q4.lora_unmerge(Wm, L["A"], L["B"], cfg.alpha, W0_out=W0u, ws=L["ws"]),
                     4.0, "lora_unmerge")):
                for _ in range(warmup):
                    fn()
                torch.cuda.synchronize(dev)
                times = []
                for _ in range(steps):
                    flush.zero_()
                    q4.qlora_profile_begin()
                    fn()
                    st = q4.qlora_profile_end()
                    times.append(sum(x["total_ms"] for x in st if x["name"] == kern))
                ms1 = statistics.median(times)
                gbs = lin.d * lin.k * bpw / 1e9 / (ms1 / 1e3)
                m = {"us": 1e3 * ms1, "gbs": gbs, "frac_of_hbm": gbs / hbm, "bytes_per_weight": bpw}
                if name == "merge" and write_ceiling:
                    m["frac_of_write_ceiling"] = gbs / write_ceiling["gbs"]
                out[f"config{ci}_{name}"] = m
            del Wm, W0u
        del layers
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    import parameter_efficient_fine_nf4_b200 as q4

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        args.gpus = world
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    q4.lib()
    cfg, T = workload(args.config, args.tokens)
    # the library's own communicator for the one exchange (sum of dA and dB)
    comm = q4.communicator_from_process_group() if world > 1 else None

    # ---- resident inputs (per rank: its own tokens, the same frozen weights)
    layers = []
    for li, lin in enumerate(cfg.linears):
        lay = synthetic.make_layer(cfg, li, T=T, with_acts=False)
        gen = torch.Generator(device=dev)
        gen.manual_seed(synthetic.seed_for(cfg.index, "X", li) + 1000 * rank)
        X = torch.randn(T, lin.k, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        dY = torch.randn(T, lin.d, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
        L = {
            "lin": lin,
            "W0": torch.from_numpy(lay.W0).to(dev),
            "A": torch.from_numpy(lay.A.view(np.int16)).view(torch.bfloat16).to(dev),
            "B": torch.from_numpy(lay.B.view(np.int16)).view(torch.bfloat16).to(dev),
            "X": X, "dY": dY,
            "qw": q4.NF4Weight(lin.d, lin.k, dev),
            "Y": torch.empty(T, lin.d, dtype=torch.bfloat16, device=dev),
            "U": torch.empty(T, cfg.r, dtype=torch.float32, device=dev),
            "dX": torch.empty(T, lin.k, dtype=torch.bfloat16, device=dev),
            "dA": torch.empty(cfg.r, lin.k, dtype=torch.float32, device=dev),
            "dB": torch.empty(lin.d, cfg.r, dtype=torch.float32, device=dev),
            "Wm": torch.empty(lin.d, lin.k, dtype=torch.bfloat16, device=dev),
            "W0u": torch.empty(lin.d, lin.k, dtype=torch.bfloat16, device=dev),
        }
        nbytes = max(q4.qlora_quantize_workspace_bytes(lin.d, lin.k),
                     q4.qlora_fwd_workspace_bytes(lin.d, lin.k, cfg.r, T),
                     q4.qlora_bwd_workspace_bytes(lin.d, lin.k, cfg.r, T),
                     q4.lora_merge_workspace_bytes(lin.d, lin.k, cfg.r))
        L["ws"] = q4.workspace(nbytes, dev)
        if args.base == "bf16":
            L["Wb"] = L["W0"].to(torch.bfloat16)
        layers.append(L)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    plain = args.base == "bf16"

    def run_layer(L, X, dY):
        """One pass of the path over one linear: QLoRA (quantise, forward,
        backward, merge, unmerge) or, with --base bf16, plain LoRA (forward,
        backward on the bf16 base)."""
        if plain:
            q4.lora_fwd(L["Wb"], L["A"], L["B"], cfg.alpha, X, Y=L["Y"], U_save=L["U"], ws=L["ws"])
            q4.lora_bwd(L["Wb"], L["A"], L["B"], cfg.alpha, X, L["U"], dY, dX=L["dX"],
                        dA=L["dA"], dB=L["dB"], ws=L["ws"])
        else:
            q4.qlora_nf4_quantize(L["W0"], out=L["qw"], ws=L["ws"])
            q4.qlora_fwd(L["qw"], L["A"], L["B"], cfg.alpha, X, Y=L["Y"], U_save=L["U"], ws=L["ws"])
            q4.qlora_bwd(L["qw"], L["A"], L["B"], cfg.alpha, X, L["U"], dY, dX=L["dX"],
                         dA=L["dA"], dB=L["dB"], ws=L["ws"])
        if comm is not None:
            q4.qlora_grad_allreduce(comm, L["dA"], L["dB"])
        if not plain:
            q4.lora_merge(L["qw"], L["A"], L["B"], cfg.alpha, W_out=L["Wm"], ws=L["ws"])
            q4.lora_unmerge(L["Wm"], L["A"], L["B"], cfg.alpha, W0_out=L["W0u"], ws=L["ws"])

    def step():
        for L in layers:
            run_layer(L, L["X"], L["dY"])

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    # clock samples are taken from before the warm-up on, and only those that
    # fall inside the timed region are kept
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    assert q4.qlora_get_device_status() == 0

    # ---- timed region (device time per step with CUDA events; L2 flushed
    # between steps outside the events)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    clocks.mark("t_begin")
    n0 = q4.qlora_launch_count()
    q4.qlora_profile_begin()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    barrier()
    clocks.mark("t_end")
    stats = q4.qlora_profile_end()
    launches = q4.qlora_launch_count() - n0
    clk = clocks.stop()
    ms_steps = [a.elapsed_time(b) for a, b in evs]
    ms = statistics.mean(ms_steps)
    t = torch.tensor([ms], device=dev, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    flops_rank = sum(algorithmic_flops(T, L["lin"].d, L["lin"].k, cfg.r) for L in layers)
    value = flops_rank * world / (ms / 1e3) / 1e12
    tokens_s = T * world / (ms / 1e3)

    # ---- e2e through the public API with host buffers: every step copies X
    # and dY of every linear in from pinned memory and reads dA and dB back.
    # The copies run on a second stream into one of two device input sets, so
    # the inputs of step i+1 (and of the second linear) arrive while step i
    # computes, as a caller streaming micro-batches would run it.
    host_in = [(L["X"].cpu().pin_memory(), L["dY"].cpu().pin_memory()) for L in layers]
    host_out = [(torch.empty_like(L["dA"], device="cpu").pin_memory(),
                 torch.empty_like(L["dB"], device="cpu").pin_memory()) for L in layers]
    h2d = sum(x.numel() * x.element_size() + y.numel() * y.element_size() for x, y in host_in)
    d2h = sum(a.numel() * a.element_size() + b.numel() * b.element_size() for a, b in host_out)
    sets = [[(L["X"], L["dY"]) for L in layers],
            [(torch.empty_like(L["X"]), torch.empty_like(L["dY"])) for L in layers]]
    copy_stream = torch.cuda.Stream(device=dev)
    ev_ready = [[torch.cuda.Event() for _ in layers] for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n, start_ev):
        copy_stream.wait_event(start_ev)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(ev_free[b])
                for li, ((hx, hdy), (X, dY)) in enumerate(zip(host_in, sets[b])):
                    X.copy_(hx, non_blocking=True)
                    dY.copy_(hdy, non_blocking=True)
                    ev_ready[b][li].record(copy_stream)
            for li, L in enumerate(layers):
                stream.wait_event(ev_ready[b][li])
                run_layer(L, *sets[b][li])
            ev_free[b].record(stream)
            for L, (ha, hb) in zip(layers, host_out):
                ha.copy_(L["dA"], non_blocking=True)
                hb.copy_(L["dB"], non_blocking=True)

    e2e_steps = max(3, min(args.steps, 8))
    barrier()
    for timed in (False, True):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b_ev = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        pipelined(e2e_steps if timed else 2, a)
        b_ev.record(stream)
        b_ev.synchronize()
        torch.cuda.synchronize(dev)
        if timed:
            e2e_ms = [a.elapsed_time(b_ev) / e2e_steps]
    barrier()
    te = torch.tensor([statistics.mean(e2e_ms)], device=dev, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = flops_rank * world / (float(te.item()) / 1e3) / 1e12
    assert q4.qlora_get_device_status() == 0

    # ---- the HBM-bound rows, in the step and alone.  Algorithmic bytes per
    # weight: quantise 4 (W0) + 0.5 (codes) + 1/64 (E4M3 constants); merge and
    # doubleDequant 0.5 + 1/64 + 2 (bf16 out); unmerge 2 + 2.
    weights = sum(L["lin"].d * L["lin"].k for L in layers)
    bpw = {"quantise": 4.5 + 1 / 64, "merge": 2.5 + 1 / 64, "unmerge": 4.0, "dequantise": 2.5 + 1 / 64}
    kernels = {"quantise": ("nf4_quantize_phase1", "nf4_quantize_dq"), "merge": ("lora_merge",),
               "unmerge": ("lora_unmerge",), "dequantise": ("nf4_dequantize",)}

    def per_call_ms(st, names, calls):
        return sum(x["total_ms"] for x in st if x["name"] in names) / calls

    alone = {}
    for name, fn in () if plain else (("quantise", lambda L: q4.qlora_nf4_quantize(L["W0"], out=L["qw"], ws=L["ws"])),
                     ("merge", lambda L: q4.lora_merge(L["qw"], L["A"], L["B"], cfg.alpha, W_out=L["Wm"],
                                                       ws=L["ws"])),
                     ("unmerge", lambda L: q4.lora_unmerge(L["Wm"], L["A"], L["B"], cfg.alpha,
                                                           W0_out=L["W0u"], ws=L["ws"])),
                     ("dequantise", lambda L: q4.qlora_nf4_dequantize(L["qw"], W_out=L["W0u"]))):
        for L in layers:
            fn(L)
        torch.cuda.synchronize(dev)
        q4.qlora_profile_begin()
        for _ in range(5):
            for L in layers:
                fn(L)
        st_alone = q4.qlora_profile_end()
        alone[name] = per_call_ms(st_alone, kernels[name], 5)
    assert q4.qlora_get_device_status() == 0

    fb_names = FWD_BWD_KERNELS
    fb_ms = sum(x["total_ms"] for x in stats if x["name"] in fb_names) / args.steps
    fwd_bwd_value = flops_rank * world / (fb_ms / 1e3) / 1e12 if fb_ms > 0 else None

    # ---- roofline of the dominant kernel (the tcgen05 base GEMM: forward and dX)
    peaks, peak_src = read_peaks()
    hbm = float(peaks.get("hbm_gbs"))
    write_ceiling = None if plain else measure_write_ceiling(torch, dev, stream)
    hbm_rows = {}
    for name in () if plain else bpw:
        gb = weights * bpw[name] / 1e9
        row = {"bytes_per_weight": round(bpw[name], 4),
               "alone_gbs": gb / (alone[name] / 1e3), "alone_frac": gb / (alone[name] / 1e3) / hbm}
        if name in ("merge", "dequantise") and write_ceiling:
            # 2 of the 2.5 bytes per weight are writes: also against a plain fill
            row["alone_frac_of_write_ceiling"] = row["alone_gbs"] / write_ceiling["gbs"]
        ms_step = per_call_ms(stats, kernels[name], args.steps)
        if ms_step > 0:
            row["in_step_gbs"] = gb / (ms_step / 1e3)
            row["in_step_frac"] = gb / (ms_step / 1e3) / hbm
        else:
            row["in_step"] = "not part of the step (the GEMMs dequantise internally)"
        hbm_rows[name] = row
    gemm_names = ("gemm_fwd_main", "gemm_bwd_dx") if plain else ("gemm_nf4_fwd", "gemm_nf4_dx")
    gemm = [s for s in stats if s["name"] in gemm_names]
    g_ms = sum(s["total_ms"] for s in gemm)
    g_launches = sum(s["launches"] for s in gemm)
    g_flops = sum(s["flops"] for s in gemm)
    achieved = g_flops / (g_ms / 1e3) / 1e12 if g_ms > 0 else 0.0
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    peak_burst = float(peaks.get("bf16_tflops"))
    traffic = read_traffic("gemm_tc_kernel" if plain else "gemm_nf4_kernel")
    per_config = None
    if rank == 0 and world == 1 and not args.no_configs and not plain:
        per_config = config_block(torch, q4, dev, stream, flush, peaks, write_ceiling)
    rows = {s["name"]: {"launches": s["launches"], "ms_per_step": s["total_ms"] / args.steps,
                        "share": s["total_ms"] / max(1e-9, sum(x["total_ms"] for x in stats))}
            for s in stats}

    if world > 1:
        dist.barrier(device_ids=[local])
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded W0/A/B from the config recipe, X and dY ~ N(0,1) drawn on device)",
            "config": {"workload": workload_name(cfg, T), "tokens_per_gpu": T,
                       "global_tokens": T * world, "r": cfg.r, "alpha": cfg.alpha,
                       "step": ("per linear: lora_fwd, lora_bwd on the bf16 base (plain LoRA)" if plain else
                                "per linear: nf4_quantize, qlora_fwd, qlora_bwd, lora_merge, lora_unmerge")
                               + (" + all-reduce(dA, dB)" if world > 1 else ""),
                       "base": "bf16" if plain else "nf4",
                       "l2": "inputs larger than L2; L2 flushed (256 MB write) between timed steps",
                       "parallelism": f"dp{world}"},
            "tokens_per_s": tokens_s,
            "fwd_bwd_only": {"value": fwd_bwd_value, "unit": "TFLOP/s",
                             "note": "same flops over the forward and backward kernels of the step alone "
                                     "(quantise, merge and unmerge launches left out)"},
            "roofline": {"kernel": ("gemm_tc_kernel<256> (fwd main + dX on the bf16 base)" if plain else
                                    "gemm_nf4_kernel (fwd + dX, NF4 dequantised inside the GEMM)"),
                         "bound": "tensor",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak if peak else None, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long, "
                                        "power-capped step)",
                         "frac_of_dense_burst": achieved / peak_burst if peak_burst else None,
                         "dense_burst_peak": peak_burst,
                         "launches": g_launches, "ms_per_launch": g_ms / max(1, g_launches)},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": float(te.item()), "steps": e2e_steps,
                    "how": "public API, pinned host X/dY in and dA/dB out every step; copies on a "
                           "second stream into two device input sets, overlapping compute"},
            "gpu_launches": launches // args.steps * args.steps,
            "gpu_launches_per_step": launches / args.steps,
            "clocks": clk,
            "rows": rows,
            "hbm_rows": {"peak_gbs": hbm, "peak_source": f"{peak_src} hbm_gbs",
                         "write_ceiling": write_ceiling,
                         "note": "in the step (clocks held down by the power-capped GEMMs) and alone "
                                 "(5 calls back to back after the timed region)", **hbm_rows},
        }
        if per_config is not None:
            line["configs"] = per_config
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(cfg)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)
        comm.close()
        dist.destroy_process_group()
    return 0


def run_deploy(args):
    """The HBM-bound rows alone on the config's first linear: quantise, merge,
    unmerge, doubleDequant and the Adam step on its A and B (warm-up, then
    `steps` calls of each, CUDA-event timing through the library profiler).
    A diagnostic, not the bench line."""
    import torch
    import parameter_efficient_fine_nf4_b200 as q4
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg, _ = workload(args.config)
    lin = cfg.linears[0]
    lay = synthetic.make_layer(cfg, 0, with_acts=False)
    W0 = torch.from_numpy(lay.W0).to(dev)
    A = torch.from_numpy(lay.A.view(np.int16)).view(torch.bfloat16).to(dev)
    B = torch.from_numpy(lay.B.view(np.int16)).view(torch.bfloat16).to(dev)
    qw = q4.NF4Weight(lin.d, lin.k, dev)
    Wm = torch.empty(lin.d, lin.k, dtype=torch.bfloat16, device=dev)
    W0u = torch.empty_like(Wm)
    ws = q4.workspace(max(q4.qlora_quantize_workspace_bytes(lin.d, lin.k),
                          q4.lora_merge_workspace_bytes(lin.d, lin.k, cfg.r)), dev)
    ops = {"quantise": (lambda: q4.qlora_nf4_quantize(W0, out=qw, ws=ws), 4.5 + 1 / 64,
                        ("nf4_quantize_phase1", "nf4_quantize_dq")),
           "merge": (lambda: q4.lora_merge(qw, A, B, cfg.alpha, W_out=Wm, ws=ws), 2.5 + 1 / 64,
                     ("lora_merge",)),
           "unmerge": (lambda: q4.lora_unmerge(Wm, A, B, cfg.alpha, W0_out=W0u, ws=ws), 4.0,
                       ("lora_unmerge",)),
           "dequantise": (lambda: q4.qlora_nf4_dequantize(qw, W_out=W0u), 2.5 + 1 / 64,
                          ("nf4_dequantize",))}
    # the optimiser step on the adapter factors (A and B together, one call each)
    opt = []
    for shape in ((cfg.r, lin.k), (lin.d, cfg.r)):
        master = torch.randn(shape, device=dev) * 0.02
        opt.append((master, master.to(torch.bfloat16), torch.zeros_like(master), torch.zeros_like(master),
                    torch.randn(shape, device=dev) * 1e-3))
    n_opt = sum(o[0].numel() for o in opt)

    def adam_both():
        for master, w16, m, v, g in opt:
            q4.lora_adam_step(master, w16, m, v, g, step=1, lr=2e-4)

    ops["adam"] = (adam_both, 30.0 * n_opt / (lin.d * lin.k), ("lora_adam_step",))
    peaks, src = read_peaks()
    hbm = float(peaks.get("hbm_gbs"))
    out = {"mode": "deploy-only", "config": {"workload": f"{lin.name}: d={lin.d}, k={lin.k}, r={cfg.r}"},
           "peak_gbs": hbm, "peak_source": f"{src} hbm_gbs"}
    for name, (fn, bpw, kernels) in ops.items():
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        q4.qlora_profile_begin()
        for _ in range(args.steps):
            fn()
        st = q4.qlora_profile_end()
        ms = sum(x["total_ms"] for x in st if x["name"] in kernels) / args.steps
        gbs = lin.d * lin.k * bpw / 1e9 / (ms / 1e3)
        out[name] = {"us_per_call": 1e3 * ms, "gbs": gbs, "frac": gbs / hbm, "bytes_per_weight": bpw}
    assert q4.qlora_get_device_status() == 0
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per GPU instead of the config's own (small profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config block (configs 1, 2, 3, 5) of the JSON line")
    ap.add_argument("--base", choices=["nf4", "bf16"], default="nf4",
                    help="nf4: the QLoRA path (default); bf16: plain LoRA on the bf16 base")
    ap.add_argument("--deploy-only", action="store_true",
                    help="time only quantise, merge, unmerge, doubleDequant and the Adam step "
                         "of the first linear")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    if args.deploy_only:
        return run_deploy(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
