#!/usr/bin/env python
"""Benchmark one DoRA-adapted layer training step on B200.

A step is the whole hot path on one batch: dora_norm (factored row norm, g and
g - 1), dora_forward (LoRA down projection, base GEMM with the near-unity
compose) and dora_backward (compose backward, du, dB, dA, dx), on the
high-rank workload d_out = d_in = 8192, r = 384, s = 0.5, 4096 tokens, bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the step on its own 4096 tokens with
replicated weights and the per-rank dm, dA, dB are summed with NCCL (weak
scaling). Rank 0 prints one JSON line.

Timing: the three calls are captured into CUDA graphs (one per call) and each
timed step replays them between CUDA events, after a 256 MB L2 flush outside
the events. Kernel durations come from the library's own event profiler on a
second, profiled capture of the same calls. `e2e` runs the public Python API
eagerly with every step's inputs copied from pinned host memory and its
results copied back inside the timed region, the copies of neighbouring steps
overlapping the compute on separate streams. `--impl reference` times the CPU float64 oracle
on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DoRA layer fwd+bwd tokens/s and norm TFLOP/s at d_in=8192 r=384 bf16; % roofline"
UNIT = "tokens/s"
WORKLOAD_KEY = "c3"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description="DoRA layer step benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD_KEY, choices=["c2", "c3", "c4a", "c4b", "c5"],
                    help="bf16 workload to time (default: the c3 layer the metric is quoted on)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ref-tokens", type=int, default=256, help="tokens per reference-arm step")
    ap.add_argument("--ref-rows", type=int, default=1024, help="output rows per reference-arm step")
    ap.add_argument("--no-merge", action="store_true",
                    help="skip the inference, full-gradient, DVoRA and deployment-merge measurements")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS if k in p}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- algorithmic work per kernel

def kernel_work(name, wl):
    """(flops, bytes) the method needs for one launch of the named kernel."""
    T, di, do, r = wl.T, wl.d_in, wl.d_out, wl.r
    b = 2  # bf16
    table = {
        "gram_gemm": (2 * r * r * di, b * r * di),
        "norm_gemm": (2 * do * di * r + 2 * do * r * r + 2 * do * di, b * (do * di + r * di + do * r)),
        "u_gemm": (2 * T * di * r, b * (T * di + r * di + T * r)),
        "fwd_compose_gemm": (2 * T * do * (di + r),
                             b * (T * di + do * di + T * r + do * r + 2 * T * do)),
        "compose_bwd": (3 * T * do, b * 3 * T * do + 4 * do),
        "du_gemm": (2 * T * do * r, b * (T * do + do * r + T * r)),
        "dB_gemm": (2 * T * do * r, b * (T * do + T * r + do * r)),
        "dA_gemm": (2 * T * di * r, b * (T * di + T * r + r * di)),
        "dx_gemm": (2 * T * di * (do + r), b * (T * do + do * di + T * r + r * di + T * di)),
        "merge_gemm": (2 * do * di * r + 3 * do * di, b * (2 * do * di + do * r + r * di) + 4 * do),
    }
    return table.get(name, (0, 0))


# Source files that define each kernel: DRAM traffic recorded by ncu stays
# valid only while these files are unchanged.
KERNEL_SOURCES = {
    "fwd_compose_gemm": ("sm100_ptx.cuh", "gemm_sm100.cuh", "dora_bf16.cu"),
    "merge_gemm": ("sm100_ptx.cuh", "gemm_sm100.cuh", "merge_sm100.cuh"),
}


def _code_only(text):
    """Source text without comments and blank lines: comment edits do not change a kernel."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line.strip())


def source_hash(kernel):
    names = KERNEL_SOURCES.get(kernel)
    if names is None:
        return None
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "dora_weight_decomposed_b200", "csrc", n), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary (profiles/ncu_traffic.md),
    if it was taken on the kernel's current sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    want = source_hash(kernel)
    if want is None or not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 3 and cells[0] == kernel and cells[1] == want:
                try:
                    return float(cells[2])
                except ValueError:
                    return None
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, torch, device_index, period_s=0.01):
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                ids = [v for v in vis.split(",") if v.strip()]
                idx = int(ids[device_index]) if ids and ids[device_index].strip().isdigit() else device_index
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report no clocks
            self.error = repr(e)
        self.period = period_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _reasons(self):
        nv = self._nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self._h))

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)
                util = self._nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((mhz, self._reasons(), util))
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t.is_alive():
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.error or "no samples"}
        # The sampler runs only inside the timed region, so every sample is under load.
        loaded = self.samples
        bits = 0
        for _, rs, _ in loaded:
            bits |= rs
        reasons = [n for b, n in sorted(self.REASONS.items()) if bits & b]
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(loaded)}


# ---------------------------------------------------------------- CPU oracle timing

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_step(inp, T, rows=None):
    """Oracle norm + forward + backward on the first T tokens (and, if given,
    the first `rows` output features: a smaller layer with the same d_in and r)."""
    import oracle
    W0, A, B, m, s = (inp[k] for k in ("W0", "A", "B", "m", "s"))
    x, dy = inp["x"][:T], inp["dy"][:T]
    if rows is not None:
        W0, B, m, dy = W0[:rows], B[:rows], m[:rows], dy[:, :rows]
    oracle.norm(W0, A, B, m, s)
    oracle.forward(x, W0, A, B, m, s)
    oracle.backward(dy, x, W0, A, B, m, s)


def time_oracle(inp, T, min_seconds=10.0, max_steps=3):
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle_step(inp, T)
        steps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or steps >= max_steps:
            return steps, el


# ---------------------------------------------------------------- reference arm

def run_reference(args, wl, cfg):
    from dora_inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = make_inputs(wl)
    T = min(args.ref_tokens, wl.T)
    rows = min(args.ref_rows, wl.d_out)
    for _ in range(args.warmup):
        oracle_step(inp, T, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inp, T, rows)
    el = time.perf_counter() - t0
    # Every term of the layer step is linear in d_out, so a step of the full
    # layer costs d_out / rows sample steps.
    full_step_s = (el / args.steps) * (wl.d_out / rows)
    value = T / full_step_s
    cores = blas_threads()
    sample = (f"{T} of {wl.T} tokens and {rows} of {wl.d_out} output rows per step of the {wl.name} layer "
              f"(norm + forward + backward in float64 NumPy, dense W0 + s*B*A), {args.steps} steps; "
              f"rate scaled by rows / d_out to the full layer")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * full_step_s, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

def run_ours(args, wl, cfg):
    import numpy as np
    import torch
    import dora_weight_decomposed_b200 as dw
    from dora_weight_decomposed_b200 import build as dbuild
    from dora_weight_decomposed_b200.dp import allreduce_gradients
    from dora_inputs import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    dbuild.build()
    dw.load_library()

    inp = make_inputs(wl, token_seed=rank)
    bf = torch.bfloat16
    td = {k: torch.from_numpy(inp[k]).to(dev).to(bf).contiguous() for k in ("W0", "A", "B", "x", "dy")}
    W0, A, B, x, dy, s = td["W0"], td["A"], td["B"], td["x"], td["dy"], wl.s
    if inp["m"] is not None:
        m = torch.from_numpy(inp["m"]).to(dev)
    else:
        # Near-unity workloads: m = C (1 + delta), delta ~ U(-delta, delta), with C the layer's own
        # norm from the library (the tests take C from the oracle instead).
        C1, _, _ = dw.dora_norm(W0, A, B, torch.ones(wl.d_out, device=dev), s)
        rng = np.random.default_rng(wl.seed + 7)
        delta = torch.from_numpy(rng.uniform(-wl.delta, wl.delta, wl.d_out)).to(dev, torch.float32)
        m = (C1 * (1.0 + delta)).contiguous()
    T, di, do, r = wl.T, wl.d_in, wl.d_out, wl.r
    f32 = dict(device=dev, dtype=torch.float32)
    C, g, gm1 = torch.empty(do, **f32), torch.empty(do, **f32), torch.empty(do, **f32)
    y = torch.empty(T, do, device=dev, dtype=bf)
    su = torch.empty(T, r, device=dev, dtype=bf)
    pre = torch.empty(T, do, device=dev, dtype=bf)
    dm = torch.empty(do, **f32)
    dA = torch.empty(r, di, device=dev, dtype=bf)
    dB = torch.empty(do, r, device=dev, dtype=bf)
    dx = torch.empty(T, di, device=dev, dtype=bf)
    ws = [torch.empty(max(dw.dora_workspace_size(do, di, r, bf, s, T, op), 256), dtype=torch.uint8, device=dev)
          for op in (dw.DORA_OP_NORM, dw.DORA_OP_FORWARD, dw.DORA_OP_BACKWARD)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def call_norm():
        dw.dora_norm(W0, A, B, m, s, norm_out=C, g_out=g, gm1_out=gm1, ws=ws[0])

    def call_fwd():
        dw.dora_forward(x, W0, A, B, gm1, s, y=y, su_save=su, pre_save=pre, ws=ws[1])

    def call_bwd():
        dw.dora_backward(dy, x, W0, A, B, C, g, su, pre, s, dm=dm, dA=dA, dB=dB, dx=dx, ws=ws[2])

    calls = (call_norm, call_fwd, call_bwd)
    # Warm the library (attributes, tensor-map entry point) before capture.
    for c in calls:
        c()
    torch.cuda.synchronize()

    def capture(profiled):
        graphs = []
        if profiled:
            dw.dora_profile_start(256)
        for c in calls:
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph):
                c()
            graphs.append(gph)
        if profiled:
            dw.dora_profile_stop()
        torch.cuda.synchronize()
        return graphs

    plain = capture(False)
    prof = capture(True)
    launches_per_step = dw.dora_profile_count()

    def replay(graphs):
        for gph in graphs:
            gph.replay()
        if dist is not None:
            allreduce_gradients(dm, dA, dB)

    # ---- warm-up
    for _ in range(args.warmup):
        flush.zero_()
        replay(plain)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()

    # ---- timed region: K steps, events around each step, L2 flushed before each
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    with ClockSampler(torch, local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            e = ev[i]
            e[0].record()
            plain[0].replay()
            e[1].record()
            plain[1].replay()
            e[2].record()
            plain[2].replay()
            e[3].record()
            if dist is not None:
                allreduce_gradients(dm, dA, dB)
            e[4].record()
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[4]) for e in ev]
    phase_ms = {"norm": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
                "forward": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
                "backward": statistics.mean(e[2].elapsed_time(e[3]) for e in ev)}
    if dist is not None:
        phase_ms["allreduce"] = statistics.mean(e[3].elapsed_time(e[4]) for e in ev)
    total_ms = sum(step_ms)
    if dist is not None:
        t = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * T * args.steps / (total_ms / 1e3)

    # ---- per-kernel durations from the profiled capture
    nprof = min(args.steps, 50)
    per = {}
    for _ in range(nprof):
        flush.zero_()
        for gph in prof:
            gph.replay()
        torch.cuda.synchronize()
        for name, ms in dw.dora_profile_read():
            per.setdefault(name, []).append(ms)
    kernels = {}
    for name, v in per.items():
        launches = len(v) / nprof
        avg = sum(v) / len(v)
        fl, by = kernel_work(name, wl)
        kernels[name] = {"ms": avg, "launches_per_step": launches, "share": 0.0,
                         "tflops": (fl / (avg * 1e-3) / 1e12) if fl else None,
                         "gbs": (by / (avg * 1e-3) / 1e9) if by else None}
    tot = sum(k["ms"] * k["launches_per_step"] for k in kernels.values()) or 1.0
    for k in kernels.values():
        k["share"] = k["ms"] * k["launches_per_step"] / tot
    dom = max(kernels, key=lambda n: kernels[n]["ms"] * kernels[n]["launches_per_step"])
    peaks, peak_src = load_peaks()
    fl, by = kernel_work(dom, wl)
    d_ms = kernels[dom]["ms"]
    if dom == "compose_bwd":
        roof = {"bound": "hbm", "achieved": by / (d_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": fl / (d_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["peak_source"] = f"{peak_src} ({'bf16_tflops_sustained' if roof['unit'] == 'TFLOP/s' else 'hbm_gbs'})"
    tr = recorded_traffic(dom)
    roof["traffic"] = tr
    roof["algorithmic_per_launch"] = fl if roof["unit"] == "TFLOP/s" else by
    norm_flops = (2 * do * di * r + 2 * r * r * di + 2 * do * r * r + 2 * do * di + 2 * do * r)

    # ---- end to end through the public API with host buffers
    # Every step copies its inputs (x, dy, and the trained A, B, m) from pinned
    # host memory and its results (y, dm, dA, dB, dx) back, inside the timed
    # region. The frozen W0 stays resident. Steps are pipelined over three
    # streams with two device buffer sets: the copies in for step i + 1 and out
    # for step i - 1 run while step i computes.
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.detach().cpu().pin_memory()
        h_in = [pin(x), pin(dy), pin(A), pin(B), pin(m)]
        h_out = [torch.empty_like(t, device="cpu").pin_memory() for t in (y, dm, dA, dB, dx)]
        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        sets = []
        for k in range(2):
            ins = [torch.empty_like(t) for t in (x, dy, A, B, m)]
            outs = [torch.empty_like(t) for t in (y, dm, dA, dB, dx)]
            extra = [torch.empty_like(t) for t in (C, g, gm1, su, pre)]
            sets.append((ins, outs, extra))
        s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_c = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            k = i % 2
            (xk, dyk, Ak, Bk, mk), outs, (Ck, gk, gm1k, suk, prek) = sets[k]
            yk, dmk, dAk, dBk, dxk = outs
            if i >= 2:
                s_in.wait_event(ev_c[k])  # step i - 2 no longer reads set k
            with torch.cuda.stream(s_in):
                for d_t, h_t in zip((xk, dyk, Ak, Bk, mk), h_in):
                    d_t.copy_(h_t, non_blocking=True)
                ev_in[k].record(s_in)
            s_c.wait_event(ev_in[k])
            if i >= 2:
                s_c.wait_event(ev_out[k])  # results of step i - 2 have left set k
            with torch.cuda.stream(s_c):
                dw.dora_norm(W0, Ak, Bk, mk, s, norm_out=Ck, g_out=gk, gm1_out=gm1k, ws=ws[0], stream=s_c)
                dw.dora_forward(xk, W0, Ak, Bk, gm1k, s, y=yk, su_save=suk, pre_save=prek, ws=ws[1], stream=s_c)
                dw.dora_backward(dyk, xk, W0, Ak, Bk, Ck, gk, suk, prek, s, dm=dmk, dA=dAk, dB=dBk, dx=dxk,
                                 ws=ws[2], stream=s_c)
                if dist is not None:
                    allreduce_gradients(dmk, dAk, dBk)
                ev_c[k].record(s_c)
            s_out.wait_event(ev_c[k])
            with torch.cuda.stream(s_out):
                for h_t, d_t in zip(h_out, outs):
                    h_t.copy_(d_t, non_blocking=True)
                ev_out[k].record(s_out)

        k_e2e = max(3, min(args.steps, 20))
        for i in range(args.warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(s_in)
        for i in range(args.warmup, args.warmup + k_e2e):
            e2e_step(i)
        e_end.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = e_start.elapsed_time(e_end)
        if dist is not None:
            t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": world * T * k_e2e / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": k_e2e, "ms_per_step": e2e_ms / k_e2e,
               "api": "dora_norm/dora_forward/dora_backward (eager, stream=), copies pipelined over three streams",
               "l2": "not flushed: every step's inputs and W0 exceed L2"}
        del sets

    # ---- cached-norm inference: forward only, norm reused, nothing saved for a backward
    infer = None
    if rank == 0 and not args.no_merge:
        wsi = torch.empty(max(dw.dora_workspace_size(do, di, r, bf, s, T, dw.DORA_OP_FORWARD), 256),
                          dtype=torch.uint8, device=dev)
        call_inf = lambda: dw.dora_forward(x, W0, A, B, gm1, s, y=y, save_for_backward=False, ws=wsi)
        call_inf()
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi):
            call_inf()
        iev = []
        for i in range(max(3, args.warmup) + 20):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gi.replay()
            e1.record()
            if i >= max(3, args.warmup):
                iev.append((e0, e1))
        torch.cuda.synchronize()
        i_ms = statistics.median(a.elapsed_time(b_) for a, b_ in iev)
        fl = 2 * T * do * (di + r) + 2 * T * di * r
        infer = {"value": T / (i_ms * 1e-3), "unit": UNIT, "ms_per_batch": i_ms, "tflops": fl / (i_ms * 1e-3) / 1e12,
                 "calls": len(iev), "api": "dora_forward(save_for_backward=False) with the norm of a prior dora_norm",
                 "l2": "flushed before every call"}
        del gi, wsi

    # ---- the backward without the detach of the norm (appendix A eq. A.1), same layer and batch
    full_bwd = None
    if rank == 0 and not args.no_merge:
        wsf = torch.empty(max(dw.dora_workspace_size(do, di, r, bf, s, T, dw.DORA_OP_BACKWARD_FULL), 256),
                          dtype=torch.uint8, device=dev)
        call_full = lambda: dw.dora_backward_full(dy, x, W0, A, B, C, g, su, pre, s, dm=dm, dA=dA, dB=dB, dx=dx,
                                                  ws=wsf)
        call_full()
        gf = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gf):
            call_full()
        fev = []
        for i in range(max(3, args.warmup) + 20):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gf.replay()
            e1.record()
            if i >= max(3, args.warmup):
                fev.append((e0, e1))
        torch.cuda.synchronize()
        f_ms = statistics.median(a.elapsed_time(b_) for a, b_ in fev)
        full_bwd = {"ms": f_ms, "detached_ms": phase_ms["backward"], "calls": len(fev),
                    "api": "dora_backward_full", "l2": "flushed before every call"}
        del gf, wsf

    # ---- DVoRA's extra calls on the same layer: form B' = diag(b) B diag(d), and db, dd from dB'
    vera = None
    if rank == 0 and not args.no_merge:
        bv = torch.linspace(0.5, 1.5, do, device=dev)
        dv = torch.linspace(-1.0, 1.0, r, device=dev)
        Bp = torch.empty_like(B)
        wsv = torch.empty(max(dw.dora_workspace_size(do, 8, r, bf, 1.0, 0, dw.DORA_OP_VERA_GRAD), 256),
                          dtype=torch.uint8, device=dev)
        timings = {}
        for name, fn in (("compose", lambda: dw.dora_vera_compose(B, bv, dv, out=Bp)),
                         ("grad", lambda: dw.dora_vera_grad(B, bv, dv, dB, ws=wsv))):
            fn()
            gv = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gv):
                fn()
            vev = []
            for i in range(max(3, args.warmup) + 20):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                gv.replay()
                e1.record()
                if i >= max(3, args.warmup):
                    vev.append((e0, e1))
            torch.cuda.synchronize()
            timings[name] = statistics.median(a.elapsed_time(b_) for a, b_ in vev)
            del gv
        vb = {"compose": 2 * (2 * do * r) + 4 * (do + r), "grad": 2 * (2 * do * r) + 8 * (do + r)}
        vera = {k: {"us": timings[k] * 1e3, "gbs": vb[k] / (timings[k] * 1e-3) / 1e9} for k in timings}
        vera["api"] = "dora_vera_compose, dora_vera_grad (one CUDA graph per call, L2 flushed)"
        del Bp, wsv

    # ---- deployment merge W' = diag(g) (W0 + s B A) on the same layer (not part of the step)
    merge = None
    if rank == 0 and not args.no_merge:
        Wm = torch.empty_like(W0)
        call_merge = lambda: dw.dora_merge(W0, A, B, g, s, out=Wm)
        for _ in range(3):
            call_merge()
        gm = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gm):
            call_merge()
        mev = []
        for _ in range(20):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gm.replay()
            e1.record()
            mev.append((e0, e1))
        torch.cuda.synchronize()
        del gm
        m_ms = statistics.median(a.elapsed_time(b_) for a, b_ in mev)
        fl, by = kernel_work("merge_gemm", wl)
        gbs, tfl = by / (m_ms * 1e-3) / 1e9, fl / (m_ms * 1e-3) / 1e12
        # Bound: the larger of HBM time and tensor time at the measured burst peaks.
        hbm_bound = by / peaks["hbm_gbs"] >= fl / (peaks["bf16_tflops"] * 1e3)
        mroof = ({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s"} if hbm_bound else
                 {"bound": "tensor", "achieved": tfl, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"})
        mroof["frac"] = mroof["achieved"] / mroof["peak"]
        mroof["peak_source"] = f"{peak_src} ({'hbm_gbs' if hbm_bound else 'bf16_tflops'}, burst)"
        mroof["traffic"] = recorded_traffic("merge_gemm")
        merge = {"us": m_ms * 1e3, "gbs": gbs, "tflops": tfl, "calls": len(mev), "roofline": mroof,
                 "l2": "flushed before every call", "api": "dora_merge (one CUDA graph per call)"}
        del Wm

    status = dw.dora_device_status()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        steps, el = time_oracle(inp, T)
        cpu = {"value": T * steps / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{steps} full step(s) of {T} tokens on the {wl.name} layer in float64 NumPy "
                         f"(dense W0 + s*B*A; norm + forward + backward), {el:.1f} s"}

    if dist is not None:
        del plain, prof
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "norm_tflops": norm_flops / (phase_ms["norm"] * 1e-3) / 1e12, "phase_ms": phase_ms,
            "roofline": roof, "kernels": kernels, "inference": infer, "backward_full": full_bwd, "merge": merge,
            "dvora": vera,
            "gpu_launches": int(launches_per_step * args.steps),
            "clocks": clocks.summary(), "e2e": e2e, "cpu_baseline": cpu, "device_status": status,
            "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms)}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    from dora_inputs import workload
    wl = workload(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    cfg = {"workload": wl.name, "d_out": wl.d_out, "d_in": wl.d_in, "r": wl.r, "s": wl.s,
           "tokens_per_gpu": wl.T, "global_tokens": wl.T * world, "parallelism": f"dp{world}",
           "l2": "flushed before every timed step (256 MB write)",
           "timing": "CUDA graphs per call, CUDA events per step, max over ranks"}
    if args.impl == "reference":
        cfg["timing"] = "wall clock over the CPU oracle steps"
        cfg["l2"] = "not applicable (host CPU)"
        return run_reference(args, wl, cfg)
    return run_ours(args, wl, cfg)


if __name__ == "__main__":
    sys.exit(main())
