"""Benchmark of the MoE layer forward (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one moe_forward (route -> dispatch -> expert GEMMs -> combine, plus
the Switch loss) over one batch of synthetic tokens of the named workload
(default: the Mixtral-shaped layer, N=4096 tokens, d_model=4096, E=8, k=2,
SwiGLU d_ff=14336, bf16).  Under torchrun every rank runs its own batch on
its own GPU (data-parallel tokens, no collective on the data path: weak
scaling); the timed region is bracketed by a barrier and a device
synchronisation, timed with CUDA events and reduced with MAX over ranks.

``--impl reference`` times the fp64 CPU oracle (single thread) on a bounded
sample of the same workload instead; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/sec (bf16, 1 B200); expert-GEMM TFLOPS as % of bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# timed regions at least this long are held against the sustained bf16 peak
# (the power cap has settled: median SM clocks near 1.1-1.3 GHz were seen
# from about half a second of back-to-back expert GEMMs on)
SUSTAINED_REGION_MS = 250.0
L2_BYTES = 126 * 1024 * 1024
# tokens of the workload the CPU oracle handles per reference step (about 1-3 s each)
REF_TOKENS_PER_STEP = {"tiny_fp32": 64, "gpt2_moe": 32, "mixtral": 1, "deepseek_v3": 1, "qwen3_skew": 8,
                       "deepseek_v3_shared": 1}


def kernels_per_step(wl) -> int:
    """libmoe kernels one moe_forward launches: the router (bf16 and E <= 32:
    one fused tcgen05 kernel; bf16 and E > 32: logits + selection; fp32: one
    CUDA-core kernel), the scan (one CTA for E <= 32, else per-expert columns
    + finalize), the row pass (scatter fused with the gather), GEMM1, GEMM2,
    the combine, and a shared expert's two GEMMs."""
    router = 2 if (wl.dtype == "bf16" and wl.E > 32) else 1
    scan = 1 if wl.E <= 32 else 2
    return router + scan + 1 + 2 + 1 + (2 if wl.d_ff_shared else 0)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="mixtral")
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--tokens", type=int, default=0, help="override N (small profiling cases)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward"],
                   help="backward: time moe_backward (fp32 gradients of <dy, y> + losses) instead")
    return p.parse_args()


def load_peaks():
    """The roofline denominators: MEASURED_PEAKS.json's numbers where it has
    them (top-level numeric keys named as in FALLBACK_PEAKS), the fallback
    figures for the rest; the source says which."""
    peaks = dict(FALLBACK_PEAKS)
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        return peaks, "fallback"
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return peaks, "fallback"
    found = {k: float(v) for k, v in d.items() if k in FALLBACK_PEAKS and isinstance(v, (int, float))} \
        if isinstance(d, dict) else {}
    peaks.update(found)
    if not found:
        return peaks, "fallback"
    return peaks, "measured" if len(found) == len(FALLBACK_PEAKS) else "measured (partly fallback)"


def tensor_peak(peaks, region_ms: float):
    """(peak TFLOP/s, its name) for a kernel timed inside a region of
    region_ms: the burst bf16 peak for short regions, the sustained one from
    SUSTAINED_REGION_MS on."""
    if region_ms >= SUSTAINED_REGION_MS:
        return peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), "bf16_tflops_sustained"
    return peaks["bf16_tflops"], "bf16_tflops (burst)"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(
        os.environ.get("WORLD_SIZE", "1"))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest per-rank value (the job's time is its slowest rank's)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weights_bytes(wl) -> int:
    es = 4 if wl.dtype == "f32" else 2
    return wl.E * wl.mats * wl.d_model * wl.d_ff * es


def gemm1_bytes(wl, experts_used: int) -> int:
    """Algorithmic DRAM bytes of GEMM1: the first-layer weights of every
    expert that has rows (W1, and W3 for SwiGLU) read once, x_sorted read,
    h written."""
    es = 4 if wl.dtype == "f32" else 2
    rows = wl.N * wl.k
    mats1 = 2 if wl.act == "swiglu" else 1
    return experts_used * mats1 * wl.d_model * wl.d_ff * es + rows * wl.d_model * es + rows * wl.d_ff * es


def gemm1_bound(flops: float, nbytes: float, tflops_peak: float, hbm_gbs: float) -> str:
    """'hbm' when the kernel's arithmetic intensity is below the ridge point
    of the two peaks (it cannot keep the tensor cores fed from HBM), else
    'tensor'."""
    return "hbm" if flops / max(nbytes, 1.0) < tflops_peak * 1e12 / (hbm_gbs * 1e9) else "tensor"


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(f"{kernel}:{workload}")
    if not ent or "sources" not in ent:
        return None
    h = sources_hash(ent["sources"])
    return ent["bytes_per_launch"] if h is not None and h == ent["sources_sha256_16"] else None


def sources_hash(sources):
    """sha256 (first 16 hex digits) of the given repository files, concatenated in order."""
    hasher = hashlib.sha256()
    for rel in sources:
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src):
            return None
        with open(src, "rb") as f:
            hasher.update(f.read())
    return hasher.hexdigest()[:16]


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons of one GPU, polled through
    NVML from a background thread every `interval_ms` (default 1 ms, so that
    even a timed region of a few tens of milliseconds holds ten or more
    samples); `mark(t0, t1)` keeps the samples of the timed region.  Falls
    back to `nvidia-smi -lms` when NVML is unavailable.  Reads only."""
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event bits (hw_slowdown includes the power brake)
    REASONS = (("hw_slowdown", 0x88), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, cuda_index: int, interval_ms: float = 1.0):
        self.cuda_index = cuda_index
        self.interval_ms = interval_ms
        self.samples = []      # (time.monotonic(), sm_mhz, reasons bitmask)
        self.sm_max = None
        self.source = None
        self.window = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        idx = self.cuda_index
        try:
            import torch
            idx = torch.cuda._get_nvml_device_index(self.cuda_index)
        except Exception:
            pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.source = "nvml"

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                        self.samples.append((time.monotonic(), sm, rs))
                    except Exception:
                        pass
                    time.sleep(self.interval_ms / 1000.0)

            self._thread = threading.Thread(target=poll, daemon=True)
            self._thread.start()
        except Exception:
            self._start_smi()
        return self

    def _start_smi(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.cuda_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"

            def read():
                for line in self._proc.stdout:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        sm, smax = float(parts[1]), float(parts[2])
                    except ValueError:
                        continue
                    self.sm_max = smax
                    rs = 0
                    for (name, bit), val in zip(self.REASONS, parts[5:9]):
                        if val.lower().startswith("active"):
                            rs |= bit
                    self.samples.append((time.monotonic(), sm, rs))

            self._thread = threading.Thread(target=read, daemon=True)
            self._thread.start()
        except OSError:
            self._proc = None

    def mark(self, t0: float, t1: float):
        """The timed region in time.monotonic() seconds; samples outside it are ignored."""
        self.window = (t0, t1)

    def __exit__(self, *exc):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None and self._proc is None:
            self._thread.join(timeout=1)

    def summary(self):
        samples = list(self.samples)
        if self.window is not None:
            t0, t1 = self.window
            samples = [s for s in samples if t0 <= s[0] <= t1]
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0, "source": self.source}
        reasons = sorted({name for _, _, rs in samples for name, bit in self.REASONS if rs & bit})
        return {"sm_mhz": statistics.median(s[1] for s in samples), "sm_max_mhz": self.sm_max, "reasons": reasons,
                "samples": len(samples), "source": self.source,
                "interval_ms": self.interval_ms if self.source == "nvml" else 50}


class OracleSample:
    """The fp64 oracle (single thread) on a bounded sample of the workload's tokens.

    Expert weights are drawn on the host on demand (same recipe as the GPU
    run) and kept in a small LRU cache; only the oracle's own calls --
    routing, the per-token expert FFNs and the weighted sum -- are timed.
    """

    def __init__(self, wl, cache_bytes: int = 6 << 30):
        import numpy as np
        import oracle as O
        import workloads as W
        self.np, self.O, self.W, self.wl = np, O, W, wl
        self.x = W.make_x(wl)
        r = W.make_router(wl)
        self.Wg = r["W_g"].float().numpy().astype(np.float64)
        self.b = None if r["b_e"] is None else r["b_e"].numpy().astype(np.float64)
        self.L = O.lib()
        sh = W.make_shared(wl)
        self.shared = None if sh is None else {
            k: (None if v is None else v.float().numpy().astype(np.float64)) for k, v in sh.items()}
        self.cache = {}
        self.cache_bytes = cache_bytes

    def _expert(self, e):
        if e in self.cache:
            self.cache[e] = self.cache.pop(e)  # most recent last
            return self.cache[e]
        ex = self.W.make_expert(self.wl, e, "cpu")
        arrs = {k: (None if v is None else v.float().numpy().astype(self.np.float64)) for k, v in ex.items()}
        size = sum(a.nbytes for a in arrs.values() if a is not None)
        while self.cache and sum(sum(a.nbytes for a in v.values() if a is not None)
                                 for v in self.cache.values()) + size > self.cache_bytes:
            self.cache.pop(next(iter(self.cache)))
        self.cache[e] = arrs
        return arrs

    def run(self, tokens):
        """Oracle forward of the given token indices; returns seconds spent in the oracle."""
        np, O, wl = self.np, self.O, self.wl
        x = self.x[tokens].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        rt = O.route(x, self.Wg, wl.k, wl.router, wl.norm_topk, wl.routed_scaling, b_sel=self.b, L=self.L)
        spent = time.perf_counter() - t0
        for s in range(len(tokens)):
            y = np.zeros(wl.d_model)
            for j in range(wl.k):
                ew = self._expert(int(rt["ids"][s, j]))
                t0 = time.perf_counter()
                o = O.expert_ffn(x[s], ew["W1"], ew["W2"], wl.act, ew["b1"], ew["W3"], ew["b2"], L=self.L)
                y += rt["w"][s, j] * o
                spent += time.perf_counter() - t0
            if self.shared is not None:
                sw = self.shared
                t0 = time.perf_counter()
                y += O.expert_ffn(x[s], sw["W1"], sw["W2"], wl.act, sw["b1"], sw["W3"], sw["b2"], L=self.L)
                spent += time.perf_counter() - t0
        return spent


def host_info():
    """Host core count and CPU model, reported beside every CPU timing."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


class PinnedToOneCore:
    """Runs the enclosed code with this process pinned to one host core (the
    lowest core it may use), restoring the previous affinity afterwards."""

    def __enter__(self):
        self.core = None
        self.prev = None
        if hasattr(os, "sched_getaffinity"):
            self.prev = os.sched_getaffinity(0)
            self.core = min(self.prev)
            os.sched_setaffinity(0, {self.core})
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            os.sched_setaffinity(0, self.prev)


def cpu_baseline(wl, tokens: int):
    """Oracle tokens/s on the first `tokens` tokens of the workload, pinned to one host core."""
    sample = OracleSample(wl)
    with PinnedToOneCore() as pin:
        t = sample.run(list(range(tokens)))
    return tokens / t, t, pin.core


def run_reference(args, wl):
    rank, _, world = dist_env()
    if rank != 0:
        return
    per = min(REF_TOKENS_PER_STEP.get(wl.name, 4), wl.N)
    sampler = OracleSample(wl)
    nxt = 0

    def take():
        nonlocal nxt
        toks = [(nxt + i) % wl.N for i in range(per)]
        nxt += per
        return toks

    with PinnedToOneCore() as pin:
        for _ in range(args.warmup):
            sampler.run(take())
        total_t = 0.0
        for _ in range(args.steps):
            total_t += sampler.run(take())
    value = per * args.steps / total_t
    sample = (f"{per} token(s) of the {wl.name} workload per step (routing + per-token expert FFNs, "
              f"fp64, single thread pinned to core {pin.core}); value = tokens/s over {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": describe(wl),
        "cpu_baseline": dict({"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                              "pinned_core": pin.core}, **host_info()),
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "the fp64 oracle on the host cores of the GPU box (rank 0 only); n_gpus is the launch's size",
    }
    print(json.dumps(line), flush=True)


def stage_bytes(wl):
    """Algorithmic bytes of the HBM-bound stages.  route: x and W_g read, ids
    and weights written; dispatch: x read, x_sorted written, ids read,
    inv_perm written; combine: y_sorted, weights and inv_perm read, y
    written."""
    es = 4 if wl.dtype == "f32" else 2
    A = wl.N * wl.k
    return {
        "route": wl.N * wl.d_model * es + wl.E * wl.d_model * es + A * 8,
        "dispatch": wl.N * wl.d_model * es + A * wl.d_model * es + A * 8,
        "combine": A * wl.d_model * es + A * 8 + wl.N * wl.d_model * es,
    }


def hbm_fracs(wl, times_us, hbm_gbs):
    """Algorithmic bytes over measured microseconds, against the copy bandwidth."""
    out = {}
    for k, b in stage_bytes(wl).items():
        us = times_us.get(k, 0.0)
        gbs = b / (us / 1e6) / 1e9 if us > 0 else 0.0
        out[k] = {"bytes": b, "us": us, "GB/s": gbs, "frac": gbs / hbm_gbs}
    return out


def isolated_stage_times(M, cfg, wl, inp, dev, rounds: int = 6, warm: int = 2):
    """The HBM-bound entry points each timed alone: moe_route, moe_dispatch
    (histogram, scan, row pass) and moe_combine.  Each call reads its own
    copy of its inputs, rotating over enough copies that they span more than
    twice L2, so every call reads from HBM, and the calls of one stage run
    back to back between one pair of CUDA events (launch gaps hidden as in a
    forward).  Returns mean microseconds per call."""
    import ctypes

    import torch
    L = M.library()
    A, d = wl.N * wl.k, wl.d_model
    es = 4 if wl.dtype == "f32" else 2
    i32 = dict(dtype=torch.int32, device=dev)

    def copies(nbytes):
        return int(max(2, min(8, -(-2 * L2_BYTES // max(nbytes, 1)) + 1)))

    ws = M.workspace(cfg, dev)
    R_x = copies(wl.N * d * es)
    xs_in = [inp["x"].clone() for _ in range(R_x)]
    ids = [torch.empty((wl.N, wl.k), **i32) for _ in range(R_x)]
    w = torch.empty((wl.N, wl.k), dtype=torch.float32, device=dev)
    x_sorted = torch.empty((A, d), dtype=wl.torch_dtype, device=dev)
    inv, offsets, counts, status = (torch.empty(A, **i32), torch.empty(wl.E + 1, **i32), torch.empty(wl.E, **i32),
                                    torch.zeros(1, **i32))
    R_y = copies(A * d * es)
    ys = [torch.randn((A, d), device=dev).to(wl.torch_dtype) for _ in range(R_y)]
    y = torch.empty((wl.N, d), dtype=wl.torch_dtype, device=dev)
    P, st, cfgp = M._ptr, M._stream(), ctypes.byref(cfg)

    def route(i):
        return L.moe_route(cfgp, P(xs_in[i % R_x]), P(inp["W_g"]), P(inp["b_e"]), P(ids[i % R_x]), P(w), None,
                           P(ws), ws.numel(), st)

    def dispatch(i):
        return L.moe_dispatch(cfgp, P(xs_in[i % R_x]), P(ids[i % R_x]), P(x_sorted), None, P(inv), P(offsets),
                              P(counts), P(status), P(ws), ws.numel(), st)

    def combine(i):
        return L.moe_combine(cfgp, P(ys[i % R_y]), P(w), P(inv), P(y), st)

    for i in range(R_x):  # every copy of x gets its routing before the dispatch reads it
        if route(i) != 0:
            raise RuntimeError("moe_route")
    out = {}
    for name, call, R in (("route", route, R_x), ("dispatch", dispatch, R_x), ("combine", combine, R_y)):
        for i in range(warm * R):
            if call(i) != 0:
                raise RuntimeError(name)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(rounds * R):
            call(i)
        e1.record()
        torch.cuda.synchronize()
        out[name] = 1000.0 * e0.elapsed_time(e1) / (rounds * R)
    assert int(status[0]) == 0
    del xs_in, ys
    return out


def describe(wl):
    import workloads as W
    d = W.describe(wl)
    d["parallelism"] = "data-parallel tokens, one batch per GPU"
    return d


def run_native(args, wl):
    import torch
    import torch.distributed as dist

    import mixture_experts_layer_53_b200 as M
    import workloads as W

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    M.library()
    cfg = M.make_config(wl.N, wl.d_model, wl.d_ff, wl.E, wl.k, wl.router, wl.norm_topk, wl.routed_scaling,
                        wl.act, wl.dtype, wl.d_ff_shared)
    inp = W.make_inputs(wl.scaled(seed=wl.seed + 100 * rank) if rank else wl, dev)
    ws = M.workspace(cfg, dev)
    out = M.forward_outputs(cfg, dev)
    b_e = inp["b_e"]
    stream = torch.cuda.current_stream()
    big_inputs = weights_bytes(wl) > 2 * L2_BYTES
    flush = None if big_inputs else torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step(events=None):
        M.moe_forward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], W3=inp["W3"], b1=inp["b1"], b2=inp["b2"],
                      b_e=b_e, gamma=wl.gamma, ws=ws, out=out, stage_events=events, shared=inp["shared"])

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # route, dispatch and combine each alone, inputs rotated past L2; timed
    # before the forwards, so that they run at the clocks a short burst of
    # work sees rather than after seconds of expert GEMMs at the power cap
    kernel_us = isolated_stage_times(M, cfg, wl, inp, dev)

    # inside the timed loop only GEMM1's two boundaries are recorded (the
    # roofline kernel); an event between two kernels of the forward stops the
    # second from being scheduled before the first drains, so the full stage
    # breakdown comes from a separate, untimed pass below
    stage_ev = [M.StageEvents(which=(M.STAGE_NAMES.index("gemm1"), M.STAGE_NAMES.index("gemm1") + 1))
                for _ in range(args.steps)]
    start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clocks:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        assert int(out["status"][0]) == 0, f"device status {int(out['status'][0])}"
        barrier()
        w0 = time.monotonic()
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        t_all0.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)
            start[i].record(stream)
            step(stage_ev[i])
            end[i].record(stream)
        t_all1.record(stream)
        barrier()
        clocks.mark(w0, time.monotonic())
    if flush is None:
        local_ms = t_all0.elapsed_time(t_all1)
    else:
        local_ms = sum(start[i].elapsed_time(end[i]) for i in range(args.steps))
    gemm1_ms = sum(ev.elapsed_ms()["gemm1"] for ev in stage_ev) / args.steps
    total_ms = max_over_ranks(local_ms, world, dev)
    experts_used = int((out["counts"] > 0).sum())  # experts whose weights GEMM1 reads

    # stage breakdown: every boundary recorded, untimed steps after the run
    n_stage = min(args.steps, 20)
    full_ev = [M.StageEvents() for _ in range(n_stage)]
    for i in range(n_stage):
        if flush is not None:
            flush.fill_(i & 0xFF)
        step(full_ev[i])
    torch.cuda.synchronize()
    stages = {k: 0.0 for k in M.STAGE_NAMES}
    for ev in full_ev:
        for k, v in ev.elapsed_ms().items():
            stages[k] += v / n_stage

    # end to end through the public call with host buffers: every step uploads
    # its x from pinned host memory, runs the layer and downloads y and the
    # loss; M.HostPipeline overlaps one step's copies with the neighbouring
    # steps' forwards (upload and download streams, double-buffered tensors).
    # The timed region starts before the first upload and ends after the last
    # download (both joined to the compute stream).
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty_like(out["y"], device="cpu").pin_memory()
    aux_host = torch.empty(1, dtype=torch.float32).pin_memory()
    weights = {k: inp[k] for k in ("W_g", "W1", "W2", "W3", "b1", "b2")}
    weights["b_e"] = b_e
    weights["shared"] = inp["shared"]
    pipe = M.HostPipeline(cfg, weights, gamma=wl.gamma, device=dev)
    for _ in range(max(6, args.warmup)):  # both parities' graphs captured (on their second use) before timing
        pipe.step(x_host, y_host, aux_host)
    pipe.finish()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.upload.wait_stream(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        pipe.step(x_host, y_host, aux_host)
    pipe.flush()  # the last forward and the downloads still owed
    stream.wait_stream(pipe.download)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)



    if rank == 0:
        peaks, peak_src = load_peaks()
        tokens = wl.N * args.steps * world
        value = tokens / (total_ms / 1000.0)
        gemm1_flops = 2 * (2 if wl.act == "swiglu" else 1) * wl.d_model * wl.d_ff * wl.N * wl.k
        gemm1_s = gemm1_ms / 1000.0
        ffn_s = (stages["gemm1"] + stages["gemm2"]) / 1000.0
        # a timed region well under the time the power cap takes to settle is
        # held against the burst bf16 peak, a longer one against the
        # sustained peak; the other fraction is reported beside it
        burst = peaks["bf16_tflops"]
        sustained = peaks.get("bf16_tflops_sustained", burst)
        peak, peak_name = tensor_peak(peaks, total_ms)
        achieved = gemm1_flops / gemm1_s / 1e12
        ffn_tflops = wl.expert_flops / ffn_s / 1e12
        fp32 = wl.dtype == "f32"
        kern = ("simt_gemm_kernel<GELU>" if fp32 else
                ("ffn_gemm_pair_kernel" if wl.N * wl.k / wl.E > 192 else "ffn_gemm_single_kernel") +
                ("<SwiGLU>" if wl.act == "swiglu" else "<GELU>")) + " (GEMM1)"
        roofline_line = {"kernel": kern, "bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} {peak_name} (timed region {total_ms:.0f} ms)",
                         "frac_of_burst_peak": achieved / burst,
                         "frac_of_sustained_peak": achieved / sustained,
                         "traffic": traffic_for("gemm1", wl.name), "flops_per_launch": gemm1_flops}
        g1_bytes = gemm1_bytes(wl, experts_used)
        if gemm1_bound(gemm1_flops, g1_bytes, burst, peaks["hbm_gbs"]) == "hbm":
            # weight streaming (few rows per expert): the kernel is held
            # against the copy bandwidth, its tensor throughput kept beside
            gbs = g1_bytes / gemm1_s / 1e9
            roofline_line.update({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                  "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs",
                                  "bytes_per_launch": g1_bytes, "tensor_tflops": achieved,
                                  "frac_of_burst_peak": achieved / burst})
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": dict(describe(wl), l2=("inputs larger than L2 (expert weights %.2f GB)" % (weights_bytes(wl) / 1e9))
                           if big_inputs else "L2 flushed between steps (256 MiB write), per-step events"),
            "roofline": roofline_line,
            "expert_ffn": {"tflops": ffn_tflops,
                           "frac_of_measured_sustained": ffn_tflops / sustained,
                           "frac_of_measured_burst": ffn_tflops / burst,
                           "frac_of_datasheet_2250": ffn_tflops / 2250.0},
            "stages_ms": stages,
            # each stage inside a forward, every boundary recorded (launch
            # latency included, L2 left warm by the previous stage)
            "hbm_stages": hbm_fracs(wl, {k: 1000.0 * v for k, v in stages.items()}, peaks["hbm_gbs"]),
            # each entry point alone, back to back over input copies larger
            # than L2: moe_route (one kernel for E <= 32), moe_dispatch
            # (histogram + scan + row pass), moe_combine
            "hbm_kernels": hbm_fracs(wl, kernel_us, peaks["hbm_gbs"]),
            "e2e": {"value": tokens / (e2e_ms / 1000.0), "unit": "tokens/s",
                    "h2d_bytes_per_step": inp["x"].numel() * inp["x"].element_size(),
                    "d2h_bytes_per_step": out["y"].numel() * out["y"].element_size() + 4},
            "gpu_launches": kernels_per_step(wl) * args.steps,
            "clocks": clocks.summary(),
        }
        if not args.no_cpu_baseline and world == 1:
            per = min(REF_TOKENS_PER_STEP.get(wl.name, 4) * 16, wl.N)
            v, dt, core = cpu_baseline(wl, per)
            line["cpu_baseline"] = dict({
                "value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "pinned_core": core,
                "sample": f"first {per} tokens of the workload, routing + per-token expert FFNs in fp64, one "
                          f"thread pinned to host core {core} ({dt:.1f} s)"}, **host_info())
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def backward_flops(wl) -> int:
    """Algorithmic FLOPs of one moe_backward: the recomputed pre-activations
    (mats - 1 products), dh = dy_s W2, dx_s (mats - 1), the weight gradients
    (mats), for N k rows of d x d_ff each; the router's 2 dz products; the
    shared expert's 3 mats - 1 products over N rows."""
    m = wl.mats
    rows = wl.N * wl.k
    per = 2 * wl.d_model * wl.d_ff
    expert = rows * per * ((m - 1) + 1 + (m - 1) + m)
    router = 2 * 2 * wl.N * wl.E * wl.d_model
    shared = wl.N * 2 * wl.d_model * wl.d_ff_shared * (3 * m - 1) if wl.d_ff_shared else 0
    return expert + router + shared


def run_backward(args, wl):
    """Times moe_backward.  bf16: the expert products run on the tensor cores
    (roofline: the measured sustained bf16 peak); fp32: on the CUDA cores
    (roofline: 148 SMs x 128 fp32 lanes x 2 FLOP x the sampled SM clock)."""
    import ctypes

    import torch

    import mixture_experts_layer_53_b200 as M
    import workloads as W

    rank, local_rank, world = dist_env()
    if rank != 0:
        return
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    M.library()
    cfg = M.make_config(wl.N, wl.d_model, wl.d_ff, wl.E, wl.k, wl.router, wl.norm_topk, wl.routed_scaling,
                        wl.act, wl.dtype, wl.d_ff_shared)
    inp = W.make_inputs(wl, dev)
    g = torch.Generator().manual_seed(wl.seed * 7 + 9)
    dy = torch.randn((wl.N, wl.d_model), generator=g).to(wl.torch_dtype).to(dev)
    n = int(M.library().moe_backward_workspace_size(ctypes.byref(cfg)))
    ws = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    ws = ws[(-ws.data_ptr()) % 256:][:n]

    def step(out=None):
        return M.moe_backward(cfg, inp["x"], inp["W_g"], inp["W1"], inp["W2"], dy, W3=inp["W3"], b1=inp["b1"],
                              b2=inp["b2"], b_e=inp["b_e"], shared=inp["shared"], aux_coef=1e-2, z_coef=1e-3,
                              ws=ws, out=out)

    out = step()
    for _ in range(max(0, args.warmup - 1)):
        step(out)
    torch.cuda.synchronize()
    assert int(out["status"][0]) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        w0 = time.monotonic()
        e0.record()
        for _ in range(args.steps):
            step(out)
        e1.record()
        torch.cuda.synchronize()
        clocks.mark(w0, time.monotonic())
    ms = e0.elapsed_time(e1) / args.steps
    cl = clocks.summary()
    flops = backward_flops(wl)
    achieved = flops / (ms / 1000.0) / 1e12
    mhz = cl.get("sm_mhz") or 1965.0
    if wl.dtype == "bf16":
        peaks, peak_src = load_peaks()
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        bound, kern = "tensor", ("ffn_gemm_pair_kernel<F32> / ffn_gemm_single_kernel<F32> (expert recompute, dgrad "
                                 "and wgrad products)")
        src = f"{peak_src} bf16_tflops_sustained"
    else:
        peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        bound, kern = "alu", "gemm_generic_kernel (all backward products)"
        src = "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x sampled SM clock"
    line = {
        "metric": "MoE-layer backward tokens/sec (fp32 gradients, 1 B200)", "value": wl.N / (ms / 1000.0),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": describe(wl),
        "roofline": {"kernel": kern, "bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": src, "flops_per_step": flops,
                     "note": "achieved = all backward FLOPs over the whole step (recomputation, element-wise and "
                             "router kernels included)"},
        "clocks": cl,
    }
    print(json.dumps(line), flush=True)


def relaunch_under_torchrun(args) -> int:
    """`--gpus N` (N > 1) outside torchrun: run this script again as N ranks
    on this node, one per GPU, and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args))
    _, _, world = dist_env()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE {world}; reporting the launched {world}",
              file=sys.stderr)
    import workloads as W
    wl = W.WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.scaled(N=args.tokens)
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.which == "backward":
        run_backward(args, wl)
    else:
        run_native(args, wl)


if __name__ == "__main__":
    main()
