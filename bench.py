"""Benchmark of the skew-aware MoE forward layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole layer (route + histogram + kappa, block plan, dispatch,
grouped SwiGLU FFN with the fused combine) over one batch of seeded synthetic inputs that
are resident in HBM.  Prints one JSON line (rank 0).  `--impl reference` times the CPU
oracle instead, on the host cores, on a bounded sample of the same workload.

With N > 1 (torchrun) every rank runs an independent replica of the layer on its own GPU:
the layer has no exchange step on one GPU, so there is no data-path collective; the
process group only carries the barrier and the max over ranks of the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from skew_aware_token_b200 import native as N  # noqa: E402
from skew_aware_token_b200 import synth  # noqa: E402

METRIC = "MoE-layer fwd routed tokens/s and TFLOP/s on 1 B200; % of roofline vs kappa"
DEFAULT_WORKLOAD = "olmoe_a1"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LAUNCHES_PER_STEP = 8  # route, kappa, block offsets, plan, rank, gather, fc1, fc2 (+ combine)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "of measured"
    return dict(FALLBACK_PEAKS), "of fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # NVML missing: report that instead of clocks
            self.nv = None
            self.error = repr(exc)

    _REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self._REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif args.impl == "ours":
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(seconds: float, dev) -> float:
    """The slowest rank's time (each rank passes its own); `dev` holds the reduction's
    tensor (a GPU for NCCL, the CPU for gloo).  One rank: the value itself."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return seconds
    t = torch.tensor([seconds], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def workload_config(wl, extra=None):
    cfg = {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f,
           "beta": wl.beta, "P": wl.P, "s": wl.s, "alpha": wl.alpha, "hot_p": wl.hot_p,
           "hot_mode": wl.hot_mode, "seed": wl.seed, "parallelism": "replicas"}
    if extra:
        cfg.update(extra)
    return cfg


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample(wl, logits, x, get_expert, n_tokens):
    """One oracle forward over the first n_tokens tokens of the workload."""
    from oracle import moe_oracle as O
    return O.moe_forward(logits[:n_tokens], x[:n_tokens], get_expert, k=wl.k, beta=wl.beta,
                         P=wl.P, s=wl.s)


class ExpertCache:
    """fp32 host copies of expert weights for the oracle, loaded on first use and kept
    while they fit in `max_bytes` (oldest dropped first)."""

    def __init__(self, load, max_bytes=6e9):
        self.load, self.max_bytes, self.cache, self.bytes = load, max_bytes, {}, 0

    def __call__(self, e):
        if e not in self.cache:
            w = self.load(e)
            size = sum(a.nbytes for a in w)
            while self.cache and self.bytes + size > self.max_bytes:
                old = next(iter(self.cache))
                self.bytes -= sum(a.nbytes for a in self.cache.pop(old))
            self.cache[e] = w
            self.bytes += size
        return self.cache[e]


def host_expert_getter(w1, w2):
    """Expert weights for the oracle, copied from the device one expert at a time."""
    return ExpertCache(lambda e: (w1[e].float().cpu().numpy(), w2[e].float().cpu().numpy()))


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_oracle(wl, logits_np, x_np, get_expert, budget_s):
    """Times the oracle on the first n tokens, n grown until one run takes about budget_s
    seconds of CPU work; when the whole workload runs faster than that, whole-layer runs
    are repeated until about budget_s has passed.  Returns (n, runs, seconds): `runs` runs
    over the first n tokens took `seconds` in total."""
    n = min(wl.T, 16)
    oracle_sample(wl, logits_np, x_np, get_expert, n)  # untimed: loads the first experts
    while True:
        t0 = time.perf_counter()
        oracle_sample(wl, logits_np, x_np, get_expert, n)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * budget_s:
            return n, 1, dt
        if n >= wl.T:
            runs, total = 1, dt
            while total < budget_s:
                t0 = time.perf_counter()
                oracle_sample(wl, logits_np, x_np, get_expert, n)
                total += time.perf_counter() - t0
                runs += 1
            return n, runs, total
        grow = budget_s / max(dt, 1e-6)
        n = int(min(wl.T, max(n + 1, n * min(grow, 8.0))))


# ------------------------------------------------------------------ our arm
def run_e2e(layer, logits_h, x_h, w1, w2, mode, wl, args, world, dev):
    """The same layer end to end through the public API (`HostPipeline`): every step copies
    that step's inputs (logits, x) from pinned host memory to the device and reads y back
    to pinned host memory; copies of neighbouring steps overlap the layer's work."""
    from skew_aware_token_b200.layer import HostPipeline
    pipe = HostPipeline(layer)
    logits_p = logits_h.pin_memory()
    x_p = x_h.pin_memory()
    y_p = torch.empty(wl.T, wl.d, dtype=torch.float32).pin_memory()
    steps = max(1, min(args.steps, 200))
    for _ in range(3):
        pipe.submit(logits_p, x_p, y_p, w1, w2, mode)
    pipe.drain()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for _ in range(steps):
        pipe.submit(logits_p, x_p, y_p, w1, w2, mode)
    e1.record(pipe.s_out)
    pipe.drain()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
    return {"value": round(wl.T * wl.k * steps * world / t, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": logits_h.numel() * 4 + x_h.numel() * 2,
            "d2h_bytes_per_step": wl.T * wl.d * 4, "steps": steps,
            "overlap": "H2D of step i+1 and D2H of step i-1 overlap the layer on step i"}


FFN_SOURCES = ("skew_aware_token_b200/csrc/ffn_tcgen05.cu", "skew_aware_token_b200/csrc/tc_util.cuh")


def ffn_source_digest() -> str:
    import hashlib
    h = hashlib.sha1()
    for rel in FFN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload: str, default_ffn: bool = True):
    """DRAM bytes (read + write) of one expert-FFN step from the committed ncu capture, or
    None when there is none for this workload, the FFN source changed since it was taken, or
    the run does not use the library's default FFN configuration (the one captured)."""
    if not default_ffn:
        return None
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh).get(workload)
    if not rec or rec.get("ffn_source_sha1") != ffn_source_digest():
        return None
    return rec["bytes_per_step"]


def ffn_one_launch(wl, mode, sms: int) -> bool:
    """Whether moe_expert_ffn runs FC1 and FC2 as one launch for this mode on a GPU with
    `sms` SMs (its rule: forced by MOE_FFN_ONE_LAUNCH, else for a fused single-SM Xp call
    with at most 2 FC1 work items per SM)."""
    if mode & N.MOE_FFN_ONE_LAUNCH:
        return True
    if mode & (N.MOE_FFN_WRITE_O | N.MOE_FFN_STRICT_SLOTS | N.MOE_FFN_SM_PAIR |
               N.MOE_FFN_GATHER_X | N.MOE_FFN_TWO_LAUNCHES):
        return False
    return wl.T * wl.k // 128 * (wl.f // 128) <= 2 * sms


def run_backward(layer, w1, w2, wl, args, dev, peak, peak_src):
    """Times the backward of the expert computation (moe_dispatch_grad, then the four
    gradient GEMMs of moe_expert_ffn_backward) after the layer's last forward: 12 N d f
    algorithmic flops per step (twice the forward's)."""
    dy = synth.make_dy(wl).to(dev)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(max(args.warmup, 3)):
        layer.backward(dy, w1, w2)
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 200))
    marks = [[ev() for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        marks[i][0].record(stream)
        N.moe_dispatch_grad(layer.cfg, dy, layer.row_token, layer.row_gate, layer.plan_info,
                            layer.d_rows, layer.status)
        marks[i][1].record(stream)
        N.moe_expert_ffn_backward(layer.cfg, layer.xp, w1, w2, layer.tiles, layer.plan_info,
                                  layer.block_off, layer.row_token, layer.d_rows,
                                  layer.a_scratch, layer.bwd_scratch, layer.dx, layer.dw1,
                                  layer.dw2, layer.status)
        marks[i][2].record(stream)
    torch.cuda.synchronize(dev)
    status = layer.read_status()
    if status != 0:
        raise RuntimeError(f"device status after backward: {N.moe_status_string(status)}")
    d_ms = statistics.mean(m[0].elapsed_time(m[1]) for m in marks)
    g_ms = statistics.mean(m[1].elapsed_time(m[2]) for m in marks)
    flops = 2 * wl.flops
    g_tflops = flops / (g_ms / 1e3) / 1e12
    return {"steps": steps, "ms_per_step": round(d_ms + g_ms, 4),
            "stages_ms": {"dispatch_grad": round(d_ms, 4), "gemms": round(g_ms, 4)},
            "flops_per_step": flops, "tokens_per_s": round(wl.T * wl.k / ((d_ms + g_ms) / 1e3), 1),
            "roofline": {"bound": "tensor", "kernel": "gradient GEMMs (dA+SwiGLU', dX, dW2, dW1)",
                         "achieved": round(g_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(g_tflops / peak, 4), "peak_source": peak_src}}


def run_ours(args, wl, world, rank, local):
    from skew_aware_token_b200.layer import MoeLayer
    dev = torch.device("cuda", local)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peaks, peak_src = load_peaks()
    logits_h = synth.make_logits(wl)
    x_h = synth.make_x(wl)
    w1, w2 = synth.make_weights(wl, dev)
    logits = logits_h.to(dev)
    x = x_h.to(dev)
    write_o = args.ffn == "write_o"
    layer = MoeLayer(wl, dev, write_o=write_o, gather_x=args.gather_x, train=args.backward)
    stream = torch.cuda.current_stream(dev)
    mode = ((N.MOE_FFN_STRICT_SLOTS if args.strict else 0) |
            (N.MOE_FFN_WRITE_O if write_o else 0) | (N.MOE_FFN_SM_PAIR if args.sm_pair else 0) |
            (N.MOE_FFN_ONE_LAUNCH if args.launches == "one" else 0) |
            (N.MOE_FFN_TWO_LAUNCHES if args.launches == "two" else 0))
    vmask = args.variant_mask

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(record=None):
        if record is None:
            layer(logits, x, w1, w2, mode=mode, variant_mask=vmask)
            return
        record[0].record(stream)
        layer.route(logits)
        record[1].record(stream)
        layer.plan(vmask)
        record[2].record(stream)
        layer.dispatch(x)
        record[3].record(stream)
        layer.ffn(w1, w2, mode, x=x)
        if write_o:
            layer.combine()
        record[4].record(stream)

    graph = None
    if args.graph:
        from skew_aware_token_b200.layer import LayerGraph
        graph = LayerGraph(layer, w1, w2, mode=mode, variant_mask=vmask)
        graph.logits.copy_(logits)
        graph.x.copy_(x)

    layer.clear_status()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = layer.read_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {N.moe_status_string(status)}")

    # per-stage events on the launching stream over the whole timed region
    recs = [[ev() for _ in range(5)] for _ in range(args.steps)]
    start, stop = ev(), ev()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()  # one graph launch per step; stage times from the pass below
            else:
                step(recs[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if graph is not None:
        for i in range(args.steps):
            step(recs[i])
        torch.cuda.synchronize(dev)
    elapsed = max_over_ranks(start.elapsed_time(stop) / 1e3, dev)
    stage_ms = {name: statistics.mean(r[i].elapsed_time(r[i + 1]) for r in recs)
                for i, name in enumerate(["route", "plan", "dispatch", "ffn"])}
    status = layer.read_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {N.moe_status_string(status)}")

    kappa = float(layer.kappa[0].item())
    pi = layer.plan_info.cpu().tolist()
    tokens = wl.T * wl.k * args.steps * world
    value = tokens / elapsed
    tflops = wl.flops * args.steps * world / elapsed / 1e12
    ffn_s = stage_ms["ffn"] / 1e3
    ffn_tflops = wl.flops / ffn_s / 1e12
    # the FFN runs inside a long loop of back-to-back steps: the sustained peak applies
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    weight_bytes = 6 * wl.d * wl.f * sum(1 for c in layer.view("counts").cpu().tolist() if c)
    roofline = {"bound": "tensor", "kernel": "expert FFN (FC1+SwiGLU, FC2+combine)",
                "achieved": round(ffn_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(ffn_tflops / peak, 4),
                "peak_source": f"bf16 sustained {peak_src} (timed inside a long step loop)",
                "traffic": None, "flops_per_launch": wl.flops,
                "ms_per_launch": round(stage_ms["ffn"], 4),
                "frac_of_burst": round(ffn_tflops / burst, 4)}
    roofline["traffic"] = measured_traffic(
        wl.name, default_ffn=mode == 0 and not args.gather_x and args.launches == "auto")

    backward = run_backward(layer, w1, w2, wl, args, dev, peak, peak_src) if args.backward \
        else None

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(layer, logits_h, x_h, w1, w2, mode, wl, args, world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, runs, dt = time_oracle(wl, logits_h.numpy(), x_h.float().numpy(),
                                  host_expert_getter(w1, w2), args.cpu_budget)
        cpu = {"value": n * wl.k * runs / dt, "unit": "tokens/s", "cores": cpu_cores(),
               "kind": "oracle",
               "sample": f"first {n} of {wl.T} tokens of {wl.name}, whole layer, {runs} "
                         f"run{'s' if runs > 1 else ''} ({dt:.1f} s, numpy fp32 + OpenBLAS)"}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; router logits N(0,1) + Zipf bias, x N(0,1), "
                "weights N(0, 1/sqrt(fan_in)), random-init)",
        "config": workload_config(wl, {"kappa": kappa, "strict_slots": bool(args.strict),
                                       "ffn": args.ffn, "sm_pair": bool(args.sm_pair),
                                       "ffn_launches": args.launches,
                                       "launch": "cuda graph replay" if args.graph else "stream launches",
                                       "fc1_rows": "gathered from x by row_token"
                                       if args.gather_x else "Xp (dispatched copy)",
                                       "l2": "inputs larger than L2 "
                                       f"(expert weights {weight_bytes / 1e9:.2f} GB > 126 MB)",
                                       "B": pi[0], "tau": pi[1], "makespan": pi[2],
                                       "fixed_makespan": pi[5], "variant": pi[3],
                                       "variant_mask": args.variant_mask,
                                       "variant_makespans": pi[N.PI["VAR_MAKESPAN"]:
                                                              N.PI["VAR_MAKESPAN"] + 5]}),
        "tflops": round(tflops, 2), "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": roofline, "cpu_baseline": cpu,
        "e2e": e2e,
        "backward": backward,
        "gpu_launches": (LAUNCHES_PER_STEP + int(write_o) - int(args.gather_x) -
                         int(ffn_one_launch(wl, mode | (N.MOE_FFN_GATHER_X if args.gather_x
                                                        else 0), sms))) * args.steps,
        "clocks": clocks.summary(),
        "impl": "ours",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ reference arm
def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    logits_h = synth.make_logits(wl)
    x_h = synth.make_x(wl)
    # the oracle reads host weights: drawn on the host with the same recipe (the host
    # generator's values differ from the device's; the work is the same)
    get_expert = ExpertCache(lambda e: tuple(w.float().numpy()
                                             for w in synth.expert_weights(wl, e, "cpu")))
    if wl.E * 3 * wl.d * wl.f * 4 <= get_expert.max_bytes:
        for e in range(wl.E):
            get_expert(e)

    logits_np, x_np = logits_h.numpy(), x_h.float().numpy()
    total = args.warmup + args.steps
    n, _, _ = time_oracle(wl, logits_np, x_np, get_expert, max(0.05, args.ref_budget / total))
    for _ in range(args.warmup):
        oracle_sample(wl, logits_np, x_np, get_expert, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(wl, logits_np, x_np, get_expert, n)
    elapsed = time.perf_counter() - t0
    value = n * wl.k * args.steps / elapsed
    sample = (f"first {n} of {wl.T} tokens of {wl.name} per step, whole layer "
              f"(numpy fp32 + OpenBLAS)")
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded)", "config": workload_config(wl),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "kind": "oracle",
                         "cores": cpu_cores(), "sample": sample},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of CPU work for the oracle baseline sample")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of CPU work for the whole reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--variant-mask", type=lambda v: int(v, 0), default=0,
                    help="planner variants (bits 0..3 bounded greedy, bit 4 quota solver; "
                         "0 = the four greedy searches), bit 5 reduction-aware selection, "
                         "bits 8..15 the quota floor u_min, bits 16..23 lambda")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the step's kernels one by one instead of replaying the whole "
                         "layer as one CUDA graph (the default)")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward of the expert computation (the forward then "
                         "keeps Z for it)")
    ap.add_argument("--launches", default="auto", choices=["auto", "one", "two"],
                    help="FC1 and FC2 in one persistent launch (per-tile-half readiness), two "
                         "launches, or the library's choice by layer size (default)")
    ap.add_argument("--gather-x", action="store_true",
                    help="FC1 gathers its rows from x by row_token (no Xp, no gather kernel)")
    ap.add_argument("--ffn", default="fused", choices=["fused", "write_o"],
                    help="fused: FC2 adds gate*O into y; write_o: FC2 stores O, then moe_combine")
    ap.add_argument("--sm-pair", action="store_true",
                    help="run the FFN on SM pairs (tcgen05 cta_group::2) instead of single SMs")
    ap.add_argument("--strict", action="store_true",
                    help="strict slots: CTA c only runs slot c mod P (one GPU standing in for P)")
    ap.add_argument("--fixed-placement", action="store_true",
                    help="plan with replica budget s = 0 (the no-replica baseline)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    wl = synth.WORKLOADS[args.workload]
    if args.fixed_placement:
        wl = wl.with_(s=0)
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, wl, world, rank)
        else:
            from skew_aware_token_b200 import build as B
            if not os.path.exists(N.LIB_PATH):
                B.build()
            run_ours(args, wl, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
