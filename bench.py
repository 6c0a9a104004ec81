"""Benchmark of the skew-aware MoE forward layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole layer (route + histogram + kappa, block plan, dispatch,
grouped SwiGLU FFN with the combine) over one batch of seeded synthetic inputs that are
resident in HBM.  The headline workload is the largest single-GPU layer (DeepSeek-V3-shaped,
T=16384, d=7168, E=256, k=8, f=2048).  Before every timed step a 256 MB buffer is written
(L2 flush), outside the step's CUDA events; per-step events on the launching stream split
the step into the stages before the FFN and the FFN itself.  The same JSON line carries:

  kappa_sweep     the skew sweep (T=16384, Qwen3 dims, all four hot experts forced into a
                  fraction p of the tokens, p = 0 .. 1 and 1 with Zipf 1.5): kappa, routed
                  tokens/s, FFN TFLOP/s and roofline fraction per point, and flatness_pct
  fixed_placement the planned layer against the no-replica plan (s = 0) with strict slots
                  (one GPU standing in for P), on the most skewed sweep point
  backward        the backward of the expert computation on the kappa = 1 sweep point
  stages_gbs      achieved HBM GB/s of the dispatch and of the unfused combine
  e2e             the headline through HostPipeline from pinned host buffers
  cpu_baseline    the CPU oracle on a bounded token sample of the headline workload

`--impl reference` times the CPU oracle instead, on the host cores, on a bounded sample of
the same workload.

With N > 1 (torchrun) every rank runs an independent replica of the layer on its own GPU:
the layer has no exchange step on one GPU, so there is no data-path collective; the
process group only carries the barriers and the max over ranks of the timed region.
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
DEFAULT_WORKLOAD = "dsv3_a1"
SWEEP_POINTS = ("sweep_all4_p0_b128", "sweep_all4_p0.1_b128", "sweep_all4_p0.3_b128",
                "sweep_all4_p0.5_b128", "sweep_all4_p1_b128", "sweep_all4_p1_b128_zipf1.5")
FIXED_WORKLOAD = "sweep_all4_p1_b128_zipf1.5"
BACKWARD_WORKLOAD = "sweep_all4_p0_b128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# a timed region of the FFN shorter than this uses the burst peak (the cuBLAS figure of a
# short run), a longer one the sustained peak (a seconds-long run under the power cap)
SUSTAINED_AFTER_S = 2.0
FLUSH_BYTES = 256 << 20
# kernels of one step: route + histogram, kappa, block offsets, plan, dispatch rank and
# gather, FC1, FC2; the dispatch adds its count and prefix kernels when the pairs span more
# than one chunk, and O rows add the combine
LAUNCHES_PER_STEP = 8
DISPATCH_CHUNK = 1024  # pairs per chunk of the dispatch's counting sort


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "of measured"
    return dict(FALLBACK_PEAKS), "of fallback"


def pick_peak(peaks, timed_s):
    """The dense bf16 peak a kernel timed for `timed_s` seconds in total is held to: burst
    for a short region, sustained for a long one."""
    if timed_s < SUSTAINED_AFTER_S:
        return peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]), "burst"
    return peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]), \
        "sustained"


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


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def workload_config(wl, extra=None):
    cfg = {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f,
           "beta": wl.beta, "P": wl.P, "s": wl.s, "alpha": wl.alpha, "hot_p": wl.hot_p,
           "hot_mode": wl.hot_mode, "seed": wl.seed, "parallelism": "replicas"}
    if extra:
        cfg.update(extra)
    return cfg


def rmax_rows(wl) -> int:
    """R_max of the configuration (moe_workspace_size(MOE_WS_ROWS))."""
    n = wl.T * wl.k
    return (n + min(wl.E, n) * (wl.beta - 1)) // wl.beta * wl.beta


def gpu_launches_per_step(wl, mode, sms: int) -> int:
    """Kernels of this library launched per step for an FFN mode (see LAUNCHES_PER_STEP)."""
    chunks = wl.T * wl.k // DISPATCH_CHUNK
    return (LAUNCHES_PER_STEP + 2 * int(chunks > 1) + int(bool(mode & N.MOE_FFN_WRITE_O)) -
            int(bool(mode & N.MOE_FFN_GATHER_X)) - int(ffn_one_launch(wl, mode, sms)))


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


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample(wl, logits, x, get_expert, n_tokens):
    """One oracle forward over the first n_tokens tokens of the workload."""
    from oracle import moe_oracle as O
    return O.moe_forward(logits[:n_tokens], x[:n_tokens], get_expert, k=wl.k, beta=wl.beta,
                         P=wl.P, s=wl.s)


def sample_experts(wl, logits_np, n_tokens):
    """Experts the first n_tokens tokens are routed to (the oracle's own top-k)."""
    from oracle import moe_oracle as O
    ids, _ = O.route_topk(logits_np[:n_tokens], wl.k)
    return sorted(set(int(e) for e in ids.ravel()))


class ExpertStore:
    """fp32 host copies of the expert weights a sample needs, loaded before timing."""

    def __init__(self, load, experts):
        self.w = {e: load(e) for e in experts}

    def __call__(self, e):
        return self.w[e]


def sample_size(wl, logits_np, max_bytes=8e9, max_tokens=4096):
    """The largest token prefix n (at most max_tokens) whose experts' fp32 weights fit in
    max_bytes of host memory."""
    per_expert = 3 * wl.d * wl.f * 4
    n = min(wl.T, max_tokens)
    while n > 1 and len(sample_experts(wl, logits_np, n)) * per_expert > max_bytes:
        n //= 2
    return n


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_oracle(wl, logits_np, x_np, get_expert, n, budget_s):
    """Repeats the oracle over the first n tokens until about budget_s seconds of CPU work
    have passed (at least one run).  Returns (runs, seconds)."""
    oracle_sample(wl, logits_np, x_np, get_expert, n)  # untimed first run
    runs, total = 0, 0.0
    while total < budget_s or runs == 0:
        t0 = time.perf_counter()
        oracle_sample(wl, logits_np, x_np, get_expert, n)
        total += time.perf_counter() - t0
        runs += 1
    return runs, total


def cpu_baseline(wl, logits_h, x_h, w1, w2, budget_s):
    """The oracle as it stands on the host cores, over a token prefix of the workload whose
    experts' weights (copied from the device) fit in host memory."""
    logits_np, x_np = logits_h.numpy(), x_h.float().numpy()
    n = sample_size(wl, logits_np)
    store = ExpertStore(lambda e: (w1[e].float().cpu().numpy(), w2[e].float().cpu().numpy()),
                        sample_experts(wl, logits_np, n))
    runs, dt = time_oracle(wl, logits_np, x_np, store, n, budget_s)
    return {"value": round(n * wl.k * runs / dt, 1), "unit": "tokens/s", "cores": cpu_cores(),
            "kind": "oracle",
            "sample": f"first {n} of {wl.T} tokens of {wl.name} ({len(store.w)} experts), "
                      f"whole layer, {runs} run{'s' if runs > 1 else ''} ({dt:.1f} s, "
                      f"numpy fp32 + OpenBLAS)"}


# ------------------------------------------------------------------ our arm
class Flusher:
    """Writes a buffer larger than L2 (126 MB) so the next step starts with a cold L2."""

    def __init__(self, dev):
        self.buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.v = 0

    def __call__(self):
        self.v ^= 1
        self.buf.fill_(self.v)


def time_layer(layer, logits, x, w1, w2, mode, vmask, steps, warmup, dev, world, flush,
               clocks=None):
    """Warm-up steps, then `steps` timed steps of the whole layer, each preceded by an L2
    flush outside its events.  Per step, events on the launching stream mark the start, the
    end of the stages before the FFN (route, block offsets, plan beside the dispatch) and
    the end of the FFN (and the combine, with O rows).  Returns per-stage mean ms, the sum
    of step times (max over ranks), the wall region and the FFN mode that ran."""
    stream = torch.cuda.current_stream(dev)
    eff = layer.ffn_mode(mode)  # the layer may run a fused-combine call with O rows
    layer.clear_status()
    for _ in range(warmup):
        flush()
        layer(logits, x, w1, w2, mode=mode, variant_mask=vmask)
    torch.cuda.synchronize(dev)
    status = layer.read_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {N.moe_status_string(status)}")
    ev = lambda: torch.cuda.Event(enable_timing=True)
    marks = [[ev() for _ in range(3)] for _ in range(steps)]
    start, stop = ev(), ev()
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter()
    ctx = clocks if clocks is not None else _NullCtx()
    with ctx:
        start.record(stream)
        for i in range(steps):
            flush()
            marks[i][0].record(stream)
            layer.pre_ffn(logits, x, vmask)
            marks[i][1].record(stream)
            layer.ffn(w1, w2, eff, x=x)
            if eff & N.MOE_FFN_WRITE_O:
                layer.combine()
            marks[i][2].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
    t_wall = time.perf_counter() - t_wall
    status = layer.read_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {N.moe_status_string(status)}")
    pre = [m[0].elapsed_time(m[1]) for m in marks]
    ffn = [m[1].elapsed_time(m[2]) for m in marks]
    step_s = sum(p + f for p, f in zip(pre, ffn)) / 1e3
    return {"pre_ms": statistics.mean(pre), "ffn_ms": statistics.mean(ffn),
            "ffn_ms_median": statistics.median(ffn),
            "steps_s": max_over_ranks(step_s, dev),
            "ffn_s": max_over_ranks(sum(ffn) / 1e3, dev),
            "region_s": start.elapsed_time(stop) / 1e3, "wall_s": t_wall, "mode": eff}


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def roofline(wl, ffn_ms, ffn_timed_s, peaks, peak_src, traffic=None):
    """The FFN against the dense bf16 peak (it is a dense contraction, tensor-bound above
    ~250 FLOP/byte): achieved = 6 T k d f (padding rows excluded) / FFN time."""
    achieved = wl.flops / (ffn_ms / 1e3) / 1e12
    peak, kind = pick_peak(peaks, ffn_timed_s)
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    return {"bound": "tensor", "kernel": "expert FFN (FC1+SwiGLU, FC2+combine)",
            "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_source": f"bf16 {kind} {peak_src} (FFN timed {ffn_timed_s:.3f} s in total; "
                           f"the burst peak applies below {SUSTAINED_AFTER_S:g} s of FFN "
                           f"time, the sustained one from there on)",
            "frac_of_burst": round(achieved / burst, 4),
            "frac_of_sustained": round(achieved / sustained, 4),
            "traffic": traffic, "flops_per_launch": wl.flops, "ms_per_launch": round(ffn_ms, 4)}


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
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for _ in range(steps):
        pipe.submit(logits_p, x_p, y_p, w1, w2, mode)
    e1.record(pipe.s_out)
    pipe.drain()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
    del pipe
    return {"value": round(wl.T * wl.k * steps * world / t, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": logits_h.numel() * 4 + x_h.numel() * 2,
            "d2h_bytes_per_step": wl.T * wl.d * 4, "steps": steps,
            "overlap": "H2D of step i+1 and D2H of step i-1 overlap the layer on step i"}


def run_kappa_sweep(args, peaks, peak_src, dev, world, flush):
    """Every all4 beta=128 sweep point: same dims and weights, growing routing skew."""
    from skew_aware_token_b200.layer import MoeLayer
    w1, w2 = synth.make_weights(synth.WORKLOADS[SWEEP_POINTS[0]], dev)
    points = []
    for name in SWEEP_POINTS:
        wl = synth.WORKLOADS[name]
        logits, x = synth.make_logits(wl).to(dev), synth.make_x(wl).to(dev)
        layer = MoeLayer(wl, dev)
        r = time_layer(layer, logits, x, w1, w2, 0, 0, args.sweep_steps, args.warmup, dev,
                       world, flush)
        step_ms = r["steps_s"] / args.sweep_steps * 1e3
        rl = roofline(wl, r["ffn_ms"], r["ffn_s"], peaks, peak_src)
        pi = layer.plan_info.cpu().tolist()
        points.append({"workload": name, "kappa": round(float(layer.kappa[0].item()), 4),
                       "hot_p": wl.hot_p, "alpha": wl.alpha,
                       "tokens_per_s": round(wl.T * wl.k * world / (step_ms / 1e3), 1),
                       "ms_per_step": round(step_ms, 4), "ffn_ms": round(r["ffn_ms"], 4),
                       "ffn_tflops": rl["achieved"], "frac": rl["frac"],
                       "frac_of_burst": rl["frac_of_burst"], "B": pi[0], "tau": pi[1],
                       "makespan": pi[2], "fixed_makespan": pi[5]})
        del layer
    torch.cuda.empty_cache()
    tps = [p["tokens_per_s"] for p in points]
    ffn = [p["ffn_tflops"] for p in points]
    return {"steps": args.sweep_steps, "points": points,
            "flatness_pct": round((max(tps) - min(tps)) / max(tps) * 100, 2),
            "flatness_ends_pct": round(abs(tps[0] - tps[-1]) / max(tps[0], tps[-1]) * 100, 2),
            "ffn_flatness_pct": round((max(ffn) - min(ffn)) / max(ffn) * 100, 2),
            "definition": "flatness_pct = (max - min) / max of layer tokens/s over the points; "
                          "flatness_ends_pct between kappa ~ 1 (p = 0) and the most skewed "
                          "point (p = 1, Zipf 1.5)"}


def run_fixed_placement(args, dev, world, flush):
    """Strict slots (unit u runs only slot u mod P: one GPU standing in for P GPUs), the
    config's replica budget s against s = 0 (the fixed-placement plan): the one-GPU analogue
    of the pages' comparison with fixed placement."""
    from skew_aware_token_b200.layer import MoeLayer
    out = {"workload": FIXED_WORKLOAD, "steps": args.sweep_steps,
           "mode": "MOE_FFN_STRICT_SLOTS (unit u runs only slot u mod P)"}
    base = synth.WORKLOADS[FIXED_WORKLOAD]
    w1, w2 = synth.make_weights(base, dev)
    logits, x = synth.make_logits(base).to(dev), synth.make_x(base).to(dev)
    for tag, wl in (("planned", base), ("fixed", base.with_(s=0))):
        layer = MoeLayer(wl, dev)
        r = time_layer(layer, logits, x, w1, w2, N.MOE_FFN_STRICT_SLOTS, 0, args.sweep_steps,
                       args.warmup, dev, world, flush)
        pi = layer.plan_info.cpu().tolist()
        step_ms = r["steps_s"] / args.sweep_steps * 1e3
        out[tag] = {"s": wl.s, "tokens_per_s": round(wl.T * wl.k * world / (step_ms / 1e3), 1),
                    "ms_per_step": round(step_ms, 4), "ffn_ms": round(r["ffn_ms"], 4),
                    "makespan_blocks": pi[2], "tau": pi[1], "replicas": pi[6]}
        del layer
    out["speedup"] = round(out["planned"]["tokens_per_s"] / out["fixed"]["tokens_per_s"], 3)
    torch.cuda.empty_cache()
    return out


def run_backward(args, peaks, peak_src, dev, world, flush):
    """The backward of the expert computation (moe_dispatch_grad, then the four gradient
    GEMMs of moe_expert_ffn_backward) after a training forward: 12 N d f algorithmic flops
    per step (twice the forward's)."""
    from skew_aware_token_b200.layer import MoeLayer
    wl = synth.WORKLOADS[BACKWARD_WORKLOAD]
    w1, w2 = synth.make_weights(wl, dev)
    logits, x = synth.make_logits(wl).to(dev), synth.make_x(wl).to(dev)
    layer = MoeLayer(wl, dev, train=True)
    layer(logits, x, w1, w2)
    dy = synth.make_dy(wl).to(dev)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(max(args.warmup, 3)):
        flush()
        layer.backward(dy, w1, w2)
    torch.cuda.synchronize(dev)
    steps = args.sweep_steps
    marks = [[ev() for _ in range(3)] for _ in range(steps)]
    barrier(world)
    for i in range(steps):
        flush()
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
    g_total = max_over_ranks(sum(m[1].elapsed_time(m[2]) for m in marks) / 1e3, dev)
    flops = 2 * wl.flops
    g_tflops = flops / (g_ms / 1e3) / 1e12
    peak, kind = pick_peak(peaks, g_total)
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    del layer
    torch.cuda.empty_cache()
    return {"workload": wl.name, "steps": steps, "ms_per_step": round(d_ms + g_ms, 4),
            "stages_ms": {"dispatch_grad": round(d_ms, 4), "gemms": round(g_ms, 4)},
            "flops_per_step": flops,
            "tokens_per_s": round(wl.T * wl.k * world / ((d_ms + g_ms) / 1e3), 1),
            "roofline": {"bound": "tensor",
                         "kernel": "gradient GEMMs (dA+SwiGLU', dX, dW2, dW1)",
                         "achieved": round(g_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(g_tflops / peak, 4),
                         "frac_of_burst": round(g_tflops / burst, 4),
                         "peak_source": f"bf16 {kind} {peak_src}"}}


def run_stage_bandwidth(layer, wl, logits, x, w1, w2, dev, flush, peaks, reps=10):
    """Achieved HBM GB/s of the two data-movement stages, timed alone after an L2 flush:
    the dispatch (rank + gather; algorithmic bytes 2 N d 2: x rows read, Xp rows written)
    and the unfused combine (N d 2 of O rows read + T d 4 of y written)."""
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    layer(logits, x, w1, w2, mode=N.MOE_FFN_WRITE_O)
    torch.cuda.synchronize(dev)
    d_ms, c_ms = [], []
    for _ in range(reps):
        flush()
        e0, e1 = ev(), ev()
        e0.record(stream)
        layer.dispatch(x)
        e1.record(stream)
        flush()
        e2, e3 = ev(), ev()
        e2.record(stream)
        layer.combine()
        e3.record(stream)
        torch.cuda.synchronize(dev)
        d_ms.append(e0.elapsed_time(e1))
        c_ms.append(e2.elapsed_time(e3))
    n = wl.T * wl.k
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    d_bytes, c_bytes = 2 * n * wl.d * 2, n * wl.d * 2 + wl.T * wl.d * 4
    dm, cm = statistics.median(d_ms), statistics.median(c_ms)
    return {"peak_gbs": hbm, "reps": reps,
            "dispatch": {"ms": round(dm, 4), "bytes": d_bytes,
                         "gbs": round(d_bytes / dm / 1e6, 1),
                         "frac": round(d_bytes / dm / 1e6 / hbm, 4),
                         "kernels": "dispatch_rank_kernel + dispatch_gather_kernel"},
            "combine": {"ms": round(cm, 4), "bytes": c_bytes,
                        "gbs": round(c_bytes / cm / 1e6, 1),
                        "frac": round(c_bytes / cm / 1e6 / hbm, 4),
                        "kernels": "combine_kernel (unfused path)"}}


FFN_SOURCES = ("skew_aware_token_b200/csrc/ffn_tcgen05.cu", "skew_aware_token_b200/csrc/ffn_wide.cu",
               "skew_aware_token_b200/csrc/tc_util.cuh", "skew_aware_token_b200/csrc/combine.cu")


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


def run_ours(args, wl, world, rank, local):
    from skew_aware_token_b200.layer import MoeLayer
    dev = torch.device("cuda", local)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peaks, peak_src = load_peaks()
    flush = Flusher(dev)
    logits_h = synth.make_logits(wl)
    x_h = synth.make_x(wl)
    w1, w2 = synth.make_weights(wl, dev)
    logits = logits_h.to(dev)
    x = x_h.to(dev)
    write_o = args.ffn == "write_o"
    layer = MoeLayer(wl, dev, write_o=True, gather_x=args.gather_x,
                     o_rows=None if args.ffn == "auto" else write_o)
    mode = ((N.MOE_FFN_STRICT_SLOTS if args.strict else 0) |
            (N.MOE_FFN_WRITE_O if write_o else 0) | (N.MOE_FFN_SM_PAIR if args.sm_pair else 0) |
            (N.MOE_FFN_ONE_LAUNCH if args.launches == "one" else 0) |
            (N.MOE_FFN_TWO_LAUNCHES if args.launches == "two" else 0))
    vmask = args.variant_mask

    clocks = ClockSampler(local)
    r = time_layer(layer, logits, x, w1, w2, mode, vmask, args.steps, args.warmup, dev, world,
                   flush, clocks=clocks)
    kappa = float(layer.kappa[0].item())
    pi = layer.plan_info.cpu().tolist()
    elapsed = r["steps_s"]
    ms_per_step = elapsed / args.steps * 1e3
    value = wl.T * wl.k * args.steps * world / elapsed
    tflops = wl.flops * args.steps * world / elapsed / 1e12
    weight_bytes = 6 * wl.d * wl.f * sum(1 for c in layer.view("counts").cpu().tolist() if c)
    rl = roofline(wl, r["ffn_ms"], r["ffn_s"], peaks, peak_src,
                  traffic=measured_traffic(wl.name, default_ffn=mode == 0 and not args.gather_x
                                           and args.launches == "auto"))

    extra = {}
    if not args.headline_only:
        extra["stages_gbs"] = run_stage_bandwidth(layer, wl, logits, x, w1, w2, dev, flush,
                                                  peaks)
    e2e = None if args.no_e2e else run_e2e(layer, logits_h, x_h, w1, w2, mode, wl, args,
                                           world, dev)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, logits_h, x_h, w1, w2, args.cpu_budget)
    del layer, w1, w2, logits, x
    torch.cuda.empty_cache()
    if not args.headline_only:
        extra["kappa_sweep"] = run_kappa_sweep(args, peaks, peak_src, dev, world, flush)
        extra["fixed_placement"] = run_fixed_placement(args, dev, world, flush)
        extra["backward"] = run_backward(args, peaks, peak_src, dev, world, flush)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; router logits N(0,1) + Zipf bias, x N(0,1), "
                "weights N(0, 1/sqrt(fan_in)), random-init)",
        "config": workload_config(wl, {
            "kappa": kappa, "strict_slots": bool(args.strict),
            "ffn": "O rows + ordered combine" if r["mode"] & N.MOE_FFN_WRITE_O
            else "FC2 with fused combine",
            "sm_pair": bool(args.sm_pair), "ffn_launches": args.launches,
            "launch": "stream launches, per-step CUDA events",
            "fc1_rows": "gathered from x by row_token" if args.gather_x
            else "Xp (dispatched copy)",
            "l2": f"flushed before every step ({FLUSH_BYTES >> 20} MB written, outside the "
                  f"step's events); expert weights {weight_bytes / 1e9:.2f} GB > 126 MB L2",
            "B": pi[0], "tau": pi[1], "makespan": pi[2], "fixed_makespan": pi[5],
            "variant": pi[3], "variant_mask": args.variant_mask,
            "executor": "work-conserving: any SM takes any slot's tiles (the plan orders "
                        "the tiles; --strict confines SM u to slot u mod P)"}),
        "tflops": round(tflops, 2),
        "stages_ms": {"pre_ffn": round(r["pre_ms"], 4), "ffn": round(r["ffn_ms"], 4)},
        "stages_note": "pre_ffn = route + histogram + kappa, block offsets, dispatch (the "
                       "planner runs beside the dispatch on a second stream); measured inside "
                       "the timed steps",
        "timed_region_s": round(r["region_s"], 4),
        "roofline": rl, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": gpu_launches_per_step(wl, r["mode"] | (N.MOE_FFN_GATHER_X
                                                               if args.gather_x else 0),
                                              sms) * args.steps,
        "clocks": clocks.summary(),
        "impl": "ours",
    }
    line.update(extra)
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ reference arm
def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    logits_h = synth.make_logits(wl)
    x_h = synth.make_x(wl)
    logits_np, x_np = logits_h.numpy(), x_h.float().numpy()
    total = args.warmup + args.steps
    # a token prefix whose experts' weights fit in host memory, then shrunk until one step
    # takes about ref_budget / total seconds
    n = sample_size(wl, logits_np, max_bytes=4e9)
    per_step = max(0.05, args.ref_budget / total)
    # the oracle reads host weights: drawn on the host with the same recipe (the host
    # generator's values differ from the device's; the work is the same)
    load = lambda e: tuple(w.float().numpy() for w in synth.expert_weights(wl, e, "cpu"))
    store = ExpertStore(load, sample_experts(wl, logits_np, n))
    while True:
        t0 = time.perf_counter()
        oracle_sample(wl, logits_np, x_np, store, n)
        dt = time.perf_counter() - t0
        if dt <= per_step or n == 1:
            break
        n = max(1, int(n * per_step / dt))
    for _ in range(args.warmup):
        oracle_sample(wl, logits_np, x_np, store, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(wl, logits_np, x_np, store, n)
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
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--sweep-steps", type=int, default=20,
                    help="timed steps per kappa-sweep point, fixed-placement run and backward")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of CPU work for the oracle baseline sample")
    ap.add_argument("--ref-budget", type=float, default=60.0,
                    help="seconds of CPU work for the whole reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the kappa sweep, fixed placement, backward and stage GB/s")
    ap.add_argument("--variant-mask", type=lambda v: int(v, 0), default=0,
                    help="planner variants (bits 0..3 bounded greedy, bit 4 quota solver; "
                         "0 = the four greedy searches), bit 5 reduction-aware selection, "
                         "bits 8..15 the quota floor u_min, bits 16..23 lambda")
    ap.add_argument("--launches", default="auto", choices=["auto", "one", "two"],
                    help="FC1 and FC2 in one persistent launch (per-tile-half readiness), two "
                         "launches, or the library's choice by layer size (default)")
    ap.add_argument("--gather-x", action="store_true",
                    help="FC1 gathers its rows from x by row_token (no Xp, no gather kernel)")
    ap.add_argument("--ffn", default="auto", choices=["auto", "fused", "write_o"],
                    help="fused: FC2 adds gate*O into y; write_o: FC2 stores O, then "
                         "moe_combine; auto: the layer's choice by the size of y (default)")
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
