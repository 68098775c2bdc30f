#!/usr/bin/env python
"""Benchmark of the MoE layer forward: routed tokens/s on B200.

One step = one whole layer forward (router, dispatch, grouped SwiGLU experts,
combine) over one batch of T tokens, through moe_forward.  Default workload:
the Mixtral-shaped dropless layer (T=8192, D=4096, F=14336, E=8, K=2, bf16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on the host cores
    python bench.py --pass train ...       # a training step: forward + backward

With --pass train one step is moe_forward_train + moe_backward (the gradient
of sum <dY, y> + 0.01 balance + 0.001 z) over one batch, and the line reports
training-step tokens/s with the backward kernels' stage times.

N > 1 runs under torchrun: one independent replica per GPU (the layer is
per-token, so ranks share nothing on the data path); value = all ranks'
tokens / the slowest rank's device time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import (WORKLOADS, Workload, make_inputs, make_output_grad,  # noqa: E402
                       make_tokens)

METRIC = "routed tokens/s per MoE layer fwd on 1 B200; % bf16 tensor peak / % HBM BW"
UNIT = "tokens/s"
METRIC_TRAIN = "routed tokens/s per MoE layer training step (fwd + bwd) on 1 B200"
C_BAL, C_Z = 0.01, 0.001  # the lab's loss coefficients
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ ranks --

def rank_info():
    r = int(os.environ.get("RANK", "0"))
    w = int(os.environ.get("WORLD_SIZE", "1"))
    lr = int(os.environ.get("LOCAL_RANK", str(r)))
    return r, w, lr


def init_dist(world: int, backend: str):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def materialize_events(event_lists, stream):
    """Give every torch event its CUDA handle before a timed region: torch
    creates it lazily at the first record, and the library's trace attach
    records a handle-less event once to obtain one, which inside the timed
    region would add an event record per stage boundary and step."""
    for evs in event_lists:
        for e in evs:
            if not e.cuda_event:
                e.record(stream)
    torch.cuda.synchronize()


def aggregate(ms_total_local: float, world: int, T: int, steps: int, device) -> tuple:
    """(ms per step, tokens/s of the whole job): the slowest rank's device time
    over all ranks' tokens (each rank processes its own T tokens per step)."""
    ms_total = max_over_ranks(ms_total_local, world, device)
    ms_step = ms_total / steps
    return ms_total, ms_step, world * T / (ms_step / 1e3)


def rank_token_seed(rank: int) -> int:
    """Each replica routes its own batch of tokens (weights are shared)."""
    return 1000 + rank


# ------------------------------------------------------------------ peaks --

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=2)
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sms.append(float(parts[0]))
                maxs.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


# ------------------------------------------------------------- the layer --

def algorithmic(wl: Workload, counts, kept_rows: int):
    """Algorithmic work of one step (the units of the roofline)."""
    s = wl.elem_bytes
    R = kept_rows
    return {
        "gateup_flop": 4.0 * R * wl.D * wl.F,
        "down_flop": 2.0 * R * wl.F * wl.D,
        "dispatch_bytes": float(wl.T * wl.D * s + R * wl.D * s),
        "combine_bytes": float(R * wl.D * s + wl.T * wl.D * s),
        "active_weight_bytes": float(sum(1 for c in counts if c > 0) * 3 * wl.D * wl.F * s),
        # gate/up GEMM: each active expert's two weight matrices, its rows of
        # x_perm read once, h written once
        "gateup_bytes": float(sum(1 for c in counts if c > 0) * 2 * wl.D * wl.F * s
                              + R * wl.D * s + R * wl.F * s),
        # router: x read once, fp32 router weight, routed ids and weights written
        "route_bytes": float(wl.T * wl.D * s + wl.D * wl.E * 4 + wl.T * wl.K * 8),
        "shared_flop": 6.0 * wl.T * wl.D * wl.F_shared,
    }


# sources that define the expert GEMM kernels (a recorded traffic figure is
# only valid while these are unchanged)
GEMM_SOURCES = ("ffn_tc.cu", "common.cuh")


def kernel_source_hash(files=GEMM_SOURCES) -> str:
    csrc = os.path.join(ROOT, "mixture_experts_layer_55_b200", "csrc")
    h = hashlib.sha256()
    for n in sorted(files):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


# and those of the backward's weight-gradient GEMM (the training step's roofline kernel)
WGRAD_SOURCES = ("wgrad_tc.cu", "common.cuh")


def recorded_traffic(workload: str, kernel: str, files=GEMM_SOURCES):
    """DRAM bytes per launch from a committed ncu summary, if the kernels have
    not changed since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(files):
        return None
    return e.get("dram_bytes_per_launch")


# the other layer shapes measured after the headline one, in the same process
# (each freed before the next); the Mixtral shape again with a shared expert of
# its own hidden size measures the shared-expert stage
EXTRA_CONFIGS = ("fine_skewed", "stmoe_capacity", "decode_e256", "tiny_fp32",
                 "mixtral_8x+shared")
# latency-bound shapes: timed as replays of one CUDA graph of the whole layer
GRAPH_CONFIGS = ("tiny_fp32", "decode_e256")
L2_BYTES = 126 * 1024 * 1024


def config_workload(name: str) -> Workload:
    if name == "mixtral_8x+shared":
        return WORKLOADS["mixtral_8x"].with_(name=name, F_shared=WORKLOADS["mixtral_8x"].F)
    return WORKLOADS[name]


def forward_roofline(wl: Workload, alg: dict, stage_ms: dict, ms_total: float):
    """Roofline of the dominant kernel, the gate/up GEMM, against the roof its
    arithmetic intensity selects (the ridge of the two measured peaks)."""
    peaks, peak_src = load_peaks()
    gu_ms = stage_ms["expert_gate_up"]
    if wl.dtype == "bf16":
        key = "bf16_tflops_sustained" if ms_total > 1000.0 else "bf16_tflops"
        peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        intensity = alg["gateup_flop"] / alg["gateup_bytes"]
        ridge = peak * 1e12 / (hbm_peak * 1e9)
        if intensity >= ridge:
            achieved = alg["gateup_flop"] / (gu_ms / 1e3) / 1e12
            roofline = {"kernel": "expert_gate_up (grouped GEMM + SwiGLU)", "bound": "tensor",
                        "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                        "frac": round(achieved / peak, 4),
                        "peak_source": f"{key} of {peak_src}"}
        else:
            achieved = alg["gateup_bytes"] / (gu_ms / 1e3) / 1e9
            roofline = {"kernel": "expert_gate_up (grouped GEMM + SwiGLU)", "bound": "hbm",
                        "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                        "frac": round(achieved / hbm_peak, 4),
                        "peak_source": f"hbm_gbs of {peak_src}"}
        roofline.update(intensity_flop_per_byte=round(intensity, 1), ridge=round(ridge, 1),
                        traffic=recorded_traffic(wl.name, "expert_gate_up"))
        return roofline
    # fp32 layer: SIMT FMA pipes; peak from unit counts and the clock:
    # 148 SMs x 128 fp32 lanes x 2 FLOP x max SM clock
    sm_mhz = float(peaks.get("sm_max_mhz", 1965.0))
    peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12
    achieved = alg["gateup_flop"] / (gu_ms / 1e3) / 1e12
    return {"kernel": "expert_gate_up (fp32 SIMT)", "bound": "alu",
            "achieved": round(achieved, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_source": "148 SMs x 128 FMA x 2 x max clock",
            "traffic": recorded_traffic(wl.name, "expert_gate_up")}


def stage_table(wl: Workload, alg: dict, stage_ms: dict) -> dict:
    peaks, _ = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    stages = {}
    for name, ms in stage_ms.items():
        ent = {"ms": round(ms, 4)}
        if name == "gather":
            gbs = alg["dispatch_bytes"] / (ms / 1e3) / 1e9
            ent.update(GBs=round(gbs, 1), hbm_frac=round(gbs / hbm, 4))
        elif name == "combine":
            gbs = alg["combine_bytes"] / (ms / 1e3) / 1e9
            ent.update(GBs=round(gbs, 1), hbm_frac=round(gbs / hbm, 4))
        elif name == "route":
            gbs = alg["route_bytes"] / (ms / 1e3) / 1e9
            ent.update(GBs=round(gbs, 1), hbm_frac=round(gbs / hbm, 4))
        elif name == "expert_gate_up":
            ent.update(TFLOPs=round(alg["gateup_flop"] / (ms / 1e3) / 1e12, 1))
        elif name == "expert_down":
            ent.update(TFLOPs=round(alg["down_flop"] / (ms / 1e3) / 1e12, 1))
        elif name == "shared_expert" and alg["shared_flop"]:
            ent.update(TFLOPs=round(alg["shared_flop"] / (ms / 1e3) / 1e12, 1))
        stages[name] = ent
    return stages


class _Flusher:
    """Writes a buffer larger than L2 between timed steps (for layers whose
    inputs fit in L2)."""

    def __init__(self, dev):
        self.buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.fill_(1)


def measure_forward(M, wl: Workload, args, rank: int, world: int, dev, *, headline: bool,
                    graph: bool, cpu_seconds: float) -> dict:
    """Time one layer shape.  Returns the fields of its JSON record (rank 0's
    view; device times are the max over ranks)."""
    inp = make_inputs(wl, device=dev)
    layer = M.MoELayer(wl.T, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], wl.K,
                       wl.capacity_factor, router_bias=inp["bias"], shared=inp["shared"])
    noise = inp["noise"]
    nbuf = 3  # a few batches of tokens, rotated between steps
    xs = [make_tokens(wl, device=dev, seed=rank_token_seed(rank) * 16 + i) for i in range(nbuf)]
    y = torch.empty_like(xs[0])
    stream = torch.cuda.current_stream(dev)
    weight_bytes = 3 * wl.E * wl.D * wl.F * wl.elem_bytes + 3 * wl.D * wl.F_shared * wl.elem_bytes
    # inputs smaller than L2: flush it before every step and time the steps one by one
    flush = None if weight_bytes > L2_BYTES else _Flusher(dev)
    nb = M._binding.lib().moe_trace_boundary_count()

    for i in range(args.warmup):
        layer.forward(xs[i % nbuf], y, logit_noise=noise)
    torch.cuda.synchronize(dev)
    # steps: at least args.steps, and enough for >= 100 ms of timed work
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    layer.forward(xs[0], y, logit_noise=noise)
    w1.record(stream)
    torch.cuda.synchronize(dev)
    est = max(w0.elapsed_time(w1), 1e-3)
    steps = args.steps if headline else max(args.steps, min(2000, int(100.0 / est) + 1))
    steps = int(max_over_ranks(float(steps), world, dev))

    def timed(run_step, per_step_events=None):
        """Device time of `steps` steps (ms, this rank), with the clock record."""
        if per_step_events is not None:
            materialize_events(per_step_events, stream)
        clocks = ClockSampler(dev.index if dev.index is not None else 0)
        clocks.start()
        time.sleep(0.3)
        barrier(world)
        torch.cuda.synchronize(dev)
        if flush is None:
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for i in range(steps):
                if per_step_events is not None:
                    M.moe_trace_attach(per_step_events[i])
                run_step(i)
            t1.record(stream)
            torch.cuda.synchronize(dev)
            total = t0.elapsed_time(t1)
        else:
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(steps)]
            for i in range(steps):
                flush()
                if per_step_events is not None:
                    M.moe_trace_attach(per_step_events[i])
                pairs[i][0].record(stream)
                run_step(i)
                pairs[i][1].record(stream)
            torch.cuda.synchronize(dev)
            total = sum(a.elapsed_time(b) for a, b in pairs)
        barrier(world)
        M.moe_trace_attach([])
        return total, clocks.stop()

    # eager: stream launches, with an event at every stage boundary inside the
    # timed region (the per-kernel times on the launching stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nb)] for _ in range(steps)]
    eager_total, eager_clk = timed(lambda i: layer.forward(xs[i % nbuf], y, logit_noise=noise),
                                   evs)
    names = M.trace_stage_names()
    stage_ms = {}
    for j in range(1, nb):
        d = [evs[i][j - 1].elapsed_time(evs[i][j]) for i in range(steps)]
        stage_ms[names[j]] = sum(d) / len(d)
    launch = "stream"
    total, clk = eager_total, eager_clk
    eager_ms_step = max_over_ranks(eager_total, world, dev) / steps
    # for reference: the same steps without the stage events (each event record
    # is a command of its own on the stream)
    plain_total, _ = timed(lambda i: layer.forward(xs[i % nbuf], y, logit_noise=noise))
    untraced_ms_step = max_over_ranks(plain_total, world, dev) / steps
    if graph:
        # one CUDA graph of the whole forward per input buffer, replayed
        graphs = [layer.capture(xs[i], y, logit_noise=noise) for i in range(nbuf)]
        for i in range(args.warmup):
            graphs[i % nbuf].replay()
        torch.cuda.synchronize(dev)
        total, clk = timed(lambda i: graphs[i % nbuf].replay())
        launch = "cuda_graph"
        del graphs
    ms_total, ms_step, value = aggregate(total, world, wl.T, steps, dev)

    counts = layer.counts.cpu().tolist()
    kept_rows = int(min(sum(min(c, M.capacity(layer.cfg)) for c in counts), M.max_rows(layer.cfg)))
    alg = algorithmic(wl, counts, kept_rows)
    rec = {"value": round(value, 1), "unit": UNIT, "ms_per_step": round(ms_step, 4),
           "steps": steps, "launch": launch, "untraced_ms_per_step": round(untraced_ms_step, 4)}
    if graph:
        rec["stream_ms_per_step"] = round(eager_ms_step, 4)

    if headline:
        # end to end from pinned host memory: every step copies its batch in and
        # its result out; copies of neighbouring steps overlap the forward
        # (MoELayer.forward_host_stream)
        x_hosts = [xs[i % nbuf].cpu().pin_memory() for i in range(nbuf)]
        y_hosts = [torch.empty_like(x_hosts[0]).pin_memory() for _ in range(nbuf)]
        seq_in = [x_hosts[i % nbuf] for i in range(steps)]
        seq_out = [y_hosts[i % nbuf] for i in range(steps)]
        layer.forward_host_stream(seq_in[:max(2, args.warmup)], seq_out[:max(2, args.warmup)],
                                  logit_noise=noise)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        layer.forward_host_stream(seq_in, seq_out, logit_noise=noise, events=(e0, e1))
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
        io_bytes = wl.T * wl.D * wl.elem_bytes
        rec["e2e"] = {"value": round(world * wl.T / (e2e_ms / 1e3), 1), "unit": UNIT,
                      "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": io_bytes,
                      "d2h_bytes_per_step": io_bytes,
                      "how": "MoELayer.forward_host_stream: per step, x in from pinned host "
                             "memory, moe_forward, y out; copies overlap neighbouring steps' "
                             "forwards"}

    flags = M.moe_get_device_status(layer.workspace)
    if flags:
        raise RuntimeError(f"device status flags {flags:#x} after the benchmark ({wl.name})")

    ffn_ms = stage_ms["expert_gate_up"] + stage_ms["expert_down"]
    rec.update({
        "config": {"workload": wl.name, "T": wl.T, "D": wl.D, "F": wl.F, "E": wl.E, "K": wl.K,
                   "capacity_factor": wl.capacity_factor, "router_bias": wl.bias,
                   "logit_noise": wl.noise, "F_shared": wl.F_shared,
                   "parallelism": f"replicas x{world}", "launch": launch,
                   "l2": ("inputs larger than L2 (expert weights "
                          f"{weight_bytes / 1e9:.2f} GB read per step)") if flush is None else
                         ("inputs fit in L2: a 252 MB buffer is written before every step and "
                          "the steps are timed one by one")},
        "dtype": wl.dtype,
        "gpu_launches": M.forward_kernel_count(layer.cfg, layer.router_terms is not None) * steps,
        "roofline": forward_roofline(wl, alg, stage_ms, ms_total),
        "stages": stage_table(wl, alg, stage_ms),
        "layer": {"assignments_per_s": round(world * wl.T * wl.K / (ms_step / 1e3), 1),
                  "kept_rows": kept_rows, "max_over_mean_load": round(
                      max(counts) / (sum(counts) / len(counts)), 3),
                  "expert_weights_GBs": round(alg["active_weight_bytes"] / (ffn_ms / 1e3) / 1e9, 1),
                  "expert_tflops": round((alg["gateup_flop"] + alg["down_flop"])
                                         / (ffn_ms / 1e3) / 1e12, 1)},
        "clocks": clk,
    })
    if wl.capacity_factor > 0:
        losses = layer.losses.cpu().tolist()
        rec["layer"].update(capacity=M.capacity(layer.cfg), z_loss=round(losses[0], 6),
                            balance_loss=round(losses[1], 6))
    del layer, inp, xs, y
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and cpu_seconds > 0:
        rec["cpu_baseline"] = cpu_baseline(wl, cpu_seconds)
    else:
        rec["cpu_baseline"] = None
    return rec


def run_gpu(args):
    import mixture_experts_layer_55_b200 as M

    rank, world, local_rank = rank_info()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    init_dist(world, "nccl")
    wl = workload_of(args)
    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    head = measure_forward(M, wl, args, rank, world, dev, headline=True, graph=args.graph,
                           cpu_seconds=cpu_s)
    extras = {}
    if args.configs == "all" and not args.override and args.workload == "mixtral_8x":
        for name in EXTRA_CONFIGS:
            cw = config_workload(name)
            extras[name] = measure_forward(M, cw, args, rank, world, dev, headline=False,
                                           graph=name in GRAPH_CONFIGS,
                                           cpu_seconds=0.0 if (args.no_cpu_baseline or
                                                               cw.F_shared) else 4.0)
    if rank != 0:
        _finish(world)
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02^2) random-init weights)",
        "config": head["config"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "untraced_ms_per_step": head["untraced_ms_per_step"],
        "roofline": head["roofline"],
        "stages": head["stages"],
        "layer": head["layer"],
        "clocks": head["clocks"],
        "cpu_baseline": head["cpu_baseline"],
    }
    if extras:
        line["configs"] = {k: {kk: vv for kk, vv in v.items()
                               if kk not in ("unit",)} for k, v in extras.items()}
    if args.warmup < 3:
        line["note"] = "fewer than 3 warm-up steps: not a valid measurement"
    print(json.dumps(line), flush=True)
    _finish(world)


def run_gpu_train(args):
    """A training step per iteration: moe_forward_train + moe_backward."""
    import mixture_experts_layer_55_b200 as M

    rank, world, local_rank = rank_info()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    init_dist(world, "nccl")
    wl = workload_of(args)
    inp = make_inputs(wl, device=dev)
    layer = M.MoELayer(wl.T, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], wl.K,
                       wl.capacity_factor, router_bias=inp["bias"])
    noise = inp["noise"]
    nbuf = 3
    xs = [make_tokens(wl, device=dev, seed=rank_token_seed(rank) * 16 + i) for i in range(nbuf)]
    dys = [make_output_grad(wl, device=dev, seed=rank_token_seed(rank) * 16 + 8 + i)
           for i in range(nbuf)]
    y = torch.empty_like(xs[0])
    stream = torch.cuda.current_stream(dev)
    grads = None

    def step(i):
        nonlocal grads
        layer.forward_train(xs[i % nbuf], y, logit_noise=noise)
        grads = layer.backward(dys[i % nbuf], C_BAL, C_Z, grads=grads)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    nf = M._binding.lib().moe_trace_boundary_count()
    nbk = M._binding.lib().moe_trace_backward_boundary_count()
    evf = [[torch.cuda.Event(enable_timing=True) for _ in range(nf)] for _ in range(args.steps)]
    evb = [[torch.cuda.Event(enable_timing=True) for _ in range(nbk)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    materialize_events(evf + evb, stream)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(args.steps):
        M.moe_trace_attach(evf[i])
        M._binding.moe_trace_attach_backward(evb[i])
        step(i)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    M.moe_trace_attach([])
    M._binding.moe_trace_attach_backward([])
    clk = clocks.stop()
    ms_total, ms_step, value = aggregate(start.elapsed_time(stop), world, wl.T, args.steps, dev)

    def stage_times(evs, names, prefix):
        out = {}
        for j in range(1, len(names)):
            d = [evs[i][j - 1].elapsed_time(evs[i][j]) for i in range(args.steps)]
            out[prefix + names[j]] = sum(d) / len(d)
        return out
    stage_ms = stage_times(evf, M.trace_stage_names(), "fwd.")
    stage_ms.update(stage_times(evb, M._binding.trace_backward_stage_names(), "bwd."))

    counts = layer.counts.cpu().tolist()
    kept_rows = int(min(sum(min(c, M.capacity(layer.cfg)) for c in counts), M.max_rows(layer.cfg)))
    R = kept_rows
    flop = {"fwd.expert_gate_up": 4.0 * R * wl.D * wl.F, "fwd.expert_down": 2.0 * R * wl.F * wl.D,
            "bwd.dgrad_h": 2.0 * R * wl.D * wl.F, "bwd.dgrad_x": 4.0 * R * wl.F * wl.D,
            "bwd.wgrad_down": 2.0 * R * wl.F * wl.D, "bwd.wgrad_gate_up": 4.0 * R * wl.D * wl.F}

    # ---------------- end to end: x and dY in from pinned memory, dx and losses out ----------
    x_h = [t.cpu().pin_memory() for t in xs]
    dy_h = [t.cpu().pin_memory() for t in dys]
    dx_h = torch.empty_like(x_h[0]).pin_memory()
    loss_h = torch.empty(3, dtype=torch.float32).pin_memory()
    xd, dyd = torch.empty_like(xs[0]), torch.empty_like(dys[0])

    def e2e_step(i):
        nonlocal grads
        xd.copy_(x_h[i % nbuf], non_blocking=True)
        dyd.copy_(dy_h[i % nbuf], non_blocking=True)
        layer.forward_train(xd, y, logit_noise=noise)
        grads = layer.backward(dyd, C_BAL, C_Z, grads=grads)
        dx_h.copy_(grads["dx"], non_blocking=True)
        loss_h.copy_(layer.losses, non_blocking=True)
    for i in range(max(2, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    io = wl.T * wl.D * wl.elem_bytes

    for ws in (layer.state, layer.bwd_workspace):
        flags = M.moe_get_device_status(ws)
        if flags:
            raise RuntimeError(f"device status flags {flags:#x} after the benchmark")
    if rank != 0:
        _finish(world)
        return

    peaks, peak_src = load_peaks()
    key = "bf16_tflops_sustained" if ms_total > 1000.0 else "bf16_tflops"
    peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # algorithmic bytes of the backward GEMMs (bf16 operands, fp32 weight gradients)
    s2, Ea = wl.elem_bytes, sum(1 for c in counts if c > 0)
    D, F, E = wl.D, wl.F, wl.E
    nbytes = {"bwd.dgrad_h": R * D * s2 + Ea * F * D * s2 + 2 * (R * 2 * F * s2),
              "bwd.dgrad_x": R * 2 * F * s2 + Ea * 2 * D * F * s2 + R * D * s2,
              "bwd.wgrad_down": R * F * s2 + R * D * s2 + E * F * D * 4,
              "bwd.wgrad_gate_up": R * D * s2 + R * 2 * F * s2 + E * 2 * D * F * 4}
    top = max(nbytes, key=lambda k: stage_ms[k])
    t_top = stage_ms[top] / 1e3
    intensity = flop[top] / nbytes[top]
    if wl.dtype == "f32":
        # fp32 layer: SIMT FMA pipes (148 SMs x 128 fp32 lanes x 2 FLOP x max SM clock)
        peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
        key = "fp32 FMA"
    ridge = peak * 1e12 / (hbm_peak * 1e9)
    if wl.dtype == "f32":
        achieved = flop[top] / t_top / 1e12
        roofline = {"kernel": top, "bound": "alu", "achieved": round(achieved, 3), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_source": "148 SMs x 128 FMA x 2 x max clock"}
    elif intensity >= ridge:
        achieved = flop[top] / t_top / 1e12
        roofline = {"kernel": top, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_source": f"{key} of {peak_src}"}
    else:
        achieved = nbytes[top] / t_top / 1e9
        roofline = {"kernel": top, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                    "peak_source": f"hbm_gbs of {peak_src}"}
    roofline.update(intensity_flop_per_byte=round(intensity, 1), ridge=round(ridge, 1),
                    traffic=recorded_traffic(wl.name, top, WGRAD_SOURCES)
                    if top.startswith("bwd.wgrad") else None)
    stages = {}
    for name, ms in stage_ms.items():
        ent = {"ms": round(ms, 4)}
        if name in flop:
            ent["TFLOPs"] = round(flop[name] / (ms / 1e3) / 1e12, 1)
        if name in nbytes:
            ent["GBs"] = round(nbytes[name] / (ms / 1e3) / 1e9, 1)
        stages[name] = ent
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_train(wl, args.cpu_seconds)
    line = {
        "metric": METRIC_TRAIN, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) tokens and output gradients, N(0,0.02^2) weights)",
        "config": {"workload": wl.name, "pass": "train", "T": wl.T, "D": wl.D, "F": wl.F,
                   "E": wl.E, "K": wl.K, "capacity_factor": wl.capacity_factor,
                   "loss": f"sum(dY*y) + {C_BAL} balance + {C_Z} z",
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (expert weights and fp32 weight gradients)"},
        "e2e": {"value": round(world * wl.T / (e2e_ms / 1e3), 1), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": 2 * io,
                "d2h_bytes_per_step": io + 12,
                "how": "per step: x and dY in from pinned host memory, moe_forward_train, "
                       "moe_backward, dx and the losses out, one stream"},
        "gpu_launches": (M.forward_kernel_count(layer.cfg)
                         + M._binding.backward_kernel_count(layer.cfg)) * args.steps,
        "roofline": roofline,
        "stages": stages,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    if args.warmup < 3:
        line["note"] = "fewer than 3 warm-up steps: not a valid measurement"
    print(json.dumps(line), flush=True)
    _finish(world)


def run_gpu_ep(args):
    """Expert parallelism: rank r of N holds experts r*E/N .. (r+1)*E/N - 1 and
    its own T tokens; a step is one ExpertParallelMoE forward on every rank
    (route, owner-sorted dispatch, NCCL all-to-all, grouped local experts,
    reverse all-to-all, weighted combine; or, with --exchange peer, the
    dispatch kernel storing rows into the owners' peer-mapped buffers, the
    experts in place and the combine kernel loading from the owners)."""
    import mixture_experts_layer_55_b200 as M
    from mixture_experts_layer_55_b200.ep import ExpertParallelMoE

    rank, world, local_rank = rank_info()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    import torch.distributed as dist
    if not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29531")
        os.environ.setdefault("RANK", str(rank))
        os.environ.setdefault("WORLD_SIZE", str(world))
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    wl = workload_of(args)
    if wl.E % world:
        raise SystemExit(f"E = {wl.E} experts do not divide among {world} ranks")
    EL = wl.E // world
    inp = make_inputs(wl, device=dev)
    sl = slice(rank * EL, (rank + 1) * EL)
    layer = ExpertParallelMoE(wl.T, inp["w_router"], inp["w_gate"][sl].contiguous(),
                              inp["w_up"][sl].contiguous(), inp["w_down"][sl].contiguous(), wl.E,
                              wl.K, wl.capacity_factor, router_bias=inp["bias"],
                              exchange=args.exchange)
    del inp["w_gate"], inp["w_up"], inp["w_down"]
    nbuf = 3
    xs = [make_tokens(wl, device=dev, seed=rank_token_seed(rank) * 16 + i) for i in range(nbuf)]
    stream = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        layer.forward(xs[i % nbuf], logit_noise=inp["noise"])
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    names = layer.stage_names()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
           for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        layer.trace_events = evs[i]
        y = layer.forward(xs[i % nbuf], logit_noise=inp["noise"])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    layer.trace_events = None
    clk = clocks.stop()
    ms_total, ms_step, value = aggregate(start.elapsed_time(stop), world, wl.T, args.steps, dev)
    stage_ms = {}
    for j, name in enumerate(names):
        d = [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)]
        stage_ms[name] = sum(d) / len(d)
    # rows this rank's experts ran on (the same every step: the batches share a shape, not
    # their routing, so read the last step's)
    local_rows = int(layer.ops.offsets_local[EL].item())
    # end to end: x in from pinned memory, y out, every step
    x_h = [t.cpu().pin_memory() for t in xs]
    y_h = torch.empty_like(x_h[0]).pin_memory()
    xd = torch.empty_like(xs[0])
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        xd.copy_(x_h[i % nbuf], non_blocking=True)
        y = layer.forward(xd, logit_noise=inp["noise"])
        y_h.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    per_step = count_library_launches(lambda: layer.forward(xs[0], logit_noise=inp["noise"]), dev)
    flags = layer.ops.status()
    if flags:
        raise RuntimeError(f"device status flags {flags:#x} after the benchmark")
    if rank == 0:
        io = wl.T * wl.D * wl.elem_bytes
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(wl, args.cpu_seconds)
        # the local experts' two grouped GEMMs (the step's dominant work), rank 0's last step
        peaks, peak_src = load_peaks()
        key = "bf16_tflops_sustained" if ms_total > 1000.0 else "bf16_tflops"
        peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
        bound, src = "tensor", f"{key} of {peak_src}"
        if wl.dtype == "f32":  # SIMT FMA pipes
            peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
            bound, src = "alu", "148 SMs x 128 FMA x 2 x max clock"
        achieved = 6.0 * local_rows * wl.D * wl.F / (stage_ms["experts"] / 1e3) / 1e12
        roof = {"kernel": "experts (grouped gate/up + SwiGLU and down GEMMs of this rank's experts)",
                "bound": bound, "achieved": round(achieved, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_source": src,
                "rows": local_rows, "traffic": None}
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": "synthetic (seeded N(0,1) tokens, N(0,0.02^2) random-init weights)",
            "config": {"workload": wl.name, "T": wl.T, "D": wl.D, "F": wl.F, "E": wl.E, "K": wl.K,
                       "capacity_factor": wl.capacity_factor,
                       "parallelism": f"expert parallel x{world} ({EL} experts per rank, "
                                      + ("NCCL all-to-all)" if args.exchange == "all_to_all" else
                                         "peer-memory dispatch and combine kernels)"),
                       "l2": "inputs larger than L2"},
            "e2e": {"value": round(world * wl.T / (e2e_ms / 1e3), 1), "unit": UNIT,
                    "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": io, "d2h_bytes_per_step": io,
                    "how": "per step: x in from pinned host memory, ExpertParallelMoE.forward, y out"},
            "gpu_launches": None if per_step is None else per_step * args.steps,
            "roofline": roof,
            "stages": {k: {"ms": round(v, 4)} for k, v in stage_ms.items()},
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        if args.warmup < 3:
            line["note"] = "fewer than 3 warm-up steps: not a valid measurement"
        print(json.dumps(line), flush=True)
    layer.close()
    dist.destroy_process_group()


def count_library_launches(step, dev):
    """Kernels of this library (namespace moe::) that one call of `step`
    launches, counted by the CUDA profiler on an extra, untimed call; None if
    the profiler is unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step()
            torch.cuda.synchronize(dev)
        return sum(1 for ev in prof.events()
                   if ev.device_type == torch.autograd.DeviceType.CUDA and "moe::" in ev.name)
    except Exception:  # pragma: no cover - profiler missing on this machine
        return None


def _finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------ CPU oracle --

def _run_experts(jobs, work, cores: int):
    """Run work(e) for every (e, n_rows) in jobs on all `cores` host threads and
    time it: an expert with at least `cores` rows runs alone, its rows spread
    over the threads by the oracle's own OpenMP loop; experts with fewer rows
    run `cores` at a time, concurrently, one OpenMP thread each (the oracle's
    results do not depend on its thread count).  Returns ({e: result}, s)."""
    import concurrent.futures as cf

    import oracle
    out, secs = {}, 0.0
    big = [e for e, n in jobs if n >= cores or cores == 1]
    small = [e for e, n in jobs if not (n >= cores or cores == 1)]
    for e in big:
        t0 = time.perf_counter()
        out[e] = work(e)
        secs += time.perf_counter() - t0
    if small:
        with cf.ThreadPoolExecutor(cores, initializer=oracle.set_num_threads,
                                   initargs=(1,)) as ex:
            t0 = time.perf_counter()
            for e, r in zip(small, ex.map(work, small)):
                out[e] = r
            secs += time.perf_counter() - t0
    return out, secs


def _sample_tokens(wl: Workload, ids, kept, order, rows_target: float):
    """Tokens of the CPU sample, in random order until about rows_target kept
    rows, limited to the experts whose weights fit a 1.5 G-element host budget
    (generating expert weights on the host is not timed, but it takes wall
    time).  Returns the sorted tokens and the experts they need."""
    e_cap = max(1, int(1.5e9 // (3 * wl.D * wl.F)))
    toks, experts, rows = [], set(), 0
    for t in order:
        te = {int(ids[t, k]) for k in range(wl.K) if kept[t, k]}
        if toks and len(experts | te) > e_cap:
            continue
        toks.append(int(t))
        experts |= te
        rows += len(te)
        if rows >= rows_target:
            break
    return sorted(toks), sorted(experts)


def cpu_baseline(wl: Workload, seconds: float = 15.0, seed: int = 0, cpu_inp=None) -> dict:
    """Time the oracle as it stands on a bounded sample of the workload.

    Router logits + routing + dispatch layout for all T tokens, then the expert
    FFN and combine for a sample of tokens sized to the time budget (a first
    call calibrates the per-row cost).  Every expert's sampled rows go to the
    oracle in one call, using all host cores (_run_experts); the expert weights
    are generated before the timed calls.  value = tokens/s extrapolated from
    the per-token costs.
    """
    import numpy as np

    import oracle
    cpu_inp = cpu_inp or _cpu_inputs_for_sample(wl)
    x = cpu_inp["x"]
    t0 = time.perf_counter()
    L = oracle.router_logits(x, cpu_inp["w_router"], cpu_inp["bias"], cpu_inp["noise"])
    ids, w, probs, lse = oracle.route(L, wl.K)
    oracle.router_stats(ids, probs, lse, wl.E)
    C = oracle.capacity(wl.T, wl.K, wl.E, wl.capacity_factor)
    d = oracle.dispatch(ids, wl.E, C)
    t_route = time.perf_counter() - t0
    kept = d["row_of"].reshape(wl.T, wl.K) >= 0
    get = cpu_inp["get_expert"]
    cores = oracle.num_threads()
    rng = np.random.default_rng(seed)
    order = rng.permutation(wl.T)
    # calibration: `cores` rows of one expert on all threads
    e0 = int(ids[order[0], 0])
    w0 = get(e0)
    xcal = x[torch.from_numpy(order[:min(cores, wl.T)].copy())]
    t1 = time.perf_counter()
    oracle.expert_rows(xcal.double().numpy(), *w0)
    sec_row = (time.perf_counter() - t1) / xcal.shape[0]
    budget = max(1.0, seconds - t_route)
    toks, experts = _sample_tokens(wl, ids, kept, order, 0.8 * budget / max(sec_row, 1e-9))
    xs = x[torch.tensor(toks)].double().numpy()
    weights = {e: get(e) for e in experts}  # generated before the timed calls
    jobs = []
    rows_of = {}
    for e in experts:
        sel = [(i, k) for i, t in enumerate(toks) for k in range(wl.K)
               if kept[t, k] and int(ids[t, k]) == e]
        rows_of[e] = sel
        jobs.append((e, len(sel)))
    res, t_ffn = _run_experts(
        jobs, lambda e: oracle.expert_rows(xs[[i for i, _ in rows_of[e]]], *weights[e]), cores)
    n_rows = sum(n for _, n in jobs)
    outs = np.zeros((len(toks), wl.K, wl.D))
    for e, sel in rows_of.items():
        for j, (i, k) in enumerate(sel):
            outs[i, k] = res[e][j]
    t1 = time.perf_counter()
    oracle.token_outputs(xs, ids[toks], w[toks], kept[toks], None, outs=outs)
    t_ffn += time.perf_counter() - t1
    n = len(toks)
    per_token = t_route / wl.T + t_ffn / n
    # the same on one thread: routing on the first tokens, the expert FFN on a
    # part of the same sample
    oracle.set_num_threads(1)
    try:
        n1 = min(wl.T, 1024)
        t0 = time.perf_counter()
        L1 = oracle.router_logits(x[:n1], cpu_inp["w_router"], cpu_inp["bias"],
                                  None if cpu_inp["noise"] is None else cpu_inp["noise"][:n1])
        ids1, _, probs1, lse1 = oracle.route(L1, wl.K)
        oracle.router_stats(ids1, probs1, lse1, wl.E)
        oracle.dispatch(ids1, wl.E, oracle.capacity(n1, wl.K, wl.E, wl.capacity_factor))
        t_route1 = time.perf_counter() - t0
        budget1 = max(0.5, seconds / 5)
        rows1, t_ffn1 = 0, 0.0
        for e in experts:
            for (i, _) in rows_of[e]:
                if t_ffn1 >= budget1:
                    break
                t1 = time.perf_counter()
                oracle.expert_rows(xs[[i]], *weights[e])
                t_ffn1 += time.perf_counter() - t1
                rows1 += 1
    finally:
        oracle.set_num_threads(cores)
    per_token1 = t_route1 / n1 + (t_ffn1 / max(rows1, 1)) * (n_rows / n)
    return {"value": round(1.0 / per_token, 3), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": (f"router + routing + dispatch layout on all {wl.T} tokens "
                       f"({t_route:.2f} s); expert FFN + combine on {n} sampled tokens = "
                       f"{n_rows} expert rows over {len(experts)} experts ({t_ffn:.2f} s on "
                       f"{cores} threads: each expert's rows in one oracle call, experts with "
                       f"fewer rows than threads run concurrently); value extrapolated per token"),
            "single_thread": {"value": round(1.0 / per_token1, 3), "unit": UNIT, "cores": 1,
                              "sample": (f"routing on {n1} tokens ({t_route1:.2f} s), "
                                         f"{rows1} expert rows ({t_ffn1:.2f} s); value "
                                         "extrapolated per token")}}


def cpu_baseline_train(wl: Workload, seconds: float = 15.0, seed: int = 0, cpu_inp=None) -> dict:
    """The oracle's training step on a bounded sample: forward routing and the
    router's backward for all T tokens, then the kept rows of sampled tokens
    through the expert backward and their share of the weight gradients (each
    expert's rows in one call, on all host cores; weights generated before
    the timed calls)."""
    import numpy as np

    import oracle
    cpu_inp = cpu_inp or _cpu_inputs_for_sample(wl)
    dy = make_output_grad(wl, device="cpu")
    t0 = time.perf_counter()
    L = oracle.router_logits(cpu_inp["x"], cpu_inp["w_router"], cpu_inp["bias"], cpu_inp["noise"])
    ids, w, probs, lse = oracle.route(L, wl.K)
    C = oracle.capacity(wl.T, wl.K, wl.E, wl.capacity_factor)
    d = oracle.dispatch(ids, wl.E, C)
    dL = oracle.router_backward(L, ids, np.zeros((wl.T, wl.K)), d["counts"], C_BAL, C_Z)
    oracle.router_linear_backward(cpu_inp["x"], cpu_inp["w_router"], dL)
    t_route = time.perf_counter() - t0
    kept = d["row_of"].reshape(wl.T, wl.K) >= 0
    get = cpu_inp["get_expert"]
    cores = oracle.num_threads()
    rng = np.random.default_rng(seed)
    order = rng.permutation(wl.T)
    budget = max(1.0, seconds - t_route)

    def rows(e, toks):
        sel = [(t, k) for t in toks for k in range(wl.K) if kept[t, k] and ids[t, k] == e]
        return (np.array([t for t, _ in sel], np.int32), np.array([w[t, k] for t, k in sel]))

    def work(e, toks, wts):
        tok, wt = rows(e, toks)
        wg, wu, wd = wts[e]
        _, _, h, dg, du = oracle.expert_backward_rows(tok, np.zeros(len(tok), np.int32), wt,
                                                      cpu_inp["x"], dy, wg, wu, wd,
                                                      intermediates=True)
        oracle.expert_wgrad(tok, wt, cpu_inp["x"], dy, h, dg, du)
        return len(tok)

    # calibration: the first token's kept rows on all threads
    cal = [int(order[0])]
    cal_e = sorted({int(ids[cal[0], k]) for k in range(wl.K) if kept[cal[0], k]})
    wts = {e: get(e) for e in cal_e}
    _, t_cal = _run_experts([(e, 1) for e in cal_e], lambda e: work(e, cal, wts), cores)
    sec_row = t_cal / max(1, len(cal_e))
    toks, experts = _sample_tokens(wl, ids, kept, order, 0.8 * budget * cores / max(sec_row, 1e-9))
    wts = {e: get(e) for e in experts}
    jobs = [(e, len(rows(e, toks)[0])) for e in experts]
    _, t_rows = _run_experts(jobs, lambda e: work(e, toks, wts), cores)
    n = len(toks)
    per_token = t_route / wl.T + t_rows / n
    return {"value": round(1.0 / per_token, 3), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": (f"routing, dispatch layout and the router's backward on all {wl.T} tokens "
                       f"({t_route:.2f} s); expert backward and weight-gradient rows of {n} "
                       f"sampled tokens = {sum(j for _, j in jobs)} rows over {len(experts)} "
                       f"experts ({t_rows:.2f} s on {cores} threads); value extrapolated per "
                       "token")}


def _cpu_inputs_for_sample(wl: Workload):
    """Host inputs for the CPU baseline: the activations, router and, for the
    experts, one expert at a time (generated on demand, seeded per expert)."""
    small = wl.E * wl.D * wl.F * wl.elem_bytes * 3 < (2 << 30)
    if small:
        inp = make_inputs(wl, device="cpu")
        get = (lambda e: (inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e]))
        return dict(inp, get_expert=get)
    # large layers: same shapes and distributions; experts drawn on demand
    x = make_tokens(wl, device="cpu", seed=7)
    g = torch.Generator().manual_seed(wl.seed)
    w_router = (torch.randn(wl.D, wl.E, generator=g) * wl.w_std).float()
    from workloads import zipf_bias
    bias = zipf_bias(wl.E) if wl.bias == "zipf" else None
    noise = None
    if wl.noise:
        noise = torch.randn(wl.T, wl.E, generator=torch.Generator().manual_seed(wl.seed + 1)) / wl.E
    cache = {}

    def get(e):
        if e not in cache:
            ge = torch.Generator().manual_seed(10_000 + e)
            mk = (lambda *s: (torch.randn(*s, generator=ge) * wl.w_std).to(wl.torch_dtype))
            cache[e] = (mk(wl.D, wl.F), mk(wl.D, wl.F), mk(wl.F, wl.D))
        return cache[e]
    return dict(x=x, w_router=w_router, bias=bias, noise=noise, get_expert=get)


def workload_of(args) -> Workload:
    """The named workload, with any --override KEY=VALUE applied (a smaller case
    of the same kernels, for profiler captures; renamed so it is never mistaken
    for the named workload)."""
    wl = WORKLOADS[args.workload]
    if args.override:
        kw = {}
        for item in args.override:
            k, v = item.split("=", 1)
            kw[k] = type(getattr(wl, k))(v)
        tag = ",".join(f"{k}={v}" for k, v in kw.items())
        wl = wl.with_(name=f"{wl.name}[{tag}]", **kw)
    return wl


def run_reference(args):
    """The oracle on the host cores, timed per step on a bounded sample.  Each
    step's value is extrapolated per token from its sample (routing on every
    token, the expert FFN on sampled tokens); ms_per_step = T / value is that
    extrapolation, not a timed step of the whole layer."""
    rank, world, _ = rank_info()
    if rank != 0:
        return
    wl = workload_of(args)
    per_step = max(2.0, args.cpu_seconds / 4)
    train = getattr(args, "pass_", "forward") == "train"
    base = cpu_baseline_train if train else cpu_baseline
    cpu_inp = _cpu_inputs_for_sample(wl)  # shared by every step (weights drawn once)
    if args.warmup > 0:
        base(wl, 2.0, cpu_inp=cpu_inp)
    vals = []
    t0 = time.perf_counter()
    for i in range(args.steps):
        vals.append(base(wl, per_step, seed=i, cpu_inp=cpu_inp))
        if time.perf_counter() - t0 > 240:
            break
    value = statistics.median(v["value"] for v in vals)
    ms_step = 1e3 * wl.T / value
    line = {
        "impl": "reference", "metric": METRIC_TRAIN if train else METRIC,
        "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": len(vals), "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3), "extrapolated": True,
        "extrapolation": ("ms_per_step = T / value: each step times the routing and dispatch "
                          "of all T tokens and the expert FFN of a bounded token sample (every "
                          "token only for small layers), and value is the per-token cost "
                          f"extrapolated (the steps together took {time.perf_counter() - t0:.1f} s)"),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "D": wl.D, "F": wl.F, "E": wl.E, "K": wl.K,
                   "capacity_factor": wl.capacity_factor, "parallelism": "host cores (oracle)"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": vals[0]["cores"],
                         "kind": "oracle", "sample": vals[0]["sample"]},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral_8x", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--override", action="append", default=[],
                    help="KEY=VALUE change of the workload shape (profiling cases only)")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "train"], default="forward",
                    help="forward (default) or a training step (forward + backward)")
    ap.add_argument("--parallel", choices=["replicas", "ep"], default="replicas",
                    help="replicas (default): every GPU holds all experts; ep: experts sharded")
    ap.add_argument("--graph", action="store_true",
                    help="forward: time replays of a CUDA graph of the whole layer")
    ap.add_argument("--configs", choices=["all", "none"], default="all",
                    help="forward at the default shape: also measure the other layer shapes "
                         "(one record each under the line's 'configs' key)")
    ap.add_argument("--exchange", choices=["all_to_all", "peer"], default="all_to_all",
                    help="with --parallel ep: NCCL all-to-all, or the library's kernels over "
                         "peer-mapped buffers")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    elif args.parallel == "ep":
        run_gpu_ep(args)
    elif args.pass_ == "train":
        run_gpu_train(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
