#!/usr/bin/env python3
"""Valid tokens/s of the padding-free GPT-3 12-layer stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl energon|reference]

One step = one energon_stack_forward call over one batch: offsets, remove,
12 GPT-3 layers (hidden 12288, 96 heads, FFN 49152, fp16) on the valid tokens,
rebuild.  Default workload: batch 32, pad_len 256, every length 128 (the
EnergonAI README's "Scaling Ability" setting: sequence length half the padding
length).  The inputs exceed L2 (43.5 GB of weights stream through every step).

Multi-GPU (torchrun, one rank per GPU): every rank runs its own replica of the
workload (sequences are independent, the path has no exchange step), weak
scaling, no collective inside the timed region.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference there is) on a
bounded sample of the same workload on the host cores.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "valid tokens/sec, GPT-3 layer stack fp16 varlen on 1 B200; % of tensor/HBM roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["energon", "reference"], default="energon")
    ap.add_argument("--workload", default="gpt3_stack_half_pad")
    ap.add_argument("--cpu-tokens", type=int, default=0,
                    help="tokens of the oracle's CPU sample (0: sized to about 15 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-padded", action="store_true")
    ap.add_argument("--no-transpose", action="store_true")
    ap.add_argument("--no-batching", action="store_true")
    ap.add_argument("--no-companions", action="store_true",
                    help="skip the other workloads (one GPT-3 layer, the dynamic batch, remove/rebuild)")
    ap.add_argument("--layers", type=int, default=0, help="override the workload's layer count (profiling)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- distributed


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend: str):
        import torch.distributed as dist
        if self.world > 1:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float, device) -> float:
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def done(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def replica_value(world: int, tokens_per_step: int, steps: int, ms_max: float) -> float:
    """Whole-job valid tokens/s of `world` replicas, timed as the slowest rank's duration."""
    return world * tokens_per_step * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- workload


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "tflops": d["bf16_tflops"], "tflops_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "tflops": 1590.0, "tflops_sustained": 1400.0, "source": "fallback"}


def config_of(wl, S: int, T: int, world: int) -> dict:
    c = {"workload": wl.name, "batch": wl.batch, "pad_len": S, "valid_tokens": T, "seq_len": S,
         "global_batch": wl.batch * world, "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}
    if wl.shape is not None:
        c.update(hidden=wl.shape.hidden, heads=wl.shape.n_heads, ffn=wl.shape.ffn, layers=wl.n_layers,
                 l2=f"inputs larger than L2 ({12 * wl.shape.hidden ** 2 * 2 * wl.n_layers / 1e9:.1f} GB of "
                    f"16-bit weights stream through every step)")
    else:
        c.update(hidden=wl.hidden, layers=0,
                 l2="inputs larger than L2 (the padded tensor alone is "
                    f"{wl.batch * S * wl.hidden * 2 / 1e6:.0f} MB); per-operator times flush L2 between launches")
    return c


def cpu_cores() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, dist: Dist):
    """The oracle (fp64, C, OpenMP on the host cores) timed on a bounded sample per step.

    Step i runs the first `tokens` tokens of sequence i mod batch through every layer
    (causal attention makes a prefix exactly the work of those tokens inside the batch).
    Layers are visited in order for all steps at once so that each layer's weights are
    generated once; every step's time is the sum of its own per-layer oracle calls."""
    if dist.rank != 0:
        return
    from padding_free_varlen_b200 import synth
    import oracle
    oracle.build()
    wl = synth.WORKLOADS[args.workload]
    lengths, S = wl.lengths(), wl.padded_len()
    T = int(lengths.sum())
    x = wl.x_padded()
    if wl.n_layers == 0:
        # the packing workload: a step is offsets + remove + rebuild over the whole batch
        secs = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            cu, _ = oracle.offsets(lengths, S)
            packed = oracle.remove_padding(x, cu)
            oracle.rebuild_padding(packed, cu, wl.batch, S)
            secs.append(time.perf_counter() - t0)
        total = sum(secs[args.warmup:])
        value = T * args.steps / total
        sample = f"per step: offsets, remove and rebuild of the whole batch ({T} valid rows; C oracle)"
    else:
        value, total, sample = reference_layers(args, oracle, wl, lengths, x)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64" if wl.n_layers else "bf16 (byte copies)", "data": "synthetic",
            "config": config_of(wl, S, T, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def reference_layers(args, oracle, wl, lengths, x):
    """Step i: the first `tokens` tokens of sequence i mod batch through every layer."""
    tokens = args.cpu_tokens or 1
    n = args.warmup + args.steps
    seqs = [i % wl.batch for i in range(n)]
    ps = [int(min(tokens, lengths[b])) for b in seqs]
    ys = [x[b:b + 1, :p].astype(np.float64) for b, p in zip(seqs, ps)]
    secs = [0.0] * n
    for l in range(wl.n_layers):
        hw = wl.layer(l)
        for i in range(n):
            t0 = time.perf_counter()
            ys[i] = oracle.layer_padded(ys[i], np.array([ps[i]], np.int32), hw, wl.shape.n_heads)
            secs[i] += time.perf_counter() - t0
        del hw
    total = sum(secs[args.warmup:])
    done = sum(ps[args.warmup:])
    return done / total, total, (f"per step: the first {tokens} tokens of one sequence through all "
                                 f"{wl.n_layers} layers (fp64 C oracle; weight generation not timed)")


# ----------------------------------------------------------------------------- our arm


def gemm_device_code_hash() -> str:
    """sha256 (16 hex digits) of the GEMM's device code: gemm_tc.cu up to its host-side
    section, plus the shared device helpers.  Host-side changes leave it unchanged."""
    csrc = os.path.join(ROOT, "padding_free_varlen_b200", "csrc")
    src = open(os.path.join(csrc, "gemm_tc.cu")).read()
    cut = src.find("// ------------------------------------------------------------------ host side")
    h = hashlib.sha256((src[:cut] if cut >= 0 else src).encode())
    h.update(open(os.path.join(csrc, "common.cuh"), "rb").read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload: str) -> int | None:
    """DRAM bytes per launch of the GEMM kernel from the committed ncu summary, if it was taken
    on this workload's launch configuration and the GEMM's device code has not changed since."""
    path = os.path.join(ROOT, "profiles", "gemm_tc_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("device_code_sha256_16") != gemm_device_code_hash() or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch_scaled")


def gemm_roofline(H: int, T: int, elem_bytes: int, launches: int, ms_total: float, peaks: dict,
                  traffic) -> dict:
    """Roofline object of the four GEMMs of a layer (QKV 3H x H, out-proj H x H, FFN1 4H x H,
    FFN2 H x 4H) on T rows, averaged per launch.  A launch of T rows does 2 T flop per weight
    element (T flop per 16-bit weight byte): below the machine's ridge (measured peak flop /
    measured HBM bytes) it is bound by streaming the weights, and is reported in bytes per
    second against the HBM rate."""
    flops_per_launch = 24 * H * H * T / 4
    weight_bytes_per_launch = 12 * H * H * elem_bytes / 4
    ms_per_launch = ms_total / max(1, launches)
    ridge = peaks["tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops_per_launch / weight_bytes_per_launch < ridge:
        achieved = weight_bytes_per_launch * launches / (ms_total / 1e3) / 1e9 if ms_total > 0 else None
        return {"bound": "hbm", "kernel": "gemm_tc (tcgen05, 4 shapes per layer), weight streaming",
                "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"] if achieved else None,
                "frac_of_datasheet": achieved / DATASHEET_HBM_GBS if achieved else None,
                "peak_note": f"{peaks['source']} HBM copy rate", "traffic": None,
                "algorithmic_bytes_per_launch": weight_bytes_per_launch, "ms_per_launch": ms_per_launch}
    achieved = flops_per_launch * launches / (ms_total / 1e3) / 1e12 if ms_total > 0 else None
    return {"bound": "tensor", "kernel": "gemm_tc (tcgen05, 4 shapes per layer)",
            "achieved": achieved, "peak": peaks["tflops_sustained"], "unit": "TFLOP/s",
            "frac": achieved / peaks["tflops_sustained"] if achieved else None,
            "frac_of_burst": achieved / peaks["tflops"] if achieved else None,
            "frac_of_datasheet": achieved / DATASHEET_TFLOPS if achieved else None,
            "peak_note": f"{peaks['source']} bf16 sustained (fp16 assumed at the bf16 rate); burst {peaks['tflops']}",
            "traffic": traffic, "algorithmic_flops_per_launch": flops_per_launch, "ms_per_launch": ms_per_launch}


DATASHEET_TFLOPS = 2250.0    # dense fp16 / bf16, for context
DATASHEET_HBM_GBS = 8000.0


def step_roofline(H: int, n_layers: int, lengths, elem_bytes: int, ms_per_step: float, peaks: dict) -> dict:
    """The whole step against its roofline: t_roof = max(algorithmic flop / sustained tensor
    peak, weight bytes / HBM rate), flop = per layer 24 H^2 T for the four GEMMs plus 4 H per
    visible key-query pair for QK^T and PV (sum over sequences of L (L + 1) / 2 pairs)."""
    T = int(sum(int(v) for v in lengths))
    pairs = sum(int(v) * (int(v) + 1) // 2 for v in lengths)
    flop = n_layers * (24 * H * H * T + 4 * H * pairs)
    weight_bytes = n_layers * 12 * H * H * elem_bytes
    t_flop = flop / (peaks["tflops_sustained"] * 1e12) * 1e3
    t_bytes = weight_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    t_roof = max(t_flop, t_bytes)
    return {"algorithmic_flop": flop, "weight_bytes": weight_bytes, "t_roof_ms": t_roof,
            "bound": "tensor" if t_flop >= t_bytes else "hbm", "ms_per_step": ms_per_step,
            "frac": t_roof / ms_per_step if ms_per_step > 0 else None}


class Timer:
    """CUDA-event timing on the launching stream, between barriers and synchronizes, max over ranks."""

    def __init__(self, dist: Dist, dev, stream):
        self.dist, self.dev, self.stream = dist, dev, stream

    def region(self, fn, k: int) -> float:
        """Milliseconds of k back-to-back calls of fn (the slowest rank's)."""
        import torch
        self.dist.barrier()
        torch.cuda.synchronize(self.dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        for _ in range(k):
            fn()
        b.record(self.stream)
        torch.cuda.synchronize(self.dev)
        self.dist.barrier()
        return self.dist.max(a.elapsed_time(b), self.dev)

    def launches(self, fn, k: int, flush=None) -> list:
        """Per-launch milliseconds of k calls of fn, each timed alone after an L2 flush."""
        import torch
        out = []
        for _ in range(k):
            if flush is not None:
                flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            fn()
            b.record(self.stream)
            torch.cuda.synchronize(self.dev)
            out.append(a.elapsed_time(b))
        return out


L2_FLUSH_BYTES = 512 << 20   # four times the 126 MB L2


def spread(vals) -> dict:
    return {"median": statistics.median(vals), "min": min(vals), "max": max(vals), "n": len(vals)}


def hbm_entry(nbytes: int, ms_list, peaks: dict, **extra) -> dict:
    ms = statistics.median(ms_list)
    gbs = nbytes / (ms / 1e3) / 1e9
    d = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
         "peak_note": f"{peaks['source']} HBM copy rate", "algorithmic_bytes_per_launch": nbytes,
         "ms_per_launch": ms, "ms_spread": spread(ms_list)}
    d.update(extra)
    return d


class CpuSample:
    """The fp64 oracle on the host cores over a bounded sample: the first p tokens of
    sequence 0 through every layer (causal attention makes a prefix exactly the work of
    those tokens).  p is sized from two calls on layer 0 (1 and 4 tokens), fitted as
    a + b p seconds per layer: a is the per-call weight decode, b the per-token work."""

    def __init__(self, x_np, lengths, n_layers: int, n_heads: int, budget_s: float, tokens: int = 0):
        import oracle
        oracle.build()
        self.oracle, self.x, self.lengths, self.L, self.nh = oracle, x_np, lengths, n_layers, n_heads
        self.budget, self.tokens = budget_s, tokens
        self.p, self.y, self.secs, self.fit = 0, None, 0.0, None

    def layer(self, l: int, hw: dict):
        o = self.oracle
        if l == 0:
            if self.tokens <= 0:
                ts = []
                for p in (1, 4):
                    t1 = time.perf_counter()
                    o.layer_padded(self.x[0:1, :p].astype(np.float64), np.array([p], np.int32), hw, self.nh)
                    ts.append(time.perf_counter() - t1)
                b = max((ts[1] - ts[0]) / 3.0, 1e-6)
                a = max(ts[0] - b, 0.0)
                self.fit = {"decode_s_per_layer_call": a, "s_per_token_per_layer": b}
                p = int((self.budget / self.L - a) / b)
            else:
                p = self.tokens
            self.p = int(max(1, min(p, int(self.lengths[0]))))
            self.y = self.x[0:1, :self.p].astype(np.float64)
        t1 = time.perf_counter()
        self.y = o.layer_padded(self.y, np.array([self.p], np.int32), hw, self.nh)
        self.secs += time.perf_counter() - t1

    def result(self) -> dict:
        r = {"value": self.p / self.secs, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
             "sample": f"first {self.p} tokens of sequence 0 through all {self.L} layers, fp64 C oracle "
                       f"({self.secs:.1f} s; weight generation not timed)"}
        if self.fit:
            r["fit"] = dict(self.fit)
            r["marginal_tokens_per_s"] = 1.0 / (self.L * self.fit["s_per_token_per_layer"])
            r["fit"]["note"] = ("a + b p seconds per layer call from 1- and 4-token calls: a is the oracle's "
                                "per-call weight decode, 1 / (layers b) its throughput once weights are decoded")
        return r


def upload_layers(wl, dist: Dist, dev, tdt, cpu: CpuSample | None = None):
    """Weights generated on the host (seeded) one layer at a time and uploaded; rank 0
    generates, the others receive a broadcast (setup only).  The CPU sample runs on each
    layer while its host copy exists."""
    import torch
    shapes = wl.shape.weight_shapes()
    dev_layers = []
    for l in range(wl.n_layers):
        hw = wl.layer(l) if dist.rank == 0 else None
        d = {}
        for name, shp in shapes.items():
            t = torch.empty(shp, dtype=tdt, device=dev)
            if hw is not None:
                src = torch.from_numpy(hw[name])
                t.copy_(src.view(torch.bfloat16) if tdt == torch.bfloat16 else src)
            if dist.pg:
                import torch.distributed as tdist
                tdist.broadcast(t, src=0)
            d[name] = t
        dev_layers.append(d)
        if cpu is not None:
            cpu.layer(l, hw)
        del hw
    return dev_layers


def prepare_folds(capi, cfg, dev_layers, H: int, dev, stream) -> float:
    """The first LayerNorm's fold vectors of every layer, computed once (weight-load time);
    returns their total device time in ms (CUDA events on the stream)."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    folds = [torch.empty(6 * H, dtype=torch.float32, device=dev) for _ in dev_layers]
    torch.cuda.synchronize(dev)
    a.record(stream)
    for d, f in zip(dev_layers, folds):
        capi.energon_layer_fold_weights(cfg, capi.make_weights(d), f, stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    for d, f in zip(dev_layers, folds):
        d["ln1_fold"] = f
    return a.elapsed_time(b)


def host_input(wl, tdt):
    import torch
    lengths, S = wl.lengths(), wl.padded_len()
    x_host = torch.empty((wl.batch, S, wl.H), dtype=tdt, pin_memory=True)
    synth_mod().fill_normal_ptr(x_host.data_ptr(), x_host.numel(), wl.seed, synth_mod().TID_X, wl.dtype)
    return x_host, torch.from_numpy(lengths).pin_memory(), lengths, S


def synth_mod():
    from padding_free_varlen_b200 import synth
    return synth


def bench_stack(args, dist: Dist, wl, dev, stream, peaks: dict, want_cpu: bool, full: bool) -> dict:
    """One workload of the layer stack: the untraced headline, a traced pass for the
    per-kernel shares and the GEMM roofline, the end-to-end leg, the padded paths; with
    `full` also the head-transposing forms, the standalone packing operators and the
    dynamic-batching comparison."""
    import torch
    from padding_free_varlen_b200 import capi, synth
    tdt = {synth.F16: torch.float16, synth.BF16: torch.bfloat16, synth.F32: torch.float32}[wl.dtype]
    edt = {synth.F16: capi.ENERGON_F16, synth.BF16: capi.ENERGON_BF16, synth.F32: capi.ENERGON_F32}[wl.dtype]
    e = 2 if tdt != torch.float32 else 4
    x_host, len_host, lengths, S = host_input(wl, tdt)
    B, H, L = wl.batch, wl.shape.hidden, wl.n_layers
    T = int(lengths.sum())
    d_in, d_len = x_host.to(dev), len_host.to(dev)
    d_out = torch.empty_like(d_in)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tm = Timer(dist, dev, stream)

    t0 = time.perf_counter()
    cpu = None
    if want_cpu:
        x_np = x_host.numpy() if tdt != torch.bfloat16 else x_host.view(torch.int16).numpy().view(np.uint16)
        cpu = CpuSample(x_np, lengths, L, wl.shape.n_heads, budget_s=25.0, tokens=args.cpu_tokens)
    dev_layers = upload_layers(wl, dist, dev, tdt, cpu)
    cfg = capi.make_config(H, wl.shape.n_heads, wl.shape.ffn, edt, wl.ln_eps)
    fold_ms = prepare_folds(capi, cfg, dev_layers, H, dev, stream)
    tables = [capi.make_weights(d) for d in dev_layers]
    setup_s = time.perf_counter() - t0

    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step(remove_padding=1):
        capi.energon_stack_forward(cfg, tables, L, d_in, d_len, B, S, remove_padding, d_out, st, ws, ws_bytes,
                                   stream)

    def check_status(what):
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())} after {what}")

    # ---- headline: K untraced steps (inputs larger than L2: the weights stream every step)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dist.local)
    clocks.start()
    ms = tm.region(step, args.steps)
    clk = clocks.stop()
    check_status("the timed steps")
    res = {"value": replica_value(dist.world, T, args.steps, ms), "ms_per_step": ms / args.steps,
           "clocks": clk, "config": config_of(wl, S, T, dist.world), "setup_s": setup_s,
           "fold_vectors": {"prepared_at_weight_load": True, "ms_all_layers": fold_ms,
                            "note": "c = W_qkv ln1_g and d = b_qkv + W_qkv ln1_b per layer "
                                    "(energon_layer_fold_weights), computed once with the weights; "
                                    "without them every step would recompute them (ms_all_layers)"}}

    # ---- a separate traced pass: per-kernel device time (one CUDA-event pair per launch)
    capi.energon_trace_start()
    ms_traced = tm.region(step, args.steps)
    trace = capi.energon_trace_stop()
    check_status("the traced steps")
    gemm_names = ("gemm_qkv", "gemm_out_proj", "gemm_ffn1", "gemm_ffn2", "gemm_ffn2_rebuild")
    g_launch = sum(trace.get(n, (0, 0.0))[0] for n in gemm_names)
    g_ms = sum(trace.get(n, (0, 0.0))[1] for n in gemm_names)
    total_ms = max(1e-9, sum(x[1] for x in trace.values()))
    res["kernels"] = {k: {"launches": v[0], "ms_per_step": v[1] / args.steps, "share": v[1] / total_ms}
                      for k, v in trace.items()}
    res["traced_pass"] = {"ms_per_step": ms_traced / args.steps,
                          "note": "per-kernel shares and the roofline come from this pass; the headline is untraced"}
    res["gpu_launches"] = sum(v[0] for v in trace.values())    # the same K steps as the headline
    res["roofline"] = gemm_roofline(H, T, e, g_launch, g_ms, peaks, traffic_from_profile(wl.name))
    res["step_roofline"] = step_roofline(H, L, lengths, e, ms / args.steps, peaks)
    aux = {}
    lo = 2 if e == 2 else 0   # the low halves of Q and K (16-bit types)
    for name, nbytes in (("layernorm_remove", 3 * T * H * e), ("zero_pads", (B * S - T) * H * e),
                         ("ln_fold", 2 * T * H * e + 8 * T), ("layernorm", T * H * (4 + e)),
                         ("ln_fold_weights", 3 * H * H * e), ("attention", T * H * e * (3 + lo + 1))):
        if name in trace and trace[name][1] > 0:
            gbs = nbytes * trace[name][0] / (trace[name][1] / 1e3) / 1e9
            aux[name] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                         "ms_per_launch": trace[name][1] / trace[name][0]}
    res["roofline_memory_kernels"] = aux

    # ---- end to end through the C ABI with host buffers: every step copies its padded input
    # (and lengths) from pinned host memory and its padded output back.  The copies run on
    # their own streams, double-buffered, so that step i+1's input and step i-1's output move
    # while step i computes; the timed region ends when the last output is in host memory.
    if not args.no_e2e:
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ins = [d_in, torch.empty_like(d_in)]
        lens = [d_len, torch.empty_like(d_len)]
        outs = [d_out, torch.empty_like(d_out)]
        hosts = [torch.empty_like(x_host, pin_memory=True) for _ in range(2)]
        ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "done", "out")}

        def e2e_run(k):
            h2d.wait_stream(stream)                 # nothing starts before the timed region does
            with torch.cuda.stream(h2d):
                ins[0].copy_(x_host, non_blocking=True)
                lens[0].copy_(len_host, non_blocking=True)
                ev["in"][0].record(h2d)
            for i in range(k):
                b = i & 1
                if i + 1 < k:                       # next input, once step i-1 has read its buffer
                    with torch.cuda.stream(h2d):
                        h2d.wait_event(ev["done"][b ^ 1])
                        ins[b ^ 1].copy_(x_host, non_blocking=True)
                        lens[b ^ 1].copy_(len_host, non_blocking=True)
                        ev["in"][b ^ 1].record(h2d)
                stream.wait_event(ev["in"][b])
                stream.wait_event(ev["out"][b])     # output buffer read back (step i-2)
                capi.energon_stack_forward(cfg, tables, L, ins[b], lens[b], B, S, 1, outs[b], st, ws, ws_bytes,
                                           stream)
                ev["done"][b].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(ev["done"][b])
                    hosts[b].copy_(outs[b], non_blocking=True)
                    ev["out"][b].record(d2h)
            stream.wait_stream(d2h)                 # the timed region ends with the last read-back
        e2e_run(2)
        torch.cuda.synchronize(dev)
        ms_e2e = tm.region(lambda: e2e_run(args.steps), 1)
        res["e2e"] = {"value": replica_value(dist.world, T, args.steps, ms_e2e), "unit": UNIT,
                      "h2d_bytes_per_step": x_host.numel() * x_host.element_size() + len_host.numel() * 4,
                      "d2h_bytes_per_step": hosts[0].numel() * hosts[0].element_size(),
                      "ms_per_step": ms_e2e / args.steps, "copies": "overlapped with compute (double-buffered streams)"}
        check_status("the end-to-end steps")
        step()                                      # the pipeline returned what one step returns
        torch.cuda.synchronize(dev)
        last = hosts[(args.steps - 1) & 1]
        if not torch.equal(last.view(torch.int16), d_out.cpu().view(torch.int16)):
            raise RuntimeError("end-to-end output differs from a plain step's output")
        del ins, outs, hosts

    # ---- the same kernels on the fully padded batch (the work elimination removes), and
    # elimination around each MLP only (attention sub-layers on the padded rows)
    if not args.no_padded:
        kp = max(1, min(args.steps, 3))
        step(0)
        ms_pad = tm.region(lambda: step(0), kp)
        pad = {"value": replica_value(dist.world, T, kp, ms_pad), "unit": UNIT, "ms_per_step": ms_pad / kp,
               "rows_per_step": B * S, "speedup_of_packed": (ms_pad / kp) / (ms / args.steps)}
        step(2)
        ms_mlp = tm.region(lambda: step(2), kp)
        pad["mlp_only"] = {"value": replica_value(dist.world, T, kp, ms_mlp), "unit": UNIT,
                           "ms_per_step": ms_mlp / kp, "speedup_over_padded": ms_pad / ms_mlp}
        check_status("the padded steps")
        res["padded_path"] = pad

    if full and not args.no_transpose and H % wl.shape.n_heads == 0:
        res["transpose_forms"] = bench_transpose(capi, wl, T, S, tdt, e, dev, stream, d_len, st, tm, peaks)
        sa = {}
        cu_sa = torch.empty(B + 1, dtype=torch.int32, device=dev)
        capi.energon_rce_offsets(d_len, B, S, cu_sa, st, stream)
        pk = torch.empty((B * S, H), dtype=tdt, device=dev)
        flush = l2_flusher(dev)
        for name, fn, nbytes in (
                ("remove_padding", lambda: capi.energon_rce_remove_padding(d_in, cu_sa, B, S, H, e, pk, stream),
                 2 * T * H * e),
                ("rebuild_padding", lambda: capi.energon_rce_rebuild_padding(pk, cu_sa, B, S, H, e, d_out, stream),
                 T * H * e + B * S * H * e)):
            fn()
            sa[name] = hbm_entry(nbytes, tm.launches(fn, max(5, args.steps), flush), peaks, standalone=True)
        res["roofline_memory_kernels"].update(sa)
        del pk
        check_status("the standalone packing operators")

    if full and not args.no_batching and dist.world == 1:
        res["dynamic_batching"] = run_batching(capi, synth, cfg, tables, L, tdt, dev, stream, tm, d_in, st)

    if cpu is not None:
        res["cpu_baseline"] = cpu.result()
    del tables, dev_layers, ws
    torch.cuda.empty_cache()
    return res


def l2_flusher(dev):
    import torch
    buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    return lambda: buf.zero_()


def bench_transpose(capi, wl, T, S, tdt, e, dev, stream, d_len, st, tm: Timer, peaks):
    """The two head-transposing forms on this workload's shapes (Q|K|V rows -> head-major
    padded, an attention output head-major padded -> packed rows), each launch moving more
    than L2 holds."""
    import torch
    B, H, nh = wl.batch, wl.shape.hidden, wl.shape.n_heads
    d = H // nh
    qkv_rows = torch.zeros((T, 3 * H), dtype=tdt, device=dev)
    heads = torch.empty((3, B, nh, S, d), dtype=tdt, device=dev)
    back = torch.empty((T, H), dtype=tdt, device=dev)
    cu_dev = torch.empty(B + 1, dtype=torch.int32, device=dev)
    capi.energon_rce_offsets(d_len, B, S, cu_dev, st, stream)
    kt = 5
    out = {}
    for name, fn, nbytes in (
            ("transpose_padding_rebuild_qkv",
             lambda: capi.energon_rce_transpose_padding_rebuild(qkv_rows, cu_dev, B, S, 3, nh, d, e, heads, stream),
             T * 3 * H * e + 3 * B * S * H * e),
            ("transpose_padding_remove_attn",
             lambda: capi.energon_rce_transpose_padding_remove(heads, cu_dev, B, S, 1, nh, d, e, back, stream),
             2 * T * H * e)):
        fn()
        out[name] = hbm_entry(nbytes, tm.launches(fn, kt), peaks)
    del qkv_rows, heads, back
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the transpose forms")
    return out


def bench_packing(args, dist: Dist, wl, dev, stream, peaks: dict, steps: int, warmup: int) -> dict:
    """The packing operators alone at their own workload (bf16 [64, 512, 4096], lengths
    U[1, 512]): a step is offsets + transpose_padding_remove + transpose_padding_rebuild.
    The headline times `steps` whole steps (the padded tensor exceeds L2); each operator is
    then timed launch by launch with a 512 MB L2 flush before every launch.  The round trip
    is checked bit for bit on the device: valid rows unchanged, pad rows all-zero bytes."""
    import torch
    from padding_free_varlen_b200 import capi, synth
    tdt = {synth.F16: torch.float16, synth.BF16: torch.bfloat16, synth.F32: torch.float32}[wl.dtype]
    e = torch.tensor([], dtype=tdt).element_size()
    x_host, len_host, lengths, S = host_input(wl, tdt)
    B, H = wl.batch, wl.H
    T = int(lengths.sum())
    d_in, d_len = x_host.to(dev), len_host.to(dev)
    cu = torch.empty(B + 1, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    packed = torch.empty((B * S, H), dtype=tdt, device=dev)
    out = torch.empty_like(d_in)
    tm = Timer(dist, dev, stream)

    def offsets():
        capi.energon_rce_offsets(d_len, B, S, cu, st, stream)

    def remove():
        capi.energon_rce_remove_padding(d_in, cu, B, S, H, e, packed, stream)

    def rebuild():
        capi.energon_rce_rebuild_padding(packed, cu, B, S, H, e, out, stream)

    def step():
        offsets()
        remove()
        rebuild()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dist.local)
    clocks.start()
    ms = tm.region(step, steps)
    clk = clocks.stop()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the packing steps")
    mask = torch.arange(S, device=dev)[None, :] < d_len[:, None]
    same = torch.equal(out.view(torch.int16)[mask], d_in.view(torch.int16)[mask])
    zero = not out.view(torch.int16)[~mask].any().item()
    if not (same and zero):
        raise RuntimeError("remove -> rebuild round trip is not the identity on valid rows with zero pads")
    flush = l2_flusher(dev)
    k = max(10, steps)
    ops = {"remove_padding": hbm_entry(2 * T * H * e, tm.launches(remove, k, flush), peaks),
           "rebuild_padding": hbm_entry(T * H * e + B * S * H * e, tm.launches(rebuild, k, flush), peaks),
           "offsets": {"bound": "latency", "ms_spread": spread(tm.launches(offsets, k, flush)),
                       "algorithmic_bytes_per_launch": 8 * B + 4}}
    ops["offsets"]["ms_per_launch"] = ops["offsets"]["ms_spread"]["median"]
    step_bytes = 2 * T * H * e + T * H * e + B * S * H * e
    gbs = step_bytes / (ms / steps / 1e3) / 1e9
    return {"value": replica_value(dist.world, T, steps, ms), "ms_per_step": ms / steps, "clocks": clk,
            "config": config_of(wl, S, T, dist.world), "dtype": "bf16" if tdt == torch.bfloat16 else str(tdt),
            "roofline": dict(ops["rebuild_padding"], kernel="rebuild_kernel (the step's larger operator)"),
            "step_hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "algorithmic_bytes_per_step": step_bytes},
            "operators": ops, "round_trip_bit_exact": True, "gpu_launches": 3 * steps}


def run_energon(args, dist: Dist):
    import torch
    from padding_free_varlen_b200 import build as cuda_build
    from padding_free_varlen_b200 import capi, synth

    if dist.rank == 0 or not os.path.exists(capi.LIB_PATH):
        cuda_build.build()
    dist.init("nccl")
    dist.barrier()
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    wl = synth.WORKLOADS[args.workload]
    if args.layers > 0 and wl.n_layers > 0:
        import dataclasses
        wl = dataclasses.replace(wl, n_layers=args.layers)
    want_cpu = dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline
    base = {"metric": METRIC, "unit": UNIT, "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)"}

    if wl.n_layers == 0:
        r = bench_packing(args, dist, wl, dev, stream, peaks, args.steps, args.warmup)
        line = dict(base, **r)
        line["e2e"] = None
        line["cpu_baseline"] = None
        line["data"] = "synthetic (seeded N(0,1) rows; lengths U[1, 512])"
    else:
        r = bench_stack(args, dist, wl, dev, stream, peaks, want_cpu, full=True)
        line = dict(base, **r)
        line["dtype"] = {synth.F16: "f16", synth.BF16: "bf16", synth.F32: "f32"}[wl.dtype]
        line.setdefault("cpu_baseline", None)
        line.setdefault("e2e", None)
        # the other workloads, timed in the same run (each its own seeded weights)
        if not args.no_companions and args.workload == "gpt3_stack_half_pad" and args.layers == 0:
            comp = {}
            cargs = argparse.Namespace(**vars(args))
            cargs.no_e2e = True
            for name in ("gpt3_layer", "gpt3_stack_dynbatch"):
                cw = synth.WORKLOADS[name]
                c = bench_stack(cargs, dist, cw, dev, stream, peaks, False, full=False)
                comp[name] = {k: c[k] for k in ("value", "ms_per_step", "config", "roofline", "step_roofline",
                                                "padded_path", "kernels", "clocks", "setup_s", "fold_vectors")
                              if k in c}
                comp[name]["unit"] = UNIT
            comp["remove_rebuild"] = bench_packing(args, dist, synth.WORKLOADS["remove_rebuild"], dev, stream,
                                                   peaks, max(10, args.steps), args.warmup)
            line["companions"] = comp
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.done()


COST_SHAPES = ((8, 32), (16, 64), (32, 64), (32, 128), (64, 128), (64, 256))


def cost_table(points, max_b: int, max_s: int):
    """cost[b-1][s-1] of b sequences padded to s tokens: linear interpolation of the measured
    (padded tokens, seconds) points in b * s, constant below the first point, extended along
    the last segment above the last one."""
    pts = sorted(points)
    xs = np.array([p[0] for p in pts], np.float64)
    ys = np.array([p[1] for p in pts], np.float64)
    n = np.arange(1, max_b + 1)[:, None] * np.arange(1, max_s + 1)[None, :]
    t = np.interp(n, xs, ys)
    if len(xs) >= 2:
        slope = (ys[-1] - ys[-2]) / (xs[-1] - xs[-2])
        t = np.where(n > xs[-1], ys[-1] + slope * (n - xs[-1]), t)
    return t.tolist()


def extend_positions(pool, n: int):
    """[B, S, H] request rows with at least n positions: a workload padded to fewer positions
    repeats its own (the values do not change the work); the batches cut from it must have
    every position their pad length claims."""
    if pool.shape[1] >= n:
        return pool
    reps = (n + pool.shape[1] - 1) // pool.shape[1]
    return pool.repeat(1, reps, 1)[:, :n].contiguous()


def run_batching(capi, synth, cfg, tables, L, tdt, dev, stream, tm: Timer, pool, st):
    """Serves 256 requests (lengths U[1, 256], all queued at once) in batches of at most 64:
    FIFO packing vs the dynamic-programming scheduler (energon_sched_plan), each batch padded
    to its longest request and run (a) on every padded row, as in the pages' comparison, and
    (b) with the padding eliminated.  The scheduler's cost table is this machine's: the
    padded stack timed at six shapes (median of 3 after a warm-up run), interpolated in the
    padded token count (cost_table).  Every arm runs once to warm its batch shapes, then 3
    timed repeats (median, min, max).  Request activations are rows of the bench batch (the
    values do not change the work)."""
    import torch
    n_req, max_b, max_s = 256, 64, 256
    lengths = [int(v) for v in synth.uniform_int(n_req, 1, max_s, 20260006, synth.TID_LENGTHS)]
    arrivals = [0.0] * n_req
    ws_bytes = capi.energon_workspace_bytes(cfg, max_b, max_s)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    pool = extend_positions(pool, max_s)
    nb = pool.shape[0]
    reps = 3

    def make_batch(members):
        s_pad = max(lengths[i] for i in members)
        x = torch.stack([pool[i % nb, :s_pad] for i in members]).contiguous()
        assert x.shape[1] == s_pad
        lens = torch.tensor([lengths[i] for i in members], dtype=torch.int32, device=dev)
        return x, lens, torch.empty_like(x), s_pad

    def runner(batches, mode):
        def go():
            for x, lens, out, s_pad in batches:
                capi.energon_stack_forward(cfg, tables, L, x, lens, x.shape[0], s_pad, mode, out, st, ws, ws_bytes,
                                           stream)
        return go

    # machine costs of the padded stack, measured at six shapes; the cost of b sequences
    # padded to s tokens is interpolated in the padded token count b * s (small batches are
    # bound by streaming the weights, large ones by the GEMMs: not one straight line)
    pts = []
    for b, s_len in COST_SHAPES:
        x = torch.stack([pool[i % nb, :s_len] for i in range(b)]).contiguous()
        assert x.shape[1] == s_len
        lens = torch.full((b,), s_len, dtype=torch.int32, device=dev)
        out = torch.empty_like(x)
        f = lambda: capi.energon_stack_forward(cfg, tables, L, x, lens, b, s_len, 0, out, st, ws, ws_bytes, stream)
        f()
        pts.append((b * s_len, statistics.median(tm.region(f, 1) for _ in range(reps)) / 1e3))
    table = cost_table(pts, max_b, max_s)
    lin = np.polyfit([p[0] for p in pts], [p[1] for p in pts], 1)

    fifo_of = capi.energon_sched_fifo(arrivals, max_b)
    fifo_groups = [[i for i in range(n_req) if fifo_of[i] == g] for g in range(max(fifo_of) + 1)]
    plan_of, order = capi.energon_sched_plan(lengths, arrivals, 0.0, max_b, table, 1.0)
    dyn_groups = [[i for i in range(n_req) if plan_of[i] == g] for g in order]
    tokens = sum(lengths)
    res = {"requests": n_req, "max_batch": max_b, "valid_tokens": tokens,
           "lengths": "U[1, 256], seed 20260006, all queued at time 0",
           "cost_model": {"kind": "piecewise-linear in padded tokens between measured points",
                          "measured_on": "padded stack at " + ", ".join(f"{b}x{s}" for b, s in COST_SHAPES)
                                         + " (median of 3 each)",
                          "points": [{"padded_tokens": int(a), "s": float(b)} for a, b in pts],
                          "straight_line_fit": {"c0_s": float(lin[1]), "c1_s_per_padded_token": float(lin[0])}}}
    for name, groups in (("fifo", fifo_groups), ("dynamic", dyn_groups)):
        batches = [make_batch(g) for g in groups]
        padded_tokens = sum(b[0].shape[0] * b[3] for b in batches)
        for mode, tag in ((0, "padded"), (1, "packed")):
            go = runner(batches, mode)
            go()                                        # warm every batch shape of this arm
            ms = [tm.region(go, 1) for _ in range(reps)]
            tps = [tokens / (m / 1e3) for m in ms]
            res[f"{name}_{tag}"] = {"tokens_per_s": statistics.median(tps), "tokens_per_s_spread": spread(tps),
                                    "ms": statistics.median(ms), "batches": len(batches),
                                    "padded_tokens": padded_tokens}
        del batches

    def gain(a, b):
        sa, sb = res[a]["tokens_per_s_spread"], res[b]["tokens_per_s_spread"]
        return {"median": sa["median"] / sb["median"], "min": sa["min"] / sb["max"], "max": sa["max"] / sb["min"]}
    res["gain_dynamic_over_fifo_padded"] = gain("dynamic_padded", "fifo_padded")
    res["gain_packed_fifo_over_fifo_padded"] = gain("fifo_packed", "fifo_padded")
    res["gain_dynamic_packed_over_fifo_padded"] = gain("dynamic_packed", "fifo_padded")
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the batching runs")
    del ws
    return res


def main():
    args = parse()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    run_energon(args, dist)


if __name__ == "__main__":
    main()
