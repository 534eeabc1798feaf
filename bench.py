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
    return {"workload": wl.name, "batch": wl.batch, "pad_len": S, "valid_tokens": T, "seq_len": S,
            "hidden": wl.shape.hidden, "heads": wl.shape.n_heads, "ffn": wl.shape.ffn, "layers": wl.n_layers,
            "global_batch": wl.batch * world, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (43.5 GB of fp16 weights stream through every step)"}


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
    value = done / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, S, T, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": f"per step: the first {tokens} tokens of one sequence through all "
                                       f"{wl.n_layers} layers (fp64 C oracle; weight generation not timed)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm


def traffic_from_profile() -> int | None:
    """DRAM bytes per launch of the GEMM kernel from the committed ncu summary, if the kernel
    source has not changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "gemm_tc_traffic.json")
    src = os.path.join(ROOT, "padding_free_varlen_b200", "csrc", "gemm_tc.cu")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if d.get("source_sha256_16") != h:
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
    wl = synth.WORKLOADS[args.workload]
    if args.layers > 0:
        import dataclasses
        wl = dataclasses.replace(wl, n_layers=args.layers)
    lengths, S = wl.lengths(), wl.padded_len()
    B, H, L = wl.batch, wl.shape.hidden, wl.n_layers
    T = int(lengths.sum())
    tdt = {synth.F16: torch.float16, synth.BF16: torch.bfloat16, synth.F32: torch.float32}[wl.dtype]
    edt = {synth.F16: capi.ENERGON_F16, synth.BF16: capi.ENERGON_BF16, synth.F32: capi.ENERGON_F32}[wl.dtype]
    want_cpu = dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline

    # ---- inputs (pinned host copies serve the end-to-end leg)
    x_host = torch.empty((B, S, H), dtype=tdt, pin_memory=True)
    synth.fill_normal_ptr(x_host.data_ptr(), x_host.numel(), wl.seed, synth.TID_X, wl.dtype)
    len_host = torch.from_numpy(lengths).pin_memory()
    d_in = x_host.to(dev)
    d_len = len_host.to(dev)
    d_out = torch.empty_like(d_in)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    # ---- weights: generated on the host (seeded) one layer at a time and uploaded; rank 0
    # generates, the other ranks receive a broadcast (setup only, outside any timed region).
    # While a layer's host copy exists, the CPU baseline runs the oracle on its sample.
    t0 = time.perf_counter()
    shapes = wl.shape.weight_shapes()
    dev_layers = []
    cpu = None
    if want_cpu:
        import oracle
        oracle.build()
        x_np = x_host.numpy() if tdt != torch.bfloat16 else x_host.view(torch.int16).numpy().view(np.uint16)
        cpu_y, cpu_p, cpu_s = None, 0, 0.0
    for l in range(L):
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
        if want_cpu:
            if l == 0:   # size the sample to about 15 s of oracle work over all layers
                tokens = args.cpu_tokens
                if tokens <= 0:
                    t1 = time.perf_counter()
                    oracle.layer_padded(x_np[0:1, :1].astype(np.float64), np.array([1], np.int32), hw,
                                        wl.shape.n_heads)
                    per_tok = (time.perf_counter() - t1) * L
                    tokens = int(max(1, min(lengths[0], 15.0 / max(per_tok, 1e-3))))
                cpu_p = int(min(tokens, lengths[0]))
                cpu_y = x_np[0:1, :cpu_p].astype(np.float64)
            t1 = time.perf_counter()
            cpu_y = oracle.layer_padded(cpu_y, np.array([cpu_p], np.int32), hw, wl.shape.n_heads)
            cpu_s += time.perf_counter() - t1
        del hw
    if want_cpu:
        cpu = {"value": cpu_p / cpu_s, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": f"first {cpu_p} tokens of sequence 0 through all {L} layers, fp64 C oracle "
                         f"({cpu_s:.1f} s; weight generation not timed)"}
    tables = [capi.make_weights(d) for d in dev_layers]
    setup_s = time.perf_counter() - t0

    cfg = capi.make_config(H, wl.shape.n_heads, wl.shape.ffn, edt, wl.ln_eps)
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(remove_padding=1):
        capi.energon_stack_forward(cfg, tables, L, d_in, d_len, B, S, remove_padding, d_out, st, ws, ws_bytes,
                                   stream)

    def timed(fn, k):
        dist.barrier()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        return dist.max(a.elapsed_time(b), dev)

    # ---- main timed region (launch tracing on: one event pair per kernel)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dist.local)
    clocks.start()
    capi.energon_trace_start()
    ms = timed(step, args.steps)
    trace = capi.energon_trace_stop()
    clk = clocks.stop()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the timed steps")
    value = replica_value(dist.world, T, args.steps, ms)

    # ---- roofline of the dominant kernel (the tcgen05 GEMM, four shapes per layer)
    peaks = load_peaks()
    gemm_names = ("gemm_qkv", "gemm_out_proj", "gemm_ffn1", "gemm_ffn2", "gemm_ffn2_rebuild")
    g_launch = sum(trace.get(n, (0, 0.0))[0] for n in gemm_names)
    g_ms = sum(trace.get(n, (0, 0.0))[1] for n in gemm_names)
    per_kernel = {k: {"launches": v[0], "ms_per_step": v[1] / args.steps,
                      "share": v[1] / max(1e-9, sum(x[1] for x in trace.values()))} for k, v in trace.items()}
    roofline = gemm_roofline(H, T, 2 if tdt != torch.float32 else 4, g_launch, g_ms, peaks, traffic_from_profile())
    whole_step = step_roofline(H, L, lengths, 2 if tdt != torch.float32 else 4, ms / args.steps, peaks)
    # memory-bound companions measured in the same region: the packing fused into the first
    # LayerNorm (reads the padded rows once, writes the packed rows and their normalisation)
    # and the pad zeroing; standalone remove / rebuild are timed after the main region
    aux = {}
    e = 2 if tdt != torch.float32 else 4
    for name, nbytes, per in (("layernorm_remove", 3 * T * H * e, 1), ("zero_pads", (B * S - T) * H * e, 1)):
        if name in trace and trace[name][1] > 0:
            gbs = nbytes * trace[name][0] / (trace[name][1] / 1e3) / 1e9
            aux[name] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                         "ms_per_launch": trace[name][1] / trace[name][0]}

    # ---- end to end through the C ABI with host buffers: every step copies its padded input
    # (and lengths) from pinned host memory and its padded output back.  The copies run on
    # their own streams, double-buffered, so that step i+1's input and step i-1's output move
    # while step i computes; the timed region ends when the last output is in host memory.
    e2e = None
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
        ms_e2e = timed(lambda: e2e_run(args.steps), 1)
        e2e = {"value": replica_value(dist.world, T, args.steps, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": x_host.numel() * x_host.element_size() + len_host.numel() * 4,
               "d2h_bytes_per_step": hosts[0].numel() * hosts[0].element_size(),
               "ms_per_step": ms_e2e / args.steps, "copies": "overlapped with compute (double-buffered streams)"}
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())} after the end-to-end steps")
        step()                                      # the pipeline returned what one step returns
        torch.cuda.synchronize(dev)
        last = hosts[(args.steps - 1) & 1]
        if not torch.equal(last.view(torch.int16), d_out.cpu().view(torch.int16)):
            raise RuntimeError("end-to-end output differs from a plain step's output")

    # ---- the same kernels on the fully padded batch (the work elimination removes)
    padded = None
    if not args.no_padded:
        kp = max(1, min(args.steps, 3))
        step(0)
        ms_pad = timed(lambda: step(0), kp)
        padded = {"value": replica_value(dist.world, T, kp, ms_pad), "unit": UNIT, "ms_per_step": ms_pad / kp,
                  "rows_per_step": B * S, "speedup_of_packed": (ms_pad / kp) / (ms / args.steps)}
        # elimination around each MLP only (attention sub-layers on the padded rows)
        step(2)
        ms_mlp = timed(lambda: step(2), kp)
        padded["mlp_only"] = {"value": replica_value(dist.world, T, kp, ms_mlp), "unit": UNIT,
                              "ms_per_step": ms_mlp / kp, "speedup_over_padded": ms_pad / ms_mlp}

    # ---- the head-transposing forms on this workload's shapes (Q|K|V rows -> head-major
    # padded, and an attention output head-major padded -> packed rows)
    transpose = None
    if not args.no_transpose and H % wl.shape.n_heads == 0:
        nh = wl.shape.n_heads
        d = H // nh
        qkv_rows = torch.zeros((T, 3 * H), dtype=tdt, device=dev)
        heads = torch.empty((3, B, nh, S, d), dtype=tdt, device=dev)
        back = torch.empty((T, H), dtype=tdt, device=dev)
        cu_dev = torch.empty(B + 1, dtype=torch.int32, device=dev)
        capi.energon_rce_offsets(d_len, B, S, cu_dev, st, stream)
        kt = max(3, args.steps)

        def t_rebuild():
            capi.energon_rce_transpose_padding_rebuild(qkv_rows, cu_dev, B, S, 3, nh, d, e, heads, stream)

        def t_remove():
            capi.energon_rce_transpose_padding_remove(heads, cu_dev, B, S, 1, nh, d, e, back, stream)
        transpose = {}
        for name, fn, nbytes in (("transpose_padding_rebuild_qkv", t_rebuild, T * 3 * H * e + 3 * B * S * H * e),
                                 ("transpose_padding_remove_attn", t_remove, 2 * T * H * e)):
            fn()
            ms_t = timed(fn, kt) / kt
            gbs = nbytes / (ms_t / 1e3) / 1e9
            transpose[name] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                               "ms_per_launch": ms_t}
        del qkv_rows, heads, back
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())} after the transpose forms")

    # ---- the standalone packing operators on this workload (energon_rce_remove_padding /
    # energon_rce_rebuild_padding), CUDA events on the launching stream
    if not args.no_transpose:
        cu_sa = torch.empty(B + 1, dtype=torch.int32, device=dev)
        capi.energon_rce_offsets(d_len, B, S, cu_sa, st, stream)
        pk = torch.empty((B * S, H), dtype=tdt, device=dev)
        ks = max(3, args.steps)
        for name, fn, nbytes in (
                ("remove_padding", lambda: capi.energon_rce_remove_padding(d_in, cu_sa, B, S, H, e, pk, stream),
                 2 * T * H * e),
                ("rebuild_padding", lambda: capi.energon_rce_rebuild_padding(pk, cu_sa, B, S, H, e, d_out, stream),
                 T * H * e + B * S * H * e)):
            fn()
            ms_t = timed(fn, ks) / ks
            gbs = nbytes / (ms_t / 1e3) / 1e9
            aux[name] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                         "ms_per_launch": ms_t, "standalone": True}
        del pk

    # ---- dynamic batching of a request stream (the pages' comparison against FIFO packing,
    # every batch padded to its longest request) on this machine's measured costs
    batching = None
    if not args.no_batching and args.workload == "gpt3_stack_half_pad" and dist.world == 1:
        batching = run_batching(args, capi, synth, cfg, tables, L, H, tdt, dev, stream, timed, d_in, st)

    launches = sum(v[0] for v in trace.values())
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16" if tdt == torch.float16 else str(tdt).replace("torch.", ""),
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
            "config": config_of(wl, S, T, dist.world), "roofline": roofline, "step_roofline": whole_step,
            "roofline_memory_kernels": aux,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
            "padded_path": padded, "transpose_forms": transpose, "dynamic_batching": batching,
            "kernels": per_kernel, "setup_s": setup_s}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    del tables
    dist.done()


def run_batching(args, capi, synth, cfg, tables, L, H, tdt, dev, stream, timed, pool, st):
    """Serves 256 requests (lengths U[1, 256], all queued at once) in batches of at most 64:
    FIFO packing vs the dynamic-programming scheduler (energon_sched_plan), each batch padded
    to its longest request and run (a) on every padded row, as in the pages' comparison, and
    (b) with the padding eliminated.  The scheduler's cost table is this machine's: the
    padded stack timed at two shapes, fitted as c0 + c1 * batch * padded length.  Request
    activations are rows of the bench batch (the values do not change the work)."""
    import torch
    n_req, max_b, max_s = 256, 64, 256
    lengths = [int(v) for v in synth.uniform_int(n_req, 1, max_s, 20260006, synth.TID_LENGTHS)]
    arrivals = [0.0] * n_req
    ws_bytes = capi.energon_workspace_bytes(cfg, max_b, max_s)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    nb = pool.shape[0]

    def make_batch(members):
        s_pad = max(lengths[i] for i in members)
        x = torch.stack([pool[i % nb, :s_pad] for i in members]).contiguous()
        lens = torch.tensor([lengths[i] for i in members], dtype=torch.int32, device=dev)
        return x, lens, torch.empty_like(x), s_pad

    def run(batches, mode):
        def go():
            for x, lens, out, s_pad in batches:
                capi.energon_stack_forward(cfg, tables, L, x, lens, x.shape[0], s_pad, mode, out, st, ws, ws_bytes,
                                           stream)
        return timed(go, 1)

    # machine costs of the padded stack
    pts = []
    for b, s_len in ((max_b, max_s), (8, 32)):
        x = torch.stack([pool[i % nb, :s_len] for i in range(b)]).contiguous()
        lens = torch.full((b,), s_len, dtype=torch.int32, device=dev)
        out = torch.empty_like(x)
        f = lambda: capi.energon_stack_forward(cfg, tables, L, x, lens, b, s_len, 0, out, st, ws, ws_bytes, stream)
        f()
        pts.append((b * s_len, timed(f, 1) / 1e3))
    c1 = max((pts[0][1] - pts[1][1]) / (pts[0][0] - pts[1][0]), 1e-12)
    c0 = max(pts[0][1] - c1 * pts[0][0], 1e-6)
    table = [[c0 + c1 * b * s_len for s_len in range(1, max_s + 1)] for b in range(1, max_b + 1)]

    fifo_of = capi.energon_sched_fifo(arrivals, max_b)
    fifo_groups = [[i for i in range(n_req) if fifo_of[i] == g] for g in range(max(fifo_of) + 1)]
    plan_of, order = capi.energon_sched_plan(lengths, arrivals, 0.0, max_b, table, 1.0)
    dyn_groups = [[i for i in range(n_req) if plan_of[i] == g] for g in order]
    tokens = sum(lengths)
    res = {"requests": n_req, "max_batch": max_b, "valid_tokens": tokens,
           "lengths": "U[1, 256], seed 20260006, all queued at time 0",
           "cost_model": {"c0_s": c0, "c1_s_per_padded_token": c1, "fitted_on": "padded stack at 64 x 256 and 8 x 32"}}
    for name, groups in (("fifo", fifo_groups), ("dynamic", dyn_groups)):
        batches = [make_batch(g) for g in groups]
        padded_tokens = sum(b[0].shape[0] * b[3] for b in batches)
        for mode, tag in ((0, "padded"), (1, "packed")):
            ms = run(batches, mode)
            res[f"{name}_{tag}"] = {"tokens_per_s": tokens / (ms / 1e3), "ms": ms, "batches": len(batches),
                                    "padded_tokens": padded_tokens}
        del batches
    res["gain_dynamic_over_fifo_padded"] = res["dynamic_padded"]["tokens_per_s"] / res["fifo_padded"]["tokens_per_s"]
    res["gain_packed_fifo_over_fifo_padded"] = res["fifo_packed"]["tokens_per_s"] / res["fifo_padded"]["tokens_per_s"]
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
