#!/usr/bin/env python3
"""Benchmark: MoE-layer tokens/s on B200 (route -> layout -> dispatch -> expert FFN -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral] [--impl ours|reference]
                    [--fp8] [--gather] [--fused] [--pipeline] [--graph]

One step = one full layer forward (every stage) over one batch of T tokens.
Default workload: the Mixtral-shaped layer (T=4096, d=4096, E=8, top-2,
f=14336, bf16 router linear, softmax top-2 renormalised), synthetic seeded
inputs.  Multi-GPU runs are replicas (one process per GPU, each with its own
token batch and a full copy of the weights, no data-path collective): weak
scaling, value = all ranks' tokens / the slowest rank's time.

``--pipeline`` runs the token-centric pipeline: after route and layout, one
persistent kernel takes dispatch chunks, GEMM-1 and GEMM-2 tiles from an
atomic ticket and (top-2 or top-1) combines in GEMM-2's epilogue.
``--fp8`` runs the layer's FP8 mode (E4M3 dispatch with a per-tensor scale
and FP8 GEMM-1; GEMM-2 and combine stay bf16); W1 is quantised once before
timing.  ``--gather`` fuses the dispatch into GEMM-1 (rows read through the
layout table with TMA gather4 loads; no dispatch kernel).  ``--fused`` runs
both expert GEMMs as one persistent kernel (GEMM-2 starts per token block as
soon as GEMM-1 has produced it).  ``--graph`` also times the same forward
captured once into a CUDA graph and replayed (launch overhead removed; the
decode configurations' second figure).  Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
(the only reference this method has) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from combine_moe_route_14_b200 import inputs as I  # noqa: E402
from combine_moe_route_14_b200 import replicas as Rp  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; HBM GB/s (dispatch/combine), TC util (GEMM)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# tokens per oracle step (the first S of the batch, all stages): the
# cpu_baseline leg and the reference arm time the same sample
ORACLE_SAMPLE = {"mixtral": 4096, "mixtral_threshold": 4096, "tiny_threshold": 256,
                 "skewed_top1": 4096, "skewed_top1_harsh": 4096, "fine_grained": 32, "tiny": 256,
                 "decode_16": 16, "decode_64": 64, "decode_256": 256, "decode_1024": 256}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------------------
# bookkeeping: algorithmic bytes / flops per stage
# ----------------------------------------------------------------------------
def stage_model(cfg, counts=None, fp8=False):  # gather form: same algorithmic bytes per stage
    """Algorithmic work of each stage for one forward (bytes moved that the math needs)."""
    T, d, E, k, f, R = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.R
    E_act = E if counts is None else int((np.asarray(counts) > 0).sum())
    m = {}
    if cfg.router == "weights":
        m["router_logits"] = {"bytes": T * d * 2 + E * d * 2 + T * E * 4, "flops": 2 * T * d * E}
    m["route"] = {"bytes": T * E * 4 + R * 8}
    m["layout"] = {"bytes": R * 4 + R * 8 + (2 * E + 1) * 4}
    m["route_layout"] = {"bytes": T * E * 4 + R * 8 + R * 8 + (2 * E + 1) * 4}
    m["dispatch"] = {"bytes": T * d * 2 + R * d * 2 + R * 4}
    m["gemm1"] = {"flops": 2 * R * d * f, "bytes": E_act * f * d * 2 + R * d * 2 + R * f * 2}
    m["gemm2"] = {"flops": 2 * R * d * f, "bytes": E_act * d * f * 2 + R * f * 2 + R * d * 2}
    m["combine"] = {"bytes": R * d * 2 + R * 8 + T * d * 2}
    if fp8:
        # absmax pass over X, then the gather writes one byte per value
        m["dispatch"] = {"bytes": 2 * T * d * 2 + R * d + R * 4}
        m["gemm1"] = {"flops": 2 * R * d * f, "bytes": E_act * f * d + R * d + R * f * 2}
        m["quantize"] = {"bytes": 2 * T * d * 2 + T * d}
    m["ffn"] = {"flops": m["gemm1"]["flops"] + m["gemm2"]["flops"],
                "bytes": m["gemm1"]["bytes"] + m["gemm2"]["bytes"]}
    # token-centric pipeline (dispatch chunks + both GEMMs + combine in one
    # launch, k <= 2): X read, dispatched rows written and read, weights, H
    # written and read, Y written; no Ye rows
    w = E_act * f * d * 2 * 2
    m["pipeline"] = {"flops": m["ffn"]["flops"],
                     "bytes": w + T * d * 2 + 2 * R * d * 2 + 2 * R * f * 2 + T * d * 2
                     if k <= 2 else w + T * d * 2 + 2 * R * d * 2 + 2 * R * f * 2
                     + m["combine"]["bytes"] + R * d * 2}
    return m


def stage_ms_hint(cfg) -> float:
    """Rough device time of one GEMM-1 launch in microseconds (sizes the queue-ahead)."""
    return max(20.0, 2 * cfg.R * cfg.d * cfg.f / 1.0e15 * 1e6)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return {k: float(j[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_sha256(text: str) -> str:
    """sha256 of C++/CUDA source with its comments and blank space removed:
    the same for two versions that differ only in comments or layout."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it still matches the code.

    profiles/<kernel>_<workload>.md carries 'traffic_bytes_per_launch:' and
    'code_sha256:' lines (the grouped GEMM source's code_sha256 when the
    counters were taken); any change to the kernel's code voids the figure.
    """
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    src = os.path.join(ROOT, "combine_moe_route_14_b200", "csrc", "grouped_gemm.cu")
    if not os.path.exists(path) or not os.path.exists(src):
        return None
    text = open(path).read()
    mt = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    ms = re.search(r"code_sha256:\s*([0-9a-f]{64})", text)
    if not mt or not ms:
        return None
    if code_sha256(open(src).read()) != ms.group(1):
        return None
    return float(mt.group(1))


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, cmax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            mx = cmax
            active = parts[4]
            if clk > 0:
                sm.append(clk)
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
            del active
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ----------------------------------------------------------------------------
def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_inputs(cfg, seed):
    """Inputs as host arrays (bf16 bits / fp32) for the oracle; weights made on a GPU if present."""
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = I.make_layer_inputs(cfg, seed, device=dev)
    out = {"X": _bits(inp["X"]), "W1": _bits(inp["W1"]), "W2": _bits(inp["W2"]),
           "logits": None if inp["logits"] is None else inp["logits"].numpy(),
           "Wr": None if inp["Wr"] is None else _bits(inp["Wr"])}
    del inp
    return out


def oracle_step(O, cfg, h, S):
    """The oracle over a bounded sample: the first S tokens of the batch, all stages."""
    X = h["X"][:S]
    L = None if h["logits"] is None else h["logits"][:S]
    return O.layer_forward(X, h["W1"], h["W2"], cfg.k, cfg.score, cfg.renormalize, logits=L,
                           Wr_bits=h["Wr"], temperature=cfg.temperature, min_prob=cfg.min_prob)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(cfg, h, S, reps=1):
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle_step(O, cfg, h, S)
    dt = time.perf_counter() - t0
    return S * reps / dt, dt


def arm_config(cfg, args, world):
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k,
            "f": cfg.f, "router": cfg.router, "score": cfg.score, "fp8": bool(args.fp8),
            "gather_on_load": bool(args.gather), "fused_ffn": bool(args.fused),
            "pipeline": bool(args.pipeline),
            "renormalize": cfg.renormalize, "temperature": cfg.temperature,
            "min_prob": cfg.min_prob, "tokens_per_gpu": cfg.T,
            "parallelism": f"replicas x{world} (no collective)",
            "l2": f"inputs larger than L2: each step streams "
                  f"{(3 if args.fp8 else 4) * cfg.E * cfg.d * cfg.f / 1e9:.2f} GB of expert weights"}


def sustained_peak_applies(loop_ms: float) -> bool:
    """Which measured GEMM peak a tensor-bound kernel is held to.

    The burst peak holds a kernel timed alone or in a short loop; the
    sustained one (cuBLAS after seconds under the 1 kW power cap) only a
    kernel timed inside a loop of a second or more.  A stray sw_power_cap
    sample in a short loop is a note, not a reason to switch peaks."""
    return loop_ms >= 1000.0


def host_cpu():
    """nproc and the CPU model name of this host (lscpu, else /proc/cpuinfo)."""
    model = None
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        m = re.search(r"^Model name:\s*(.+)$", out, re.M)
        model = m.group(1).strip() if m else None
    except (OSError, subprocess.SubprocessError):
        pass
    if model is None and os.path.exists("/proc/cpuinfo"):
        m = re.search(r"^model name\s*:\s*(.+)$", open("/proc/cpuinfo").read(), re.M)
        model = m.group(1).strip() if m else None
    return {"nproc": os.cpu_count(), "cpu_model": model}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def run_ours(args, cfg, rank, world, local_rank):
    import combine_moe_route_14_b200 as moe
    from combine_moe_route_14_b200 import build as B

    if rank == 0:
        B.build()
    if world > 1:
        torch.distributed.barrier()
    moe.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    inp = I.make_layer_inputs(cfg, args.seed, device=dev)  # weights: same on every rank
    X_host = inp["X"] if rank == 0 else I.random_bf16((cfg.T, cfg.d),
                                                       Rp.replica_token_seed(args.seed, rank), "X")
    X = X_host.to(dev)
    logits = inp["logits"].to(dev) if inp["logits"] is not None else None
    Wr = inp["Wr"].to(dev) if inp["Wr"] is not None else None
    layer = moe.MoeLayer(inp["W1"], inp["W2"], cfg.k, cfg.score, cfg.renormalize, Wr=Wr,
                         temperature=cfg.temperature, min_prob=cfg.min_prob, fp8=args.fp8,
                         gather_on_load=args.gather, fused_ffn=args.fused,
                         pipeline=args.pipeline)
    Y = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    counts = torch.empty((cfg.E,), dtype=torch.int32, device=dev)
    ws = layer.workspace(cfg.T)

    def step():
        layer(X, logits=logits, Y=Y, counts_out=counts)

    def sync_all():
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()

    def max_over_ranks(x: float) -> float:
        return Rp.max_over_ranks(x, device=dev)

    for _ in range(args.warmup):
        step()
    sync_all()
    bits = moe.moe_device_status(clear=True)
    if bits:
        raise RuntimeError(f"device status bits {bits} after warm-up")

    def step_percentiles(durs_ms):
        a = np.asarray(durs_ms) * 1e3
        return {"p10": float(np.percentile(a, 10)), "p50": float(np.percentile(a, 50)),
                "p90": float(np.percentile(a, 90))}

    graph_res = None
    if args.graph:
        # one forward captured on a side stream (per-device set-up already done
        # by the warm-up), replayed W times untimed, then K times with events
        gs = torch.cuda.Stream(device=dev)
        gs.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gs):
            with torch.cuda.graph(graph, stream=gs):
                step()
            for _ in range(args.warmup):
                graph.replay()
        gs.synchronize()
        gev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        sync_all()
        with torch.cuda.stream(gs):
            gev[0].record(gs)
            for i in range(args.steps):
                graph.replay()
                gev[i + 1].record(gs)
        gs.synchronize()
        sync_all()
        g_ms = max_over_ranks(gev[0].elapsed_time(gev[-1]))
        graph_res = {"value": Rp.weak_scaling_throughput(cfg.T, args.steps, world, g_ms),
                     "ms_per_step": g_ms / args.steps,
                     "step_us": step_percentiles([gev[i].elapsed_time(gev[i + 1])
                                                  for i in range(args.steps)])}
        del graph
        torch.cuda.synchronize(dev)

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    try:
        # ---- value: K whole-layer forwards, inputs resident in HBM
        vev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        sync_all()
        vev[0].record(stream)
        for i in range(args.steps):
            step()
            vev[i + 1].record(stream)
        sync_all()
        t_ms = max_over_ranks(vev[0].elapsed_time(vev[-1]))
        step_us = step_percentiles([vev[i].elapsed_time(vev[i + 1]) for i in range(args.steps)])

        # ---- per-stage times: the same kernels, launched stage by stage with events between
        # the layer's bf16 path ranks the slots in its routing kernel (no
        # layout launch); its staged form is moe_route_layout
        ranked = not (args.gather or args.fp8 or args.pipeline) and cfg.E <= 32
        stage_names = (["router_logits"] if Wr is not None else []) + (
            ["route_layout"] if ranked else ["route", "layout"]) + (
            ["pipeline"] if args.pipeline else
            (["quantize"] if args.gather and args.fp8 else [] if args.gather else ["dispatch"]) +
            (["ffn"] if args.fused else ["gemm1", "gemm2"]) + ["combine"])
        R = cfg.R
        L_buf = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=dev) if Wr is not None else logits
        idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
        g = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
        offs = torch.empty((cfg.E + 1,), dtype=torch.int32, device=dev)
        row_of = torch.empty((R,), dtype=torch.int32, device=dev)
        src_of = torch.empty((R,), dtype=torch.int32, device=dev)
        lws = torch.empty(max(16, moe.moe_layout_workspace_size(cfg.T, cfg.E, cfg.k)),
                          dtype=torch.uint8, device=dev)
        Xe = torch.empty((R, cfg.d), dtype=torch.uint8 if args.fp8 else torch.bfloat16, device=dev)
        Xq = torch.empty((cfg.T, cfg.d), dtype=torch.uint8, device=dev)
        ffn_ws = torch.empty(max(16, moe.moe_expert_ffn_fused_workspace_size(cfg.E, R)),
                             dtype=torch.uint8, device=dev)
        xs = torch.empty((2,), dtype=torch.float32, device=dev)
        pws = torch.empty(max(16, moe.moe_ffn_pipeline_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k,
                                                                       cfg.f)),
                          dtype=torch.uint8, device=dev) if args.pipeline else None
        H = torch.empty((R, cfg.f), dtype=torch.bfloat16, device=dev)
        Ye = torch.empty((R, cfg.d), dtype=torch.bfloat16, device=dev)
        fns = {
            "router_logits": lambda: moe.moe_router_logits(X, Wr, logits=L_buf),
            "route": lambda: moe.moe_route_ex(L_buf, cfg.k, cfg.score, cfg.renormalize,
                                              cfg.temperature, cfg.min_prob, idx, g),
            "layout": lambda: moe.moe_layout(idx, cfg.E, counts, offs, row_of, src_of, lws),
            "route_layout": lambda: route_layout_into(L_buf),
            # the layer's form: walked by token through row_of
            "dispatch": (lambda: moe.moe_dispatch_fp8_by_token(X, row_of, cfg.k, Xe, xs))
                        if args.fp8 else (lambda: moe.moe_dispatch_by_token(X, row_of, cfg.k, Xe)),
            "quantize": lambda: moe.moe_quantize_fp8(X, Xq, xs),
            "gemm1": ((lambda: moe.moe_expert_gemm_gather_fp8(Xq, xs, src_of, cfg.k, offs,
                                                              layer.W1q, layer.w1_scale, True, H))
                      if args.gather else
                      (lambda: moe.moe_expert_gemm_fp8(Xe, xs, offs, layer.W1q, layer.w1_scale,
                                                       True, H))) if args.fp8 else
                     ((lambda: moe.moe_expert_gemm_gather(X, src_of, cfg.k, offs, inp["W1"], True,
                                                          H)) if args.gather else
                      (lambda: moe.moe_expert_gemm(Xe, offs, inp["W1"], True, H))),
            "gemm2": lambda: moe.moe_expert_gemm(H, offs, inp["W2"], False, Ye),
            "ffn": (lambda: moe.moe_expert_ffn_fused_fp8(Xe, xs, offs, layer.W1q, layer.w1_scale,
                                                         inp["W2"], H, Ye, ffn_ws)) if args.fp8 else
                   (lambda: moe.moe_expert_ffn_fused(Xe, offs, inp["W1"], inp["W2"], H, Ye,
                                                     ffn_ws)),
            "combine": lambda: moe.moe_combine(Ye, row_of, g, Y),
            "pipeline": lambda: moe.moe_ffn_pipeline(X, src_of, row_of, g, offs, inp["W1"],
                                                     inp["W2"], Y=Y, ws=pws),
        }
        rl_ws = torch.empty(max(16, moe.load_library().moe_route_layout_workspace_size(
            cfg.T, cfg.E)), dtype=torch.uint8, device=dev)

        def route_layout_into(Lb):
            moe.moe_route_layout(Lb, cfg.k, cfg.score, cfg.renormalize, cfg.temperature,
                                 cfg.min_prob, out=(idx, g, counts, offs, row_of, src_of),
                                 ws=rl_ws)

        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stage_names) + 1)]
               for _ in range(args.steps)]
        # one untimed pass fills every staged buffer (offsets, row_of, ...) before
        # the queue-ahead GEMM launches below read them
        for n in stage_names:
            fns[n]()
        sync_all()
        # Queue ahead: a few untimed GEMM launches keep the GPU busy while the
        # host enqueues every staged call below, so the events between stages
        # measure device time, not the binding's per-call host overhead.
        for _ in range(max(2, (args.steps * len(stage_names) * 40) // max(1, int(stage_ms_hint(cfg))))):
            fns["pipeline" if args.pipeline else "gemm1"]()
        for s in range(args.steps):
            evs[s][0].record(stream)
            for i, n in enumerate(stage_names):
                fns[n]()
                evs[s][i + 1].record(stream)
        sync_all()
        stage_ms = {n: float(np.mean([evs[s][i].elapsed_time(evs[s][i + 1])
                                      for s in range(args.steps)]))
                    for i, n in enumerate(stage_names)}
        staged_total_ms = sum(stage_ms.values())

        # ---- e2e: host buffers in, host buffer out, every step's copies inside
        # the timed region, through the C ABI's host-buffer entry point: one
        # call runs the K batches, the library overlaps the copies of
        # neighbouring batches with the current forward (its own H2D, compute
        # and D2H streams, two device buffer sets)
        X_pin = X_host.pin_memory()
        L_pin = inp["logits"].pin_memory() if logits is not None else None
        Y_pin = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16).pin_memory()
        h2d = X_pin.numel() * 2 + (L_pin.numel() * 4 if L_pin is not None else 0)
        d2h = Y_pin.numel() * 2
        host_ws = torch.empty(max(16, moe.moe_host_workspace_size(
            moe.make_desc(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.score, cfg.renormalize,
                          cfg.temperature, cfg.min_prob, **layer.flags), L_pin is not None)),
            dtype=torch.uint8, device=dev)

        def host_batches(n):
            moe.moe_layer_forward_host(
                [X_pin] * n, layer.W1q if args.fp8 else inp["W1"], inp["W2"], cfg.k, [Y_pin] * n,
                score=cfg.score, renormalize=cfg.renormalize,
                logits_host=None if L_pin is None else [L_pin] * n,
                Wr=None if L_pin is not None else Wr, w1_scale=layer.w1_scale if args.fp8 else None,
                ws=host_ws, stream=stream, temperature=cfg.temperature, min_prob=cfg.min_prob,
                **layer.flags)

        host_batches(max(3, args.warmup))  # the first pass over pinned buffers runs slower
        sync_all()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        host_batches(args.steps)
        f1.record(stream)
        sync_all()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1))

    finally:
        if sampler:
            sampler.__exit__(None, None, None)

    bits = moe.moe_device_status(clear=True)
    if bits:
        raise RuntimeError(f"device status bits {bits} after the timed region")

    # ---- roofline of the dominant kernel
    counts_h = counts.cpu().numpy()
    model = stage_model(cfg, counts_h, args.fp8)
    dom = max(stage_ms, key=lambda n: stage_ms[n])
    peaks, peak_src = load_peaks()
    clocks = sampler.summary() if sampler else None
    sustained = sustained_peak_applies(max(t_ms, staged_total_ms * args.steps))
    per = model[dom]
    dur_s = stage_ms[dom] / 1e3
    # an FP8 contraction's peak: the measured bf16 peak x the nominal fp8:bf16 ratio (2);
    # the fused FFN in FP8 mode does half its FLOPs at each rate (harmonic mean)
    tc_ratio = 2.0 if (args.fp8 and dom == "gemm1") else (
        4.0 / 3.0 if (args.fp8 and dom == "ffn") else 1.0)
    if "flops" in per and per["flops"] / max(per["bytes"], 1) > (
            tc_ratio * peaks["bf16_tflops"] * 1e12) / (peaks["hbm_gbs"] * 1e9):
        peak = tc_ratio * (peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": per["flops"] / dur_s / 1e12, "peak": peak,
                "unit": "TFLOP/s"}
        roof["frac_vs_burst"] = roof["achieved"] / (tc_ratio * peaks["bf16_tflops"])
        roof["frac_vs_sustained"] = roof["achieved"] / (tc_ratio * peaks["bf16_tflops_sustained"])
    else:
        roof = {"bound": "hbm", "achieved": per["bytes"] / dur_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["peak_source"] = (f"{peak_src} ("
                           f"{'sustained: timed loop of 1 s or more' if sustained and roof['bound'] == 'tensor' else 'burst: timed loop under 1 s'})"
                           + ("" if tc_ratio == 1.0 else
                              " x 2 (fp8:bf16 nominal ratio)" if tc_ratio == 2.0 else
                              " x 4/3 (half the FLOPs at the fp8 rate, half at bf16)"))
    kname = {"gemm1": ("grouped_gemm_fp8_gelu" if args.fp8 else "grouped_gemm_gelu")
                      + ("_gather" if args.gather else ""),
             "gemm2": "grouped_gemm",
             "ffn": "fused_ffn_fp8" if args.fp8 else "fused_ffn",
             "pipeline": "ffn_pipeline"}.get(dom, dom)
    tr = ncu_traffic(kname, cfg.name)
    roof["traffic"] = tr
    roof["algorithmic_bytes"] = per["bytes"]

    stages = {}
    for n, ms in stage_ms.items():
        st = {"us": ms * 1e3}
        if "bytes" in model[n]:
            st["GB/s"] = model[n]["bytes"] / (ms / 1e3) / 1e9
            st["hbm_frac"] = st["GB/s"] / peaks["hbm_gbs"]
        if "flops" in model[n]:
            st["TFLOP/s"] = model[n]["flops"] / (ms / 1e3) / 1e12
        stages[n] = st

    value = Rp.weak_scaling_throughput(cfg.T, args.steps, world, t_ms)
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "step_us": step_us,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 (dispatch, GEMM-1) + bf16" if args.fp8 else "bf16", "data": "synthetic",
        "config": arm_config(cfg, args, world),
        "roofline": roof,
        "stages": stages,
        "expert_counts": {"max": int(counts_h.max()), "mean": float(counts_h.mean()),
                          "min": int(counts_h.min()),
                          "dropped_slots": int(cfg.R - counts_h.sum())},
        "e2e": {"value": Rp.weak_scaling_throughput(cfg.T, args.steps, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps,
                "path": "C ABI moe_layer_forward_host: H2D, forward and D2H of neighbouring "
                        "batches overlapped on the library's streams, two device buffer sets"},
        "gpu_launches": args.steps * (moe.moe_kernel_launches_per_forward_fp8 if args.fp8 else
                                      moe.moe_kernel_launches_per_forward)(
            moe.make_desc(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.score, cfg.renormalize,
                          gather_on_load=args.gather, fused_ffn=args.fused,
                          pipeline=args.pipeline),
            Wr is not None),
        "clocks": clocks,
    }
    if graph_res is not None:
        res["graph"] = graph_res
    del X, logits, Wr, layer, inp, ws, Xe, H, Ye
    torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral", choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 mode: E4M3 dispatch with a per-tensor scale and FP8 GEMM-1")
    ap.add_argument("--gather", action="store_true",
                    help="fuse the dispatch into GEMM-1 (gather-on-load)")
    ap.add_argument("--fused", action="store_true",
                    help="both expert GEMMs in one persistent kernel")
    ap.add_argument("--pipeline", action="store_true",
                    help="token-centric pipeline: dispatch, both GEMMs and the combine in one "
                         "persistent kernel after route and layout")
    ap.add_argument("--graph", action="store_true",
                    help="also time the forward replayed from a CUDA graph")
    args = ap.parse_args()
    if args.gather and (args.fused or args.pipeline):
        ap.error("--gather cannot be combined with --fused or --pipeline")
    if args.pipeline and (args.fp8 or args.fused):
        ap.error("--pipeline is a bf16 path of its own (no --fp8, no --fused)")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = I.workload(args.workload)

    if args.impl == "reference":
        if rank != 0:
            return 0
        # the same sample per step as the cpu_baseline leg (the first S tokens,
        # all stages), so that the two CPU figures measure the same work
        S = ORACLE_SAMPLE.get(cfg.name, 64)
        h = host_inputs(cfg, args.seed)
        for _ in range(args.warmup):
            time_oracle(cfg, h, S)
        v, dt = time_oracle(cfg, h, S, reps=args.steps)
        cores = blas_threads()
        res = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
               "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "impl": "reference",
               "config": arm_config(cfg, args, args.gpus),
               "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                **host_cpu(),
                                "sample": f"first {S} of the {cfg.T} tokens per step, all stages"},
               "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}}
        print(json.dumps(res), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, cfg, rank, world, local_rank)
        if rank == 0 and args.fp8:
            res["cpu_baseline"] = {"skipped": "FP8 mode: the oracle's E4M3 quantisation of W1 "
                                              "takes ~10 s per expert; the bf16 line carries "
                                              "the oracle baseline"}
        elif rank == 0 and world == 1 and not args.no_cpu_baseline:
            S_base = ORACLE_SAMPLE.get(cfg.name, 64)
            h = host_inputs(cfg, args.seed)
            runs, tot = 0, 0.0
            while runs == 0 or tot < 10.0:  # about 10 s of oracle work
                _, dt = time_oracle(cfg, h, S_base)
                runs, tot = runs + 1, tot + dt
            v = S_base * runs / tot
            res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": blas_threads(),
                                   "kind": "oracle", **host_cpu(),
                                   "sample": f"first {S_base} of the {cfg.T} tokens, all stages, "
                                             f"{runs} run(s), {tot:.1f} s"}
            try:  # the same oracle on one core (BLAS limited to one thread)
                from threadpoolctl import threadpool_limits
                S1 = min(S_base, 256)
                with threadpool_limits(limits=1):
                    v1, dt1 = time_oracle(cfg, h, S1)
                res["cpu_baseline"]["single_thread"] = {
                    "value": v1, "unit": UNIT, "cores": 1,
                    "sample": f"first {S1} of the {cfg.T} tokens, all stages, one run ({dt1:.1f} s)"}
            except ImportError:
                pass
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
