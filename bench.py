#!/usr/bin/env python
"""Benchmark of the MXFP4 MoE expert layer (libmxmoe, sm_100a).

One step = one pass of the whole layer over one batch of tokens: router GEMM,
top-k routing, grouping by expert, gate/up + SwiGLU, down projection, weighted
combine, through the library's C ABI. Metric: layer tokens/s, with the
expert-weight HBM GB/s and its fraction of the measured HBM peak alongside.

Default run: the five layer workloads in one process on one layer of 384 MXFP4
experts (top-8, hidden 6144, expert intermediate 2048; the tiny one on its own
small layer). The JSON line's headline is the largest single-GPU workload,
prefill8192 (8192 tokens, tensor-bound); `per_config` holds the same fields
for tiny, verify8 (one DFlash verify block of 8 tokens, the block size of the
"MiMo-V2.5-Pro-FP4-DFlash" model card, section 3), verify256 (32 such blocks)
and zipf1024 (1024 tokens, Zipf-skewed routing). Inputs are synthetic
(datagen); every step streams the touched experts' weights (>1 GB) through
HBM, far above the 126 MB L2.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                       [--config NAME] [--no-per-config]
Under torchrun each rank runs an independent replica on its own GPU (no
collective on the data path; weak scaling); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import datagen  # noqa: E402

METRIC = "MXFP4 MoE-layer tokens/s; expert-weight HBM GB/s as % of peak (1×B200)"
UNIT = "tokens/s"
LARGE_PATH_ROWS = 16384  # grouped rows (tokens x top-k) from which both FFN stages run on the large-token kernel
PERSISTENT_MAX_TOKENS = 0  # mxmoe_layer_forward runs one persistent kernel up to this many tokens


def front_path(T: int, k: int, E: int) -> bool:
    """Whether mxmoe_layer_forward (MXFP4 weights) takes its front path: router,
    routing, grouping and activation terms in one cooperative kernel, below
    128 tokens with T*k <= 4096 and k <= E <= 384."""
    return 1 <= T < 128 and T * k < LARGE_PATH_ROWS and T * k <= 4096 and k <= E <= 384


def kernels_per_step(T: int, k: int, E: int, H: int) -> int:
    """Kernels one layer step launches, following the library's dispatch: on
    the front path the front kernel, the two FFN stages and the combine;
    otherwise router GEMM (one kernel either way), route, grouping (one kernel,
    or three above 4096 pairs with E <= 1024), then the FFN -- E2M1-term path:
    x_terms + two stages; large-token path: passes + slot rows + x8_terms + two
    stages; both from 128 tokens below 16384 grouped rows -- then combine."""
    if front_path(T, k, E):
        return 4
    rows = T * k
    n = 3 if (rows > 4096 and E <= 1024) else 1
    n += 2  # router GEMM, route
    large_all = rows >= LARGE_PATH_ROWS
    hybrid = not large_all and T >= 128
    if not large_all:
        n += 3
    if large_all or hybrid:
        n += 5
    return n + 1  # combine


PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


HEADLINE = "prefill8192"  # the largest workload that fits one GPU


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default=HEADLINE, choices=[c.name for c in datagen.CONFIGS],
                    help="the workload of the line's headline value")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure the headline workload only (no per_config object)")
    ap.add_argument("--min-timed-s", type=float, default=0.25,
                    help="per_config entries: at least this many seconds of timed steps per workload")
    ap.add_argument("--batches", type=int, default=16, help="distinct rotating input batches (small token counts)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=8, help="tokens of the oracle's timed CPU sample")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling only: shrink the layer to this many experts (0 = the workload's)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling only: this many tokens per step (0 = the workload's)")
    ap.add_argument("--workload", choices=["layer", "verify_block"], default="layer",
                    help="layer: the MoE layer (the headline); verify_block: block verification of drafts")
    ap.add_argument("--blocks", type=int, default=32, help="verify_block: drafted blocks per step")
    ap.add_argument("--vocab", type=int, default=datagen.VERIFY_VOCAB, help="verify_block: vocabulary size")
    ap.add_argument("--temperature", type=float, default=1.0, help="verify_block: 0 = greedy verification")
    return ap.parse_args()


def workload_config(cfg, world: int, batches: int):
    big = cfg.T * cfg.k * cfg.H * 2 > (126 << 20)  # the step's x rows alone exceed L2
    return {
        "workload": "%s: MXFP4 MoE layer, T=%d tokens, H=%d, E=%d experts, top-%d, I=%d, block 32"
                    % (cfg.name, cfg.T, cfg.H, cfg.E, cfg.k, cfg.I),
        "tokens_per_step": cfg.T,
        "global_batch": cfg.T * world,
        "hidden": cfg.H,
        "experts": cfg.E,
        "top_k": cfg.k,
        "intermediate": cfg.I,
        "router_bias_zipf": cfg.zipf_s,
        "parallelism": "replicas x%d" % world,
        "l2": "inputs larger than L2: each step streams the touched experts' MXFP4 weights (%s) and "
              "%d input batches rotate" % (">7 GB" if big else ">0.4 MB" if cfg.E <= 16 else ">1 GB", batches),
    }


def load_peaks():
    """(HBM GB/s, sustained bf16 TFLOP/s, source): the machine's measured copy
    bandwidth and cuBLAS bf16 GEMM rate under the power cap, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1400.0, "fallback"


# Device code whose DRAM traffic a committed ncu capture describes: the
# E2M1-term gate/up kernel (decode-sized workloads) and the large-token gate/up
# kernel (from 16384 grouped rows).
TRAFFIC_SOURCES = {
    "ffn_gate_up": ("mxfp4_quantized_moe_router_b200/csrc/ffn.cu", "mxfp4_quantized_moe_router_b200/csrc/common.cuh",
                    "mxfp4_quantized_moe_router_b200/csrc/tcgen05.cuh"),
    "ffn_f8_gate_up": ("mxfp4_quantized_moe_router_b200/csrc/ffn_prefill8.cu",
                       "mxfp4_quantized_moe_router_b200/csrc/common.cuh",
                       "mxfp4_quantized_moe_router_b200/csrc/tcgen05.cuh"),
}


def kernel_source_sha(kind: str = "ffn_gate_up") -> str:
    """Hash of a kernel's code (comments, blank lines and the file's C entry
    points left out), which keys the committed traffic capture to the device
    code it was taken on."""
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES[kind]:
        with open(os.path.join(ROOT, rel)) as f:
            src = f.read()
        src = src.split('extern "C"', 1)[0]  # the kernels and their launchers, not the argument checks
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(line.rstrip() for line in src.splitlines() if line.strip()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kind: str, workload: str, touched: float):
    """DRAM bytes (read + write) per launch of the gate/up stage, from the
    committed ncu capture of the same kernel source (null once the source has
    changed). A capture keeps either its bytes per launch (taken on this very
    workload) or its bytes per touched expert (taken on a shrunk layer), which
    are scaled to this run's mean number of touched experts per launch."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        ent = d.get(kind, {}).get(workload)
        if ent and ent.get("source_sha") == kernel_source_sha(kind):
            if "dram_bytes_per_launch" in ent:
                return float(ent["dram_bytes_per_launch"])
            return float(ent["dram_bytes_per_touched_expert"]) * touched
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# replicas (one process per GPU under torchrun; no collective on the data path)
# ---------------------------------------------------------------------------
def dist_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_input_seed(seed: int, rank: int, batch: int) -> int:
    """Seed of input batch `batch` on rank `rank`: every replica runs its own tokens."""
    return seed + 1000 * rank + batch


def max_over_ranks(v: float, world: int, device="cpu") -> float:
    """Largest v over all ranks (every rank must call it, in the same order)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_step_per_rank * steps * world / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock and throttle-reason samples of this process's GPU,
    every 50 ms from start() to stop(). start() returns once the first sample
    has arrived (or after 3 s), so that every timed loop after it is covered;
    summary() reads the samples that fall inside the given timed windows."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.samples = []
        self.proc = None
        self.thread = None
        self.first = threading.Event()

    def start(self, wait_s: float = 3.0):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        self.first.wait(wait_s)

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9 or not parts[0].endswith(self.uuid):
                continue
            try:
                self.samples.append(dict(t=time.time(), sm=float(parts[1]), max=float(parts[2]),
                                         hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                self.first.set()
            except ValueError:
                pass

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, windows):
        """Median SM clock, max clock and active throttle reasons over the
        samples taken inside the (t0, t1) windows (host time around each timed
        loop, widened by one sampling period); if no sample fell inside a
        window, the two samples nearest to it."""
        pad = self.PERIOD_MS / 1e3
        win = [s for s in self.samples if any(t0 - pad <= s["t"] <= t1 + pad for t0, t1 in windows)]
        nearest = False
        if not win and self.samples and windows:
            mid = 0.5 * (windows[0][0] + windows[-1][1])
            win = sorted(self.samples, key=lambda s: abs(s["t"] - mid))[:2]
            nearest = True
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for s in win:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if s[key].lower().startswith("active"):
                    reasons.add(name)
        out = {"sm_mhz": statistics.median(s["sm"] for s in win), "sm_max_mhz": max(s["max"] for s in win),
               "reasons": sorted(reasons), "samples": len(win), "period_ms": self.PERIOD_MS}
        if nearest:
            out["nearest_to_window"] = True
        return out


# ---------------------------------------------------------------------------
# host description and CPU oracle timing (baseline and reference arm)
# ---------------------------------------------------------------------------
def host_cpu():
    """(logical cores the host offers, CPU model name)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 0, model


def oracle_setup(cfg, seed, token_rows, x_bf16, bias):
    """Route the sample tokens with the oracle and quantise (untimed) the experts
    they touch. Returns the experts dict."""
    import oracle
    import torch

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wg = datagen.make_router_weight(cfg, seed, dev).cpu()
    xs = x_bf16[token_rows].cpu()
    logits = oracle.router_logits(xs, wg, bias)
    ids, _ = oracle.route(logits, cfg.k)
    experts = {}
    for e in sorted(set(ids.ravel().tolist())):
        w13 = datagen.make_w13(cfg, e, seed, dev).cpu()
        w2 = datagen.make_w2(cfg, e, seed, dev).cpu()
        p13, s13 = oracle.quantize(w13)
        p2, s2 = oracle.quantize(w2)
        experts[e] = (p13, s13, p2, s2)
    return wg, xs, experts


def oracle_layer_time(cfg, wg, xs, bias, experts):
    import oracle

    t = time.perf_counter()
    oracle.moe_layer(xs, wg, bias, lambda e: experts[e], cfg.k, threads=1)
    return time.perf_counter() - t


def cpu_baseline(cfg, seed, x_cpu, bias, n_tokens):
    """The oracle as it stands on a seeded sample of the workload's tokens, one
    thread on the host cores."""
    rows = sorted(datagen.sample_tokens(cfg.T, min(n_tokens, cfg.T), seed).tolist())
    wg, xs, experts = oracle_setup(cfg, seed, rows, x_cpu, bias)
    dt = oracle_layer_time(cfg, wg, xs, bias, experts)
    cores, model = host_cpu()
    return {"value": len(rows) / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d seeded token(s) of the %s workload through the float64 C oracle (router, routing, %d experts "
                      "decoded and run, combine; experts quantised beforehand, untimed), one thread"
                      % (len(rows), cfg.name, len(experts)),
            "seconds": dt, "host_cores": cores, "cpu_model": model}


def run_reference(args):
    """--impl reference: the float64 CPU oracle as it stands, on host cores."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cfg = datagen.BY_NAME[args.config]
    x = datagen.make_x(cfg, args.seed)
    bias = datagen.make_router_bias(cfg, args.seed)
    # one token per step (all of its k experts); a step is a bounded sample
    n = min(cfg.T, max(1, args.warmup + args.steps))
    tokens = sorted(datagen.sample_tokens(cfg.T, n, args.seed).tolist())
    steps_tokens = [[tokens[i % len(tokens)]] for i in range(args.warmup + args.steps)]
    need = sorted(set(t for s in steps_tokens for t in s))
    wg, _, experts = oracle_setup(cfg, args.seed, need, x, bias)
    times = []
    for i, rows in enumerate(steps_tokens):
        xs = x[rows]
        dt = oracle_layer_time(cfg, wg, xs, bias, experts)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = len(times) / total
    cores, model = host_cpu()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, 1, 1),
        "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": UNIT,
                         "sample": "each step: 1 seeded token of the %s workload through the float64 C oracle "
                                   "(router, routing, its %d experts decoded and run, combine), one thread"
                                   % (cfg.name, cfg.k), "host_cores": cores, "cpu_model": model},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------
def make_layer(mx, cfg, seed, dev, fmt="mxfp4"):
    """A layer's router weight and prepacked experts on the device (generated
    by datagen, quantised and prepacked by the library): MXFP4, or with
    fmt="fp8" FP8 (E4M3, one E8M0 scale per 32)."""
    import torch

    wg = datagen.make_router_weight(cfg, seed, dev)
    ew = (mx.ExpertWeightsFp8 if fmt == "fp8" else mx.ExpertWeights)(cfg.E, cfg.H, cfg.I, dev)
    for e in range(cfg.E):
        ew.quantize_expert(e, datagen.make_w13(cfg, e, seed, dev), datagen.make_w2(cfg, e, seed, dev))
    ew.prepack()
    torch.cuda.synchronize()
    prepacked = ew.prepacked
    del ew  # the kernels stream the prepacked blob only
    torch.cuda.empty_cache()
    return wg, prepacked


def fp8_expert_bytes(cfg) -> int:
    """FP8 bytes of one expert: 3*H*I one-byte codes plus one scale byte per 32."""
    n = 3 * cfg.H * cfg.I
    return n + n // 32


def measure_layer(mx, cfg, wg, prepacked, args, steps, warmup, world, rank, dev, clocks, want_e2e=True, fmt="mxfp4",
                  path="auto"):
    """Time one workload: the whole layer (device-resident inputs), its
    dominant unit (CUDA events on the launching stream: the gate/up stage, or
    for FP8 experts the whole expert FFN), and the end-to-end leg with host
    copies. Every rank takes the same collective steps."""
    fp8 = fmt == "fp8"
    import torch
    import torch.distributed as dist

    T, H, E, k, I = cfg.T, cfg.H, cfg.E, cfg.k, cfg.I
    nb = max(1, args.batches if T * H * 2 <= (16 << 20) else 2)  # rotate batches of small token counts
    xs = [datagen.make_x(cfg, replica_input_seed(args.seed, rank, b), dev) for b in range(nb)]
    bias_np = datagen.make_router_bias(cfg, args.seed)
    bias = torch.from_numpy(bias_np).to(dev) if bias_np is not None else None
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    src_row = torch.empty(T * k, dtype=torch.int32, device=dev)
    dst_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    fws = torch.empty((mx.mxmoe_ffn_workspace_size_fp8 if fp8 else mx.mxmoe_ffn_workspace_size)(T, k, E, H, I),
                      dtype=torch.uint8, device=dev)
    pms = torch.empty(max(1, mx.mxmoe_permute_scratch_size(T, k, E)), dtype=torch.uint8, device=dev)
    y_perm = torch.empty((T * k, H), dtype=torch.float32, device=dev)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    L = mx.load()
    P = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    fws_bytes = fws.numel()
    lws = torch.empty((mx.mxmoe_workspace_size_fp8 if fp8 else mx.mxmoe_workspace_size)(T, H, I, E, k),
                      dtype=torch.uint8, device=dev)
    forward = (L.mxmoe_layer_forward_fp8 if fp8 else
               {"auto": L.mxmoe_layer_forward, "chained": L.mxmoe_layer_forward_chained,
                "persistent": L.mxmoe_layer_forward_persistent}[path])
    lws_bytes = lws.numel()

    def layer_step(b, x=None, y_out=None):
        x = xs[b % nb] if x is None else x
        y_out = y if y_out is None else y_out
        rc = forward(P(x), P(wg), P(bias), P(prepacked), T, H, I, E, k, P(y_out), P(ids), P(w), P(lws), lws_bytes, sp)
        if rc:
            raise RuntimeError("mxmoe_layer_forward failed: " + mx.last_error())

    def split_step(b, ev):
        """The same layer through the per-step entry points, with events around
        the gate/up stage (the unit that streams 2/3 of the weight bytes)."""
        x = xs[b % nb]
        rc = L.mxmoe_router_gemm(P(x), P(wg), P(bias), T, H, E, P(logits), sp)
        rc |= L.mxmoe_route(P(logits), T, E, k, P(ids), P(w), sp)
        rc |= L.mxmoe_permute_ws(P(ids), T, k, E, P(offsets), P(src_row), P(dst_of), P(pms), pms.numel(), sp)
        if fp8:  # the FP8 FFN has no separate stage entry points: the unit is the whole expert FFN
            ev[0].record(stream)
            rc |= L.mxmoe_expert_ffn_fp8(P(x), P(offsets), P(src_row), P(prepacked), T, k, E, H, I, P(y_perm),
                                         P(fws), fws_bytes, sp)
            ev[1].record(stream)
        else:
            ev[0].record(stream)
            rc |= L.mxmoe_ffn_gate_up(P(x), P(offsets), P(src_row), P(prepacked), T, k, E, H, I, P(fws), fws_bytes,
                                      sp)
            ev[1].record(stream)
            rc |= L.mxmoe_ffn_down(P(offsets), P(prepacked), T, k, E, H, I, P(y_perm), P(fws), fws_bytes, sp)
        rc |= L.mxmoe_combine(P(y_perm), P(dst_of), P(w), T, k, H, P(y), sp)
        if rc:
            raise RuntimeError("libmxmoe call failed: " + mx.last_error())

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(v: float) -> float:
        return max_over_ranks(v, world, dev)

    # touched experts per batch (untimed), for the weight-byte accounting; the
    # same calls give a first step-time estimate
    touched = []
    est0 = time.perf_counter()
    for b in range(nb):
        layer_step(b)
        torch.cuda.synchronize()
        touched.append(int(torch.unique(ids).numel()))
    est_s = (time.perf_counter() - est0) / nb
    assert mx.mxmoe_read_status(lws) == mx.OK
    if steps is None:  # per_config entries: at least min_timed_s of timed steps (same count on every rank)
        steps = max(args.steps, int(np.ceil(rank_max(args.min_timed_s / max(est_s, 1e-6)))))
        steps = min(steps, 20000)
    windows = []

    # --- device-resident timed region: the whole layer per step
    for i in range(warmup):
        layer_step(i)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for i in range(steps):
        layer_step(warmup + i)
    end.record(stream)
    torch.cuda.synchronize()
    windows.append((t0, time.time()))
    barrier()
    ms = start.elapsed_time(end)
    ms_max = rank_max(ms)

    # --- roofline region: same steps through the per-step entry points, with
    # CUDA events on the launching stream around the gate/up stage
    for i in range(warmup):
        split_step(i, (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
    ev_unit = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(steps):
        split_step(warmup + i, ev_unit[i])
    torch.cuda.synchronize()
    windows.append((t0, time.time()))
    barrier()
    unit_ms = [a.elapsed_time(b) for a, b in ev_unit]

    # --- end to end through the public API with host buffers: every step
    # uploads its x from pinned host memory and downloads its y. The copies
    # run on their own streams into double-buffered device x and y, ordered
    # by events, so that step i+1's upload and step i-1's download overlap
    # step i's layer, as in a serving loop.
    ms_e2e = None
    if want_e2e:
        x_host = [xb.cpu().pin_memory() for xb in xs]
        y_host = [torch.empty((T, H), dtype=torch.float32).pin_memory() for _ in range(2)]
        x_dev = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        y_dev = [torch.empty((T, H), dtype=torch.float32, device=dev) for _ in range(2)]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        x_ready, x_free = [torch.cuda.Event() for _ in range(2)], [torch.cuda.Event() for _ in range(2)]
        y_ready, y_free = [torch.cuda.Event() for _ in range(2)], [torch.cuda.Event() for _ in range(2)]

        def e2e_step(s):
            j = s & 1
            up.wait_event(x_free[j])  # the layer two steps back has read x_dev[j]
            with torch.cuda.stream(up):
                x_dev[j].copy_(x_host[s % nb], non_blocking=True)
            x_ready[j].record(up)
            stream.wait_event(x_ready[j])
            stream.wait_event(y_free[j])  # y_dev[j] of two steps back is downloaded
            layer_step(s, x_dev[j], y_dev[j])
            x_free[j].record(stream)
            y_ready[j].record(stream)
            down.wait_event(y_ready[j])
            with torch.cuda.stream(down):
                y_host[j].copy_(y_dev[j], non_blocking=True)
            y_free[j].record(down)

        def e2e_run(first, n):
            for i in range(first, first + n):
                e2e_step(i)
            for j in range(2):  # the last downloads end the region
                stream.wait_event(y_free[j])

        e2e_run(0, warmup)
        barrier()
        torch.cuda.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        s2.record(stream)
        up.wait_event(s2)
        e2e_run(warmup, steps)
        e2.record(stream)
        torch.cuda.synchronize()
        windows.append((t0, time.time()))
        barrier()
        ms_e2e = rank_max(s2.elapsed_time(e2))

    peak, peak_tf, peak_kind = load_peaks()
    steps_batches = [(warmup + i) % nb for i in range(steps)]
    mean_touched = float(np.mean([touched[b] for b in steps_batches]))
    value = whole_job_rate(T, steps, world, ms_max)
    expert_bytes = fp8_expert_bytes(cfg) if fp8 else cfg.expert_bytes
    weight_gbs = mean_touched * expert_bytes * steps / (ms / 1e3) / 1e9
    unit_ms_mean = float(np.mean(unit_ms))
    if fp8:
        # dominant unit: mxmoe_expert_ffn_fp8 (act_terms + both FP8 stages); algorithmic bytes = the touched
        # experts' FP8 bytes + x read + h written and read back + y_perm written
        unit_bytes = mean_touched * expert_bytes + T * H * 2 + 2 * T * k * I * 2 + T * k * H * 4
        achieved = unit_bytes / (unit_ms_mean / 1e3) / 1e9
        roofline = {"kernel": "mxmoe_expert_ffn_fp8 (act_terms_kernel + ffn_mxf4_kernel<gate_up|down, fp8 weights>)",
                    "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
                    else "fallback 6.65 TB/s", "traffic": None, "unit_ms": unit_ms_mean,
                    "algorithmic_bytes_per_launch": unit_bytes}
        dtype = "e2m1 digit terms x e4m3 -> f32"
    elif T * k >= LARGE_PATH_ROWS:
        # dominant unit: mxmoe_ffn_gate_up on block-scaled tensor cores (passes, slot rows, x8_terms +
        # ffn_f8_kernel<gate_up>); algorithmic work = the dense gate/up contraction of every grouped row,
        # 2 * rows * 2I * H flops, against the bf16 peak: x enters as two E4M3 terms on the fp8 kind,
        # whose rate is twice bf16's, so the two terms take the time of one bf16 contraction (the same
        # fraction as the issued term work against the fp8 peak)
        unit_flops = 2.0 * T * k * 2 * I * H
        achieved = unit_flops / (unit_ms_mean / 1e3) / 1e12
        roofline = {"kernel": "mxmoe_ffn_gate_up (x8_terms_kernel + ffn_f8_kernel<gate_up>)", "bound": "tensor",
                    "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
                    "peak_source": "%s (MEASURED_PEAKS.json bf16_tflops_sustained; the fp8 kind's issued two-term "
                                   "work is twice the flops at twice the rate)" % peak_kind
                    if peak_kind == "measured" else "fallback 1.4 PFLOP/s sustained",
                    "traffic": profiled_traffic("ffn_f8_gate_up", cfg.name, mean_touched), "unit_ms": unit_ms_mean,
                    "algorithmic_flops_per_launch": unit_flops,
                    "issued_fp8_frac": 2 * achieved / (2 * peak_tf)}
        dtype = "e2m1 x e4m3 terms -> f32"
    else:
        # dominant unit: mxmoe_ffn_gate_up (x_terms + gate/up stage); algorithmic
        # bytes = gate/up MXFP4 bytes of the touched experts + x read + h written
        w13_bytes = 2 * I * H * 17 // 32
        unit_bytes = mean_touched * w13_bytes + T * H * 2 + T * k * I * 2
        achieved = unit_bytes / (unit_ms_mean / 1e3) / 1e9
        hybrid = T >= 128
        roofline = {"kernel": "mxmoe_ffn_gate_up (act_terms_kernel + ffn_mxf4_kernel<gate_up>%s)"
                              % (" + the large-token kernels for experts with >= 128 rows" if hybrid else ""),
                    "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
                    else "fallback 6.65 TB/s",
                    "traffic": profiled_traffic("ffn_gate_up", cfg.name, mean_touched), "unit_ms": unit_ms_mean,
                    "algorithmic_bytes_per_launch": unit_bytes}
        dtype = "e2m1 x e2m1 digit terms -> f32"
    out = {
        "value": value, "unit": UNIT, "steps": steps, "warmup": warmup, "ms_per_step": ms_max / steps,
        "dtype": dtype, "config": workload_config(cfg, world, nb), "weight_gbs": weight_gbs,
        "weight_frac_of_hbm_peak": weight_gbs / peak, "touched_experts_per_step": mean_touched,
        "roofline": roofline, "clocks": clocks.summary(windows),
        "gpu_launches": (kernels_per_step(T, k, E, H) if not fp8 else (3 if T * k > 4096 and E <= 1024 else 1) + 6)
        * steps,
    }
    if fp8:
        out["weight_format"] = "fp8 (E4M3, one E8M0 scale per 32)"
    persistent = path == "persistent" or (path == "auto" and not fp8 and T <= PERSISTENT_MAX_TOKENS and E <= 384)
    out["layer_path"] = ("persistent kernel" if persistent else
                         "front kernel + chained launches" if not fp8 and front_path(T, k, E) else "chained launches")
    if persistent:  # one cooperative launch per step (plus the status clear)
        out["gpu_launches"] = steps
    if ms_e2e is not None:
        out["e2e"] = {"value": T * steps * world / (ms_e2e / 1e3), "unit": UNIT, "h2d_bytes_per_step": T * H * 2,
                      "d2h_bytes_per_step": T * H * 4,
                      "api": "mxmoe_layer_forward with pinned host x/y copies on their own streams, double-buffered "
                             "(step i+1's upload and step i-1's download overlap step i)"}
    out["_x0"] = xs[0].cpu()
    out["_bias"] = bias_np
    return out


def run_native(args):
    import dataclasses

    import torch
    import torch.distributed as dist

    import mxfp4_quantized_moe_router_b200 as mx

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())

    def shaped(cfg):
        if args.experts:
            cfg = dataclasses.replace(cfg, name=cfg.name + "-E%d" % args.experts, E=args.experts)
        if args.tokens:
            cfg = dataclasses.replace(cfg, name=cfg.name + "-T%d" % args.tokens, T=args.tokens)
        return cfg

    head = shaped(datagen.BY_NAME[args.config])
    names = [c.name for c in datagen.CONFIGS] if not args.no_per_config else [args.config]
    cfgs = [shaped(datagen.BY_NAME[n]) for n in names]
    # one set of weights per distinct layer (H, E, I); the tiny workload has its own
    layers = {}
    for c in cfgs:
        key = (c.H, c.E, c.I)
        if key not in layers:
            layers[key] = make_layer(mx, c, args.seed, dev)

    clocks = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    results = {}
    for c in cfgs:  # the headline last, after the others have warmed the GPU
        if c.name == head.name:
            continue
        wg, prepacked = layers[(c.H, c.E, c.I)]
        results[c.name] = measure_layer(mx, c, wg, prepacked, args, None, args.warmup, world, rank, dev, clocks)
        torch.cuda.empty_cache()
    fp8_name = None
    extra = []
    if not args.no_per_config and not args.experts and not args.tokens:
        # the persistent layer kernel against the chained launches, on the decode-sized workloads
        for name, path in (("verify8", "persistent"), ("verify256", "persistent")):
            c = datagen.BY_NAME[name]
            wg_c, pre_c = layers[(c.H, c.E, c.I)]
            key = "%s_%s" % (name, path)
            results[key] = measure_layer(mx, c, wg_c, pre_c, args, None, args.warmup, world, rank, dev, clocks,
                                         want_e2e=False, path=path)
            extra.append(key)
            torch.cuda.empty_cache()
        # the verify8 workload with FP8 experts (the pages' 8-bit baseline), to set its weight stream against MXFP4's
        c = datagen.BY_NAME["verify8"]
        wg8, pre8 = make_layer(mx, c, args.seed, dev, fmt="fp8")
        fp8_name = "verify8_fp8"
        results[fp8_name] = measure_layer(mx, c, wg8, pre8, args, None, args.warmup, world, rank, dev, clocks,
                                          fmt="fp8")
        del wg8, pre8
        torch.cuda.empty_cache()
    wg, prepacked = layers[(head.H, head.E, head.I)]
    res = measure_layer(mx, head, wg, prepacked, args, args.steps, args.warmup, world, rank, dev, clocks)
    clocks.stop()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    x0, bias_np = res.pop("_x0"), res.pop("_bias")
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": res["dtype"],
        "data": "synthetic (seeded datagen: x~N(0,1), router W~N(0,0.02), expert W~N(0,0.02) quantised to MXFP4 by "
                "the library)",
        "config": res["config"],
    }
    for key in ("weight_gbs", "weight_frac_of_hbm_peak", "touched_experts_per_step", "roofline", "clocks",
                "gpu_launches", "e2e"):
        line[key] = res[key]
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(head, args.seed, x0, bias_np, args.cpu_tokens)
    if results:
        line["per_config"] = {}
        for name in [c.name for c in cfgs] + extra + ([fp8_name] if fp8_name else []):
            if name == head.name:
                r = dict(res)
            else:
                r = results[name]
                r.pop("_x0")
                r.pop("_bias")
            line["per_config"][name] = {key: r[key] for key in (
                "value", "unit", "ms_per_step", "steps", "dtype", "weight_gbs", "weight_frac_of_hbm_peak",
                "touched_experts_per_step", "roofline", "e2e", "clocks", "gpu_launches", "weight_format",
                "layer_path") if key in r}
            line["per_config"][name]["workload"] = r["config"]["workload"]
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# block verification workload
# ---------------------------------------------------------------------------
VERIFY_K = 8  # drafted tokens per block (the model card's verify block)
VERIFY_METRIC = "verified draft blocks/s (8 drafted tokens each); logit HBM GB/s as % of peak (1xB200)"
VERIFY_UNIT = "blocks/s"


def verify_config(args, world: int, nb: int):
    mode = "greedy" if args.temperature == 0 else "rejection sampling, temperature %g" % args.temperature
    return {
        "workload": "verify_block: %d blocks of %d drafted tokens, vocabulary %d, %s"
                    % (args.blocks, VERIFY_K, args.vocab, mode),
        "blocks_per_step": args.blocks, "block_size": VERIFY_K, "vocab": args.vocab,
        "temperature": args.temperature, "parallelism": "replicas x%d" % world,
        "l2": "inputs larger than L2: %d rotating input batches of fp32 logits" % nb,
    }


def run_verify_reference(args):
    """--impl reference --workload verify_block: the float64 oracle on host cores."""
    import oracle

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    tau = args.temperature
    z, w, d, u = datagen.make_verify_inputs(1, VERIFY_K, args.vocab, seed=args.seed)
    times = []
    for i in range(args.warmup + args.steps):  # one block per step: a bounded sample
        t0 = time.perf_counter()
        oracle.verify_block(z, w if tau > 0 else None, d, u, tau)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = len(times) / total
    print(json.dumps({
        "impl": "reference", "metric": VERIFY_METRIC, "value": value, "unit": VERIFY_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": verify_config(args, 1, 1),
        "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": VERIFY_UNIT,
                         "sample": "each step: 1 block through the float64 C oracle, one thread"},
        "e2e": {"value": value, "unit": VERIFY_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_verify(args):
    import torch
    import torch.distributed as dist

    import mxfp4_quantized_moe_router_b200 as mx

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    B, K, V, tau = args.blocks, VERIFY_K, args.vocab, args.temperature
    rows = 2 * K + 1 if tau > 0 else K + 1
    step_bytes = B * rows * V * 4
    nb = max(1, min(args.batches, 1 + (512 << 20) // max(step_bytes, 1)))  # rotate over more than L2
    batches = []
    for i in range(nb):
        z, w, d, u = datagen.make_verify_inputs(B, K, V, seed=replica_input_seed(args.seed, rank, i))
        batches.append((torch.from_numpy(z).to(dev), torch.from_numpy(w).to(dev) if tau > 0 else None,
                        torch.from_numpy(d).to(dev), torch.from_numpy(u).to(dev)))
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    tok = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    ws = torch.empty(max(mx.mxmoe_verify_workspace_size(B, K, V), 1), dtype=torch.uint8, device=dev)
    L = mx.load()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: None if t is None else t.data_ptr()  # noqa: E731

    def step(i, inputs=None, out=None):
        zt, wt, dt, ut = inputs if inputs is not None else batches[i % nb]
        a, t = out if out is not None else (acc, tok)
        rc = L.mxmoe_verify_block(P(zt), P(wt), P(dt), P(ut), B, K, V, tau, P(a), P(t), P(ws), ws.numel(), sp)
        if rc:
            raise RuntimeError("mxmoe_verify_block failed: " + mx.last_error())

    def barrier():
        if world > 1:
            dist.barrier()

    accepted_mean = []
    for i in range(nb):
        step(i)
        torch.cuda.synchronize()
        accepted_mean.append(float(acc.float().mean()))
    clocks = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    for i in range(args.warmup):
        step(i)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    clk = clocks.summary([(t0, t1)])
    # end to end: each step uploads its logits, drafts and uniforms from pinned
    # host memory and downloads the verdicts, copies on their own streams
    # (double-buffered) so that they overlap the neighbouring steps' kernels
    hosts = [tuple(None if x is None else x.cpu().pin_memory() for x in bt) for bt in batches[:2]]
    devs = [tuple(None if x is None else torch.empty_like(x) for x in batches[0]) for _ in range(2)]
    outs = [(torch.empty_like(acc), torch.empty_like(tok)) for _ in range(2)]
    outs_h = [(torch.empty(B, dtype=torch.int32).pin_memory(), torch.empty((B, K + 1), dtype=torch.int32).pin_memory())
              for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
    in_ready, in_free, out_ready, out_free = ev(), ev(), ev(), ev()

    def e2e_step(s):
        j = s & 1
        up.wait_event(in_free[j])
        with torch.cuda.stream(up):
            for dst, src in zip(devs[j], hosts[s % len(hosts)]):
                if dst is not None:
                    dst.copy_(src, non_blocking=True)
        in_ready[j].record(up)
        stream.wait_event(in_ready[j])
        stream.wait_event(out_free[j])
        step(s, devs[j], outs[j])
        in_free[j].record(stream)
        out_ready[j].record(stream)
        down.wait_event(out_ready[j])
        with torch.cuda.stream(down):
            outs_h[j][0].copy_(outs[j][0], non_blocking=True)
            outs_h[j][1].copy_(outs[j][1], non_blocking=True)
        out_free[j].record(down)

    e2e_steps = max(3, min(args.steps, 50))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    up.wait_event(s2)
    for i in range(e2e_steps):
        e2e_step(i)
    for j in range(2):
        stream.wait_event(out_free[j])
    e2.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(s2.elapsed_time(e2), world, dev)
    clocks.stop()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    peak, _, peak_kind = load_peaks()
    ms_step = ms / args.steps
    achieved = step_bytes / (ms_step / 1e3) / 1e9
    line = {
        "metric": VERIFY_METRIC, "value": B * args.steps * world / (ms / 1e3), "unit": VERIFY_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded datagen: peaked fp32 logits, drafts = the drafter's argmax, uniforms)",
        "config": verify_config(args, world, nb),
        "mean_accepted": float(np.mean(accepted_mean)),
        "roofline": {"kernel": "mxmoe_verify_block (all %d kernels of the call)" % (4 if tau > 0 else 2),
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
                     else "fallback 6.65 TB/s",
                     "traffic": None, "unit_ms": ms_step, "algorithmic_bytes_per_launch": step_bytes},
        "clocks": clk,
        "gpu_launches": (4 if tau > 0 else 2) * args.steps,
        "e2e": {"value": B * e2e_steps * world / (ms_e2e / 1e3), "unit": VERIFY_UNIT,
                "h2d_bytes_per_step": step_bytes + B * K * 4 + B * (K + 1) * 4,
                "d2h_bytes_per_step": B * 4 + B * (K + 1) * 4,
                "api": "mxmoe_verify_block with pinned host logits/drafts/uniforms and verdict copies on their own "
                       "streams (double-buffered)"},
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle

        z, w, d, u = datagen.make_verify_inputs(1, K, V, seed=args.seed)
        t_cpu = time.perf_counter()
        n_cpu = 0
        while n_cpu < 3 or time.perf_counter() - t_cpu < 2.0:
            oracle.verify_block(z, w if tau > 0 else None, d, u, tau)
            n_cpu += 1
        v_cpu = n_cpu / (time.perf_counter() - t_cpu)
        line["cpu_baseline"] = {"value": v_cpu, "unit": VERIFY_UNIT, "cores": 1, "kind": "oracle",
                                "sample": "%d single blocks through the float64 C oracle, one thread" % n_cpu}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.workload == "verify_block":
        if args.impl == "reference":
            run_verify_reference(args)
        else:
            run_verify(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
