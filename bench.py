#!/usr/bin/env python
"""Benchmark of the GPTQ layer quantizer (sm_100a) on synthetic Llama-shaped layers.

One step = the whole hot path on one layer: H = 2 X^T X over the calibration
tokens, damping / act-order / inverse factor, the column walk with OBQ
feedback and lazy updates, and code packing.  Inputs are resident in HBM when
the timed region starts; each step is timed with CUDA events on the launching
stream, with the working copy of W restored and L2 flushed between steps
(outside the events).  Each stage's launches are captured once in a CUDA graph
after the warm-up and replayed (--no-graph: launched on the stream).  Multi-GPU runs are independent replicas (one layer per
rank, no collective on the data path): weak scaling, max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama7b_q_proj]

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "GPTQ layer quantize: weights/s and ms/layer (4-bit g128); Hessian TFLOP/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# dram__bytes_read.sum + dram__bytes_write.sum of one Hessian launch at 65,536
# tokens x 4,096 (ncu, current kernel: 256 x 256 blocks as two MMA halves
# sharing B, 32,768-token drains, eight drain warps): 608.4 MB read + 40.1 MB
# written
TRAFFIC_65K = 648.5e6


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama7b_q_proj")
    p.add_argument("--tokens", type=int, default=None,
                   help="override the calibration token count (profiling of a smaller case)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="launch each stage on the stream instead of replaying captured CUDA graphs")
    p.add_argument("--dequant-matmul", type=int, default=0, metavar="TOKENS",
                   help="instead of the quantizer step, time the product of TOKENS tokens with a "
                        "quantized Llama-70B down_proj (gptq_dequant_matmul)")
    p.add_argument("--dequant-gemm", type=int, default=0, metavar="TOKENS",
                   help="instead of the quantizer step, time the many-token product of TOKENS "
                        "tokens with a quantized Llama-70B down_proj (gptq_dequant_gemm, tcgen05)")
    p.add_argument("--hessian-only", action="store_true",
                   help="instead of the whole step, time the Hessian stage alone (X and H only on "
                        "the device: the profiling case for large d_col)")
    p.add_argument("--gemm-peaks", action="store_true",
                   help="instead of the quantizer step, measure the library-GEMM denominators of the "
                        "fp32 stages: cuBLAS 8192^3 fp32 with TF32 tensor cores and with plain FFMA")
    return p.parse_args()


def run_gemm_peaks():
    """cuBLAS (through torch.matmul) 8192^3 fp32 products, best of 10 after
    3 warm-up: with TF32 tensor cores allowed (the kind::tf32 roof of the
    3xTF32 GEMMs, which run three MMAs per product) and without (the FFMA
    roof of an fp32-exact SIMT product)."""
    n = 8192
    a = torch.randn(n, n, device="cuda")
    b = torch.randn(n, n, device="cuda")
    c = torch.empty(n, n, device="cuda")
    out = {}
    for name, tf32 in (("tf32_tflops", True), ("fp32_ffma_tflops", False)):
        torch.backends.cuda.matmul.allow_tf32 = tf32
        for _ in range(3):
            torch.matmul(a, b, out=c)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        out[name] = 2 * n ** 3 / (best * 1e-3) / 1e12
    torch.backends.cuda.matmul.allow_tf32 = False
    print(json.dumps({"gemm_peaks": out, "how": "torch.matmul fp32 8192^3, best of 10 (burst)",
                      "gpu": torch.cuda.get_device_name()}), flush=True)


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- replicas
# The layers of a model are independent quantization problems, so N GPUs run
# N replicas: rank k quantizes its own layer (seed offset k) with no
# collective on the data path.  The step time is the slowest rank's; the
# job's throughput counts every rank's weights.
def replica_seed_offset(rank: int) -> int:
    return int(rank)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest per-rank value (a device-timed step: the job waits for the
    slowest rank).  All ranks call it; all get the maximum."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_weights_per_s(world: int, d_row: int, d_col: int, ms_max: float) -> float:
    """Whole-job throughput: every rank quantizes one d_row x d_col layer per
    step, and a step lasts as long as the slowest rank's."""
    return world * d_row * d_col / (ms_max / 1e3)


# ---------------------------------------------------------------- clocks
_SAMPLER_SRC = r"""
import select, sys, time
import pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1].encode())
period = float(sys.argv[2])
print("ready", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
out = []
while not select.select([sys.stdin], [], [], period)[0]:
    try:
        out.append((time.monotonic(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                    pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
    except Exception:
        pass
for t, mhz, mask in out:
    print(t, mhz, mask)
"""


class ClockSampler:
    """SM clock and clock-event reasons through NVML, sampled every few ms by
    a separate process (a thread of this one would wait for the interpreter
    lock while the main thread blocks in a device synchronize).  Samples are
    kept between start() and stop()."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        import subprocess
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.error = None
        self.t0 = self.t1 = None
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_SRC, uuid, str(period_s)],
                                         stdin=subprocess.PIPE, stdout=subprocess.PIPE,
                                         stderr=subprocess.PIPE, text=True)
            import select
            if not select.select([self.proc.stdout], [], [], 30.0)[0]:
                raise RuntimeError("clock sampler did not report within 30 s")
            first = self.proc.stdout.readline().split()
            if len(first) != 2 or first[0] != "ready":
                raise RuntimeError("clock sampler did not start: "
                                   + self.proc.stderr.read()[-300:].strip())
            self.max_mhz = int(first[1])
        except Exception as exc:  # NVML missing: report that, do not guess
            self.error = repr(exc)
            if self.proc is not None and self.proc.poll() is None:
                self.proc.kill()
            self.proc = None

    def start(self):
        self.t0 = time.monotonic()

    def stop(self):
        self.t1 = time.monotonic()
        if self.proc is None:
            return
        try:
            out, _ = self.proc.communicate(input="", timeout=30)
        except Exception as exc:
            self.proc.kill()
            self.error = repr(exc)
            return
        for ln in out.splitlines():
            t, mhz, mask = ln.split()
            if self.t0 <= float(t) <= self.t1:
                self.samples.append(int(mhz))
                for bit, name in self.REASONS.items():
                    if int(mask) & bit:
                        self.reasons.add(name)

    def summary(self):
        if self.proc is None and self.max_mhz is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_min_mhz": min(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "period_ms": 5}


# ---------------------------------------------------------------- oracle timing
_SAMPLES: dict = {}


def oracle_sample(wl: workloads.Workload, seed_offset: int = 0, n_tokens: int = 32768,
                  n_rows: int = 256) -> dict:
    """Time the float64 oracle on a bounded sample of one full-width layer:
    H = 2 X^T X over a token sample, the dead-column / act-order / damping
    step and the inverse factor U (library Cholesky and triangular inverse of
    the flipped matrix) at the full d_col, and the OBQ column loop driven by
    U's rows on a row sample.  The oracle's work is linear in the tokens (H)
    and in the rows (the column loop) and has no other sampled dimension, so
    the full layer's time is t_H (N / n) + t_U + t_rows (R / r)."""
    import oracle
    n_s = min(wl.n_tokens, n_tokens)
    r_s = min(wl.d_row, n_rows)
    key = (wl.name, n_s, r_s, seed_offset)
    if key not in _SAMPLES:  # the inputs are drawn once (not timed)
        _SAMPLES.clear()
        _SAMPLES[key] = (workloads.activations(wl, n_tokens=n_s, seed_offset=seed_offset),
                         workloads.gaussian_weights(r_s, wl.d_col, wl.w_std, wl.seed))
    X, W = _SAMPLES[key]
    t0 = time.perf_counter()
    H = oracle.hessian(X)
    t_h = time.perf_counter() - t0
    t0 = time.perf_counter()
    prep = oracle.prepare(H, W, damp=wl.damp, desc_act=wl.desc_act)
    U = oracle.upper_factor_flip(prep["H_damped"])
    t_u = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.gptq_columns_u(prep["W0"], U, wl.bits, wl.group_size)
    t_r = time.perf_counter() - t0
    total = t_h * wl.n_tokens / n_s + t_u + t_r * wl.d_row / r_s
    spent = t_h + t_u + t_r
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return dict(value=wl.d_row * wl.d_col / total, seconds_extrapolated=total, spent=spent,
                cores=cores, fraction=spent / total,
                sample=(f"oracle (numpy/LAPACK + C, float64, OpenMP): H on {n_s} of {wl.n_tokens} "
                        f"tokens (x{wl.n_tokens / n_s:g}), the full {wl.d_col}^2 inverse factor, "
                        f"the column loop on {r_s} of {wl.d_row} rows (x{wl.d_row / r_s:g}); "
                        f"{spent:.1f} s of host work for {spent / total:.3f} of a layer"))


def run_reference(args, rank: int, world: int):
    """The oracle timed as it stands (no GPU work).  Each step is a bounded
    sample of the layer (oracle_sample); ms_per_step is the wall time the
    step really took, value the layer throughput those measured parts imply
    (the extrapolation is labelled in the line)."""
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_sample(wl)
    vals, spent, frac = [], [], []
    last = None
    for _ in range(args.steps):
        last = oracle_sample(wl)
        vals.append(last["value"])
        spent.append(last["spent"])
        frac.append(last["fraction"])
    value = statistics.mean(vals)
    ms = statistics.mean(spent) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "weights/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(wl, world),
            "extrapolation": {"layer_fraction_per_step": statistics.mean(frac),
                              "full_layer_ms": wl.d_row * wl.d_col / value * 1e3,
                              "how": "t_H (tokens / sampled tokens) + t_U + t_rows (rows / sampled rows)"},
            "cpu_baseline": {"value": value, "unit": "weights/s", "cores": last["cores"],
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(wl, world):
    return {"workload": wl.name, "d_row": wl.d_row, "d_col": wl.d_col, "tokens": wl.n_tokens,
            "bits": wl.bits, "group_size": wl.group_size, "desc_act": wl.desc_act,
            "damp": wl.damp, "block": wl.block_size, "parallelism": f"replicas{world}",
            "l2": "flushed between steps (256 MiB write); X (2 bytes x tokens x d_col) is larger "
                  "than L2"}


# ---------------------------------------------------------------- our path
def run_ours(args, rank: int, world: int, dist):
    import post_weight_quantization_gptq_b200 as g

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens:
        wl = dataclasses.replace(wl, n_tokens=args.tokens)
    r, d, n = wl.d_row, wl.d_col, wl.n_tokens
    cfg = g.GPTQConfig(bits=wl.bits, group_size=wl.group_size, desc_act=wl.desc_act, damp=wl.damp)

    X = workloads.activations(wl, device=dev, seed_offset=replica_seed_offset(rank))
    W0 = workloads.weights(wl, device=dev, seed_offset=replica_seed_offset(rank))
    W = torch.empty_like(W0)
    H = torch.empty(d, d, dtype=torch.float32, device=dev)
    U = torch.empty(d, d, dtype=torch.float32, device=dev)
    perm = torch.empty(d, dtype=torch.int32, device=dev)
    dead = torch.empty(d, dtype=torch.uint8, device=dev)
    ng = g.n_groups(d, wl.group_size)
    codes = torch.empty(r, d, dtype=torch.uint8, device=dev)
    scales = torch.empty(ng, r, dtype=torch.float32, device=dev)
    zeros = torch.empty(ng, r, dtype=torch.int32, device=dev)
    packed = torch.empty(r, g.packed_words(d, wl.bits), dtype=torch.int32, device=dev)
    ws = torch.empty(g.gptq_workspace_size(cfg, r, d), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        H.zero_()
        g.gptq_hessian_accumulate(X, H, st)
        if ev is not None:
            ev[0].record(stream)
        g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
        if ev is not None:
            ev[1].record(stream)
        g.gptq_quantize_layer(W, U, perm, dead, cfg, codes, scales, zeros, st, ws)
        if ev is not None:
            ev[2].record(stream)
        g.gptq_pack(codes, wl.bits, packed)

    def between():
        W.copy_(W0)
        flush.fill_(1)

    for _ in range(args.warmup):
        between()
        step()
    status = g.gptq_sync_status(st)
    if status != 0:
        raise RuntimeError(f"device status {g.STATUS.get(status, status)} during warm-up")

    # Each stage's launch sequence (hundreds of dependent kernels in prepare_hinv,
    # with their cross-stream events) is captured once in a CUDA graph and
    # replayed in the timed steps; the library's side streams join the capture
    # through its events.  Their one-time set-up ran in the warm-up above.
    stages = [lambda: g.gptq_hessian_accumulate(X, H, st),
              lambda: g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws),
              lambda: g.gptq_quantize_layer(W, U, perm, dead, cfg, codes, scales, zeros, st, ws),
              lambda: g.gptq_pack(codes, wl.bits, packed)]
    launches_per_step = None
    if not args.no_graph:
        between()
        H.zero_()
        torch.cuda.synchronize(dev)
        graphs = []
        l0 = g.gptq_launch_counter()
        for fn in stages:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, capture_error_mode="thread_local"):
                fn()
            graphs.append(gr)
        launches_per_step = g.gptq_launch_counter() - l0  # kernels in the captured graphs
        torch.cuda.synchronize(dev)
        stages = [gr.replay for gr in graphs]

    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_h0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_mid = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clocks = ClockSampler(dev.index)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = g.gptq_launch_counter()
    clocks.start()
    for k in range(K):
        between()
        ev_s[k].record(stream)
        H.zero_()
        ev_h0[k].record(stream)
        stages[0]()
        ev_mid[k][0].record(stream)
        stages[1]()
        ev_mid[k][1].record(stream)
        stages[2]()
        ev_mid[k][2].record(stream)
        stages[3]()
        ev_e[k].record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clocks.stop()
    launches = (g.gptq_launch_counter() - launches0) / K if launches_per_step is None else launches_per_step
    status = g.gptq_sync_status(st)
    if status != 0:
        raise RuntimeError(f"device status {g.STATUS.get(status, status)} in the timed steps")

    step_ms = [ev_s[k].elapsed_time(ev_e[k]) for k in range(K)]
    hess_ms = [ev_h0[k].elapsed_time(ev_mid[k][0]) for k in range(K)]
    prep_ms = [ev_mid[k][0].elapsed_time(ev_mid[k][1]) for k in range(K)]
    quant_ms = [ev_mid[k][1].elapsed_time(ev_mid[k][2]) for k in range(K)]
    pack_ms = [ev_mid[k][2].elapsed_time(ev_e[k]) for k in range(K)]
    ms = statistics.mean(step_ms)
    ms_max = max_over_ranks(ms, dist, dev)

    # ------------------------------------------------ end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        Xh = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
        Xh.copy_(X)
        Wh = torch.empty(W0.shape, dtype=W0.dtype, pin_memory=True)
        Wh.copy_(W0)
        ph = torch.empty(packed.shape, dtype=packed.dtype, pin_memory=True)
        sh = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
        zh = torch.empty(zeros.shape, dtype=zeros.dtype, pin_memory=True)
        Ke = max(2, min(K, 5))
        # X streams from pinned host memory through a two-slot staging buffer
        # (copies overlap the Hessian GEMM); W's copy runs on a second stream
        # beside it and is waited for before the column walk
        staging = torch.empty(g.gptq_hessian_staging_size(d, 32768), dtype=torch.uint8,
                              device=dev)
        wcopy = torch.cuda.Stream(dev)

        def e2e_step(e0=None, e1=None):
            flush.fill_(1)
            if e0 is not None:
                e0.record(stream)
            wcopy.wait_stream(stream)
            with torch.cuda.stream(wcopy):
                W.copy_(Wh, non_blocking=True)
            H.zero_()
            g.gptq_hessian_accumulate_host(Xh, H, staging, st)
            g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
            stream.wait_stream(wcopy)
            g.gptq_quantize_layer(W, U, perm, dead, cfg, codes, scales, zeros, st, ws)
            g.gptq_pack(codes, wl.bits, packed)
            ph.copy_(packed, non_blocking=True)
            sh.copy_(scales, non_blocking=True)
            zh.copy_(zeros, non_blocking=True)
            if e1 is not None:
                e1.record(stream)

        e2e_step()  # warm-up: the library's copy stream and events are created here
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
        for k in range(Ke):
            e2e_step(e_s[k], e_e[k])
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(statistics.mean(e_s[k].elapsed_time(e_e[k]) for k in range(Ke)),
                              dist, dev)
        if g.gptq_sync_status(st) != 0:
            raise RuntimeError("device status error in the end-to-end steps")
        e2e = {"value": job_weights_per_s(world, r, d, e_ms), "unit": "weights/s",
               "h2d_bytes_per_step": X.numel() * X.element_size() + W0.numel() * 4,
               "d2h_bytes_per_step": packed.numel() * 4 + scales.numel() * 4 + zeros.numel() * 4,
               "ms_per_step": e_ms}

    if rank != 0:
        return
    pk, which = peaks()
    hess_flops = n * d * (d + 1)
    # DRAM traffic of one Hessian launch from ncu (one launch at 65,536 tokens,
    # d = 4,096); X reads and the per-32k-token drains both grow with the tokens.
    traffic = (TRAFFIC_65K * n / 65536
               if (TRAFFIC_65K is not None and d == 4096 and n % 32768 == 0) else None)
    h_ms = statistics.mean(hess_ms)
    achieved = hess_flops / (h_ms / 1e3) / 1e12
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    stages = stage_rooflines(wl, pk, which, {"hessian": h_ms, "prepare_hinv": statistics.mean(prep_ms),
                                             "quantize_layer": statistics.mean(quant_ms),
                                             "pack": statistics.mean(pack_ms)}, ms)
    line = {
        "metric": METRIC, "value": job_weights_per_s(world, r, d, ms_max), "unit": "weights/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16-in/fp32", "data": "synthetic (seeded; Student-t / half-normal activations "
                                         "with outlier channels, Gaussian weights)",
        "config": _config(wl, world),
        "ms_per_layer": ms_max,
        "hessian_tflops": achieved,
        # the same launch counted as a dense d x d product (2 n d^2 flop), for
        # comparison with GEMM figures; the roofline uses the algorithmic count
        "hessian_tflops_dense_equivalent": 2.0 * n * d * d / (h_ms / 1e3) / 1e12,
        "stage_ms": {"hessian": h_ms, "prepare_hinv": statistics.mean(prep_ms),
                     "quantize_layer": statistics.mean(quant_ms), "pack": statistics.mean(pack_ms)},
        "quantize_only_weights_per_s": r * d / ((ms - h_ms) / 1e3),
        "roofline": {"kernel": "hessian_syrk_tcgen05", "bound": "tensor", "achieved": achieved,
                     "peak": peak, "peak_source": f"{which} bf16 dense (burst)", "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "algorithmic": f"n*d*(d+1) = {hess_flops:.4e} flop per launch"},
        "stage_rooflines": stages,
        "gpu_launches": launches,
        "launch": "stream" if args.no_graph else "CUDA graphs (one per stage, captured once)",
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        # a larger sample than the per-step one of --impl reference: about
        # 10-30 s of host work in one measurement
        cb = oracle_sample(wl, n_tokens=131072, n_rows=1024)
        line["cpu_baseline"] = {"value": cb["value"], "unit": "weights/s", "cores": cb["cores"],
                                "kind": "oracle", "sample": cb["sample"]}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- stage rooflines
# Nominal dense tf32 / bf16 tensor ratio (1.1 / 2.25 PFLOP/s): the tf32 peak
# is the measured bf16 one times this ratio; a 3xTF32 product issues three
# tf32 MMAs per fp32-accurate product.  FFMA: 148 SMs x 128 lanes x 2 flop x
# the 1.965 GHz maximum SM clock.
TF32_PER_BF16 = 1.1 / 2.25
FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def stage_rooflines(wl, pk, which, stage_ms, layer_ms):
    """Each stage's algorithmic work, the time its bound allows, and the
    fraction of that bound the measured stage reaches; their sum is the
    layer's roofline."""
    r, d, n, b = wl.d_row, wl.d_col, wl.n_tokens, wl.bits
    bf16 = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tf32x3 = bf16 * TF32_PER_BF16 / 3.0
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    B = wl.block_size
    nb = -(-d // B)
    # lazy update: sum over blocks of 2 r B (d - end of block) flop
    lazy = sum(2.0 * r * min(B, d - B * k) * max(0, d - B * (k + 1)) for k in range(nb))
    walk = float(r) * d * B  # in-block feedback, r d B flop
    rows = {
        "hessian": dict(bound="tensor (bf16)", work=f"n d (d+1) = {n * d * (d + 1):.3e} flop",
                        bound_ms=n * d * (d + 1) / (bf16 * 1e12) * 1e3,
                        peak=f"{bf16:g} TFLOP/s bf16 dense ({which})"),
        "prepare_hinv": dict(bound="tensor (3xTF32)", work=f"2/3 d^3 = {2 * d ** 3 / 3:.3e} flop",
                             bound_ms=(2.0 * d ** 3 / 3) / (tf32x3 * 1e12) * 1e3,
                             peak=f"{tf32x3:.1f} TFLOP/s fp32-accurate = {which} bf16 x "
                                  f"{TF32_PER_BF16:.3f} (nominal tf32/bf16) / 3 MMAs"),
        "quantize_layer": dict(bound="tensor (3xTF32) + alu (FFMA)",
                               work=f"lazy update {lazy:.3e} flop + column walk r d B = {walk:.3e} flop",
                               bound_ms=(lazy / (tf32x3 * 1e12) + walk / (FFMA_TFLOPS * 1e12)) * 1e3,
                               peak=f"{tf32x3:.1f} TFLOP/s 3xTF32; {FFMA_TFLOPS:.1f} TFLOP/s FFMA "
                                    f"(148 SMs x 128 x 2 x 1.965 GHz)"),
        "pack": dict(bound="hbm", work=f"r d (1 + b/8) = {r * d * (1 + b / 8):.3e} bytes",
                     bound_ms=r * d * (1 + b / 8) / (hbm * 1e9) * 1e3,
                     peak=f"{hbm:g} GB/s HBM copy ({which})"),
    }
    total_bound = 0.0
    for name, row in rows.items():
        row["measured_ms"] = stage_ms[name]
        row["frac"] = row["bound_ms"] / stage_ms[name] if stage_ms[name] > 0 else None
        total_bound += row["bound_ms"]
    return {"stages": rows, "sum_bound_ms": total_bound, "layer_ms": layer_ms,
            "layer_frac_of_summed_bound": total_bound / layer_ms}


# ---------------------------------------------------------------- Hessian alone
def run_hessian_only(args, rank: int, world: int, dist):
    """H = 2 X^T X of the workload (token count from --tokens), timed alone:
    only X and H live on the device."""
    import post_weight_quantization_gptq_b200 as g

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens:
        wl = dataclasses.replace(wl, n_tokens=args.tokens)
    n, d = wl.n_tokens, wl.d_col
    X = workloads.activations(wl, device=dev, seed_offset=replica_seed_offset(rank))
    H = torch.empty(d, d, dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        H.zero_()
        g.gptq_hessian_accumulate(X, H, st)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(dev.index)
    torch.cuda.synchronize(dev)
    clocks.start()
    for k in range(K):
        flush.fill_(1)
        H.zero_()
        ev[k][0].record(stream)
        g.gptq_hessian_accumulate(X, H, st)
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    if g.gptq_sync_status(st) != 0:
        raise RuntimeError("device status error in the timed Hessians")
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), dist, dev)
    if rank != 0:
        return
    pk, which = peaks()
    flops = n * d * (d + 1)
    tf = flops / (ms / 1e3) / 1e12
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    print(json.dumps({
        "metric": "Hessian H = 2 X^T X: TFLOP/s (n d (d+1) flop)", "value": world * tf,
        "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16-in/fp32",
        "data": "synthetic", "config": {"workload": wl.name + "_hessian", "d_col": d, "tokens": n,
                                        "x_bytes": 2 * n * d},
        "roofline": {"kernel": "hessian_syrk_tcgen05", "bound": "tensor", "achieved": tf,
                     "peak": peak, "peak_source": f"{which} bf16 dense (burst)", "unit": "TFLOP/s",
                     "frac": tf / peak, "traffic": None},
        "clocks": clocks.summary()}), flush=True)


# ---------------------------------------------------------------- the product
def run_dequant_matmul(args, rank: int, world: int, dist):
    """Y = X W_hat^T for a quantized 8192 x 28672 layer (4-bit, g128, act-order):
    the decode form (HBM-bound on the packed words for one token), or with
    --dequant-gemm the many-token form on the tensor cores (bf16 dense
    contraction, 2 tokens x d_row x d_col flop)."""
    import post_weight_quantization_gptq_b200 as g

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    gemm = args.dequant_gemm > 0
    n_tok = args.dequant_gemm if gemm else args.dequant_matmul
    d_row, d_col, bits, gs = 8192, 28672, 4, 128
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321 + rank)
    ng = d_col // gs
    packed = torch.randint(-(1 << 31), 1 << 31, (d_row, d_col * bits // 32), dtype=torch.int64,
                           device=dev, generator=gen).to(torch.int32)
    scales = torch.rand(ng, d_row, device=dev, generator=gen) * 0.02 + 1e-3
    zeros = torch.randint(0, 1 << bits, (ng, d_row), dtype=torch.int32, device=dev, generator=gen)
    perm = torch.randperm(d_col, device=dev, generator=gen).to(torch.int32)
    X = torch.randn(n_tok, d_col, device=dev, generator=gen).to(torch.bfloat16)
    Y = torch.empty(n_tok, d_row, dtype=torch.float32, device=dev)
    wsz = (g.gptq_dequant_gemm_workspace_size if gemm else g.gptq_dequant_matmul_workspace_size)(
        n_tok, d_col)
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def product():
        if gemm:
            g.gptq_dequant_gemm(X, packed, scales, zeros, perm, bits, gs, Y, ws, st)
        else:
            g.gptq_dequant_matmul(X, packed, scales, zeros, perm, bits, gs, Y, ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        product()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(dev.index)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = g.gptq_launch_counter()
    clocks.start()
    for k in range(K):
        flush.fill_(1)
        ev[k][0].record(stream)
        product()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clocks.stop()
    launches = (g.gptq_launch_counter() - launches0) / K
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_max = max_over_ranks(ms, dist, dev)
    kernel_ms = None
    if gemm:
        # the contraction kernel alone (the activations already in
        # quantization order: no gather launch), for its roofline
        kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        for k in range(K):
            flush.fill_(1)
            kev[k][0].record(stream)
            g.gptq_dequant_gemm(X, packed, scales, zeros, None, bits, gs, Y, ws, st)
            kev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        kernel_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in kev), dist, dev)
    if rank != 0:
        return
    if g.gptq_sync_status(st) != 0:
        raise RuntimeError("device status error in the timed products")
    pk, which = peaks()
    nbytes = (d_row * d_col * bits // 8 + 8 * ng * d_row + 2 * n_tok * d_col + 4 * d_col
              + 4 * n_tok * d_row)
    gbs = nbytes / (ms / 1e3) / 1e9
    peak = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    if gemm:
        flops = 2.0 * n_tok * d_row * d_col
        tf = flops / (kernel_ms / 1e3) / 1e12
        bpk = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        roof = {"kernel": "dequant_gemm_kernel", "bound": "tensor", "achieved": tf, "peak": bpk,
                "peak_source": f"{which} bf16 dense (burst)", "unit": "TFLOP/s", "frac": tf / bpk,
                "traffic": None, "kernel_ms": kernel_ms, "gather_ms": ms_max - kernel_ms,
                "algorithmic": f"2 tokens d_row d_col = {flops:.4e} flop (bf16 operands, fp32 sums)"}
    else:
        roof = {"kernel": "dequant_matmul_kernel", "bound": "hbm", "achieved": gbs,
                "peak": peak, "peak_source": f"{which} HBM copy", "unit": "GB/s",
                "frac": gbs / peak, "traffic": None,
                "algorithmic": f"packed codes + scales + zeros + X + perm + Y = {nbytes} bytes"}
    line = {
        "metric": f"dequantized product with a quantized layer ({n_tok} token(s)): weights/s",
        "value": world * d_row * d_col / (ms_max / 1e3), "unit": "weights/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16-in/fp32",
        "data": "synthetic (seeded random codes, scales, zeros, act-order permutation)",
        "config": {"workload": "llama70b_down_proj_dequant_" + ("gemm" if gemm else "matmul"),
                   "d_row": d_row, "d_col": d_col,
                   "tokens": n_tok, "bits": bits, "group_size": gs, "desc_act": True,
                   "l2": "flushed between steps (256 MiB write)"},
        "roofline": roof,
        "gpu_launches": launches, "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    if args.gemm_peaks:
        run_gemm_peaks()
        return
    try:
        if args.dequant_matmul > 0 or args.dequant_gemm > 0:
            run_dequant_matmul(args, rank, world, dist)
        elif args.hessian_only:
            run_hessian_only(args, rank, world, dist)
        else:
            run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
