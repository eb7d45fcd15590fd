"""Benchmark of the fused attention forward (libattn) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of the workload
(for the FP8 workload: Hadamard rotation + quantisation of Q, K, V and the
FP8 attention).  The default workload is the throughput case the headline
target is stated on: B=2, H=16, N=8192, d=128, non-causal, bf16
(``--workload sweep8192c`` is its causal half).  Rank 0 prints one JSON line.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronisation; each step's kernels are timed with CUDA events on the
launching stream, and the L2 cache (126 MB) is flushed by writing a 256 MB
buffer between steps, outside the timed events.  Multi-GPU runs are weak
scaling: every rank runs its own copy of the workload (independent batches,
no data-path collective) and the job time is the max over ranks.

--impl reference times the fp64 CPU oracle on this machine's host cores on a
bounded sample of the same workload (the reference arm; there is no other
implementation of these pages to run).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import attn_inputs as gen  # noqa: E402

METRIC = "attn fwd TFLOP/s (4·B·H·N²·d, causal/2) and % of B200 dense BF16 peak"
GEMM_METRIC = "A@B+C TFLOP/s (2·M·N·K)"
# the small-K A@B+C workload (a separate line, not the attention metric)
GEMM_WORKLOADS = {"gemm_add": dict(M=8192, N=8192, K=128)}
L2_FLUSH_BYTES = 256 << 20
# the configuration the headline target is stated on (BF16, N = 8192, d = 128)
DEFAULT_WORKLOAD = "sweep8192"
# a timed region at least this long runs into the power cap: the sustained
# GEMM peak is then the fair denominator, otherwise the burst one
SUSTAINED_MIN_S = 1.0


def workloads():
    w = {
        "tiny": dict(B=1, Hq=1, Hkv=1, N=128, d=64, causal=False, dtype="bf16"),
        "gpt2": dict(B=8, Hq=12, Hkv=12, N=1024, d=64, causal=True, dtype="bf16"),
        "gqa": dict(B=4, Hq=32, Hkv=8, N=4096, d=128, causal=True, dtype="bf16"),
        "mqa": dict(B=4, Hq=32, Hkv=1, N=4096, d=128, causal=True, dtype="bf16"),
        "d256": dict(B=2, Hq=8, Hkv=8, N=4096, d=256, causal=False, dtype="bf16"),
        "fp8": dict(B=4, Hq=16, Hkv=16, N=8192, d=128, causal=False, dtype="fp8"),
        # decode-shaped (16 query rows against 32K keys), split-KV + combine;
        # HBM-bound: the roofline is the K/V read
        "decode": dict(B=4, Hq=32, Hkv=8, N=32768, Nq=16, d=128, causal=False, dtype="bf16", split=True),
    }
    for n in (512, 1024, 2048, 4096, 8192, 16384):
        for c in (False, True):
            w[f"sweep{n}{'c' if c else ''}"] = dict(B=16384 // n, Hq=16, Hkv=16, N=n, d=128, causal=c, dtype="bf16")
    return w


def n_query(cfg) -> int:
    """Query rows per head (N unless the workload sets Nq); N is the key count."""
    return cfg.get("Nq", cfg["N"])


def flops(cfg) -> float:
    f = 4.0 * cfg["B"] * cfg["Hq"] * n_query(cfg) * cfg["N"] * cfg["d"]
    return f / 2 if cfg["causal"] else f


def describe(name, cfg):
    n = f"N={cfg['N']}" if n_query(cfg) == cfg["N"] else f"Nq={n_query(cfg)} Nk={cfg['N']}"
    return (f"{name}: B={cfg['B']} Hq={cfg['Hq']} Hkv={cfg['Hkv']} {n} d={cfg['d']} "
            f"{'causal' if cfg['causal'] else 'non-causal'} {cfg['dtype']}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(bf16=j["bf16_tflops"], bf16_sustained=j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                    hbm=j["hbm_gbs"], src="measured")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, src="fallback")


def tensor_roofline(achieved, peaks, timed_s, fp8=False):
    """Roofline record of a tensor-bound kernel: the burst peak for a short timed
    region, the sustained one (power-capped) for a region of SUSTAINED_MIN_S or
    more; both fractions are reported."""
    ratio = 2.0 if fp8 else 1.0
    burst, sustained = peaks["bf16"] * ratio, peaks["bf16_sustained"] * ratio
    use_sustained = timed_s >= SUSTAINED_MIN_S
    peak = sustained if use_sustained else burst
    kind = "sustained" if use_sustained else "burst"
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "frac_burst": achieved / burst, "frac_sustained": achieved / sustained,
            "peak_source": f"{peaks['src']} {kind} bf16{' x2 (fp8 nominal ratio)' if fp8 else ''}",
            "timed_region_s": timed_s}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, dev_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.stop_ev, self.thread = period_s, threading.Event(), None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.nv = None

    def _run(self):
        while not self.stop_ev.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:  # noqa: BLE001
            pass

    def __enter__(self):
        if self.nv is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop_ev.set()
            self.thread.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def make_inputs(cfg, seed=gen.BASE_SEED):
    outl = cfg["dtype"] == "fp8"
    return gen.qkv_bf16(cfg["B"], cfg["Hq"], cfg["Hkv"], n_query(cfg), cfg["N"], cfg["d"], seed=seed, outliers=outl)


def _row_flops(cfg, rows):
    nq, nk = n_query(cfg), cfg["N"]
    i = rows % nq
    keys = np.clip(i + (nk - nq) + 1, 0, nk) if cfg["causal"] else np.full(rows.shape, nk)
    return float(np.sum(4.0 * cfg["d"] * keys))


def oracle_sample(cfg, qb, kb, vb, target_s: float, n_rows: int | None = None, seed: int = 0):
    """Times the fp64 oracle on a bounded uniform sample of query rows (all their
    keys).  With n_rows None the sample is grown until one run takes about
    target_s.  Returns (TFLOP/s, description, seconds, n_rows)."""
    import oracle
    B, Hq, d = cfg["B"], cfg["Hq"], cfg["d"]
    total_rows = B * Hq * n_query(cfg)
    q, k, v = gen.bf16_bits_to_f64(qb), gen.bf16_bits_to_f64(kb), gen.bf16_bits_to_f64(vb)
    rng = np.random.default_rng(seed)
    n = min(total_rows, n_rows or 256)
    while True:
        rows = np.sort(rng.choice(total_rows, size=n, replace=False))
        t0 = time.perf_counter()
        oracle.attn_fwd_rows(q, k, v, cfg["causal"], 1.0 / math.sqrt(d), rows)
        dt = time.perf_counter() - t0
        if n_rows is not None or dt >= 0.8 * target_s or n == total_rows:
            break
        n = min(total_rows, max(n * 2, int(n * target_s / max(dt, 1e-3))))
    tf = _row_flops(cfg, rows) / dt / 1e12
    desc = f"{n} of {total_rows} query rows (uniform sample), all their keys, fp64"
    return tf, desc, dt, n


def rank_seed(rank: int) -> int:
    """Input seed of a rank: every rank attends over its own batch (weak scaling)."""
    return gen.BASE_SEED + 1000 * rank


def max_over_ranks(values, device, world: int):
    """Element-wise max of per-rank values (step counts, device times) over the
    job; the only collective of a multi-GPU run, outside every timed region."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return units_per_rank_step * steps * world / (max_ms * 1e-3)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, cfg, name):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    qb, kb, vb = make_inputs(cfg)
    per_step = max(0.5, min(10.0, 60.0 / max(1, args.steps + args.warmup)))
    _, _, _, n_rows = oracle_sample(cfg, qb, kb, vb, per_step)  # size the per-step sample
    vals = []
    desc = ""
    for i in range(args.warmup + args.steps):
        tf, desc, dt, _ = oracle_sample(cfg, qb, kb, vb, per_step, n_rows=n_rows, seed=i)
        if i >= args.warmup:
            vals.append(tf)
    v = float(statistics.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": flops(cfg) / (v * 1e12) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(name, cfg), "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, cfg, name):
    import torch
    import torch.distributed as dist

    import exact_attention_140_b200 as ea

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    B, Hq, Hkv, N, d, causal = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"], cfg["causal"]
    Nq = n_query(cfg)
    scale = 1.0 / math.sqrt(d)
    fp8 = cfg["dtype"] == "fp8"

    qb, kb, vb = make_inputs(cfg, seed=rank_seed(rank))
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (qb, kb, vb)]
    q, k, v = (h.to(dev) for h in host)
    o = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    o_host = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    if fp8:
        signs = torch.from_numpy(gen.hadamard_signs(gen.BASE_SEED + 3, d)).to(dev)
        q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
        k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
        v8 = torch.empty(v.shape, dtype=torch.uint8, device=dev)
        desc = torch.empty(3, dtype=torch.float32, device=dev)
        ws = torch.empty(3 * ea.attn_hadamard_quant_fp8_workspace_bytes(), dtype=torch.uint8, device=dev)
        wsb = ea.attn_hadamard_quant_fp8_workspace_bytes()

        def step(qq, kk, vv):
            ea.attn_hadamard_quant_fp8(qq, q8, desc.data_ptr(), ws.data_ptr(), B * N * Hq, d, signs, stream)
            ea.attn_hadamard_quant_fp8(kk, k8, desc.data_ptr() + 4, ws.data_ptr() + wsb, B * N * Hkv, d, signs,
                                       stream)
            ea.attn_hadamard_quant_fp8(vv, v8, desc.data_ptr() + 8, ws.data_ptr() + 2 * wsb, B * N * Hkv, d, None,
                                       stream)
            ea.attn_fwd_fp8(q8, k8, v8, o, lse, B, Hq, Hkv, N, N, d, causal, scale, desc.data_ptr(),
                            desc.data_ptr() + 4, desc.data_ptr() + 8, stream)
        launches_per_step = 7  # 3 x (amax + quantise) + attention
    elif cfg.get("split"):
        ws_bytes = ea.attn_splitkv_workspace_bytes(B, Hq, Hkv, Nq, N, d, 0)
        ws_split = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

        def step(qq, kk, vv):
            ea.attn_fwd_splitkv(qq, kk, vv, o, lse, B, Hq, Hkv, Nq, N, d, causal, scale, 0, ws_split, ws_bytes,
                                stream)
        launches_per_step = 2 if ws_bytes > 0 else 1  # windows' attention + combine
    else:
        def step(qq, kk, vv):
            ea.attn_fwd(qq, kk, vv, o, lse, B, Hq, Hkv, Nq, N, d, causal, scale, ea.ATTN_BF16, stream)
        launches_per_step = 1

    for _ in range(max(3, args.warmup)):
        step(q, k, v)
    torch.cuda.synchronize()
    if args.steps <= 0:  # size the timed region to about 1.5 s (L2 flush included)
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record(stream)
        for i in range(5):
            flush.fill_(float(i))
            step(q, k, v)
        w1.record(stream)
        torch.cuda.synchronize()
        per = w0.elapsed_time(w1) / 5 * 1e-3
        args.steps = int(max_over_ranks([int(min(20000, max(20, 1.5 / per)))], dev, world)[0])
    rc, word = ea.attn_get_last_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    kstarts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)] if fp8 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record(stream)
            if fp8:
                ea.attn_hadamard_quant_fp8(q, q8, desc.data_ptr(), ws.data_ptr(), B * N * Hq, d, signs, stream)
                ea.attn_hadamard_quant_fp8(k, k8, desc.data_ptr() + 4, ws.data_ptr() + wsb, B * N * Hkv, d, signs,
                                           stream)
                ea.attn_hadamard_quant_fp8(v, v8, desc.data_ptr() + 8, ws.data_ptr() + 2 * wsb, B * N * Hkv, d,
                                           None, stream)
                kstarts[i].record(stream)
                ea.attn_fwd_fp8(q8, k8, v8, o, lse, B, Hq, Hkv, N, N, d, causal, scale, desc.data_ptr(),
                                desc.data_ptr() + 4, desc.data_ptr() + 8, stream)
            else:
                step(q, k, v)
            ends[i].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kern_ms = [s.elapsed_time(e) for s, e in zip(kstarts, ends)] if fp8 else step_ms
    total_ms = float(sum(step_ms))
    rc, word = ea.attn_get_last_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")

    # end to end with host buffers: H2D inputs, kernel(s), D2H outputs.  The bf16
    # forward goes through attn_fwd_host (the C ABI's host-buffer entry point,
    # which pipelines the copies and kernels over chunks of heads); the FP8 and
    # split-KV lines copy around their device entry points.
    e2e_steps = max(3, min(args.steps, 50))
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
    host_path = not fp8 and not cfg.get("split")

    def e2e_step():
        if host_path:
            ea.attn_fwd_host(host[0], host[1], host[2], o_host, lse_host, dq, dk, dv, o, lse, B, Hq, Hkv, Nq, N, d,
                             causal, scale, 0, stream)
            return
        dq.copy_(host[0], non_blocking=True)
        dk.copy_(host[1], non_blocking=True)
        dv.copy_(host[2], non_blocking=True)
        step(dq, dk, dv)
        o_host.copy_(o, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    e2e_step()  # first call creates the pipeline's streams and events
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        e_st[i].record(stream)
        e2e_step()
        e_en[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = float(sum(s.elapsed_time(e) for s, e in zip(e_st, e_en)))

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev, world)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = load_peaks()
    f = flops(cfg)
    value = job_throughput(f, args.steps, world, total_ms) / 1e12
    e2e_value = job_throughput(f, e2e_steps, world, e2e_ms) / 1e12
    kern_avg_s = float(np.mean(kern_ms)) * 1e-3
    achieved = f / kern_avg_s / 1e12
    peak = peaks["bf16"] * (2.0 if fp8 else 1.0)
    traffic = traffic_bytes(name)
    if cfg.get("split"):
        # HBM-bound: algorithmic bytes = Q + K + V read once, O + LSE written once
        alg_bytes = float(sum(x.numel() * x.element_size() for x in (q, k, v, o, lse)))
        roofline = {"bound": "hbm", "achieved": alg_bytes / kern_avg_s / 1e9, "peak": peaks["hbm"], "unit": "GB/s",
                    "frac": alg_bytes / kern_avg_s / 1e9 / peaks["hbm"], "traffic": traffic,
                    "peak_source": f"{peaks['src']} hbm copy", "kernel": "attn_fwd_kernel (key windows) + combine",
                    "algorithmic_bytes": alg_bytes}
    else:
        roofline = tensor_roofline(achieved, peaks, float(np.sum(kern_ms)) * 1e-3, fp8)
        roofline.update(traffic=traffic,
                        kernel="attn_fwd_persistent_kernel" if ea.attn_fwd_schedule(N, d, causal) == 1 else "attn_fwd_kernel")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": {"workload": describe(name, cfg), "global_batch": cfg["B"] * world, "seq_len": N,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed between steps (256 MB write)",
                   "pct_of_peak": round(100.0 * value / world / peak, 2)},
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in host)),
                "d2h_bytes_per_step": int(o.numel() * o.element_size() + lse.numel() * lse.element_size()),
                "api": ("attn_fwd_host (pinned host buffers, copies and kernels pipelined over 8 chunks)"
                        if host_path else "pinned-host copies around the device entry point")},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        tf, desc, dt, _ = oracle_sample(cfg, qb, kb, vb, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                                "sample": desc + f"; {dt:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


def kernel_source_hash() -> str:
    import hashlib
    csrc = os.path.join(ROOT, "exact_attention_140_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(f.encode())
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_bytes(name):
    """DRAM bytes per launch from the committed ncu record, or None when the
    kernel sources changed since it was taken (or the workload has none)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("source_hash") != kernel_source_hash():
        return None
    return rec.get(name)


def run_prep(args, cfg, name):
    """FP8 input preparation alone (Hadamard rotation of Q and K, per-tensor
    amax, E4M3 codes of Q, K, V) on the FP8 workload's tensors: HBM-bound, so
    the line is GB/s of algorithmic bytes (each bf16 input read once, each
    code written once).  --impl reference times the fp64 oracle's preparation
    on a bounded sample of rows."""
    B, Hq, Hkv, N, d = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"]
    rows = [B * N * Hq, B * N * Hkv, B * N * Hkv]
    alg_bytes = float(sum(r * d * 3 for r in rows))  # 2 bytes in + 1 byte out per element
    metric = "FP8 prep GB/s (rotate + amax + E4M3 of Q, K, V; algorithmic bytes)"
    qb, kb, vb = make_inputs(dict(cfg, dtype="fp8"))
    signs_np = gen.hadamard_signs(gen.BASE_SEED + 3, d)

    def oracle_rows(n_rows, seed):
        import oracle
        rng = np.random.default_rng(seed)
        t0 = time.perf_counter()
        for x, rot in ((qb, True), (kb, True), (vb, False)):
            flat = x.reshape(-1, d)
            pick = np.sort(rng.choice(flat.shape[0], size=n_rows, replace=False))
            oracle.fp8_prepare(gen.bf16_bits_to_f64(flat[pick]), signs_np.astype(np.float64) if rot else None)
        dt = time.perf_counter() - t0
        return 3 * n_rows * d * 3 / dt / 1e9, f"{n_rows} rows of each of Q, K, V (uniform sample), fp64; {dt:.1f} s"

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        steps = args.steps if args.steps > 0 else 3
        vals, desc = [], ""
        for i in range(args.warmup + steps):
            v, desc = oracle_rows(20000, i)
            if i >= args.warmup:
                vals.append(v)
        v = float(statistics.median(vals))
        print(json.dumps({
            "impl": "reference", "metric": metric, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": steps,
            "warmup": args.warmup, "ms_per_step": alg_bytes / (v * 1e9) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(name, cfg), "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    import torch
    import torch.distributed as dist

    import exact_attention_140_b200 as ea
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    if rank != 0:
        qb, kb, vb = make_inputs(dict(cfg, dtype="fp8"), seed=rank_seed(rank))
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (qb, kb, vb)]
    xs = [h.to(dev) for h in host]
    x8s = [torch.empty(x.shape, dtype=torch.uint8, device=dev) for x in xs]
    x8_host = [torch.empty(x.shape, dtype=torch.uint8).pin_memory() for x in xs]
    signs = torch.from_numpy(signs_np).to(dev)
    desc = torch.empty(3, dtype=torch.float32, device=dev)
    wsb = ea.attn_hadamard_quant_fp8_workspace_bytes()
    ws = torch.empty(3 * wsb, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step(ins):
        for i, (x, rot) in enumerate(zip(ins, (True, True, False))):
            ea.attn_hadamard_quant_fp8(x, x8s[i], desc.data_ptr() + 4 * i, ws.data_ptr() + i * wsb, rows[i], d,
                                       signs if rot else None, stream)
    for _ in range(max(3, args.warmup)):
        step(xs)
    torch.cuda.synchronize()
    if args.steps <= 0:
        args.steps = 200
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record(stream)
            step(xs)
            ends[i].record(stream)
        torch.cuda.synchronize()
    rc, word = ea.attn_get_last_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")
    total_ms = float(sum(x.elapsed_time(y) for x, y in zip(starts, ends)))
    e2e_steps = max(3, min(args.steps, 20))
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    ds = [torch.empty_like(x) for x in xs]
    for i in range(e2e_steps):
        e_st[i].record(stream)
        for dd, h in zip(ds, host):
            dd.copy_(h, non_blocking=True)
        step(ds)
        for hh, x8 in zip(x8_host, x8s):
            hh.copy_(x8, non_blocking=True)
        e_en[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = float(sum(x.elapsed_time(y) for x, y in zip(e_st, e_en)))
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev, world)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks = load_peaks()
    value = job_throughput(alg_bytes, args.steps, world, total_ms) / 1e9
    kern_s = total_ms / args.steps * 1e-3
    line = {
        "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16->e4m3 (fp32 math)", "data": "synthetic",
        "config": {"workload": describe(name, cfg) + " (prep only)",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed between steps (256 MB write)"},
        "roofline": {"bound": "hbm", "achieved": alg_bytes / kern_s / 1e9, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": alg_bytes / kern_s / 1e9 / peaks["hbm"], "traffic": traffic_bytes(name),
                     "peak_source": f"{peaks['src']} hbm copy", "kernel": "fp8_prep_kernel (amax + quantise passes)",
                     "algorithmic_bytes": alg_bytes},
        "e2e": {"value": job_throughput(alg_bytes, e2e_steps, world, e2e_ms) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in host)),
                "d2h_bytes_per_step": int(sum(x.numel() for x in x8s))},
        "gpu_launches": 6 * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        v, desc_s = oracle_rows(20000, 0)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc_s}
    print(json.dumps(line), flush=True)
    return 0


def run_gemm(args, g, name):
    """D = A B + C (bf16, fp32 accumulation): HBM-bound for small K, so the
    roofline is bytes (A + B + C + D) over time.  --impl reference times the
    fp64 oracle on a bounded sample of rows."""
    M, N, K = g["M"], g["N"], g["K"]
    ab, bb, cb = gen.normal_bf16(11, (M, K)), gen.normal_bf16(12, (K, N)), gen.normal_bf16(13, (M, N))
    f = 2.0 * M * N * K

    def oracle_rows(n_rows, seed):
        import oracle
        rows = np.sort(np.random.default_rng(seed).choice(M, size=n_rows, replace=False))
        a64, b64, c64 = (gen.bf16_bits_to_f64(x) for x in (ab[rows], bb, cb[rows]))
        t0 = time.perf_counter()
        oracle.gemm_add(a64, b64, c64)
        dt = time.perf_counter() - t0
        return 2.0 * n_rows * N * K / dt / 1e12, f"{n_rows} of {M} rows of D (uniform sample), fp64; {dt:.1f} s"

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        steps = args.steps if args.steps > 0 else 3
        vals = []
        desc = ""
        for i in range(args.warmup + steps):
            tf, desc = oracle_rows(256, i)
            if i >= args.warmup:
                vals.append(tf)
        v = float(statistics.median(vals))
        print(json.dumps({
            "impl": "reference", "metric": GEMM_METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": f / (v * 1e12) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{name}: M={M} N={N} K={K} bf16", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    import torch
    import torch.distributed as dist

    import exact_attention_140_b200 as ea
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (ab, bb, cb)]
    a, b, c = (h.to(dev) for h in host)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    d_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step(aa, bb_, cc):
        ea.attn_gemm_add(aa, bb_, cc, d, M, N, K, stream)
    for _ in range(max(3, args.warmup)):
        step(a, b, c)
    torch.cuda.synchronize()
    if args.steps <= 0:
        args.steps = 200
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record(stream)
            step(a, b, c)
            ends[i].record(stream)
        torch.cuda.synchronize()
    rc, word = ea.attn_get_last_device_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")
    step_ms = [x.elapsed_time(y) for x, y in zip(starts, ends)]
    total_ms = float(sum(step_ms))
    e2e_steps = max(3, min(args.steps, 20))
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    da, db, dc = (torch.empty_like(x) for x in (a, b, c))
    for i in range(e2e_steps):
        e_st[i].record(stream)
        da.copy_(host[0], non_blocking=True)
        db.copy_(host[1], non_blocking=True)
        dc.copy_(host[2], non_blocking=True)
        step(da, db, dc)
        d_host.copy_(d, non_blocking=True)
        e_en[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = float(sum(x.elapsed_time(y) for x, y in zip(e_st, e_en)))
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev, world)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks = load_peaks()
    value = job_throughput(f, args.steps, world, total_ms) / 1e12
    kern_s = total_ms / args.steps * 1e-3
    alg_bytes = float(sum(x.numel() * x.element_size() for x in (a, b, c, d)))
    line = {
        "metric": GEMM_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{name}: M={M} N={N} K={K} bf16 (D = A B + C)",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed between steps (256 MB write)"},
        "roofline": {"bound": "hbm", "achieved": alg_bytes / kern_s / 1e9, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": alg_bytes / kern_s / 1e9 / peaks["hbm"], "traffic": traffic_bytes(name),
                     "peak_source": f"{peaks['src']} hbm copy", "kernel": "gemm_add_kernel",
                     "algorithmic_bytes": alg_bytes},
        "e2e": {"value": job_throughput(f, e2e_steps, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in host)),
                "d2h_bytes_per_step": int(d.numel() * d.element_size())},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        tf, desc = oracle_rows(256, 0)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0 = enough for about 1.5 s)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads()) + sorted(GEMM_WORKLOADS) + ["fp8prep"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.workload in GEMM_WORKLOADS:
        return run_gemm(args, GEMM_WORKLOADS[args.workload], args.workload)
    if args.workload == "fp8prep":
        return run_prep(args, workloads()["fp8"], args.workload)
    cfg = workloads()[args.workload]
    if args.impl == "reference":
        if args.steps <= 0:
            args.steps = 3
        return run_reference(args, cfg, args.workload)
    return run_ours(args, cfg, args.workload)


if __name__ == "__main__":
    sys.exit(main())
