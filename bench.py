"""Benchmark of the hot path: exact attention forward (fa_fwd) then backward (fa_bwd).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = fa_fwd + fa_bwd on one batch of synthetic inputs already resident in device
memory (the default workload is B=2, H=16, N=8192, d=128, causal, bf16).  The value is
credited TFLOP/s: forward 4*B*H*N^2*d plus backward 10*B*H*N^2*d, halved for causal, per
second of device time, summed over ranks.  Under torchrun every rank runs the same
workload on its own GPU (replicas of independent heads: weak scaling, no data-path
collective); the time is the max over ranks.

Rank 0 prints one JSON line.  Besides the contract keys it carries:
  roofline      the dominant kernel's achieved TFLOP/s against the measured bf16 peak
  cpu_baseline  the fp64 oracle timed on this host on a bounded sample (rank 0, N=1)
  e2e           the same metric with host buffers: pinned host -> device copies of the
                inputs, fa_fwd, fa_bwd and device -> host copies of the results, all
                inside the timed region; pipelined over three streams (uploads, compute,
                downloads), with the one-stream figure beside it ("serial") and the
                time of the same copies alone, both directions at once
                ("copy_floor_ms": no pipelined step can be faster)
  clocks        SM clocks and throttle reasons sampled during the timed region
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_64_b200 import dist as fa_dist  # noqa: E402
from exact_io_aware_64_b200 import inputs as fa_inputs  # noqa: E402
from exact_io_aware_64_b200 import traffic  # noqa: E402

DEFAULT_WORKLOAD = "n8192_d128_causal_bwd"
METRIC = "attention TFLOP/s (fwd, bwd) vs N and % of B200 dense BF16 peak, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_NAMES_BF16 = ("fwd_sm100_kernel", "bwd_prep_kernel", "bwd_dkdv_kernel", "bwd_dq_kernel")
KERNEL_NAMES_F32 = ("fwd_f32_kernel", "bwd_f32_prep_kernel", "bwd_f32_dkdv_kernel",
                    "bwd_f32_dq_kernel")
# float32 FMA on the CUDA cores: 148 SMs x 128 lanes x 2 FLOP per clock at 1965 MHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

KERNEL_SOURCES = {
    "fwd_sm100_kernel": ("fwd_sm100.cu", "sm100.cuh"),
    "bwd_prep_kernel": ("bwd_sm100.cu", "sm100.cuh"),
    "bwd_dkdv_kernel": ("bwd_sm100.cu", "sm100.cuh"),
    "bwd_dq_kernel": ("bwd_sm100.cu", "sm100.cuh"),
}


def kernel_digest(kernel: str) -> str:
    """Hash of the sources that define `kernel` (its translation unit and the sm_100a
    primitives it includes)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_64_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel's current sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_SOURCES:
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_digest") != kernel_digest(kernel):
        return None
    return e.get("bytes_per_launch")


def add_rates(kernels: dict) -> dict:
    """Per-kernel rates from mean launch times: TFLOP/s for kernels credited with FLOPs
    (and executed TFLOP/s where the executed work differs), GB/s for the ones credited
    with bytes."""
    for kinfo in kernels.values():
        sec = kinfo["ms"] * 1e-3
        if "flops" in kinfo:
            kinfo["tflops"] = kinfo["flops"] / sec / 1e12
        else:
            kinfo["gbs"] = kinfo["bytes"] / sec / 1e9
        if "executed_flops" in kinfo:
            kinfo["executed_tflops"] = kinfo["executed_flops"] / sec / 1e12
    return kernels


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.seek(0)
        rows = [r.strip().split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                power.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        loaded = [s for s, p in zip(sm, power) if p > 200.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def config_dict(w, with_bwd: bool, world: int) -> dict:
    """The workload as both arms name it in their JSON line."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "step": "fa_fwd + fa_bwd" if with_bwd else "fa_fwd",
            "l2": "inputs larger than L2 (no flush)" if w.B * w.H * w.N * w.d * 2 > (126 << 20)
            else "inputs smaller than L2 (resident between steps)",
            "parallelism": f"replicas x{world} (independent heads per GPU)"}


def step_flops(w) -> float:
    return traffic.fwd_flops(w.B, w.H, w.N, w.d, w.causal) + \
        traffic.bwd_flops(w.B, w.H, w.N, w.d, w.causal)


# ------------------------------------------------------------------ CPU oracle timing
def time_oracle(w, max_seconds: float = 20.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the forward
    and backward of whole heads (b, h) = (0, 0), (0, 1), ... until about max_seconds of
    CPU work.  Returns (TFLOP/s credited, threads, sample description, seconds)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()
                       if i.get("user_api") == "blas"), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    ins = fa_inputs.make_inputs(1, 1, w.N, w.d, w.seed, sigma_qk=w.sigma_qk,
                                sigma_v=w.sigma_v, with_dO=True)
    Q, K, V, dO = (ins[n][0, 0].double().numpy() for n in ("Q", "K", "V", "dO"))
    heads = 0
    t0 = time.perf_counter()
    while True:
        oracle.attention_head(Q, K, V, w.scale, w.causal)
        oracle.attention_bwd_head(Q, K, V, dO, w.scale, w.causal)
        heads += 1
        el = time.perf_counter() - t0
        if el > max_seconds / 2 or heads >= 4:
            break
    flops = heads * (traffic.fwd_flops(1, 1, w.N, w.d, w.causal) +
                     traffic.bwd_flops(1, 1, w.N, w.d, w.causal))
    sample = (f"fp64 oracle forward+backward of {heads} whole head(s) of the workload "
              f"(N={w.N}, d={w.d}, causal={w.causal}); credited FLOPs per second; "
              f"extrapolated full step ({w.B * w.H} heads) = {el * w.B * w.H / heads:.0f} s")
    return flops / el / 1e12, int(threads), sample, el


# The checked subset of each named workload (the oracle is O(N^2 d) per head in fp64):
# whole heads, and seeded rows of every head (each output row needs only its own query
# and the head's keys and values; the backward's dQ rows likewise).
CHECK_PLAN = {
    "tiny_f32": {"full_heads": ((0, 0),), "rows": 0},
    "n4096_d64": {"full_heads": ((0, 0),), "rows": 256},
    "n4096_d64_causal": {"full_heads": ((0, 0),), "rows": 256},
    "n10000_d128_causal": {"full_heads": ((0, 31),), "rows": 512},
    "n32768_d128_causal_sigma3": {"full_heads": (), "rows": 512, "extra_rows": 128},
    "n8192_d128_causal_bwd": {"full_heads": ((0, 3), (1, 7)), "rows": 256},
}


def parity_check(w, ins, outs, with_bwd):
    """Errors of the timed run's outputs against the fp64 oracle on the workload's checked
    subset (CHECK_PLAN), and the oracle's time for that subset on this host, with its
    extrapolation to the whole problem (by the oracle's executed products).  ins and outs
    are the device tensors of the run (inputs Q, K, V, dO; outputs O, LSE, dQ, dK, dV)."""
    import numpy as np
    import oracle
    plan = CHECK_PLAN[w.name]
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()  # noqa: E731
    rows = sorted(set(fa_inputs.sample_rows(w.N, plan["rows"], seed=1234)) |
                  set(range(min(plan.get("extra_rows", 0), w.N)))) if plan["rows"] else []
    rows = np.array(rows, dtype=np.int64)
    got = {n: [] for n in ("O", "LSE", "dQ", "dK", "dV")}
    ref = {n: [] for n in got}
    t_or, units = 0.0, 0.0  # oracle seconds; its products in units of N*d multiply-adds
    for b in range(w.B):
        for h in range(w.H):
            full = (b, h) in plan["full_heads"]
            if not full and rows.size == 0:
                continue
            Q, K, V = (f64(ins[n][b, h]) for n in ("Q", "K", "V"))
            dO = f64(ins["dO"][b, h]) if with_bwd else None
            O64, L64 = f64(outs["O"][b, h]), f64(outs["LSE"][b, h])
            t0 = time.perf_counter()
            if full:
                rO, rL, _ = oracle.attention_head(Q, K, V, w.scale, w.causal)
                units += 2 * w.N
                if with_bwd:
                    rg = oracle.attention_bwd_head(Q, K, V, dO, w.scale, w.causal)
                    units += 6 * w.N
            else:
                rO, rL, _ = oracle.attention_head(Q[rows], K, V, w.scale, w.causal,
                                                  q_index=rows)
                units += 2 * rows.size
                if with_bwd:
                    rdq, _ = oracle.attention_bwd_dq_rows(Q[rows], K, V, dO[rows], w.scale,
                                                          w.causal, rows)
                    units += 4 * rows.size
            t_or += time.perf_counter() - t0
            sel = slice(None) if full else rows
            got["O"].append(O64[sel].ravel())
            ref["O"].append(rO.ravel())
            got["LSE"].append(L64[sel].ravel())
            ref["LSE"].append(rL.ravel())
            if with_bwd:
                gq = f64(outs["dQ"][b, h])
                if full:
                    for k_, n in enumerate(("dQ", "dK", "dV")):
                        got[n].append(f64(outs[n][b, h]).ravel())
                        ref[n].append(rg[k_].ravel())
                else:
                    got["dQ"].append(gq[rows].ravel())
                    ref["dQ"].append(rdq.ravel())
    res = {}
    for n in got:
        if not got[n]:
            continue
        g, r = np.concatenate(got[n]), np.concatenate(ref[n])
        diff = g - r
        res[n] = {"max_abs": float(np.abs(diff).max()),
                  "rel_l2": float(np.linalg.norm(diff) / np.linalg.norm(r)),
                  "values": int(g.size)}
    full_units = w.B * w.H * (2 + (6 if with_bwd else 0)) * w.N
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()
                       if i.get("user_api") == "blas"), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    res["subset"] = (f"whole heads {list(plan['full_heads'])}; "
                     f"{rows.size} seeded rows of every head" if rows.size else
                     f"whole heads {list(plan['full_heads'])}")
    res["oracle_s"] = t_or
    res["oracle_threads"] = int(threads)
    res["oracle_est_full_s"] = t_or * full_units / units if units else None
    return res


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step = []
    value = threads = sample = None
    for i in range(args.warmup + args.steps):
        v, threads, sample, el = time_oracle(w, max_seconds=args.ref_seconds)
        if i >= args.warmup:
            per_step.append((v, el))
    value = statistics.median(v for v, _ in per_step)
    ms = statistics.median(el for _, el in per_step) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, not args.fwd_only, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle",
                         "sample": sample + "; run on the host cores (rank 0 only), each "
                         "step one bounded sample of the workload"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, w):
    from exact_io_aware_64_b200 import binding
    info = fa_dist.rank_info()
    fa_dist.init(info, "nccl")
    rank, world, local = info.rank, info.world, info.local_rank
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, N, d = w.B, w.H, w.N, w.d
    with_bwd = not args.fwd_only
    f32 = w.dtype == "f32"
    ins = fa_inputs.make_inputs(B, H, N, d, fa_dist.replica_seed(w.seed, info), sigma_qk=w.sigma_qk,
                                sigma_v=w.sigma_v, with_dO=True, device=str(dev),
                                dtype=torch.float32 if f32 else torch.bfloat16)
    q, k, v, do = ins["Q"], ins["K"], ins["V"], ins["dO"]
    O = torch.empty_like(q)
    LSE = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dQ, dK, dV = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(binding.workspace_bytes(B, H, N, d), 1), device=dev,
                     dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(marks=None):
        # marks: [fwd before, fwd after, bwd before, prep done, dkdv done, dq done], recorded
        # by the library at its kernel boundaries (fa_trace_events)
        if marks is None:
            binding.fwd(q, k, v, scale=w.scale, causal=w.causal, O=O, LSE=LSE)
        else:
            with binding.trace_kernels(marks[0:2]):
                binding.fwd(q, k, v, scale=w.scale, causal=w.causal, O=O, LSE=LSE)
        if with_bwd:
            if marks is None:
                binding.bwd(q, k, v, O, do, LSE, scale=w.scale, causal=w.causal, dQ=dQ, dK=dK,
                            dV=dV, workspace=ws)
            else:
                with binding.trace_kernels(marks[2:6]):
                    binding.bwd(q, k, v, O, do, LSE, scale=w.scale, causal=w.causal, dQ=dQ,
                                dK=dK, dV=dV, workspace=ws)

    for _ in range(args.warmup):
        step()
    binding.check_device_error()
    marks = [[ev() for _ in range(6)] for _ in range(args.steps)]
    fa_dist.barrier(info)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        start, end = ev(), ev()
        start.record(stream)
        for i in range(args.steps):
            step(marks[i])
        end.record(stream)
        torch.cuda.synchronize()
    fa_dist.barrier(info)
    binding.check_device_error()
    ms_local = start.elapsed_time(end) / args.steps
    ms = fa_dist.max_over_ranks(ms_local, info, device=str(dev))
    def span(a, b):
        return statistics.mean(m[a].elapsed_time(m[b]) for m in marks)

    fwd_ms = span(0, 1)
    bwd_ms = span(2, 5) if with_bwd else 0.0
    # per-step device time (first kernel start to last kernel end of each step)
    per_step = sorted(m[0].elapsed_time(m[5 if with_bwd else 1]) for m in marks)
    pct = statistics.quantiles(per_step, n=10) if len(per_step) > 1 else per_step * 9
    step_pct = {"p10": pct[0], "p50": statistics.median(per_step), "p90": pct[-1]}
    f_fwd = traffic.fwd_flops(B, H, N, d, w.causal)
    f_bwd = traffic.bwd_flops(B, H, N, d, w.causal) if with_bwd else 0.0
    # per kernel: mean launch time and algorithmic work (FLOPs credited to that kernel,
    # or bytes for the bandwidth-bound preparation)
    kn = KERNEL_NAMES_F32 if f32 else KERNEL_NAMES_BF16
    kernels = {kn[0]: {"ms": fwd_ms, "flops": f_fwd}}
    if with_bwd:
        half = 0.5 if w.causal else 1.0
        kernels[kn[1]] = {"ms": span(2, 3),
                          "bytes": traffic.bwd_prep_bytes(B, H, N, d, 4 if f32 else 2)}
        kernels[kn[2]] = {"ms": span(3, 4), "flops": 8.0 * B * H * N * N * d * half}
        # credited: the dQ product; executed: the S and dP recomputes as well
        kernels[kn[3]] = {"ms": span(4, 5), "flops": 2.0 * B * H * N * N * d * half,
                          "executed_flops": 6.0 * B * H * N * N * d * half}
    add_rates(kernels)
    value = fa_dist.aggregate_throughput(f_fwd + f_bwd, ms * 1e-3, info) / 1e12

    # ---- end to end through the public API with host buffers
    pin = lambda t: t.detach().to("cpu").pin_memory()  # noqa: E731
    hq, hk, hv, hdo = pin(q), pin(k), pin(v), pin(do)
    hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    hL = torch.empty(LSE.shape, dtype=LSE.dtype, pin_memory=True)
    hdQ, hdK, hdV = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(3))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    outs = [(O, hO), (LSE, hL)] + ([(dQ, hdQ), (dK, hdK), (dV, hdV)] if with_bwd else [])
    d2h = sum(dt.numel() * dt.element_size() for dt, _ in outs)

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        do.copy_(hdo, non_blocking=True)
        step()
        for dt, ht in outs:
            ht.copy_(dt, non_blocking=True)

    # (a) one stream: copy in, compute, copy out, step after step
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    fa_dist.barrier(info)
    e0, e1 = ev(), ev()
    e0.record(stream)
    # enough steps that the pipelined figure below is not dominated by filling and
    # draining its three-stage pipeline
    e2e_steps = max(2, min(args.steps, 30))
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    serial_ms = fa_dist.max_over_ranks(e0.elapsed_time(e1) / e2e_steps, info, device=str(dev))

    # (b) pipelined, as a throughput-minded caller would run it: step i's inputs go up
    # on one stream while step i-1 computes and step i-2's results come down on a third
    # (PCIe carries both directions at once).  Three sets of device buffers take turns
    # (one more than the three stages strictly need, so that a slow copy in one direction
    # does not stall the other); events order each copy after the step that last used
    # its buffers.  Every step still moves all its inputs in and all its results out
    # inside the timed region.
    n_sets = 3
    sets = []
    for _ in range(n_sets):
        di = {n: torch.empty_like(t) for n, t in (("q", q), ("k", k), ("v", v), ("do", do))}
        do_ = {"O": torch.empty_like(O), "LSE": torch.empty_like(LSE)}
        if with_bwd:
            do_.update(dQ=torch.empty_like(dQ), dK=torch.empty_like(dK), dV=torch.empty_like(dV))
        ho = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in do_.items()}
        sets.append((di, do_, ho))
    s_up, s_cmp, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    hin = {"q": hq, "k": hk, "v": hv, "do": hdo}

    def pipelined(n_steps):
        computed, downloaded = [], []
        for i in range(n_steps):
            di, dout, ho = sets[i % n_sets]
            up = torch.cuda.Event()
            with torch.cuda.stream(s_up):
                if i >= n_sets:
                    s_up.wait_event(computed[i - n_sets])
                for n, t in di.items():
                    t.copy_(hin[n], non_blocking=True)
                up.record(s_up)
            cmp_done = torch.cuda.Event()
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up)
                if i >= n_sets:
                    s_cmp.wait_event(downloaded[i - n_sets])
                binding.fwd(di["q"], di["k"], di["v"], scale=w.scale, causal=w.causal,
                            O=dout["O"], LSE=dout["LSE"], stream=s_cmp)
                if with_bwd:
                    binding.bwd(di["q"], di["k"], di["v"], dout["O"], di["do"], dout["LSE"],
                                scale=w.scale, causal=w.causal, dQ=dout["dQ"], dK=dout["dK"],
                                dV=dout["dV"], workspace=ws, stream=s_cmp)
                cmp_done.record(s_cmp)
            computed.append(cmp_done)
            dn = torch.cuda.Event()
            with torch.cuda.stream(s_down):
                s_down.wait_event(cmp_done)
                for n, t in dout.items():
                    ho[n].copy_(t, non_blocking=True)
                dn.record(s_down)
            downloaded.append(dn)

    pipelined(n_sets + 1)
    torch.cuda.synchronize()
    fa_dist.barrier(info)
    p0, p1 = ev(), ev()
    p0.record(s_up)
    s_cmp.wait_event(p0)
    s_down.wait_event(p0)
    pipelined(e2e_steps)
    s_down.wait_stream(s_up)
    s_down.wait_stream(s_cmp)
    p1.record(s_down)
    torch.cuda.synchronize()
    binding.check_device_error()
    e2e_ms = fa_dist.max_over_ranks(p0.elapsed_time(p1) / e2e_steps, info, device=str(dev))
    e2e_value = fa_dist.aggregate_throughput(f_fwd + f_bwd, e2e_ms * 1e-3, info) / 1e12
    serial_value = fa_dist.aggregate_throughput(f_fwd + f_bwd, serial_ms * 1e-3, info) / 1e12

    # (c) the copy floor of (b): one step's uploads and downloads, both directions at once
    # on the same streams, with no compute.  No pipelined step can be faster.
    di0, dout0, ho0 = sets[0]

    def copies():
        with torch.cuda.stream(s_up):
            for n, t in di0.items():
                t.copy_(hin[n], non_blocking=True)
        with torch.cuda.stream(s_down):
            for n, t in dout0.items():
                ho0[n].copy_(t, non_blocking=True)

    copies()
    torch.cuda.synchronize()
    c0, c1 = ev(), ev()
    c0.record(s_up)
    s_down.wait_event(c0)
    copy_reps = 5
    for _ in range(copy_reps):
        copies()
    s_down.wait_stream(s_up)
    c1.record(s_down)
    torch.cuda.synchronize()
    copy_ms = fa_dist.max_over_ranks(c0.elapsed_time(c1) / copy_reps, info, device=str(dev))
    del sets

    if rank != 0:
        fa_dist.shutdown(info)
        return 0

    peaks, peak_src = load_peaks()
    # dominant kernel: the one with the longest mean launch time
    dom_name = max(kernels, key=lambda k: kernels[k]["ms"])
    dom = kernels[dom_name]
    peak = peaks.get("bf16_tflops_sustained" if args.sustained_peak else "bf16_tflops")
    bound, peak_source = "tensor", (f"{peak_src} "
                                    f"{'sustained' if args.sustained_peak else 'burst'} bf16")
    if f32:
        # the float32 path runs on the CUDA cores: nominal FMA rate at the maximum clock
        peak, bound = FP32_ALU_TFLOPS, "alu"
        peak_source = "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz"
    achieved = dom["tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if f32 else "bf16",
        "data": "synthetic",
        "config": config_dict(w, with_bwd, world),
        "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "step_ms_percentiles": step_pct,
        "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": (f_bwd / (bwd_ms * 1e-3) / 1e12) if with_bwd else None,
        # tensor-core work the split backward executes (its dQ kernel recomputes S and dP)
        "bwd_executed_tflops": (traffic.bwd_executed_flops(B, H, N, d, w.causal)
                                / (bwd_ms * 1e-3) / 1e12) if with_bwd else None,
        "roofline": {"kernel": dom_name, "bound": bound, "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": peak_source, "traffic": recorded_traffic(dom_name),
                     **({} if f32 else {
                         "peak_sustained": peaks.get("bf16_tflops_sustained"),
                         "frac_sustained": achieved / peaks["bf16_tflops_sustained"]
                         if peaks.get("bf16_tflops_sustained") else None})},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "mode": "pipelined: uploads, compute and downloads on three streams",
                "copy_floor_ms": copy_ms, "frac_of_copy_floor": copy_ms / e2e_ms,
                "serial": {"value": serial_value, "ms_per_step": serial_ms}},
        "gpu_launches": args.steps * (1 + (3 if with_bwd else 0)),
        "clocks": clocks.summary(),
    }
    if args.check and world == 1:
        line["parity"] = parity_check(
            w, ins, {"O": O, "LSE": LSE, "dQ": dQ, "dK": dK, "dV": dV}, with_bwd)
    if world == 1 and not args.no_cpu_baseline:
        v_cpu, threads, sample, _ = time_oracle(w, max_seconds=args.ref_seconds)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)
    fa_dist.shutdown(info)
    return 0


# ------------------------------------------------------------------ N sweep
SWEEP_N = (256, 512, 1024, 2048, 4096, 8192, 16384, 32768)
SWEEP_CHUNK_NQ = (256, 1024, 2048, 4096)


def run_sweep(args):
    """TFLOP/s of fa_fwd and fa_bwd against N (the metric's "vs N"): B*N = 16384 tokens
    (B = max(1, 16384 / N)), H = 2048 / d, d in {64, 128}, causal in {0, 1}, bf16.
    Each call is timed alone with CUDA events; for N <= 1024 a 256 MB buffer is
    rewritten between calls so every call starts with a cold L2.  One JSON line per
    point."""
    from exact_io_aware_64_b200 import binding
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    for d in (64, 128):
        for causal in (False, True):
            for N in SWEEP_N:
                B, H = max(1, 16384 // N), 2048 // d
                ins = fa_inputs.make_inputs(B, H, N, d, seed=N + d, with_dO=True, device="cuda")
                q, k, v, do = ins["Q"], ins["K"], ins["V"], ins["dO"]
                O = torch.empty_like(q)
                LSE = torch.empty((B, H, N), device=dev, dtype=torch.float32)
                dQ, dK, dV = (torch.empty_like(q) for _ in range(3))
                ws = torch.empty(max(binding.workspace_bytes(B, H, N, d), 1), device=dev,
                                 dtype=torch.uint8)
                fwd = lambda: binding.fwd(q, k, v, causal=causal, O=O, LSE=LSE)  # noqa: E731
                bwd = lambda: binding.bwd(q, k, v, O, do, LSE, causal=causal, dQ=dQ,  # noqa: E731
                                          dK=dK, dV=dV, workspace=ws)
                res = {}
                for name, fn, flops, nbytes in (
                        ("fwd", fwd, traffic.fwd_flops(B, H, N, d, causal),
                         traffic.fwd_compulsory_bytes(B, H, N, d)),
                        ("bwd", bwd, traffic.bwd_flops(B, H, N, d, causal),
                         traffic.bwd_compulsory_bytes(B, H, N, d))):
                    for _ in range(args.warmup):
                        fn()
                    times = []
                    for _ in range(args.steps):
                        if N <= 1024:
                            flush.fill_(1)
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record()
                        fn()
                        e1.record()
                        torch.cuda.synchronize()
                        times.append(e0.elapsed_time(e1))
                    ms = statistics.median(times)
                    pct = statistics.quantiles(times, n=10) if len(times) > 1 else [ms] * 9
                    # roofline: the slower of the tensor-core time and the time to move
                    # the compulsory bytes once at the measured HBM bandwidth
                    t_tensor = flops / (peak * 1e12) * 1e3
                    t_hbm = nbytes / (hbm * 1e9) * 1e3
                    res[name] = {"ms": ms, "ms_p10": pct[0], "ms_p90": pct[-1],
                                 "tflops": flops / (ms * 1e-3) / 1e12,
                                 "frac": flops / (ms * 1e-3) / 1e12 / peak,
                                 "gbs": nbytes / (ms * 1e-3) / 1e9,
                                 "bound": "tensor" if t_tensor >= t_hbm else "hbm",
                                 "roofline_frac": max(t_tensor, t_hbm) / ms}
                binding.check_device_error()
                print(json.dumps({"sweep": "attention TFLOP/s vs N", "N": N, "B": B, "H": H, "d": d,
                                  "causal": causal, "dtype": "bf16", "peak": peak,
                                  "hbm_gbs": hbm, "peak_source": f"{peak_src} burst bf16, "
                                  f"{peak_src} HBM copy", **res}), flush=True)
                del ins, q, k, v, do, O, LSE, dQ, dK, dV, ws
    # chunks of queries at the end of a long key sequence (fa_fwd_qk / fa_bwd_qk):
    # B=1, H=16, Nk=8192, d=128, causal
    for Nq in SWEEP_CHUNK_NQ:
        B, H, Nk, d = 1, 16, 8192, 128
        qi = fa_inputs.make_inputs(B, H, Nq, d, seed=Nq, with_dO=True, device="cuda")
        ki = fa_inputs.make_inputs(B, H, Nk, d, seed=Nq + 1, device="cuda")
        q, do, k, v = qi["Q"], qi["dO"], ki["K"], ki["V"]
        O = torch.empty_like(q)
        LSE = torch.empty((B, H, Nq), device=dev, dtype=torch.float32)
        dQ, dK, dV = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(binding.workspace_bytes(B, H, Nq, d), 1), device=dev,
                         dtype=torch.uint8)
        fwd = lambda: binding.fwd(q, k, v, causal=True, O=O, LSE=LSE)  # noqa: E731
        bwd = lambda: binding.bwd(q, k, v, O, do, LSE, causal=True, dQ=dQ, dK=dK,  # noqa: E731
                                  dV=dV, workspace=ws)
        res = {}
        for name, fn, flops in (("fwd", fwd, traffic.fwd_flops_qk(B, H, Nq, Nk, d, True)),
                                ("bwd", bwd, traffic.bwd_flops_qk(B, H, Nq, Nk, d, True))):
            for _ in range(args.warmup):
                fn()
            times = []
            for _ in range(args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            ms = statistics.median(times)
            res[name] = {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12,
                         "frac": flops / (ms * 1e-3) / 1e12 / peak}
        binding.check_device_error()
        print(json.dumps({"sweep": "prefill chunk TFLOP/s", "Nq": Nq, "Nk": Nk, "B": B, "H": H,
                          "d": d, "causal": True, "dtype": "bf16", "peak": peak, **res}),
              flush=True)
        del qi, ki, q, do, k, v, O, LSE, dQ, dK, dV, ws
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(fa_inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--sustained-peak", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=20.0)
    ap.add_argument("--check", action="store_true",
                    help="after timing, compare the outputs with the fp64 oracle on the "
                    "workload's checked subset and time the oracle on it")
    ap.add_argument("--sweep", action="store_true",
                    help="print TFLOP/s of fa_fwd and fa_bwd against N instead of the step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = fa_inputs.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.sweep:
        return run_sweep(args)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
