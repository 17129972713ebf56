"""Benchmark of Skip Softmax attention on B200 (prefill and decode).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference] [--quick]

One JSON line on stdout (rank 0).

Headline (``value``): prefill dense-equivalent TFLOP/s on the causal
Llama-3.3-70B attention-layer shape at 128K context (B=1, Hq=64, Hkv=8,
N=131072, d=128, Br=Bc=128, tau=inf), the largest workload and the one the
Skip Softmax page reports on.  A step is one attn_prefill call over that
layer, inputs resident in HBM.

``configs`` holds one entry per workload (the five shapes of
``inputs.WORKLOADS``) at each of its thresholds: prefill dense-equivalent and
executed TFLOP/s, the skipped fraction, latency and the fraction of the
measured bf16 peak; decode KV-read GB/s, latency and the fraction of the
measured HBM bandwidth.  ``extras`` holds the rest (8-bit Q K^T, varlen,
decode rule variants, paged decode, and an input on which the skip rule
fires), none of which is one of the five workloads.

Timing: W untimed warm-up steps (at least 3), then exactly K steps between
two CUDA events on the launching stream, bracketed by a barrier and a device
synchronise, max over ranks.  Every timed workload but the 256-token one has
inputs larger than the 126 MB L2 (the 8B layer: 168 MB); the 256-token one
fits in L2 by construction and is launch-bound.  Multi-GPU: every rank runs
its own copy of the workload (independent sequences; no collective on the
data path) -> weak scaling.

``--impl reference`` times the fp64 CPU oracle (the deliberately slow
reference program) on a bounded sample of the headline workload, on this
host's cores, in the same unit.
"""
from __future__ import annotations

import argparse
import gc
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "llama33_70b_causal_N131072"
ENCODER = "encoder_64x32x512_d128"
DECODE = "gqa_decode_16x32q8kv_L32768"
LAYER_8B = "llama3_8b_causal_N8192"
SMALL = "causal_1x1x256_d64"
CONFIG_ORDER = [SMALL, ENCODER, DECODE, LAYER_8B, HEADLINE]
METRIC = "prefill attn TFLOP/s (dense-equiv) & % tensor peak; decode KV-read GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PAGES_CONTEXT = {
    "source": "Accelerating Long-Context Inference with Skip Softmax in NVIDIA TensorRT-LLM "
              "(Key Points; Detailed Analysis)",
    "decode_end_to_end_speedup": "about 1.4x, Llama 3.3 70B, NVIDIA GB200 system",
    "prefill_speedup": "about 40% at 128K context, Llama 3.3 70B, NVIDIA GB200 system",
    "turboattention_profiling_hardware": "NVIDIA A100 (TurboAttention: Efficient Attention "
                                         "Approximation for High-Throughput LLM Serving)",
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def measured_traffic(key: str, cu_file: str):
    """DRAM bytes per launch from the committed ncu record, or None when the
    kernel's source changed since the counters were taken.  ``key`` names the
    kernel and the workload the counters were taken on."""
    import hashlib

    csrc = os.path.join(ROOT, "block_skipping_softmax_b200", "csrc")
    h = hashlib.sha256()
    for f in (cu_file, "ptx.cuh", "kernels.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.txt")) as fh:
            for line in fh:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == key and parts[1] == digest:
                    return int(parts[2])
    except OSError:
        pass
    return None


def dense_flops(w):
    f = 4.0 * w["B"] * w["Hq"] * w["N"] * w["N"] * w["d"]
    return f / 2 if w["causal"] else f


def compulsory_prefill_bytes(w):
    return 2 * w["B"] * w["Hq"] * w["N"] * w["d"] * 2 + 2 * w["B"] * w["Hkv"] * w["N"] * w["d"] * 2


def headline_config(w, world):
    return {"workload": HEADLINE, "B": w["B"], "Hq": w["Hq"], "Hkv": w["Hkv"], "N": w["N"], "d": w["d"],
            "causal": w["causal"], "Br": w["Br"], "Bc": w["Bc"], "tau": "inf",
            "parallelism": f"replicas x{world} (independent sequences)",
            "l2": "inputs 4.83 GB per step > 126 MB L2 (no flush needed)"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.rows = []
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        rows = [r for t, r in self.rows if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        window = "timed region"
        if len(rows) < 2:
            rows = [r for _, r in self.rows]
            window = "whole GPU phase"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows), "window": window,
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()),
                                   default=None)}


def dist_setup():
    from block_skipping_softmax_b200.replicas import rank_info

    return rank_info()


def cpu_cores():
    return len(os.sched_getaffinity(0))


# --------------------------------------------------------------------------- CPU oracle
_ORACLE_INPUTS = {}


def oracle_sample_headline(target_s, seed=1, heads=None, n_units=None):
    """Time the fp64 oracle on a random sample of row blocks of the headline
    workload (~target_s of CPU work on all host cores).

    The row blocks come from a few query heads, each drawn on its own with its
    KV head (bit for bit the heads of the full layer) and stacked as a small
    batch of independent heads, since the oracle's output buffers for all 64
    heads of a 128K-token layer would not fit in host memory.  ``n_units``
    fixes the sample size (row blocks per call); otherwise a short calibration
    run sizes it to ``target_s``.  Returns (TFLOP/s, seconds, row blocks,
    cores, heads)."""
    import numpy as np
    import torch

    import oracle
    from block_skipping_softmax_b200 import inputs

    w = inputs.WORKLOADS[HEADLINE]
    rng = np.random.default_rng(seed)
    if heads is None:
        heads = sorted(int(h) for h in rng.choice(w["Hq"], 4, replace=False))
    key = tuple(heads)
    if key not in _ORACLE_INPUTS:  # drawn once per set of heads
        drawn = [inputs.prefill_head_inputs(w["Hq"], w["Hkv"], w["N"], w["d"], 0, h, seed=0, **w["gen"])
                 for h in heads]
        # head i of the stack is query head heads[i] with its own KV head
        _ORACLE_INPUTS.clear()
        _ORACLE_INPUTS[key] = tuple(torch.cat([t[j] for t in drawn], dim=1) for j in range(3))
    Q, K, V = _ORACLE_INPUTS[key]
    n_rb = -(-w["N"] // w["Br"])
    cores = cpu_cores()

    def run(units):
        t = time.perf_counter()
        oracle.prefill(Q, K, V, True, math.inf, w["Br"], w["Bc"], units=units, want_exact=False,
                       nthreads=cores)
        return time.perf_counter() - t

    def pick(n):
        flat = rng.choice(len(heads) * n_rb, n, replace=False)
        return [(0, int(x) // n_rb, int(x) % n_rb) for x in flat]

    if n_units is None:
        run(pick(1))  # the first call pays for thread start-up
        n = 2 * cores
        t = run(pick(n))
        n_units = int(min(len(heads) * n_rb, max(cores, n * target_s / max(t, 1e-3))))
    units = pick(n_units)
    t = run(units)
    # dense-equivalent: half of 4 * rows * keys * d per row block under the causal mask
    f = sum(4.0 * w["Br"] * min(w["N"], (rb + 1) * w["Br"]) * w["d"] * 0.5 for _, _, rb in units)
    return f / t / 1e12, t, n_units, cores, heads


def reference_arm(args, world, rank):
    if rank != 0:
        return 0
    from block_skipping_softmax_b200 import inputs

    w = inputs.WORKLOADS[HEADLINE]
    # each step: a fresh random sample of row blocks, ~1.5 s of CPU time
    rates, secs = [], []
    heads = n_units = None
    cores = 0
    for i in range(args.warmup + args.steps):
        r, t, n_units, cores, heads = oracle_sample_headline(2.0, seed=100 + i, heads=heads,
                                                             n_units=n_units)
        if i >= args.warmup:
            rates.append(r)
            secs.append(t)
    value = statistics.mean(rates)
    sample = (f"{n_units} random row blocks (128 queries each, causal) of query heads {heads} of "
              f"{HEADLINE} per step, {statistics.mean(secs):.1f} s of fp64 CPU work each")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.mean(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": headline_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--quick", action="store_true", help="headline, e2e and the five workloads only")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup()

    if args.impl == "reference":
        return reference_arm(args, world, rank)

    import torch

    import block_skipping_softmax_b200 as bss
    from block_skipping_softmax_b200 import build as bss_build
    from block_skipping_softmax_b200 import inputs

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        bss_build.build()
    if dist:
        dist.barrier()
    bss.lib()
    peaks, peak_src = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    steps_x = max(3, args.steps // 4)  # steps of the secondary lines

    def barrier():
        if dist:
            dist.barrier()

    def max_over_ranks(x):
        from block_skipping_softmax_b200.replicas import max_over_ranks as mor

        return mor(x, dev)

    attempts_log = []

    def timed(fn, steps, warmup, label="step"):
        """Exactly `steps` calls between two events on the launching stream.

        Per-call events inside the region separate GPU time from host gaps
        (time the GPU sat idle because the host had not launched yet).  If
        the host gaps exceed 2% of the region, the region is measured again
        (at most 3 attempts); every attempt is reported in `timing_attempts`.
        """
        for _ in range(warmup):
            fn()
        tries = []
        for attempt in range(3):
            gc.collect()
            gc.disable()  # no collector pauses between the two events
            barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            marks = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps)]
            t0 = time.time()
            e0.record(stream)
            for i in range(steps):
                marks[2 * i].record(stream)
                fn()
                marks[2 * i + 1].record(stream)
            e1.record(stream)
            torch.cuda.synchronize()
            t1 = time.time()
            gc.enable()
            barrier()
            st = bss.attn_sync_status()
            if st != 0:
                raise RuntimeError(f"kernel status {bss.attn_status_string(st)}")
            total = e0.elapsed_time(e1)
            busy = sum(marks[2 * i].elapsed_time(marks[2 * i + 1]) for i in range(steps))
            gap = max(0.0, total - busy)
            tries.append({"ms_total": total, "host_gap_ms": gap})
            if gap <= 0.02 * total:
                break
        attempts_log.append({"region": label, "attempts": tries})
        return max_over_ranks(total / steps), t0, t1

    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    clocks = ClockSampler(int(vis[local]) if local < len(vis) and vis[local].strip().isdigit() else local)
    if rank == 0:
        clocks.start()

    configs = {name: {"config": i + 1, "workload": name, "runs": []} for i, name in enumerate(CONFIG_ORDER)}

    def prefill_run(name, wl, Qd, Kd, Vd, tau, steps, warmup, label=None, record=True):
        """Time one prefill line; returns its entry (dense and executed
        TFLOP/s, skipped fraction, latency, fractions of the bf16 peaks)."""
        Od = torch.empty_like(Qd)
        ms_x, t0, t1 = timed(lambda: bss.prefill(Qd, Kd, Vd, wl["causal"], tau, wl["Br"], wl["Bc"], out=Od),
                             steps, warmup, label or f"{name}@tau={tau}")
        _, mask = bss.prefill(Qd, Kd, Vd, wl["causal"], tau, wl["Br"], wl["Bc"], out=Od, skip_mask=True)
        mk = mask[mask != 2]
        f = dense_flops(wl)
        skipped = float((mk == 1).float().mean().item())
        visited = mk.numel()
        del mask, mk, Od
        # executed MMA FLOPs: every visited tile's Q K^T, every kept tile's P V
        executed = visited * 2.0 * wl["Br"] * wl["Bc"] * wl["d"] * (2.0 - skipped)
        tfl = f / (ms_x * 1e-3) / 1e12
        entry = {"tau": "inf" if math.isinf(tau) else tau, "ms": ms_x, "latency_us": ms_x * 1e3,
                 "steps": steps, "dense_tflops": tfl,
                 "executed_tflops": executed / (ms_x * 1e-3) / 1e12,
                 "frac_of_peak": tfl / peaks["bf16_tflops"],
                 # a launch of 50 ms or more runs under the power cap: compare it
                 # with the sustained GEMM figure as well
                 "frac_of_sustained_peak": tfl / peaks["bf16_tflops_sustained"] if ms_x >= 50.0 else None,
                 "skipped_fraction": skipped, "tiles_visited": visited,
                 "gpu_launches": steps}
        if record:
            configs[name]["runs"].append(entry)
        return entry, t0, t1

    # ================= headline: the 70B layer at 128K, tau = inf
    wh = inputs.WORKLOADS[HEADLINE]
    # drawn by the GPU's generator (the same recipe; a CPU draw of the 2.1 GB
    # Q would take minutes)
    Qh, Kh, Vh = inputs.prefill_inputs(wh["B"], wh["Hq"], wh["Hkv"], wh["N"], wh["d"], seed=rank,
                                       device=str(dev), **wh["gen"])
    Oh = torch.empty_like(Qh)

    def step():
        bss.prefill(Qh, Kh, Vh, wh["causal"], math.inf, wh["Br"], wh["Bc"], out=Oh)

    ms, t0, t1 = timed(step, args.steps, args.warmup, "prefill " + HEADLINE)
    clk = clocks.summary(t0, t1) if rank == 0 else None
    flops = dense_flops(wh)
    achieved = flops / (ms * 1e-3) / 1e12
    value = world * achieved
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
                "sustained_peak": peaks["bf16_tflops_sustained"],
                "traffic": measured_traffic("prefill_split_kernel@" + HEADLINE, "prefill_split_sm100.cu"),
                "algorithmic_bytes": compulsory_prefill_bytes(wh),
                "peak_source": f"{peak_src} bf16 burst; the sustained figure (seconds-long GEMM loop "
                               f"under the power cap) is given beside it",
                "kernel": "prefill_split_kernel<128, causal, no poly, no skip test> (tau = inf; one "
                          "128-row block per work item, softmax warpgroups splitting each key tile's "
                          "columns, persistent)",
                "algorithmic": "2*B*Hq*N^2*d dense-equivalent FLOPs per launch (causal half of 4*N^2*d "
                               "per head); one launch per step"}
    configs[HEADLINE]["runs"].append(
        {"tau": "inf", "ms": ms, "latency_us": ms * 1e3, "steps": args.steps, "dense_tflops": achieved,
         "executed_tflops": None, "frac_of_peak": achieved / peaks["bf16_tflops"],
         "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"], "gpu_launches": args.steps,
         "skipped_fraction": 0.0, "note": "headline region; tau = inf skips nothing by definition"})

    # ---------------- end to end through the public API, from pinned host memory
    Qp = torch.empty(Qh.shape, dtype=Qh.dtype, pin_memory=True)
    Kp = torch.empty(Kh.shape, dtype=Kh.dtype, pin_memory=True)
    Vp = torch.empty(Vh.shape, dtype=Vh.dtype, pin_memory=True)
    Op = torch.empty(Qh.shape, dtype=Qh.dtype, pin_memory=True)
    Qp.copy_(Qh)
    Kp.copy_(Kh)
    Vp.copy_(Vh)

    def e2e_step():
        # one public call: host inputs in, host output back; the library cuts
        # the layer into chunks of KV-head groups whose copies overlap the kernels
        bss.prefill_host(Qp, Kp, Vp, wh["causal"], math.inf, wh["Br"], wh["Bc"], out=Op, stream=stream)

    ms_e2e, _, _ = timed(e2e_step, steps_x, 2, "e2e " + HEADLINE)
    torch.cuda.synchronize()
    e2e_equal = bool(torch.equal(Op[0, :2].to(dev), Oh[0, :2]))  # the path computes the same output
    e2e = {"value": world * flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": Qp.numel() * 2 + Kp.numel() * 2 + Vp.numel() * 2,
           "d2h_bytes_per_step": Op.numel() * 2, "ms_per_step": ms_e2e, "steps": steps_x,
           "output_equals_device_path": e2e_equal,
           "path": "attn_prefill_host: pinned host -> chunks of KV-head groups, copies overlapping "
                   "attn_prefill_ex -> pinned host"}
    del Qp, Kp, Vp, Op
    # tau = 4 on the headline layer, plus its skipped fraction
    prefill_run(HEADLINE, wh, Qh, Kh, Vh, 4.0, steps_x, 2)
    del Qh, Kh, Vh, Oh
    torch.cuda.empty_cache()

    # ================= the other workloads, each at its thresholds
    ws = inputs.WORKLOADS[SMALL]
    Qs, Ks, Vs = (t.to(dev) for t in inputs.prefill_inputs(ws["B"], ws["Hq"], ws["Hkv"], ws["N"], ws["d"],
                                                           seed=rank, **ws["gen"]))
    for tau in ws["taus"]:
        prefill_run(SMALL, ws, Qs, Ks, Vs, tau, max(args.steps, 200), args.warmup)
    configs[SMALL]["note"] = ("4 CTAs on a 148-SM GPU: launch-bound, inputs resident in L2; "
                              "reported for completeness")
    del Qs, Ks, Vs

    we = inputs.WORKLOADS[ENCODER]
    Qm, Km, Vm = inputs.prefill_inputs(we["B"], we["Hq"], we["Hkv"], we["N"], we["d"], seed=rank, **we["gen"])
    Qe, Ke, Ve = Qm.to(dev), Km.to(dev), Vm.to(dev)
    del Qm, Km, Vm
    for tau in we["taus"]:
        prefill_run(ENCODER, we, Qe, Ke, Ve, tau, args.steps, args.warmup)

    extras = {}

    def qk8_extra(name, wl, Qd, Kd, Vd, tau, steps, warmup, int8=False):
        """The 8-bit Q K^T paths: e4m3 (or int8) Q and K, quantised once,
        outside the timed region (the quantiser is timed on its own), bf16 P*V."""
        quant = bss.quantize_i8 if int8 else bss.quantize_e4m3
        prefill8 = bss.prefill_qki8 if int8 else bss.prefill_qk8
        tag = "qki8" if int8 else "qk8"
        Q8, qs = quant(Qd)
        K8, ks = quant(Kd)
        Od = torch.empty_like(Qd)
        run = lambda: prefill8(Q8, K8, qs, ks, Vd, wl["causal"], tau, wl["Br"], wl["Bc"], out=Od)
        ms_x, _, _ = timed(run, steps, warmup, f"{name} {tag}@tau={tau}")
        _, mask = prefill8(Q8, K8, qs, ks, Vd, wl["causal"], tau, wl["Br"], wl["Bc"], out=Od,
                           skip_mask=True)
        skipped = float((mask[mask != 2] == 1).float().mean().item())
        f = dense_flops(wl)
        # half the dense FLOPs (Q K^T) run at the 8-bit rate, twice the bf16
        # rate (nominal ratio); the mixed peak is 4/3 of the bf16 peak
        mixed_peak = peaks["bf16_tflops"] * 4.0 / 3.0
        entry = {"ms": ms_x, "dense_tflops": f / (ms_x * 1e-3) / 1e12,
                 "frac_of_mixed_peak": f / (ms_x * 1e-3) / 1e12 / mixed_peak,
                 "mixed_peak_tflops": mixed_peak, "skipped_fraction": skipped}
        if tau == math.inf:
            ms_q, _, _ = timed(lambda: (quant(Qd, out=(Q8, qs)), quant(Kd, out=(K8, ks))),
                               steps, warmup, f"{name} quantize {tag}")
            qbytes = (Qd.numel() + Kd.numel()) * 3  # read bf16, write 8-bit
            entry["quantize_q_and_k_ms"] = ms_q
            entry["quantize_gbs"] = qbytes / (ms_q * 1e-3) / 1e9
        extras[f"{name} {tag}@tau={tau}"] = entry
        del Q8, K8, Od

    if not args.quick:
        # the same batch packed as variable-length sequences ([tokens, H, d],
        # cu_seqlens), the serving layout
        Qv = Qe.permute(0, 2, 1, 3).reshape(-1, we["Hq"], we["d"]).contiguous()
        Kv = Ke.permute(0, 2, 1, 3).reshape(-1, we["Hkv"], we["d"]).contiguous()
        Vv = Ve.permute(0, 2, 1, 3).reshape(-1, we["Hkv"], we["d"]).contiguous()
        Ov = torch.empty_like(Qv)
        cu = torch.arange(0, we["B"] * we["N"] + 1, we["N"], dtype=torch.int32, device=dev)
        ms_v, _, _ = timed(lambda: bss.prefill_varlen(Qv, Kv, Vv, cu, we["N"], we["causal"], math.inf,
                                                      we["Br"], we["Bc"], out=Ov),
                           steps_x, 2, f"{ENCODER} varlen@tau=inf")
        extras[f"{ENCODER} varlen@tau=inf"] = {
            "ms": ms_v, "dense_tflops": dense_flops(we) / (ms_v * 1e-3) / 1e12,
            "frac_of_peak": dense_flops(we) / (ms_v * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "layout": f"{we['B']} sequences of {we['N']} tokens packed as [tokens, H, d]"}
        del Qv, Kv, Vv, Ov, cu
        qk8_extra(ENCODER, we, Qe, Ke, Ve, math.inf, steps_x, 2)
        qk8_extra(ENCODER, we, Qe, Ke, Ve, math.inf, steps_x, 2, int8=True)
    del Qe, Ke, Ve
    torch.cuda.empty_cache()

    # ---------------- decode: KV-read GB/s
    wd = inputs.WORKLOADS[DECODE]
    qh, Kdh, Vdh = inputs.decode_inputs(wd["B"], wd["Hq"], wd["Hkv"], wd["L"], wd["d"], seed=rank, **wd["gen"])
    q, Kd, Vd = qh.to(dev), Kdh.to(dev), Vdh.to(dev)
    del Kdh, Vdh
    o = torch.empty_like(q)
    kv_bytes = wd["B"] * wd["Hkv"] * wd["L"] * wd["d"] * 2
    dec_traffic = measured_traffic("decode_partial_kernel@" + DECODE, "decode_sm100.cu")
    for tau in wd["taus"]:
        ms_d, _, _ = timed(lambda: bss.decode(q, Kd, Vd, tau, out=o), args.steps, args.warmup,
                           f"decode@tau={tau}")
        _, mask = bss.decode(q, Kd, Vd, tau, out=o, skip_mask=True)
        kept = 1.0 - float((mask == 1).float().mean().item())
        read = kv_bytes * (1.0 + kept)
        gbs = read / (ms_d * 1e-3) / 1e9
        configs[DECODE]["runs"].append({
            "tau": "inf" if math.isinf(tau) else tau, "ms": ms_d, "latency_us": ms_d * 1000,
            "steps": args.steps, "kv_read_gbs": gbs,
            "dense_equiv_gbs": 2 * kv_bytes / (ms_d * 1e-3) / 1e9, "skipped_fraction": 1.0 - kept,
            "frac_of_hbm": gbs / peaks["hbm_gbs"], "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"],
                         "traffic": dec_traffic if math.isinf(tau) else None,
                         "peak_source": f"{peak_src} HBM copy bandwidth",
                         "kernel": "decode_partial_kernel<128,4> + decode_combine_kernel<128>",
                         "algorithmic": "K bytes + kept fraction x V bytes per launch"},
            "split_len": bss.attn_decode_split_len(wd["B"], wd["Hkv"], wd["L"])})
    if not args.quick:
        # the decode rule variants (per-head test, sink-seeded splits) at the
        # thresholds where the skip rule acts
        g = wd["Hq"] // wd["Hkv"]
        ls = bss.attn_decode_split_len(wd["B"], wd["Hkv"], wd["L"])
        n_splits = -(-wd["L"] // ls)
        variants = {}
        for rule, rname in ((bss.RULE_PER_HEAD, "per_head"), (bss.RULE_SINK_SEED, "sink_seed"),
                            (bss.RULE_PER_HEAD | bss.RULE_SINK_SEED, "per_head+sink_seed")):
            for tau in (2.0, 4.0):
                ms_v, _, _ = timed(lambda: bss.decode(q, Kd, Vd, tau, out=o, rule=rule),
                                   steps_x, 2, f"decode {rname}@tau={tau}")
                _, mask = bss.decode(q, Kd, Vd, tau, out=o, skip_mask=True, rule=rule)
                if rule & bss.RULE_PER_HEAD:
                    m4 = mask.view(wd["B"], wd["Hkv"], g, -1)
                    v_kept = float((m4 == 0).any(dim=2).float().mean().item())
                    row_skip = float((mask == 1).float().mean().item())
                else:
                    v_kept = 1.0 - float((mask == 1).float().mean().item())
                    row_skip = 1.0 - v_kept
                seed_bytes = (wd["B"] * wd["Hkv"] * (n_splits - 1) * 64 * wd["d"] * 2
                              if rule & bss.RULE_SINK_SEED else 0)
                read = kv_bytes * (1.0 + v_kept) + seed_bytes
                gbs = read / (ms_v * 1e-3) / 1e9
                variants[f"{rname}@tau={tau}"] = {
                    "kv_read_gbs": gbs, "latency_us": ms_v * 1000,
                    "v_tiles_skipped": 1.0 - v_kept, "row_tiles_skipped": row_skip,
                    "bytes_read": read, "frac_of_hbm": gbs / peaks["hbm_gbs"]}
        extras["decode_rule_variants"] = variants
        # the same cache as a pool of 64-key pages in shuffled order, read
        # through a block table (the serving layout)
        B_, Hkv_, L_, d_ = wd["B"], wd["Hkv"], wd["L"], wd["d"]
        npg = L_ // 64
        gen = torch.Generator(device="cpu").manual_seed(7)
        perm = torch.randperm(B_ * npg, generator=gen).to(dev)
        Kp = torch.empty(B_ * npg, Hkv_, 64, d_, dtype=torch.bfloat16, device=dev)
        Vp = torch.empty_like(Kp)
        Kp[perm] = Kd.view(B_, Hkv_, npg, 64, d_).permute(0, 2, 1, 3, 4).reshape(B_ * npg, Hkv_, 64, d_)
        Vp[perm] = Vd.view(B_, Hkv_, npg, 64, d_).permute(0, 2, 1, 3, 4).reshape(B_ * npg, Hkv_, 64, d_)
        table = perm.view(B_, npg).to(torch.int32).contiguous()
        lens = torch.full((B_,), L_, dtype=torch.int32, device=dev)
        ms_p, _, _ = timed(lambda: bss.decode_paged(q, Kp, Vp, table, lens, L_, math.inf, out=o),
                           steps_x, 2, "decode paged@tau=inf")
        gbs = 2 * kv_bytes / (ms_p * 1e-3) / 1e9
        extras["decode paged@tau=inf"] = {"kv_read_gbs": gbs, "latency_us": ms_p * 1000,
                                          "frac_of_hbm": gbs / peaks["hbm_gbs"],
                                          "layout": "pool [B*L/64, Hkv, 64, d], pages in a seeded random order"}
        del Kp, Vp, table, lens, perm
    del q, Kd, Vd, o
    torch.cuda.empty_cache()

    # ---------------- the causal 8B layer (inputs drawn on the GPU)
    w8 = inputs.WORKLOADS[LAYER_8B]
    Q8d, K8d, V8d = inputs.prefill_inputs(w8["B"], w8["Hq"], w8["Hkv"], w8["N"], w8["d"], seed=rank,
                                          device=str(dev), **w8["gen"])
    for tau in w8["taus"]:
        prefill_run(LAYER_8B, w8, Q8d, K8d, V8d, tau, args.steps, args.warmup)
    if not args.quick:
        for tau in (math.inf, 4.0):
            qk8_extra(LAYER_8B, w8, Q8d, K8d, V8d, tau, steps_x, 2)
        qk8_extra(LAYER_8B, w8, Q8d, K8d, V8d, math.inf, steps_x, 2, int8=True)
        # part of the exponentials on the FMA-pipe polynomial instead of MUFU
        for pairs in (4, 8):
            Od = torch.empty_like(Q8d)
            ms_p, _, _ = timed(lambda: bss.prefill_poly(Q8d, K8d, V8d, True, math.inf, pairs, out=Od),
                               steps_x, 2, f"{LAYER_8B} poly{pairs}@tau=inf")
            tfl = dense_flops(w8) / (ms_p * 1e-3) / 1e12
            extras[f"{LAYER_8B} poly{pairs}/16@tau=inf"] = {
                "ms": ms_p, "dense_tflops": tfl, "frac_of_peak": tfl / peaks["bf16_tflops"],
                "exp2_on_fma_pipes": f"{pairs} of every 16 pairs"}
            del Od
    del Q8d, K8d, V8d
    torch.cuda.empty_cache()

    if not args.quick:
        # Not one of the five workloads: the parity suite's skip-exercising
        # input (strong sinks: q = 2z + 8u, sink keys 6 sqrt(d) u) at the 8B
        # layer's shape, where the every-row rule does skip tiles.  The same
        # input at tau = inf is the time a skip is measured against.
        gen_s = dict(q_sigma=2.0, q_u=8.0, sink_scale=6.0)
        Qx, Kx, Vx = inputs.prefill_inputs(w8["B"], w8["Hq"], w8["Hkv"], w8["N"], w8["d"], seed=rank,
                                           device=str(dev), **gen_s)
        runs = {}
        for tau in (math.inf, 4.0, 2.0):
            e, _, _ = prefill_run(LAYER_8B, w8, Qx, Kx, Vx, tau, args.steps, args.warmup,
                                  label=f"skip-exercising 8B shape@tau={tau}", record=False)
            runs["inf" if math.isinf(tau) else str(tau)] = e
        base = runs["inf"]["ms"]
        for k, e in runs.items():
            e["time_vs_tau_inf"] = e["ms"] / base
            # if a skipped tile cost nothing, time would fall with the P*V half of the work
            e["pv_work_fraction_left"] = 1.0 - 0.5 * e["skipped_fraction"]
        extras["skip_exercising_8b_shape"] = {
            "not_a_baseline_config": True,
            "input": "B=1, Hq=32, Hkv=8, N=8192, d=128, causal, Br=Bc=128; q = 2z + 8u, "
                     "sink keys 6 sqrt(d) u (the parity suite's skip-exercising recipe)",
            "runs": runs}
        del Qx, Kx, Vx
        torch.cuda.empty_cache()
    if rank == 0:
        clocks.stop()

    cpu_base = None
    if rank == 0 and world == 1 and not args.quick:
        r, t, n, cores, heads = oracle_sample_headline(12.0)
        cpu_base = {"value": r, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                    "sample": f"{n} random row blocks (128 queries each, causal) of query heads "
                              f"{heads} of {HEADLINE}, {t:.1f} s of fp64 CPU work"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": headline_config(wh, world),
            "roofline": roofline, "e2e": e2e, "gpu_launches": args.steps, "clocks": clk,
            "cpu_baseline": cpu_base,
            "configs": [configs[n] for n in CONFIG_ORDER],
            "extras": extras,
            # the pages report no kernel-level figure; their numbers are
            # end-to-end model speedups on other hardware (context only)
            "pages_context": PAGES_CONTEXT,
            "timing_attempts": attempts_log,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
