"""Benchmark of causal packed-document attention, forward + backward.

One step = one fwd + bwd pass over the whole workload (every query head, every
document) through the C ABI.  Default workload: 32768 packed tokens,
log-normal document lengths (median 2048, sigma 1, clipped to [64, 16384]),
32 heads, d = 128, 1% of tokens x8 (seed 0).  Metric: causal-aware TFLOP/s
with the algorithmic FLOP count 14 d Hq sum_k L_k (L_k + 1) / 2 (masked work is
never counted), and its fraction of the B200 tensor peaks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fapk|reference]
                  [--config 1..5]

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no cross-GPU exchange), timings are max-reduced over ranks and
``value`` counts the work of all ranks.  ``--impl reference`` times the fp64
CPU oracle on a bounded sample of the same workload on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "causal fwd+bwd attention TFLOP/s (bf16, MXFP8 incl. quant) & % of B200 tensor peak"
# the library's precision constant of each path name
PREC = {"bf16": "BF16", "mxfp8": "MXFP8", "nvfp4": "NVFP4_MIXED"}
# mixed NVFP4/FP8 path: the scores' MMAs run FP4 (twice the FP8 rate), the
# other products FP8; the time-weighted peak of each kernel in units of the
# FP8 peak: forward S + PV = 2 + 2 -> 4 / (1 + 2); dK/dV S, dP, dV, dK ->
# 8 / (1 + 6); dQ S, dP, dQ -> 6 / (1 + 4)
NV_PEAK_FACTOR = {"fwd_kernel": 4.0 / 3.0, "dkdv_kernel": 8.0 / 7.0, "dq_kernel": 6.0 / 5.0}
DENSE_BF16_TFLOPS = 2250.0   # NVIDIA B200 datasheet, dense
DENSE_FP8_TFLOPS = 4500.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk["bf16_tflops_sustained"],
                "sm_max_mhz": float(pk.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


def tensor_peak(peaks, clk, fp8: bool):
    """Tensor denominator for a kernel timed in a short region: the measured
    burst bf16 GEMM peak (taken at the maximum SM clock), scaled to the median
    SM clock sampled during the timed region, times the nominal FP8/bf16 ratio
    of 2 for the MXFP8 path.  Returns (peak TFLOP/s, description)."""
    mhz = clk.get("sm_mhz") if clk else None
    top = peaks["sm_max_mhz"]
    f = min(1.0, mhz / top) if mhz else 1.0
    base = peaks["bf16_tflops"] * f
    desc = (f"{peaks['source']} bf16 burst GEMM peak {peaks['bf16_tflops']:.1f} TFLOP/s (MEASURED_PEAKS.json) "
            f"x median SM clock {mhz if mhz else 'unknown'} / {top:.0f} MHz")
    if fp8:
        return 2.0 * base, "2 x " + desc + " (nominal FP8/bf16 ratio; no FP8 GEMM measured)"
    return base, desc


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fapk_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def cpu_oracle_sample(w, target_s: float = 15.0):
    """Time the fp64 oracle (fwd + bwd) on a bounded sample of the workload:
    query heads 0..h-1 of the first documents whose cost fits about
    `target_s` seconds on this host's cores.  Returns (TFLOP/s, cores, text)."""
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    q, k, v, do = w.tensors()
    cu = w.cu
    # sample: a prefix of whole documents, KV head 0 and its query heads
    G = w.Hq // w.Hkv
    lengths = np.diff(cu.astype(np.int64))
    # calibrate on the first document
    n_docs = 1
    T1 = int(cu[1])
    sl = slice(0, T1)
    args = [t[sl, :G].double().numpy() if i != 1 and i != 2 else t[sl, :1].double().numpy()
            for i, t in enumerate((q, k, v, do))]
    t0 = time.perf_counter()
    oracle.attn_bwd(*args, cu[:2], w.scale)
    dt = time.perf_counter() - t0
    flops1 = 14.0 * w.d * G * float(lengths[0] * (lengths[0] + 1) // 2)
    rate = flops1 / max(dt, 1e-9)
    # grow the prefix while it fits the budget
    budget = target_s * rate
    acc = flops1
    while n_docs < len(lengths):
        nxt = 14.0 * w.d * G * float(lengths[n_docs] * (lengths[n_docs] + 1) // 2)
        if acc + nxt > budget:
            break
        acc += nxt
        n_docs += 1
    Tn = int(cu[n_docs])
    sl = slice(0, Tn)
    args = [t[sl, :G].double().numpy() if i not in (1, 2) else t[sl, :1].double().numpy()
            for i, t in enumerate((q, k, v, do))]
    t0 = time.perf_counter()
    oracle.attn_bwd(*args, cu[: n_docs + 1], w.scale)
    dt = time.perf_counter() - t0
    tflops = acc / dt / 1e12
    text = (f"oracle fp64 fwd+bwd on the first {n_docs} document(s) ({Tn} tokens), KV head 0 and its "
            f"{G} query head(s): {acc:.3g} FLOP in {dt:.1f} s")
    return tflops, cores, text, dt


def run_reference(args, w, world, rank):
    """--impl reference: the fp64 CPU oracle, as it stands, on a bounded sample."""
    if rank != 0:
        return
    vals = []
    text = ""
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.steps):
        v, cores, text, _ = cpu_oracle_sample(w, target_s=args.ref_seconds)
        vals.append(v)
    val = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**w.describe(), "path": "oracle fp64 (CPU)"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": text},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


KERNELS = {
    # per path: names of the intervals between the events the library records
    "bf16": (["schedule_fwd", "convert_v_f16", "fwd_kernel"],
             ["schedule_kv", "schedule_q", "convert_k_f16", "delta_kernel", "dkdv_kernel", "dq_kernel"]),
    "mxfp8": (["schedule_fwd", "quantize_kv", "fwd_kernel"],
              ["schedule_kv", "schedule_q", "delta_quantize_do", "dkdv_kernel", "dq_kernel"]),
}
KERNELS["nvfp4"] = KERNELS["mxfp8"]  # the same launches (the K pass also writes K's NVFP4 form)
# algorithmic tensor work of each attention kernel per visible (query, key)
# pair and query head, in units of d: forward S and PV = 4; dK/dV kernel S,
# dP, dV, dK = 8; dQ kernel S, dP, dQ = 6
KERNEL_FLOPS = {"fwd_kernel": 4.0, "dkdv_kernel": 8.0, "dq_kernel": 6.0}
# DRAM bytes (read + written) of one launch of each attention kernel on the
# 32K workload (config 4), from dram__bytes_read.sum + dram__bytes_write.sum
# of an ncu capture of the kernels as they stand; None where not measured.
# These must be taken again whenever a kernel changes.
MEASURED_TRAFFIC = {
    4: {"bf16": {"fwd_kernel": 1.325e9, "dkdv_kernel": 2.131e9, "dq_kernel": 1.610e9},
        # (the MXFP8 dK/dV kernel changed after its last capture: not measured)
        "mxfp8": {"fwd_kernel": 1.594e9, "dkdv_kernel": None, "dq_kernel": 1.354e9,
                  "quantize_kv": 1.034e9, "delta_quantize_do": 1.052e9},
        "nvfp4": {"fwd_kernel": 1.324e9, "dkdv_kernel": None, "dq_kernel": 1.368e9,
                  "quantize_kv": 1.111e9, "delta_quantize_do": 1.052e9}},
}


class Path:
    """Buffers and one timed fwd+bwd step of one precision path."""

    def __init__(self, fapk, w, prec, dev, tensors):
        self.fapk, self.w, self.prec, self.dev = fapk, w, prec, dev
        self.qd, self.kd, self.vd, self.dod = tensors
        seq = fapk.Seqlens(w.cu, dev)
        self.seq = seq
        self.P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=getattr(fapk, PREC[prec]))
        self.ws_f = fapk.workspace(self.P, fapk.FWD, dev)
        self.ws_b = fapk.workspace(self.P, fapk.BWD, dev)
        self.o = torch.empty((w.T, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((w.Hq, w.T), dtype=torch.float32, device=dev)
        self.dq = torch.empty((w.T, w.Hq, w.d), dtype=torch.float32, device=dev)
        self.dk = torch.empty((w.T, w.Hkv, w.d), dtype=torch.float32, device=dev)
        self.dv = torch.empty((w.T, w.Hkv, w.d), dtype=torch.float32, device=dev)
        self.ctx = torch.empty(max(fapk.ctx_size(self.P), 256), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)

    def step(self, timers=None):
        f = self.fapk
        Pf = timers[0].with_events(self.P) if timers else self.P
        Pb = timers[1].with_events(self.P) if timers else self.P
        f.attn_fwd(Pf, self.qd, self.kd, self.vd, o=self.o, lse=self.lse, ctx=self.ctx, ws=self.ws_f,
                   stream=self.stream)
        f.attn_bwd(Pb, self.qd, self.kd, self.vd, self.o, self.lse, self.dod, ctx=self.ctx, dq=self.dq,
                   dk=self.dk, dv=self.dv, ws=self.ws_b, stream=self.stream)

    def balance(self, num_sms):
        """One untimed fwd + bwd with per-CTA time records: mean / max of the
        CTAs' busy times (start of the earliest CTA to each CTA's end), per
        persistent kernel, next to the same ratio of causal tile work when the
        units are handed out in order to the SM that frees up first."""
        f = self.fapk
        P = f.make_problem(self.seq, self.w.Hq, self.w.Hkv, self.w.d, self.w.scale,
                           prec=getattr(f, PREC[self.prec]), flags=f.FLAG_CTA_TIMES)
        f.attn_fwd(P, self.qd, self.kd, self.vd, o=self.o, lse=self.lse, ctx=self.ctx, ws=self.ws_f,
                   stream=self.stream)
        fwd = f.cta_times(P, f.FWD, 0, self.ws_f, self.stream)
        f.attn_bwd(P, self.qd, self.kd, self.vd, self.o, self.lse, self.dod, ctx=self.ctx, dq=self.dq,
                   dk=self.dk, dv=self.dv, ws=self.ws_b, stream=self.stream)
        kv = f.cta_times(P, f.BWD, 0, self.ws_b, self.stream)
        qk = f.cta_times(P, f.BWD, 1, self.ws_b, self.stream)
        ana = analytic_balance(self.w, self.prec, num_sms)
        out = {}
        for name, t in (("fwd_kernel", fwd), ("dkdv_kernel", kv), ("dq_kernel", qk)):
            busy = (t[:, 1] - t[:, 0].min()).astype(np.float64)
            out[name] = {"measured": float(busy.mean() / busy.max()), "analytic": ana[name], "ctas": int(len(t)),
                         "max_ms": float(busy.max() / 1e6)}
        return out

    def status_ok(self):
        return self.fapk.status(self.ws_f) == 0 and self.fapk.status(self.ws_b) == 0

    def timed_graph(self, steps, warmup):
        """ms per step of the same fwd + bwd captured once into a CUDA graph and
        replayed (no host launch work inside the timed region)."""
        s = torch.cuda.Stream(self.dev)
        s.wait_stream(self.stream)
        saved = self.stream
        self.stream = s
        with torch.cuda.stream(s):
            self.step()  # eager once on the capturing stream
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self.step()
        self.stream = saved
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize(self.dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize(self.dev)
        del g
        return e0.elapsed_time(e1) / steps

    def timed(self, steps, warmup, world):
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize(self.dev)
        if not self.status_ok():
            raise RuntimeError(f"{self.prec}: device status {self.fapk.status(self.ws_f)}/{self.fapk.status(self.ws_b)}")
        nf, nb = (len(x) + 1 for x in KERNELS[self.prec])
        timers = [(self.fapk.KernelTimer(nf), self.fapk.KernelTimer(nb)) for _ in range(steps)]
        launches0 = self.fapk.launch_count()
        barrier(world)
        torch.cuda.synchronize(self.dev)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(self.stream)
        for i in range(steps):
            self.step(timers[i])
        end.record(self.stream)
        torch.cuda.synchronize(self.dev)
        barrier(world)
        launches = self.fapk.launch_count() - launches0
        total_ms = max_over_ranks(start.elapsed_time(end), world, self.dev)
        names = KERNELS[self.prec][0] + KERNELS[self.prec][1]
        per = [tf.durations_ms() + tb.durations_ms() for tf, tb in timers]
        kern_ms = {n: max_over_ranks(statistics.mean(row[i] for row in per), world, self.dev)
                   for i, n in enumerate(names)}
        return total_ms / steps, kern_ms, launches


def analytic_balance(w, prec, num_sms):
    """Mean / max per-SM causal tile work (128 x 128 tile pairs) of each
    persistent kernel when its units, in the scheduler's order (documents by
    tile count, longest first; head by head; each head's tiles longest work
    first), go one by one to the SM that frees up first."""
    import heapq
    lengths = np.diff(w.cu.astype(np.int64))
    G = w.Hq // w.Hkv

    def units(rows, H, work_of):
        nts = [int((L + rows - 1) // rows) for L in lengths]
        order = sorted([k for k in range(len(lengths)) if nts[k] > 0], key=lambda k: -nts[k])
        for k in order:
            for _ in range(H):
                for r in range(nts[k]):
                    yield work_of(k, nts[k], r)

    def fwd_pair(k, nt, r):  # 256-row unit: query tiles 2u (and 2u + 1 if present)
        u = nt - 1 - r
        n0 = 2 * u + 1
        n1 = 2 * u + 2 if 256 * u + 128 < lengths[k] else 0
        return n0 + n1

    def ratio(gen):
        heap = [(0.0, i) for i in range(num_sms)]
        loads = [0.0] * num_sms
        n = 0
        for work in gen:
            t, i = heapq.heappop(heap)
            loads[i] += work
            heapq.heappush(heap, (t + work, i))
            n += 1
        used = loads[: min(n, num_sms)]
        return float(np.mean(used) / max(used)) if used and max(used) > 0 else 1.0

    if prec != "bf16":
        fwd = ratio(units(128, w.Hq, lambda k, nt, r: nt - r))
    else:
        fwd = ratio(units(256, w.Hq, fwd_pair))
    nq = lambda k: (lengths[k] + 127) // 128
    return {"fwd_kernel": fwd,
            "dkdv_kernel": ratio(units(128, w.Hkv, lambda k, nt, r: G * (nt - r))),
            "dq_kernel": ratio(units(128, w.Hq, lambda k, nt, r: nt - r))}


def path_report(w, prec, ms_per_step, kern_ms, launches, world, peaks, clk, config=None):
    flops = w.flops()
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    pairs = w.pairs()
    fwd_names, bwd_names = KERNELS[prec]
    fwd_ms = sum(kern_ms[n] for n in fwd_names)
    bwd_ms = sum(kern_ms[n] for n in bwd_names)
    dom = max(KERNEL_FLOPS, key=lambda n: kern_ms[n])
    dom_flops = KERNEL_FLOPS[dom] * w.d * w.Hq * pairs
    achieved = dom_flops / (kern_ms[dom] * 1e-3) / 1e12
    peak, peak_src = tensor_peak(peaks, clk, prec != "bf16")
    kpeak = {n: peak * (NV_PEAK_FACTOR[n] if prec == "nvfp4" else 1.0) for n in KERNEL_FLOPS}
    if prec == "nvfp4":
        peak *= NV_PEAK_FACTOR[dom]
        peak_src = (f"{NV_PEAK_FACTOR[dom]:.4f} x " + peak_src + " (the scores' FP4 MMAs at twice the FP8 "
                    "rate, weighted by the kernel's products)")
    dense = DENSE_BF16_TFLOPS if prec == "bf16" else DENSE_FP8_TFLOPS
    traffic = MEASURED_TRAFFIC.get(config, {}).get(prec, {}).get(dom)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "traffic_unit": "bytes per launch",
                "kernel": dom, "peak_source": peak_src,
                "sm_mhz_median": clk.get("sm_mhz") if clk else None,
                "frac_of_dense_datasheet": achieved / dense,
                "kernels_ms": kern_ms,
                "kernels_tflops": {n: KERNEL_FLOPS[n] * w.d * w.Hq * pairs / (kern_ms[n] * 1e-3) / 1e12
                                   for n in KERNEL_FLOPS},
                "kernels_frac": {n: KERNEL_FLOPS[n] * w.d * w.Hq * pairs / (kern_ms[n] * 1e-3) / 1e12 / kpeak[n]
                                 for n in KERNEL_FLOPS},
                "fwd": {"ms": fwd_ms, "tflops": 4.0 * w.d * w.Hq * pairs / (fwd_ms * 1e-3) / 1e12},
                "bwd": {"ms": bwd_ms, "tflops": 10.0 * w.d * w.Hq * pairs / (bwd_ms * 1e-3) / 1e12}}
    out = {"value": value, "ms_per_step": ms_per_step, "pct_of_dense_peak": 100.0 * (value / world) / dense,
           "dense_peak_tflops": dense, "roofline": roofline, "gpu_launches": launches}
    if prec != "bf16":
        # the standalone quantisation launch of the forward (K and V, both
        # forms; HBM bound), algorithmic bytes per element: 2 B bf16 read, then
        # per form 1 B of E4M3 codes and 1/32 B of scales written.  Q is
        # quantised on load inside the forward kernel, dO inside the D pass.
        qbytes = 2 * w.T * w.Hkv * w.d * (2.0 + 2 * (1.0 + 1.0 / 32))
        if prec == "nvfp4":  # K's NVFP4 form too: 1/2 B of codes and 1/16 B of scales per element
            qbytes += w.T * w.Hkv * w.d * (0.5 + 1.0 / 16)
        gbs = qbytes / (kern_ms["quantize_kv"] * 1e-3) / 1e9
        qtraffic = MEASURED_TRAFFIC.get(config, {}).get(prec, {})
        out["roofline_quantize"] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": gbs / peaks["hbm_gbs"], "traffic": qtraffic.get("quantize_kv"),
                                    "algorithmic_bytes": qbytes,
                                    "kernel": "quantize_mxfp8_kernel (K and V in one launch; both forms)"}
        # the D pass with dO's quantisation: reads dO, O and O's residual
        # (6 B), writes dO's two forms (2 + 1/16 B) per element and D
        dbytes = w.T * w.Hq * w.d * (6.0 + 2 * (1.0 + 1.0 / 32)) + 4.0 * w.T * w.Hq
        gbs = dbytes / (kern_ms["delta_quantize_do"] * 1e-3) / 1e9
        out["roofline_delta_quantize_do"] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                                             "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                                             "traffic": qtraffic.get("delta_quantize_do"),
                                             "algorithmic_bytes": dbytes}
        out["quantize_ms_per_step"] = kern_ms["quantize_kv"] + kern_ms["delta_quantize_do"]
    return out


def time_qkv_proj(fapk, w, dev, peaks, clk, warmup, steps):
    """CUDA-event time of fapk_qkv_proj_mxfp8 on the workload's tokens: x
    [T, Hq d] bf16 against w [(Hq + 2 Hkv) d, Hq d]; 2 T d_model N FLOP."""
    g = torch.Generator(device=dev).manual_seed(5)
    Dm = w.Hq * w.d
    N = (w.Hq + 2 * w.Hkv) * w.d
    x = torch.randn((w.T, Dm), generator=g, device=dev).to(torch.bfloat16)
    wt = (torch.randn((N, Dm), generator=g, device=dev) / Dm ** 0.5).to(torch.bfloat16)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.MXFP8)
    ws = fapk.workspace(P, fapk.FWD, dev)
    for _ in range(warmup):
        fapk.qkv_proj_mxfp8(P, x, wt, ws=ws)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fapk.qkv_proj_mxfp8(P, x, wt, ws=ws)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    flops = 2.0 * w.T * Dm * N
    tf = flops / (ms * 1e-3) / 1e12
    peak, src = tensor_peak(peaks, clk, False)
    return {"ms": ms, "tflops": tf, "frac": tf / peak, "peak": peak, "peak_source": src,
            "shape": {"tokens": w.T, "d_model": Dm, "n_out": N}, "status_ok": fapk.status(ws) == 0,
            "note": "includes the schedule launch and the MX forms of K and V written by the epilogue"}


def time_quantized_kv(fapk, w, dev, tensors, peaks, clk, warmup, steps):
    """CUDA-event time of fapk_attn_fwd_quantized_kv (the MXFP8 forward over
    K and V given in both MX forms, as a cache would hold them: no
    quantisation launch) on the workload; 4 d Hq pairs FLOP."""
    qd, kd, vd = tensors[:3]
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.MXFP8)
    kf = fapk.quantize_mxfp8(kd, seq)
    vf = fapk.quantize_mxfp8(vd, seq)
    ws = fapk.workspace(P, fapk.FWD, dev)
    o = torch.empty((w.T, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.Hq, w.T), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        fapk.attn_fwd_quantized_kv(P, qd, kf, vf, o=o, lse=lse, ws=ws)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fapk.attn_fwd_quantized_kv(P, qd, kf, vf, o=o, lse=lse, ws=ws)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    tf = 4.0 * w.d * w.Hq * w.pairs() / (ms * 1e-3) / 1e12
    peak, src = tensor_peak(peaks, clk, True)
    return {"ms": ms, "tflops": tf, "frac": tf / peak, "peak": peak, "peak_source": src,
            "status_ok": fapk.status(ws) == 0,
            "note": "forward only, K and V pre-quantised; includes the schedule launch"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fapk", choices=["fapk", "reference"])
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--paths", default="bf16,mxfp8,nvfp4")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--ref-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--qkv-proj", type=int, default=1, help="also time the fused QKV projection (0: skip)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from causal_flash_attention_packed_b200 import workloads as W
    w = W.config(args.config, args.seed)

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return

    world, rank, local = dist_setup()
    from causal_flash_attention_packed_b200 import fapk
    fapk.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()

    q, k, v, do = w.tensors()
    dev_tensors = tuple(t.to(dev) for t in (q, k, v, do))
    paths = [p for p in args.paths.split(",") if p]
    runners = {p: Path(fapk, w, p, dev, dev_tensors) for p in paths}

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    timed = {}
    for p in paths:
        timed[p] = runners[p].timed(args.steps, args.warmup, world)
    clk = clocks.stop() if clocks else None
    results = {p: path_report(w, p, *timed[p], world, peaks, clk, config=args.config) for p in paths}
    st_ok = all(r.status_ok() for r in runners.values())
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    balance = {p: runners[p].balance(num_sms) for p in paths}
    st_ok = st_ok and all(r.status_ok() for r in runners.values())

    # the fused QKV projection with K's and V's MX quantisation in its epilogue,
    # on the same tokens (d_model = Hq d, as for a model whose heads span it);
    # timed on its own: it precedes the attention step in a training step
    proj = None
    if args.qkv_proj and w.d == 128:
        proj = time_qkv_proj(fapk, w, dev, peaks, clk, args.warmup, min(args.steps, 20))

    # the main path's step captured into a CUDA graph and replayed
    graph = None
    if world == 1:
        gms = runners[paths[0]].timed_graph(args.steps, args.warmup)
        graph = {"ms_per_step": gms, "value": w.flops() / (gms * 1e-3) / 1e12, "unit": "TFLOP/s",
                 "path": paths[0], "note": "fwd + bwd captured once into a CUDA graph, replayed"}

    # the forward over pre-quantised K and V (a quantised KV cache)
    qkv_cached = None
    if w.d == 128:
        qkv_cached = time_quantized_kv(fapk, w, dev, dev_tensors, peaks, clk, args.warmup, min(args.steps, 20))

    # end to end through the C ABI with host buffers (pinned), copies included:
    # every step copies its inputs host -> device and its outputs device ->
    # host.  The copies run on their own streams, pipelined with the kernels
    # (the inputs of step i + 1 and the outputs of step i - 1 move while step
    # i computes), with two sets of device buffers, as a training loop that
    # streams its batches would run it.
    e2e = None
    main_path = paths[0]
    if args.e2e_steps > 0:
        sets = [runners[main_path],
                Path(fapk, w, main_path, dev, tuple(torch.empty_like(t) for t in dev_tensors))]
        comp = sets[0].stream
        s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        hin = [t.pin_memory() for t in (q, k, v, do)]
        outs_of = lambda R: (R.o, R.lse, R.dq, R.dk, R.dv)  # noqa: E731
        houts = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs_of(R)] for R in sets]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in houts[0])
        n = args.e2e_steps
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, comp_done, out_done = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
        barrier(world)
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_h2d)
        for i in range(n):
            b = i % 2
            R = sets[b]
            if i >= 2:
                s_h2d.wait_event(comp_done[i - 2])  # step i - 2 has read this set's inputs
            with torch.cuda.stream(s_h2d):
                for src, dst in zip(hin, (R.qd, R.kd, R.vd, R.dod)):
                    dst.copy_(src, non_blocking=True)
            in_ready[i].record(s_h2d)
            comp.wait_event(in_ready[i])
            if i >= 2:
                comp.wait_event(out_done[i - 2])  # step i - 2's outputs have left this set
            R.step()
            comp_done[i].record(comp)
            s_d2h.wait_event(comp_done[i])
            with torch.cuda.stream(s_d2h):
                for src, dst in zip(outs_of(R), houts[b]):
                    dst.copy_(src, non_blocking=True)
            out_done[i].record(s_d2h)
        e1.record(s_d2h)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n
        e2e = {"value": w.flops() * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "path": main_path, "steps": n,
               "copies": "H2D and D2H on their own streams, pipelined with the kernels (two buffer sets)"}
        st_ok = st_ok and sets[1].status_ok()

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v_cpu, cores, text, _ = cpu_oracle_sample(w, target_s=15.0)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": text}
    head = results[main_path]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if main_path == "bf16" else "e4m3/e8m0", "data": "synthetic",
        "config": {**w.describe(), "path": main_path, "parallelism": f"replicas x{world}",
                   "l2": f"inputs {sum(t.numel() * 2 for t in (q, k, v, do)) / 1e9:.2f} GB > 126 MB L2, no flush"},
        "pct_of_dense_bf16_peak": head["pct_of_dense_peak"] if main_path == "bf16" else None,
        "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": sum(r["gpu_launches"] for r in results.values()),
        "clocks": clk, "status_ok": st_ok, "qkv_proj": proj, "fwd_quantized_kv": qkv_cached, "graph": graph,
        "scheduler_balance": balance,
    }
    for p in paths[1:]:
        line[p] = results[p]
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
