#!/usr/bin/env python
"""Throughput of the quantized attention forward pass on B200.

One step = the whole hot path on one batch of synthetic input: the smooth +
quantize pre-pass (K mean, INT8 Q/K, E4M3 V) followed by the attention kernel
(INT8 QK^T, online softmax, E4M3 P~V).  Metric: attention TOPS =
4*B*H*S^2*D / time (halved for causal), the figure the SageAttention pages
quote for their kernels.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one process per GPU; every rank runs
the same workload on its own GPU (independent problems, no data-path
collective: weak scaling) and the elapsed time is the maximum over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "b2_h32_s4096_d128"
METRIC = "attention TOPS (4BHS²D/t) at D=128, S=4K–32K; % of B200 INT8/FP8 peak"
FALLBACK_BF16 = 1590.0             # TFLOP/s burst, used only without the measured peaks file
FALLBACK_BF16_SUSTAINED = 1400.0   # TFLOP/s sustained, likewise
FP8_OVER_BF16 = 2.0                # nominal dense ratio (4.5 / 2.25 PFLOP/s); INT8 = FP8 on B200
SUSTAINED_AFTER_S = 2.0            # timed regions longer than this are compared with the sustained peak


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=WORKLOAD)
    ap.add_argument("--pv", default="fp8", choices=["fp8", "fp16"])
    ap.add_argument("--pv-accum", default="fp32", choices=["fp32", "fp32+fp32", "fp32_lazy", "fp32+fp16"])
    ap.add_argument("--gran", default="per_block", choices=["per_block", "per_warp", "per_thread", "per_token"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the attention-kernel sweep over S")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return d, "measured"
    except Exception:
        return {"bf16_tflops": FALLBACK_BF16, "bf16_tflops_sustained": FALLBACK_BF16_SUSTAINED,
                "hbm_gbs": 6650.0}, "fallback"


def tensor_peak(pk: dict, region_s: float):
    """Dense INT8/FP8 peak (TOPS) for a kernel timed over a region of
    region_s seconds: 2 x the measured bf16 burst figure for short regions,
    2 x the sustained (power-capped) figure for regions of seconds."""
    if region_s > SUSTAINED_AFTER_S:
        return FP8_OVER_BF16 * float(pk.get("bf16_tflops_sustained", FALLBACK_BF16_SUSTAINED)), "sustained"
    return FP8_OVER_BF16 * float(pk.get("bf16_tflops", FALLBACK_BF16)), "burst"


class NvmlClocks:
    """In-process NVML sampling (read-only queries) of the SM clock and the
    clock-event reasons every ~1 ms, so that even a region of ~10 ms has a
    clock record of its own."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int, period_s: float = 0.001):
        self.idx, self.period = gpu_index, period_s
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        self.stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self.stop.set()
        if self.ok:
            self.t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, in-process, ~1 ms"}


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed
    region (used when NVML cannot be opened in-process)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.idx)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def strip_comments(src: str) -> str:
    """C/C++ source without its // and /* */ comments, every run of whitespace
    outside string and character literals collapsed to one space, so that an
    edit of comments or layout leaves the hash alone."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c.isspace():
            out.append(" ")
            i += 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash():
    """Hash of the attention kernel's sources without comments: the recorded
    ncu traffic is used only while it matches."""
    h = hashlib.sha256()
    for f in ("attn_fwd.cu", "sage_common.cuh", "sage_launch.cuh"):
        src = open(os.path.join(ROOT, "quantized_attention_token_b200", "csrc", f), encoding="utf-8").read()
        h.update(strip_comments(src).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, mode: str):
    """dram bytes per launch of the attention kernel in `mode` ("pv/accum")
    from the committed ncu summary, if it was taken on the current kernel
    source; else None."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    e = d.get(f"{workload} {mode}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def max_over_ranks(x: float, device) -> float:
    """The maximum of x over the ranks of the default process group (x itself
    without one): a multi-GPU time is the slowest rank's."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(world: int, ops_per_step: float, steps: int, elapsed_ms: float) -> float:
    """Whole-job TOPS: each of `world` ranks ran `steps` steps of
    `ops_per_step` ops in `elapsed_ms` (the slowest rank's time)."""
    return world * ops_per_step * steps / (elapsed_ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- CPU oracle
def cpu_baseline(spec: synth.Spec, q, k, v, pv: str, budget_s: float):
    """The oracle as it stands, on a bounded sample of the workload: whole
    query tiles (128 rows, all keys) of a few heads, pre-pass included."""
    import oracle
    oracle.lib()
    tiles_per_head = (spec.S + 127) // 128
    heads = [(b, h) for b in range(spec.B) for h in range(spec.Hq)]
    rng = np.random.default_rng(0)
    order = rng.permutation(len(heads))
    done_rows, t0, sample = 0, time.perf_counter(), []
    grp = spec.Hq // spec.Hkv
    for i in order:
        b, h = heads[i]
        hk = h // grp
        qt = int(rng.integers(0, tiles_per_head))
        rows = (qt * 128, min(spec.S, qt * 128 + 128))
        if spec.layout == "HND":
            qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1]
        else:
            qs, ks, vs = q[b:b + 1, :, h:h + 1], k[b:b + 1, :, hk:hk + 1], v[b:b + 1, :, hk:hk + 1]
        oracle.attention(qs, ks, vs, spec.layout, spec.causal, pv=pv, q_rows={(0, 0): rows})
        done_rows += rows[1] - rows[0]
        sample.append(f"b{b}h{h}t{qt}")
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    ops = 4.0 * done_rows * spec.S * spec.D * (0.5 if spec.causal else 1.0)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{len(sample)} query tiles x 128 rows x all {spec.S} keys (+ their K/V/Q pre-pass) of "
                      f"{spec.name}, {dt:.1f} s, scaled by the ops of the rows computed"}


# ----------------------------------------------------------------------------- S sweep
def sweep_s(sage, dev, gran, n=20):
    """The attention kernel alone over the metric's sequence axis: S in
    1K..32K with B = 32768 / S, H = 32, D = 128, FP8 and 16-bit P~V, causal
    and not (one-level accumulation), on seeded iid N(0,1) fp16 inputs drawn
    on the device.  TOPS from CUDA events over n launches, and the fraction
    of the burst dense FP8/INT8 peak."""
    pk, _ = peaks()
    peak, _ = tensor_peak(pk, 0.0)
    g = torch.Generator(device=dev)
    res = {}
    for S in (1024, 2048, 4096, 8192, 16384, 32768):
        Bs, H, D = 32768 // S, 32, 128
        g.manual_seed(S)
        q, k, v = (torch.randn(Bs, H, S, D, generator=g, device=dev, dtype=torch.float32).half() for _ in range(3))
        o = torch.empty_like(q)
        w = torch.empty(sage.sage_workspace_bytes(Bs, H, H, S, D, 1, 0), dtype=torch.uint8, device=dev)
        for pv in ("fp8", "fp16"):
            sage.quant_qkv(q, k, v, w, "HND", gran, pv)
            for causal in (False, True):
                def f():
                    sage.attn_quantized(o, w, Bs, H, H, S, D, "HND", causal, None, gran, pv, "fp32")
                for _ in range(3):
                    f()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                e0.record()
                for _ in range(n):
                    f()
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / n
                tops = 4.0 * Bs * H * S * S * D * (0.5 if causal else 1.0) / (ms * 1e-3) / 1e12
                res[f"S{S}/{pv}/{'causal' if causal else 'full'}"] = {"tops": round(tops, 1),
                                                                       "frac": round(tops / peak, 4)}
        del q, k, v, o, w
    return {"workload": "B=32768/S, H=32, D=128, fp16 iid N(0,1), HND, one-level accumulation", "gran": gran,
            "peak": peak, "points": res}


def bench_config(spec: synth.Spec, args) -> dict:
    """The workload description both arms print (the reference arm times the
    oracle on the same workload)."""
    elem = spec.total_tokens * spec.D
    return {"workload": spec.name, "B": spec.B, "H": spec.Hq, "Hkv": spec.Hkv, "S": spec.S, "D": spec.D,
            "layout": spec.layout, "causal": spec.causal, "input_dtype": spec.dtype, "qk_gran": args.gran,
            "pv": args.pv, "pv_accum": args.pv_accum,
            "l2": "inputs larger than L2: Q/K/V %s = %d MiB per GPU, L2 126 MB" % (
                spec.dtype, (spec.Hq + 2 * spec.Hkv) * elem * 2 >> 20)}


# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    spec = synth.CONFIGS[args.config]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    ops = spec.attention_ops()

    if args.impl == "reference":
        if rank != 0:
            return
        q, k, v = synth.make(spec)
        per_step, wall_ms = [], []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            cb = cpu_baseline(spec, q, k, v, args.pv, max(1.0, args.cpu_seconds / max(1, args.steps)))
            if i >= args.warmup:
                per_step.append(cb["value"])
                wall_ms.append((time.perf_counter() - t0) * 1e3)
        val = float(np.median(per_step))
        cb["value"] = val
        # each step times a bounded sample of the workload (cpu_baseline's
        # "sample"): ms_per_step is what one such step took; the whole
        # workload at the same rate is reported beside it
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TOPS", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.median(wall_ms)),
                "ms_per_full_workload_at_this_rate": ops / (val * 1e12) * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8+e4m3 (f64 oracle)",
                "data": "synthetic",
                "config": bench_config(spec, args),
                "cpu_baseline": cb,
                "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import quantized_attention_token_b200 as sage
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    q_h, k_h, v_h = synth.make(spec)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    out = torch.empty_like(q)
    B, H, S, D = spec.B, spec.Hq, spec.S, spec.D
    layout = spec.layout
    pv_code = sage.PV[args.pv]
    ws = torch.empty(sage.sage_workspace_bytes(B, spec.Hq, spec.Hkv, S, D, pv_code, 0), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        sage.quant_qkv(q, k, v, ws, layout, args.gran, args.pv)
        if ev is not None:
            ev[1].record(stream)
        sage.attn_quantized(out, ws, B, spec.Hq, spec.Hkv, S, D, layout, spec.causal, None, args.gran, args.pv,
                            args.pv_accum)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, bits = sage.get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with NvmlClocks(local) as nclk, Clocks(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = start.elapsed_time(stop)
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    pre_ms = [e[0].elapsed_time(e[1]) for e in evs]
    elapsed_ms = max_over_ranks(elapsed_ms, dev)
    st, bits = sage.get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} after the timed region")

    ms_per_step = elapsed_ms / args.steps
    value = job_tops(world, ops, args.steps, elapsed_ms)

    # the attention kernel alone in the other modes the workload names (and
    # the conditional-rescaling mode), inputs resident, CUDA events
    def kernel_ms(pv, acc, n=100):
        sage.quant_qkv(q, k, v, ws, layout, args.gran, pv)

        def f():
            sage.attn_quantized(out, ws, B, spec.Hq, spec.Hkv, S, D, layout, spec.causal, None, args.gran, pv, acc)

        for _ in range(3):
            f()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        m0.record(stream)
        for _ in range(n):
            f()
        m1.record(stream)
        torch.cuda.synchronize()
        return m0.elapsed_time(m1) / n

    other_ms = {(pv, acc): kernel_ms(pv, acc)
                for pv, acc in [("fp8", "fp32+fp32"), ("fp8", "fp32_lazy"), ("fp8", "fp32+fp16"), ("fp16", "fp32"),
                                ("fp16", "fp32+fp32"), ("fp16", "fp32_lazy")] if (pv, acc) != (args.pv, args.pv_accum)}
    other_modes = {f"{pv}/{acc}": ops / (ms * 1e-3) / 1e12 for (pv, acc), ms in other_ms.items()}
    sweep = None if args.no_sweep or world > 1 else sweep_s(sage, dev, args.gran)

    # end to end through the public API with host buffers: every step copies
    # q, k, v in from pinned host memory, runs sageattn and copies the output
    # back.  Steps are pipelined over three streams (inputs in, compute,
    # output out) with two sets of device buffers and workspaces, so step
    # i's input copy overlaps step i-1's pass and step i-2's output copy; the
    # host link's input bandwidth bounds the rate.
    qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
    op = [torch.empty_like(q_h).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dbuf = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(q)) for _ in range(2)]
    wss = [ws, torch.empty_like(ws)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_done + ev_out:
        e.record(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step(i):
        b = i % 2
        qd, kd, vd, od = dbuf[b]
        with torch.cuda.stream(s_in):              # buffer b is free once step i-2 computed and copied out
            s_in.wait_event(ev_done[b])
            s_in.wait_event(ev_out[b])
            qd.copy_(qp, non_blocking=True)
            kd.copy_(kp, non_blocking=True)
            vd.copy_(vp, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        sage.sageattn(qd, kd, vd, layout, spec.causal, qk_quant_gran=args.gran, pv_dtype=args.pv,
                      pv_accum_dtype=args.pv_accum, out=od, workspace=wss[b])
        ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            op[b].copy_(od, non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(args.e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    pk, pk_kind = peaks()
    peak, peak_kind = tensor_peak(pk, elapsed_ms * 1e-3)
    attn_avg = float(np.mean(attn_ms))
    achieved = ops / (attn_avg * 1e-3) / 1e12
    two = ("fp8", "fp32+fp32") if args.pv == "fp8" else ("fp16", "fp32+fp32")
    two_ms = other_ms.get(two)
    pre_avg = float(np.mean(pre_ms))
    elem = spec.total_tokens * D
    pre_bytes = elem * (2 * spec.Hq + 4 * spec.Hkv) + elem * (spec.Hq + 2 * spec.Hkv)   # 9 B/elem at Hq=Hkv
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8+e4m3" if args.pv == "fp8" else "int8+f16", "data": "synthetic",
        "config": bench_config(spec, args),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(spec.name, f"{args.pv}/{args.pv_accum}"),
                     "kernel": "attn_fwd_kernel", "kernel_ms": attn_avg,
                     "mode": f"{args.pv}/{args.pv_accum}",
                     "peak_source": f"2 x bf16_tflops {peak_kind} ({pk_kind}: the dense FP8/INT8 rate is twice "
                                    f"bf16's); timed region {elapsed_ms:.1f} ms"},
        "roofline_two_level": None if two_ms is None else {
            "bound": "tensor", "achieved": ops / (two_ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
            "frac": ops / (two_ms * 1e-3) / 1e12 / peak, "traffic": recorded_traffic(spec.name, f"{two[0]}/{two[1]}"),
            "kernel": "attn_fwd_kernel",
            "kernel_ms": two_ms, "mode": f"{two[0]}/{two[1]}",
            "note": "the two-level accumulation (the API default), attention kernel alone, 100 launches"},
        "prepass": {"ms": pre_avg, "achieved_gbs": pre_bytes / (pre_avg * 1e-3) / 1e9,
                    "peak_gbs": float(pk.get("hbm_gbs", 0)),
                    "frac": pre_bytes / (pre_avg * 1e-3) / 1e9 / float(pk.get("hbm_gbs", 1))},
        "e2e": {"value": job_tops(world, ops, 1, e2e_ms), "unit": "TOPS",
                "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))),
                "d2h_bytes_per_step": int(q_h.numel() * q_h.element_size())},
        "attention_modes_tops": other_modes,   # attention kernel alone, other P~V / accumulation modes
        "attention_modes_frac": {m: t / peak for m, t in other_modes.items()},
        "sweep": sweep,
        "gpu_launches": 3 * args.steps,     # pre-pass launches A and B + the attention kernel
        "clocks": nclk.summary() or clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(spec, q_h, k_h, v_h, args.pv, args.cpu_seconds)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
