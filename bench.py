"""Benchmark: gated delta-rule chunked forward (Gated DeltaNet, B=8 H=8 T=4096 d=128,
chunk 64, bf16 in / fp32 state) on B200, plus the decode step (B=256 H=16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0. A step is one chunked forward over the whole batch
(o and S_T). Timing: W untimed steps, then K steps between CUDA events on the
launching stream, bracketed by a barrier and a device synchronize; the time is
the max over ranks. Two input sets (each 270 MB, larger than the 126 MB L2) are
alternated so no step reads the previous step's inputs from L2.
Multi-GPU: every rank runs its own batch (weak scaling, no data-path collective).
``--impl reference`` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gated_delta_rule_143_b200.inputs import (CHUNK_WORKLOADS, DECODE_WORKLOADS, WORKLOAD_SEEDS,  # noqa: E402
                                              make_decode_state, make_decode_step, workload_inputs)

WORKLOAD = "gdn_bf16_b8_h8_t4096_d128"
DECODE = "gdn_decode_bf16_b256_h16_d128"
METRIC = "gated-delta-rule fwd tokens/s on 1 B200; % of roofline (TC FLOP/s or HBM GB/s)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- counts --
def chunk_flops_per_token_head(C, dk, dv):
    """Dense chunk-tile flops of the chunk form per token-head: A, W, QK^T (C*dk each),
    U and P.Delta (C*dv each), W S^T, Delta^T K and Q S^T (dk*dv each)."""
    return 2 * (C * (3 * dk + 2 * dv) + 3 * dk * dv)


def chunk_bytes(w):
    """Algorithmic HBM bytes of one forward: q, k, v read once and o written once, all in the input
    dtype; beta and g read once; S_T written once (S0 is null for these workloads). 1032 bytes per
    token-head for bf16 Gated DeltaNet at d = 128, plus 64 KiB of S_T per (b, h)."""
    eb = 2 if w.dtype == "bf16" else 4
    th = w.B * w.T * w.H
    g = 0 if w.mode == "none" else (4 if w.mode == "scalar" else 4 * w.dk)
    per_th = eb * (2 * w.dk + w.dv) + eb * w.dv + 4 + g
    return th * per_th + w.B * w.H * w.dv * w.dk * 4


def o_fp32_extra_bytes(w):
    """Bytes the default fp32 output writes beyond an output in the input dtype (implementation
    traffic of the precision choice, not algorithmic)."""
    eb = 2 if w.dtype == "bf16" else 4
    return w.B * w.T * w.H * w.dv * (4 - eb)


def kernel_bytes(w, plan, c1):
    """Algorithmic HBM bytes per launch of each kernel of the chosen plan, as (name, bytes) in launch
    order. The inputs q, k, v, beta, g are read once by whichever kernel prepares a chunk; o and
    S_T are written once by the kernel that runs the state passes. Hand-off blocks exchanged
    through the workspace or the ring are implementation traffic, not algorithmic bytes (they
    show up in the ncu DRAM counters)."""
    eb = 2 if w.dtype == "bf16" else 4
    th = w.B * w.T * w.H
    g = 0 if w.mode == "none" else (4 if w.mode == "scalar" else 4 * w.dk)
    inputs = th * (eb * (2 * w.dk + w.dv) + 4 + g)
    outputs = th * eb * w.dv + w.B * w.H * w.dv * w.dk * 4
    if plan == "two_pass":
        return [("chunk_prep", inputs), ("chunk_state", outputs)]
    if plan == "prep_fused":
        nc = -(-w.T // w.chunk)
        pre = inputs * c1 // nc
        return [("chunk_prep", pre), ("chunk_fused", inputs - pre + outputs)]
    if plan == "scan":
        # prep reads the inputs; the state kernel's o^0 and read-outs are intermediate; the carry
        # writes S_T and the correction writes o
        st = w.B * w.H * w.dv * w.dk * 4
        return [("chunk_prep", inputs), ("chunk_state", 0), ("scan_carry", st), ("scan_correct", outputs - st)]
    return [("chunk_fused" if plan == "fused" else "chunk_simt", inputs + outputs)]


def decode_bytes(w):
    """S read and written once (fp32); q, k, v read and o written in the input dtype; beta and g
    read (2 * 4 * d_k * d_v + 1032 bytes per head-step for bf16 Gated DeltaNet at d = 128)."""
    eb = 2 if w.dtype == "bf16" else 4
    nh = w.B * w.H
    g = 0 if w.mode == "none" else (4 if w.mode == "scalar" else 4 * w.dk)
    return nh * (2 * 4 * w.dk * w.dv + eb * (2 * w.dk + w.dv) + eb * w.dv + 4 + g)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks --
class NvmlClockSampler:
    """SM clock, power and clock-event reasons read through NVML every ~0.5 ms on a host thread, from
    start() to stop(); summary() keeps the samples taken between mark_begin() and mark_end() (the
    timed region), so that a region of a few milliseconds still has samples. Reads only."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, dev_index: int):
        import pynvml
        import threading
        self.nv = pynvml
        pynvml.nvmlInit()
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
        except Exception:
            pass
        h = None
        if uuid:
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = None
        if h is None:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[dev_index]) if vis and vis.split(",")[dev_index].strip().isdigit() else dev_index
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
        self.h = h
        self.samples = []
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        try:
            mx = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception:
            mx = None
        pw, k = 0.0, 0
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = getr(self.h)
                if k % 8 == 0:
                    pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                k += 1
                self.samples.append((t, sm, mx, rs, pw))
            except Exception:
                pass
            time.sleep(0.0005)

    def start(self):
        self._thread.start()
        time.sleep(0.01)

    def mark_begin(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self._stop.set()
        self._thread.join(timeout=2)
        rows = [r for r in self.samples if self.t0 is not None and self.t0 <= r[0] <= (self.t1 or r[0])]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvml"}
        reasons = sorted({name for r in rows for bit, name in self.REASONS.items() if r[3] & bit})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max((r[2] or 0) for r in rows) or None,
                "reasons": reasons, "samples": len(rows), "power_w_max": round(max(r[4] for r in rows), 1),
                "source": "nvml, every ~0.5 ms during the timed region"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        """Starts sampling every 20 ms and returns once the first sample has arrived (so the
        samples cover the timed region that follows), or after 5 s."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            self.out.flush()
            if os.path.getsize(self.out.name) > 0:
                break
            time.sleep(0.01)
        self.size0 = os.path.getsize(self.out.name)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.out.flush()
        rows = []
        try:
            with open(self.out.name) as f:
                f.seek(self.size0)  # only samples taken after start() returned
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            os.unlink(self.out.name)
        return self._summary(rows)

    @staticmethod
    def _summary(rows):
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def smi_id(dev, local):
    """nvidia-smi --id for this process's device: its UUID when torch exposes it, else the
    physical index from CUDA_VISIBLE_DEVICES, else the local ordinal."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


# ------------------------------------------------------------- distributed --
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif n_gpus > 1:
        raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run (one process per GPU)")
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# Records whose device status check failed once and were run again: the expired wait's diagnostics
# (kind, block, thread, barrier or flag) as gdr_sync_status reports them. A second failure raises.
STATUS_RETRIES = []


def with_status_retry(name, fn, world):
    """Runs fn (a record ending in gdr.sync_status()) and, if the device status reports an error on
    any rank, runs it once more on every rank (the decision is reduced over ranks, so all ranks take
    the same collective steps); the failure is kept in STATUS_RETRIES and printed in the line."""
    import gated_delta_rule_143_b200 as gdr
    for attempt in range(2):
        err = None
        try:
            out = fn()
        except gdr.GdrError as e:
            out, err = None, str(e)
        if max_over_ranks(1.0 if err else 0.0, world) == 0.0:
            return out
        STATUS_RETRIES.append({"record": name, "attempt": attempt + 1, "error": err or "on another rank"})
    raise RuntimeError(f"{name}: the device status reported an error twice: {STATUS_RETRIES[-2:]}")


def max_over_ranks(x, world):
    """The maximum of a per-rank number over all ranks (device tensor under NCCL, host under gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, ms_per_step, world):
    """Whole-job rate under weak scaling: every rank processes `units_per_rank` per step and the
    step time is the slowest rank's (already the max over ranks)."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def rank_seed(base, rank, input_set):
    """Seed of one rank's input set: each rank runs its own independent batch."""
    return base + 1000 * rank + input_set


# ------------------------------------------------------------------- ours --
def time_device(fn, steps, warmup, world, stream):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)  # ms over `steps`


def run_ours(args):
    import gated_delta_rule_143_b200 as gdr

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    w = CHUNK_WORKLOADS[WORKLOAD]
    if args.batch:
        w = dataclasses.replace(w, B=args.batch)
    if args.seq:
        w = dataclasses.replace(w, T=args.seq)
    stream = torch.cuda.current_stream(dev)

    # two resident input sets, each larger than L2; one seed per rank (weak scaling)
    sets = []
    for s in range(2):
        x = workload_inputs(w, seed=rank_seed(WORKLOAD_SEEDS[WORKLOAD], rank, s))
        sets.append({k: (None if t is None else t.to(dev)) for k, t in x.items()})
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=dev)
    st = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
    ws_n = gdr.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.mode, torch.bfloat16, torch.float32)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev) if ws_n else None

    # per-kernel durations: an event before each step and one the library records after each of
    # its kernels (gdr_profile_next_call), all on the launching stream
    kernels_per_step = gdr_kernels_per_step(w)
    plan, c1 = gdr.chunk_fwd_plan(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.mode, torch.bfloat16, torch.float32)
    kb = kernel_bytes(w, plan, c1)
    assert len(kb) == kernels_per_step, (plan, kernels_per_step)
    names = [n for n, _ in kb]
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(kernels_per_step)] for _ in range(args.steps)]
    for e in ev0 + [e for row in evk for e in row]:
        e.record(stream)  # creates the event (torch creates them lazily)

    def step(i=0):
        x = sets[i & 1]
        ev0[i].record(stream)
        gdr.profile_next_call(evk[i])
        gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], mode=w.mode, chunk=w.chunk,
                      out=o, state_out=st, workspace=ws)

    def timed():
        try:
            clocks = NvmlClockSampler(local)
        except Exception:
            clocks = None
        if clocks is not None:
            clocks.start()  # sampling from the start of the warm-up, kept for the timed region only
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        if clocks is None:
            smi = ClockSampler(smi_id(dev, local))
            smi.start()
        else:
            clocks.mark_begin()
        ms = time_device(step, args.steps, 0, world, stream)
        if clocks is None:
            clk = smi.stop()
        else:
            clocks.mark_end()
            clk = clocks.stop()
        gdr.sync_status()
        return ms, clk

    ms, clk = with_status_retry("main", timed, world)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    tokens = w.B * w.T
    value = job_throughput(tokens, ms_step, world)

    nbytes = chunk_bytes(w)
    flops = chunk_flops_per_token_head(w.chunk, w.dk, w.dv) * w.B * w.T * w.H
    achieved_gbs = nbytes / (ms_step * 1e-3) / 1e9
    kb = dict(kb)
    kernels = []
    for j, name in enumerate(names):
        us = [1e3 * (evk[i][j - 1] if j else ev0[i]).elapsed_time(evk[i][j]) for i in range(args.steps)]
        us = max_over_ranks(statistics.mean(us), world)
        gbs = kb[name] / (us * 1e-6) / 1e9
        kernels.append({"kernel": name, "launch_us": round(us, 2), "share": None,
                        "algorithmic_bytes_per_launch": kb[name], "achieved_gbs": round(gbs, 1),
                        "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic_from_profile(name)})
    tot = sum(k["launch_us"] for k in kernels)
    for k in kernels:
        k["share"] = round(k["launch_us"] / tot, 4)
    dom = max(kernels, key=lambda k: k["launch_us"])
    roofline = {"bound": "hbm", "achieved": dom["achieved_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": dom["frac"], "traffic": dom["traffic"], "kernel": dom["kernel"],
                "launch_us": dom["launch_us"], "algorithmic_bytes_per_launch": dom["algorithmic_bytes_per_launch"],
                "plan": plan, "precomputed_chunks_per_head": c1,
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)" if peak_src == "measured"
                else "fallback 6650 GB/s",
                "kernels": kernels,
                "step": {"achieved": round(achieved_gbs, 1), "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
                         "algorithmic_bytes": nbytes,
                         "roofline_us": round(max(nbytes / (peaks["hbm_gbs"] * 1e9),
                                                  flops / (peaks["bf16_tflops"] * 1e12)) * 1e6, 2)},
                "bytes_note": "algorithmic bytes count q, k, v and o in the input dtype (bf16); the default "
                              "call writes o in fp32, o_fp32_extra_bytes_per_step more (see o_bf16 for the "
                              "bf16-output call)",
                "o_fp32_extra_bytes_per_step": o_fp32_extra_bytes(w),
                "tensor_view": {"flops_per_step": flops,
                                "achieved_tflops": round(flops / (ms_step * 1e-3) / 1e12, 1),
                                "peak_tflops": peaks["bf16_tflops"],
                                "frac": round(flops / (ms_step * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}}

    if args.only == "fwd":
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
                              "ms_per_step": round(ms_step, 5), "config": {"workload": WORKLOAD, "B": w.B, "T": w.T},
                              "plan": plan, "precomputed_chunks_per_head": c1,
                              "roofline_frac": round(nbytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                              "kernels": [(k["kernel"], k["launch_us"]) for k in kernels]}))
        return

    # the same forward with o in the input dtype (bf16): the call shape of the C ABI's definition
    o16 = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
    ws16_n = gdr.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.mode, torch.bfloat16, torch.bfloat16)
    ws16 = ws if (ws is not None and ws16_n <= ws.numel()) else (
        torch.empty(max(ws16_n, 1), dtype=torch.uint8, device=dev) if ws16_n else None)

    def step16(i=0):
        x = sets[i & 1]
        gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], mode=w.mode, chunk=w.chunk,
                      out=o16, state_out=st, workspace=ws16)

    n16 = max(3, min(args.steps, 200))

    def run16():
        ms = max_over_ranks(time_device(step16, n16, args.warmup, world, stream), world) / n16
        gdr.sync_status()
        return ms

    ms16 = with_status_retry("o_bf16", run16, world)
    o_bf16 = {"ms_per_step": round(ms16, 5), "tokens_per_s": round(job_throughput(tokens, ms16, world), 1),
              "steps": n16, "roofline_frac": round(nbytes / (ms16 * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
              "algorithmic_bytes": nbytes}

    # end to end: pinned host inputs -> device -> kernels -> host outputs, every step
    hx = {k: (None if t is None else t.cpu().pin_memory()) for k, t in sets[0].items()}
    h_o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, pin_memory=True)
    h_s = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, pin_memory=True)

    def e2e_step(i=0):
        gdr.chunk_fwd(hx["q"], hx["k"], hx["v"], hx["g"], hx["beta"], None, mode=w.mode, chunk=w.chunk,
                      out=h_o, state_out=h_s)

    e2e_steps = max(3, min(args.steps, 20))

    def run_e2e():
        ms = max_over_ranks(time_device(e2e_step, e2e_steps, max(1, min(args.warmup, 3)), world, stream), world)
        gdr.sync_status()
        return ms

    e2e_ms = with_status_retry("e2e", run_e2e, world)
    h2d = sum(t.numel() * t.element_size() for t in hx.values() if t is not None)
    d2h = h_o.numel() * h_o.element_size() + h_s.numel() * h_s.element_size()

    dec = with_status_retry("decode", lambda: bench_decode(args, dev, peaks, world), world)
    others = with_status_retry("workloads", lambda: bench_workloads(args, dev, peaks), world) if world == 1 else None
    pro = with_status_retry("prologue", lambda: bench_prologue(args, w, dev, ws, o, st, stream, world, rank, ms_step),
                            world)
    gdn2 = with_status_retry("gated_deltanet2", lambda: bench_gdn2(dev, peaks, stream), world) if world == 1 else None
    bwd = with_status_retry("backward", lambda: bench_backward(args, w, sets[0], dev, peaks, stream, world), world)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.dk, "d_v": w.dv, "chunk": w.chunk,
                   "decay": w.mode, "inputs": "bf16 q/k/v, fp32 g/beta, fp32 state; S0 = 0; returns o (fp32) and S_T",
                   "l2": "two resident input sets alternated, each 270 MB > 126 MB L2 (no flush)",
                   "parallelism": f"replicas x{world} (independent batches per GPU)"},
        "e2e": {"value": round(job_throughput(tokens, e2e_ms / e2e_steps, world), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": kernels_per_step * args.steps,
        "roofline": roofline,
        "clocks": clk,
        "o_bf16": o_bf16,
        "decode": dec,
        "prologue": pro,
        "backward": bwd,
        "status_retries": STATUS_RETRIES,
    }
    if others is not None:
        line["extra"] = {"workloads": others, "gated_deltanet2": gdn2}
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_prologue(args, w, dev, ws, o, st, stream, world, rank, ms_plain):
    """The same step on raw inputs (q/k unnormalised, beta and gate logits), with the mixer prologue
    fused into the kernels (gdr_chunk_fwd_ex), against the prologue as separate torch ops (F.normalize,
    sigmoid, softplus: library kernels, for comparison only) followed by the plain call."""
    import torch.nn.functional as F

    import gated_delta_rule_143_b200 as gdr
    from gated_delta_rule_143_b200.inputs import make_raw_chunk_inputs

    sets = []
    for s in range(2):
        x = make_raw_chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, w.mode, w.dtype, rank_seed(97, rank, s))
        sets.append({k: (None if t is None else t.to(dev)) for k, t in x.items()})
    gate = w.mode != "none"

    def fused(i=0):
        x = sets[i & 1]
        gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, mode=w.mode, chunk=w.chunk, out=o,
                      state_out=st, workspace=ws, l2norm_qk=True, beta_sigmoid=True, gate_softplus=gate,
                      gate_scale=x["gate_scale"])

    def unfused(i=0):
        x = sets[i & 1]
        q = F.normalize(x["q"].float(), dim=-1, eps=0.0).to(x["q"].dtype)
        k = F.normalize(x["k"].float(), dim=-1, eps=0.0).to(x["k"].dtype)
        b = torch.sigmoid(x["beta"])
        g = None
        if gate:
            A = x["gate_scale"].view((1, 1, -1) + ((1,) if w.mode == "channel" else ()))
            g = -A * F.softplus(x["g"])
        gdr.chunk_fwd(q, k, x["v"], g, b, None, mode=w.mode, chunk=w.chunk, out=o, state_out=st, workspace=ws)

    n = max(3, min(args.steps, 100))
    ms_f = max_over_ranks(time_device(fused, n, args.warmup, world, stream), world) / n
    ms_u = max_over_ranks(time_device(unfused, n, args.warmup, world, stream), world) / n
    gdr.sync_status()
    tokens = w.B * w.T
    return {"fused_ms_per_step": round(ms_f, 5), "fused_tokens_per_s": round(job_throughput(tokens, ms_f, world), 1),
            "torch_ops_then_call_ms_per_step": round(ms_u, 5), "plain_step_ms": round(ms_plain, 5),
            "steps": n, "fused_gpu_launches_per_step": gdr_kernels_per_step(w),
            "note": "raw q/k (unnormalised, bf16), beta logits, gate logits and A [H]; fused = "
                    "l2norm_qk + beta_sigmoid + gate_softplus in the library's kernels"}


def bench_gdn2(dev, peaks, stream):
    """Gated DeltaNet-2 (gdr_chunk_fwd_gdn2) at the Kimi Delta Attention workload's shape: the same
    inputs plus fp32 erase [B,T,H,d_k] and write [B,T,H,d_v] gates in place of beta. Bytes as that
    workload's, with the two gates in place of beta (2 * 512 B more per token-head)."""
    import gated_delta_rule_143_b200 as gdr
    from gated_delta_rule_143_b200.inputs import make_gdn2_gates
    w = CHUNK_WORKLOADS["kda_bf16_b4_h16_t8192_d128"]
    x = {k: (None if t is None else t.to(dev)) for k, t in workload_inputs(w).items()}
    gates = {k: t.to(dev) for k, t in make_gdn2_gates(w.B, w.T, w.H, w.dk, w.dv, 77).items()}
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=dev)
    st = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)

    def step(i=0):
        gdr.chunk_fwd_gdn2(x["q"], x["k"], x["v"], x["g"], gates["erase"], gates["write"], None, mode=w.mode, out=o,
                           state_out=st)

    n = 10
    ms = time_device(step, n, 3, 1, stream) / n
    gdr.sync_status()
    nbytes = chunk_bytes(w) + w.B * w.T * w.H * 4 * (w.dk + w.dv - 1)
    return {"workload": "gdn2 at " + w.name, "ms_per_step": round(ms, 5),
            "tokens_per_s": round(w.B * w.T / (ms * 1e-3), 1), "steps": n, "algorithmic_bytes": nbytes,
            "roofline_frac": round(nbytes / (peaks["hbm_gbs"] * 1e9) / (ms * 1e-3), 4),
            "path": "channel gate's tensor-core passes with the erase / write gates"}


def bench_backward(args, w, x, dev, peaks, stream, world):
    """gdr_chunk_bwd on the same workload (all gradients, dS0 included): device time per call and
    the bytes its two kernels must move (inputs and dO read twice, the per-token state history
    written once and read once, gradients written)."""
    import gated_delta_rule_143_b200 as gdr

    gen = torch.Generator().manual_seed(4242)
    dO = torch.randn(w.B, w.T, w.H, w.dv, generator=gen).to(torch.bfloat16).to(dev)
    ws_n = gdr._lib.lib().gdr_chunk_bwd_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, gdr._mode(w.mode), 1)
    ws_b = torch.empty(ws_n, dtype=torch.uint8, device=dev)

    n = max(3, min(args.steps, 10))
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for e in ev0 + [e for row in evk for e in row]:
        e.record(stream)
    calls = [0]

    def step(i=0):
        j = calls[0] - min(args.warmup, 3)  # timed calls record per-kernel events
        calls[0] += 1
        if 0 <= j < n:
            ev0[j].record(stream)
            gdr.profile_next_call(evk[j])
        gdr.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dO, S0=x["S0"], mode=w.mode, workspace=ws_b)

    ms = max_over_ranks(time_device(step, n, min(args.warmup, 3), world, stream), world) / n
    gdr.sync_status()
    k_ms = [statistics.mean((ev0[j] if c == 0 else evk[j][0]).elapsed_time(evk[j][c]) for j in range(n))
            for c in range(2)]
    ntok = w.B * w.T * w.H
    hist = w.B * w.H * w.T * w.dv * w.dk * 4
    gbytes = w.dk * 4 if w.mode == "channel" else (4 if w.mode == "scalar" else 0)
    nbytes = (2 * ntok * (2 * w.dk * 2 + w.dv * 2 + 4 + gbytes) + ntok * w.dv * 2  # q, k, v, beta, g twice; dO
              + 2 * hist  # the state history, written and read
              + ntok * (2 * w.dk + w.dv + 1) * 4 + ntok * gbytes + w.B * w.H * w.dv * w.dk * 4)  # gradients
    del ws_b
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms_per_call": round(ms, 4), "tokens_per_s": round(job_throughput(w.B * w.T, ms, world), 1),
            "calls": n, "gpu_launches_per_call": 2, "bytes_per_call": nbytes,
            "kernels_ms": {"bwd_history": round(k_ms[0], 4), "bwd_reverse": round(k_ms[1], 4)},
            "achieved_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "note": "fp32 CUDA-core backward: state-history kernel + reverse kernel, d_v / 8 CTAs per head"}


def gdr_kernels_per_step(w):
    import gated_delta_rule_143_b200 as gdr
    return gdr.launches_per_chunk_fwd(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.mode, torch.bfloat16, torch.float32)


def kernel_code_digest(text=None):
    """sha256 of the tensor-core kernel sources (gdr_chunk_tc.cu and the device helpers it
    includes, gdr_sm100.cuh), or of `text`, with comments and blank lines removed: an edit of the
    code makes recorded counters stale, an edit of a comment does not."""
    import hashlib
    import re
    if text is None:
        csrc = os.path.join(ROOT, "gated_delta_rule_143_b200", "csrc")
        text = ""
        for name in ("gdr_chunk_tc.cu", "gdr_sm100.cuh"):
            with open(os.path.join(csrc, name)) as f:
                text += f.read() + "\n"
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()


def traffic_from_profile(kernel):
    """DRAM bytes (read + write) per launch of `kernel` on this workload, from the committed ncu
    summary (profiles/traffic.json), or None when none was recorded for the current kernel code."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if not kernel_code_digest().startswith(d.get("_kernel_code_sha256_prefix", "-")):
        return None  # the kernel code changed since the counters were taken
    return d.get(WORKLOAD, {}).get(kernel)


def bench_decode(args, dev, peaks, world):
    import gated_delta_rule_143_b200 as gdr
    w = DECODE_WORKLOADS[DECODE]
    S = make_decode_state(w, WORKLOAD_SEEDS[DECODE]).to(dev)
    toks = []
    for s in range(2):
        x = make_decode_step(w, WORKLOAD_SEEDS[DECODE], s)
        toks.append({k: (None if t is None else t.to(dev)) for k, t in x.items()})
    o = torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                    device=dev)  # o in the input dtype, as decode_bytes counts it
    stream = torch.cuda.current_stream(dev)

    def step(i=0):
        x = toks[i & 1]
        gdr.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S, mode=w.mode, out=o)

    n = max(20, min(args.steps, 200))
    ms = max_over_ranks(time_device(step, n, max(3, args.warmup), world, stream), world) / n
    gdr.sync_status()
    nbytes = decode_bytes(w)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": DECODE, "ms_per_step": round(ms, 5), "tokens_per_s": round(world * w.B / (ms * 1e-3), 1),
            "steps": n, "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                                     "algorithmic_bytes_per_launch": nbytes},
            "l2": "state 537 MB > L2, streamed once per step"}


def bench_workloads(args, dev, peaks):
    """Every named chunked-forward workload, forward only (default call: fp32 o), timed with CUDA
    events over a few steps after a warm-up: ms per step, tokens/s, the plan, and the fraction of
    the roofline max(bytes / HBM peak, flops / bf16 peak) with bytes and flops counted as above."""
    import gated_delta_rule_143_b200 as gdr
    stream = torch.cuda.current_stream(dev)
    out = {}
    # the small fp32 workload's T = 256 runs the token recurrence; the same shape at T = 320 (five
    # chunks) keeps the fp32 chunk form measured
    extra = dataclasses.replace(CHUNK_WORKLOADS["gdn_f32_b1_h2_t256_d64"], name="gdn_f32_b1_h2_t320_d64_chunk_form",
                                T=320)
    for name, w in list(CHUNK_WORKLOADS.items()) + [(extra.name, extra)]:
        x = {k: (None if t is None else t.to(dev)) for k, t in workload_inputs(w, seed=WORKLOAD_SEEDS.get(name, 1)).items()}
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=dev)
        st = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
        nws = gdr.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.mode, dt, torch.float32)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev) if nws else None

        def step(i=0):
            gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], mode=w.mode, chunk=w.chunk,
                          out=o, state_out=st, workspace=ws)

        n = 50 if w.B * w.T * w.H <= (1 << 20) else 10
        ms = time_device(step, n, 3, 1, stream) / n
        nbytes = chunk_bytes(w)
        flops = chunk_flops_per_token_head(w.chunk, w.dk, w.dv) * w.B * w.T * w.H
        roof_us = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12)) * 1e6
        plan, c1 = gdr.chunk_fwd_plan(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.mode, dt, torch.float32)
        out[name] = {"ms_per_step": round(ms, 5), "tokens_per_s": round(w.B * w.T / (ms * 1e-3), 1), "steps": n,
                     "plan": plan, "precomputed_chunks_per_head": c1, "roofline_us": round(roof_us, 2),
                     "roofline_frac": round(roof_us / (ms * 1e3), 4), "algorithmic_bytes": nbytes,
                     "flops": flops}
        del x, o, st, ws
    gdr.sync_status()
    return out


# ------------------------------------------------------------------- oracle --
def _oracle_sample(w, b_count=1):
    """A bounded sample of the workload for the CPU oracle: the first b_count sequences
    (all heads, all tokens)."""
    x = workload_inputs(w)
    return {k: (None if t is None else t[:b_count].contiguous()) for k, t in x.items()}


def cpu_baseline(w):
    import oracle
    x = _oracle_sample(w, b_count=w.B)
    t0 = time.perf_counter()
    oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], w.mode, S0=x["S0"])
    dt = time.perf_counter() - t0
    return {"value": round(w.B * w.T / dt, 1), "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"full workload once ({w.B}x{w.T} tokens x {w.H} heads), fp64 token-by-token recurrence",
            "seconds": round(dt, 3)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = CHUNK_WORKLOADS[WORKLOAD]
    x = _oracle_sample(w, b_count=1)
    sample_tokens = x["q"].shape[0] * w.T

    def once():
        oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], w.mode, S0=x["S0"])

    for _ in range(args.warmup):
        once()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        once()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = round(sample_tokens / dt, 1)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "d_k": w.dk, "d_v": w.dv, "chunk": w.chunk,
                   "decay": w.mode},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"1 of {w.B} sequences per step ({w.T} tokens x {w.H} heads)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    global WORKLOAD
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)  # about 0.25 s timed: a dozen clock samples
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--only", choices=("all", "fwd", "decode", "bwd"), default="all",
                    help="fwd: time the forward only (no e2e, decode or CPU baseline); decode: the decode step "
                         "only; bwd: the backward only; all three for profiling runs")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch size (profiling runs)")
    ap.add_argument("--seq", type=int, default=0, help="override the workload's sequence length (profiling runs)")
    ap.add_argument("--workload", choices=sorted(CHUNK_WORKLOADS), default=WORKLOAD,
                    help="chunked-forward workload (default: the headline one; others for --only fwd runs)")
    args = ap.parse_args()
    if args.workload != WORKLOAD:
        if args.only not in ("fwd", "bwd") or args.impl != "ours":
            ap.error("other workloads are timed with --only fwd or bwd (the full line describes the headline one)")
        WORKLOAD = args.workload
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only == "decode":
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        peaks, _ = load_peaks()
        print(json.dumps({"metric": "decode step", "decode": bench_decode(args, dev, peaks, 1)}))
    elif args.only == "bwd":
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        peaks, _ = load_peaks()
        w = CHUNK_WORKLOADS[WORKLOAD]
        if args.batch:
            w = dataclasses.replace(w, B=args.batch)
        if args.seq:
            w = dataclasses.replace(w, T=args.seq)
        x = {k: (None if t is None else t.to(dev)) for k, t in workload_inputs(w).items()}
        bwd = bench_backward(args, w, x, dev, peaks, torch.cuda.current_stream(dev), 1)
        print(json.dumps({"metric": "backward", "config": {"workload": WORKLOAD, "B": w.B, "T": w.T},
                          "backward": bwd}))
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
