"""Benchmark of the GQE attention forward pass on B200 (routed prefill and decode).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl gqe|reference]

A step is one pass of the whole routed path over one batch of seeded synthetic
input, with inputs resident in HBM:
  prefill workloads: gqe_route (router, per-group top-k, compaction) +
                     gqe_attn_prefill (routed causal attention + gated scatter)
  decode workload:   gqe_route on the new tokens + gqe_attn_decode
Metric: active-head TFLOP/s for prefill (4*d_h*(t+1) per routed row), KV-cache
GB/s for decode (2*g*d_h*L_b bf16 elements per sequence).  The headline is the
largest prefill config (gqe_prefill: B=8 T=4096 h=32 g=8 k=2); every config's
attention time and roofline fraction go into the line's "configs" map.  The L2 is flushed
before every timed step, outside the step's CUDA events: a 256 MB buffer is
written, then read back, so the step starts with clean, unrelated lines in L2.

With N > 1 (torchrun) every rank runs an independent replica on its own batch
(the path has no exchange step); value = all ranks' work / the slowest rank's time.
``--impl reference`` times the CPU oracle instead, on bounded samples of the
same workload, on the host cores.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gqe_synth  # noqa: E402

PRIMARY = "gqe_prefill"
# Every config, in order, in the line's compact "configs" map (the primary included).
CONFIG_ORDER = ["tiny_f32", "dense_gqa", "gqe_prefill", "gqe_long", "gqe_decode", "gqe_32k"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernels, from `ncu` captures
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel
# source they were taken on (sha256 of the listed files).  See profiles/.
NCU_TRAFFIC = {
    ("prefill_tc_kernel", "gqe_prefill"): {
        "sha": "f93b2665924b3811", "bytes_per_launch": 1060030000 + 231494144,
        "note": "ncu SpeedOfLight + MemoryWorkloadAnalysis, one launch (profiles/prefill_tc_kernel_gqe_prefill.md)"},
    ("prefill_tc_kernel", "gqe_long"): {
        "sha": "f93b2665924b3811", "bytes_per_launch": 169284608 + 37322752,
        "note": "ncu SpeedOfLight + MemoryWorkloadAnalysis, one launch (profiles/prefill_tc_kernel_gqe_long.md)"},
    ("prefill_tc_kernel", "dense_gqa"): {
        "sha": "f93b2665924b3811", "bytes_per_launch": 104842752 + 30646272,
        "note": "ncu SpeedOfLight + MemoryWorkloadAnalysis, one launch (profiles/prefill_tc_kernel_dense_gqa.md)"},
    ("decode_partial_kernel", "gqe_decode"): {
        "sha": "2ffadcebec633c3d", "bytes_per_launch": 2263625728 + 8142592,
        "note": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch of the partial kernel "
                "(profiles/decode_partial_kernel_gqe_decode.md)"},
}


def kernel_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "routed_head_gqa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_FILES = {
    "prefill_tc_kernel": ["prefill_tc.cu", "sm100.cuh", "units.cuh", "common.cuh"],
    "decode_partial_kernel": ["decode.cu", "common.cuh"],
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clocks and clock-event reasons of the benchmarked GPU during the
    timed region.  A thread polls NVML (read-only queries) every `poll_ms`,
    so a region of a few milliseconds still holds samples; nvidia-smi's own
    query runs beside it.  Every sample carries its host time, and the summary
    takes the samples between mark_start() and mark_end() (NVML's if it
    answered, else nvidia-smi's, else the nearest ones)."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    NVML_BITS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
                 "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
                 "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
                 "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, device_index: int, uuid: str | None = None, poll_ms: float = 2.0,
                 smi_interval_ms: int = 100, smi_cmd: str = "nvidia-smi"):
        self.dev = device_index
        self.uuid = uuid
        self.poll_s = poll_ms * 1e-3
        self.smi_interval_ms = smi_interval_ms
        self.smi_cmd = smi_cmd
        self.proc = None
        self.thread = None
        self.smi = []    # (host time, csv line)
        self.nvml = []   # (host time, sm MHz, max MHz, reasons)
        self.nvml_thread = None
        self.stop_flag = threading.Event()
        self.nvml_ready = threading.Event()
        self.smi_ready = threading.Event()
        self.t0 = self.t1 = None

    # -- nvidia-smi -----------------------------------------------------------
    def _read(self):
        for line in self.proc.stdout:
            self.smi.append((time.perf_counter(), line.strip()))
            self.smi_ready.set()

    # -- NVML -------------------------------------------------------------------
    def _nvml_handle(self, nv):
        if self.uuid:
            try:
                return nv.nvmlDeviceGetHandleByUUID(self.uuid)
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def _poll(self):
        try:
            import pynvml as nv

            nv.nvmlInit()
        except Exception:
            self.nvml_ready.set()
            return
        try:
            hdl = self._nvml_handle(nv)
            mx = float(nv.nvmlDeviceGetMaxClockInfo(hdl, nv.NVML_CLOCK_SM))
            bits = {n: getattr(nv, attr) for n, attr in self.NVML_BITS.items()}
            while not self.stop_flag.is_set():
                mhz = float(nv.nvmlDeviceGetClockInfo(hdl, nv.NVML_CLOCK_SM))
                mask = int(nv.nvmlDeviceGetCurrentClocksEventReasons(hdl))
                self.nvml.append((time.perf_counter(), mhz, mx, {n for n, b in bits.items() if mask & b}))
                self.nvml_ready.set()
                time.sleep(self.poll_s)
        except Exception:
            pass
        finally:
            self.nvml_ready.set()
            try:
                nv.nvmlShutdown()
            except Exception:
                pass

    def start(self, wait_s: float = 3.0):
        """Start both samplers and wait (at most wait_s) for their first samples."""
        try:
            self.proc = subprocess.Popen(
                [self.smi_cmd, f"--id={self.dev}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", str(self.smi_interval_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None
            self.smi_ready.set()
        self.nvml_thread = threading.Thread(target=self._poll, daemon=True)
        self.nvml_thread.start()
        deadline = time.perf_counter() + wait_s
        self.nvml_ready.wait(max(0.0, deadline - time.perf_counter()))
        self.smi_ready.wait(max(0.0, deadline - time.perf_counter()))

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def _parse_smi(self):
        out = []
        for t, line in self.smi:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            reasons = {n for n, v in zip(self.REASONS, parts[5:9]) if v.lower().startswith("active")}
            out.append((t, mhz, mx, reasons))
        return out

    def _window(self, samples):
        if not samples:
            return []
        if self.t0 is None or self.t1 is None:
            return samples
        inside = [s for s in samples if self.t0 <= s[0] <= self.t1]
        if inside:
            return inside
        # none inside a region shorter than the period: the first sample after it starts
        after = [s for s in samples if s[0] >= self.t0]
        return after[:1] if after else samples[-1:]

    def stop(self):
        if self.proc is not None:
            time.sleep(2 * self.smi_interval_ms * 1e-3)
        self.stop_flag.set()
        if self.nvml_thread is not None:
            self.nvml_thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)
        nvml_all, smi_all = list(self.nvml), self._parse_smi()
        nvml_in, smi_in = self._window(nvml_all), self._window(smi_all)
        inside = lambda s: self.t0 is not None and self.t1 is not None and self.t0 <= s[0] <= self.t1  # noqa: E731
        use, source = (nvml_in, "nvml") if any(inside(s) for s in nvml_in) or not smi_in else (smi_in, "nvidia-smi")
        if not use:
            return None
        reasons = set()
        for s in nvml_in + smi_in:
            reasons |= s[3]
        return {"sm_mhz": statistics.median(s[1] for s in use), "sm_max_mhz": max(s[2] for s in nvml_all + smi_all),
                "reasons": sorted(reasons), "samples": sum(1 for s in use if inside(s)), "source": source,
                "nvidia_smi_samples": sum(1 for s in smi_all if inside(s))}


def device_uuid(dev):
    """NVML's name of the torch device ("GPU-<uuid>"), or None."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None
    return u if u.startswith("GPU-") else "GPU-" + u


def l2_flush(buf):
    """Evict the L2 between timed steps: write a 256 MB buffer (twice the L2),
    then read it back, so that the L2 is left holding clean lines of an
    unrelated buffer and the timed kernels do not pay for writing the flush's
    dirty lines back to HBM."""
    buf.zero_()
    buf.view(torch.int32).max()


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only: barrier and max of the step times)
# ---------------------------------------------------------------------------
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(work: float, ws: int, steps: int, step_ms_max: float, scale: float) -> float:
    """Whole-job throughput: the work of all ranks' steps over the slowest rank's time."""
    return work * ws * steps / (step_ms_max * 1e-3) * scale


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def workload_for_rank(w, rank):
    if rank == 0:
        return w
    import dataclasses

    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


class Runner:
    """Holds one workload's device inputs and buffers; runs steps."""

    def __init__(self, w, dev):
        import routed_head_gqa_b200 as g

        self.g = g
        self.w = w
        self.inp = gqe_synth.make_inputs(w)
        self.dev = dev
        self.d = {k: (v.to(dev) if v is not None else None) for k, v in self.inp.items()}
        T = 1 if w.decode else w.T
        self.shape = g.make_shape(w.B, T, w.d_model, w.h, w.g, w.d_h, w.k, w.torch_dtype)
        self.buf = g.Buffers(self.shape, dev, Lmax=w.Lmax if w.decode else 0)
        self.stream = torch.cuda.current_stream()

    def route(self):
        self.buf.route(self.d["x"], self.d["W_r"], self.d["bias"])

    def attend(self):
        if self.w.decode:
            self.buf.decode(self.d["q"], self.d["K_cache"], self.d["V_cache"], self.d["lengths"])
        else:
            self.buf.prefill(self.d["Q"], self.d["K"], self.d["V"])

    def step(self):
        self.route()
        self.attend()

    def launches_per_step(self):
        # router (+ a separate count pass unless the tensor-core router fuses the
        # counts: bf16, h % 8 == 0, h <= 256, d_model % 8 == 0, h/g <= 64, T % 32 == 0)
        # + one scan-and-scatter pass; then one prefill or two decode kernels
        w = self.w
        fused = (w.dtype == "bf16" and w.h % 8 == 0 and w.h <= 256 and w.d_model % 8 == 0
                 and w.h // w.g <= 64 and w.T % 32 == 0)
        route = 2 if fused else 3
        return route + (2 if w.decode else 1)

    def work(self):
        """(work units per step, unit string, scale to the unit)."""
        from routed_head_gqa_b200 import metrics

        w = self.w
        if w.decode:
            return float(metrics.decode_kv_bytes(self.inp["lengths"], w.g, w.d_h, 2)), "GB/s", 1e-9
        flops = metrics.prefill_active_flops(w.B, w.T, w.g, w.k, w.d_h)
        return float(flops), "TFLOP/s", 1e-12


def time_workload(w, steps, warmup, ws, rank, peaks, peak_kind, with_clocks, with_e2e):
    dev = torch.device("cuda", torch.cuda.current_device())
    r = Runner(workload_for_rank(w, rank), dev)
    work, unit, scale = r.work()
    if not w.decode:
        from routed_head_gqa_b200 import metrics

        r.step()
        torch.cuda.synchronize()
        assert metrics.prefill_active_flops_from_routing(r.buf.idx, w.d_h) == int(work)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        l2_flush(flush)
        r.step()
    torch.cuda.synchronize()
    st = r.buf.status()
    if st != 0:
        raise RuntimeError(f"device status {r.g.gqe_status_string(st)} during warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(dev.index, uuid=device_uuid(dev)) if with_clocks else None
    if sampler:
        sampler.start()
    barrier(ws)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_start()
    for i in range(steps):
        l2_flush(flush)
        e0, e1, e2 = ev[i]
        e0.record()
        r.route()
        e1.record()
        r.attend()
        e2.record()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_end()
    barrier(ws)
    clocks = sampler.stop() if sampler else None
    st = r.buf.status()
    if st != 0:
        raise RuntimeError(f"device status {r.g.gqe_status_string(st)} in the timed region")
    step_ms = sum(a.elapsed_time(c) for a, _, c in ev)
    attn_ms = [b.elapsed_time(c) for _, b, c in ev]
    route_ms = [a.elapsed_time(b) for a, b, _ in ev]
    step_ms_max = max_over_ranks(step_ms, ws)
    value = aggregate_value(work, ws, steps, step_ms_max, scale)

    kern = "decode_partial_kernel" if w.decode else "prefill_tc_kernel"
    attn_avg_ms = sum(attn_ms) / len(attn_ms)
    if w.dtype == "f32" and not w.decode:
        achieved = work / (attn_avg_ms * 1e-3) * 1e-12
        alu_peak = SM_COUNT * FP32_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 * 1e-12
        kern = "prefill_simt_kernel"
        roof = {"bound": "alu", "achieved": round(achieved, 4), "peak": round(alu_peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / alu_peak, 6),
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 x 1965 MHz (derived)",
                "kernel": "gqe_attn_prefill (prefill_simt_kernel, fp32 CUDA cores)"}
    elif w.decode:
        achieved = work / (attn_avg_ms * 1e-3) * 1e-9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": f"hbm_gbs ({peak_kind})",
                "kernel": "gqe_attn_decode (decode_partial_kernel + decode_combine_kernel)"}
    else:
        achieved = work / (attn_avg_ms * 1e-3) * 1e-12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "peak_source": f"bf16_tflops burst ({peak_kind})",
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "kernel": "gqe_attn_prefill (prefill_tc_kernel)"}
    tr = NCU_TRAFFIC.get((kern, w.name))
    roof["traffic"] = None
    if tr and kern in KERNEL_FILES and tr["sha"] == kernel_sha(KERNEL_FILES[kern]):
        roof["traffic"] = tr["bytes_per_launch"]
        roof["traffic_note"] = tr["note"]
    roof["algorithmic_per_launch"] = work
    res = {
        "value": value, "unit": unit, "ms_per_step": step_ms_max / steps,
        "attn_ms": attn_avg_ms, "route_ms": sum(route_ms) / len(route_ms),
        "roofline": roof, "clocks": clocks, "gpu_launches": r.launches_per_step() * steps,
    }
    if with_e2e:
        res["e2e"] = time_e2e(r, steps, ws, work, scale, unit)
    del r, flush
    torch.cuda.empty_cache()
    return res


def time_layer_ops(w, steps, warmup, peaks, peak_kind):
    """The GQE layer's calls around the routed attention, on the workload's
    shapes, each timed alone with CUDA events (L2 flushed before each call,
    outside the events): the routed query projection (a tensor-core grouped
    GEMM over the routed rows only), the always-active shared head (one dense
    causal head over KV group 0, on the routed prefill's kernel) and the
    per-group slots (concatenated expert outputs + gate-weighted sum, HBM-bound)."""
    from routed_head_gqa_b200 import metrics

    dev = torch.device("cuda", torch.cuda.current_device())
    r = Runner(w, dev)
    g = r.g
    r.step()
    Qs = gqe_synth.make_shared_query(w).to(dev)
    Os = torch.empty((w.B, w.T, w.d_h), dtype=w.torch_dtype, device=dev)
    W_Q = gqe_synth.make_qproj_weight(w).to(dev)
    Qp = torch.empty((w.B, w.T, w.h, w.d_h), dtype=w.torch_dtype, device=dev)
    W_Z = gqe_synth.make_oproj_weight(w).to(dev)
    Y = torch.empty((w.B, w.T, w.d_model), dtype=w.torch_dtype, device=dev)
    cat = torch.empty((w.B, w.T, w.g, w.k, w.d_h), dtype=w.torch_dtype, device=dev)
    wsum = torch.empty((w.B, w.T, w.g, w.d_h), dtype=w.torch_dtype, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def shared():
        g.gqe_attn_shared_head(r.shape, Qs, r.d["K"], r.d["V"], 0, Os, r.buf.workspace)

    def slots():
        g.gqe_group_slots(r.shape, r.buf.O, r.buf.idx, r.buf.gate, cat, wsum)

    def qproj():
        g.gqe_routed_qproj(r.shape, r.d["x"], W_Q, r.buf.idx, r.buf.head_offsets, r.buf.head_pos, Qp, r.buf.workspace)

    def oproj():  # over the prefill's gated output (zeros in the unselected slots)
        g.gqe_routed_oproj(r.shape, r.buf.O, r.buf.idx, W_Z, Y, r.buf.workspace)

    def timed(fn):
        for _ in range(warmup):
            l2_flush(flush)
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for a, b in ev:
            l2_flush(flush)
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / steps

    sh_ms = timed(shared)
    sl_ms = timed(slots)
    qp_ms = timed(qproj)
    op_ms = timed(oproj)
    st = r.buf.status()
    if st != 0:
        raise RuntimeError(f"device status {g.gqe_status_string(st)} in the output construction")
    sh_flops = 4.0 * w.d_h * w.B * w.T * (w.T + 1) / 2  # one head, causal
    el = 2 if w.dtype == "bf16" else 4
    rows = w.B * w.T * w.g * w.k
    sl_bytes = float(rows * w.d_h * el * 2 + w.B * w.T * w.g * w.d_h * el + rows * 8)  # O rows in, cat + wsum out
    qp_flops = 2.0 * w.d_model * w.d_h * rows  # routed rows only
    qp_tf = qp_flops / (qp_ms * 1e-3) * 1e-12
    op_flops = 2.0 * w.d_model * w.d_h * rows  # the selected heads' rows only
    op_dense = 2.0 * w.d_model * w.d_h * w.B * w.T * w.h  # every head slot, as a dense GEMM would
    op_tf = op_flops / (op_ms * 1e-3) * 1e-12
    sh_tf = sh_flops / (sh_ms * 1e-3) * 1e-12
    sl_gbs = sl_bytes / (sl_ms * 1e-3) * 1e-9
    del r, flush
    torch.cuda.empty_cache()
    return {
        "routed_qproj": {"ms": qp_ms, "value": qp_tf, "unit": "TFLOP/s", "flops": qp_flops,
                         "roofline": {"bound": "tensor", "achieved": round(qp_tf, 1), "peak": peaks["bf16_tflops"],
                                      "unit": "TFLOP/s", "frac": round(qp_tf / peaks["bf16_tflops"], 4),
                                      "peak_source": f"bf16_tflops burst ({peak_kind})",
                                      "kernel": "gqe_routed_qproj (qproj_kernel)"}},
        "routed_oproj": {"ms": op_ms, "value": op_tf, "unit": "TFLOP/s", "flops": op_flops,
                         "roofline": {"bound": "tensor", "achieved": round(op_tf, 1), "peak": peaks["bf16_tflops"],
                                      "unit": "TFLOP/s", "frac": round(op_tf / peaks["bf16_tflops"], 4),
                                      "frac_of_dense_equivalent": round(op_dense / (op_ms * 1e-3) * 1e-12
                                                                        / peaks["bf16_tflops"], 4),
                                      "peak_source": f"bf16_tflops burst ({peak_kind})",
                                      "kernel": "gqe_routed_oproj (oproj_kernel)"}},
        "shared_head": {"ms": sh_ms, "value": sh_tf, "unit": "TFLOP/s", "flops": sh_flops,
                        "roofline": {"bound": "tensor", "achieved": round(sh_tf, 1), "peak": peaks["bf16_tflops"],
                                     "unit": "TFLOP/s", "frac": round(sh_tf / peaks["bf16_tflops"], 4),
                                     "peak_source": f"bf16_tflops burst ({peak_kind})",
                                     "kernel": "gqe_attn_shared_head (prefill_tc_kernel, identity routing)"}},
        "group_slots": {"ms": sl_ms, "value": sl_gbs, "unit": "GB/s", "bytes": sl_bytes,
                        "roofline": {"bound": "hbm", "achieved": round(sl_gbs, 1), "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "frac": round(sl_gbs / peaks["hbm_gbs"], 4),
                                     "peak_source": f"hbm_gbs ({peak_kind})",
                                     "kernel": "gqe_group_slots (group_slots_kernel)"}},
        "shape": w.describe(),
    }


FP32_LANES_PER_SM = 128  # B200: 4 sub-partitions x 32 fp32 FMA lanes
SM_COUNT = 148
SM_MAX_MHZ = 1965.0


def time_backward(w, steps, warmup, peaks, peak_kind):
    """The routed attention's backward (gqe_attn_prefill_backward) on the
    workload's shapes, after one forward step, timed alone with CUDA events (L2
    flushed before each call, outside the events).  Algorithmic FLOPs: the
    five contractions of an attention backward over the visible (row, key)
    pairs of the routed rows, 2.5x the forward's 4*d_h per pair.  bf16 inputs
    with d_h = 128 run on the tensor cores (the roofline is the bf16 tensor
    peak); other inputs run on the fp32 CUDA cores (the roofline is the fp32
    FMA peak: 148 SMs x 128 lanes x 2 FLOP x the 1965 MHz SM clock)."""
    from routed_head_gqa_b200 import metrics

    dev = torch.device("cuda", torch.cuda.current_device())
    r = Runner(w, dev)
    r.step()
    tensor = w.dtype == "bf16" and w.d_h == 128 and w.k <= 4 and w.h // w.g <= 32
    if tensor:
        r.buf.prefill_train(r.d["Q"], r.d["K"], r.d["V"])
    dO = gqe_synth.make_output_grad(w).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def attn():  # from the training forward's saved rows where the tensor-core path has them
        r.buf.backward(r.d["Q"], r.d["K"], r.d["V"], dO, saved=tensor)

    def attn_recompute():
        r.buf.backward(r.d["Q"], r.d["K"], r.d["V"], dO)

    def router():
        r.buf.route_backward(r.d["x"], r.d["W_r"], r.buf._bwd[3])

    def timed(fn):
        for _ in range(warmup):
            l2_flush(flush)
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for a, b in ev:
            l2_flush(flush)
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / steps

    ms = timed(attn)
    ms_recompute = timed(attn_recompute) if tensor else None
    rms = timed(router)
    st = r.buf.backward_status()
    if st != 0:
        raise RuntimeError(f"device status {r.g.gqe_status_string(st)} in the backward")
    flops = 2.5 * metrics.prefill_active_flops(w.B, w.T, w.g, w.k, w.d_h)
    tf = flops / (ms * 1e-3) * 1e-12
    alu_peak = SM_COUNT * FP32_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 * 1e-12
    el = 2 if w.dtype == "bf16" else 4
    BT = w.B * w.T
    # x read once per 32 heads and dx written (fp32); dlogits read twice; W_r, dW_r, dbias are small
    r_bytes = float(BT * w.d_model * (el * -(-w.h // 32) + 4) + 2 * BT * w.h * 4 + w.d_model * w.h * (el + 4))
    r_gbs = r_bytes / (rms * 1e-3) * 1e-9
    del r, flush
    torch.cuda.empty_cache()
    if tensor:
        roof = {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tf / peaks["bf16_tflops"], 4), "peak_source": f"bf16_tflops burst ({peak_kind})",
                "kernel": "gqe_attn_prefill_backward_saved (bwd_pack_kernel + dq_tc_kernel + dkdv_tc_kernel)"}
    else:
        roof = {"bound": "alu", "achieved": round(tf, 2), "peak": round(alu_peak, 1), "unit": "TFLOP/s",
                "frac": round(tf / alu_peak, 4),
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 x 1965 MHz (derived)",
                "frac_of_bf16_tensor": round(tf / peaks["bf16_tflops"], 4),
                "kernel": "gqe_attn_prefill_backward (bwd_dq_kernel + bwd_rows_kernel + bwd_dkdv_kernel)"}
    out = {"ms": ms, "value": tf, "unit": "TFLOP/s", "flops": flops, "launches": 3,
           "roofline": roof}
    if tensor:  # gqe_attn_prefill_backward: the forward's rows recomputed first (prefill_tc_kernel<train>)
        out["recompute"] = {"ms": ms_recompute, "value": flops / (ms_recompute * 1e-3) * 1e-12, "launches": 4}
    return {**out,
            "router": {"ms": rms, "value": r_gbs, "unit": "GB/s", "bytes": r_bytes, "launches": 4,
                       "roofline": {"bound": "hbm", "achieved": round(r_gbs, 1), "peak": peaks["hbm_gbs"],
                                    "unit": "GB/s", "frac": round(r_gbs / peaks["hbm_gbs"], 4),
                                    "peak_source": f"hbm_gbs ({peak_kind})",
                                    "kernel": "gqe_route_backward (dx, dW_r partials + reduce, dbias)"}},
            "shape": w.describe()}


def time_paged_decode(w, steps, warmup, peaks, peak_kind, page_size=256):
    """The decode workload with its caches cut into pages of page_size rows,
    scattered over the pool in a seeded random order (gqe_attn_decode_paged),
    timed like the contiguous decode: CUDA events around the decode call, L2
    flushed before each, outside the events."""
    from routed_head_gqa_b200 import metrics

    dev = torch.device("cuda", torch.cuda.current_device())
    r = Runner(w, dev)
    g = r.g
    r.route()
    Kp, Vp, bt = gqe_synth.make_paged_cache(r.inp["K_cache"], r.inp["V_cache"], page_size)
    Kp, Vp, bt = Kp.to(dev), Vp.to(dev), bt.to(dev)
    del r.d["K_cache"], r.d["V_cache"]
    O = torch.empty_like(r.buf.O)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def paged():
        g.gqe_attn_decode_paged(r.shape, r.d["q"], Kp, Vp, page_size, bt, r.d["lengths"], r.buf.idx, r.buf.gate, O,
                                r.buf.workspace)

    for _ in range(warmup):
        l2_flush(flush)
        paged()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        l2_flush(flush)
        a.record()
        paged()
        b.record()
    torch.cuda.synchronize()
    st = r.buf.status()
    if st != 0:
        raise RuntimeError(f"device status {g.gqe_status_string(st)} in the paged decode")
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    nbytes = float(metrics.decode_kv_bytes(r.inp["lengths"], w.g, w.d_h, 2))
    gbs = nbytes / (ms * 1e-3) * 1e-9
    del r, Kp, Vp, flush
    torch.cuda.empty_cache()
    return {"page_size": page_size, "ms": ms, "value": gbs, "unit": "GB/s",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"hbm_gbs ({peak_kind})",
                         "kernel": "gqe_attn_decode_paged (decode_partial_kernel paged + decode_combine_kernel)"}}


def time_e2e(r, steps, ws, work, scale, unit):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory to the device and its output back, all
    inside the timed region.  As a serving loop would, the copies run on their
    own streams with double-buffered device inputs and outputs: step i+1's
    inputs go in and step i-1's output comes out (PCIe is full duplex) while
    step i computes."""
    import routed_head_gqa_b200 as g

    w = r.w
    names = ["x", "q"] if w.decode else ["x", "Q", "K", "V"]
    host = {n: r.inp[n].pin_memory() for n in names}
    bufs = [r.buf, g.Buffers(r.shape, r.dev, Lmax=w.Lmax if w.decode else 0)]
    dev_in = [{n: torch.empty_like(r.d[n]) for n in names} for _ in range(2)]
    out_host = [torch.empty(r.buf.O.shape, dtype=r.buf.O.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        k = i % 2
        if i >= 2:
            s_in.wait_event(comp_done[k])  # step i-2 has finished reading dev_in[k]
        with torch.cuda.stream(s_in):
            for n in names:
                dev_in[k][n].copy_(host[n], non_blocking=True)
            in_done[k].record(s_in)
        comp.wait_event(in_done[k])
        if i >= 2:
            comp.wait_event(out_done[k])  # step i-2's output has left bufs[k].O
        bufs[k].route(dev_in[k]["x"], r.d["W_r"], r.d["bias"])
        if w.decode:
            bufs[k].decode(dev_in[k]["q"], r.d["K_cache"], r.d["V_cache"], r.d["lengths"])
        else:
            bufs[k].prefill(dev_in[k]["Q"], dev_in[k]["K"], dev_in[k]["V"])
        comp_done[k].record(comp)
        s_out.wait_event(comp_done[k])
        with torch.cuda.stream(s_out):
            out_host[k].copy_(bufs[k].O, non_blocking=True)
            out_done[k].record(s_out)

    def run(n):
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        for i in range(n):
            one(i)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    e0.record()
    run(steps)
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), ws)
    note = ("KV caches stay resident (decoder state); per step: x and q in, O out" if w.decode
            else "per step: x, Q, K, V in; O out")
    return {"value": work * ws * steps / (ms * 1e-3) * scale, "unit": unit, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "note": note + "; copies on their own streams, double-buffered, overlapping the neighbouring steps"}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample(w, inp, n_rows, seed):
    """Run the oracle on a sample of n_rows token rows of the workload.  Returns
    (work done in the metric's units, seconds, sample description)."""
    import numpy as np

    import oracle

    if w.decode:
        gen = torch.Generator().manual_seed(seed)
        bs = torch.randperm(w.B, generator=gen)[: max(1, min(w.B, n_rows))].sort().values
        t0 = time.perf_counter()
        idx, gate, _, _ = oracle.route(inp["x"][bs], inp["W_r"], w.h, w.g, w.k, bias=inp["bias"])
        oracle.decode(inp["q"][bs], inp["K_cache"][bs], inp["V_cache"][bs], inp["lengths"][bs], idx, gate)
        dt = time.perf_counter() - t0
        work = float(inp["lengths"][bs].to(torch.int64).sum().item()) * 2 * w.g * w.d_h * 2
        return work, dt, f"{len(bs)} of {w.B} sequences (full cache each)"
    rows = gqe_synth.sample_rows(w, n_rows, seed=seed).numpy()
    t0 = time.perf_counter()
    xr = inp["x"].reshape(w.B * w.T, w.d_model)[torch.from_numpy(rows)]
    idx_s, gate_s, _, _ = oracle.route(xr, inp["W_r"], w.h, w.g, w.k, bias=inp["bias"])
    idx = np.zeros((w.B * w.T, w.g, w.k), np.int32)
    gate = np.zeros((w.B * w.T, w.g, w.k), np.float64)
    # rows outside the sample keep a valid placeholder routing (never computed)
    idx[:] = (np.arange(w.g)[:, None] * w.hpg + np.arange(w.k)[None, :])[None]
    idx[rows] = idx_s
    gate[rows] = gate_s
    oracle.attn_rows(inp["Q"], inp["K"], inp["V"], idx.reshape(w.B, w.T, w.g, w.k),
                     gate.reshape(w.B, w.T, w.g, w.k), rows=rows)
    dt = time.perf_counter() - t0
    t = rows % w.T
    work = float(4 * w.d_h * w.g * w.k * (t + 1).sum())
    return work, dt, f"{len(rows)} of {w.B * w.T} token rows (route + all routed heads)"


def cpu_baseline(w, inp, target_s):
    """Calibrate a sample to about target_s seconds of oracle work, time it."""
    n = 8 if w.decode else 64
    work, dt, _ = oracle_sample(w, inp, n, 7)
    total = w.B if w.decode else w.B * w.T
    per = dt / n
    n2 = int(min(total, max(n, target_s / max(per, 1e-9))))
    work, dt, desc = oracle_sample(w, inp, n2, 8)
    scale = 1e-9 if w.decode else 1e-12
    unit = "GB/s" if w.decode else "TFLOP/s"
    return {"value": work / dt * scale, "unit": unit, "cores": os.cpu_count(), "kind": "oracle",
            "sample": desc, "seconds": round(dt, 2)}


def run_reference(w, steps, warmup):
    inp = gqe_synth.make_inputs(w)
    # size each step to ~2 s of oracle work so K+W steps end within minutes
    n = 8 if w.decode else 64
    work, dt, _ = oracle_sample(w, inp, n, 1)
    total = w.B if w.decode else w.B * w.T
    n_step = int(min(total, max(1, 2.0 / max(dt / n, 1e-9))))
    for i in range(warmup):
        oracle_sample(w, inp, max(1, n_step // 8), 100 + i)
    tot_work, tot_s, desc = 0.0, 0.0, ""
    for i in range(steps):
        wk, s, desc = oracle_sample(w, inp, n_step, 200 + i)
        tot_work += wk
        tot_s += s
    scale = 1e-9 if w.decode else 1e-12
    unit = "GB/s" if w.decode else "TFLOP/s"
    value = tot_work / tot_s * scale
    return value, unit, tot_s, desc


def compact_entry(r):
    """One config's figures for the line's "configs" map."""
    roof = r["roofline"]
    e = {"value": round(r["value"], 3), "unit": r["unit"], "attn_ms": round(r["attn_ms"], 5),
         "route_ms": round(r["route_ms"], 5), "bound": roof["bound"], "achieved": roof["achieved"],
         "frac": roof["frac"]}
    if roof.get("traffic") is not None:
        e["traffic"] = roof["traffic"]
    return e


# ---------------------------------------------------------------------------
def workload_config(w, ws):
    """The line's "config": the workload and how it is run, the same for both
    arms (the GPU arm and the CPU oracle arm print identical configs)."""
    return {"workload": w.name, "shape": w.describe(), "per_gpu_batch": w.B, "global_batch": w.B * ws,
            "parallelism": f"replicas x{ws} (no exchange step)",
            "l2": "GPU arm: flushed before every timed step, outside the step events (256 MB written, "
                  "read back); CPU oracle arm: not applicable"}


def gqe_line(metric, w, ws, steps, warmup, res, cpu, configs, extras):
    """The GPU arm's JSON line from one timed run (res: time_workload's result)."""
    line = {
        "metric": metric, "value": res["value"], "unit": res["unit"], "n_gpus": ws, "steps": steps,
        "warmup": warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded, gqe_synth recipe)",
        "config": workload_config(w, ws),
        "step_breakdown_ms": {"route": round(res["route_ms"], 5), "attn": round(res["attn_ms"], 5)},
        "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res.get("e2e"), "clocks": res["clocks"],
        "gpu_launches": res["gpu_launches"],
    }
    if configs:
        line["configs"] = configs
    if extras:
        line["extras"] = {"paged_decode_frac": extras["paged_decode"]["roofline"]["frac"],
                          "qproj_frac": extras["layer_ops"]["routed_qproj"]["roofline"]["frac"],
                          "oproj_frac": extras["layer_ops"]["routed_oproj"]["roofline"]["frac"],
                          "shared_head_frac": extras["layer_ops"]["shared_head"]["roofline"]["frac"],
                          "group_slots_frac": extras["layer_ops"]["group_slots"]["roofline"]["frac"],
                          "backward_ms": round(extras["backward"]["ms"], 3),
                          "backward_frac": extras["backward"]["roofline"]["frac"],
                          "route_backward_ms": round(extras["backward"]["router"]["ms"], 4)}
    return line


def reference_line(metric, w, ws, steps, warmup, value, unit, secs, desc):
    """The CPU oracle arm's JSON line."""
    return {"metric": metric, "impl": "reference", "value": value, "unit": unit, "n_gpus": ws,
            "steps": steps, "warmup": warmup, "ms_per_step": secs * 1e3 / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, gqe_synth recipe)",
            "config": workload_config(w, ws),
            "cpu_baseline": {"value": value, "unit": unit, "cores": os.cpu_count(), "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=PRIMARY, choices=sorted(gqe_synth.WORKLOADS))
    ap.add_argument("--impl", default="gqe", choices=["gqe", "reference"])
    ap.add_argument("--no-secondary", action="store_true", help="skip the other configs")
    ap.add_argument("--extras", action="store_true",
                    help="also time the calls around the hot path (paged decode, Q projection, shared head, "
                         "group slots, backward); a summary goes into the line")
    ap.add_argument("--extras-out", default=None, help="write the extras' full figures to this JSON file")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--layer-ops-only", action="store_true",
                    help="time only the calls around the routed attention (for profiling)")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the routed attention's backward (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = gqe_synth.WORKLOADS[args.workload]
    metric = "routed GQE attn TFLOP/s (prefill), KV-read GB/s (decode), % of B200 roofline"

    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        value, unit, secs, desc = run_reference(w, args.steps, args.warmup)
        line = reference_line(metric, w, args.gpus, args.steps, args.warmup, value, unit, secs, desc)
        print(json.dumps(line))
        return

    ws, rank, local = dist_setup()
    from routed_head_gqa_b200 import build as gqe_build

    if rank == 0:
        gqe_build.build()
    barrier(ws)
    peaks, peak_kind = load_peaks()
    if args.backward_only:
        bw = time_backward(w, args.steps, args.warmup, peaks, peak_kind)
        if rank == 0:
            print(json.dumps({"workload": w.name, "gqe_backward": bw}))
        if ws > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return
    if args.layer_ops_only:
        ops = time_layer_ops(w, args.steps, args.warmup, peaks, peak_kind)
        if rank == 0:
            print(json.dumps({"workload": w.name, "gqe_layer_ops": ops}))
        if ws > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return
    res = time_workload(w, args.steps, args.warmup, ws, rank, peaks, peak_kind, with_clocks=(rank == 0),
                        with_e2e=True)
    configs = {}
    if not args.no_secondary and args.workload == PRIMARY:
        for name in CONFIG_ORDER:
            if name == w.name:
                r2 = res
            else:
                r2 = time_workload(gqe_synth.WORKLOADS[name], max(5, args.steps // 2), 3, ws, rank, peaks,
                                   peak_kind, with_clocks=False, with_e2e=False)
            configs[name] = compact_entry(r2)
    extras = None
    if args.extras and args.workload == PRIMARY:
        extras = {}
        dw = gqe_synth.WORKLOADS["gqe_decode"]
        extras["paged_decode"] = time_paged_decode(dw, max(5, args.steps // 2), 3, peaks, peak_kind)
        lw = gqe_synth.WORKLOADS["dense_gqa"]
        extras["layer_ops"] = time_layer_ops(lw, max(5, args.steps // 2), 3, peaks, peak_kind)
        extras["backward"] = time_backward(lw, 3, 3, peaks, peak_kind)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, gqe_synth.make_inputs(w), args.cpu_seconds)
    if rank == 0:
        if extras and args.extras_out:
            with open(args.extras_out, "w") as f:
                json.dump(extras, f)
        line = gqe_line(metric, w, ws, args.steps, args.warmup, res, cpu, configs, extras)
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
