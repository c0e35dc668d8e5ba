#!/usr/bin/env python
"""Throughput of the Lighthouse selection layer, forward + backward, on B200.

One step is one pass of the whole hot path over one batch of synthetic input: the pyramid and
scores, the stratified top-K, the gather, the causal attention on the S rows and the
scatter-back, then the backward through all of them. Every stage runs in liblh.so. Inputs are
resident in HBM before the timed region; each input tensor (1 GiB at 128K) is larger than the
126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 128k] [--impl reference]

Under torchrun each rank runs its own copy of the workload (heads are independent problems),
there is no data-path collective, and rank 0 prints one JSON line with the whole-job tokens/s.
`--impl reference` times the CPU oracle (test infrastructure) on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "Lighthouse layer fwd+bwd tokens/s at N=128K, 1 B200; % of HBM / tensor roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one call of a stage, from one ncu
# capture, with the digest of the kernel sources the capture ran. `roofline.traffic` reports them
# only while those sources are unchanged; after any change it is null and `traffic_stale` true.
# (workload, stage) -> (bytes per call, source digest, how the bytes were obtained)
MEASURED_TRAFFIC = {
    ("128k", "attn_bwd"): (
        996068352, "4e12501af0a2f120",
        "ncu dram__bytes_read.sum + dram__bytes_write.sum of the D and one-pass kernels at 16 of the "
        "32 heads (two of four head groups), x2; reads grow in proportion to head groups (8 -> 16 "
        "heads: 156 -> 312 MB), writes faster (51 -> 186 MB), so the write part is a lower bound"),
}
# the sources whose kernels run in each stage
STAGE_SOURCES = {
    "pyramid_score": ["pool.cu"], "select": ["select.cu"], "gather": ["gather_scatter.cu"],
    "attn_fwd": ["attn_tc_fwd.cu", "tc.cuh"], "scatter": ["gather_scatter.cu"],
    "scatter_bwd": ["pool.cu"], "attn_bwd": ["attn_tc_bwd.cu", "tc.cuh"],
    "gather_bwd": ["gather_scatter.cu"],
}


def source_digest(stage):
    """sha256 (first 16 hex digits) of the CUDA sources of a stage's kernels, plus common.cuh."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_hierarchical_attention_b200", "csrc")
    for name in STAGE_SOURCES[stage] + ["common.cuh"]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_of(workload, stage):
    """(bytes or None, stale flag, note) of the measured DRAM traffic of one stage call."""
    rec = MEASURED_TRAFFIC.get((workload, stage))
    if rec is None:
        return None, False, "not captured for this workload"
    nbytes, digest, how = rec
    if digest != source_digest(stage):
        return None, True, "kernel sources changed since the capture"
    return nbytes, False, how


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="128k", choices=sorted(WORKLOADS))
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads (profiling captures on a smaller "
                         "case; 0 = the workload's own)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--also", default="1m",
                    help="comma-separated workloads also device-timed in the same run ('' for none)")
    ap.add_argument("--no-sdpa", action="store_true",
                    help="skip the dense causal SDPA context timing (run when N <= 128K)")
    args = ap.parse_args()
    args.also = [x for x in args.also.split(",") if x]
    for x in args.also:
        if x not in WORKLOADS:
            ap.error(f"--also: unknown workload {x}")
    return args


# ----------------------------------------------------------------------------- process group
def dist_setup(backend="nccl"):
    """One process per GPU (torchrun env). `gloo` serves the CPU tests of this host logic."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        kw = {"timeout": datetime.timedelta(seconds=300)}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(total_ms_local, steps, tokens_per_rank, world):
    """Whole-job tokens/s and ms per step. Every rank runs its own replica (weak scaling); the
    slowest rank's device time over the timed steps sets the job's time."""
    total_ms = max_over_ranks(total_ms_local, world)
    ms_step = total_ms / steps
    return tokens_per_rank * world / (ms_step / 1e3), ms_step


# ----------------------------------------------------------------------------- clocks
class Clocks:
    """SM clock, power and clock-event reasons sampled during the timed region.

    NVML is polled every 5 ms from a background thread (read-only queries), so that even a
    timed region of a few tens of milliseconds yields samples. The NVML device is found by the
    CUDA device's PCI bus id. Without NVML, nvidia-smi samples every 200 ms instead."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index, period_s=0.005):
        import threading
        self.samples, self.max_mhz, self.err = [], None, None
        self._stop = threading.Event()
        try:
            import pynvml as nv
            nv.nvmlInit()
            p = torch.cuda.get_device_properties(device_index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.bits = {name: getattr(nv, attr) for name, attr in self.REASONS}
        except Exception as e:  # noqa: BLE001  (no NVML: the nvidia-smi path below)
            self.nv, self.err = None, repr(e)
        if self.nv is None:
            self.smi = _SmiClocks(device_index)
            return
        self.thread = threading.Thread(target=self._poll, args=(period_s,), daemon=True)
        self.thread.start()

    def _poll(self, period_s):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                watts = nv.nvmlDeviceGetPowerUsage(self.h) / 1e3
                self.samples.append((mhz, mask, watts))
            except Exception as e:  # noqa: BLE001
                self.err = repr(e)
            self._stop.wait(period_s)

    def stop(self):
        if self.nv is None:
            return self.smi.stop()
        self._stop.set()
        self.thread.join(timeout=5)
        sm = [m for m, _, _ in self.samples]
        reasons = sorted({name for _, mask, _ in self.samples for name, bit in self.bits.items()
                          if mask & bit})
        load = [x for x in sm if x > 0.5 * self.max_mhz] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm), "source": "nvml, 5 ms",
                "power_w_max": round(max((w for _, _, w in self.samples), default=0.0), 1)}


class _SmiClocks:
    """nvidia-smi samples (200 ms) during the timed region, when NVML is not importable."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.file.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.file.read())) if len(r) >= 9]
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], None, set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(nm)
        load = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 200 ms"}


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK, "fallback"


# ----------------------------------------------------------------------------- algorithmic work
def stage_work(w, geo):
    """Algorithmic bytes (HBM-bound stages) or FLOPs (attention) per launch of each stage."""
    B, H, N, d, S = w.B, w.H, w.N, w.d, w.S
    e = torch.tensor([], dtype=w.dtype).element_size()
    R = geo["R"]
    BH = B * H
    return {
        "pyramid_score": ("hbm", 3 * BH * N * d * e + 3 * BH * R * d * e + BH * (N + R) * 4),
        "select": ("hbm", BH * (N + R) * 4 + BH * S * 4),
        "gather": ("hbm", 2 * 3 * BH * S * d * e + BH * S * 4),
        "attn_fwd": ("tensor", 2 * BH * S * S * d),
        "scatter": ("hbm", BH * S * d * 4 + BH * N * d * e + BH * S * 4),
        "scatter_bwd": ("hbm", BH * N * d * e + BH * S * d * e + BH * S * 4),
        "attn_bwd": ("tensor", 5 * BH * S * S * d),
        "gather_bwd": ("hbm", 3 * BH * S * d * 4 + 3 * BH * N * d * e + BH * S * 4),
    }


# ----------------------------------------------------------------------------- our arm
def make_stages(lh, w, dev, seed):
    """Device buffers of one workload and the eight stage calls of one step, in order."""
    from sparse_hierarchical_attention_b200 import Shape
    shape = Shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S, w.dtype)
    geo = lh.lh_validate(shape)
    B, H, N, d, S, dt = w.B, w.H, w.N, w.d, w.S, w.dtype
    R = geo["R"]
    q, k, v, d_o = make_inputs(w, dev, seed=seed)
    E = lambda *s, t=dt: torch.empty(*s, dtype=t, device=dev)  # noqa: E731
    pq, pk, pv = E(B, H, max(R, 1), d), E(B, H, max(R, 1), d), E(B, H, max(R, 1), d)
    score = E(B, H, N + R, t=torch.float32)
    idx = E(B, H, S, t=torch.int32)
    qs, ks, vs = (E(B, H, S, d) for _ in range(3))
    os_ = E(B, H, S, d, t=torch.float32)
    lse = E(B, H, S, t=torch.float32)
    o = E(B, H, N, d)
    dos = E(B, H, S, d)
    dqs, dks, dvs = (E(B, H, S, d, t=torch.float32) for _ in range(3))
    dq, dk, dv = (E(B, H, N, d) for _ in range(3))
    ws = torch.zeros(lh.lh_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    stages = [
        ("pyramid_score", lambda: lh.lh_build_pyramid(shape, q, k, v, pq, pk, pv, score, ws)),
        ("select", lambda: lh.lh_select_topk(shape, score, idx)),
        ("gather", lambda: lh.lh_gather(shape, q, k, v, pq, pk, pv, idx, qs, ks, vs, ws)),
        ("attn_fwd", lambda: lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)),
        ("scatter", lambda: lh.lh_scatter(shape, idx, os_, o)),
        ("scatter_bwd", lambda: lh.lh_scatter_bwd(shape, idx, d_o, dos, ws)),
        ("attn_bwd", lambda: lh.lh_attn_bwd(shape, qs, ks, vs, os_, lse, dos, dqs, dks, dvs, ws)),
        ("gather_bwd", lambda: lh.lh_gather_bwd(shape, idx, dqs, dks, dvs, dq, dk, dv)),
    ]
    return shape, geo, (q, k, v, d_o), ws, stages


def time_stages(lh, stages, ws, K, W, world, local):
    """W warm-up steps, then exactly K timed steps between a barrier and a synchronize on both
    sides. Returns (per-stage mean ms, per-step ms, device ms of the K steps, clocks, wall s)."""
    for _ in range(W):
        for _, fn in stages:
            fn()
    torch.cuda.synchronize()
    rc, flags = lh.lh_check(ws)
    if rc:
        raise RuntimeError(f"device fault flags {flags:#x} during warm-up")
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    clocks = Clocks(local)
    t_wall = time.perf_counter()
    for s in range(K):
        ev[s][0].record(stream)
        for i, (_, fn) in enumerate(stages):
            fn()
            ev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t_wall
    barrier(world)
    clk = clocks.stop()
    rc, flags = lh.lh_check(ws)
    if rc:
        raise RuntimeError(f"device fault flags {flags:#x} in the timed steps")
    step_ms = [ev[s][0].elapsed_time(ev[s][-1]) for s in range(K)]
    per_stage = {name: sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(K)) / K
                 for i, (name, _) in enumerate(stages)}
    return per_stage, step_ms, sum(step_ms), clk, wall


def report_stages(w, geo, per_stage):
    """Each stage's achieved rate and fraction of the measured peak, and the dominant stage's
    roofline object."""
    pk_, src = peaks()
    work = stage_work(w, geo)
    stage_report = {}
    for name, ms in per_stage.items():
        kind, amount = work[name]
        if kind == "hbm":
            ach, peak, unit = amount / (ms / 1e3) / 1e9, pk_["hbm_gbs"], "GB/s"
        else:
            ach, peak, unit = amount / (ms / 1e3) / 1e12, pk_["bf16_tflops"], "TFLOP/s"
        stage_report[name] = {"ms": round(ms, 4), "achieved": round(ach, 2), "unit": unit,
                              "frac": round(ach / peak, 4), "bound": kind}
        if kind != "hbm":  # against the sustained (power-capped) GEMM figure as well
            stage_report[name]["frac_sustained"] = round(ach / pk_["bf16_tflops_sustained"], 4)
    dom = max(per_stage, key=per_stage.get)
    kind, amount = work[dom]
    rf = stage_report[dom]
    traffic, stale, note = traffic_of(w.name, dom)
    if w.H != WORKLOADS[w.name].H:  # a profiling run on fewer heads: the table is per workload
        traffic, stale, note = None, False, "heads override: no measured traffic for this size"
    roofline = {"kernel": dom, "bound": "hbm" if kind == "hbm" else "tensor",
                "achieved": rf["achieved"], "peak": pk_["hbm_gbs"] if kind == "hbm" else pk_["bf16_tflops"],
                "unit": rf["unit"], "frac": rf["frac"], "traffic": traffic, "traffic_stale": stale,
                "traffic_note": note,
                "traffic_scope": "bytes of one stage call (all its launches), like achieved",
                "peak_source": f"{src} ({'hbm_gbs' if kind == 'hbm' else 'bf16_tflops'})",
                "units_per_launch": amount}
    return stage_report, roofline


def run_ours(args, world, rank, local):
    import dataclasses

    import sparse_hierarchical_attention_b200 as lh

    w = WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, H=args.heads)
    dev = torch.device("cuda", local)
    K, W = args.steps, args.warmup
    shape, geo, (q, k, v, d_o), ws, stages = make_stages(lh, w, dev, 1000 * rank)
    per_stage, step_ms, total_ms, clk, wall = time_stages(lh, stages, ws, K, W, world, local)
    value, ms_step = throughput(total_ms, K, w.B * w.N, world)
    stage_report, roofline = report_stages(w, geo, per_stage)
    nf, nb = lh.lh_launches(shape)
    del stages, ws
    torch.cuda.empty_cache()

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(lh, shape, w, dev, q, k, v, d_o, K, W, world)
    context = None
    if world == 1 and not args.no_sdpa and w.N <= 131072 and w.dtype == torch.bfloat16:
        context = dense_sdpa_context(q, k, v, d_o, ms_step)
    del q, k, v, d_o
    torch.cuda.empty_cache()
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms_step, 4),
        "ms_per_step_median_rank0": round(statistics.median(step_ms), 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded N(0,1) Q/K/V with the workload's row-scale recipe; dO N(0,1))",
        "config": workload_config(w, world),
        "stages": stage_report, "roofline": roofline, "gpu_launches": (nf + nb) * K,
        "clocks": clk, "wall_s_timed": round(wall, 3),
    }
    if e2e:
        out["e2e"] = e2e
    if context:
        out["context"] = context
    # further workloads in the same run, device-timed the same way (no e2e, no context)
    extra = {}
    for name in args.also:
        if name == w.name:
            continue
        wx = WORKLOADS[name]
        shape_x, geo_x, ins, ws_x, stages_x = make_stages(lh, wx, dev, 1000 * rank)
        per_x, steps_x, total_x, clk_x, _ = time_stages(lh, stages_x, ws_x, K, W, world, local)
        value_x, ms_x = throughput(total_x, K, wx.B * wx.N, world)
        rep_x, roof_x = report_stages(wx, geo_x, per_x)
        nfx, nbx = lh.lh_launches(shape_x)
        extra[name] = {"value": round(value_x, 1), "unit": "tokens/s", "ms_per_step": round(ms_x, 4),
                       "steps": K, "warmup": W, "config": workload_config(wx, world),
                       "stages": rep_x, "roofline": roof_x, "gpu_launches": (nfx + nbx) * K,
                       "clocks": clk_x}
        del ins, ws_x, stages_x
        torch.cuda.empty_cache()
    if extra:
        out["also"] = extra
    return out


def dense_sdpa_context(q, k, v, d_o, ms_layer):
    """Dense causal SDPA (torch's fused backends) fwd+bwd on the layer's own Q, K, V and dO, for
    context only: what full attention over all N tokens costs on the same GPU."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    qq, kk, vv = (t.detach().clone().requires_grad_(True) for t in (q, k, v))
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION):
        try:
            with sdpa_kernel([backend]):
                def step():
                    o = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
                    o.backward(d_o)
                step()
                torch.cuda.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(2):
                    step()
                b.record()
                torch.cuda.synchronize()
            ms = a.elapsed_time(b) / 2
            B, H, N, d = q.shape
            return {"what": "dense causal SDPA fwd+bwd over all N tokens, same shape and GPU",
                    "backend": backend.name, "ms_per_step": round(ms, 3),
                    "tflops": round(7 * B * H * N * N * d / (ms / 1e3) / 1e12, 1),  # causal: 2+5 N^2 d
                    "layer_speedup": round(ms / ms_layer, 2)}
        except RuntimeError:
            continue
    return {"what": "dense causal SDPA fwd+bwd", "unavailable": "no torch SDPA backend ran"}


def run_e2e(lh, shape, w, dev, q, k, v, d_o, K, W, world):
    """Same metric through the public layer API from pinned host buffers. Every step copies its
    Q, K, V, dO in, runs lh_layer_fwd + lh_layer_bwd and copies O, dQ, dK, dV out. Two buffer
    sets and two copy streams pipeline the steps: step t+1's inputs cross the host link while step
    t's outputs cross it the other way (the link is full duplex) and while the GPU computes."""
    from sparse_hierarchical_attention_b200 import LighthouseLayer
    layer = LighthouseLayer(shape, dev)
    h_in = [t.cpu().pin_memory() for t in (q, k, v, d_o)]
    h_out = [[torch.empty_like(h_in[0]).pin_memory() for _ in range(4)] for _ in range(2)]
    d_in = [[torch.empty_like(q) for _ in range(4)] for _ in range(2)]
    d_out = [[torch.empty_like(q) for _ in range(4)] for _ in range(2)]
    saved = layer.new_saved()
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    state = {"computed": [None, None], "copied": [None, None]}

    def step(t, after=None):
        b = t % 2
        if after is not None:
            s_in.wait_event(after)
        if state["computed"][b] is not None:  # d_in[b] is free once the step before last computed
            s_in.wait_event(state["computed"][b])
        with torch.cuda.stream(s_in):
            for h, dbuf in zip(h_in, d_in[b]):
                dbuf.copy_(h, non_blocking=True)
        ev_in = torch.cuda.Event()
        ev_in.record(s_in)
        main.wait_event(ev_in)
        if state["copied"][b] is not None:  # d_out[b] is free once its outputs left
            main.wait_event(state["copied"][b])
        layer.forward(d_in[b][0], d_in[b][1], d_in[b][2], o=d_out[b][0], saved=saved)
        layer.backward(saved, d_in[b][3], dq=d_out[b][1], dk=d_out[b][2], dv=d_out[b][3])
        ev_c = torch.cuda.Event()
        ev_c.record(main)
        state["computed"][b] = ev_c
        s_out.wait_event(ev_c)
        with torch.cuda.stream(s_out):
            for h, dbuf in zip(h_out[b], d_out[b]):
                h.copy_(dbuf, non_blocking=True)
        ev_o = torch.cuda.Event()
        ev_o.record(s_out)
        state["copied"][b] = ev_o

    for t in range(W):
        step(t)
    torch.cuda.synchronize()
    state["computed"], state["copied"] = [None, None], [None, None]
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for t in range(K):
        step(t, after=a if t == 0 else None)
    for ev in state["copied"]:  # the last outputs have reached the host
        if ev is not None:
            main.wait_event(ev)
    b.record(main)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world) / K
    layer.check()
    nbytes = sum(t.numel() * t.element_size() for t in h_in)
    return {"value": round(w.B * w.N * world / (ms / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in h_out[0]),
            "api": "LighthouseLayer.forward/backward -> lh_layer_fwd/lh_layer_bwd",
            "pipelining": "two buffer sets; copies in, compute and copies out on three streams"}


# ----------------------------------------------------------------------------- CPU oracle
def workload_config(w, world):
    """The `config` object of both arms' JSON lines: the workload, named by what it is."""
    return {"workload": w.name, "describe": w.describe, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "p": w.p, "L": w.L, "S": w.S, "global_batch": w.B * world, "seq_len": w.N,
            "parallelism": f"replicas x{world} (independent heads, no collective)",
            "l2": "inputs larger than L2 (each input tensor > 126 MB); no flush"}


def oracle_sample(w, frac, seed=0):
    """One head, the first N/frac tokens (same p, L and rows per chunk), on the host."""
    N, S = w.N // frac, w.S // frac
    q, k, v, d_o = make_inputs(w, "cpu", seed=seed, B=1, H=1, N=N)
    return [t.to(torch.float64).numpy() for t in (q, k, v, d_o)], N, S


def single_threaded():
    """Limits the BLAS thread pools to one thread while the oracle is timed; returns the
    limiter (a context manager) and the number of threads the timing then uses."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1), 1


def time_oracle(w, frac, steps=1):
    """Seconds of one oracle forward + backward over one head of N/frac tokens."""
    import oracle as O
    (q, k, v, d_o), N, S = oracle_sample(w, frac)
    geo = O.Geometry(N, w.p, w.L, S).check()
    store = "bf16" if w.dtype == torch.bfloat16 else "f32"
    g = 8 if w.dtype == torch.bfloat16 else 4
    t0 = time.perf_counter()
    for _ in range(steps):
        o, sv = O.layer_fwd(q, k, v, geo, g, store=store)
        O.layer_bwd(sv, d_o)
    dt = (time.perf_counter() - t0) / steps
    # layer tokens/s: this head's N tokens took dt; the layer runs B*H such heads
    value = N / (dt * w.H * w.B)
    return value, dt, N, S


def pick_sample(w, budget_s, runs):
    """Largest head prefix (1, 1/4 or 1/16 of the tokens) whose `runs` oracle passes are
    projected to fit `budget_s`, from one timed pass at 1/16. The oracle's time grows about as
    the sample's tokens to the power 1.5 (its attention is quadratic in the kept rows)."""
    _, t16, _, _ = time_oracle(w, 16)
    for frac in (1, 4):
        if runs * t16 * (16 / frac) ** 1.5 <= budget_s:
            return frac, t16
    return 16, t16


def sample_note(w, N, S):
    return (f"head 0 of {w.B * w.H}, first {N} of {w.N} tokens (S={S}, same p, L, rows per "
            f"chunk)" + ("" if N == w.N else "; a prefix has cheaper attention per token than "
            "the whole sequence, so this overstates the oracle's full-workload rate"))


def cpu_baseline(w, budget_s=30.0):
    """The oracle, single-threaded, on one head: the whole head if it fits the budget, else the
    longest prefix that does."""
    limiter, cores = single_threaded()
    with limiter:
        frac, _ = pick_sample(w, budget_s, 1)
        value, dt, N, S = time_oracle(w, frac)
    return {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{sample_note(w, N, S)}; fwd+bwd in {dt:.2f}s on one thread; tokens/s = "
                      f"{N}/({dt:.2f}s x {w.B * w.H} heads)"}


def run_reference(args, world, rank, budget_s=180.0):
    """The reference arm: the CPU oracle as it stands, single-threaded, on the GPU arm's
    workload and config. Each step is a bounded sample of it: one head (every head is the same
    problem), whole if all warm-up and timed steps fit about three minutes, else its longest
    prefix that does. The value is the layer's tokens/s if the B*H heads ran one after another
    on this core. This process imports only the oracle and the input generator, never the CUDA
    library."""
    w = WORKLOADS[args.workload]
    if rank != 0:
        return None
    limiter, cores = single_threaded()
    with limiter:
        frac, _ = pick_sample(w, budget_s, args.steps + args.warmup)
        for _ in range(args.warmup):
            time_oracle(w, frac)
        t0 = time.perf_counter()
        runs = [time_oracle(w, frac) for _ in range(args.steps)]
        total = time.perf_counter() - t0
    dt = sum(r[1] for r in runs) / len(runs)
    N, S = runs[0][2], runs[0][3]
    value = N / (dt * w.H * w.B)
    cb = {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
          "sample": f"each step: {sample_note(w, N, S)}; fwd+bwd on one thread; tokens/s = "
                    f"{N}/(seconds per step x {w.B * w.H} heads)"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * dt, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (same recipe as our arm)",
            "config": workload_config(w, world), "cpu_baseline": cb, "wall_s": round(total, 2),
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world, rank, local = dist_setup() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    out = run_ours(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(WORKLOADS[args.workload])
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
