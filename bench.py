#!/usr/bin/env python
"""Benchmark of rank-major MoE EP dispatch + combine on B200 (virtual EP ranks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the routing plan and
EPLB gather, the dispatch row copy, and the BF16 combine, on the prefill
workload (ep 8, 256 experts, top_k 8, 4096 tokens per rank, hidden 7168 BF16,
64 extra bytes per token, EPLB statistics).  Inputs are resident in HBM when
the timed region starts; they are larger than L2, so no flush is needed.
Rank 0 prints one JSON line.

With N > 1 (torchrun, one process per GPU) every rank runs its own independent
replica of the workload (the path has no exchange between GPUs: all EP ranks
are virtual ranks of one GPU); the timed region is bracketed by barriers and
the max over ranks is reported (weak scaling).

`--impl reference` times the plain CPU oracle on the host cores instead (rank 0
only), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "c4_ep8_prefill"
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------- #
# Process group helpers (also exercised on CPU with gloo by the tests)
# --------------------------------------------------------------------------- #

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_group(backend: str, timeout_s: float = 120.0):
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist if ws > 1 else None


def reduce_max(value: float, dist, device=None) -> float:
    """Max over ranks (identity on one rank)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None):
    if dist is None:
        return
    if device is not None and device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


class CudaTimer:
    """Device time between two events on the launching stream."""

    def __init__(self, stream):
        import torch
        self.torch = torch
        self.stream = stream
        self.a = torch.cuda.Event(enable_timing=True)
        self.b = torch.cuda.Event(enable_timing=True)

    def start(self):
        self.torch.cuda.synchronize()
        self.a.record(self.stream)

    def stop(self) -> float:
        self.b.record(self.stream)
        self.torch.cuda.synchronize()
        return float(self.a.elapsed_time(self.b))


def run_timed_flushed(step, flush, steps: int, warmup: int, stream, dist, device=None,
                      during=None) -> float:
    """Like run_timed, but L2 is flushed before every step and only the steps
    are timed (one event pair around each); returns the summed milliseconds,
    max over ranks."""
    import torch
    for _ in range(warmup):
        flush()
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(dist, device)
    torch.cuda.synchronize()
    if during is not None:
        during.start()
    for a, b in ev:
        flush()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    if during is not None:
        during.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev)
    barrier(dist, device)
    return reduce_max(ms, dist, device)


class WallTimer:
    """Host clock; used only by the CPU tests of the harness and the oracle arm."""

    def start(self):
        self.t = time.perf_counter()

    def stop(self) -> float:
        return (time.perf_counter() - self.t) * 1e3


def run_timed(step, steps: int, warmup: int, timer, dist, device=None,
              during=None, on_start=None) -> float:
    """W untimed steps, then exactly K timed steps bracketed by barriers and
    synchronisation; returns the max over ranks of the elapsed milliseconds.
    `on_start` runs after the warm-up, before the timed region opens."""
    for _ in range(warmup):
        step()
    if on_start is not None:
        on_start()
    barrier(dist, device)
    timer.start()
    if during is not None:
        during.start()
    for _ in range(steps):
        step()
    ms = timer.stop()
    if during is not None:
        during.stop()
    barrier(dist, device)
    return reduce_max(ms, dist, device)


# --------------------------------------------------------------------------- #
# Clocks during the timed region (NVML reads only; nothing is changed)
# --------------------------------------------------------------------------- #

_REASONS = [(0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
            (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
            (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
            (0x100, "display_clock_setting")]


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.error = None
        self.handle = None
        try:
            import pynvml
            self.nvml = pynvml
            pynvml.nvmlInit()
            try:
                import torch
                p = torch.cuda.get_device_properties(device_index)
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.reason_fn = fn
        except Exception as e:  # no NVML: report it, do not fail the bench
            self.error = f"{type(e).__name__}: {e}"

    def _loop(self):
        while not self.stop_flag.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.handle,
                                                                     self.nvml.NVML_CLOCK_SM))
                self.reasons |= int(self.reason_fn(self.handle))
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            time.sleep(self.period)

    def start(self):
        self.stop_flag = threading.Event()
        if self.handle is None:
            return
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def stop(self):
        self.stop_flag.set()
        if self.handle is not None:
            self.thread.join()

    def record(self):
        r = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
             "sm_max_mhz": self.max_mhz,
             "reasons": [n for bit, n in _REASONS if self.reasons & bit],
             "samples": len(self.samples)}
        if self.error:
            r["error"] = self.error
        return r


# --------------------------------------------------------------------------- #
# Algorithmic bytes (what the method must move; invalid rows and the dense
# ep x tpr capacity excluded)
# --------------------------------------------------------------------------- #

@dataclasses.dataclass
class Bytes:
    copy: int          # dispatch row copy: rows read once + written once per destination
    combine: int       # combine: valid rows read + output written
    route: int         # ids read, per-destination ids / valid rows, plan, counts, EPLB
    step: int


def algorithmic_bytes(w, n_tok: int, sum_d: int, live: int, fp8: bool,
                      live_slots: int = 0) -> Bytes:
    """live_slots > 0: the combine of per-expert outputs, which reads one bf16
    row per (token, slot) whose expert a live rank owns, plus ids and weights."""
    rb = sum(w.payload_row_bytes())
    k, ep, tpr, E, H = w.top_k, w.ep_size, w.tokens_per_rank, w.num_experts, w.hidden
    copy = n_tok * rb + sum_d * rb
    if live_slots:
        combine = live_slots * H * 2 + n_tok * k * 8 + n_tok * H * 2
    else:
        combine = sum_d * H * (1 if fp8 else 2) + n_tok * H * 2
    route = n_tok * k * 4 * (1 + 0) + sum_d * k * 4 + live * ep * tpr + ep * ep * 4
    if w.eplb:
        route += ep * E * 4 + live * ep * E * 4
    return Bytes(copy, combine, route, copy + combine + route)


def parse_options(items):
    """[("COMBINE_PIPELINE", 2), ...] from NAME=VALUE strings."""
    out = []
    for it in items or []:
        name, _, value = it.partition("=")
        out.append((name.strip().upper(), int(value)))
    return out


def l2_note(flushed: bool, step_bytes: int, l2_bytes: int) -> str:
    """How the timed steps meet the L2 rule, for the JSON line's config."""
    if flushed:
        return "512 MB L2 flush before every step, each step timed alone"
    mb, l2 = step_bytes / 1e6, l2_bytes / 1e6
    if step_bytes > 4 * l2_bytes:
        return f"inputs larger than L2 (no flush): each step moves {mb:.0f} MB, L2 holds {l2:.0f} MB"
    return (f"no flush, warm L2: each step moves {mb:.0f} MB and part of it stays in the "
            f"{l2:.0f} MB L2 between steps")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C++ source without comments and blank space, so that editing a comment
    does not count as changing a kernel (the sources hold no string literals
    with comment markers)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_sources_hash() -> str:
    """Hash of the CUDA sources' code (comments and spacing ignored), to tell
    whether committed ncu counters still describe the kernels that run."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_route_plan_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode())
                h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def device_mb_in_use(device) -> float:
    """Device memory in use (total minus free, cudaMemGetInfo) in MB: torch's
    tensors plus the library's own workspace, which torch does not see."""
    import torch
    free, total = torch.cuda.mem_get_info(device)
    return round((total - free) / 1e6, 1)


def committed_traffic(kernel: str, workload: str):
    """dram bytes per launch from profiles/dram_traffic.json, if it was taken on
    these exact kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("sources_hash") != kernel_sources_hash():
            return None
        e = d["kernels"][kernel]
        if e.get("workload") != workload:
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------------- #
# Every workload on the record: one measurement per (workload, combine input)
# --------------------------------------------------------------------------- #

# (workload, combine inputs) measured for the `workloads` record of the
# default line, besides the headline's prefill step: bf16 rows, E4M3 rows,
# E4M3 rows with a per-row scale, per-(token, slot) expert outputs.
RECORD_CASES = [
    ("c1_ep4_tiny", ("bf16", "fp8", "fp8s", "experts", "experts_fp8")),
    ("c2_ep8_decode", ("bf16", "fp8", "fp8s", "experts", "experts_fp8")),
    ("c3_ep16_zipf_nvfp4", ("bf16", "fp8", "fp8s", "experts", "experts_fp8")),
    ("c3_ep16_zipf_mxfp8", ("bf16",)),
    ("c3_ep16_zipf_dsfp8", ("bf16",)),
    ("c5_ep64_wide_masked", ("bf16", "fp8", "fp8s", "experts", "experts_fp8")),
]
COMBINE_KINDS = {"bf16": "BF16 rows", "fp8": "FP8 E4M3 rows",
                 "fp8s": "FP8 E4M3 rows + per-row fp32 scale",
                 "experts": "per-(token, slot) BF16 expert outputs, weighted reduction fused",
                 "experts_fp8": "per-(token, slot) BF16 expert outputs, weighted reduction and "
                                "per-row E4M3 quantisation fused (sender-side FP8)"}


def live_slot_count(w, x) -> int:
    """(token, slot) pairs of existing tokens whose expert a live rank owns: the
    rows the combine of per-slot expert outputs reads."""
    idn = x.token_selected_experts.numpy()
    n = x.local_num_tokens
    owner = np.where((idn >= 0) & (idn < w.num_experts), idn // w.experts_per_rank, -1)
    alive = np.array([r not in w.masked_ranks for r in range(w.ep_size)] + [False])
    exists = (np.arange(w.tokens_per_rank)[None, :] < n[:, None]) & alive[:w.ep_size, None]
    return int((alive[owner] & exists[:, :, None]).sum())


class DeviceCase:
    """One workload's inputs on the device and a handle, with the step of each
    combine input.  Combine inputs are drawn on the device from a seeded CUDA
    generator (their values do not change the work), unless given."""

    def __init__(self, w, x, device, kinds, xo=None):
        import torch
        from combine_route_plan_b200 import ep_a2a
        self.w, self.x = w, x
        self.ids = x.token_selected_experts.to(device)
        self.payloads = [p.to(device) for p in x.payloads]
        self.stats = x.eplb_local_stats.to(device) if x.eplb_local_stats is not None else None
        self.n, self.mask = x.local_num_tokens, x.active_rank_mask
        ep, tpr, k, H = w.ep_size, w.tokens_per_rank, w.top_k, w.hidden
        gen = torch.Generator(device=device).manual_seed(w.seed + 55)
        if xo is None and set(kinds) & {"bf16", "fp8", "fp8s"}:
            xo = torch.randn((ep, ep * tpr, H), generator=gen, device=device,
                             dtype=torch.bfloat16)
        self.xo = xo
        self.xo8 = ep_a2a.quantize_e4m3(xo) if "fp8" in kinds else None
        self.codes = self.row_scales = None
        if "fp8s" in kinds:
            self.codes, self.row_scales = ep_a2a.quantize_e4m3_rows(xo)
        self.y = self.wts = None
        if "experts" in kinds or "experts_fp8" in kinds:
            self.y = torch.randn((ep, tpr, k, H), generator=gen, device=device,
                                 dtype=torch.bfloat16)
            self.wts = self.payloads[-1].view(torch.float32).view(ep, tpr, k)
        self.out = torch.empty((ep, tpr, H), dtype=torch.bfloat16, device=device)
        self.comm = ep_a2a.EpA2A(ep, w.num_experts, k, tpr, H, w.payload_row_bytes(),
                                 eplb_stats_num_experts=w.num_experts if w.eplb else 0,
                                 enable_rank_mask=self.mask is not None)
        d = self.comm.dispatch(self.ids, self.n, self.payloads, tpr, self.stats, self.mask)
        torch.cuda.synchronize()
        self.sum_d = int(d.send_counts.sum().item())
        self.live = ep - len(w.masked_ranks)
        self.n_tok = int(sum(int(self.n[r]) for r in range(ep) if r not in w.masked_ranks))
        self.live_slots = live_slot_count(w, x) if ("experts" in kinds or
                                                    "experts_fp8" in kinds) else 0

    def step(self, kind):
        c, tpr = self.comm, self.w.tokens_per_rank

        def dispatch():
            c.dispatch(self.ids, self.n, self.payloads, tpr, self.stats, self.mask, views=False)
        if kind == "bf16":
            return lambda: (dispatch(), c.combine(self.xo, self.out))
        if kind == "fp8":
            return lambda: (dispatch(), c.combine(self.xo8, self.out))
        if kind == "fp8s":
            return lambda: (dispatch(), c.combine_scaled(self.codes, self.row_scales, self.out))
        if kind == "experts_fp8":
            return lambda: (dispatch(), c.combine_experts_fp8(self.wts, self.y, self.out))
        return lambda: (dispatch(), c.combine_experts(self.wts, self.y, self.out))

    def bytes(self, kind) -> "Bytes":
        by = algorithmic_bytes(self.w, self.n_tok, self.sum_d, self.live, kind in ("fp8", "fp8s"),
                               self.live_slots if kind in ("experts", "experts_fp8") else 0)
        if kind == "fp8s":        # the row scales travel with the codes
            by = dataclasses.replace(by, combine=by.combine + self.sum_d * 4,
                                     step=by.step + self.sum_d * 4)
        return by

    def destroy(self):
        self.comm.destroy()


def measure_case(case, kind, steps, warmup, stream, flush_buf, graph, peak, clean_buf=None):
    """Step time (CUDA events; with flush_buf, L2 is flushed before every step
    and each step is timed alone), per-kernel times from an eager pass with
    events around each launch, and the roofline figures of both.  With
    clean_buf, a second timed loop flushes the same way and then reads
    clean_buf (larger than L2), so each step also starts with no dirty lines
    in L2: the write flush leaves L2 full of dirty lines that the step would
    otherwise write back to DRAM on its own time."""
    import torch
    from combine_route_plan_b200 import ep_a2a
    step = case.step(kind)

    def flushed():
        if flush_buf is not None:
            flush_buf.zero_()
        step()
    for _ in range(warmup):
        flushed()
    torch.cuda.synchronize()
    ep_a2a.ep_a2a_profile_start(case.comm.handle, 4 * steps + 8)
    for _ in range(steps):
        flushed()
    kt = ep_a2a.ep_a2a_profile_stop(case.comm.handle)
    timed = step
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g):
            step()
        timed = g.replay
    if flush_buf is not None:
        ms = run_timed_flushed(timed, lambda: flush_buf.zero_(), steps, warmup, stream, None)
    else:
        ms = run_timed(timed, steps, warmup, CudaTimer(stream), None)
    ms_clean = None
    if flush_buf is not None and clean_buf is not None:
        def clean_flush():
            flush_buf.zero_()
            clean_buf.amax()
        ms_clean = run_timed_flushed(timed, clean_flush, steps, warmup, stream, None)
    torch.cuda.synchronize()
    del g
    if case.comm.get_status() != ep_a2a.OK:
        raise RuntimeError("device error word set")
    by = case.bytes(kind)
    step_s = ms / steps / 1e3
    kbytes = {"route_plan": by.route, "copy_vec": by.copy, "copy_bulk": by.copy,
              "copy_staged": by.copy, "combine": by.combine, "combine_experts": by.combine,
              "combine_experts_fp8": by.combine}
    if not kt["route_plan"][0]:     # the copy kernel routed the tokens itself
        kbytes["copy_vec"] = by.copy + by.route
    kernels = {}
    for name, (cnt, tot) in kt.items():
        if cnt:
            avg_s = tot / cnt / 1e3
            kernels[name] = {"avg_us": avg_s * 1e6, "algorithmic_bytes": kbytes[name],
                             "gbs": kbytes[name] / avg_s / 1e9,
                             "frac": kbytes[name] / avg_s / 1e9 / peak}
    rec = {"workload": case.w.name, "combine": kind, "step_us": step_s * 1e6,
           "tokens_per_s": case.n_tok / step_s, "step_algorithmic_bytes": by.step,
           "step_gbs": by.step / step_s / 1e9, "step_frac": by.step / step_s / 1e9 / peak,
           "tokens": case.n_tok, "mean_distinct_ranks": case.sum_d / max(case.n_tok, 1),
           "kernels": kernels}
    if ms_clean is not None:
        clean_s = ms_clean / steps / 1e3
        rec["clean_l2"] = {"step_us": clean_s * 1e6, "tokens_per_s": case.n_tok / clean_s,
                           "step_frac": by.step / clean_s / 1e9 / peak}
    return rec


def workloads_record(args, device, stream, peak, prefill_case=None):
    """The `workloads` record: every other workload with every combine input
    (L2 flushed before each step, CUDA-graph replay of the step), and the
    prefill step with the other combine inputs (eager, inputs larger than L2)."""
    import gc
    import torch
    from combine_route_plan_b200 import workloads as W
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    clean_buf = torch.ones(512 << 20, dtype=torch.uint8, device=device)
    out = []
    for name, kinds in RECORD_CASES:
        w = W.BY_NAME[name]
        case = DeviceCase(w, W.make_inputs(w, with_expert_output=False), device, kinds)
        for kind in kinds:
            r = measure_case(case, kind, args.workload_steps, 5, stream, flush_buf, True, peak,
                             clean_buf=clean_buf)
            r["timing"] = ("CUDA-graph replay, 512 MB L2 flush (written) before each step, steps "
                           "timed alone; clean_l2: the same flush followed by a 512 MB read, so "
                           "the step also starts with no dirty lines in L2")
            out.append(r)
        case.destroy()
        del case
        gc.collect()
        torch.cuda.empty_cache()
    del flush_buf, clean_buf
    if prefill_case is not None:
        for kind in ("fp8", "fp8s", "experts", "experts_fp8"):
            r = measure_case(prefill_case, kind, args.workload_steps, 5, stream, None, False, peak)
            r["timing"] = "eager, inputs larger than L2 (no flush)"
            out.append(r)
    return out


# --------------------------------------------------------------------------- #
# Our arm
# --------------------------------------------------------------------------- #

def run_ours(args):
    import torch
    from combine_route_plan_b200 import ep_a2a
    from combine_route_plan_b200 import workloads as W

    ws, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_group("nccl")
    w = W.BY_NAME[args.workload]
    if args.tokens_per_rank:
        w = W.scaled(w, args.tokens_per_rank)
    x = W.make_inputs(w)
    if args.e2e_steps > 0:
        # the end-to-end leg copies from pinned host memory: pin the inputs once
        # (in place of the pageable copies, so the host holds one copy)
        x = dataclasses.replace(
            x, token_selected_experts=x.token_selected_experts.pin_memory(),
            payloads=[p.pin_memory() for p in x.payloads],
            eplb_local_stats=(x.eplb_local_stats.pin_memory()
                              if x.eplb_local_stats is not None else None),
            expert_output=x.expert_output.pin_memory())
    stream = torch.cuda.current_stream()

    ids = x.token_selected_experts.to(device)
    payloads = [p.to(device) for p in x.payloads]
    stats = x.eplb_local_stats.to(device) if x.eplb_local_stats is not None else None
    xo = x.expert_output.to(device)
    # the E4M3 rows only when something reads them (profiling runs keep the
    # device footprint small)
    xo8 = ep_a2a.quantize_e4m3(xo) if (args.combine == "fp8" or args.fp8_steps > 0) else None
    experts = args.combine in ("experts", "experts_fp8")
    experts_fp8 = args.combine == "experts_fp8"
    scaled = args.combine == "fp8s"
    if scaled:
        codes, row_scales = ep_a2a.quantize_e4m3_rows(xo)
    if experts:
        # one bf16 row per (token, slot), drawn on the device (seeded)
        gen = torch.Generator(device=device).manual_seed(w.seed + 77)
        y = torch.randn((w.ep_size, w.tokens_per_rank, w.top_k, w.hidden), generator=gen,
                        device=device).to(torch.bfloat16)
        wts = payloads[-1].view(torch.float32).view(w.ep_size, w.tokens_per_rank, w.top_k)
    n = x.local_num_tokens
    mask = x.active_rank_mask
    comm = ep_a2a.EpA2A(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank, w.hidden,
                        w.payload_row_bytes(), eplb_stats_num_experts=w.num_experts if w.eplb else 0,
                        enable_rank_mask=mask is not None)
    if args.no_pdl:
        comm.set_option(ep_a2a.OPT_PDL, 0)
    for name, value in parse_options(args.opt):
        comm.set_option(getattr(ep_a2a, "OPT_" + name), value)
    out = torch.empty((w.ep_size, w.tokens_per_rank, w.hidden), dtype=torch.bfloat16, device=device)
    tpr = w.tokens_per_rank
    fp8 = args.combine == "fp8"
    comb_in = xo8 if fp8 else xo

    dense = args.variant == "agrs"
    if dense:
        # the all-gather writes into the same receive arrays the rank-major
        # dispatch uses (taken from one dispatch result)
        res0 = comm.dispatch(ids, n, payloads, tpr, stats, mask, views=False)
        recv_ptrs = [res0.recv_payloads[i] for i in range(len(payloads))]
        pay_ptrs = [p.data_ptr() for p in payloads]
        rows = w.payload_row_bytes()
        dense_calls = [
            lambda: ep_a2a.ep_a2a_allgather(w.ep_size, tpr, n, pay_ptrs, rows, recv_ptrs,
                                            res0.rank_stride_bytes, mask),
            lambda: ep_a2a.ep_a2a_reduce_scatter(w.ep_size, tpr, w.hidden, n, xo.data_ptr(),
                                                 out.data_ptr(), mask)]

    def step():
        if dense:
            for call in dense_calls:
                call()
            return
        comm.dispatch(ids, n, payloads, tpr, stats, mask, views=False)
        if experts_fp8:
            comm.combine_experts_fp8(wts, y, out)
        elif experts:
            comm.combine_experts(wts, y, out)
        elif scaled:
            comm.combine_scaled(codes, row_scales, out)
        else:
            comm.combine(comb_in, out)

    step()
    torch.cuda.synchronize()
    d = comm.dispatch(ids, n, payloads, tpr, stats, mask)
    torch.cuda.synchronize()
    assert comm.get_status() == ep_a2a.OK
    sum_d = int(d.send_counts.sum().item())
    live = w.ep_size - len(w.masked_ranks)
    n_tok = int(sum(int(n[r]) for r in range(w.ep_size) if r not in w.masked_ranks))
    live_slots = live_slot_count(w, x) if experts else 0
    if dense:       # every existing token goes to, and is summed over, every live rank
        sum_d = n_tok * live
    by = algorithmic_bytes(w, n_tok, sum_d, live, fp8 or scaled, live_slots)
    if scaled:      # the row scales travel with the codes
        by = dataclasses.replace(by, combine=by.combine + sum_d * 4, step=by.step + sum_d * 4)

    clocks = ClockSampler(local)
    flush_buf = None
    if args.l2_flush:
        flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    if args.graph or flush_buf is not None:
        # per-kernel times from an eager profiled pass (flushing L2 before each
        # step when the timed loop does), then the timed loop without events
        # between the kernels
        def flushed_step():
            if flush_buf is not None:
                flush_buf.zero_()
            step()
        if dense:
            for _ in range(args.warmup):
                flushed_step()
            kt = dense_call_times(dense_calls, args.steps, stream,
                                  flush=(lambda: flush_buf.zero_()) if flush_buf is not None
                                  else None)
        else:
            run_timed(flushed_step, args.steps, args.warmup, CudaTimer(stream), dist, device,
                      on_start=lambda: ep_a2a.ep_a2a_profile_start(comm.handle,
                                                                   4 * args.steps + 8))
            kt = ep_a2a.ep_a2a_profile_stop(comm.handle)
        timed_step = step
        if args.graph:
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                step()
            torch.cuda.current_stream().wait_stream(side)
            with torch.cuda.graph(graph):
                step()
            timed_step = graph.replay
        if flush_buf is not None:
            ms = run_timed_flushed(timed_step, lambda: flush_buf.zero_(), args.steps, args.warmup,
                                   stream, dist, device, during=clocks)
        else:
            ms = run_timed(timed_step, args.steps, args.warmup, CudaTimer(stream), dist, device,
                           during=clocks)
    elif dense:
        ms = run_timed(step, args.steps, args.warmup, CudaTimer(stream), dist, device,
                       during=clocks)
        kt = dense_call_times(dense_calls, args.steps, stream)
    else:
        # the headline: K steps with nothing recorded between the kernels (an
        # event between two kernels would stop them from overlapping)
        ms = run_timed(step, args.steps, args.warmup, CudaTimer(stream), dist, device,
                       during=clocks)
        # per-kernel durations: a second timed region of K steps, each kernel
        # bracketed by CUDA events on its launch stream
        run_timed(step, args.steps, 0, CudaTimer(stream), dist, device,
                  on_start=lambda: ep_a2a.ep_a2a_profile_start(comm.handle, 4 * args.steps + 8))
        kt = ep_a2a.ep_a2a_profile_stop(comm.handle)
    torch.cuda.synchronize()
    assert comm.get_status() == ep_a2a.OK
    ms_per_step = ms / args.steps
    tokens_total = ws * n_tok * args.steps
    value = tokens_total / (ms / 1e3)
    peak, peak_kind = load_peaks()

    per_kernel = {}
    for name, (cnt, tot) in kt.items():
        if cnt:
            per_kernel[name] = {"launches": cnt, "avg_ms": tot / cnt}
    kbytes = {"route_plan": by.route, "copy_bulk": by.copy, "copy_vec": by.copy,
              "copy_staged": by.copy, "combine": by.combine, "combine_experts": by.combine,
              "combine_experts_fp8": by.combine,
              "allgather": by.copy, "reduce_scatter": by.combine}
    if "copy_vec" in per_kernel and "route_plan" not in per_kernel:
        kbytes["copy_vec"] = by.copy + by.route     # the copy kernel routed the tokens itself
    for name, e in per_kernel.items():
        e["algorithmic_bytes"] = kbytes[name]
        e["achieved_gbs"] = kbytes[name] / (e["avg_ms"] / 1e3) / 1e9
        e["frac_of_peak"] = e["achieved_gbs"] / peak
    dominant = max(per_kernel, key=lambda k: per_kernel[k]["avg_ms"] * per_kernel[k]["launches"])
    dk = per_kernel[dominant]
    step_gbs = by.step / (ms_per_step / 1e3) / 1e9

    # FP8 combine, timed alone on the same plan (context, not the headline)
    fp8_ctx = None
    if not fp8 and not experts and not scaled and not dense and args.fp8_steps > 0:
        comm.dispatch(ids, n, payloads, tpr, stats, mask)
        t8 = run_timed(lambda: comm.combine(xo8, out), args.fp8_steps, 3, CudaTimer(stream),
                       dist, device, on_start=lambda: ep_a2a.ep_a2a_profile_start(
                           comm.handle, args.fp8_steps + 4))
        k8 = ep_a2a.ep_a2a_profile_stop(comm.handle)["combine"]
        b8 = algorithmic_bytes(w, n_tok, sum_d, live, True).combine
        avg8 = k8[1] / k8[0]
        fp8_ctx = {"avg_ms": avg8, "algorithmic_bytes": b8,
                   "achieved_gbs": b8 / (avg8 / 1e3) / 1e9, "frac_of_peak": b8 / (avg8 / 1e3) / 1e9 / peak,
                   "loop_ms_per_launch": t8 / args.fp8_steps}

    e2e = None
    if args.e2e_steps > 0:
        e2e = None if (scaled or dense) else run_e2e(args, w, x, comm, device, stream, dist, n_tok, ws,
                                          y_dev=y if experts else None,
                                          experts_fp8=experts_fp8)

    # every other workload and combine input on the record (one GPU only; the
    # headline above is unaffected: it was timed before any of this ran)
    records = None
    if (rank == 0 and ws == 1 and args.workload_steps > 0 and not dense and not experts
            and not scaled and not fp8 and args.workload == DEFAULT_WORKLOAD
            and not args.tokens_per_rank):
        pc = DeviceCase(w, x, device, ("fp8", "fp8s", "experts", "experts_fp8"), xo=xo)
        records = workloads_record(args, device, stream, peak, pc)
        pc.destroy()
        del pc

    cpu = cpu_all = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)
        if args.cpu_all_cores_seconds > 0:
            cpu_all = cpu_baseline_all_cores(w, args.cpu_all_cores_seconds)

    if rank == 0:
        rec = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": f"{w.name}: ep_size {w.ep_size}, num_experts {w.num_experts}, "
                            f"top_k {w.top_k}, {tpr} tokens/rank, hidden {w.hidden} BF16, "
                            f"extra {w.extra_bytes} B/token, EPLB stats, "
                            + ("combine of per-expert outputs (weighted local reduction "
                               "and per-row E4M3 quantisation fused, fp32 accumulate)"
                               if experts_fp8 else
                               "combine of per-expert outputs (weighted local reduction "
                               "fused, fp32 accumulate)" if experts else
                               f"{'FP8 E4M3 with a per-row fp32 scale' if scaled else 'FP8 E4M3' if fp8 else 'BF16'} combine (fp32 accumulate)"),
                "tokens_per_step_per_gpu": n_tok, "mean_distinct_ranks": sum_d / n_tok,
                "l2": l2_note(args.l2_flush, by.step,
                              getattr(torch.cuda.get_device_properties(device),
                                      "L2_cache_size", 0) or (126 << 20)),
                "launch": ("CUDA graph replay" if args.graph else "eager") +
                          (", programmatic dependent launch" if not args.no_pdl else ""),
                "kernel_times": "CUDA events around each launch, in a second timed region of "
                                "the same K steps (events between kernels stop them overlapping)",
                "parallelism": f"{ws} independent replicas" if ws > 1 else "1 GPU, virtual ranks",
                "variant": ("dense: all-gather dispatch + reduce-scatter combine (vllm AgRs)"
                            if dense else "rank-major dispatch + combine"),
                "options": dict(parse_options(args.opt)) or "library defaults",
            },
            "hbm": {"step_algorithmic_bytes": by.step, "achieved_gbs": step_gbs,
                    "peak_gbs": peak, "peak_kind": peak_kind, "frac": step_gbs / peak},
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": dk["achieved_gbs"],
                         "peak": peak, "unit": "GB/s", "frac": dk["frac_of_peak"],
                         "peak_kind": peak_kind,
                         "traffic": committed_traffic(dominant, w.name)},
            "kernels": per_kernel,
            "gpu_launches": sum(e["launches"] for e in per_kernel.values()),
            "clocks": clocks.record(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "cpu_baseline_all_cores": cpu_all,
            "kernel_sources": kernel_sources_hash(),
            "device_mb_in_use": device_mb_in_use(device),
        }
        if fp8_ctx:
            rec["fp8_combine"] = fp8_ctx
        if records is not None:
            rec["workloads"] = records
        print(json.dumps(rec), flush=True)
    comm.destroy()
    if dist is not None:
        dist.destroy_process_group()


def dense_call_times(calls, steps, stream, flush=None):
    """{name: (launches, total ms)} of the dense variant's two calls, each
    bracketed by CUDA events on the stream (they have no handle to profile)."""
    import torch
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(steps)] for _ in calls]
    for i in range(steps):
        if flush is not None:
            flush()
        for c, call in enumerate(calls):
            evs[c][i][0].record(stream)
            call()
            evs[c][i][1].record(stream)
    torch.cuda.synchronize()
    return {name: (steps, sum(a.elapsed_time(b) for a, b in ev))
            for name, ev in zip(("allgather", "reduce_scatter"), evs)}


def run_e2e(args, w, x, comm, device, stream, dist, n_tok, ws, y_dev=None, experts_fp8=False):
    """Same step through the public API with the inputs in pinned host memory:
    every step copies the inputs host->device and the result device->host.
    With y_dev (the combine of per-expert outputs) the combine input is the
    per-(token, slot) expert outputs instead of per-rank rows."""
    import torch
    h_ids = x.token_selected_experts.pin_memory()
    h_pay = [p.pin_memory() for p in x.payloads]
    h_stats = x.eplb_local_stats.pin_memory() if x.eplb_local_stats is not None else None
    h_xo = (y_dev.cpu() if y_dev is not None else x.expert_output).pin_memory()
    h_out = torch.empty((w.ep_size, w.tokens_per_rank, w.hidden), dtype=torch.bfloat16).pin_memory()
    d_ids = torch.empty_like(h_ids, device=device)
    d_pay = [torch.empty_like(p, device=device) for p in h_pay]
    d_stats = torch.empty_like(h_stats, device=device) if h_stats is not None else None
    d_xo = torch.empty_like(h_xo, device=device)
    d_out = torch.empty_like(h_out, device=device)
    h2d = h_ids.nbytes + sum(p.nbytes for p in h_pay) + h_xo.nbytes + \
        (h_stats.nbytes if h_stats is not None else 0)
    d2h = h_out.nbytes

    # Three streams: the inputs go up on s_in once the previous step's kernels
    # are done with the device buffers, the result comes down on s_out, so a
    # step's result download overlaps the next step's upload (separate copy
    # engines, PCIe is full duplex); the kernels run on `stream`.
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def step():
        s_in.wait_stream(stream)
        with torch.cuda.stream(s_in):
            d_ids.copy_(h_ids, non_blocking=True)
            for d, h in zip(d_pay, h_pay):
                d.copy_(h, non_blocking=True)
            if d_stats is not None:
                d_stats.copy_(h_stats, non_blocking=True)
            d_xo.copy_(h_xo, non_blocking=True)
        stream.wait_stream(s_in)
        comm.dispatch(d_ids, x.local_num_tokens, d_pay, w.tokens_per_rank, d_stats,
                      x.active_rank_mask, stream=stream, views=False)
        stream.wait_stream(s_out)        # d_out: the previous download is done
        if y_dev is not None:
            wts = d_pay[-1].view(torch.float32).view(w.ep_size, w.tokens_per_rank, w.top_k)
            if experts_fp8:
                comm.combine_experts_fp8(wts, d_xo, d_out, stream=stream)
            else:
                comm.combine_experts(wts, d_xo, d_out, stream=stream)
        else:
            comm.combine(d_xo, d_out, stream=stream)
        s_out.wait_stream(stream)
        with torch.cuda.stream(s_out):
            h_out.copy_(d_out, non_blocking=True)

    class JoinTimer(CudaTimer):
        """Stops only after the last step's download."""

        def stop(self) -> float:
            self.stream.wait_stream(s_out)
            return super().stop()

    ms = run_timed(step, args.e2e_steps, 2, JoinTimer(stream), dist, device)
    return {"value": ws * n_tok * args.e2e_steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": args.e2e_steps, "ms_per_step": ms / args.e2e_steps}


# --------------------------------------------------------------------------- #
# The oracle on the host cores
# --------------------------------------------------------------------------- #

def oracle_step(w, x):
    """One pass of the whole path in the CPU oracle."""
    import oracle
    plan = oracle.route(w.ep_size, w.num_experts, w.top_k, w.tokens_per_rank,
                        x.token_selected_experts.numpy(), x.local_num_tokens, x.active_rank_mask)
    for p in x.payloads:
        oracle.dispatch_payload(plan, p.numpy())
    if x.eplb_local_stats is not None:
        oracle.eplb_gather(w.ep_size, x.eplb_local_stats.numpy(), x.active_rank_mask)
    xo = x.expert_output.view(__import__("torch").int16).numpy().view(np.uint16)
    oracle.combine(plan, xo, w.hidden)
    return int(sum(int(x.local_num_tokens[r]) for r in range(w.ep_size)
                   if r not in w.masked_ranks))


def cpu_baseline(w, seconds: float, tokens_per_rank: int = 1024):
    """The oracle as it stands, single-threaded, on a bounded sample of the
    workload: the same shapes with fewer tokens per rank, repeated for at
    least `seconds`."""
    from combine_route_plan_b200 import workloads as W
    import oracle
    oracle.build()
    ws = W.scaled(w, min(tokens_per_rank, w.tokens_per_rank))
    xs = W.make_inputs(ws)
    oracle_step(ws, xs)            # untimed: page in buffers
    t0 = time.perf_counter()
    toks = reps = 0
    while True:
        toks += oracle_step(ws, xs)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": toks / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{ws.name}: {ws.tokens_per_rank} tokens/rank "
                      f"({toks // reps} tokens) x {reps} steps, route + dispatch + EPLB + "
                      f"BF16 combine, {dt:.1f} s, single thread",
            "host_cpus": os.cpu_count()}


def _oracle_worker(name: str, tokens_per_rank: int, seconds: float, barrier_, results):
    """One process of the all-cores baseline: the oracle, single-threaded, on
    its own copy of the sample, from the moment every process is ready."""
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import torch
    torch.set_num_threads(1)
    from combine_route_plan_b200 import workloads as W
    ws = W.scaled(W.BY_NAME[name], tokens_per_rank)
    xs = W.make_inputs(ws)
    oracle_step(ws, xs)            # untimed: page in buffers
    barrier_.wait()
    t0 = time.perf_counter()
    toks = reps = 0
    while True:
        toks += oracle_step(ws, xs)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    results.put((toks, time.perf_counter() - t0, reps))


def cpu_baseline_all_cores(w, seconds: float, tokens_per_rank: int = 128, procs: int = 0):
    """The oracle as it stands on every host core: one single-threaded process
    per core, each on its own copy of a bounded sample (the same shapes with
    fewer tokens per rank), started together; tokens of all processes over
    the slowest one's time.  Processes are spawned (never forked after CUDA
    work)."""
    import multiprocessing as mp
    import oracle
    oracle.build()
    n = procs or len(os.sched_getaffinity(0))
    ctx = mp.get_context("spawn")
    barrier_ = ctx.Barrier(n)
    results = ctx.Queue()
    tpr = min(tokens_per_rank, w.tokens_per_rank)
    ps = [ctx.Process(target=_oracle_worker, args=(w.name, tpr, seconds, barrier_, results))
          for _ in range(n)]
    for p in ps:
        p.start()
    got = [results.get(timeout=600) for _ in ps]
    for p in ps:
        p.join(timeout=60)
    toks = sum(g[0] for g in got)
    dt = max(g[1] for g in got)
    reps = min(g[2] for g in got)
    return {"value": toks / dt, "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"{w.name} at {tpr} tokens/rank: {n} single-threaded processes, each on "
                      f"its own copy, >= {reps} steps of route + dispatch + EPLB + BF16 combine "
                      f"in {dt:.1f} s"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return                      # rank 0 alone runs the CPU oracle
    from combine_route_plan_b200 import workloads as W
    import oracle
    oracle.build()
    w = W.BY_NAME[args.workload]
    # size each step's sample so that warm-up + K steps take about args.ref_budget_s
    probe = W.scaled(w, 64)
    xp = W.make_inputs(probe)
    oracle_step(probe, xp)
    t0 = time.perf_counter()
    tok = oracle_step(probe, xp)
    per_tok = (time.perf_counter() - t0) / max(tok, 1)
    per_step_s = args.ref_budget_s / max(1, args.steps + args.warmup)
    tpr = int(min(w.tokens_per_rank, max(8, per_step_s / per_tok / w.ep_size)))
    ws_ = W.scaled(w, tpr)
    xs = W.make_inputs(ws_)
    n_tok = [0]

    def step():
        n_tok[0] = oracle_step(ws_, xs)

    ms = run_timed(step, args.steps, args.warmup, WallTimer(), None)
    value = n_tok[0] * args.steps / (ms / 1e3)
    sample = (f"{ws_.name}: {tpr} tokens/rank ({n_tok[0]} tokens) per step, route + dispatch + "
              f"EPLB + BF16 combine, single thread")
    rec = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name} (bounded samples of {tpr} tokens/rank per step)",
                   "l2": "host run"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "host_cpus": os.cpu_count()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(rec), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--tokens-per-rank", type=int, default=0,
                    help="run the workload with this many tokens per rank (small profiling cases)")
    ap.add_argument("--combine", choices=["bf16", "fp8", "fp8s", "experts", "experts_fp8"],
                    default="bf16",
                    help="combine input: bf16 / fp8 / fp8 with a per-row scale rows per rank, "
                         "or bf16 outputs per (token, slot) reduced with topk_weights inside "
                         "the combine (experts_fp8: and each rank's row quantised to E4M3 "
                         "with one scale before the sum)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--fp8-steps", type=int, default=100)
    ap.add_argument("--workload-steps", type=int, default=30,
                    help="steps per entry of the `workloads` record (every other workload "
                         "and combine input, measured after the headline); 0 = skip")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-all-cores-seconds", type=float, default=10.0,
                    help="also time the oracle on every host core (one process each); 0 = skip")
    ap.add_argument("--ref-budget-s", type=float, default=120.0)
    ap.add_argument("--graph", action="store_true",
                    help="time CUDA-graph replays of the step (small workloads)")
    ap.add_argument("--l2-flush", action="store_true",
                    help="flush L2 before every step and time steps alone (small workloads)")
    ap.add_argument("--variant", choices=["rank-major", "agrs"], default="rank-major",
                    help="agrs: the dense all-gather / reduce-scatter formulation of the same "
                         "step, for comparison")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch")
    ap.add_argument("--opt", action="append", default=[],
                    help="library tuning option NAME=VALUE (ep_a2a_option without the "
                         "EP_A2A_OPT_ prefix, e.g. COMBINE_PIPELINE=2); repeatable")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
