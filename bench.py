#!/usr/bin/env python
"""Benchmark: expert-parallel layout -> dispatch -> combine on B200, one JSON line.

A step is one pass of the whole hot path over one batch: ``ep_layout``,
``ep_dispatch`` and ``ep_combine`` (plus ``ep_reroute`` first for the replica
workload) through the C ABI, on inputs already resident in HBM.  The default
workload is the prefill shape (R=8 emulated ranks, E=256 experts, top-8 with
Zipf(1.2) popularity, T=4096 tokens per rank, hidden 7168): its token rows
(470 MB) and receive slab (120 GB) are far larger than L2, so no flush is
needed between steps.  Smaller workloads (token rows under twice L2) write a
256 MB buffer before every timed step, outside the step's event pair.

Reported:
  value        effective HBM GB/s of the whole step: the algorithmic bytes of
               dispatch + combine (one read of every live token row plus one
               write per live pair, and the mirror image for combine) divided
               by the step time, summed over ranks and divided by the slowest
               rank's time;
  dispatch/combine/layout microseconds per call, from CUDA events recorded on
               the launching stream around every call in the timed region, and
               layout + dispatch end to end (the events before the layout and
               after the dispatch of each step; with --graph, a graph of the two);
  roofline     the dominant kernel's achieved GB/s against the measured copy
               bandwidth of this GPU type (MEASURED_PEAKS.json);
  e2e          the same metric with host buffers: every step copies its inputs
               from pinned host memory and reads the output back; two device
               buffer sets let one step's upload overlap the previous step's
               download and compute;
  clocks       SM clock (median) and clock-event reasons sampled through NVML
               every 5 ms while the timed region runs;
  cpu_baseline the plain single-threaded CPU oracle, pinned to one host core,
               over the same workload once (rank 0, one GPU only), timed per
               stage.

``--impl reference`` times that CPU oracle alone as the reference arm.
Multi-GPU (torchrun): every rank runs an independent replica (the emulated
EP world lives inside one GPU); NCCL only carries the barrier and the max of
the per-rank times.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from combine_get_dispatch_histogram_b200 import inputs  # noqa: E402

METRIC = "dispatch & combine µs/call and effective HBM GB/s (fraction of ~8 TB/s)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = {"dispatch_kernel": "ep_dispatch.cu", "dispatch_vec_kernel": "ep_dispatch.cu",
                  "combine_kernel": "ep_combine.cu", "combine_vec_kernel": "ep_combine.cu"}


def kernel_names(args, k):
    """Names of the dispatch / combine kernels the launch configuration selects."""
    dv = (args.dispatch_cfg or {}).get("variant", 0)
    cv = (args.combine_cfg or {}).get("variant", 0)
    dispatch = "dispatch_vec_kernel" if dv == 2 else "dispatch_kernel"
    combine = "combine_vec_kernel" if (cv == 2 or (cv == 0 and k <= 8)) else "combine_kernel"
    return dispatch, combine


# ----------------------------------------------------------------------------- helpers

def measured_hbm_gbs():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_sha(fname: str) -> str:
    path = os.path.join(ROOT, "combine_get_dispatch_histogram_b200", "csrc", fname)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    if rec.get("source_sha") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    per = rec.get("per_workload", {}).get(workload)
    return None if per is None else int(per)


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs.

    NVML (the library nvidia-smi reads) is polled every 5 ms from a thread, so even a timed
    region of a few tens of milliseconds yields several samples; without NVML it falls back to
    ``nvidia-smi -lms 200``.  The GPU is found by its PCI address, so the sample is of the device
    the timed kernels ran on.  Nothing is ever set: clocks are only read.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits worth reporting (idle, application clocks and sync boost are not)
    REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                   0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    PERIOD_S = 0.005

    def __init__(self, gpu_index: int, device=None):
        self.gpu_index = gpu_index
        self.device = device
        self.proc = None
        self.thread = None
        self.samples = []
        self.max_mhz = None
        self.path = os.path.join("/tmp", f"ep_bench_clocks_{os.getpid()}.csv")

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        if self.device is not None:
            import torch

            pr = torch.cuda.get_device_properties(self.device)
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(
                    f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0")
            except Exception:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu_index)

    def _poll(self, nv, h):
        reasons_of = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), int(reasons_of(h))))
            except Exception:
                pass
            self.stop.wait(self.PERIOD_S)

    def __enter__(self):
        import threading

        try:
            nv, h = self._nvml_handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu_index), "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.thread is not None:
            if not self.samples:
                return None
            seen = 0
            for _, bits in self.samples:
                seen |= bits
            return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(name for bit, name in self.REASON_BITS.items() if seen & bit),
                    "samples": len(self.samples), "source": "nvml, every 5 ms"}
        if self.proc is None:
            return None
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        rows.append(parts)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(float(r[2]) for r in rows),
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi, every 200 ms"}


# ----------------------------------------------------------------------------- rank plumbing

def rank_barrier(world: int, local_rank: int = 0):
    """Barrier over all ranks (no-op on one rank); NCCL needs the rank's device."""
    if world <= 1:
        return
    import torch.distributed as dist

    if dist.get_backend() == "nccl":
        dist.barrier(device_ids=[local_rank])
    else:
        dist.barrier()


def reduce_over_ranks(values, world: int, device, op: str = "max"):
    """Element-wise max (or sum) of a list of floats over all ranks."""
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return t.tolist()


def whole_job_gbs(total_bytes: float, ms: float) -> float:
    """GB/s of bytes moved by all ranks in the slowest rank's time."""
    return total_bytes / (ms * 1e-3) / 1e9


def stats_ms(samples):
    """Median, min and max of per-call times (ms)."""
    return {"median": statistics.median(samples), "min": min(samples), "max": max(samples)}


L2_BYTES = 126 * 1000 * 1000   # B200 L2
L2_FLUSH_BYTES = 256 << 20     # written between timed steps when a step's inputs could stay in L2


def needs_l2_flush(w: inputs.Workload) -> bool:
    """True when the token rows one step reads (x, and the slab rows the combine reads back) are
    less than twice L2: then a step could find the previous step's data still cached."""
    return w.num_ranks * w.num_tokens * w.hidden * 2 < 2 * L2_BYTES


def config_of(w: inputs.Workload, world: int) -> dict:
    """The workload description both arms report (identical dicts for the same run)."""
    R, T, H = w.num_ranks, w.num_tokens, w.hidden
    slab_bytes = w.num_physical * R * T * H * 2
    if needs_l2_flush(w):
        l2 = ("flushed: %d MB written before every timed step and every per-kernel replay, outside "
              "its event pair (x %.0f MB)" % (L2_FLUSH_BYTES >> 20, R * T * H * 2 / 1e6))
    else:
        l2 = "no flush: inputs larger than L2 (x %.0f MB, receive slab %.1f GB)" % (R * T * H * 2 / 1e6,
                                                                                   slab_bytes / 1e9)
    return {"workload": f"{w.name} " + " ".join(f"{k_}={v}" for k_, v in w.describe().items()),
            **w.describe(), "parallelism": f"replicas{world}" if world > 1 else "single-gpu",
            "emulated_ep_ranks": R, "l2": l2}


# ----------------------------------------------------------------------------- our arm

def algorithmic_bytes(H: int, tokens_sent: int, live_pairs: int, tokens_out: int):
    row = 2 * H
    return row * (tokens_sent + live_pairs), row * (live_pairs + tokens_out)


def run_ours(args, rank, world, local_rank, w, inp):
    import torch

    from combine_get_dispatch_histogram_b200 import ep

    ep.load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    R, T, k, H = w.num_ranks, w.num_tokens, w.num_topk, w.hidden
    E = w.num_physical
    cap = R * T
    reroute = w.num_extra > 0

    slab_bytes = E * cap * H * 2
    free, _ = torch.cuda.mem_get_info(dev)
    if free < slab_bytes + (4 << 30):
        raise SystemExit(f"workload {w.name} needs {slab_bytes / 1e9:.1f} GB for the receive slab; "
                         f"{free / 1e9:.1f} GB free")

    # device-resident inputs and preallocated outputs (the library allocates nothing)
    idx_log = torch.from_numpy(inp.topk_idx).to(dev)
    wts = torch.from_numpy(inp.topk_weights).to(dev)
    act = torch.from_numpy(inp.active).to(dev)
    x = torch.from_numpy(inp.x.view(np.int16)).to(dev).view(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    recv_x = torch.empty((E, cap, H), dtype=torch.bfloat16, device=dev)
    src_info = torch.empty((E, cap, 2), dtype=torch.int32, device=dev)
    out = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    lay_ws = torch.zeros(max(16, ep.ep_layout_workspace_bytes(R, T, k, E, H)), dtype=torch.uint8, device=dev)
    rr_ws = rr_out = None
    if reroute:
        rr_ws = torch.empty(max(16, ep.ep_reroute_workspace_bytes(R, T, k, w.num_experts)), dtype=torch.uint8,
                            device=dev)
        rr_out = dict(load=torch.empty(w.num_experts, dtype=torch.int32, device=dev),
                      num_replicas=torch.empty(w.num_experts, dtype=torch.int32, device=dev),
                      phys_base=torch.empty(w.num_experts + 1, dtype=torch.int32, device=dev),
                      topk_idx_phys=torch.empty((R, T, k), dtype=torch.int32, device=dev))
    lay = ep.DispatchLayout(torch.empty((R, E), dtype=torch.int32, device=dev),
                            torch.empty((R, R), dtype=torch.int32, device=dev),
                            torch.empty((R, T, R), dtype=torch.uint8, device=dev),
                            torch.empty((E,), dtype=torch.int32, device=dev),
                            torch.empty((E, R), dtype=torch.int32, device=dev),
                            torch.empty((R, T, k), dtype=torch.int32, device=dev), status)
    stream = torch.cuda.Stream(dev)
    n_ev = 4
    layout_launches = 3 if ep.ep_layout_path(R, T, k, E, H) == ep.EP_LAYOUT_CHUNKED else 1
    launches_per_step = layout_launches + 2 + (1 if reroute else 0)  # layout, dispatch, combine (+ reroute)

    # the step reads its inputs from and writes its result to the current buffer set (the end-to-end
    # leg alternates two sets so that one step's copies overlap the next step's)
    cur = {"b": dict(idx=idx_log, w=wts, act=act, x=x, out=out)}

    def idx_phys():
        return rr_out["topk_idx_phys"] if reroute else cur["b"]["idx"]

    def do_layout():
        b = cur["b"]
        if reroute:
            ep.ep_reroute(b["idx"], w.num_experts, w.num_extra, workspace=rr_ws, out=rr_out, status=status,
                          stream=stream)
        ep.ep_layout(idx_phys(), b["act"], E, hidden=H, workspace=lay_ws, out=lay, status=status, stream=stream)

    def do_dispatch():
        ep.ep_dispatch(cur["b"]["x"], idx_phys(), lay.pair_row, E, recv_x=recv_x, src_info=src_info,
                       status=status, stream=stream, cfg=args.dispatch_cfg)

    def do_combine():
        b = cur["b"]
        ep.ep_combine(recv_x, idx_phys(), b["w"], lay.pair_row, b["act"], out=b["out"], status=status,
                      stream=stream, cfg=args.combine_cfg)

    parts = (do_layout, do_dispatch, do_combine)

    def step(events=None):
        for i, part in enumerate(parts):
            if events is not None:
                events[i].record(stream)
            part()
        if events is not None:
            events[len(parts)].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} after warm-up")
    live_pairs = int(lay.recv_count.sum().item())
    tokens_sent = int(lay.is_token_in_rank.view(R * T, R).amax(dim=1).sum().item())
    tokens_out = R * T
    d_bytes, c_bytes = algorithmic_bytes(H, tokens_sent, live_pairs, tokens_out)

    # ---------------------------------------------------------------- timed region (device resident)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    graphs = None
    if args.graph:
        # one graph for the whole step, one per part (for the per-kernel split), one of layout + dispatch
        graphs = []
        for fns in ([step],) + tuple((p,) for p in parts) + ((do_layout, do_dispatch),):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for fn in fns:
                    fn()
            graphs.append(g)
        torch.cuda.synchronize(dev)
        for g in graphs:
            for _ in range(args.warmup):
                g.replay()
        torch.cuda.synchronize(dev)
    # small steps: a buffer larger than L2 is written before every timed step, outside the step's
    # event pair, and the step time is the sum of the per-step pairs
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if needs_l2_flush(w) else None
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    rank_barrier(world, local_rank)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_index_of(local_rank), dev)
    with sampler, torch.cuda.stream(stream):
        # ~1 ms of GPU sleep ahead of the start event, so the host has queued the first steps when
        # the timed region begins (else the first layout waited on the host: 100-200 us)
        torch.cuda._sleep(2_000_000)
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
                step_ev[i][0].record(stream)
            if graphs is not None:
                graphs[0].replay()
            else:
                step(events[i])
            if flush is not None:
                step_ev[i][1].record(stream)
        t_end.record(stream)
        stream.synchronize()
    torch.cuda.synchronize(dev)
    rank_barrier(world, local_rank)
    total_ms = t_start.elapsed_time(t_end) if flush is None else sum(e0.elapsed_time(e1) for e0, e1 in step_ev)
    if graphs is None:
        per_part = [[e[i].elapsed_time(e[i + 1]) for e in events] for i in range(len(parts))]
        per_part.append([e[0].elapsed_time(e[2]) for e in events])  # layout + dispatch
    else:
        # each part replayed alone as its own graph, one event pair per replay
        per_part = []
        for g in graphs[1:]:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            with torch.cuda.stream(stream):
                for e0, e1 in evs:
                    if flush is not None:
                        flush.zero_()
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
            stream.synchronize()
            per_part.append([e0.elapsed_time(e1) for e0, e1 in evs])
    part_stats = [stats_ms(v) for v in per_part]  # layout, dispatch, combine, layout + dispatch
    lay_ms, dis_ms, com_ms = (st["median"] for st in part_stats[:3])
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} after the timed steps")

    # ---------------------------------------------------------------- e2e: host buffers
    # Every step copies its inputs from pinned host memory and its result back.  Two device buffer
    # sets alternate: step i's inputs go up on one copy stream while step i-1 computes and step i-2's
    # result comes down on another (PCIe carries both directions at once).  A set is refilled only
    # after the step that read it has finished, and its result buffer only after it has been read out.
    e2e = None
    if args.e2e_steps > 0:
        h_idx = torch.from_numpy(inp.topk_idx).pin_memory()
        h_w = torch.from_numpy(inp.topk_weights).pin_memory()
        h_act = torch.from_numpy(inp.active).pin_memory()
        h_x = torch.from_numpy(inp.x.view(np.int16)).pin_memory()
        h_out = [torch.empty((R, T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
        h2d = h_idx.numel() * 4 + h_w.numel() * 4 + h_act.numel() + h_x.numel() * 2
        d2h = h_out[0].numel() * 2
        sets = [cur["b"], dict(idx=torch.empty_like(idx_log), w=torch.empty_like(wts), act=torch.empty_like(act),
                               x=torch.empty_like(x), out=torch.empty_like(out))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        n = args.e2e_steps
        rank_barrier(world, local_rank)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(n):
            b = i % 2
            B = sets[b]
            if i >= 2:
                s_in.wait_event(ev_done[b])      # step i-2 has finished reading this set
            with torch.cuda.stream(s_in):
                B["idx"].copy_(h_idx, non_blocking=True)
                B["w"].copy_(h_w, non_blocking=True)
                B["act"].copy_(h_act, non_blocking=True)
                B["x"].view(torch.int16).copy_(h_x, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])     # step i-2's result has been read out of this set
            cur["b"] = B
            with torch.cuda.stream(stream):
                step()
                ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                h_out[b].copy_(B["out"].view(torch.int16), non_blocking=True)
                ev_out[b].record(s_out)
        for b in range(min(2, n)):
            stream.wait_event(ev_out[b])
        e1.record(stream)
        stream.synchronize()
        cur["b"] = sets[0]
        rank_barrier(world, local_rank)
        e2e_ms = e0.elapsed_time(e1) / n
        e2e = dict(ms=e2e_ms, h2d=h2d, d2h=d2h)
        assert np.array_equal(h_out[(n - 1) % 2].numpy(), out.view(torch.int16).cpu().numpy())

    # ---------------------------------------------------------------- dispatch ceilings (after the timed region)
    # The paced dispatch kernel with its row loads left out: mode 0 times the scatter's stores alone,
    # mode 1 the stores plus the paced prefetch of the rows -- the dispatch's own HBM traffic with no
    # store waiting for a read.  Each is timed like the steps: warm-up, then one event pair per call.
    ceil_ms = []
    for mode in (0, 1):
        def ceiling_call():
            ep.ep_diag_dispatch_ceiling(cur["b"]["x"], idx_phys(), lay.pair_row, E, mode, recv_x=recv_x,
                                        src_info=src_info, status=status, stream=stream)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                ceiling_call()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for e0, e1 in evs:
                e0.record(stream)
                ceiling_call()
                e1.record(stream)
        stream.synchronize()
        ceil_ms.append(statistics.median(e0.elapsed_time(e1) for e0, e1 in evs))
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} after the ceiling calls")

    # ---------------------------------------------------------------- reduce over ranks
    flat = [v for st in part_stats for v in (st["median"], st["min"], st["max"])]
    total_ms, e2e_ms, c0_ms, c1_ms, *flat = reduce_over_ranks(
        [total_ms, e2e["ms"] if e2e else 0.0] + ceil_ms + flat, world, dev, "max")
    part_stats = [dict(median=flat[3 * i], min=flat[3 * i + 1], max=flat[3 * i + 2]) for i in range(len(flat) // 3)]
    lay_ms, dis_ms, com_ms = (st["median"] for st in part_stats[:3])
    ms_per_step = total_ms / args.steps
    step_bytes = d_bytes + c_bytes
    (job_bytes,) = reduce_over_ranks([step_bytes], world, dev, "sum")
    value = whole_job_gbs(job_bytes, ms_per_step)
    dis_gbs = d_bytes / (dis_ms * 1e-3) / 1e9
    com_gbs = c_bytes / (com_ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_gbs()
    d_name, c_name = kernel_names(args, k)
    dispatch_path = ep.ep_dispatch_path(R, T, k, E, H, cfg=args.dispatch_cfg)
    dom = (d_name, d_bytes, dis_ms) if dis_ms >= com_ms else (c_name, c_bytes, com_ms)
    achieved = dom[1] / (dom[2] * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(w, world),
        "dispatch_us": round(dis_ms * 1e3, 2),
        "combine_us": round(com_ms * 1e3, 2),
        "layout_us": round(lay_ms * 1e3, 2),
        "kernel_us": {name: {k_: round(v * 1e3, 2) for k_, v in st.items()}
                      for name, st in zip(("layout", "dispatch", "combine"), part_stats)},
        "kernel_us_stat": "median over the timed steps (min, max beside it); max over ranks",
        "layout_dispatch_us": {k_: round(v * 1e3, 2) for k_, v in part_stats[3].items()},
        "dispatch_gbs": round(dis_gbs, 1),
        "combine_gbs": round(com_gbs, 1),
        "dispatch_frac_of_8tbs": round(dis_gbs / NOMINAL_HBM_GBS, 4),
        "combine_frac_of_8tbs": round(com_gbs / NOMINAL_HBM_GBS, 4),
        "bytes_per_direction": d_bytes,
        "roofline": {"bound": "hbm", "kernel": dom[0], "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(dom[0], w.name),
                     "algorithmic_bytes": dom[1]},
        "gpu_launches": launches_per_step * args.steps,
        "dispatch_path": {ep.EP_VARIANT_BULK: "bulk", ep.EP_VARIANT_PACED: "paced",
                          ep.EP_VARIANT_VECTOR: "vector"}.get(dispatch_path, str(dispatch_path)),
        "dispatch_ceiling": {
            "what": "the paced dispatch kernel without its row loads (ep_diag_dispatch_ceiling), timed after the "
                    "steps: stores alone, and stores plus the paced L2 prefetch of the rows (the dispatch's HBM "
                    "traffic with no store waiting on a read); compared with the dispatch only when the dispatch "
                    "itself took the paced path",
            "stores_only_us": round(c0_ms * 1e3, 2),
            "stores_and_row_reads_us": round(c1_ms * 1e3, 2),
            "dispatch_over_stores_and_reads": (round(dis_ms / c1_ms, 4) if dispatch_path == ep.EP_VARIANT_PACED
                                               else None),
        },
    }
    if args.graph:
        line["graph"] = True
    if args.dispatch_cfg or args.combine_cfg:
        line["launch_cfg"] = {"dispatch": args.dispatch_cfg, "combine": args.combine_cfg}
    if e2e is not None:
        line["e2e"] = {"value": round(whole_job_gbs(job_bytes, e2e_ms), 1), "unit": "GB/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e_ms, 3)}
    clk = sampler.summary()
    if clk is not None:
        line["clocks"] = clk
    return line


def gpu_index_of(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[local_rank])
        except Exception:
            pass
    return local_rank


# ----------------------------------------------------------------------------- CPU oracle arm

class one_core:
    """Pin the calling thread to one host core for the duration (restores the old set after)."""

    def __enter__(self):
        self.old = None
        self.core = None
        try:
            self.old = os.sched_getaffinity(0)
            self.core = min(self.old)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            self.old = None
        return self

    def __exit__(self, *exc):
        if self.old is not None:
            os.sched_setaffinity(0, self.old)


def oracle_sample(w: inputs.Workload, sample_tokens=None, inp=None):
    """Time the CPU oracle, pinned to one core, stage by stage.

    ``sample_tokens`` None (the default) runs the whole workload once; a number
    runs the first that many tokens of every rank.
    """
    import oracle

    inp = inp if inp is not None else inputs.make_inputs(w)
    Ts = w.num_tokens if sample_tokens is None else min(int(sample_tokens), w.num_tokens)
    idx = np.ascontiguousarray(inp.topk_idx[:, :Ts])
    x = np.ascontiguousarray(inp.x[:, :Ts])
    wts = np.ascontiguousarray(inp.topk_weights[:, :Ts])
    E, H, R = w.num_physical, w.hidden, w.num_ranks
    oracle.load()
    stages = {}
    with one_core() as pin:
        t0 = time.perf_counter()
        if w.num_extra:
            idx = oracle.reroute(idx, w.num_experts, w.num_extra)["topk_idx_phys"]
            stages["reroute"] = time.perf_counter() - t0
        t1 = time.perf_counter()
        ref = oracle.layout(idx, inp.active, E)
        t2 = time.perf_counter()
        packed, _ = oracle.dispatch(x, idx, ref)
        t3 = time.perf_counter()
        oracle.combine(packed, ref.list_base[:-1], idx, wts, ref.pair_row, inp.active, E)
        t4 = time.perf_counter()
    del packed
    stages.update(layout=t2 - t1, dispatch=t3 - t2, combine=t4 - t3)
    secs = t4 - t0
    live = int(ref.recv_count.sum())
    sent = int(ref.is_token_in_rank.reshape(R * Ts, R).max(axis=1).sum())
    d_b, c_b = algorithmic_bytes(H, sent, live, R * Ts)
    what = ("the whole workload" if Ts == w.num_tokens else f"first {Ts} of {w.num_tokens} tokens of each rank")
    return dict(value=round((d_b + c_b) / secs / 1e9, 3), unit="GB/s", cores=1, kind="oracle",
                sample=f"{what}: {R} ranks x {Ts} tokens (reroute + layout + dispatch + combine, "
                       f"single-threaded C, float64 combine, one pass)",
                pinned_core=pin.core, seconds=round(secs, 3),
                stage_seconds={k_: round(v, 4) for k_, v in stages.items()})


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def run_reference(args, world):
    w = inputs.named(args.workload)
    inp = inputs.make_inputs(w)
    samples = []
    for _ in range(args.warmup):
        oracle_sample(w, args.cpu_sample_tokens, inp)
    for _ in range(args.steps):
        samples.append(oracle_sample(w, args.cpu_sample_tokens, inp))
    secs = sum(s["seconds"] for s in samples) / len(samples)
    value = round(statistics.median(s["value"] for s in samples), 4)
    base = dict(samples[0])
    base["value"] = value
    base["seconds"] = round(secs, 3)
    base["stage_seconds"] = {k_: round(statistics.median(s_["stage_seconds"][k_] for s_ in samples), 4)
                             for k_ in samples[0]["stage_seconds"]}
    base["host_cores"] = os.cpu_count()
    base["cpu_model"] = cpu_model()
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main

def parse_cfg(text: str) -> dict:
    cfg = {}
    for part in filter(None, text.split(",")):
        key, val = part.split("=")
        if key not in ("max_ctas", "threads", "stages", "variant"):
            raise argparse.ArgumentTypeError(f"unknown launch-config key {key}")
        cfg[key] = int(val)
    return cfg


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill",
                    help="prefill | decode | replica | tiny | sweep_T<n>[_mask5] | prefill_T<n> | replica_T<n> | "
                         "small_slab | paced_slab")
    ap.add_argument("--e2e-steps", type=int, default=30,
                    help="steps of the host-buffer pipeline (its fill and drain are spread over them)")
    ap.add_argument("--graph", action="store_true",
                    help="replay the step as a CUDA graph (per-kernel split from per-kernel graphs)")
    ap.add_argument("--cpu-sample-tokens", type=int, default=None,
                    help="tokens per rank in the CPU oracle's timed pass (default: the whole workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dispatch-cfg", type=parse_cfg, default=None,
                    help="launch config of ep_dispatch, e.g. max_ctas=296,stages=7")
    ap.add_argument("--combine-cfg", type=parse_cfg, default=None,
                    help="launch config of ep_combine, e.g. stages=8,threads=256")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    try:
        w = inputs.named(args.workload)
        inp = inputs.make_inputs(w)
        line = run_ours(args, rank, world, local_rank, w, inp)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cb = oracle_sample(w, args.cpu_sample_tokens, inp)
            cb["host_cores"] = os.cpu_count()
            cb["cpu_model"] = cpu_model()
            line["cpu_baseline"] = cb
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
