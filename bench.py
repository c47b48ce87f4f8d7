#!/usr/bin/env python
"""Paged decode attention benchmark (KV-read GB/s, % of HBM peak, seqs/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2|all|1..5]
                    [--impl ours|reference]

One step = one pa_decode call over the whole batch of the workload (every
page of every sequence read once, the split-KV combine included when the
planner splits).  Default workload: the Llama-style MHA decode batch
(64 sequences x 4096 tokens, 32/32 heads, head size 128, bf16, 4 GiB of K/V
per step: larger than L2, so no flush is needed between steps; smaller
workloads flush L2 by writing a 256 MiB buffer between timed steps).

On one GPU, with one workload asked for (the default), the line also
carries `per_config`: for each of the five workloads, its own timed region of
at least 0.3 s, with GB/s, % of the 8 TB/s spec and of the measured copy
rate, the roofline fraction and DRAM traffic, the plan, and the SM clock
sampled every 5 ms (at least 12 samples).

With N > 1 (torchrun), every rank runs its own batch of the same workload
(weak scaling, no collective on the data path); the time is the max over ranks.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on this host's cores (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak) and seqs/s at 1 GPU"
UNIT = "GB/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_NAME = "pa_decode_kernel"
DATA = "synthetic (seeded N(0,1) K/V/Q, seeded random block tables)"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


# --------------------------------------------------------------------------- helpers
def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
            return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The device code of the default decode path: pa_decode_kernel, pa_combine_kernel
# and the page body they share.  (The dynamic schedule's kernel lives in its own
# header and does not change what these kernels read or write.)
KERNEL_SOURCES = ("pa_decode_kernels.cuh", "pa_ptx.cuh")


def kernel_source_hash() -> str:
    """Hash of the default path's device code: its kernel headers with
    comments and whitespace removed (host-side ABI code does not change what
    the kernels read or write, and neither do comments)."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_471_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        text = " ".join(text.split())
        h.update(name.encode())
        h.update(text.encode())
    return h.hexdigest()[:16]


def traffic_per_launch(config_idx: int):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except Exception:
        return None
    if t.get("source_hash") != kernel_source_hash():
        return None
    ent = t.get("configs", {}).get(str(config_idx))
    return None if ent is None else float(ent["dram_bytes_per_launch"])


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, device, period_s: float = 0.02):
        self.device, self.period = device, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def _handle(self, nv):
        """NVML handle of the CUDA device (NVML ignores CUDA_VISIBLE_DEVICES)."""
        import torch
        props = torch.cuda.get_device_properties(self.device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        try:
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def _run(self):
        nv = self._nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for k, bit in names.items():
                    if r & bit and k != "gpu_idle":
                        self.reasons.add(k)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join(timeout=1.0)

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- GPU arm
def bytes_of(wl):
    """Algorithmic bytes of one step: K+V of every token read once, plus Q and
    out.  With a shared prefix the K/V of shared blocks count once (unique
    bytes), the conservative figure; the logical count is reported beside it."""
    kv = wl.unique_kv_bytes if wl.cfg.shared_prefix_blocks else wl.kv_bytes
    return kv + wl.q_out_bytes


def workload_config(idx: int, num_seqs: int = 0):
    """The named workload, or the same shape with fewer sequences and a pool
    sized to them (used for small profiler captures)."""
    from paged_kv_cache_471_b200 import workloads as W
    if num_seqs and num_seqs < W.WORKLOADS[idx].num_seqs:
        return W.reduced(idx, num_seqs=num_seqs)
    return W.WORKLOADS[idx]


def time_gpu(idx: int, steps: int, warmup: int, device, want_e2e=True, rank=0, num_seqs=0,
             cascade=True, alibi=False, schedule="auto", min_region_ms=0.0,
             min_clock_samples=12, extras=True, mha_cuda_cores=False, fp8_compute=False,
             partition_pages=0, stages=0):
    import torch

    import paged_kv_cache_471_b200 as pa
    from paged_kv_cache_471_b200 import workloads as W

    cfg = workload_config(idx, num_seqs)
    wl = W.make_workload(cfg, device)
    out = torch.empty_like(wl.query)
    # A workload whose sequences share a prompt prefix declares it, so the
    # prefix pages are streamed once per group of query rows (cascade decode).
    prefix = cfg.shared_prefix_blocks if (cascade and not alibi) else 0
    slopes = None
    if alibi:  # geometric ALiBi slopes 2^(-8 i / H)
        slopes = torch.tensor([2.0 ** (-8.0 * (i + 1) / cfg.num_heads)
                               for i in range(cfg.num_heads)], dtype=torch.float32, device=device)
    if prefix and schedule == "balanced":
        schedule = "auto"  # balanced ranges do not take a shared prefix
    fp8_compute = fp8_compute and cfg.kv_dtype == W.FP8_E4M3
    plan = pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size, cfg.block_size,
                   cfg.max_seq_len, cfg.kv_dtype, shared_prefix_blocks=prefix, schedule=schedule,
                   fp8_compute=fp8_compute, partition_pages=partition_pages, stages=stages)
    ws = torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    alg_bytes = bytes_of(wl)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = alg_bytes < 4 * l2
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device) if flush else None

    def step():
        pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale,
                  wl.block_tables, wl.seq_lens, cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
                  wl.k_scale, wl.v_scale, workspace_tensor=ws, stream=stream,
                  shared_prefix_blocks=prefix, alibi_slopes=slopes, schedule=schedule,
                  mha_cuda_cores=mha_cuda_cores, fp8_compute=fp8_compute,
                  partition_pages=partition_pages, stages=stages)

    for _ in range(max(warmup, 3)):
        if flush:
            scratch.fill_(1)
        step()
    torch.cuda.synchronize(device)
    # Estimated time of one call (warm), to size a timed region of at least
    # min_region_ms and the extra calls that keep the clock sampler busy.
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        if flush:
            scratch.fill_(1)
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    est_ms = max(e0.elapsed_time(e1) / 3, 1e-3)
    if min_region_ms > 0:
        steps = max(steps, int(math.ceil(min_region_ms / est_ms)))

    # Per-launch device time: events bracket only the pa_decode call.  Large
    # workloads are timed as `steps` bare back-to-back calls (an event between
    # calls would keep each launch from overlapping the previous call's end),
    # and their per-launch statistics come from a second pass of the same
    # calls; small workloads need the per-launch events in the timed region to
    # leave the L2 flushes out of the step time.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]

    def per_launch_pass():
        for i in range(steps):
            if flush:
                scratch.fill_(1)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    # Clocks are sampled every 5 ms through the timed region and the
    # per-launch pass after it; when those are too short for
    # min_clock_samples samples, the same calls keep running, untimed, until
    # there are enough.
    extra_calls = 0
    with ClockSampler(device, period_s=0.005) as clk:
        t_start.record(stream)
        if flush:
            per_launch_pass()
        else:
            for _ in range(steps):
                step()
        t_end.record(stream)
        torch.cuda.synchronize(device)
        region_samples = len(clk.samples)
        barrier(device)
        if not flush:
            per_launch_pass()
            torch.cuda.synchronize(device)
        chunk = max(1, int(20.0 / est_ms))
        while clk.ok and len(clk.samples) < min_clock_samples and extra_calls < 200000:
            for _ in range(chunk):
                step()
            torch.cuda.synchronize(device)
            extra_calls += chunk
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    region_ms = t_start.elapsed_time(t_end)
    # With flushes in the timed region, the step time is the per-call event
    # time, which leaves them out.
    step_ms = sum(kern_ms) / steps if flush else region_ms / steps
    local_step_ms = step_ms
    status = pa.read_status(ws)

    extra = {}
    if flush and extras:
        # Small workloads: also the time per call of back-to-back calls with a
        # warm L2 (bound by the host's launch rate for tiny batches) and of 100
        # calls replayed from one CUDA graph (no launch overhead), labelled as
        # such; the headline value above stays cold-L2 per call.
        torch.cuda.synchronize(device)
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record(stream)
        for _ in range(steps):
            step()
        w1.record(stream)
        torch.cuda.synchronize(device)
        extra["warm_l2_back_to_back_ms_per_call"] = round(w0.elapsed_time(w1) / steps, 5)
        gs = torch.cuda.Stream(device)
        gs.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gs):
            step_on = lambda st: pa.decode(out, wl.query, wl.key_cache, wl.value_cache,
                                           cfg.num_kv_heads, cfg.scale, wl.block_tables,
                                           wl.seq_lens, cfg.block_size, cfg.max_seq_len,
                                           cfg.kv_dtype, wl.k_scale, wl.v_scale,
                                           workspace_tensor=ws, stream=st, schedule=schedule,
                                           mha_cuda_cores=mha_cuda_cores, fp8_compute=fp8_compute,
                  partition_pages=partition_pages, stages=stages)
            step_on(gs)  # warm on the capture stream
            gs.synchronize()
            with torch.cuda.graph(graph, stream=gs):
                for _ in range(100):
                    step_on(gs)
        stream.wait_stream(gs)
        graph.replay()
        torch.cuda.synchronize(device)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(5):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize(device)
        extra["graph_of_100_ms_per_call"] = round(g0.elapsed_time(g1) / 500, 5)
        del graph

    clocks = clk.summary()
    clocks["samples_in_timed_region"] = region_samples
    clocks["sampled_over"] = ("the timed region and the per-launch pass"
                              + (f", then {extra_calls} more of the same calls" if extra_calls
                                 else ""))
    res = dict(cfg=cfg, wl=wl, plan=plan, alg_bytes=alg_bytes, kern_ms=kern_ms,
               region_ms=region_ms, step_ms=step_ms, local_step_ms=local_step_ms, flush=flush,
               steps=steps, clocks=clocks, status=status,
               launches_per_step=1 + plan["combine"],
               shared_prefix_blocks=prefix, alibi=alibi, extra=extra,
               options={"schedule": schedule, "mha_cuda_cores": bool(mha_cuda_cores),
                        "fp8_compute": bool(fp8_compute), "partition_pages": partition_pages,
                        "stages": stages})

    if want_e2e:
        # End to end through the public call, as a serving loop runs it: every
        # step uploads its own inputs (queries, block tables, sequence lengths)
        # from pinned host memory, decodes against the resident KV cache and
        # downloads its output to pinned host memory.  Uploads and downloads run
        # on their own streams with two buffer sets, so step i+1's upload and
        # step i-1's download overlap step i's decode; each decode waits for its
        # own upload, and the timed region ends when the last download landed.
        q_h = wl.query.cpu().pin_memory()
        bt_h = wl.block_tables.cpu().pin_memory()
        sl_h = wl.seq_lens.cpu().pin_memory()
        nb = 2
        out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(nb)]
        q_d = [torch.empty_like(wl.query) for _ in range(nb)]
        bt_d = [torch.empty_like(wl.block_tables) for _ in range(nb)]
        sl_d = [torch.empty_like(wl.seq_lens) for _ in range(nb)]
        out_d = [torch.empty_like(out) for _ in range(nb)]
        up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_used = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]

        def run_e2e(n):
            for i in range(n):
                b = i % nb
                with torch.cuda.stream(up):
                    if i >= nb:
                        up.wait_event(ev_used[b])
                    q_d[b].copy_(q_h, non_blocking=True)
                    bt_d[b].copy_(bt_h, non_blocking=True)
                    sl_d[b].copy_(sl_h, non_blocking=True)
                    ev_in[b].record(up)
                stream.wait_event(ev_in[b])
                if i >= nb:
                    stream.wait_event(ev_out[b])
                pa.decode(out_d[b], q_d[b], wl.key_cache, wl.value_cache, cfg.num_kv_heads,
                          cfg.scale, bt_d[b], sl_d[b], cfg.block_size, cfg.max_seq_len,
                          cfg.kv_dtype, wl.k_scale, wl.v_scale, workspace_tensor=ws,
                          stream=stream, shared_prefix_blocks=prefix, alibi_slopes=slopes,
                          schedule=schedule, mha_cuda_cores=mha_cuda_cores, fp8_compute=fp8_compute,
                  partition_pages=partition_pages, stages=stages)
                ev_used[b].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(ev_used[b])
                    out_h[b].copy_(out_d[b], non_blocking=True)
                    ev_out[b].record(down)

        run_e2e(4)
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(up)
        run_e2e(steps)
        e1.record(down)
        torch.cuda.synchronize(device)
        barrier(device)
        assert torch.equal(out_h[(steps - 1) % nb], out.cpu()), "e2e output differs"
        # Small workloads run this loop with a warm L2, as a serving loop
        # repeating a small batch would (no flush between steps).
        e2e_ms = e0.elapsed_time(e1) / steps
        h2d = (q_h.numel() * q_h.element_size() + bt_h.numel() * bt_h.element_size()
               + sl_h.numel() * sl_h.element_size())
        d2h = out_h[0].numel() * out_h[0].element_size()
        res.update(e2e_ms=e2e_ms, h2d=h2d, d2h=d2h)
    return res


# --------------------------------------------------------------------------- CPU arm
def cpu_sample(idx: int, wl, budget_s: float = 12.0, max_seqs=None):
    """Time the fp64 oracle on whole sequences of the workload (all heads),
    growing the sample until it takes about budget_s.  Returns GB/s over the
    sample's algorithmic bytes, the sample description and thread count."""
    import torch

    import oracle
    from paged_kv_cache_471_b200 import workloads as W

    cfg = wl.cfg
    threads = len(os.sched_getaffinity(0))
    kv = oracle.KV_E4M3 if cfg.kv_dtype == W.FP8_E4M3 else oracle.KV_BF16
    elem = cfg.elem_bytes

    def host_inputs(seqs):
        bt = wl.block_tables[seqs].cpu()
        ids = bt[bt >= 0].unique()
        remap = torch.full((cfg.num_blocks,), -1, dtype=torch.int64)
        remap[ids] = torch.arange(ids.numel())
        btn = torch.where(bt >= 0, remap[bt.clamp(min=0).long()], torch.tensor(-1)).to(torch.int32)
        idd = ids.to(wl.key_cache.device)
        return (wl.query[seqs].cpu(), wl.key_cache[idd].cpu(), wl.value_cache[idd].cpu(), btn,
                wl.seq_lens[seqs].cpu())

    def run(seqs):
        q, kc, vc, bt, sl = host_inputs(seqs)
        t0 = time.perf_counter()
        oracle.pa_decode(q, kc, vc, cfg.num_kv_heads, cfg.scale, bt, sl, cfg.block_size, kv,
                         cfg.k_scale, cfg.v_scale, threads=threads)
        dt = time.perf_counter() - t0
        tok = int(sl.clamp(min=0).sum())
        nbytes = 2 * tok * cfg.num_kv_heads * cfg.head_size * elem + \
            2 * len(seqs) * cfg.num_heads * cfg.head_size * 2
        return dt, nbytes

    limit = max_seqs or cfg.num_seqs
    n = 1
    dt, nb = run(list(range(n)))
    if dt < budget_s and n < limit:
        n = min(limit, max(1, int(n * budget_s / max(dt, 1e-3))))
        dt, nb = run(list(range(n)))
    reps = 1
    while dt < budget_s and reps < 64:  # the whole batch is quick: repeat it
        d2, _ = run(list(range(n)))
        dt += d2
        reps += 1
    return dict(gbs=nb * reps / dt / 1e9, seconds=dt, seqs=n, threads=threads, bytes=nb * reps,
                reps=reps)


# --------------------------------------------------------------------------- main
def workload_config_dict(idx, cfg, wl, alg_bytes, n_gpus):
    """The line's `config`: what the workload is (the same for both arms)."""
    return {
        "workload": cfg.name,
        "config_index": idx,
        "num_seqs": cfg.num_seqs, "num_heads": cfg.num_heads,
        "num_kv_heads": cfg.num_kv_heads, "head_size": cfg.head_size,
        "block_size": cfg.block_size, "num_blocks": cfg.num_blocks,
        "kv_dtype": cfg.kv_dtype,
        "shared_prefix_blocks": cfg.shared_prefix_blocks,
        "sum_seq_lens": int(wl.seq_lens.sum()),
        "bytes_per_step": alg_bytes,
        "logical_bytes_per_step": wl.kv_bytes + wl.q_out_bytes,
        "parallelism": f"weak x{n_gpus} (independent batches per GPU)" if n_gpus > 1
        else "1 GPU",
    }


def result_line(idx, r, n_gpus, steps, warmup, cpu=None):
    cfg = r["cfg"]
    peak, peak_kind = measured_hbm_peak()
    gbs = r["alg_bytes"] / (r["step_ms"] * 1e-3) / 1e9
    kern_avg = sum(r["kern_ms"]) / len(r["kern_ms"])
    # This rank's own device time per step over the timed region (each step is
    # the decode launch, plus the combine when the plan splits).
    achieved = r["alg_bytes"] / (r["local_step_ms"] * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(gbs * n_gpus, 2),
        "unit": UNIT,
        "n_gpus": n_gpus,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(r["step_ms"], 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8_e4m3 KV, f16 MMA, fp32 softmax" if cfg.kv_dtype == "fp8_e4m3"
        else "bf16",
        "data": DATA,
        "config": workload_config_dict(idx, cfg, r["wl"], r["alg_bytes"], n_gpus),
        "seqs_per_s": round(cfg.num_seqs * n_gpus / (r["step_ms"] * 1e-3), 1),
        "pct_of_8TBs_spec": round(100 * gbs / SPEC_HBM_GBS, 2),
        f"pct_of_{peak_kind}_hbm": round(100 * gbs / peak, 2),
        "l2": ("flushed between steps (256 MiB write, excluded from step time)"
               if r["flush"] else "inputs larger than L2, no flush"),
        "plan": r["plan"],
        "shared_prefix_blocks_declared": r["shared_prefix_blocks"],
        "alibi": r["alibi"],
        "options": r["options"],
        **({"small_workload": {
            **r["extra"],
            "warm_l2_back_to_back_gbs": round(r["alg_bytes"] / (r["extra"]["warm_l2_back_to_back_ms_per_call"] * 1e-3) / 1e9, 2),
            "graph_of_100_gbs": round(r["alg_bytes"] / (r["extra"]["graph_of_100_ms_per_call"] * 1e-3) / 1e9, 2)}}
           if r["extra"] else {}),
        "roofline": {
            "bound": "hbm",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic_per_launch(idx),
            "kernel": KERNEL_NAME + (" + pa_combine_kernel" if r["launches_per_step"] > 1 else ""),
            "bytes_per_launch": r["alg_bytes"],
            "launch_ms": {"mean": round(kern_avg, 5),
                          "median": round(statistics.median(r["kern_ms"]), 5),
                          "min": round(min(r["kern_ms"]), 5),
                          "how": ("events around each call in the timed region" if r["flush"]
                                  else "events around each call, in a second pass after the "
                                       "timed region of back-to-back calls")},
        },
        "gpu_launches": steps * r["launches_per_step"],
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    if "e2e_ms" in r:
        line["e2e"] = {"value": round(r["alg_bytes"] / (r["e2e_ms"] * 1e-3) / 1e9 * n_gpus, 2),
                       "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                       "d2h_bytes_per_step": r["d2h"], "ms_per_step": round(r["e2e_ms"], 5),
                       "note": "per step: pinned H2D of its queries/block tables/seq_lens, decode "
                               "over the resident KV cache, D2H of its out; uploads and "
                               "downloads pipelined on two copy streams with two buffer sets"
                               + ("; L2 warm (no flush between steps)" if r["flush"] else "")}
    if cpu is not None:
        line["cpu_baseline"] = {
            "value": round(cpu["gbs"], 4), "unit": UNIT, "cores": cpu["threads"],
            "kind": "oracle",
            "sample": f"{cpu['seqs']} of {cfg.num_seqs} sequences (all heads) x {cpu['reps']} "
                      f"repetitions, {cpu['seconds']:.1f} s, fp64 C + OpenMP"}
    return line


def config_entry(idx, r):
    """One workload's figures for the per_config object of the default line:
    the same quantities as the line's own, for a timed region of at least
    0.3 s (so that the clock sampler sees it many times)."""
    cfg = r["cfg"]
    peak, peak_kind = measured_hbm_peak()
    gbs = r["alg_bytes"] / (r["step_ms"] * 1e-3) / 1e9
    ent = {
        "workload": cfg.name,
        "steps": r["steps"],
        "ms_per_step": round(r["step_ms"], 5),
        "gbs": round(gbs, 2),
        "pct_of_8TBs_spec": round(100 * gbs / SPEC_HBM_GBS, 2),
        f"pct_of_{peak_kind}_hbm": round(100 * gbs / peak, 2),
        "seqs_per_s": round(cfg.num_seqs / (r["step_ms"] * 1e-3), 1),
        "bytes_per_step": r["alg_bytes"],
        "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(gbs / peak, 4),
                     "traffic": traffic_per_launch(idx)},
        "launch_ms": {"mean": round(sum(r["kern_ms"]) / len(r["kern_ms"]), 5),
                      "median": round(statistics.median(r["kern_ms"]), 5),
                      "min": round(min(r["kern_ms"]), 5)},
        "plan": r["plan"],
        "shared_prefix_blocks_declared": r["shared_prefix_blocks"],
        "l2": ("flushed between steps (256 MiB write, excluded from step time)"
               if r["flush"] else "inputs larger than L2, no flush"),
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    if cfg.shared_prefix_blocks:
        logical = r["wl"].kv_bytes + r["wl"].q_out_bytes
        ent["bytes_counted"] = "unique (shared prefix blocks once)"
        ent["logical_bytes_per_step"] = logical
        ent["logical_gbs"] = round(logical / (r["step_ms"] * 1e-3) / 1e9, 2)
    for k, v in r["extra"].items():
        ent[k] = v
    return ent


def run_copy_blocks(args, device):
    """Bandwidth of pa_copy_blocks (copy on write of whole blocks) on the
    Llama-style MHA block geometry: 4096 random (src, dst) pairs per call,
    256 KiB of K+V per pair, so each call reads and writes 1 GiB."""
    import torch

    import paged_kv_cache_471_b200 as pa
    from paged_kv_cache_471_b200 import workloads as W
    cfg = W.WORKLOADS[2]
    kc = torch.empty(cfg.key_cache_shape(), dtype=torch.bfloat16, device=device)
    vc = torch.empty(cfg.value_cache_shape(), dtype=torch.bfloat16, device=device)
    kc.view(torch.int16).fill_(1)
    vc.view(torch.int16).fill_(2)
    n = 4096
    g = torch.Generator().manual_seed(17)
    perm = torch.randperm(cfg.num_blocks, generator=g)
    src, dst = perm[:n].to(device), perm[n:2 * n].to(device)
    moved = 2 * 2 * n * cfg.page_bytes() * cfg.num_kv_heads  # (K+V) x (read+write)
    for _ in range(args.warmup):
        pa.copy_blocks(kc, vc, src, dst)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        pa.copy_blocks(kc, vc, src, dst)
    b.record()
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / args.steps
    peak, kind = measured_hbm_peak()
    gbs = moved / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "block copy (copy on write) GB/s, read+write", "value": round(gbs, 2),
                      "unit": "GB/s", "ms_per_step": round(ms, 5), "steps": args.steps,
                      "config": {"workload": f"{n} random block pairs, {cfg.num_kv_heads} kv heads "
                                             f"x 128 x 16 bf16 (K+V 256 KiB per pair)",
                                 "bytes_per_step": moved},
                      "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak,
                                   "peak_kind": kind, "unit": "GB/s",
                                   "frac": round(gbs / peak, 4)}}), flush=True)


def run_reference(args):
    """The oracle as the reference arm: each step one bounded sample."""
    import torch
    ws, rank, local = dist_env()
    if rank != 0:
        return 0
    from paged_kv_cache_471_b200 import workloads as W
    idx = int(args.config) if args.config not in ("all",) else 2
    cfg = W.WORKLOADS[idx]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    wl = W.make_workload(cfg, dev) if dev.type == "cuda" else W.make_workload(
        W.reduced(idx, num_seqs=2), dev)
    per = []
    for i in range(args.warmup + args.steps):
        r = cpu_sample(idx, wl, budget_s=args.ref_budget / max(args.steps, 1), max_seqs=2)
        if i >= args.warmup:
            per.append(r)
    gbs = sum(r["bytes"] for r in per) / sum(r["seconds"] for r in per) / 1e9
    ms = 1e3 * sum(r["seconds"] for r in per) / len(per)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": DATA,
        "config": workload_config_dict(idx, cfg, wl, bytes_of(wl), args.gpus),
        "cpu_baseline": {"value": round(gbs, 4), "unit": UNIT, "cores": per[0]["threads"],
                         "kind": "oracle",
                         "sample": f"per step {per[0]['seqs']} sequence(s) of {cfg.num_seqs}, "
                                   "all heads, fp64 C + OpenMP"},
        "e2e": {"value": round(gbs, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="2", help="workload 1..5, or 'all' (one line each)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--extra", default="", choices=["", "copy_blocks"],
                    help="measure a side kernel instead of decode")
    ap.add_argument("--alibi", action="store_true", help="decode with ALiBi slopes")
    ap.add_argument("--schedule", default="auto",
                    choices=["auto", "balanced", "partitioned", "dynamic"],
                    help="how CTAs share the work (pa_options.schedule)")
    ap.add_argument("--stages", type=int, default=0,
                    help="force this many page buffers per warp (pa_options.stages)")
    ap.add_argument("--partition-pages", type=int, default=0,
                    help="force split-KV partitions of this many blocks (pa_options.partition_pages)")
    ap.add_argument("--fp8-compute", action="store_true",
                    help="e4m3 x e4m3 tensor-core products for an FP8 cache (pa_options.fp8_compute)")
    ap.add_argument("--mha-cuda-cores", action="store_true",
                    help="q.K and P.V on the CUDA cores for one query head per kv head")
    ap.add_argument("--no-cascade", action="store_true",
                    help="do not declare a workload's shared prefix (plain per-sequence decode)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config figures of the other workloads (1 GPU only)")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="run the workload with fewer sequences (profiling captures only)")
    ap.add_argument("--ref-budget", type=float, default=20.0,
                    help="seconds of CPU time for the reference arm's timed steps")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(device)
    import paged_kv_cache_471_b200 as pa
    pa.lib()

    if args.extra == "copy_blocks":
        if rank == 0:
            run_copy_blocks(args, device)
        return 0
    cfg_ids = [1, 2, 3, 4, 5] if args.config == "all" else [int(args.config)]
    for idx in cfg_ids:
        r = time_gpu(idx, args.steps, args.warmup, device, want_e2e=not args.no_e2e, rank=rank,
                     num_seqs=args.num_seqs, cascade=not args.no_cascade, alibi=args.alibi,
                     schedule=args.schedule, mha_cuda_cores=args.mha_cuda_cores,
                     fp8_compute=args.fp8_compute, partition_pages=args.partition_pages,
                     stages=args.stages)
        r["step_ms"] = reduce_max(r["step_ms"], device)
        if "e2e_ms" in r:
            r["e2e_ms"] = reduce_max(r["e2e_ms"], device)
        cpu = None
        if rank == 0 and ws == 1 and not args.no_cpu and idx == cfg_ids[0]:
            cpu = cpu_sample(idx, r["wl"])
        line = result_line(idx, r, ws, args.steps, args.warmup, cpu) if rank == 0 else None
        del r
        torch.cuda.empty_cache()
        # One GPU, one workload asked for: the line also carries every
        # workload's figures (each its own timed region of >= 0.3 s).
        if (ws == 1 and len(cfg_ids) == 1 and not args.no_per_config and not args.num_seqs
                and not args.alibi and args.schedule == "auto" and not args.mha_cuda_cores
                and not args.fp8_compute and not args.partition_pages and not args.stages):
            per = {}
            for j in (1, 2, 3, 4, 5):
                rj = time_gpu(j, args.steps, args.warmup, device, want_e2e=False,
                              min_region_ms=300.0, extras=(j == 1),
                              cascade=not args.no_cascade)
                per[str(j)] = config_entry(j, rj)
                del rj
                torch.cuda.empty_cache()
            line["per_config"] = per
        if rank == 0:
            print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
