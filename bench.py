"""Benchmark of one DSA sparse-attention prefill layer on B200.

A step is one pass of the whole layer (indexer scores -> exact top-k ->
sparse attention) through dsa_prefill_layer over one synthetic chunk: by
default the 8,192-query chunk at positions 9,216..17,407 of a 17,408-token
context (top-2048, 32 heads, 512 + 64 latent/rope, indexer 32 x 128).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line. ``value`` is whole-job queries per second per layer
(device time, inputs resident in HBM, L2 flushed between steps); ``e2e`` is
the same metric through the same C-ABI call with host buffers, the
host->device copies of the inputs and the device->host copy of the output
inside the timed region. ``--impl reference`` times the float64 CPU oracle on
a bounded sample of the same workload instead.

Multi-GPU (torchrun): by default every rank runs its own chunk of the same
shape (weak scaling, no data-path collective); with ``--split query`` one chunk
is split by queries over the ranks (strong scaling: the chunk's new cache rows
and the outputs are all-gathered over NCCL inside each step). The step time is
the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

SPEC_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of a
# kernel inside the layer on a workload, from one ncu capture of that launch
# (bench.py --layer-only on the same workload). An entry is removed whenever
# its kernel changes after the capture.
# key: (CUDA kernel, workload); value: bytes per launch
PROFILED_DRAM_BYTES_PER_LAUNCH: dict = {
    ("index_scores_tc", "chunk8k_ctx17k"): 256_191_488 + 394_599_936,
    ("topk_window_kernel", "chunk8k_ctx17k"): 515_052_288 + 56_298_752,
    ("sparse_attn_tc", "chunk8k_ctx17k"): 389_540_352 + 242_374_656,
}
# the CUDA kernel behind each timed entry point (the layer's own launch configuration)
KERNEL_OF = {"index_scores": "index_scores_tc", "topk_select": "topk_window_kernel",
             "sparse_attn": "sparse_attn_tc"}

def kernels_per_layer(d) -> int:
    """Kernels one layer call launches: the two key-norm passes, the indexer,
    the top-k's window select and its redo pass over handed-back rows (whose
    CTAs exit at once when there are none), a second top-k pass for rows past
    49,152 keys, and the attention; the FP8 indexer adds the e4m3 forms of the
    keys and of the queries."""
    two_pass = d.q_pos0 + d.n_q > 49152
    return 6 + (1 if two_pass else 0) + (2 if d.flags & 1 else 0)
E2E_SUB_CHUNKS = (2, 4, 8, 16, 64)  # query sub-chunk counts tried for the host-buffer call (copies overlap the layer)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------- distributed


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's synthetic chunk: every rank works on its own chunk."""
    return seed + 1000 * rank


def whole_job_rate(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Units per second over all ranks, for a step time that is the max over ranks."""
    return world * units_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons while running.

    Reads NVML every few milliseconds from a background thread (read-only
    queries); falls back to `nvidia-smi -lms` when NVML is unavailable.
    """

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_s: float = 0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []  # (sm_mhz, max_mhz, set of reason names)
        self.stop = threading.Event()
        self.thread = None
        self.proc = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            masks = [(n, getattr(pynvml, attr, 0)) for n, attr in self.REASONS]

            def loop():
                while not self.stop.is_set():
                    try:
                        mhz = pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM)
                        bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                        self.samples.append((float(mhz), float(max_mhz),
                                             {n for n, m in masks if m and bits & m}))
                    except pynvml.NVMLError:
                        pass
                    self.stop.wait(self.period)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
        except Exception:  # no NVML: sample with nvidia-smi instead
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100", "-i", str(self.gpu)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.thread = threading.Thread(target=self._read_smi, daemon=True)
                self.thread.start()
            except (OSError, FileNotFoundError):
                self.proc = None
        return self

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                self.samples.append((float(parts[1]), float(parts[2]),
                                     {n for n, v in zip(names, parts[5:9])
                                      if v.lower().startswith("active")}))
            except ValueError:
                continue

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": self.samples[-1][1], "reasons": sorted(reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------ our GPU path


def kernel_rates(d, per_kernel_ms, peaks):
    """Useful rate and roofline fraction of each entry point's kernels.

    The indexer and the attention are contractions (useful FLOP / time against
    the bf16 peak); the top-k reads each causal score once and writes the
    selection (algorithmic bytes / time against the HBM copy bandwidth)."""
    fl = workloads.useful_flops(d)
    t = d.q_pos0 + np.arange(d.n_q, dtype=np.int64)
    topk_bytes = float(((t + 1) * 4).sum() + d.n_q * d.top_k * 4)
    out = {}
    for name, ms in per_kernel_ms.items():
        if name == "topk_select":
            ach = topk_bytes / (ms / 1e3) / 1e9
            out[name] = {"ms": ms, "bound": "hbm", "achieved": ach, "unit": "GB/s",
                         "algorithmic": topk_bytes, "frac": ach / peaks["hbm_gbs"]}
        else:
            f = fl["indexer"] if name == "index_scores" else fl["attention"]
            ach = f / (ms / 1e3) / 1e12
            out[name] = {"ms": ms, "bound": "tensor", "achieved": ach, "unit": "TFLOP/s",
                         "algorithmic": float(f), "frac": ach / peaks["bf16_tflops"]}
    return out


def time_steps(step, flush, steps, stream, flushed=True):
    """CUDA-event time of each of `steps` calls of step() on `stream`; with
    flushed=True the L2 is overwritten (untimed) before each step."""
    import torch

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for s in range(steps):
        if flushed:
            flush.zero_()
        starts[s].record(stream)
        step()
        ends[s].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in zip(starts, ends)]


def attn_variants(dsa, d, xd, idx, out, lse, flush, stream, steps):
    """Median CUDA-event time (ms) of the attention step alone in each of its
    forms on the layer's own selection: the per-query pipelined kernel, the
    decode split and the block-sparse union over groups of 1 and 2 queries."""
    import torch

    ws = {}

    def ws_for(which):
        if which not in ws:
            ws[which] = torch.empty(max(256, dsa.dsa_workspace_size(d, which)), dtype=torch.uint8,
                                    device="cuda")
        return ws[which]

    calls = {
        "per_query": lambda: dsa.dsa_sparse_attn_prefill(
            d, xd["q"], xd["latent"], xd["rope"], idx, out, lse, ws_for(dsa.DSA_WS_ATTN),
            stream=stream),
        "sm_pair": lambda: dsa.dsa_sparse_attn_prefill(
            dataclasses.replace(d, flags=dsa.DSA_FLAG_ATTN_PAIR), xd["q"], xd["latent"],
            xd["rope"], idx, out, lse, ws_for(dsa.DSA_WS_ATTN), stream=stream),
        "decode_split": lambda: dsa.dsa_sparse_attn_decode(
            d, xd["q"], xd["latent"], xd["rope"], idx, out, lse, ws_for(dsa.DSA_WS_DECODE_ATTN),
            stream=stream),
        "block_qb1": lambda: dsa.dsa_sparse_attn_block(
            d, xd["q"], xd["latent"], xd["rope"], idx, out, lse, 1, ws_for(dsa.DSA_WS_BLOCK_ATTN),
            stream=stream),
        "block_qb2": lambda: dsa.dsa_sparse_attn_block(
            d, xd["q"], xd["latent"], xd["rope"], idx, out, lse, 2, ws_for(dsa.DSA_WS_BLOCK_ATTN),
            stream=stream),
    }
    res = {}
    for name, call in calls.items():
        dsa.check(call())  # warm-up
        res[name] = statistics.median(
            time_steps(lambda: dsa.check(call()), flush, max(3, steps), stream))
    return res


def run_ours(args):
    import torch

    import sparse_attention_prefill_dsa_b200 as dsa

    world, rank, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(local)
    dsa.library()
    wl = workloads.ALL_BY_NAME[args.workload]
    d = wl.dims
    w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    x = workloads.generate(d, rank_seed(wl.seed, rank), wl.kind, w_mode)
    if args.fp8_indexer:  # the FP8 indexer variant of the layer (its own selection contract)
        d = dataclasses.replace(d, flags=dsa.DSA_FLAG_FP8_INDEXER)
    if args.l2_scores:  # the layer's scores and selection over L2-resident query sub-blocks
        d = dataclasses.replace(d, flags=d.flags | dsa.DSA_FLAG_L2_SCORES)
    stream = torch.cuda.current_stream()

    def to_dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    xd = {k: (to_dev_bf16(v) if v.dtype == np.uint16 else torch.from_numpy(v).cuda())
          for k, v in x.items()}
    out = torch.empty(d.n_q, d.n_heads, d.d_latent, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(d.n_q, d.n_heads, dtype=torch.float32, device="cuda")
    idx = torch.empty(d.n_q, d.top_k, dtype=torch.int32, device="cuda")
    # (sized for the whole-chunk schedule too: the end-to-end leg's host call uses it)
    ws_layer = torch.empty(max(dsa.dsa_workspace_size(d, dsa.DSA_WS_LAYER),
                               dsa.dsa_workspace_size(dataclasses.replace(
                                   d, flags=d.flags & ~dsa.DSA_FLAG_L2_SCORES), dsa.DSA_WS_LAYER)),
                           dtype=torch.uint8,
                           device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def layer():
        dsa.check(dsa.dsa_prefill_layer(d, xd["q"], xd["latent"], xd["rope"], xd["q_idx"],
                                        xd["k_idx"], xd["w_idx"], out, lse, idx, ws_layer,
                                        stream=stream))

    for _ in range(args.warmup):
        layer()
        flush.zero_()
    dsa.check(dsa.dsa_device_status(ws_layer, stream=stream))
    torch.cuda.synchronize()

    # ---- timed region: K steps of the layer, L2 flushed (untimed) between steps
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        step_ms = time_steps(layer, flush, args.steps, stream)
    barrier(world)
    dsa.check(dsa.dsa_device_status(ws_layer, stream=stream))
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, d.n_q, ms_per_step)
    fl = workloads.useful_flops(d)
    peaks, peaks_src = load_peaks()
    tflops = fl["total"] / (ms_per_step / 1e3) / 1e12
    if args.layer_only:  # the layer alone (for profiler captures): no other legs
        if rank == 0:
            print(json.dumps({"metric": "DSA prefill queries/s per layer", "value": value,
                              "unit": "queries/s", "ms_per_step": ms_per_step,
                              "workload": wl.name, "tflops": tflops,
                              "clocks": clocks.summary()}), flush=True)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    # ---- the same layer with a warm L2 (no flush between steps)
    warm_ms = time_steps(layer, flush, args.steps, stream, flushed=False)
    warm_ms_per_step = max_over_ranks(statistics.median(warm_ms), world)

    # ---- per-kernel durations, same inputs and launch configuration
    ld = (d.ctx_len + 127) // 128 * 128
    scores = torch.empty(d.n_q, ld, dtype=torch.float32, device="cuda")
    # one workspace for the three single-step calls: the largest they need (the
    # top-k's candidate buffer on rows past 49,152 keys)
    ws_small = torch.empty(max(dsa.dsa_workspace_size(d, w) for w in
                               (dsa.DSA_WS_INDEX_SCORES, dsa.DSA_WS_TOPK, dsa.DSA_WS_ATTN)),
                           dtype=torch.uint8, device="cuda")
    names = ("index_scores", "topk_select", "sparse_attn")
    d1 = dataclasses.replace(d, flags=0)  # the single-step calls take no flag
    if args.fp8_indexer:
        # the e4m3 keys are formed once per cache (as in the layer); the
        # queries' e4m3 form is part of the timed indexer step
        q_rows = d.n_q * d.n_idx_heads
        k8 = torch.empty(d.ctx_len, d.d_idx, dtype=torch.uint8, device="cuda")
        ks = torch.empty(d.ctx_len, dtype=torch.float32, device="cuda")
        kh = torch.empty(d.ctx_len, d.d_idx, dtype=torch.int16, device="cuda")
        q8 = torch.empty(q_rows, d.d_idx, dtype=torch.uint8, device="cuda")
        qs = torch.empty(q_rows, dtype=torch.float32, device="cuda")
        qh = torch.empty(q_rows, d.d_idx, dtype=torch.int16, device="cuda")
        dsa.check(dsa.dsa_quantize_fp8(xd["k_idx"], d.ctx_len, d.d_idx, k8, ks, kh, stream=stream))
        q_in, k_in = qh, kh
    else:
        q_in, k_in = xd["q_idx"], xd["k_idx"]
    ev = []
    for s in range(args.steps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(stream)
        if args.fp8_indexer:
            dsa.check(dsa.dsa_quantize_fp8(xd["q_idx"], q_rows, d.d_idx, q8, qs, qh, stream=stream))
            dsa.check(dsa.dsa_index_scores_fp8(d1, q8, qs, k8, ks, xd["w_idx"], scores, ld,
                                               ws_small, stream=stream))
        else:
            dsa.check(dsa.dsa_index_scores(d1, xd["q_idx"], xd["k_idx"], xd["w_idx"], scores, ld,
                                           ws_small, stream=stream))
        e[1].record(stream)
        dsa.check(dsa.dsa_topk_select(d1, scores, ld, q_in, k_in, xd["w_idx"], idx,
                                      ws_small, stream=stream))
        e[2].record(stream)
        dsa.check(dsa.dsa_sparse_attn_prefill(d1, xd["q"], xd["latent"], xd["rope"], idx, out,
                                              lse, ws_small, stream=stream))
        e[3].record(stream)
        ev.append(e)
    torch.cuda.synchronize()
    per_kernel = {n: statistics.median(e[j].elapsed_time(e[j + 1]) for e in ev)
                  for j, n in enumerate(names)}
    rates = kernel_rates(d, per_kernel, peaks)
    variants = attn_variants(dsa, d1, xd, idx, out, lse, flush, stream, args.steps) \
        if args.attn_variants else None

    # ---- end to end through the library's host-buffer call: every step copies
    # all inputs in from page-locked host memory and the output back, the
    # copies of one query sub-chunk overlapping the layer on another
    pinned = {k: (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
                  if v.dtype == np.uint16 else torch.from_numpy(v)).pin_memory()
              for k, v in x.items()}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = out_host.numel() * out_host.element_size()
    e2e_streams = (torch.cuda.Stream(), stream, torch.cuda.Stream())  # copy in, layer, copy out
    e2e_events = (torch.cuda.Event(), torch.cuda.Event())
    for ev_ in e2e_events:
        ev_.record(stream)  # creates the CUDA events
    dev_tensors = {k: xd[k] for k in ("q", "latent", "rope", "q_idx", "k_idx", "w_idx")}
    dev_tensors["out"] = out
    # two sets of device tensors used in turn (DSA_FLAG_HOST_UNORDERED): the
    # copy-in of one step overlaps the layers and the copy-out of the previous
    # one; a set is reused only after the copy-out of the step that last used
    # it (an event on the copy-out stream)
    dev_sets = (dev_tensors, {k: torch.empty_like(v) for k, v in dev_tensors.items()})
    set_free = [torch.cuda.Event(), torch.cuda.Event()]
    for ev_ in set_free:
        ev_.record(e2e_streams[2])
    # (the host call schedules its own sub-chunks: no L2 sub-blocks there)
    d_host = dataclasses.replace(d, flags=(d.flags & ~dsa.DSA_FLAG_L2_SCORES) | dsa.DSA_FLAG_HOST_UNORDERED)
    e2e_calls = [0]

    def e2e_step(n_sub):
        b = e2e_calls[0] & 1
        e2e_calls[0] += 1
        e2e_streams[0].wait_event(set_free[b])
        e2e_streams[1].wait_event(set_free[b])
        dsa.check(dsa.dsa_prefill_layer_host(
            d_host, pinned["q"], pinned["latent"], pinned["rope"], pinned["q_idx"], pinned["k_idx"],
            pinned["w_idx"], out_host, None, None, dev_sets[b], ws_layer, e2e_streams, e2e_events,
            n_sub=n_sub))
        set_free[b].record(e2e_streams[2])

    # warm-up doubles as the choice of the sub-chunk count: per candidate two
    # untimed steps, then three back to back timed as a whole (consecutive
    # steps overlap), the fastest per step is used for the timed steps
    tried = {}
    for n_sub in E2E_SUB_CHUNKS:
        for _ in range(2):
            e2e_step(n_sub)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(e2e_streams[0])
        for _ in range(3):
            e2e_step(n_sub)
        t1.record(e2e_streams[2])
        torch.cuda.synchronize()
        tried[n_sub] = max_over_ranks(t0.elapsed_time(t1), world) / 3
    n_best = min(tried, key=tried.get)
    for _ in range(max(1, args.warmup)):
        e2e_step(n_best)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(e2e_streams[0])
    for _ in range(args.steps):
        e2e_step(n_best)
    e1.record(e2e_streams[2])
    torch.cuda.synchronize()
    dsa.check(dsa.dsa_device_status(ws_layer, stream=stream))
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    barrier(world)
    # the copies alone, as the bound of the end-to-end figure: every input in
    # (one copy per tensor, pinned host memory) and the output back, each
    # direction by itself, median of the steps
    def copy_ms(h2d_on, d2h_on):
        ts = []
        for _ in range(max(3, args.steps)):
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            joined = torch.cuda.Event()
            c0.record(e2e_streams[0])
            e2e_streams[2].wait_event(c0)
            if h2d_on:
                with torch.cuda.stream(e2e_streams[0]):
                    for k_, v_ in pinned.items():
                        dev_tensors[k_].copy_(v_, non_blocking=True)
            if d2h_on:
                with torch.cuda.stream(e2e_streams[2]):
                    out_host.copy_(out, non_blocking=True)
            joined.record(e2e_streams[2])
            e2e_streams[0].wait_event(joined)
            c1.record(e2e_streams[0])
            torch.cuda.synchronize()
            ts.append(c0.elapsed_time(c1))
        return max_over_ranks(statistics.median(ts), world)
    h2d_only_ms, d2h_only_ms = copy_ms(True, False), copy_ms(False, True)
    both_ms = copy_ms(True, True)  # both directions at once, as in the end-to-end call

    # the dominant kernel's roofline, with its DRAM traffic when a capture of
    # the current kernel on this workload exists
    dom_name = max(per_kernel, key=per_kernel.get)
    r = rates[dom_name]
    kernel = KERNEL_OF[dom_name]
    if dom_name == "sparse_attn" and d.flags & dsa.DSA_FLAG_ATTN_PAIR:
        kernel = "sparse_attn_pair"
    prof = PROFILED_DRAM_BYTES_PER_LAUNCH.get((kernel, wl.name)) if not args.fp8_indexer else None
    roof = {"kernel": kernel, "bound": r["bound"], "achieved": r["achieved"],
            "peak": peaks["bf16_tflops"] if r["bound"] == "tensor" else peaks["hbm_gbs"],
            "unit": r["unit"], "frac": r["frac"],
            "traffic": prof if prof else None,
            "traffic_source": ("ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch of "
                               "this kernel inside the layer on this workload" if prof else None),
            "peak_source": (f"{peaks_src} bf16 burst (kernel timed alone)" if r["bound"] == "tensor"
                            else f"{peaks_src} copy bandwidth")}

    result = {
        "metric": "DSA prefill queries/s per layer",
        "value": value,
        "unit": "queries/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "about": wl.about, "n_q": d.n_q, "q_pos0": d.q_pos0,
                   "ctx_len": d.ctx_len, "top_k": d.top_k, "n_heads": d.n_heads,
                   "d_latent": d.d_latent, "d_rope": d.d_rope, "n_idx_heads": d.n_idx_heads,
                   "d_idx": d.d_idx, "parallelism": f"dp{world} (independent chunks)",
                   "indexer": "fp8 (e4m3) variant" if args.fp8_indexer else "bf16",
                   "scores": "L2-resident query sub-blocks" if args.l2_scores else "whole chunk",
                   "l2": "flushed: 256 MB write between timed steps"},
        "tflops": tflops,
        "pct_of_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
        "bf16_peak": {"tflops": peaks["bf16_tflops"], "source": peaks_src},
        "pct_of_spec_bf16_peak": 100.0 * tflops / SPEC_BF16_TFLOPS,
        "useful_flop_per_step": fl["total"],
        "ms_per_step_median": max_over_ranks(statistics.median(step_ms), world),
        "warm_l2": {"ms_per_step_median": warm_ms_per_step,
                    "value": whole_job_rate(world, d.n_q, warm_ms_per_step)},
        "per_kernel_ms": per_kernel,
        **({"attn_variants_ms": variants} if variants else {}),
        "per_kernel": rates,
        "e2e": {"value": whole_job_rate(world, d.n_q, e2e_ms), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "call": "dsa_prefill_layer_host", "sub_chunks": n_best,
                "h2d_alone_ms": h2d_only_ms, "d2h_alone_ms": d2h_only_ms,
                "h2d_and_d2h_together_ms": both_ms,
                "warmup_ms_by_sub_chunks": {str(k): round(v, 3) for k, v in tried.items()}},
        "gpu_launches": kernels_per_layer(d) * args.steps,
        "roofline": roof,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(d, x, args.cpu_rows)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_split(args):
    """One chunk split by queries over the ranks (strong scaling): each step
    gathers the chunk's new cache rows, runs the layer on this rank's query
    range (dsa_partition_queries) and gathers the outputs, all over NCCL."""
    import datetime

    import torch
    import torch.distributed as dist

    import sparse_attention_prefill_dsa_b200 as dsa
    from sparse_attention_prefill_dsa_b200 import multi_gpu

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dsa.library()
    wl = workloads.ALL_BY_NAME[args.workload]
    d = wl.dims
    w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    x = workloads.generate(d, wl.seed, wl.kind, w_mode)  # one chunk, the same on every rank
    stream = torch.cuda.current_stream()

    def to_dev(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
            else torch.from_numpy(a)
        return t.cuda()

    cache = {k: to_dev(x[k]) for k in ("latent", "rope", "k_idx")}
    chunk = {k: to_dev(x[k]) for k in ("q", "q_idx", "w_idx")}
    outputs = {"out": torch.empty(d.n_q, d.n_heads, d.d_latent, dtype=torch.bfloat16,
                                  device="cuda")}
    ranges = multi_gpu.query_ranges(d, world)
    s0, e0 = ranges[rank]
    ws = torch.empty(dsa.dsa_workspace_size(multi_gpu.sub_dims(d, s0, e0), dsa.DSA_WS_LAYER),
                     dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def layer_fn(sd, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx):
        dsa.check(dsa.dsa_prefill_layer(sd, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx,
                                        ws, stream=stream))

    def step():
        multi_gpu.prefill_layer_sharded(d, rank, world, cache, chunk, outputs, layer_fn)

    for _ in range(args.warmup):
        step()
        flush.zero_()
    dsa.check(dsa.dsa_device_status(ws, stream=stream))
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        step_ms = time_steps(step, flush, args.steps, stream)
    barrier(world)
    dsa.check(dsa.dsa_device_status(ws, stream=stream))
    ms_per_step = max_over_ranks(sum(step_ms), world) / args.steps
    value = d.n_q / (ms_per_step / 1e3)

    # end to end: this rank's inputs (its chunk rows and the prefix cache) in
    # from page-locked host memory, the gathered output back out, every step
    pinned = {k: (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
                  if v.dtype == np.uint16 else torch.from_numpy(v)).pin_memory()
              for k, v in x.items()}
    out_host = torch.empty(outputs["out"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = 0
    for k in ("latent", "rope", "k_idx"):
        h2d += (d.q_pos0 + e0 - s0) * pinned[k][0].numel() * pinned[k].element_size()
    for k in ("q", "q_idx", "w_idx"):
        h2d += (e0 - s0) * pinned[k][0].numel() * pinned[k].element_size()
    d2h = out_host.numel() * out_host.element_size()

    def e2e():
        for k in ("latent", "rope", "k_idx"):
            cache[k][: d.q_pos0].copy_(pinned[k][: d.q_pos0], non_blocking=True)
            cache[k][d.q_pos0 + s0: d.q_pos0 + e0].copy_(
                pinned[k][d.q_pos0 + s0: d.q_pos0 + e0], non_blocking=True)
        for k in ("q", "q_idx", "w_idx"):
            chunk[k][s0:e0].copy_(pinned[k][s0:e0], non_blocking=True)
        step()
        out_host.copy_(outputs["out"], non_blocking=True)

    for _ in range(args.warmup):
        e2e()
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        e2e()
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world) / args.steps
    fl = workloads.useful_flops(d)
    peaks, _ = load_peaks()
    tflops = fl["total"] / (ms_per_step / 1e3) / 1e12
    result = {
        "metric": "DSA prefill queries/s per layer", "value": value, "unit": "queries/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "about": wl.about, "n_q": d.n_q, "ctx_len": d.ctx_len,
                   "top_k": d.top_k, "parallelism": f"query split over {world} ranks "
                   "(cache rows and outputs all-gathered over NCCL)",
                   "ranges": ranges, "l2": "flushed: 256 MB write between timed steps"},
        "tflops": tflops, "pct_of_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
        "e2e": {"value": d.n_q / (e2e_ms / 1e3), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": kernels_per_layer(d) * args.steps,
        "clocks": clocks.summary(),
    }
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ----------------------------------------------------------- CPU reference


def oracle_sample(d, x, n_rows):
    """Times the float64 oracle on n_rows query rows spread over the chunk."""
    import oracle

    rows = np.linspace(0, d.n_q - 1, n_rows).round().astype(np.int32)
    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.prefill_layer(d, **x, rows=rows, n_threads=cores)
    dt = time.perf_counter() - t0
    return n_rows / dt, cores, dt


def sized_rows(d, x, seconds):
    """Rows of a CPU-oracle sample that takes about `seconds` on this host."""
    _, _, dt = oracle_sample(d, x, 8)
    return int(min(d.n_q, max(8, round(8 * seconds / max(dt, 1e-3)))))


def cpu_baseline(d, x, n_rows=None, seconds=12.0):
    if not n_rows:
        n_rows = sized_rows(d, x, seconds)
    qps, cores, dt = oracle_sample(d, x, n_rows)
    return {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": f"{n_rows} of {d.n_q} query rows spread over the chunk, full layer per "
                      f"row (float64 oracle, {cores} threads, {dt:.1f} s wall)"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle

    oracle.build()
    wl = workloads.ALL_BY_NAME[args.workload]
    d = wl.dims
    w_mode = "ones" if wl.kind == "ternary_ties" else "uniform"
    x = workloads.generate(d, wl.seed, wl.kind, w_mode)
    rows_per_step = args.cpu_rows or sized_rows(d, x, 6.0)
    for _ in range(args.warmup):
        oracle_sample(d, x, max(1, rows_per_step // 4))
    times = []
    cores = os.cpu_count() or 1
    for _ in range(args.steps):
        _, cores, dt = oracle_sample(d, x, rows_per_step)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = rows_per_step / (ms / 1e3)
    result = {
        "impl": "reference", "metric": "DSA prefill queries/s per layer", "value": value,
        "unit": "queries/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "about": wl.about, "n_q": d.n_q, "ctx_len": d.ctx_len,
                   "top_k": d.top_k},
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} of {d.n_q} query rows per step, full "
                                   f"layer per row (float64 oracle, {cores} threads)"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="chunk8k_ctx17k", choices=sorted(workloads.ALL_BY_NAME))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="query rows of the bounded CPU-oracle sample (0: about 12 s of work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", default="chunks", choices=("chunks", "query"),
                    help="chunks: every rank runs its own chunk (weak scaling, default); "
                         "query: one chunk split by queries over the ranks (strong scaling)")
    ap.add_argument("--attn-variants", action="store_true",
                    help="also time the attention step's other forms (decode split, block union)")
    ap.add_argument("--fp8-indexer", action="store_true",
                    help="the layer with the FP8 indexer variant (dims.flags = DSA_FLAG_FP8_INDEXER)")
    ap.add_argument("--l2-scores", action="store_true",
                    help="the layer's indexer and top-k over query sub-blocks whose scores stay in L2 "
                         "(dims.flags = DSA_FLAG_L2_SCORES)")
    ap.add_argument("--layer-only", action="store_true",
                    help="time the layer alone and print a short line (for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.split == "query":
        run_split(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
