"""Benchmark of the CSA / HCA decode hot path on B200.

Default workload: one CSA decode step at 128K context, batch 32 (64 query
heads x 512, FP8 entries with a scale per 64, MXFP4 indexer 64 x 128, top-k
512, window 128 bf16, sink).  A step is one csa_decode call: indexer ->
top-k -> sparse attention (+ split-K combine) over the whole batch.  The HCA
decode step at 1M context, batch 8, is timed in the same run and reported
under "hca_decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Timing: W untimed steps, then K steps, each bracketed by CUDA events on the
launching stream with an L2 flush (a 256 MB write) between steps outside the
events; barrier + synchronize on both sides; max over ranks.  The device-side
step is the library call captured once in a CUDA graph and replayed (the way
a decode loop runs it); the e2e number calls the library eagerly, with every
step's host-to-device input copies and device-to-host output read inside the
timed region, overlapped with the neighbouring steps' compute on separate
streams (the caches rotate over three copies larger than L2 together, since
no flush runs between overlapped steps).  Multi-GPU runs are independent
replicas (weak scaling): each rank decodes its own batch.
The reference arm (--impl reference) is the CPU oracle on a bounded sample of
the same workload.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA attn decode tok/s @128K–1M; HBM GB/s & tensor-core % of B200 peak"
WORKLOAD = "csa_decode_128k_b32"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------ algorithmic bytes
def csa_decode_bytes(w):
    """Bytes the method must move in one CSA decode step (per batch): the
    indexer keys of every visible block (E2M1 + E8M0: 68 B at dI = 128), the
    indexer query and weights, the selected FP8 entries (codes + scales), the
    bf16 window, q, and the bf16 output.  The scores and the selection are
    this design's intermediates, not the method's bytes, and are not counted."""
    nb = w.n_ctx // w.m
    ne = (w.n_ctx - w.W) // w.m
    key = w.dI // 2 + w.dI // 32
    ent = w.d + 4 * (w.d // 64)
    idx = ne * key + w.HI * key + w.HI * 4
    att = w.k * ent + w.W * w.d * 2 + 2 * w.H * w.d * 2
    return {"indexer": w.batch * idx, "attention": w.batch * att, "step": w.batch * (idx + att),
            "n_blocks": nb}


def hca_decode_bytes(w):
    ne = (w.n_ctx - w.W) // w.m
    ent = w.d + 4 * (w.d // 64)
    return w.batch * (ne * ent + w.W * w.d * 2 + 2 * w.H * w.d * 2)


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU while the timed
    region runs.  NVML is polled from a host thread every `period` seconds
    (read-only queries); without NVML, nvidia-smi is sampled every 100 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int, period: float = 0.0005):
        self.index, self.period = index, period
        self.proc = self.thread = None
        self.samples, self.max_mhz, self.lines = [], None, []
        self.marks = {}
        self._sample = None

    def mark(self, name):
        """Record the host time of an event (the timed region's start / end)
        and take one sample right there, so that a short timed region still
        has samples at its edges."""
        self.marks[name] = time.perf_counter()
        if self._sample is not None:
            try:
                self._sample()
            except Exception:
                pass

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:  # the same physical GPU as the CUDA device, whatever the visible-device mapping
            import torch
            pr = torch.cuda.get_device_properties(self.index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def __enter__(self):
        try:
            import threading
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop = threading.Event()

            def sample():
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, {n for n, b in bits.items() if rs & b}, time.perf_counter()))

            def poll():
                while not self.stop.is_set():
                    try:
                        sample()
                    except Exception:
                        return
                    self.stop.wait(self.period)

            self._sample = sample

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
            for ln in self.lines:
                f = [x.strip() for x in ln.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm, self.max_mhz = float(f[1]), float(f[2])
                except ValueError:
                    continue
                self.samples.append((sm, {n for n, v in zip(self.NAMES, f[5:9]) if v.lower() == "active"},
                                     None))

    def summary(self):
        """Median SM clock and the reasons seen over every sample (the whole
        measurement: warm-up, timed steps and the per-kernel legs), plus the
        same over the samples taken inside the timed region alone."""
        sm = [x for x, _, _ in self.samples]
        reasons = set().union(*(r for _, r, _ in self.samples)) if self.samples else set()
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
               "reasons": sorted(reasons), "samples": len(sm), "period_ms": self.period * 1e3,
               "source": "nvml" if self.thread else ("nvidia-smi" if self.proc else None)}
        t0, t1 = self.marks.get("timed_start"), self.marks.get("timed_end")
        if t0 is not None and t1 is not None:
            tr = [(x, r) for x, r, ts in self.samples if ts is not None and t0 <= ts <= t1 + 1e-3]
            out["timed_region"] = {"sm_mhz": statistics.median([x for x, _ in tr]) if tr else None,
                                   "reasons": sorted(set().union(*(r for _, r in tr))) if tr else [],
                                   "samples": len(tr), "seconds": round(t1 - t0, 4)}
        return out


# ------------------------------------------------------------------ our arm
def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (all ranks call this, in the same
    order): a multi-GPU step is as slow as its slowest replica."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(batch: int, steps: int, world: int, t_ms: float) -> float:
    """Tokens per second of the whole job: every replica decodes `batch`
    sequences per step, and the job takes the slowest replica's time."""
    return batch * steps * world / (t_ms / 1e3)


def setup_csa_decode(w, dev):
    import torch

    import compressed_sparse_attention_13_b200 as K
    from synth.workloads import draw_torch

    B, H, d, HI, dI, m, W, k = w.batch, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = w.n_ctx // m
    p = K.params(m, W, k, H, d, HI, dI, w.scale, K.BF16, K.FP8_S64, K.MXFP4)

    def quant(name, fmt):
        v = draw_torch(w, name, device=dev)
        v = v.reshape(-1, v.shape[-1])
        st = K.empty_stored(fmt, v.shape[0], v.shape[1], device=dev)
        K.csa_quantize(v, st)
        torch.cuda.synchronize()
        return st

    S = {"p": p, "nb": nb}
    S["kv"] = quant("kv", K.FP8_S64)
    S["kI"] = quant("kI", K.MXFP4)
    S["qI"] = quant("qI", K.MXFP4)
    S["q"] = draw_torch(w, "q", device=dev)
    S["w"] = draw_torch(w, "w", device=dev)
    S["window"] = draw_torch(w, "window", device=dev)
    S["sinks"] = draw_torch(w, "sinks", device=dev)
    q_pos = torch.full((B,), w.n_ctx, dtype=torch.int64, device=dev)
    S["q_pos"], S["raw_pos0"] = q_pos, q_pos - W + 1
    S["out"] = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    S["sel"] = torch.empty(B, k, dtype=torch.int32, device=dev)
    S["ws"] = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, B, 1, nb), dtype=torch.uint8, device=dev)
    return S


def csa_decode_call(w, S, stream=None):
    import compressed_sparse_attention_13_b200 as K
    K.csa_decode(S["p"], w.batch, S["q"], S["qI"], S["w"], S["kv"], S["kI"], S["nb"], S["window"],
                 w.W, S["raw_pos0"], S["q_pos"], S["sinks"], S["out"], S["sel"], S["ws"], stream)


def e2e_pipelined(w, S, dev, steps, warmup, full_window=False, n_sets=3):
    """End to end through the public call (csa_decode) with the host copies
    inside the timed region.  Every step copies the inputs a decode loop
    receives for the new token of each sequence -- q, qI (MXFP4 codes and
    scales), w, the token's raw row for the sliding window, the positions --
    from one packed pinned host buffer to the device, appends the raw row to
    the device-resident window (whose other W - 1 rows are cache state, like
    the pooled entries), and reads the output back.  With full_window the
    whole window is copied from the host every step instead.  The copies run
    on their own streams and overlap the neighbouring steps' compute (two
    buffer sets, events between the streams), as a decode server's loop does;
    the caches rotate over three copies (3 x 89 MB, more than the 126 MB L2),
    so no step finds its cache rows in L2 from the steps before.  Returns the
    elapsed ms of `steps` steps after `warmup` and the bytes copied per step."""
    import torch

    import compressed_sparse_attention_13_b200 as K

    comp = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    new_row = S["window"][:, -1].contiguous()           # the new token's raw row per sequence
    parts = [("q", S["q"]), ("w", S["w"]), ("q_pos", S["q_pos"]), ("raw_pos0", S["raw_pos0"]),
             ("qI", S["qI"].data), ("qI_s", S["qI"].scales)]
    parts.append(("window", S["window"]) if full_window else ("new_row", new_row))
    offs, off = {}, 0
    for n, t in parts:                      # 256-byte aligned slots of one byte buffer
        offs[n] = off
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(off, dtype=torch.uint8).pin_memory()
    for n, t in parts:
        nb = t.numel() * t.element_size()
        host[offs[n]:offs[n] + nb].copy_(t.detach().contiguous().view(-1).view(torch.uint8).cpu())

    def views(buf):
        v = {}
        for n, t in parts:
            nb = t.numel() * t.element_size()
            v[n] = buf[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape)
        return v

    bufs = []
    for _ in range(2):
        raw = torch.empty(off, dtype=torch.uint8, device=dev)
        d = views(raw)
        d["raw"] = raw
        d["qI"] = K.Stored(S["qI"].fmt, d["qI"], d.pop("qI_s"))
        if not full_window:
            d["window"] = S["window"].clone()   # resident window rows; the last one is appended per step
        d["out"], d["sel"] = torch.empty_like(S["out"]), torch.empty_like(S["sel"])
        d["out_h"] = torch.empty(S["out"].shape, dtype=S["out"].dtype).pin_memory()
        bufs.append(d)
    clone = lambda st: K.Stored(st.fmt, st.data.clone(), st.scales.clone())
    caches = [(S["kv"], S["kI"])] + [(clone(S["kv"]), clone(S["kI"])) for _ in range(n_sets - 1)]
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]

    def run(i0, n):
        for i in range(i0, i0 + n):
            b, d = i % 2, bufs[i % 2]
            kv, kI = caches[i % n_sets]
            if i >= 2:
                h2d_s.wait_event(in_free[b])        # step i - 2 is done with these inputs
            with torch.cuda.stream(h2d_s):
                d["raw"].copy_(host, non_blocking=True)
            in_ready[b].record(h2d_s)
            comp.wait_event(in_ready[b])
            if i >= 2:
                comp.wait_event(out_read[b])        # step i - 2's output has been read back
            if not full_window:
                d["window"][:, -1].copy_(d["new_row"])   # append the new token's raw row
            K.csa_decode(S["p"], w.batch, d["q"], d["qI"], d["w"], kv, kI, S["nb"], d["window"], w.W,
                         d["raw_pos0"], d["q_pos"], S["sinks"], d["out"], d["sel"], S["ws"], comp)
            in_free[b].record(comp)
            d2h_s.wait_event(in_free[b])
            with torch.cuda.stream(d2h_s):
                d["out_h"].copy_(d["out"], non_blocking=True)
            out_read[b].record(d2h_s)

    run(0, warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    h2d_s.wait_event(e0)
    run(warmup, steps)
    comp.wait_stream(d2h_s)
    e1.record(comp)
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for _, t in parts)
    d2h = bufs[0]["out_h"].numel() * bufs[0]["out_h"].element_size()
    return {"ms": e0.elapsed_time(e1), "steps": steps, "unit": "tok/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "inputs": ("q, qI, w, positions and the whole window" if full_window else
                       "q, qI, w, positions and the new token's raw row (appended to the resident window)"),
            "pipelined": "one packed input copy and the output read per step, on their own streams, "
            "overlap the neighbouring steps' compute; caches rotate over 3 copies (3 x 89 MB > L2)"}


def time_steps(fn, steps, warmup, flush, stream, clk=None):
    """Per-step CUDA-event times (ms) with an L2 flush before every step.
    With a clock sampler, the timed region (after the warm-up, until the last
    step has completed) is marked on it."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if clk is not None:
        clk.mark("timed_start")
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    if clk is not None:
        clk.mark("timed_end")
    return [a.elapsed_time(b) for a, b in ev]


def kernel_times_in_step(fns, steps, warmup, flush, stream):
    """Mean CUDA-event time (ms) of each of `fns`, run one after another as one
    step (an L2 flush before every step), over `steps` steps after `warmup`."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        for f in fns:
            f()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)] for _ in range(steps)]
    for e in ev:
        flush.zero_()
        e[0].record(stream)
        for f, b in zip(fns, e[1:]):
            f()
            b.record(stream)
    torch.cuda.synchronize()
    return [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev) for i in range(len(fns))]


def graphed(fn):
    """Capture fn (a sequence of library calls on the current stream) in a
    CUDA graph after one eager call; returns a replay function.  The decode
    step is a handful of short launches, so host enqueue time would otherwise
    show up as idle time inside the events."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g.replay


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "compressed_sparse_attention_13_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, src_hash):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the current source of that kernel."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel)
        if rec and rec.get("source_sha") == src_hash:
            return rec["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def run_ours(args):
    import torch
    import torch.distributed as dist

    import compressed_sparse_attention_13_b200 as K
    from synth.workloads import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    K.lib()
    hbm_peak, bf16_peak, peak_kind = peaks()
    if args.only_legs:
        # one GPU, the named extra legs alone (a small command to profile them)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        legs = {"hca": lambda: bench_hca(args, dev, flush, stream, hbm_peak),
                "prefill": lambda: bench_prefill(dev, flush, stream, bf16_peak),
                "stack": lambda: bench_stack(dev, flush, stream, hbm_peak, bf16_peak),
                "schedule": lambda: bench_schedule(dev, flush, stream, hbm_peak),
                "indexer": lambda: bench_indexer_variants(args, dev, flush, stream, hbm_peak),
                "shard": lambda: bench_shard(args, dev, flush, stream)}
        print(json.dumps({n: legs[n]() for n in args.only_legs.split(",")}), flush=True)
        return

    w = WORKLOADS[WORKLOAD]
    S = setup_csa_decode(w, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    eager_step = lambda: csa_decode_call(w, S)
    step = graphed(eager_step)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # warm-up + timed steps; the clock sampler runs across them and the
    # per-kernel legs below, and marks the timed region
    barrier()
    clk = ClockSampler(local).__enter__()
    times = time_steps(step, args.steps, args.warmup, flush, stream, clk)
    barrier()
    t_ms = max_over_ranks(sum(times), dev)
    assert K.csa_device_status(reset=True) == 0
    value = job_throughput(w.batch, args.steps, world, t_ms)

    # The step's kernels one at a time: the three entry points csa_decode
    # calls, with the same arguments (the same launches), enqueued eagerly with
    # CUDA events between them on the launching stream, over the same number of
    # steps, each step after an L2 flush.  The 256 MB flush runs for longer
    # than the host takes to enqueue the step, so the events time the kernels,
    # not the host.  Each is also timed alone (graph-replayed after a flush).
    nb = S["nb"]
    scores = S["ws"].view(torch.float32)[: w.batch * nb].view(w.batch, nb)
    ws_attn = torch.empty(K.csa_workspace_size(S["p"], K.OP_SPARSE_ATTN, w.batch, 1, 0),
                          dtype=torch.uint8, device=dev)
    kfn = {
        "indexer_score": lambda: K.indexer_score(S["p"], w.batch, 1, S["qI"], S["w"], S["kI"], nb,
                                                 S["q_pos"], scores, nb),
        "topk_select": lambda: K.topk_select(S["p"], w.batch, 1, scores, nb, nb, S["q_pos"], S["sel"]),
        "sparse_mqa_attn": lambda: K.sparse_mqa_attn(
            S["p"], w.batch, 1, S["q"], S["kv"], nb, S["sel"], S["window"], w.W, S["raw_pos0"],
            S["q_pos"], S["sinks"], S["out"], ws_attn),
    }
    in_step = kernel_times_in_step(list(kfn.values()), args.steps, args.warmup, flush, stream)
    in_step = dict(zip(kfn.keys(), in_step))
    kt = {name: statistics.mean(time_steps(graphed(fn), max(20, args.steps // 5), 3, flush, stream))
          for name, fn in kfn.items()}
    clk.__exit__(None, None, None)
    by = csa_decode_bytes(w)
    src = {"indexer_score": kernel_source_hash(["k_indexer_tc.cu", "sm100.cuh", "common.cuh"]),
           "sparse_mqa_attn": kernel_source_hash(["k_attn_tc.cu", "sm100.cuh", "common.cuh"]),
           "topk_select": kernel_source_hash(["k_topk.cu", "common.cuh"])}
    kname = {"indexer_score": "indexer_tc_kernel", "sparse_mqa_attn": "attn_tc_kernel",
             "topk_select": "topk"}
    alg = {"indexer_score": by["indexer"], "sparse_mqa_attn": by["attention"]}
    stage_roof = {}
    for n, ms in in_step.items():
        if n in alg:
            gbs = alg[n] / (ms / 1e3) / 1e9
            stage_roof[n] = {"kernel": kname[n], "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak,
                             "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
                             "traffic": recorded_traffic(kname[n], src[n]), "algorithmic_bytes": alg[n],
                             "us_in_step": round(ms * 1e3, 2), "peak_source": peak_kind}
        else:
            stage_roof[n] = {"kernel": kname[n], "bound": "latency", "us_in_step": round(ms * 1e3, 2),
                             "score_bytes_read": w.batch * (by["n_blocks"] - w.W // w.m) * 4}
    dominant = max(in_step, key=in_step.get)
    if dominant not in alg:   # the roofline names an HBM-bound kernel; take the slower of the two
        dominant = max(alg, key=lambda n: in_step[n])

    # end to end: host inputs (pinned) -> device, step, output -> host
    n_e2e = max(20, args.steps // 2)
    e2e = e2e_pipelined(w, S, dev, n_e2e, max(3, args.warmup))
    e2e = {"value": round(job_throughput(w.batch, e2e.pop("steps"), world, max_over_ranks(e2e.pop("ms"), dev)), 1),
           **e2e}
    full = e2e_pipelined(w, S, dev, n_e2e, max(3, args.warmup), full_window=True)
    e2e["full_window"] = {"value": round(job_throughput(w.batch, full.pop("steps"), world,
                                                        max_over_ranks(full.pop("ms"), dev)), 1),
                          "h2d_bytes_per_step": full["h2d_bytes_per_step"]}

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp4 indexer + bf16 attention (fp32 accumulate)", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": WORKLOAD, "batch": w.batch, "context": w.n_ctx, "heads": w.H,
                   "head_dim": w.d, "idx_heads": w.HI, "idx_dim": w.dI, "m": w.m, "top_k": w.k,
                   "window": w.W, "kv": "fp8_e4m3_scale64", "indexer": "mxfp4",
                   "parallelism": f"replicas x{world}", "l2": "flushed (256 MB write) between steps"},
        # the slowest HBM-bound kernel of the step, timed inside the step
        "roofline": dict(stage_roof[dominant], kernel=f"{dominant} ({kname[dominant]})"),
        "stage_roofline": stage_roof,
        "kernels_us_in_step": {n: round(v * 1e3, 2) for n, v in in_step.items()},
        # each entry point alone, graph-replayed after an L2 flush (cold scores)
        "kernels_us_isolated": {n: round(v * 1e3, 2) for n, v in kt.items()},
        "step_bytes": by["step"],
        "step_gbs": round(by["step"] / (t_ms / args.steps / 1e3) / 1e9, 1),
        "e2e": e2e,
        # indexer, top-k and attention (the split combine runs in the attention's cluster)
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }
    legs = set(args.legs.split(",")) if args.legs else {"hca", "indexer", "shard", "prefill", "stack", "schedule"}
    if world == 1 and rank == 0 and not args.no_extra:
        if "hca" in legs:
            result["hca_decode"] = bench_hca(args, dev, flush, stream, hbm_peak)
        del S
        torch.cuda.empty_cache()
        if "indexer" in legs:
            try:
                result["indexer_write_path"] = bench_indexer_variants(args, dev, flush, stream, hbm_peak)
            except Exception as exc:  # an extra leg must not lose the main line
                result["indexer_write_path"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        torch.cuda.empty_cache()
        for key, name, leg in (("sharded_decode_1m", "shard", lambda: bench_shard(args, dev, flush, stream)),
                               ("prefill_8k_bf16", "prefill", lambda: bench_prefill(dev, flush, stream, bf16_peak)),
                               ("stack_c4", "stack", lambda: bench_stack(dev, flush, stream, hbm_peak, bf16_peak)),
                               ("schedule_v4_pro", "schedule", lambda: bench_schedule(dev, flush, stream, hbm_peak))):
            if name not in legs:
                continue
            try:
                result[key] = leg()
            except Exception as exc:  # an extra leg must not lose the main line
                result[key] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def bench_hca(args, dev, flush, stream, hbm_peak):
    """HCA decode at 1M context, batch 8: pool the context (m' = 128) into FP8
    entries once, then time hca_attn steps."""
    import torch

    import compressed_sparse_attention_13_b200 as K
    from synth.workloads import WORKLOADS, draw_torch

    w = WORKLOADS["hca_decode_1m_b8"]
    B, N, H, d, m, W = w.batch, w.n_ctx, w.H, w.d, w.m, w.W
    nb = N // m
    p = K.params(m, W, 1, H, d, 1, 32, w.scale, K.BF16, K.FP8_S64, K.MXFP4)
    kv = K.empty_stored(K.FP8_S64, B * nb, d, device=dev)
    bias = draw_torch(w, "bias", device=dev)
    x = draw_torch(w, "x", device=dev)
    z = draw_torch(w, "z", device=dev)
    comp = lambda: K.csa_compress(p, d, x, z, bias, B * N, kv)
    t_comp = statistics.mean(time_steps(graphed(comp), 5, 3, flush, stream))
    comp_bytes = 2 * B * N * d * 2 + B * nb * (d + 4 * d // 64)
    win = torch.cat([x[:, N - W + 1:], draw_torch(w, "x_new", device=dev)[:, None]], 1).contiguous()
    del x, z
    torch.cuda.empty_cache()
    q, sinks = draw_torch(w, "q", device=dev), draw_torch(w, "sinks", device=dev)
    q_pos = torch.full((B,), N, dtype=torch.int64, device=dev)
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, B, 1, nb), dtype=torch.uint8, device=dev)
    raw_pos0 = q_pos - W + 1
    fn = graphed(lambda: K.hca_attn(p, B, 1, q, kv, nb, win, W, raw_pos0, q_pos, sinks, out, ws))
    times = time_steps(fn, args.steps, args.warmup, flush, stream)
    t = statistics.mean(times)
    by = hca_decode_bytes(w)
    gbs = by / (t / 1e3) / 1e9
    return {"workload": "hca_decode_1m_b8", "value": round(B / (t / 1e3), 1), "unit": "tok/s",
            "ms_per_step": round(t, 5), "step_bytes": by,
            "roofline": {"kernel": "hca_attn", "bound": "hbm", "achieved": round(gbs, 1),
                         "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4)},
            "compress": {"workload": "pool 8 x 1M bf16 tokens at m'=128 -> FP8",
                         "ms": round(t_comp, 3), "bytes": comp_bytes,
                         "achieved_gbs": round(comp_bytes / (t_comp / 1e3) / 1e9, 1)}}


def bench_indexer_variants(args, dev, flush, stream, hbm_peak):
    """The indexer of the 128K x 32 decode step on its write-path variants,
    each graph-replayed after an L2 flush: MXFP4 queries stored beforehand
    (the default), the same with the separate fp32 -> MXFP4 quantise launch
    in the step, bf16 queries quantised inside the indexer, and the exact
    E2M1 -> E4M3 expansion on the MXFP8 MMA (alone and with bf16 queries)."""
    import torch

    import compressed_sparse_attention_13_b200 as K
    from synth.workloads import WORKLOADS, draw_torch

    w = WORKLOADS[WORKLOAD]
    B, HI, dI, m, W = w.batch, w.HI, w.dI, w.m, w.W
    nb = w.n_ctx // m
    kv = draw_torch(w, "kI", device=dev).reshape(-1, dI)
    kI = K.empty_stored(K.MXFP4, B * nb, dI, device=dev)
    K.csa_quantize(kv, kI)
    del kv
    qf = draw_torch(w, "qI", device=dev).reshape(-1, dI).contiguous()
    qb = qf.to(torch.bfloat16)
    qs = K.empty_stored(K.MXFP4, B * HI, dI, device=dev)
    wt = draw_torch(w, "w", device=dev)
    q_pos = torch.full((B,), w.n_ctx, dtype=torch.int64, device=dev)
    scores = torch.empty(B, nb, dtype=torch.float32, device=dev)
    K.csa_quantize(qf, qs)
    prm = lambda f: K.params(m, W, w.k, w.H, w.d, HI, dI, w.scale, K.BF16, K.FP8_S64, K.MXFP4, flags=f)
    p0, pq, p8, pq8 = prm(0), prm(K.FLAG_QI_BF16), prm(K.FLAG_INDEXER_FP8), prm(K.FLAG_QI_BF16 | K.FLAG_INDEXER_FP8)
    cases = {
        "mxfp4_stored_query": lambda: K.indexer_score(p0, B, 1, qs, wt, kI, nb, q_pos, scores, nb),
        "quantise_then_mxfp4": lambda: (K.csa_quantize(qf, qs),
                                        K.indexer_score(p0, B, 1, qs, wt, kI, nb, q_pos, scores, nb)),
        "mxfp4_bf16_query_fused": lambda: K.indexer_score(pq, B, 1, K.Stored(K.BF16, qb), wt, kI, nb, q_pos,
                                                          scores, nb),
        "fp8_expanded": lambda: K.indexer_score(p8, B, 1, qs, wt, kI, nb, q_pos, scores, nb),
        "fp8_expanded_bf16_query": lambda: K.indexer_score(pq8, B, 1, K.Stored(K.BF16, qb), wt, kI, nb,
                                                           q_pos, scores, nb),
    }
    n_vis = max(0, min((w.n_ctx - W) // m, nb))
    key_bytes = B * n_vis * (dI // 2 + dI // 32)
    res = {"workload": WORKLOAD, "key_bytes": key_bytes}
    for name, fn in cases.items():
        t = statistics.mean(time_steps(graphed(fn), args.steps, args.warmup, flush, stream))
        res[name] = {"us": round(t * 1e3, 2), "key_gbs": round(key_bytes / (t / 1e3) / 1e9, 1),
                     "frac": round(key_bytes / (t / 1e3) / 1e9 / hbm_peak, 4)}
    assert K.csa_device_status(reset=True) == 0
    return res


def bench_shard(args, dev, flush, stream, world=8):
    """One 1M-token sequence (batch 1) split over `world` ranks, emulated on
    this GPU: every rank's phases are timed one by one (graph-replayed after
    an L2 flush), the per-GPU step is the slowest rank's select + attend plus
    the merge; the exchanges (two all-gathers of a few KB to a few MB) are not
    timed here (one GPU).  The unsharded call on the whole cache is timed
    beside it."""
    import torch

    import compressed_sparse_attention_13_b200 as K
    from compressed_sparse_attention_13_b200 import shard as SH
    from synth import tensor_torch

    N, H, d, HI, dI, W, k = 1 << 20, 64, 512, 64, 128, 128, 1024
    res = {"workload": f"one sequence at 1M tokens sharded over {world} emulated ranks", "ranks": world}
    t_of = lambda fn: statistics.mean(time_steps(graphed(fn), args.steps, args.warmup, flush, stream)) * 1e3

    def st(name, rows, width, fmt):
        v = tensor_torch(0, f"shard/{name}", (rows, width), device=dev)
        o = K.empty_stored(fmt, rows, width, device=dev)
        K.csa_quantize(v, o)
        return o

    q = tensor_torch(0, "shard/q", (1, H, d), dtype="bf16", device=dev)
    win = tensor_torch(0, "shard/win", (1, W, d), dtype="bf16", device=dev)
    sinks = tensor_torch(0, "shard/sinks", (H,), device=dev)
    q_pos = torch.full((1,), N, dtype=torch.int64, device=dev)
    raw_pos0 = q_pos - W + 1
    out = torch.empty(1, H, d, dtype=torch.bfloat16, device=dev)
    for kind, m in (("csa", 4), ("hca", 128)):
        nb = N // m
        p = K.params(m, W, k if kind == "csa" else 1, H, d, HI, dI, 1 / math.sqrt(d), K.BF16, K.FP8_S64, K.MXFP4)
        kv = st(f"{kind}/kv", nb, d, K.FP8_S64)
        kI = st("csa/kI", nb, dI, K.MXFP4) if kind == "csa" else None
        shards = SH.make_shards(kv, kI, 1, nb, world)
        r = {"entries": nb}
        if kind == "csa":
            qI = st("csa/qI", HI, dI, K.MXFP4)
            wt = tensor_torch(0, "shard/w", (1, HI), 0.1, device=dev)
            cand = [SH.csa_select(p, 1, qI, wt, sh, q_pos, dev) for sh in shards]
            all_s, all_i = torch.stack([c[0] for c in cand]), torch.stack([c[1] for c in cand])
            r["select_us"] = [round(t_of(lambda sh=sh: SH.csa_select(p, 1, qI, wt, sh, q_pos, dev)), 2)
                              for sh in shards]
            r["attend_us"] = [round(t_of(lambda sh=sh: SH.csa_attend(p, 1, q, all_s, all_i, sh, win, W, raw_pos0,
                                                                     q_pos, None, dev)), 2) for sh in shards]
            parts = [SH.csa_attend(p, 1, q, all_s, all_i, sh, win, W, raw_pos0, q_pos, None, dev) for sh in shards]
            ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, 1, 1, nb), dtype=torch.uint8, device=dev)
            sel = torch.empty(1, k, dtype=torch.int32, device=dev)
            r["unsharded_us"] = round(t_of(lambda: K.csa_decode(p, 1, q, qI, wt, kv, kI, nb, win, W, raw_pos0,
                                                                q_pos, sinks, out, sel, ws)), 2)
        else:
            r["attend_us"] = [round(t_of(lambda sh=sh: SH.hca_attend(p, 1, q, sh, win, W, raw_pos0, q_pos, dev)), 2)
                              for sh in shards]
            parts = [SH.hca_attend(p, 1, q, sh, win, W, raw_pos0, q_pos, dev) for sh in shards]
            ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, 1, 1, nb), dtype=torch.uint8, device=dev)
            r["unsharded_us"] = round(t_of(lambda: K.hca_attn(p, 1, 1, q, kv, nb, win, W, raw_pos0, q_pos, sinks,
                                                              out, ws)), 2)
        all_o, all_ml = torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts])
        r["merge_us"] = round(t_of(lambda: SH.merge(p, 1, all_o, all_ml, sinks, out)), 2)
        r["per_gpu_compute_us"] = round(max(r.get("select_us", [0.0])) + max(r["attend_us"]) + r["merge_us"], 2)
        r["exchange_bytes_per_rank"] = SH.exchange_bytes(1, k, H, d, csa=kind == "csa")
        res[kind] = r
        del kv, kI, shards, parts, all_o, all_ml
        torch.cuda.empty_cache()
    assert K.csa_device_status(reset=True) == 0
    return res


def _causal_pairs(T, m, W, k, t0=0):
    """(indexer (query, block) pairs, attended (query, item) pairs) of a chunk
    of T queries at positions t0 .. t0 + T - 1."""
    idx = att = 0
    for t in range(t0, t0 + T):
        ne = max(0, (t - W) // m)
        idx += ne
        att += min(k, ne) + min(W, t + 1)
    return idx, att


def bench_prefill(dev, flush, stream, bf16_peak):
    """CSA prefill, bf16, T = 8192 (pool the chunk, indexer, top-k, attention)."""
    import torch

    import compressed_sparse_attention_13_b200 as K
    from synth.workloads import WORKLOADS, draw_torch

    w = WORKLOADS["csa_prefill_8k_bf16"]
    B, T, H, d, HI, dI, m, W, k = w.batch, w.n_ctx, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = T // m
    p = K.params(m, W, k, H, d, HI, dI, w.scale, K.BF16, K.BF16, K.BF16)
    t_ = {n: draw_torch(w, n, device=dev) for n in ("x", "z", "bias", "q", "qI", "kI", "w", "sinks")}
    kv = K.empty_stored(K.BF16, B * nb, d, device=dev)
    qI, kI = K.Stored(K.BF16, t_["qI"]), K.Stored(K.BF16, t_["kI"])
    out = torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev)
    sel = torch.empty(B, T, k, dtype=torch.int32, device=dev)
    ws = torch.empty(K.csa_workspace_size(p, K.OP_PREFILL, B, T, nb), dtype=torch.uint8, device=dev)
    fn = lambda: K.csa_prefill(p, B, T, 0, t_["x"], T, 0, t_["z"], t_["bias"], t_["q"], qI, t_["w"], kv,
                               kI, nb, t_["sinks"], out, sel, ws)
    times = time_steps(fn, 5, 3, flush, stream)
    t = statistics.median(times)
    pi, pa = _causal_pairs(T, m, W, k)
    f_idx, f_att = B * pi * 2 * HI * dI, B * pa * 4 * H * d
    flops = f_idx + f_att
    tf = flops / (t / 1e3) / 1e12
    # the stages alone, on the entries and selections the chunk produced
    scores = torch.empty(B * T, nb, dtype=torch.float32, device=dev)
    q_pos = torch.arange(T, dtype=torch.int64, device=dev).repeat(B)
    pos0 = torch.zeros(B, dtype=torch.int64, device=dev)
    stages = {
        "indexer_score": lambda: K.indexer_score(p, B, T, qI, t_["w"], kI, nb, q_pos, scores, nb),
        "topk_select": lambda: K.topk_select(p, B, T, scores, nb, nb, q_pos, sel),
        "sparse_mqa_attn": lambda: K.sparse_mqa_attn(p, B, T, t_["q"], kv, nb, sel, t_["x"], T, pos0, q_pos,
                                                     t_["sinks"], out, ws),
    }
    st = {n: statistics.median(time_steps(f, 5, 3, flush, stream)) for n, f in stages.items()}
    assert K.csa_device_status(reset=True) == 0
    tf_idx = f_idx / (st["indexer_score"] / 1e3) / 1e12
    tf_att = f_att / (st["sparse_mqa_attn"] / 1e3) / 1e12
    roof = lambda kern, a: {"kernel": kern, "bound": "tensor", "achieved": round(a, 2), "peak": bf16_peak,
                            "unit": "TFLOP/s", "frac": round(a / bf16_peak, 4)}
    return {"workload": "csa_prefill_8k_bf16", "value": round(B * T / (t / 1e3), 1), "unit": "tok/s",
            "ms_per_step": round(t, 3), "flop": flops,
            "roofline": roof("csa_prefill (all stages)", tf),
            "stages_ms": {n: round(v, 4) for n, v in st.items()},
            "stage_roofline": {"indexer_score": roof("indexer_bf16_tc_kernel", tf_idx),
                               "sparse_mqa_attn": roof("attn_tc_kernel<1> (bf16 entries)", tf_att)}}


def bench_stack(dev, flush, stream, hbm_peak, bf16_peak):
    """Four layers CSA, HCA, CSA, HCA on one sequence at 1M context: a prior
    cache of 1,044,480 tokens, a 4096-token prefill chunk, then 256 decode steps
    with incremental pooling (every 4 tokens for CSA, 128 for HCA)."""
    import math

    import torch

    import compressed_sparse_attention_13_b200 as K
    from compressed_sparse_attention_13_b200.stack import Layer, LayerSpec
    from synth import tensor_torch

    PRIOR, CHUNK, STEPS, TOPK, W, H, d, HI, dI = 1_044_480, 4096, 256, 1024, 128, 64, 512, 64, 128
    scale = 1 / math.sqrt(d)
    n_new = CHUNK + STEPS
    g = lambda li, name, shape, std=1.0, dt="f32": tensor_torch(0, f"stack_c4/{li}/{name}", shape, std, dt,
                                                            device=dev)
    layers = []
    for li, kind in enumerate(["csa", "hca", "csa", "hca"]):
        m = 4 if kind == "csa" else 128
        p = K.params(m, W, TOPK if kind == "csa" else 1, H, d, HI, dI, scale, K.BF16, K.FP8_S64, K.MXFP4)
        L = Layer(LayerSpec(kind, p, PRIOR, n_new), dev)
        K.csa_quantize(g(li, "prior_kv", (PRIOR // m, d)), K.Stored(K.FP8_S64, L.kv.data[:PRIOR // m],
                                                                    L.kv.scales[:PRIOR // m]))
        L.set_prior_window(g(li, "x_prior", (W - 1, d), dt="bf16"))
        inp = dict(kind=kind, L=L, x=g(li, "x", (n_new, d), dt="bf16"), z=g(li, "z", (n_new, d), dt="bf16"),
                   bias=g(li, "bias", (m, d), 0.1), q=g(li, "q", (n_new, H, d), dt="bf16"),
                   sinks=g(li, "sinks", (H,)), out=torch.empty(n_new, H, d, dtype=torch.bfloat16, device=dev),
                   sel=torch.empty(n_new, TOPK, dtype=torch.int32, device=dev))
        if kind == "csa":
            K.csa_quantize(g(li, "prior_kI", (PRIOR // m, dI)),
                           K.Stored(K.MXFP4, L.kI.data[:PRIOR // m], L.kI.scales[:PRIOR // m]))
            qI = K.empty_stored(K.MXFP4, n_new * HI, dI, device=dev)
            K.csa_quantize(g(li, "qI", (n_new * HI, dI)), qI)
            inp.update(xI=g(li, "xI", (n_new, dI), dt="bf16"), zI=g(li, "zI", (n_new, dI), dt="bf16"),
                       biasI=g(li, "biasI", (m, dI), 0.1), qI=qI, w=g(li, "w", (n_new, HI), 0.1))
        layers.append(inp)
    torch.cuda.synchronize()

    def rows(st, a, b):
        return K.Stored(st.fmt, st.data[a:b], st.scales[a:b])

    # prefill chunk (all four layers): one untimed pass first (it loads the
    # kernels and lets the allocator reserve the prefill workspaces), then the
    # layers are put back to the state before the chunk and the pass is timed
    # (re-appending the same tokens rewrites the same rows and entries)
    before = [ly["L"].state() for ly in layers]

    def prefill_pass():
        for ly in layers:
            L, csa = ly["L"], ly["kind"] == "csa"
            L.append(ly["x"][:CHUNK], ly["z"][:CHUNK], ly["xI"][:CHUNK] if csa else None,
                     ly["zI"][:CHUNK] if csa else None)
            L.prefill(CHUNK, ly["q"][:CHUNK], rows(ly["qI"], 0, CHUNK * HI) if csa else None,
                      ly["w"][:CHUNK] if csa else None, ly["sinks"], ly["out"][:CHUNK],
                      ly["sel"][:CHUNK] if csa else None, ly["bias"], ly.get("biasI"))

    prefill_pass()
    torch.cuda.synchronize()
    for ly, st in zip(layers, before):
        ly["L"].restore(st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush.zero_()
    e0.record(stream)
    prefill_pass()
    e1.record(stream)
    torch.cuda.synchronize()
    t_prefill = e0.elapsed_time(e1)
    assert K.csa_device_status(reset=True) == 0
    # decode steps: one eager pass (loads every kernel), then the same steps
    # captured once in a graph and replayed (appends and pooling rewrite the
    # same rows, so a replay recomputes the same outputs)
    qpos = torch.arange(PRIOR + CHUNK, PRIOR + n_new, dtype=torch.int64, device=dev)
    start = [ly["L"].state() for ly in layers]

    def steps():
        for s in range(STEPS):
            i = CHUNK + s
            for ly in layers:
                L, csa = ly["L"], ly["kind"] == "csa"
                L.append(ly["x"][i:i + 1], ly["z"][i:i + 1], ly["xI"][i:i + 1] if csa else None,
                         ly["zI"][i:i + 1] if csa else None)
                L.decode(ly["q"][i], rows(ly["qI"], i * HI, (i + 1) * HI) if csa else None,
                         ly["w"][i] if csa else None, ly["sinks"], ly["out"][i], ly["sel"][i] if csa else None,
                         ly["bias"], ly.get("biasI"), q_pos=qpos[s:s + 1])

    steps()
    torch.cuda.synchronize()
    assert K.csa_device_status(reset=True) == 0
    for ly, st in zip(layers, start):
        ly["L"].restore(st)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        steps()
    dec = []
    for _ in range(3):
        flush.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        dec.append(e0.elapsed_time(e1))
    assert K.csa_device_status(reset=True) == 0
    del graph
    t_dec = statistics.median(dec) / STEPS
    # algorithmic bytes of one decode step (four layers, at the middle step):
    # CSA: 68 B per visible indexer key + the query and weights, the selected
    # FP8 entries and the bf16 window; HCA: every visible FP8 entry + the window
    by = 0
    for ly in layers:
        t = PRIOR + CHUNK + STEPS // 2
        if ly["kind"] == "csa":
            ne = (t - W) // 4
            by += ne * (dI // 2 + dI // 32) + HI * (dI // 2 + dI // 32 + 4) + TOPK * (d + 4 * d // 64) + W * d * 2
        else:
            ne = (t - W) // 128
            by += ne * (d + 4 * d // 64) + W * d * 2
    gbs = by / (t_dec / 1e3) / 1e9
    # work of the prefill chunk: the MXFP4 indexer (2 HI dI per visible
    # (query, block) pair) and the bf16 attention (4 H d per attended item)
    f_idx = f_att = 0
    for ly in layers:
        m = 4 if ly["kind"] == "csa" else 128
        for t in range(PRIOR, PRIOR + CHUNK):
            ne = max(0, (t - W) // m)
            if ly["kind"] == "csa":
                f_idx += ne * 2 * HI * dI
                f_att += (min(TOPK, ne) + W) * 4 * H * d
            else:
                f_att += (ne + W) * 4 * H * d
    fp4_peak = 4 * bf16_peak      # derived: the FP4 tensor rate is 4x the measured bf16 rate
    roof_ms = (f_idx / fp4_peak + f_att / bf16_peak) / 1e12 * 1e3
    return {"workload": "csa_hca_stack_1m_4layers", "prior_tokens": PRIOR, "chunk": CHUNK, "decode_steps": STEPS,
            "prefill_ms": round(t_prefill, 3), "prefill_tok_s": round(CHUNK / (t_prefill / 1e3), 1),
            "prefill_flop": {"indexer_mxfp4": f_idx, "attention_bf16": f_att},
            "prefill_tflops": round((f_idx + f_att) / (t_prefill / 1e3) / 1e12, 1),
            "prefill_roofline": {"bound": "tensor", "roofline_ms": round(roof_ms, 3),
                                 "frac": round(roof_ms / t_prefill, 4),
                                 "peaks_tflops": {"bf16": bf16_peak, "fp4": fp4_peak},
                                 "note": "frac = time at the tensor peaks (indexer at the derived FP4 "
                                         "peak, attention at the measured bf16 peak) / measured time"},
            "decode_us_per_step": round(t_dec * 1e3, 2), "decode_tok_s": round(1 / (t_dec / 1e3), 1),
            "decode_step_bytes": by,
            "roofline": {"kernel": "decode step (4 layers)", "bound": "hbm", "achieved": round(gbs, 1),
                         "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4)}}


def bench_schedule(dev, flush, stream, hbm_peak, steps=8):
    """Decode steps through the DeepSeek-V4-Pro layer schedule as synthetic
    layers (no weights): 61 layers -- HCA at layers 0-1, then CSA and HCA
    alternating -- and the MTP block with the sliding window only, one
    sequence with a prior cache of 1,044,480 tokens per layer.  Each step
    appends the new token to every layer (pooling completed blocks) and
    attends with it; the steps are replayed from one CUDA graph."""
    import math

    import torch

    import compressed_sparse_attention_13_b200 as K
    from compressed_sparse_attention_13_b200.stack import Layer, LayerSpec, v4_pro_schedule
    from synth import tensor_torch

    PRIOR, TOPK, W, H, d, HI, dI = 1_044_480, 1024, 128, 64, 512, 64, 128
    scale = 1 / math.sqrt(d)
    g = lambda li, name, shape, std=1.0, dt="f32": tensor_torch(0, f"schedule/{li}/{name}", shape, std, dt,
                                                            device=dev)
    kinds = v4_pro_schedule()
    layers = []
    for li, kind in enumerate(kinds):
        m = 128 if kind == "hca" else 4
        p = K.params(m, W, TOPK if kind == "csa" else 1, H, d, HI, dI, scale, K.BF16, K.FP8_S64, K.MXFP4)
        L = Layer(LayerSpec(kind, p, PRIOR, steps), dev)
        if L.kv is not None:
            K.csa_quantize(g(li, "prior_kv", (PRIOR // m, d)), K.Stored(K.FP8_S64, L.kv.data[:PRIOR // m],
                                                                        L.kv.scales[:PRIOR // m]))
        L.set_prior_window(g(li, "x_prior", (W - 1, d), dt="bf16"))
        ly = dict(kind=kind, L=L, x=g(li, "x", (steps, d), dt="bf16"), z=g(li, "z", (steps, d), dt="bf16"),
                  bias=g(li, "bias", (m, d), 0.1), q=g(li, "q", (steps, H, d), dt="bf16"),
                  sinks=g(li, "sinks", (H,)), out=torch.empty(steps, H, d, dtype=torch.bfloat16, device=dev),
                  sel=torch.empty(steps, TOPK, dtype=torch.int32, device=dev))
        if kind == "csa":
            K.csa_quantize(g(li, "prior_kI", (PRIOR // m, dI)),
                           K.Stored(K.MXFP4, L.kI.data[:PRIOR // m], L.kI.scales[:PRIOR // m]))
            qI = K.empty_stored(K.MXFP4, steps * HI, dI, device=dev)
            K.csa_quantize(g(li, "qI", (steps * HI, dI)), qI)
            ly.update(xI=g(li, "xI", (steps, dI), dt="bf16"), zI=g(li, "zI", (steps, dI), dt="bf16"),
                      biasI=g(li, "biasI", (m, dI), 0.1), qI=qI, w=g(li, "w", (steps, HI), 0.1))
        layers.append(ly)
    torch.cuda.synchronize()
    qpos = torch.arange(PRIOR, PRIOR + steps, dtype=torch.int64, device=dev)

    def run():
        for s_ in range(steps):
            for ly in layers:
                L, csa = ly["L"], ly["kind"] == "csa"
                L.append(ly["x"][s_:s_ + 1], ly["z"][s_:s_ + 1], ly["xI"][s_:s_ + 1] if csa else None,
                         ly["zI"][s_:s_ + 1] if csa else None)
                qI = K.Stored(K.MXFP4, ly["qI"].data[s_ * HI:(s_ + 1) * HI],
                              ly["qI"].scales[s_ * HI:(s_ + 1) * HI]) if csa else None
                L.decode(ly["q"][s_], qI, ly["w"][s_] if csa else None, ly["sinks"], ly["out"][s_],
                         ly["sel"][s_] if csa else None, ly["bias"], ly.get("biasI"), q_pos=qpos[s_:s_ + 1])

    start = [ly["L"].state() for ly in layers]
    run()
    torch.cuda.synchronize()
    assert K.csa_device_status(reset=True) == 0
    for ly, st in zip(layers, start):
        ly["L"].restore(st)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(3):
        flush.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / steps)
    assert K.csa_device_status(reset=True) == 0
    del graph
    t = statistics.median(times)
    # algorithmic bytes of one step over all blocks (as in the four-layer stack)
    tq = PRIOR + steps // 2
    by = 0
    for ly in layers:
        if ly["kind"] == "csa":
            ne = (tq - W) // 4
            by += ne * (dI // 2 + dI // 32) + HI * (dI // 2 + dI // 32 + 4) + TOPK * (d + 4 * d // 64) + W * d * 2
        elif ly["kind"] == "hca":
            by += (tq - W) // 128 * (d + 4 * d // 64) + W * d * 2
        else:
            by += W * d * 2
    gbs = by / (t / 1e3) / 1e9
    counts = {k_: kinds.count(k_) for k_ in ("csa", "hca", "window")}
    return {"workload": "v4_pro_schedule_61_layers_mtp_1m", "layers": counts, "prior_tokens": PRIOR,
            "decode_steps": steps, "decode_us_per_step": round(t * 1e3, 1), "decode_tok_s": round(1e3 / t, 1),
            "step_bytes": by,
            "roofline": {"kernel": "decode step (61 layers + MTP)", "bound": "hbm", "achieved": round(gbs, 1),
                         "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4)}}


def run_case(name, reps=3):
    """One small named workload, run `reps` times, for profiling a kernel
    under ncu (the bench's own timed region is not involved).  Inputs are
    seeded; device memory stays at a few GB at most."""
    import torch

    import compressed_sparse_attention_13_b200 as K
    from synth import tensor_torch
    from synth.workloads import WORKLOADS, draw_torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if name == "decode_128k_b32":       # indexer, top-k, sparse attention (one csa_decode)
        w = WORKLOADS[WORKLOAD]
        S = setup_csa_decode(w, dev)
        fn = lambda: csa_decode_call(w, S)
    elif name == "hca_1m_b8":           # HCA attention over 8 x 8192 FP8 entries (+ the split combine)
        w = WORKLOADS["hca_decode_1m_b8"]
        B, N, H, d, m, W = w.batch, w.n_ctx, w.H, w.d, w.m, w.W
        nb = N // m
        p = K.params(m, W, 1, H, d, 1, 32, w.scale, K.BF16, K.FP8_S64, K.MXFP4)
        kv = K.empty_stored(K.FP8_S64, B * nb, d, device=dev)
        K.csa_quantize(tensor_torch(0, "case/hca/kv", (B * nb, d), device=dev), kv)
        q = tensor_torch(0, "case/hca/q", (B, H, d), dtype="bf16", device=dev)
        win = tensor_torch(0, "case/hca/win", (B, W, d), dtype="bf16", device=dev)
        sinks = tensor_torch(0, "case/hca/sinks", (H,), device=dev)
        q_pos = torch.full((B,), N, dtype=torch.int64, device=dev)
        out = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, B, 1, nb), dtype=torch.uint8, device=dev)
        fn = lambda: K.hca_attn(p, B, 1, q, kv, nb, win, W, q_pos - W + 1, q_pos, sinks, out, ws)
    elif name == "pool_hca":            # pooling 8 x 65,536 bf16 tokens at m' = 128 into FP8 entries
        B, N, d, m = 8, 65536, 512, 128
        p = K.params(m, 128, 1, 64, d, 1, 32, 1.0, K.BF16, K.FP8_S64, K.MXFP4)
        x = tensor_torch(0, "case/pool/x", (B * N, d), dtype="bf16", device=dev)
        z = tensor_torch(0, "case/pool/z", (B * N, d), dtype="bf16", device=dev)
        bias = tensor_torch(0, "case/pool/bias", (m, d), 0.1, device=dev)
        kv = K.empty_stored(K.FP8_S64, B * N // m, d, device=dev)
        fn = lambda: K.csa_compress(p, d, x, z, bias, B * N, kv)
    elif name == "prefill_topk":        # top-k of the 8K bf16 prefill: 8192 rows of up to 2048 scores
        w = WORKLOADS["csa_prefill_8k_bf16"]
        T, nb = w.n_ctx, w.n_ctx // w.m
        p = K.params(w.m, w.W, w.k, w.H, w.d, w.HI, w.dI, w.scale, K.BF16, K.BF16, K.BF16)
        scores = tensor_torch(0, "case/topk/s", (T, nb), device=dev)
        q_pos = torch.arange(T, dtype=torch.int64, device=dev)
        sel = torch.empty(T, w.k, dtype=torch.int32, device=dev)
        fn = lambda: K.topk_select(p, 1, T, scores, nb, nb, q_pos, sel)
    elif name == "decode_128k_b32_fp8_indexer":   # the indexer's exact E2M1 -> E4M3 variant on C2
        w = WORKLOADS[WORKLOAD]
        S = setup_csa_decode(w, dev)
        S["p"] = K.params(w.m, w.W, w.k, w.H, w.d, w.HI, w.dI, w.scale, K.BF16, K.FP8_S64, K.MXFP4,
                          flags=K.FLAG_INDEXER_FP8)
        fn = lambda: csa_decode_call(w, S)
    elif name == "prefill_8k_attn":     # the bf16 prefill's attention stage (8192 rows, bf16 entries)
        w = WORKLOADS["csa_prefill_8k_bf16"]
        T, nb, H, d = w.n_ctx, w.n_ctx // w.m, w.H, w.d
        p = K.params(w.m, w.W, w.k, H, d, w.HI, w.dI, w.scale, K.BF16, K.BF16, K.BF16)
        kv = K.Stored(K.BF16, tensor_torch(0, "case/pa/kv", (nb, d), dtype="bf16", device=dev))
        q = tensor_torch(0, "case/pa/q", (T, H, d), dtype="bf16", device=dev)
        raw = tensor_torch(0, "case/pa/x", (1, T, d), dtype="bf16", device=dev)
        sinks = tensor_torch(0, "case/pa/sinks", (H,), device=dev)
        q_pos = torch.arange(T, dtype=torch.int64, device=dev)
        # a valid selection: the k most recent eligible entries of each row
        e = torch.arange(w.k, device=dev)[None, :]
        ne = torch.clamp((q_pos[:, None] - w.W) // w.m, min=0)
        idx = torch.where(e < ne, ne - 1 - e, torch.full_like(e, -1)).flip(1).to(torch.int32)
        idx = torch.sort(torch.where(idx < 0, torch.full_like(idx, 1 << 30), idx), dim=1).values
        idx = torch.where(idx == (1 << 30), torch.full_like(idx, -1), idx).contiguous()
        out = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(K.csa_workspace_size(p, K.OP_SPARSE_ATTN, 1, T, 0), dtype=torch.uint8, device=dev)
        pos0 = torch.zeros(1, dtype=torch.int64, device=dev)
        fn = lambda: K.sparse_mqa_attn(p, 1, T, q, kv, nb, idx, raw, T, pos0, q_pos, sinks, out, ws)
    else:
        raise SystemExit(f"unknown case {name}")
    torch.cuda.empty_cache()   # only the case's own tensors stay on the device
    for _ in range(reps):
        fn()
    torch.cuda.synchronize()
    assert K.csa_device_status(reset=True) == 0
    print(json.dumps({"case": name, "reps": reps, "ok": True}))


# ------------------------------------------------------------- CPU oracle
def _oracle_sample(w, seqs):
    """Host inputs for the sampled sequences, quantised by the oracle."""
    import oracle
    from synth.workloads import draw_np
    sinks = draw_np(w, "sinks")
    rows = []
    for b in seqs:
        v = {n: draw_np(w, n, b) for n in ("q", "qI", "w", "kv", "kI", "window")}
        rows.append(dict(q=oracle.Stored(oracle.BF16, v["q"]), kv=oracle.quantize_fp8_s64(v["kv"]),
                         qI=oracle.quantize_mxfp4(v["qI"]), w=v["w"][None], kI=oracle.quantize_mxfp4(v["kI"]),
                         win=oracle.Stored(oracle.BF16, v["window"])))
    return rows, sinks


def _oracle_step(w, rows, sinks, threads):
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    t = w.n_ctx

    def one(r):
        return oracle.csa(r["q"], r["kv"], r["qI"], r["w"], r["kI"], r["win"], t - w.W + 1, sinks,
                          [t], w.H, w.HI, w.m, w.W, w.k, w.scale, 1)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, rows))


def host_threads() -> int:
    """Host cores this process may run on (all of them for the CPU baseline)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, seconds):
    """The oracle, as it stands (its source compiled -O3 -march=native with
    OpenMP for this host), on all host cores: one sequence per thread,
    repeated until about `seconds` of CPU work."""
    import oracle
    oracle.use_native()
    threads = host_threads()
    n = min(threads, w.batch)
    rows, sinks = _oracle_sample(w, list(range(n)))
    t0 = time.perf_counter()
    reps = 0
    while True:
        _oracle_step(w, rows, sinks, n)
        reps += 1
        el = time.perf_counter() - t0
        if el * n >= seconds or el > seconds:
            break
    return {"value": round(reps * n / el, 3), "unit": "tok/s", "cores": n, "host_cores": os.cpu_count(),
            "threads": n, "kind": "oracle", "build": "g++ -O3 -march=native -fopenmp",
            "sample": f"{reps} x {n} sequences of the {w.batch}-sequence batch (one per thread), "
                      f"{el:.1f} s wall"}


def run_reference(args):
    """The CPU oracle timed as the reference arm on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from synth.workloads import WORKLOADS
    oracle.use_native()
    w = WORKLOADS[WORKLOAD]
    threads = host_threads()
    n = min(threads, w.batch)
    rows, sinks = _oracle_sample(w, list(range(n)))
    for _ in range(args.warmup):
        _oracle_step(w, rows, sinks, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(w, rows, sinks, n)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    res = {"metric": METRIC, "value": round(value, 3), "unit": "tok/s", "impl": "reference",
           "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1))",
           "config": {"workload": WORKLOAD, "batch": w.batch, "context": w.n_ctx, "heads": w.H,
                      "head_dim": w.d, "top_k": w.k, "window": w.W},
           "cpu_baseline": {"value": round(value, 3), "unit": "tok/s", "cores": n,
                            "host_cores": os.cpu_count(), "threads": n, "kind": "oracle",
                            "build": "g++ -O3 -march=native -fopenmp",
                            "sample": f"each step: {n} of the {w.batch} sequences, one per thread"},
           "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the extra legs")
    ap.add_argument("--legs", default="", help="extra legs to run, comma-separated among hca, indexer, shard, "
                    "prefill, stack, schedule (default: all)")
    ap.add_argument("--only-legs", default="", help="run only these extra legs (comma-separated among "
                    "hca, indexer, shard, prefill, stack, schedule) and print their results, without the main line")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--case", default="", help="run one small named workload (decode_128k_b32, hca_1m_b8, "
                    "pool_hca, prefill_topk) a few times, for profiling, and exit")
    args = ap.parse_args()
    if args.case:
        run_case(args.case)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
