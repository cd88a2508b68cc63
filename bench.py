"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME] [--no-detail]

A step is one forward of the workload for every normalizer the workload names
(the Qwen3-8B-shaped prefill layer by default: B=2, Hq=32, Hkv=8 (GQA 4:1),
T=4096, d=128, causal; softmax and softmax1).  Inputs are seeded synthetic
bf16 tensors resident in HBM before timing starts; L2 is flushed (a 256 MiB
write) before every timed step and the flush is outside the per-step CUDA
events.  The headline value is useful TFLOP/s by the accounting rule of
"Attention variants" (TensorCAD, "What the engine does today"):
4 * T_eff * head_dim FLOPs per query row and head, halved when causal.

Under torchrun each rank runs its own batch (independent problems, weak
scaling, no data-path collective); the time is the max over ranks.

--impl reference times the float64 CPU oracle on a bounded sample of the same
workload on the host cores (the reference arm of this benchmark).
"""

import argparse
import json
from dataclasses import replace
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}


def peak_label(key, extra=""):
    """'of measured <key>' or 'of fallback <key>', by where the peaks came
    from (MEASURED_PEAKS.json, else the pool's earlier measurement)."""
    return f"of {load_peaks()[1]} {key}{extra}"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return PEAKS_FALLBACK, "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv",
                 "-i", str(self.index), "-lms", "20"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
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
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f.read().splitlines()[1:]:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm = float(parts[1].split()[0])
                    smax = float(parts[2].split()[0])
                except ValueError:
                    continue
                rows.append((sm, smax, parts[5:9]))
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, x in enumerate(r)
                          if x.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


class NvmlSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML
    every ``period_s`` on a background thread (read-only queries), so that
    even a timed region of a few milliseconds holds several samples.  Falls
    back to the nvidia-smi sampler when NVML is not usable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device, period_s=0.002):
        self.device = device
        self.period = period_s
        self.rows = []
        self.thread = None
        self.fallback = None

    def start(self):
        import threading
        try:
            import pynvml as N
            import torch
            N.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(self.device)
            h = N.nvmlDeviceGetHandleByIndex(idx)
            smax = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            bits = [(n, getattr(N, a)) for n, a in self.REASONS]
        except Exception:
            self.fallback = ClockSampler(int(getattr(self.device, "index", 0) or 0))
            self.fallback.start()
            return
        self.stop_evt = threading.Event()

        def loop():
            while not self.stop_evt.is_set():
                try:
                    sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                    rs = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.rows.append((sm, smax, [n for n, b in bits if rs & b]))
                except Exception:
                    pass
                self.stop_evt.wait(self.period)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.fallback is not None:
            return self.fallback.stop()
        if self.thread is None:
            return None
        self.stop_evt.set()
        self.thread.join(timeout=5)
        if not self.rows:
            return None
        return {"sm_mhz": statistics.median(r[0] for r in self.rows),
                "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": sorted({x for r in self.rows for x in r[2]}),
                "samples": len(self.rows), "source": "nvml"}


# --------------------------------------------------------------------------
# native arm
# --------------------------------------------------------------------------
def kv_bytes_decode(x, w):
    lens = x["seqlens"].long()
    return int(lens.sum()) * w.Hkv * (w.d + w.dv) * 2 + \
        2 * w.B * w.Hq * w.Tq * w.d * 2


class Runner:
    """Preallocated arguments and scratch for one workload on one device."""

    def __init__(self, w, dev, seed_offset=0):
        import torch
        from alternative_normalizers_b200 import binding
        from alternative_normalizers_b200.workloads import make_inputs
        self.w = w
        self.binding = binding
        x = make_inputs(w, seed=w.seed + seed_offset)
        self.host = x
        self.x = {k: v.to(dev) for k, v in x.items()}
        if w.paged:
            self.out = torch.empty(w.B, w.Hq, w.Tq, w.dv, dtype=torch.bfloat16,
                                   device=dev)
            self.max_len = w.len_range[1]
        else:
            self.out = torch.empty(w.B, w.Hq, w.Tq, w.dv, dtype=torch.bfloat16,
                                   device=dev)
        self.stat = torch.empty(w.B, w.Hq, w.Tq, dtype=torch.float32, device=dev)
        self.args = {}
        self.ws = {}
        stream = torch.cuda.current_stream(dev).cuda_stream
        for n in w.normalizers:
            a = self._args(n, self.x, self.out, self.stat, stream)
            need = binding.nattn_workspace_size(a)
            if need:
                self.ws[n] = torch.empty(need, dtype=torch.uint8, device=dev)
                a.workspace, a.workspace_bytes = self.ws[n].data_ptr(), need
            self.args[n] = a

    def _args(self, n, x, out, stat, stream):
        w = self.w
        if w.paged:
            return self.binding.build_args(
                x["q"], x["k_pool"], x["v_pool"], out, stat, None,
                normalizer=n, causal=w.causal, window=w.window,
                softcap=w.softcap, scale=w.scale, block_table=x["block_table"],
                seqlens=x["seqlens"], page_size=w.page_size,
                max_seqlen=self.max_len, stream=stream)
        return self.binding.build_args(
            x["q"], x["k"], x["v"], out, stat, None, normalizer=n,
            causal=w.causal, window=w.window, softcap=w.softcap,
            scale=w.scale, stream=stream)

    def call(self, n):
        rc = self.binding.nattn_fwd_ex(self.args[n])
        if rc != 0:
            raise RuntimeError(f"nattn_fwd_ex({n}) failed: {rc}")

    def units(self):
        """Useful FLOPs (prefill) or K/V bytes (decode) of one normalizer."""
        if self.w.paged:
            return kv_bytes_decode(self.host, self.w)
        return self.w.useful_flops()


# this library's kernels per call: the pair kernel for softmax / softmax1;
# threshold pass, apply, wide and row-wise kernels for the sparse ones (the
# last two exit at once when no row overflowed)
LAUNCHES = {"softmax": 1, "softmax1": 1, "sparsemax": 4, "entmax15": 4}

# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of the current kernel (the profile summary named beside it).
# An entry is removed whenever the kernel changes after its capture.
NCU_TRAFFIC = {
    ("qwen3_8b_prefill", "softmax"): (
        131_220_224, "profiles/prefill_pair_qwen3_8b_softmax.md"),
}
# decode: split kernel and combine; sparse: score pass, threshold kernel,
# apply pass and combine
LAUNCHES_DECODE = {"softmax": 2, "softmax1": 2, "sparsemax": 4, "entmax15": 4}


def shard_seed(w, rank):
    """Seed of rank `rank`'s batch: every GPU runs an independent problem of
    the same shape (weak scaling; the path has no exchange step)."""
    return w.seed + rank


def max_over_ranks(ms, dist, device):
    """The slowest rank's time: the job finishes when the last rank does."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_runner(r, steps, warmup, flush):
    """Per-normalizer average kernel time (ms) over `steps` timed steps, each
    preceded by an L2 flush outside the events."""
    import torch
    for _ in range(warmup):
        for n in r.w.normalizers:
            r.call(n)
    torch.cuda.synchronize()
    ev = {n: [] for n in r.w.normalizers}
    for _ in range(steps):
        for n in r.w.normalizers:
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(
                enable_timing=True)
            s.record()
            r.call(n)
            e.record()
            ev[n].append((s, e))
    torch.cuda.synchronize()
    return {n: sum(s.elapsed_time(e) for s, e in v) / len(v)
            for n, v in ev.items()}


def e2e_measure(r, steps, dev):
    """Same metric through the C ABI with host buffers: every step copies the
    inputs from pinned host memory and reads the output and row statistics
    back, all inside the timed region."""
    import torch
    host = {k: v.pin_memory() for k, v in r.host.items()}
    dst = {k: torch.empty_like(v, device=dev) for k, v in r.host.items()}
    out_h = torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory()
    stat_h = torch.empty(r.stat.shape, dtype=r.stat.dtype).pin_memory()
    stream = torch.cuda.current_stream(dev).cuda_stream
    args = {n: r._args(n, dst, r.out, r.stat, stream) for n in r.w.normalizers}
    for n, a in args.items():
        if n in r.ws:
            a.workspace = r.ws[n].data_ptr()
            a.workspace_bytes = r.ws[n].numel()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h.numel() * out_h.element_size() + stat_h.numel() * 4

    def one():
        for k in host:
            dst[k].copy_(host[k], non_blocking=True)
        for n in r.w.normalizers:
            if r.binding.nattn_fwd_ex(args[n]) != 0:
                raise RuntimeError("nattn_fwd_ex failed")
            out_h.copy_(r.out, non_blocking=True)
            stat_h.copy_(r.stat, non_blocking=True)

    one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        one()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    nn = len(r.w.normalizers)
    return ms, h2d, d2h * nn


def e2e_chunks(B, Hkv):
    """(batch entry, first KV head, end KV head) of each chunk of the
    end-to-end loop: every batch entry, cut into two halves of its KV heads
    (one piece when Hkv is odd).  A chunk's q rows (its KV heads' query
    heads), k/v rows and out/row_stat rows are contiguous in the dense
    layouts."""
    gs = Hkv // 2 if Hkv % 2 == 0 else Hkv
    return [(b, g0, g0 + gs) for b in range(B) for g0 in range(0, Hkv, gs)]


def e2e_measure_dense(r, steps, dev):
    """The same metric through the C ABI with host buffers, as a serving loop
    would run it: every step copies its inputs from pinned host memory and
    reads every normalizer's output and row statistics back, all inside the
    timed region.  The work is cut into chunks of (batch entry, half of the
    KV heads) whose q/k/v/out slices are contiguous; one stream copies the
    chunks in, one runs nattn_fwd_ex on each chunk as soon as its inputs have
    landed, one copies each chunk's results out as soon as they are done, so
    the host-to-device copies, the products and the device-to-host copies
    overlap (PCIe runs both directions at once).  Outputs alternate between
    two device buffers so that a step's products never wait for the
    previous step's copies out; a chunk's next inputs wait until every
    normalizer of the step has read them.  Returns (ms per step, bytes in,
    bytes out, max |difference| from one unchunked call per normalizer)."""
    import torch
    w = r.w
    grp = w.Hq // w.Hkv
    chunks = e2e_chunks(w.B, w.Hkv)
    host = {k: r.host[k].pin_memory() for k in ("q", "k", "v")}
    din = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    norms = list(w.normalizers)
    outs = [[torch.empty(r.out.shape, dtype=r.out.dtype, device=dev) for _ in norms]
            for _ in range(2)]
    stats = [[torch.empty(r.stat.shape, dtype=torch.float32, device=dev) for _ in norms]
             for _ in range(2)]
    out_h = [torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory() for _ in norms]
    stat_h = [torch.empty(r.stat.shape, dtype=torch.float32).pin_memory() for _ in norms]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def qs(t, c):
        b, g0, g1 = c
        return t[b:b + 1, g0 * grp:g1 * grp]

    def kvs(t, c):
        b, g0, g1 = c
        return t[b:b + 1, g0:g1]

    args, keep = {}, []
    for par in range(2):
        for ni, n in enumerate(norms):
            for ci, c in enumerate(chunks):
                a = r.binding.build_args(
                    qs(din["q"], c), kvs(din["k"], c), kvs(din["v"], c),
                    qs(outs[par][ni], c), qs(stats[par][ni], c), None, normalizer=n,
                    causal=w.causal, window=w.window, softcap=w.softcap,
                    scale=w.scale, stream=s_cmp.cuda_stream)
                need = r.binding.nattn_workspace_size(a)
                if need:
                    ws = torch.empty(need, dtype=torch.uint8, device=dev)
                    keep.append(ws)
                    a.workspace, a.workspace_bytes = ws.data_ptr(), need
                args[par, ni, ci] = a
    ev_in = [torch.cuda.Event() for _ in chunks]
    ev_read = [torch.cuda.Event() for _ in chunks]
    ev_cmp = {key: torch.cuda.Event() for key in args}
    ev_out = {key: torch.cuda.Event() for key in args}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = len(norms) * (out_h[0].numel() * out_h[0].element_size() + stat_h[0].numel() * 4)

    def step(i):
        par = i & 1
        for ci, c in enumerate(chunks):
            with torch.cuda.stream(s_in):
                if i > 0:
                    s_in.wait_event(ev_read[ci])
                qs(din["q"], c).copy_(qs(host["q"], c), non_blocking=True)
                kvs(din["k"], c).copy_(kvs(host["k"], c), non_blocking=True)
                kvs(din["v"], c).copy_(kvs(host["v"], c), non_blocking=True)
                ev_in[ci].record(s_in)
        for ni in range(len(norms)):
            for ci, c in enumerate(chunks):
                key = (par, ni, ci)
                with torch.cuda.stream(s_cmp):
                    if ni == 0:
                        s_cmp.wait_event(ev_in[ci])
                    if i >= 2:
                        s_cmp.wait_event(ev_out[key])
                    if r.binding.nattn_fwd_ex(args[key]) != 0:
                        raise RuntimeError("nattn_fwd_ex failed")
                    ev_cmp[key].record(s_cmp)
                    if ni == len(norms) - 1:
                        ev_read[ci].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[key])
                    qs(out_h[ni], c).copy_(qs(outs[par][ni], c), non_blocking=True)
                    qs(stat_h[ni], c).copy_(qs(stats[par][ni], c), non_blocking=True)
                    ev_out[key].record(s_out)

    def join():
        e = torch.cuda.Event()
        e.record(s_out)
        s_in.wait_event(e)
        e2 = torch.cuda.Event()
        e2.record(s_cmp)
        s_in.wait_event(e2)

    step(0)
    step(1)
    join()
    torch.cuda.synchronize()
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record(s_in)
    for i in range(steps):
        step(i)
    join()
    en.record(s_in)
    torch.cuda.synchronize()
    ms = st.elapsed_time(en) / steps
    # the chunked results against one unchunked call per normalizer
    diff = 0.0
    for ni, n in enumerate(norms):
        r.call(n)
        torch.cuda.synchronize()
        diff = max(diff, float((out_h[ni].float() - r.out.float().cpu()).abs().max()))
    return ms, h2d, d2h, diff


def cpu_baseline_prefill(w, x, budget_s=10.0):
    """The float64 oracle on a bounded sample of query rows (evenly spaced
    rows of batch 0, head after head, about budget_s seconds of CPU work),
    scaled to useful TFLOP/s."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max(i.get("num_threads", 1) for i in threadpool_info()) \
            if threadpool_info() else os.cpu_count()
    except Exception:
        cores = os.cpu_count()
    flops, secs, nrows, heads = 0.0, 0.0, 0, 0
    stride = max(1, w.Tq // 512)
    rows_all = np.arange(w.Tq - 1, -1, -stride)
    ok = oracle.allowed_matrix(w.Tq, w.Tk, w.causal, w.window)
    t_start = time.perf_counter()
    for h in range(w.Hq):
        g = h // (w.Hq // w.Hkv)
        q = x["q"][:1, h:h + 1]
        k = x["k"][:1, g:g + 1]
        v = x["v"][:1, g:g + 1]
        for n in w.normalizers:
            for i0 in range(0, len(rows_all), 64):
                sel = rows_all[i0:i0 + 64]
                rows = np.stack([np.zeros_like(sel), np.zeros_like(sel), sel], 1)
                t0 = time.perf_counter()
                oracle.attention_rows(q, k, v, rows, w.scale, n, w.causal,
                                      w.window, w.softcap)
                secs += time.perf_counter() - t0
                flops += float(ok[sel].sum()) * 4 * w.d
                nrows += len(sel)
        heads += 1
        if time.perf_counter() - t_start > budget_s:
            break
    return {"value": flops / secs / 1e12 if secs else None, "unit": "TFLOP/s",
            "cores": cores, "kind": "oracle",
            "sample": f"{nrows} query rows of batch 0 ({len(rows_all)} evenly "
                      f"spaced rows of each of {heads} head(s), latest first, "
                      f"every normalizer), float64 numpy, {secs:.1f} s; FLOPs "
                      f"counted per visible key"}


def main_native(args):
    import torch
    import torch.distributed as dist
    from alternative_normalizers_b200 import binding
    from alternative_normalizers_b200.workloads import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.lib()

    w = WORKLOADS[args.workload]
    if args.normalizer:
        w = replace(w, normalizers=(args.normalizer,))
    if args.batch:
        w = replace(w, B=args.batch)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    r = Runner(w, dev, seed_offset=shard_seed(w, rank) - w.seed)
    for n in w.normalizers:  # warm-up, also the launch configuration checks
        r.call(n)
    torch.cuda.synchronize()
    if binding.nattn_get_device_status() != 0:
        raise RuntimeError("device status after warm-up")

    sampler = NvmlSampler(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    per = time_runner(r, args.steps, args.warmup, flush)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_step = sum(per.values())
    if world > 1:
        ms_step = max_over_ranks(ms_step, dist, dev)
        dist.barrier()

    units = r.units()
    total_units = units * len(w.normalizers) * world
    if w.paged:
        value = total_units / (ms_step * 1e-3) / 1e9
        unit, metric = "GB/s", "decode K/V GB/s (paged, split-KV)"
    else:
        value = total_units / (ms_step * 1e-3) / 1e12
        unit, metric = "TFLOP/s", "fwd attention useful TFLOP/s (prefill)"

    peaks, peak_src = load_peaks()
    # dominant kernel: the prefill (or decode split) launch of one normalizer
    dom = max(per, key=per.get)
    if w.paged:
        ach = units / (per[dom] * 1e-3) / 1e9
        peak_key = "hbm_gbs"
        roof = {"bound": "hbm", "achieved": round(ach, 1), "unit": "GB/s"}
    else:
        ach = units / (per[dom] * 1e-3) / 1e12
        # each launch is timed alone (L2 flush in between), at full clocks:
        # the burst GEMM figure is the matching denominator
        peak_key = "bf16_tflops"
        roof = {"bound": "tensor", "achieved": round(ach, 1), "unit": "TFLOP/s"}
    peak = peaks[peak_key]
    roof["peak"] = peak
    roof["frac"] = round(ach / peak, 4)
    if not w.paged:
        roof["frac_vs_sustained"] = round(ach / peaks["bf16_tflops_sustained"], 4)
    tr = NCU_TRAFFIC.get((w.name, dom))
    roof["traffic"] = tr[0] if tr else None
    roof["traffic_source"] = tr[1] if tr else None
    roof["kernel"] = f"{dom} launch"
    roof["peak_source"] = f"{peak_src} {peak_key}"

    line = {
        "metric": metric, "value": round(value, 2), "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, see workloads.py)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
                   "Tq": w.Tq, "Tk": w.Tk, "d": w.d, "dv": w.dv,
                   "causal": w.causal, "window": w.window,
                   "softcap": w.softcap,
                   "normalizers": list(w.normalizers),
                   "parallelism": f"independent batch per GPU x{world}",
                   "l2": "flushed (256 MiB write) before every timed launch, "
                         "outside the CUDA events"},
        "per_normalizer_ms": {n: round(v, 4) for n, v in per.items()},
        "per_normalizer_value": {
            n: round(units / (v * 1e-3) / (1e9 if w.paged else 1e12), 2)
            for n, v in per.items()},
        "roofline": roof,
        "clocks": clocks,
        "gpu_launches": args.steps * sum(
            (LAUNCHES_DECODE if w.paged else LAUNCHES)[n]
            for n in w.normalizers),
    }
    if rank == 0 and args.quick:
        print(json.dumps(line), flush=True)
    elif not args.quick:
        # every rank streams its own batch through the C ABI at the same
        # time; the whole job's figure is all ranks' work over the slowest
        # rank's time
        e2e_steps = max(4, args.steps // 4)
        if world > 1:
            dist.barrier()
        if w.paged:
            e2e_ms, h2d, d2h = e2e_measure(r, e2e_steps, dev)
            how, diff = "copy in, compute, copy out on one stream", None
        else:
            e2e_ms, h2d, d2h, diff = e2e_measure_dense(r, e2e_steps, dev)
            how = ("chunks of (batch entry, half the KV heads): copies in, "
                   "products and copies out on three streams, overlapped")
        if world > 1:
            e2e_ms = max_over_ranks(e2e_ms, dist, dev)
        e2e_val = units * world * len(w.normalizers) / (e2e_ms * 1e-3) / (
            1e9 if w.paged else 1e12)
        line["e2e"] = {"value": round(e2e_val, 3), "unit": unit,
                       "h2d_bytes_per_step": h2d * world,
                       "d2h_bytes_per_step": d2h * world,
                       "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                       "schedule": how}
        if diff is not None:
            line["e2e"]["max_abs_diff_vs_unchunked"] = diff
    if rank == 0 and not args.quick:
        if world == 1 and not w.paged:
            line["cpu_baseline"] = cpu_baseline_prefill(w, r.host)
        if args.detail and world == 1:
            line["other_workloads"] = detail(args, dev, flush)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def sparse_prefill_stats(r, n):
    """Support statistics of one sparse normalizer on a dense workload: the
    rows' thresholds come from the kernel (row_stat), the scores are
    recomputed in float32 with torch (measurement only).  Returns the mean
    threshold, the support size (mean / p99 / max) and the fraction of
    visible weights that are exactly zero."""
    import torch
    w = r.w
    r.call(n)
    if r.stat.is_cuda:
        torch.cuda.synchronize()
    tau = r.stat.float()
    half = 0.5 if n == "entmax15" else 1.0
    sup_all, vis_all = [], 0
    ii = torch.arange(w.Tq, device=tau.device)[:, None]
    jj = torch.arange(w.Tk, device=tau.device)[None, :]
    off = w.Tk - w.Tq
    allowed = torch.ones(w.Tq, w.Tk, dtype=torch.bool, device=tau.device)
    if w.causal:
        allowed &= jj <= ii + off
    if w.window > 0:
        allowed &= jj > ii + off - w.window
    vis_all = int(allowed.sum()) * w.B * w.Hq
    grp = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hq):
            q = r.x["q"][b, h].float()
            k = r.x["k"][b, h // grp].float()
            z = (q @ k.T) * w.scale
            if w.softcap > 0:
                z = w.softcap * torch.tanh(z / w.softcap)
            u = z * half
            u = u.masked_fill(~allowed, float("-inf"))
            sup_all.append((u > tau[b, h][:, None]).sum(dim=1))
    sup = torch.cat(sup_all).float()
    return {"tau_mean": round(float(tau[torch.isfinite(tau)].mean()), 4),
            "support_mean": round(float(sup.mean()), 2),
            "support_p99": float(torch.quantile(sup[:1 << 20], 0.99)),
            "support_max": int(sup.max()),
            "exact_zero_fraction": round(1.0 - float(sup.sum()) / vis_all, 6)}


def sparse_decode_bytes(r, n):
    """Bytes a sparse decode step actually moves, next to the dense-equivalent
    K/V count: every K page (the score pass), the fp32 scores written once
    and read twice (threshold, then apply), the V pages that carry a nonzero
    weight for some query head of their group, and Q/O.  Which V pages are
    loaded is recomputed here from the kernel's thresholds and float32
    scores (measurement only); split partials (under 1 % here) are left
    out."""
    import torch
    w = r.w
    r.call(n)
    if r.stat.is_cuda:
        torch.cuda.synchronize()
    tau = r.stat.float()
    half = 0.5 if n == "entmax15" else 1.0
    grp = w.Hq // w.Hkv
    ps = w.page_size
    kb = vb = sb = 0
    vpages = 0
    for b in range(w.B):
        L = int(r.host["seqlens"][b])
        npg = (L + ps - 1) // ps
        pages = r.x["block_table"][b, :npg].long()
        kseq = r.x["k_pool"][pages]                      # [npg, Hkv, ps, d]
        kseq = kseq.permute(1, 0, 2, 3).reshape(w.Hkv, npg * ps, w.d)[:, :L]
        q = r.x["q"][b, :, 0].float()                    # [Hq, d]
        z = torch.einsum("hgd,htd->hgt", q.view(w.Hkv, grp, w.d),
                         kseq.float()) * w.scale         # [Hkv, grp, L]
        if w.softcap > 0:
            z = w.softcap * torch.tanh(z / w.softcap)
        t = tau[b, :, 0].view(w.Hkv, grp, 1)
        hit = (z * half > t).any(dim=1)                  # [Hkv, L]
        pad = npg * ps - L
        if pad:
            hit = torch.nn.functional.pad(hit, (0, pad))
        vpages += int(hit.view(w.Hkv, npg, ps).any(dim=2).sum())
        kb += npg * ps * w.Hkv * w.d * 2
        sb += 3 * w.Hq * L * 4
    vb = vpages * ps * w.dv * 2
    qo = w.B * w.Hq * (w.d + w.dv) * 2
    return {"k_bytes": kb, "v_bytes": vb, "score_bytes": sb, "qo_bytes": qo,
            "total": kb + vb + sb + qo, "v_pages": vpages}


class BwdRunner:
    """The backward pass of one dense workload: the forward runs once to give
    the saved output and row statistic, then every timed call is one
    nattn_bwd (delta pass, dQ kernel, dK/dV kernel).  Useful FLOPs are 2.5x
    the forward's (five products of the forward's size against two)."""

    def __init__(self, w, dev):
        import torch
        from alternative_normalizers_b200 import binding
        from alternative_normalizers_b200.workloads import make_inputs
        self.w, self.binding = w, binding
        x = make_inputs(w)
        g = torch.Generator().manual_seed(w.seed + 500)
        dout = torch.randn(w.B, w.Hq, w.Tq, w.dv, generator=g).to(torch.bfloat16)
        self.x = {k: v.to(dev) for k, v in x.items()}
        self.dout = dout.to(dev)
        self.args, self.keep = {}, []
        for n in w.normalizers:
            out, st, _ = binding.attention(self.x["q"], self.x["k"], self.x["v"],
                                           normalizer=n, causal=w.causal,
                                           window=w.window, softcap=w.softcap,
                                           scale=w.scale)
            dq, dk, dv = (torch.empty_like(self.x[t]) for t in ("q", "k", "v"))
            a = binding.build_bwd_args(self.x["q"], self.x["k"], self.x["v"], out, st,
                                       self.dout, dq, dk, dv, normalizer=n,
                                       causal=w.causal, window=w.window,
                                       softcap=w.softcap, scale=w.scale)
            ws = torch.empty(binding.nattn_bwd_workspace_size(a), dtype=torch.uint8,
                             device=dev)
            a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
            self.keep += [out, st, dq, dk, dv, ws]
            self.args[n] = a

    def call(self, n):
        rc = self.binding.nattn_bwd(self.args[n])
        if rc != 0:
            raise RuntimeError(f"nattn_bwd({n}) failed: {rc}")

    def units(self):
        return 2.5 * self.w.useful_flops()


class ArgsRunner:
    """Timing target for prebuilt argument blocks: one nattn_fwd_ex per call."""

    def __init__(self, name, normalizers, args, keep, units):
        from types import SimpleNamespace
        from alternative_normalizers_b200 import binding
        self.w = SimpleNamespace(name=name, normalizers=tuple(normalizers))
        self.binding, self.args, self.keep, self._units = binding, args, keep, units

    def call(self, n):
        rc = self.binding.nattn_fwd_ex(self.args[n])
        if rc != 0:
            raise RuntimeError(f"nattn_fwd_ex({n}) failed: {rc}")

    def units(self):
        return self._units


def varlen_runner(dev):
    """The headline layer's heads (Hq=32, Hkv=8, d=128, causal) over one
    packed batch of four requests of 4096, 2048, 1536 and 512 tokens
    ([total, H, d] layouts, cumulative lengths)."""
    import torch
    from alternative_normalizers_b200 import binding
    lens = [4096, 2048, 1536, 512]
    tot, Hq, Hkv, d = sum(lens), 32, 8, 128
    g = torch.Generator().manual_seed(2024)
    mk = lambda *sh: torch.randn(*sh, generator=g).to(torch.bfloat16).to(dev)
    q, k, v = mk(tot, Hq, d), mk(tot, Hkv, d), mk(tot, Hkv, d)
    cu = torch.tensor([0] + list(__import__("itertools").accumulate(lens)),
                      dtype=torch.int32, device=dev)
    out = torch.empty(tot, Hq, d, dtype=torch.bfloat16, device=dev)
    st = torch.empty(tot, Hq, dtype=torch.float32, device=dev)
    args, keep = {}, [q, k, v, cu, out, st]
    for n in ("softmax", "sparsemax"):
        a = binding.NattnArgs()
        a.q, a.k, a.v, a.out, a.row_stat = (t.data_ptr() for t in (q, k, v, out, st))
        a.B, a.Hq, a.Hkv, a.d, a.dv, a.Tq, a.Tk = len(lens), Hq, Hkv, d, d, max(lens), max(lens)
        a.scale, a.normalizer, a.causal = d ** -0.5, binding.NORMALIZER_IDS[n], 1
        a.cu_seqlens_q = a.cu_seqlens_k = cu.data_ptr()
        a.total_q = a.total_k = tot
        a.stream = torch.cuda.current_stream(dev).cuda_stream
        need = binding.nattn_workspace_size(a)
        if need:
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
            keep.append(ws)
            a.workspace, a.workspace_bytes = ws.data_ptr(), need
        args[n] = a
    pairs = sum(L * (L + 1) // 2 for L in lens)
    return ArgsRunner("packed_varlen", args.keys(), args, keep, 4.0 * d * pairs * Hq)


def paged_prefill_runner(dev):
    """Chunked prefill into a paged cache: 8 requests, each with 1024 new
    query tokens after 3072 cached ones (4096 keys), Hq=32, Hkv=8, d=128,
    64-token pages in a random permutation of the pool, causal."""
    import torch
    from alternative_normalizers_b200 import binding
    B, Tq, L, Hq, Hkv, d, ps = 8, 1024, 4096, 32, 8, 128, 64
    g = torch.Generator().manual_seed(2025)
    mk = lambda *sh: torch.randn(*sh, generator=g).to(torch.bfloat16).to(dev)
    npg = L // ps
    q = mk(B, Hq, Tq, d)
    kp, vp = mk(B * npg, Hkv, ps, d), mk(B * npg, Hkv, ps, d)
    table = torch.randperm(B * npg, generator=g).to(torch.int32).view(B, npg).to(dev)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, Tq, d, dtype=torch.bfloat16, device=dev)
    st = torch.empty(B, Hq, Tq, dtype=torch.float32, device=dev)
    args, keep = {}, [q, kp, vp, table, lens, out, st]
    for n in ("softmax", "sparsemax"):
        a = binding.build_args(q, kp, vp, out, st, None, normalizer=n, causal=True,
                               scale=d ** -0.5, block_table=table, seqlens=lens,
                               page_size=ps, max_seqlen=L)
        need = binding.nattn_workspace_size(a)
        if need:
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
            keep.append(ws)
            a.workspace, a.workspace_bytes = ws.data_ptr(), need
        args[n] = a
    # query i of a request sits at key position i + 3072: sees 3073 + i keys
    pairs = Tq * (L - Tq) + Tq * (Tq + 1) // 2
    return ArgsRunner("paged_prefill", args.keys(), args, keep, 4.0 * d * pairs * B * Hq)


def detail(args, dev, flush):
    """The other workload shapes, each normalizer timed like the headline."""
    import torch
    from alternative_normalizers_b200.workloads import WORKLOADS
    res = {}
    names = ["sparse_prefill_t1", "sparse_prefill_t4", "sparse_prefill_wide",
             "gemma2_9b_local", "gemma2_9b_global", "paged_decode"]
    for name in names:
        w = WORKLOADS[name]
        try:
            r = Runner(w, dev)
            per = time_runner(r, max(3, args.steps // 2), 2, flush)
            u = r.units()
            if w.paged:
                vals = {n: round(u / (t * 1e-3) / 1e9, 1) for n, t in per.items()}
                unit = "GB/s (dense-equivalent K/V bytes)"
            else:
                vals = {n: round(u / (t * 1e-3) / 1e12, 1) for n, t in per.items()}
                unit = "useful TFLOP/s"
            peaks = load_peaks()[0]
            if w.paged:
                frac = {n: round(v / peaks["hbm_gbs"], 4) for n, v in vals.items()}
                fkind = peak_label("hbm_gbs", " (dense-equivalent bytes)")
            else:
                frac = {n: round(v / peaks["bf16_tflops"], 4)
                        for n, v in vals.items()}
                fkind = peak_label("bf16_tflops", " (burst)")
            res[name] = {"unit": unit, "value": vals,
                         "ms": {n: round(t, 4) for n, t in per.items()},
                         "roofline_frac": frac, "roofline_denominator": fkind}
            sparse = [n for n in per if n in ("sparsemax", "entmax15")]
            if w.paged and sparse:
                peak = load_peaks()[0]["hbm_gbs"]
                act = {}
                for n in sparse:
                    by = sparse_decode_bytes(r, n)
                    gbs = by["total"] / (per[n] * 1e-3) / 1e9
                    act[n] = {"GB/s": round(gbs, 1), "bytes": by,
                              "frac_of_hbm": round(gbs / peak, 4)}
                res[name]["actual_bytes"] = act
            elif sparse:
                res[name]["support"] = {n: sparse_prefill_stats(r, n)
                                        for n in sparse}
            del r
            torch.cuda.empty_cache()
        except Exception as exc:  # report, keep the headline line
            res[name] = {"error": repr(exc)[:200]}
    peaks = load_peaks()[0]
    # backward pass (fused, recomputing the weights from the saved statistic)
    for name in ("qwen3_8b_prefill", "sparse_prefill_t1"):
        w = WORKLOADS[name]
        try:
            r = BwdRunner(w, dev)
            per = time_runner(r, max(3, args.steps // 2), 2, flush)
            u = r.units()
            vals = {n: round(u / (t * 1e-3) / 1e12, 1) for n, t in per.items()}
            res[name + "_backward"] = {
                "unit": "useful TFLOP/s (2.5x the forward's useful FLOPs)",
                "value": vals, "ms": {n: round(t, 4) for n, t in per.items()},
                "roofline_frac": {n: round(v / peaks["bf16_tflops"], 4)
                                  for n, v in vals.items()},
                "roofline_denominator": peak_label("bf16_tflops", " (burst)")}
            del r
            torch.cuda.empty_cache()
        except Exception as exc:
            res[name + "_backward"] = {"error": repr(exc)[:200]}
    # learned per-head sinks on the headline shape (softmax with sinks[h])
    try:
        w = replace(WORKLOADS["qwen3_8b_prefill"], normalizers=("softmax",))
        r = Runner(w, dev)
        g = torch.Generator().manual_seed(77)
        sinks = (torch.randn(w.Hq, generator=g) * 2).to(dev)
        r.args["softmax"].sinks = sinks.data_ptr()
        per = time_runner(r, max(3, args.steps // 2), 2, flush)
        v = r.units() / (per["softmax"] * 1e-3) / 1e12
        res["qwen3_8b_prefill_sinks"] = {
            "unit": "useful TFLOP/s", "value": {"softmax+sinks": round(v, 1)},
            "ms": {"softmax+sinks": round(per["softmax"], 4)},
            "roofline_frac": {"softmax+sinks": round(v / peaks["bf16_tflops"], 4)},
            "roofline_denominator": peak_label("bf16_tflops", " (burst)")}
        del r, sinks
        torch.cuda.empty_cache()
    except Exception as exc:
        res["qwen3_8b_prefill_sinks"] = {"error": repr(exc)[:200]}
    # block mask: the headline shape packed with four causal documents of
    # 1024 tokens (block-diagonal mask); useful FLOPs = 4 * d per allowed
    # (query, key) pair, counted exactly
    try:
        w = WORKLOADS["qwen3_8b_prefill"]
        r = Runner(w, dev)
        doc = 1024 // 128
        nq = (w.Tq + 127) // 128
        bm = torch.zeros(w.B, w.Hq, nq, nq, dtype=torch.uint8)
        for d0 in range(0, nq, doc):
            bm[..., d0:d0 + doc, d0:d0 + doc] = 1
        bm = bm.to(dev)
        for n in w.normalizers:
            r.args[n].block_mask = bm.data_ptr()
        per = time_runner(r, max(3, args.steps // 2), 2, flush)
        pairs = (w.Tq // 1024) * (1024 * 1025 // 2)
        u = 4.0 * w.d * pairs * w.B * w.Hq
        vals = {n: round(u / (t * 1e-3) / 1e12, 1) for n, t in per.items()}
        res["qwen3_8b_prefill_doc_mask"] = {
            "unit": "useful TFLOP/s (exact allowed pairs)", "value": vals,
            "ms": {n: round(t, 4) for n, t in per.items()},
            "roofline_frac": {n: round(v / peaks["bf16_tflops"], 4) for n, v in vals.items()},
            "roofline_denominator": peak_label("bf16_tflops", " (burst)")}
        del r, bm
        torch.cuda.empty_cache()
    except Exception as exc:
        res["qwen3_8b_prefill_doc_mask"] = {"error": repr(exc)[:200]}
    # packed variable-length batch and chunked paged prefill (exact pairs)
    for make in (varlen_runner, paged_prefill_runner):
        try:
            r = make(dev)
            per = time_runner(r, max(3, args.steps // 2), 2, flush)
            vals = {n: round(r.units() / (t * 1e-3) / 1e12, 1) for n, t in per.items()}
            res[r.w.name] = {
                "unit": "useful TFLOP/s (exact allowed pairs)", "value": vals,
                "ms": {n: round(t, 4) for n, t in per.items()},
                "roofline_frac": {n: round(v / peaks["bf16_tflops"], 4)
                                  for n, v in vals.items()},
                "roofline_denominator": peak_label("bf16_tflops", " (burst)")}
            del r
            torch.cuda.empty_cache()
        except Exception as exc:
            res[make.__name__] = {"error": repr(exc)[:200]}
    return res


# --------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# --------------------------------------------------------------------------
def main_reference(args):
    from alternative_normalizers_b200.workloads import WORKLOADS, make_inputs
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    x = make_inputs(w)
    # one head's rows per step (under a second), so that --steps K stays
    # within minutes
    budget = 0.1
    vals = []
    cb = None
    for _ in range(args.warmup):
        cpu_baseline_prefill(w, x, budget_s=budget)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cb = cpu_baseline_prefill(w, x, budget_s=budget)
        vals.append(cb["value"])
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": "fwd attention useful TFLOP/s (prefill)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(wall / max(1, args.steps) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded, see workloads.py)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
                   "Tq": w.Tq, "Tk": w.Tk, "d": w.d, "causal": w.causal,
                   "normalizers": list(w.normalizers)},
        "cpu_baseline": dict(cb, value=value),
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def spawn_ranks(n):
    """Run this same command as ``n`` ranks, one per GPU, under
    torch.distributed.run (rendezvous on 127.0.0.1); returns its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--workload", default="qwen3_8b_prefill")
    p.add_argument("--no-detail", dest="detail", action="store_false")
    p.add_argument("--normalizer", default=None,
                   help="time only this normalizer of the workload")
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's batch (profiling a smaller "
                        "case of the same kernel)")
    p.add_argument("--quick", action="store_true",
                   help="timed steps only (no e2e, CPU baseline or other "
                        "workloads): the profiling target")
    args = p.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is not None and int(env_world) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={env_world}")
    if env_world is None and args.gpus > 1:
        sys.exit(spawn_ranks(args.gpus))
    if args.impl == "reference":
        main_reference(args)
    else:
        main_native(args)


if __name__ == "__main__":
    main()
