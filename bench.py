#!/usr/bin/env python
"""MLA paged decode benchmark (one JSON line on rank 0).

A step is one pass of the whole decode path over one batch: split-KV
scheduling (mla_get_metadata), the decode kernel and the split combine, all
through the C ABI of libmla_b200.so on inputs already resident in HBM.
Default workload: the DeepSeek-V3-shaped batch (64 requests x 128 heads,
4096 cached tokens each, bf16 latent cache in 64-token pages), whose 302 MB
cache is larger than L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores

With N > 1 (launched by torch.distributed.run) every rank decodes its own
replica of the workload (requests are independent; no collective is needed
on the data path), timing is the max over ranks and `value` sums all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import mla_workloads as W  # noqa: E402

METRIC = "MLA decode TFLOPS & HBM GB/s on 1 B200, as fraction of roofline"
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAK_FALLBACK), "fallback"


KERNEL_SOURCE = {"mla_decode_pair_kernel": "mla_decode_pair.cu", "mla_decode_kernel": "mla_decode.cu",
                 "mla_decode_page_kernel": "mla_decode_page.cu"}


def strip_c_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines, trailing spaces
    dropped; string and character literals (inline PTX) are kept as written."""
    out, i, n = [], 0, len(src)
    while i < n:
        j = min((k for k in (src.find("//", i), src.find("/*", i), src.find('"', i), src.find("'", i)) if k >= 0),
                default=n)
        out.append(src[i:j])
        if j >= n:
            break
        if src.startswith("//", j):
            k = src.find("\n", j)
            i = n if k < 0 else k
        elif src.startswith("/*", j):
            k = src.find("*/", j + 2)
            i = n if k < 0 else k + 2
        else:  # a literal: copy it through its closing quote
            q, k = src[j], j + 1
            while k < n and src[k] != q:
                k += 2 if src[k] == "\\" else 1
            out.append(src[j:k + 1])
            i = k + 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_source_hash(kernel: str) -> str:
    """Hash of what one decode kernel is built from: its own .cu file and the
    shared headers, without comments (the scheduler, combine and host-side
    files, and comments, do not change the kernel's memory traffic)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "head_latent_attention_get_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith(".cuh") or f == KERNEL_SOURCE[kernel]:
            with open(os.path.join(csrc, f), encoding="utf-8") as fh:
                h.update(strip_c_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def decode_kernel_name(w, rows: int) -> str:
    """The decode kernel the library launches for this workload: CTA pairs for
    units of 65-128 rows on the BF16 cache (paged or token-sparse), one CTA per
    row group otherwise; the FP8 and NVFP4 paged caches have a page kernel."""
    if w.kv == "bf16" and rows > 64:
        return "mla_decode_pair_kernel"
    if w.kv in ("fp8", "nvfp4") and w.topk == 0:
        return "mla_decode_page_kernel"
    return "mla_decode_kernel"


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel") not in KERNEL_SOURCE or e.get("kernel_source_sha") != kernel_source_hash(e["kernel"]):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons while the timed loop runs.

    A separate `nvidia-smi -lms` process does the sampling, so the Python
    thread that enqueues the kernels cannot starve it; only samples whose
    timestamps fall inside the timed window are kept. Falls back to an NVML
    thread when nvidia-smi is not available."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device, period_ms: int = 20):
        self.samples, self.reasons = [], set()
        self.period_ms = period_ms
        self.max_mhz = None
        self.proc = None
        self.source = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not self.uuid.startswith("GPU-"):
                self.uuid = "GPU-" + self.uuid
        except Exception:
            self.uuid = None

    def __enter__(self):
        import subprocess
        if self.uuid:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", self.uuid, "--query-gpu=timestamp,clocks.sm,clocks.max.sm,"
                     "clocks_event_reasons.active", "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.proc.stdout.readline()   # sampling has started
                self.source = "nvidia-smi"
            except Exception:
                self.proc = None
        self.t0 = time.time()
        return self

    def __exit__(self, *a):
        self.t1 = time.time()
        if self.proc is None:
            return
        import datetime
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 4:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                mhz, mx, bits = float(f[1]), float(f[2]), int(f[3], 16)
            except ValueError:
                continue
            if self.t0 - 0.05 <= ts <= self.t1 + 0.05:
                self.samples.append(mhz)
                self.max_mhz = mx
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        self.reasons.add(name)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no clock samples"],
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": self.source,
                "window_s": round(self.t1 - self.t0, 3)}


def workload_config(inp, work):
    w = inp.workload
    cfg = {"workload": f"{w.name}: {w.note}", "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q,
           "h_kv": 1, "d_qk": w.d_qk, "d_v": 512, "page": 64, "kv_cache": w.kv,
           "causal": w.causal, "softmax_scale": w.scale,
           "tokens_cached": int(sum(int(x) for x in inp.cache_seqlens.tolist())),
           "algorithmic_flops": work["flops"], "algorithmic_bytes": work["bytes"],
           "l2": ("a step reads %.0f MB (more than twice the 126 MB L2), no flush" if
                  work["bytes"] >= 2 * L2_BYTES else
                  "a step reads %.0f MB (less than twice L2): 256 MB written before every step, "
                  "outside the events that time it") % (
               work["bytes"] / 1e6)}
    if w.topk:
        cfg["topk"] = w.topk
    if inp.sink is not None:
        cfg["sink"] = "seeded per-head logits, N(0,1) + 1"
    return cfg


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(inp, budget_s: float):
    """Time the fp64 oracle on whole requests until about budget_s elapses."""
    from oracle import mla_oracle as O
    from threadpoolctl import threadpool_info
    w = inp.workload
    order = list(range(w.batch))
    flops = 0.0
    elapsed = 0.0
    done = []
    for b in order:
        sub = W.restrict(inp, [b])
        work = W.algorithmic_work(sub)
        t0 = time.perf_counter()
        O.reference_decode(sub)
        elapsed += time.perf_counter() - t0
        flops += work["flops"]
        done.append(b)
        if elapsed >= budget_s:
            break
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": int(threads),
            "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{len(done)} of {w.batch} requests of the workload (whole requests, "
                      f"{flops:.3g} FLOPs in {elapsed:.2f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = W.make_inputs(W.get_workload(args.workload))
    from oracle import mla_oracle as O
    from threadpoolctl import threadpool_info
    w = inp.workload
    # each step decodes one request of the workload (a bounded sample)
    times, flops = [], []
    for s in range(args.warmup + args.steps):
        b = s % w.batch
        sub = W.restrict(inp, [b])
        t0 = time.perf_counter()
        O.reference_decode(sub)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            flops.append(W.algorithmic_work(sub)["flops"])
    tot = sum(times)
    value = sum(flops) / tot / 1e12
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    work = W.algorithmic_work(inp)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(inp, work),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": int(threads),
                             "host_cores": os.cpu_count(), "kind": "oracle",
                             "sample": "one whole request of the workload per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ranks
def init_ranks(device=None, backend="nccl"):
    """(world, rank, local rank, process group module or None) from the
    torchrun environment; one process per GPU, a short collective timeout so
    that ranks waiting on a lost peer end with an error."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": device} if backend == "nccl" and device is not None else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
        pg = dist
    return world, rank, local, pg


def max_over_ranks(pg, x: float, device) -> float:
    """The largest of every rank's x (a time: the job is as slow as its slowest rank)."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank decodes its own replica of the workload."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- GPU path
L2_BYTES = 126 * 2 ** 20
CONFIGS = ["tiny", "dsv3", "mtp", "fp8", "sparse"]   # the five configurations, in order


def build_runner(inp, dev, M, C):
    w = inp.workload
    d = {k: (None if v is None else v.to(dev)) for k, v in dict(
        q=inp.q, kc=inp.kcache, bt=inp.block_table, sl=inp.cache_seqlens, idx=inp.indices, sink=inp.sink,
        qs=inp.q_scale, ks=inp.kv_scale).items()}
    runner = M.DecodeRunner(d["q"], d["kc"], d["bt"], d["sl"], softmax_scale=w.scale, causal=w.causal,
                            indices=d["idx"], sink=d["sink"], q_scale=d["qs"], kv_scale=d["ks"])
    return runner, d


def measure(inp, steps: int, warmup: int, dev, pg=None):
    """Times `steps` decode steps (scheduler + decode kernel + combine) on
    resident inputs with CUDA events on the launching stream: once back to
    back (the step time), then again with an event around each kernel (the
    per-kernel times). The decode kernel is launched with the combine held
    back and the combine enqueued right after it, so each kernel has its own
    events. When the bytes a step reads are less than twice L2 (the tiny and
    token-sparse workloads), a 256 MB buffer is written before each step
    (outside the per-kernel events) so that every step reads from HBM."""
    import head_latent_attention_get_b200 as M
    from head_latent_attention_get_b200 import _capi as C
    w = inp.workload
    runner, d = build_runner(inp, dev, M, C)
    runner.args.debug_flags = C.MLA_DEBUG_SKIP_COMBINE
    U, R, P = runner.units, runner.rows, runner.parts
    ws_bytes = runner.workspace.numel()
    stream = torch.cuda.current_stream()
    # the bytes a step touches (not the whole cache: a token-sparse step reads
    # only its indexed rows) decide whether L2 could serve the next step
    touched = W.algorithmic_work(inp)["bytes"]
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev) if touched < 2 * L2_BYTES else None

    def step(ev=None):
        """ev: four events (one around each kernel) or two (around the whole
        step, whose kernels then stay chained)."""
        each = ev is not None and len(ev) == 4
        if flush is not None:
            flush.fill_(1)
        if ev is not None:
            ev[0].record(stream)
        runner.plan(stream)
        if each:
            ev[1].record(stream)
        runner.run(stream)
        if each:
            ev[2].record(stream)
        M.mla_combine_sink(runner.workspace, ws_bytes, runner.num_splits, U, R, P, w.h_q, d["sink"], runner.out,
                           runner.lse, stream)
        if ev is not None:
            ev[-1].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    code, bits = runner.status()
    if code != C.MLA_OK:
        raise RuntimeError(f"{w.name}: device status after warm-up: {M.mla_status_string(code)} bits={bits}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    whole = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    bad_reasons = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    remeasured = False
    for attempt in range(2):
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        with ClockSampler(dev) as clocks:
            # whole steps back to back (the kernels of a step overlap their
            # launches), then the same steps with events around each whole
            # step (the L2 flush stays outside them), then with an event
            # around each kernel
            t_start.record(stream)
            for s in range(steps):
                step()
            t_end.record(stream)
            for s in range(steps):
                step(whole[s])
            for s in range(steps):
                step(evs[s])
            torch.cuda.synchronize()
        if pg:
            pg.barrier()
        if attempt == 0 and bad_reasons & set(clocks.summary().get("reasons", [])):
            remeasured = True      # slowdown seen while timing: measure once more
            continue
        break
    meta = [e[0].elapsed_time(e[1]) for e in evs]
    dec = [e[1].elapsed_time(e[2]) for e in evs]
    comb = [e[2].elapsed_time(e[3]) for e in evs]
    return {"runner": runner, "rows": runner.rows, "dev_inputs": d, "total_ms": t_start.elapsed_time(t_end), "steps": steps,
            "flushed": flush is not None, "metadata_ms": sum(meta) / steps, "kernel_ms": sum(dec) / steps,
            "combine_ms": sum(comb) / steps, "step_kernels_ms": (sum(meta) + sum(dec) + sum(comb)) / steps,
            "step_chained_ms": sum(e[0].elapsed_time(e[1]) for e in whole) / steps,
            "clocks": dict(clocks.summary(), remeasured=remeasured), "launches": 3 * steps}


def roofline_of(inp, m, peaks, peak_src):
    """Roofline figures of the decode kernel from its measured average time."""
    w = inp.workload
    work = W.algorithmic_work(inp)
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"])
    k_ms = m["kernel_ms"]
    achieved_gbs = work["bytes"] / (k_ms * 1e-3) / 1e9
    achieved_tf = work["flops"] / (k_ms * 1e-3) / 1e12
    t_hbm = work["bytes"] / (hbm_peak * 1e9)
    t_tc = work["flops"] / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    mhz = m["clocks"].get("sm_mhz")
    # with an L2 flush before every step: events around each whole step;
    # otherwise whole steps back to back
    step_ms = m["step_chained_ms"] if m["flushed"] else m["total_ms"] / m["steps"]
    return {"bound": bound,
            "achieved": achieved_gbs if bound == "hbm" else achieved_tf,
            "peak": hbm_peak if bound == "hbm" else tc_peak,
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": (achieved_gbs / hbm_peak) if bound == "hbm" else (achieved_tf / tc_peak),
            "traffic": recorded_traffic(w.name),
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst figures)" if peak_src == "measured"
            else "fallback",
            "kernel": decode_kernel_name(w, m["rows"]),
            "kernel_ms": k_ms,
            "kernel_kclk_at_median_sm_mhz": None if mhz is None else k_ms * mhz,
            "achieved_tflops": achieved_tf, "achieved_gbs": achieved_gbs,
            "hbm_frac": achieved_gbs / hbm_peak, "tensor_frac": achieved_tf / tc_peak,
            "roofline_frac": max(t_hbm, t_tc) / (k_ms * 1e-3),
            "combine_ms": m["combine_ms"], "metadata_ms": m["metadata_ms"],
            "step_ms": step_ms, "step_overhead_ms": step_ms - k_ms,
            "timing": "kernel_ms, metadata_ms, combine_ms: each kernel between its own events (its launch "
                      "gap included); step_ms: scheduler, decode and combine chained by programmatic dependent "
                      "launch; step_overhead_ms = step_ms - kernel_ms, what the scheduler and combine add (the two come "
                      "from separate passes: where the power cap moves the SM clock between them it can read "
                      "below zero)"}


def run_gpu(args):
    import head_latent_attention_get_b200 as M

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    world, rank, local, pg = init_ranks(dev, "nccl")
    peaks, peak_src = load_peaks()

    inp = W.make_inputs(W.get_workload(args.workload))
    if args.sink:
        inp = W.with_sink(inp, seed=inp.workload.seed)
    work = W.algorithmic_work(inp)
    w = inp.workload
    m = measure(inp, args.steps, args.warmup, dev, pg)
    # with an L2 flush before every step, the step is timed between events
    # around it (the flush outside); otherwise steps run back to back
    ms_step = max_over_ranks(pg, m["step_chained_ms"] if m["flushed"] else m["total_ms"] / args.steps, dev)
    runner, d = m["runner"], m["dev_inputs"]
    stream = torch.cuda.current_stream()

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs from pinned host memory, decodes, and copies out and
    # lse back. Two buffer sets and three streams (copy in, decode, copy out)
    # chained by events, so step i's decode overlaps step i+1's upload and
    # step i-1's download, as a serving loop would run them.
    q_h = inp.q.pin_memory()
    bt_h = inp.block_table.pin_memory()
    sl_h = inp.cache_seqlens.pin_memory()
    idx_h = inp.indices.pin_memory() if inp.indices is not None else None
    qs_h = inp.q_scale.pin_memory() if inp.q_scale is not None else None
    sets = []
    for _ in range(2):
        dq = torch.empty_like(d["q"])
        dbt = torch.empty_like(d["bt"])
        dsl = torch.empty_like(d["sl"])
        didx = torch.empty_like(d["idx"]) if d["idx"] is not None else None
        dqs = torch.empty_like(d["qs"]) if d["qs"] is not None else None
        r = M.DecodeRunner(dq, d["kc"], dbt, dsl, softmax_scale=w.scale, causal=w.causal, indices=didx,
                           sink=d["sink"], q_scale=dqs, kv_scale=d["ks"])
        out_h = torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory()
        lse_h = torch.empty(r.lse.shape, dtype=r.lse.dtype).pin_memory()
        sets.append(dict(q=dq, bt=dbt, sl=dsl, idx=didx, qs=dqs, r=r, out_h=out_h, lse_h=lse_h,
                         loaded=torch.cuda.Event(), done=torch.cuda.Event(), fetched=torch.cuda.Event()))
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step(i):
        b = sets[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(b["done"])          # the decode two steps back has read this set
            b["q"].copy_(q_h, non_blocking=True)
            b["bt"].copy_(bt_h, non_blocking=True)
            b["sl"].copy_(sl_h, non_blocking=True)
            if idx_h is not None:
                b["idx"].copy_(idx_h, non_blocking=True)
            if qs_h is not None:
                b["qs"].copy_(qs_h, non_blocking=True)
            b["loaded"].record(s_in)
        s_run.wait_event(b["loaded"])
        s_run.wait_event(b["fetched"])          # its previous outputs have been copied out
        b["r"].plan(s_run)
        b["r"].run(s_run)
        b["done"].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(b["done"])
            b["out_h"].copy_(b["r"].out, non_blocking=True)
            b["lse_h"].copy_(b["r"].lse, non_blocking=True)
            b["fetched"].record(s_out)

    for i in range(max(2, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_e2e = max(2, min(args.steps, 200))
    e0.record(s_in)
    s_run.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(n_e2e):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1) / n_e2e, dev)
    h2d = q_h.numel() * q_h.element_size() + bt_h.numel() * 4 + sl_h.numel() * 4
    if idx_h is not None:
        h2d += idx_h.numel() * 4
    if qs_h is not None:
        h2d += qs_h.numel()
    d2h = sets[0]["out_h"].numel() * sets[0]["out_h"].element_size() + sets[0]["lse_h"].numel() * 4
    del sets

    # ---- the other configurations, timed the same way in the same run (rank 0 reports them)
    per_config = {}
    if not args.no_per_config:
        for name in CONFIGS:
            if name == args.workload and not args.sink:
                continue
            pi = W.make_inputs(W.get_workload(name))
            pm = measure(pi, min(args.steps, args.per_config_steps), args.warmup, dev, pg)
            r = roofline_of(pi, pm, peaks, peak_src)
            r.update({"workload": W.get_workload(name).note, "steps": pm["steps"],
                      "l2_flush_between_steps": pm["flushed"], "clocks": pm["clocks"]})
            r["step_tflops"] = W.algorithmic_work(pi)["flops"] / (r["step_ms"] * 1e-3) / 1e12
            per_config[name] = r
            del pm
            torch.cuda.empty_cache()

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0

    roof = roofline_of(inp, m, peaks, peak_src)
    value = job_tflops(world, work["flops"], ms_step)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"bf16": "bf16", "fp8": "fp8-e4m3 cache, bf16 mma",
                      "nvfp4": "nvfp4 (e2m1 + ue4m3) query and cache, dequantised exactly to bf16 mma"}[w.kv],
            "data": "synthetic", "config": workload_config(inp, work),
            "hbm_gbs": world * work["bytes"] / (ms_step * 1e-3) / 1e9,
            "roofline": roof, "clocks": m["clocks"],
            "e2e": {"value": job_tflops(world, work["flops"], e2e_ms), "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": m["launches"]}
    if per_config:
        line["per_config"] = per_config
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(inp, args.cpu_budget)
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="dsv3",
                    choices=[w.name for w in W.named_workloads() + W.extra_workloads()])
    ap.add_argument("--sink", action="store_true", help="seeded per-head attention-sink logits")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="time only the chosen workload")
    ap.add_argument("--per-config-steps", type=int, default=1000,
                    help="timed steps of each of the other configurations (capped by --steps)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
