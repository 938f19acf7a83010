#!/usr/bin/env python
"""Benchmark of one ragged paged attention pass (rpa_forward) on B200.

A step is one rpa_forward call over one synthetic batch: the fused cache
update, the decode / prefill kernels, the split-KV combine -- every part of
the method.  The headline line is the 128-sequence decode batch shaped like a
Llama-3-8B attention layer (metric: decode HBM GB/s); the prefill (causal and
not), mixed-batch and head_dim-256 long-context workloads are measured in the
same run.  Each workload prints one short JSON line of its own (value,
dominant-kernel roofline fraction, end-to-end and CUDA-graph numbers) as it
finishes; the headline line comes last.

Timing: W untimed warm-up steps, then K steps timed on the device with CUDA
events on the launching stream, a 256 MiB write between steps to flush the
126 MB L2, barrier + synchronize on both sides, max over ranks.  Algorithmic
bytes and FLOPs follow the method's minimum work: K and V of every visible
position read once, the new K/V written once, Q read and out / lse written
once, the page-table entries read once; FLOPs count visible (q, k) pairs only.
The dominant kernel's roofline comes from a second pass over the same steps
with the library's per-kernel CUDA-event tracing on, so that the step's own
timing has no events between its launches.

``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample
of the same workload (the only other place this script runs the oracle).

``--ablate-write`` measures the cost of the fused cache update: every listed
workload's kernels are timed with this library and, in a child process, with
a timing-only build whose cache stores are compiled out
(RPA_ABLATE_CACHE_WRITE); one line per workload gives both kernel times.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ragged_paged_attention_03_b200 import inputs as I  # noqa: E402

FLUSH_BYTES = 256 << 20
WORKLOAD_TEXT = {
    "decode_128": "decode: 128 seqs, q_len 1, kv_len U[1024,8192], Hq 32 / Hkv 8, D 128, page 16, "
                  "bf16, 0.5*N(0,1), shuffled 1.25x page pool",
    "prefill_8x2048": "prefill: 8 fresh seqs q_len = kv_len = 2048, Hq 32 / Hkv 8, D 128, page 16, "
                      "bf16, N(0,1), shuffled 1.25x pool",
    "mixed_96d_4c": "mixed: 96 decode seqs kv log-U[512,16384] + 4 chunked seqs q_len 512 after "
                    "log-U[1024,8192] context, Hq 32 / Hkv 8, D 128, page 16, bf16, causal",
    "long_d256": "long context: 32 decode seqs kv 131072 + 4 prefill seqs 4096, Hq 16 / Hkv 4, "
                 "D 256, page 64, bf16, causal",
    "prefill_4x4096_d256": "prefill: 4 fresh seqs q_len = kv_len = 4096, Hq 16 / Hkv 4, D 256, page 64, "
                           "bf16, N(0,1), shuffled 1.25x pool (the prefill rows of the long-context batch)",
}


# ------------------------------------------------------------ work counting
def algorithmic(prob: I.Problem) -> dict:
    """Minimum bytes and FLOPs of one pass (see module docstring)."""
    e = 4 if prob.dtype == I.F32 else 2
    hq, hkv, d, p = prob.num_q_heads, prob.num_kv_heads, prob.head_dim, prob.page_size
    q = prob.q_lens.astype(np.int64)
    k = prob.kv_lens.astype(np.int64)
    t = int(q.sum())
    kv_read = int(k.sum()) * hkv * d * 2 * e
    cache_write = t * hkv * d * 2 * e
    q_out = 2 * t * hq * d * e
    lse = 4 * t * hq
    table = 4 * int(((k + p - 1) // p)[q > 0].sum())
    if prob.causal:
        pairs = q * (k - q) + q * (q + 1) // 2
    else:
        pairs = q * k
    flops = 4 * d * hq * int(pairs.sum())
    dec = q == 1
    dec_bytes = (int(k[dec].sum()) * hkv * d * 2 * e + int(dec.sum()) * hkv * d * 2 * e
                 + int(dec.sum()) * hq * d * e + 4 * int(((k[dec] + p - 1) // p).sum()))
    return dict(bytes=kv_read + cache_write + q_out + lse + table, flops=flops, tokens=t,
                decode_kernel_bytes=dec_bytes, prefill_flops=4 * d * hq * int(pairs[q > 1].sum()))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return dict(hbm=float(m["hbm_gbs"]), tc=float(m["bf16_tflops"]),
                    tc_sustained=float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, tc=1590.0, tc_sustained=1400.0, source="fallback")


PREFILL_KERNEL_OPTION = 0   # RPA_OPT_PREFILL_KERNEL of this run (--prefill-kernel)


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source has not changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(f"{kernel}/{workload}")
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    # the counters belong to the kernel that the RPA_OPT_PREFILL_KERNEL of the capture picks
    if PREFILL_KERNEL_OPTION != rec.get("prefill_kernel_option", 0):
        return None
    src = os.path.join(ROOT, rec["source"])
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    return rec["dram_bytes_per_launch"] if sha == rec["source_sha256"] else None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device)
            self.bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0),
                                             getattr(props, "pci_bus_id", 0),
                                             getattr(props, "pci_device_id", 0))
        except Exception:
            self.bus = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if self.bus:
            cmd += ["-i", self.bus]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ------------------------------------------------------------------ GPU arm
def device_problem(name: str, causal, device, max_seqs=None, head_shard=None) -> I.Problem:
    return I.make_workload(name, device=device, causal=causal, poison=False, max_seqs=max_seqs,
                           head_shard=head_shard)


def time_steps(prob, steps, warmup, flush, stream, profile=False):
    from ragged_paged_attention_03_b200 import binding
    out = torch.empty_like(prob.q)
    lse = torch.empty(prob.q.shape[0], prob.num_q_heads, dtype=torch.float32, device=prob.q.device)

    def call():
        binding.rpa_forward(prob.q, prob.k_new, prob.v_new, prob.k_cache, prob.v_cache,
                            prob.page_table, prob.cu_q_lens, prob.kv_lens, prob.distribution,
                            prob.scale, prob.causal, out, lse, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.add_(1)
            call()
        stream.synchronize()
        if profile:
            binding.rpa_profile_read()
            binding.rpa_profile_enable(True)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for a, b in evs:
            flush.add_(1)            # 256 MiB write evicts the step's data from L2
            a.record(stream)
            call()
            b.record(stream)
        stream.synchronize()
        if profile:
            binding.rpa_profile_enable(False)
    kern = binding.rpa_profile_read() if profile else None
    flags = binding.rpa_device_status(stream)
    if flags:
        raise RuntimeError(f"device error flags {flags:#x}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    return ms, kern


def time_graph(prob, steps, warmup, flush, stream):
    """rpa_forward_device (lengths in device memory, planned by a kernel)
    captured once in a CUDA graph and replayed every step.  Returns the mean
    device ms per step and the host microseconds one replay takes to launch."""
    from ragged_paged_attention_03_b200 import binding
    dev = prob.q.device
    out = torch.empty_like(prob.q)
    lse = torch.empty(prob.q.shape[0], prob.num_q_heads, dtype=torch.float32, device=dev)
    cu = torch.as_tensor(np.asarray(prob.cu_q_lens), dtype=torch.int32).to(dev)
    kv = torch.as_tensor(np.asarray(prob.kv_lens), dtype=torch.int32).to(dev)
    n = torch.tensor([prob.num_seqs], dtype=torch.int32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    dims = binding.make_dims(prob.q, prob.k_cache, prob.page_table)
    ws = torch.empty(binding.rpa_device_workspace_size(dims, prob.num_seqs), dtype=torch.uint8, device=dev)

    def call():
        binding.rpa_forward_device(prob.q, prob.k_new, prob.v_new, prob.k_cache, prob.v_cache,
                                   prob.page_table, cu, kv, n, prob.scale, prob.causal, out, ws,
                                   lse=lse, dev_flags=flags)

    with torch.cuda.stream(stream):
        call()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            call()
        for _ in range(warmup):
            flush.add_(1)
            graph.replay()
        stream.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        host = []
        for a, b in evs:
            flush.add_(1)
            a.record(stream)
            t0 = time.perf_counter()
            graph.replay()
            host.append(time.perf_counter() - t0)
            b.record(stream)
        stream.synchronize()
    if int(flags.item()):
        raise RuntimeError(f"device error flags {int(flags.item()):#x}")
    del graph
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    return ms, float(np.median(host)) * 1e6


def host_call_us(prob, calls, stream):
    """Host microseconds one host-planned rpa_forward call takes (planning,
    plan upload and launches), median over `calls`."""
    from ragged_paged_attention_03_b200 import binding
    out = torch.empty_like(prob.q)
    lse = torch.empty(prob.q.shape[0], prob.num_q_heads, dtype=torch.float32, device=prob.q.device)
    ts = []
    with torch.cuda.stream(stream):
        for _ in range(calls):
            t0 = time.perf_counter()
            binding.rpa_forward(prob.q, prob.k_new, prob.v_new, prob.k_cache, prob.v_cache,
                                prob.page_table, prob.cu_q_lens, prob.kv_lens, prob.distribution,
                                prob.scale, prob.causal, out, lse, stream=stream)
            ts.append(time.perf_counter() - t0)
            stream.synchronize()
    return float(np.median(ts)) * 1e6


def time_e2e(prob, steps, warmup, flush, stream):
    """Host buffers in, host buffers out, through rpa_forward_host: each step
    copies this step's Q, new K/V and page table from pinned host memory,
    runs the attention pass and copies out and lse back (the library overlaps
    the copies with the kernels, group by group), all inside the timed
    region.  The caches stay resident on the device."""
    from ragged_paged_attention_03_b200 import binding
    h = {k: getattr(prob, k).cpu().pin_memory() for k in ("q", "k_new", "v_new", "page_table")}
    h_out = torch.empty(prob.q.shape, dtype=prob.q.dtype).pin_memory()
    h_lse = torch.empty(prob.q.shape[0], prob.num_q_heads, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * 4

    def call():
        binding.rpa_forward_host(h["q"], h["k_new"], h["v_new"], prob.k_cache, prob.v_cache, h["page_table"],
                                 prob.cu_q_lens, prob.kv_lens, prob.distribution, prob.scale, prob.causal,
                                 h_out, h_lse, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.add_(1)
            call()
        stream.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for a, b in evs:
            flush.add_(1)
            a.record(stream)
            call()
            b.record(stream)
        stream.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs])), h2d, d2h


def metric_of(name):
    if name.startswith("decode"):
        return "decode HBM GB/s", "GB/s"
    if name.startswith("prefill"):
        return "prefill TFLOP/s", "TFLOP/s"
    if name.startswith("mixed"):
        return "mixed-batch tokens/s", "tokens/s"
    return "long-context HBM GB/s", "GB/s"


def rank_work(work: dict, world: int, shard: str) -> dict:
    """One rank's share of the job's work, as value_of counts it (value =
    world x a rank's share / time).  Replicas: each rank does the whole
    batch.  KV-head shards: bytes and FLOPs split over the ranks, but every
    rank serves all the batch's tokens (for its heads), so its share of the
    job's tokens is tokens / world."""
    if shard != "heads" or world == 1:
        return work
    return {**work, "tokens": work["tokens"] / world}


def value_of(name, work, ms, n):
    metric, unit = metric_of(name)
    if unit == "GB/s":
        return n * work["bytes"] / (ms * 1e-3) / 1e9
    if unit == "TFLOP/s":
        return n * work["flops"] / (ms * 1e-3) / 1e12
    return n * work["tokens"] / (ms * 1e-3)


def roofline(name, work, kern, pk, steps):
    """The dominant kernel class of the step against its own roofline: its
    device time per step (a class may launch more than once per step, e.g.
    decode for long and for packed short sequences)."""
    launches = {k: v for k, v in kern.items() if v[0] > 0}
    top = max(launches, key=lambda k: launches[k][1])
    n, total_ms = launches[top]
    avg_s = total_ms / steps * 1e-3
    if top == "prefill":
        achieved = work["prefill_flops"] / avg_s / 1e12
        r = {"bound": "tensor", "achieved": achieved, "peak": pk["tc"], "unit": "TFLOP/s",
             "peak_source": f"{pk['source']} bf16 dense (burst)"}
        b = work["bytes"] - work["decode_kernel_bytes"]
    else:
        b = work["decode_kernel_bytes"] if top == "decode" else work["bytes"]
        achieved = b / avg_s / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
             "peak_source": f"{pk['source']} HBM copy"}
    r["alg_bytes"] = b
    r["frac"] = r["achieved"] / r["peak"]
    r["kernel"] = top
    r["kernel_ms"] = total_ms / steps
    r["kernel_launches_per_step"] = n / steps
    r["traffic"] = traffic_for(top, name)
    r["kernel_share"] = {k: round(v[1] / sum(x[1] for x in launches.values()), 4)
                         for k, v in launches.items()}
    return r


# ----------------------------------------------------------- oracle (CPU)
def oracle_sample(prob_dev: I.Problem, budget_s: float):
    """Sequences of the workload for a bounded oracle run: decode sequences
    in order, then prefill sequences, until the estimated fp64 work fills
    about `budget_s` seconds of the host's cores."""
    import oracle
    rate = 0.4e9 * max(1, oracle.num_threads())          # fp64 multiply-adds / s, rough
    q = prob_dev.q_lens.astype(np.int64)
    k = prob_dev.kv_lens.astype(np.int64)
    pairs = q * (k - q) + q * (q + 1) // 2 if prob_dev.causal else q * k
    cost = 2.0 * pairs * prob_dev.num_q_heads * prob_dev.head_dim
    order = [s for s in range(prob_dev.num_seqs) if q[s] == 1] + \
            [s for s in range(prob_dev.num_seqs) if q[s] > 1]
    pick, acc = [], 0.0
    for s in order:
        if pick and acc + cost[s] > rate * budget_s:
            continue
        pick.append(s)
        acc += cost[s]
    return sorted(pick)


def run_oracle_sample(sub: I.Problem):
    import oracle
    kc = I.to_storage(sub.k_cache).copy()
    vc = I.to_storage(sub.v_cache).copy()
    args = (I.to_storage(sub.q), I.to_storage(sub.k_new), I.to_storage(sub.v_new))
    t0 = time.perf_counter()
    oracle.forward(*args, kc, vc, sub.page_table.numpy(), sub.cu_q_lens, sub.kv_lens, sub.scale,
                   sub.causal, sub.dtype)
    return time.perf_counter() - t0


def cpu_baseline(name, prob_dev, budget_s):
    import oracle
    seqs = oracle_sample(prob_dev, budget_s)
    sub = I.sub_problem(prob_dev, seqs)
    dt = run_oracle_sample(sub)
    work = algorithmic(sub)
    metric, unit = metric_of(name)
    v = value_of(name, work, dt * 1e3, 1)
    return {"value": v, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(seqs)} of {prob_dev.num_seqs} sequences "
                      f"({work['tokens']} new tokens, {work['bytes'] / 1e9:.3f} GB, "
                      f"{work['flops'] / 1e9:.1f} GFLOP), one fp64 oracle pass, {dt:.1f} s"}


# ------------------------------------------------------------ output lines
def _r(x, digits=4):
    """x rounded to `digits` significant digits (floats only)."""
    if isinstance(x, float):
        return float(f"{x:.{digits}g}") if math.isfinite(x) else x
    if isinstance(x, dict):
        return {k: _r(v, digits) for k, v in x.items()}
    if isinstance(x, list):
        return [_r(v, digits) for v in x]
    return x


def workload_line(line: dict) -> dict:
    """The short per-workload line: value, the dominant kernel against its
    roofline, and the end-to-end and graph-replay values in the same unit."""
    rf = line["roofline"]
    short = {"workload": line["workload"], "metric": line["metric"], "value": line["value"],
             "unit": line["unit"], "ms_per_step": line["ms_per_step"],
             "roofline": {"kernel": rf["kernel"], "frac": rf["frac"], "achieved": rf["achieved"],
                          "peak": rf["peak"], "unit": rf["unit"], "kernel_ms": rf["kernel_ms"],
                          "traffic": rf["traffic"], "alg_bytes": rf.get("alg_bytes")},
             "e2e": line["e2e"]["value"], "graph": line["device_planned_graph"]["value"]}
    return _r(short)


# --------------------------------------------------- cache-write ablation
def kernel_times(spec, steps, warmup, dev):
    """Per kernel class (launches, ms per step) of one workload, kernels run
    serially (a mixed batch's concurrent schedule would overlap the events)."""
    from ragged_paged_attention_03_b200 import binding as rb
    name, _, opt = spec.partition(":")
    prob = device_problem(name, False if opt == "noncausal" else None, dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    old = rb.rpa_set_option(rb.RPA_OPT_CONCURRENT_MIXED, -1)
    try:
        ms, kern = time_steps(prob, steps, warmup, flush, stream, profile=True)
    finally:
        rb.rpa_set_option(rb.RPA_OPT_CONCURRENT_MIXED, old)
    return {k: (v[0] / steps, v[1] / steps) for k, v in kern.items() if v[0] > 0}, ms


def ablate_write(args, dev):
    """The fused cache update's cost: each workload's kernel times with the
    library as built and with the timing-only build whose cache stores are
    compiled out, run in a child process that loads that build."""
    from ragged_paged_attention_03_b200 import build
    build.build()
    build.build(ablate_write=True)
    for spec in [w for w in args.workloads.split(",") if w]:
        with_w, step_w = kernel_times(spec, args.steps, args.warmup, dev)
        env = dict(os.environ, RPA_ABLATE_CACHE_WRITE="1")
        kopt = [] if args.prefill_kernel is None else ["--prefill-kernel", str(args.prefill_kernel)]
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--ablate-child", "--workloads", spec,
                            "--steps", str(args.steps), "--warmup", str(args.warmup)] + kopt,
                           env=env, capture_output=True, text=True, check=True)
        child = json.loads(r.stdout.strip().splitlines()[-1])
        without, step_wo = child["kern"], child["ms_per_step"]
        line = {"ablation": "fused cache write", "workload": spec,
                "kernel_ms_with_write": {k: v[1] for k, v in with_w.items()},
                "kernel_ms_without_write": {k: v[1] for k, v in without.items()},
                "step_ms_with_write": step_w, "step_ms_without_write": step_wo,
                "write_cost_frac": {k: (with_w[k][1] - without[k][1]) / with_w[k][1]
                                    for k in with_w if k in without and with_w[k][1] > 0}}
        print(json.dumps(_r(line)), flush=True)


# ----------------------------------------------------------------- main
def dist_setup(args, backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        if backend == "nccl":
            # each rank's GPU before the group forms, so that NCCL (and the
            # first barrier) binds this rank to its own device
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks: each rank runs its own replica, and the
    slowest one sets the whole job's step time.  Every rank must call it at
    the same point (it is a collective when more than one rank runs)."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workloads", default="decode_128,prefill_8x2048,prefill_8x2048:noncausal,"
                                           "mixed_96d_4c,long_d256,prefill_4x4096_d256")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--max-seqs", type=int, default=None,
                    help="keep only the first N sequences of each workload (profiler captures)")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="replicas: every GPU runs the whole batch (weak scaling); heads: every GPU "
                         "runs its Hkv/N KV heads of the same batch (strong scaling; no collective)")
    ap.add_argument("--prefill-kernel", type=int, default=None,
                    help="RPA_OPT_PREFILL_KERNEL (0, the default: two tiles per CTA at head_dim 128, CTA "
                         "pairs at 256; 1: two tiles per CTA, one tile per CTA at 256; 2: CTA pairs; 3: one "
                         "tile per CTA at 128)")
    ap.add_argument("--ablate-write", action="store_true",
                    help="time each workload's kernels with and without the fused cache stores "
                         "(a separate timing-only build; off by default)")
    ap.add_argument("--ablate-child", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.prefill_kernel is not None:
        global PREFILL_KERNEL_OPTION
        from ragged_paged_attention_03_b200 import binding as rb
        rb.rpa_set_option(rb.RPA_OPT_PREFILL_KERNEL, args.prefill_kernel)
        PREFILL_KERNEL_OPTION = args.prefill_kernel
    if args.ablate_write or args.ablate_child:
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(dev)
        if args.ablate_child:
            if os.environ.get("RPA_ABLATE_CACHE_WRITE") != "1":
                raise SystemExit("--ablate-child runs only under RPA_ABLATE_CACHE_WRITE=1")
            kern, ms = kernel_times(args.workloads.split(",")[0], args.steps, args.warmup, dev)
            print(json.dumps({"kern": kern, "ms_per_step": ms}), flush=True)
        elif int(os.environ.get("RANK", "0")) == 0:
            ablate_write(args, dev)
        return
    world, rank, local = dist_setup(args)
    n = world
    wl = [w for w in args.workloads.split(",") if w]

    if args.impl == "reference":
        if rank != 0:
            return
        name = wl[0].split(":")[0]
        prob = I.make_workload(name, device="cpu", poison=False)
        seqs = oracle_sample(prob, max(1.0, 150.0 / max(1, args.steps + args.warmup)))
        sub = I.sub_problem(prob, seqs)
        for _ in range(args.warmup):
            run_oracle_sample(sub)
        times = [run_oracle_sample(sub) for _ in range(args.steps)]
        work = algorithmic(sub)
        ms = float(np.mean(times)) * 1e3
        metric, unit = metric_of(name)
        v = value_of(name, work, ms, 1)
        import oracle
        line = {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": n,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic",
                "config": {"workload": WORKLOAD_TEXT[name], "sample_seqs": len(seqs)},
                "cpu_baseline": {"value": v, "unit": unit, "cores": oracle.num_threads(),
                                 "kind": "oracle",
                                 "sample": f"{len(seqs)} of {prob.num_seqs} sequences per step"},
                "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    from ragged_paged_attention_03_b200 import build
    if rank == 0 and not os.path.exists(os.path.join(ROOT, "ragged_paged_attention_03_b200",
                                                     "librpa_b200.so")):
        build.build()
    if world > 1:
        torch.distributed.barrier()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    pk = peaks()
    clocks = ClockSampler(local)
    results = []
    cpu_base = None
    for i, spec in enumerate(wl):
        name, _, opt = spec.partition(":")
        causal = False if opt == "noncausal" else None
        prob = device_problem(name, causal, dev, args.max_seqs,
                              head_shard=(rank, world) if args.shard == "heads" else None)
        work = rank_work(algorithmic(prob), world, args.shard)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        # a batch with prefill and decode rows runs them concurrently (two
        # streams); its per-kernel event times overlap, so the kernel
        # rooflines of such a step come from a serial run of the same step
        mixed = work["prefill_flops"] > 0 and work["decode_kernel_bytes"] > 0
        if i == 0:
            clocks.start()
        # the step as a user runs it: no per-kernel events between the launches
        ms, _ = time_steps(prob, args.steps, args.warmup, flush, stream, profile=False)
        if i == 0:
            clk = clocks.stop()
        # per-kernel device times from a second pass over the same steps with
        # the library's CUDA-event tracing on (events on the launching
        # stream around every kernel); a batch with prefill and decode rows
        # runs them serially in this pass, since its step runs them
        # concurrently and their events would overlap
        from ragged_paged_attention_03_b200 import binding as rb
        old = rb.rpa_set_option(rb.RPA_OPT_CONCURRENT_MIXED, -1) if mixed else None
        try:
            traced_ms, kern = time_steps(prob, args.steps, args.warmup, flush, stream, profile=True)
        finally:
            if mixed:
                rb.rpa_set_option(rb.RPA_OPT_CONCURRENT_MIXED, old)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(ms, dev)
        if world > 1:
            torch.distributed.barrier()
        e2e_ms, h2d, d2h = time_e2e(prob, max(10, args.steps // 4), 3, flush, stream)
        e2e_ms = max_over_ranks(e2e_ms, dev)
        g_ms, g_host_us = time_graph(prob, args.steps, args.warmup, flush, stream)
        g_ms = max_over_ranks(g_ms, dev)
        h_host_us = host_call_us(prob, 20, stream)
        metric, unit = metric_of(name)
        line = {"metric": metric, "value": value_of(name, work, ms, n), "unit": unit,
                "ms_per_step": ms,
                "workload": name + ("" if prob.causal else " (non-causal)"),
                "config": {"workload": WORKLOAD_TEXT[name] + ("" if prob.causal else ", non-causal"),
                           "l2": "flushed between steps (256 MiB write)",
                           "tokens": work["tokens"], "bytes": work["bytes"],
                           "flops": work["flops"]},
                "roofline": {**roofline(name, work, kern, pk, args.steps),
                             "kernel_timing": (f"serial traced pass of the same steps ({traced_ms:.4f} ms per step), "
                                               "since the step itself runs prefill and decode concurrently")
                             if mixed else f"traced pass of the same steps ({traced_ms:.4f} ms per step)"},
                "e2e": {"value": value_of(name, work, e2e_ms, n), "unit": unit,
                        "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": int(sum(v[0] for v in kern.values())),
                "device_planned_graph": {"value": value_of(name, work, g_ms, n), "unit": unit,
                                         "ms_per_step": g_ms, "host_us_per_replay": g_host_us,
                                         "host_us_per_host_planned_call": h_host_us}}
        if rank == 0 and i == 0 and world == 1:
            cpu_base = cpu_baseline(name, prob, args.cpu_budget)
        if rank == 0:
            print(json.dumps(workload_line(line)), flush=True)
        results.append(line)
        del prob
        torch.cuda.empty_cache()
    if rank == 0:
        head = results[0]
        out = {"metric": head["metric"], "value": head["value"], "unit": head["unit"],
               "n_gpus": n, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": head["ms_per_step"], "higher_is_better": True,
               "scaling": "strong" if args.shard == "heads" else "weak",
               "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
               "config": {**head["config"],
                          "parallelism": "1 GPU" if n == 1 else
                          (f"KV-head shards x{n}" if args.shard == "heads" else f"replicas x{n}")},
               "roofline": head["roofline"], "e2e": head["e2e"],
               "gpu_launches": head["gpu_launches"], "clocks": clk,
               "cpu_baseline": cpu_base,
               "workloads": [r["workload"] for r in results]}
        print(json.dumps(_r(out, 6)), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
