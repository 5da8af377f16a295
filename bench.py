"""Benchmark of the recurrent gated-delta-rule decode step on B200.

One step = one call of the fused-gate decode (every step of the op: gather the
state slot, gate prologue, decay, memory read, delta update, output, padding,
scatter) over one batch of seeded synthetic inputs of the large-batch workload
(B=512 items, 64 heads, T=1, 64x512 bfloat16 state per head, 2 GiB pool).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdr|reference]
                    [--all-workloads] [--op decode|gate]

Prints one JSON line (rank 0); --all-workloads adds one line for each of the
single-sequence, grouped-head and speculative workloads after it. Multi-GPU:
one process per GPU under torchrun; one logical call of N x 512 items is
split by item over the ranks (each holds its items' pool slots; weak
scaling, no collective on the data path); the timed region is bracketed by
barriers and the max over ranks is reported.

``--impl reference`` times the CPU oracle (fp64 NumPy) on this machine's host
cores on a bounded sample of the same workload; it is a deliberately slow
baseline, not a target.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gated_delta_rule_recurrent_b200 import distributed, metrics, workloads  # noqa: E402

METRIC = "decode tokens/s and achieved HBM GB/s vs ~8 TB/s peak for gated-delta step"
PREFILL_METRIC = "prefill tokens/s and achieved HBM GB/s (long-prompt gated-delta recurrence)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
DEFAULT_WORKLOAD = 4
# What the large-batch kernel's traffic record depends on: the single-token
# kernel's headers, and in gdr_api.cu its launch configuration (the section
# between the two markers) and its tile-width table.
KERNEL_SOURCE_FILES = ("gated_delta_rule_recurrent_b200/csrc/gdr_decode.cuh",
                       "gated_delta_rule_recurrent_b200/csrc/gdr_ptx.cuh",
                       "gated_delta_rule_recurrent_b200/csrc/gdr_decode_tma.cuh")
LAUNCH_SOURCE = "gated_delta_rule_recurrent_b200/csrc/gdr_api.cu"
LAUNCH_SECTION = ("// ---------------------------------------------------------------- TMA path",
                  "// ---------------------------------------------------------------- chunk path")
LAUNCH_TABLE = "static const SliceKernel k64_one[]"
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "decode_gated_B512_H64_64x512_dram.txt")


# --------------------------------------------------------------------------- helpers

def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            peaks = json.load(f)
        return float(peaks["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    import hashlib

    h = hashlib.sha256()
    for rel in KERNEL_SOURCE_FILES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    with open(os.path.join(ROOT, LAUNCH_SOURCE)) as f:
        api = f.read()
    a, b = api.index(LAUNCH_SECTION[0]), api.index(LAUNCH_SECTION[1])
    h.update(api[a:b].encode())
    t = api.index(LAUNCH_TABLE)
    h.update(api[t:api.index(";", t)].encode())
    return h.hexdigest()


def decode_kernel_name(w, layout):
    """The kernel the library launches for this workload (one per call)."""
    if w.D_k == 128 and w.D_v % 128 == 0:
        return "gdr::decode_chunk_tc_kernel"
    if w.T == 1:
        return "gdr::decode_tma_kernel" if layout == "kv" else "gdr::decode_rows_kernel"
    return "gdr::decode_chunk_kernel"


def recorded_traffic(workload_name, layout):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    this workload and layout with the current kernel source; else None."""
    try:
        rec = {}
        with open(TRAFFIC_RECORD) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    rec[k.strip()] = v.strip()
        if rec.get("kernel_source_sha256") != kernel_source_hash():
            return None
        if rec.get("workload") != workload_name or rec.get("state_layout", "kv") != layout:
            return None
        return int(float(rec["dram_bytes_per_launch"]))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every ``period_ms``."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, period_ms: int = 10):
        self.samples = []  # (host time, sm_mhz, max_mhz, power, reasons set)
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            cmd = ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}",
                   "--format=csv,noheader,nounits", f"-lms={period_ms}"]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, smax, power = float(parts[0]), float(parts[1]), float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                     "sw_power_cap"]
            reasons = {n for n, v in zip(names, parts[4:8]) if v.lower().startswith("active")}
            self.samples.append((time.time(), sm, smax, power, reasons))

    def wait_first(self, timeout=10.0):
        t0 = time.time()
        while self.proc is not None and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.02)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window": "unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if not inside:  # timed region shorter than the sampling period
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            window = "nearest to timed region"
        reasons = sorted(set().union(*[s[4] for s in inside]))
        return {"sm_mhz": float(np.median([s[1] for s in inside])),
                "sm_max_mhz": max(s[2] for s in inside),
                "power_w_max": max(s[3] for s in inside),
                "reasons": reasons, "samples": len(inside), "window": window}


def oracle_tokens_per_s(x, gated, items_per_call, budget_s, items_order=None):
    """Time the fp64 oracle on consecutive chunks of batch items until ``budget_s``."""
    from threadpoolctl import threadpool_limits

    from oracle.gdr_oracle import (recurrent_gated_delta_rule,
                                   recurrent_gated_delta_rule_gated)

    B = x["query"].shape[0]
    order = np.arange(B) if items_order is None else items_order
    asl = x["actual_seq_lengths"].to(torch.int64).numpy()
    idx = x["ssm_state_indices"].to(torch.int64).numpy()
    T = x["query"].shape[2]

    def f64(t):
        return t.to(torch.float64).numpy()

    tokens = 0
    items_done = 0
    elapsed = 0.0
    pos = 0
    with threadpool_limits(limits=1):
        while elapsed < budget_s:
            sel = order[pos:pos + items_per_call]
            if sel.size == 0:
                pos = 0
                continue
            pos += items_per_call
            st = torch.from_numpy(idx[sel])
            pool = f64(x["state_pool"][st])  # gathered slots (inputs, not timed)
            args = {k: f64(x[k][torch.from_numpy(sel)]) for k in
                    ("query", "key", "value", "gk", "a", "b", "beta", "g")}
            local_idx = np.arange(sel.size)
            t0 = time.perf_counter()
            if gated:
                recurrent_gated_delta_rule_gated(
                    args["query"], args["key"], args["value"], args["a"], args["b"],
                    f64(x["dt_bias"]), f64(x["decay_scale"]), pool, asl[sel], local_idx,
                    args["gk"], asl[sel], x["scale_value"])
            else:
                recurrent_gated_delta_rule(
                    args["query"], args["key"], args["value"], args["beta"], pool, asl[sel],
                    local_idx, args["g"], args["gk"], asl[sel], x["scale_value"])
            elapsed += time.perf_counter() - t0
            tokens += int(np.clip(asl[sel], 0, T).sum())
            items_done += sel.size
    return tokens / elapsed, tokens, items_done, elapsed


def measure_e2e(args, w, x, xd, out, dev, step, barrier, max_over_ranks, world, n_tokens):
    """End to end through the public API with host buffers.

    Every timed step copies its per-token inputs from pinned host memory to the
    device, runs the decode call, and copies its output back to pinned host
    memory; the state pool stays resident, as it does in serving. Steps are
    pipelined over three streams with double-buffered device inputs and
    outputs, so step i+1's upload and step i-1's download overlap step i's
    kernel; the state pool's updates stay in call order on the compute stream.
    """
    gated = w.gated
    per_step = ["query", "key", "value", "gk", "actual_seq_lengths", "ssm_state_indices",
                "num_accepted_tokens"] + (["a", "b"] if gated else ["beta", "g"])
    host = {k: x[k].pin_memory() for k in per_step}
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(host[k].numel() * host[k].element_size() for k in per_step)
    d2h = host_out[0].numel() * host_out[0].element_size()
    dev_in = [{k: torch.empty_like(xd[k]) for k in per_step} for _ in range(2)]
    dev_out = [out, torch.empty_like(out)]
    up, comp, down = (torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    ev_in = [torch.cuda.Event() for _ in range(2)]         # inputs of a slot uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]       # kernel done with a slot's inputs
    ev_done = [torch.cuda.Event() for _ in range(2)]       # kernel wrote a slot's output
    ev_fetched = [torch.cuda.Event() for _ in range(2)]    # output of a slot downloaded
    for e in ev_used + ev_fetched:
        e.record(torch.cuda.current_stream(dev))

    def run(n):
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(up):
                up.wait_event(ev_used[j])
                for k in per_step:
                    dev_in[j][k].copy_(host[k], non_blocking=True)
                ev_in[j].record(up)
            with torch.cuda.stream(comp):
                comp.wait_event(ev_in[j])
                comp.wait_event(ev_fetched[j])
                step(o=dev_out[j], inputs=dev_in[j])
                ev_used[j].record(comp)
                ev_done[j].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[j])
                host_out[j].copy_(dev_out[j], non_blocking=True)
                ev_fetched[j].record(down)

    run(max(1, args.warmup))
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(up)
    run(args.steps)
    down.wait_event(ev_fetched[(args.steps - 1) % 2])
    e1.record(down)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    tokens = distributed.sum_over_ranks(n_tokens * args.steps, dev)
    return {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": e2e_ms / args.steps,
            "pipelining": "upload, kernel and download on 3 streams, double-buffered"}


# --------------------------------------------------------------------------- CUDA arm

def _place(x, dev, layout):
    """Device copies of one call's inputs (the pool in the requested layout)."""
    xd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    if layout == "vk":  # the same state, stored [pool, H_v, D_v, D_k]
        xd["state_pool"] = xd["state_pool"].transpose(2, 3).contiguous()
    return xd


def _capture(step, K, dev):
    """The K steps captured once as a CUDA graph (the library's per-call host
    work, configuration and tensor maps, happens at capture; a replay queues
    only the K kernel launches)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(g, stream=s):
        for i in range(K):
            step(i)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    return g


def _timed_region(step, K, stream, dev, barrier, max_over_ranks, graph=None):
    """K steps back to back between two events on the launching stream,
    bracketed by a barrier and a device synchronisation on both sides (as one
    replay of ``graph`` when given); the max over ranks of the region, and the
    host times of its ends."""
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    host_t0 = time.time()
    r0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(K):
            step(i)
    r1.record(stream)
    torch.cuda.synchronize(dev)
    host_t1 = time.time()
    barrier()
    return max_over_ranks(r0.elapsed_time(r1)), host_t0, host_t1


def bench_decode_workload(args, wkey, ctx, with_e2e, cpu_seconds, op="decode"):
    """One JSON line for one decode (or, op="prefill", long-prompt) workload on
    this rank's GPU."""
    import gated_delta_rule_recurrent_b200 as gdr

    world, rank, dev, barrier, max_over_ranks, sampler = ctx
    w = workloads.workload(wkey)
    if args.batch is not None and wkey == args.workload:
        w = w.replace(name=f"{w.name}_B{args.batch}", B=args.batch, pool=args.batch)
    gated = w.gated
    # One logical call of N x B items over N x pool slots, split by item
    # (distributed.shard_call's contiguous item split): rank r holds items
    # [r B, (r + 1) B) and the slots they name. Its share is drawn from its own
    # seed, so no rank builds the others' inputs.
    x = workloads.make_inputs(w, seed=distributed.rank_seed(w.seed, rank))
    lengths = x["actual_seq_lengths"].tolist()
    n_tokens = int(sum(min(max(L, 0), w.T) for L in lengths))
    step_bytes = metrics.algorithmic_bytes(w.B, w.H_qk, w.H_v, w.T, w.D_k, w.D_v, lengths,
                                           gated)
    # Every step must read its inputs from HBM: a workload smaller than a few
    # L2s rotates over copies of its inputs and pool that together exceed it.
    n_copies = max(1, min(64, math.ceil(3 * L2_BYTES / step_bytes)))
    copies = [_place(x, dev, args.layout) for _ in range(n_copies)]
    outs = [torch.empty(w.B, w.H_v, w.T, w.D_v, dtype=torch.bfloat16, device=dev)
            for _ in range(n_copies)]
    stream = torch.cuda.current_stream(dev)

    def call(z, o):
        if op == "prefill":
            if gated:
                gdr.prefill_gated(z["query"], z["key"], z["value"], z["a"], z["b"],
                                  z["dt_bias"], z["decay_scale"], z["state_pool"],
                                  z["actual_seq_lengths"], z["ssm_state_indices"], z["gk"],
                                  z["num_accepted_tokens"], z["scale_value"], out=o)
            else:
                gdr.prefill(z["query"], z["key"], z["value"], z["beta"], z["state_pool"],
                            z["actual_seq_lengths"], z["ssm_state_indices"], z["g"], z["gk"],
                            z["num_accepted_tokens"], z["scale_value"], out=o)
        elif gated:
            gdr.decode_gated(z["query"], z["key"], z["value"], z["a"], z["b"],
                             z["dt_bias"], z["decay_scale"], z["state_pool"],
                             z["actual_seq_lengths"], z["ssm_state_indices"], z["gk"],
                             z["num_accepted_tokens"], z["scale_value"], out=o,
                             state_layout=args.layout)
        else:
            gdr.decode(z["query"], z["key"], z["value"], z["beta"], z["state_pool"],
                       z["actual_seq_lengths"], z["ssm_state_indices"], z["g"], z["gk"],
                       z["num_accepted_tokens"], z["scale_value"], out=o,
                       state_layout=args.layout)

    def step(i):
        call(copies[i % n_copies], outs[i % n_copies])

    # ---- kernel-resident timing: inputs already in HBM
    for i in range(max(args.warmup, n_copies)):
        step(i)
    torch.cuda.synchronize(dev)
    kernel = gdr.last_launch()
    K = args.steps
    # Events only at the two ends of the region: the steps run back to back
    # (the host enqueues a call in ~25 us, ahead of the device), one decode
    # launch per step, so the average launch duration is the region over the
    # launches. (An event pair around every launch leaves the device idle for
    # a few microseconds between launches, which a short step would count.)
    # The steps are replayed from a CUDA graph: a small step is shorter than the
    # ~25 us the Python binding takes to queue a call, and a graph is how a
    # serving loop issues it. (--no-graph times direct calls instead.)
    graph = None if args.no_graph else _capture(step, K, dev)
    region_ms, host_t0, host_t1 = _timed_region(step, K, stream, dev, barrier, max_over_ranks,
                                                graph)
    clocks = sampler.summary(host_t0, host_t1)
    # the same region again, back to back: its spread shows the run's noise
    repeats = [_timed_region(step, K, stream, dev, barrier, max_over_ranks, graph)[0] / K
               for _ in range(args.repeats)]
    del graph
    launches = K  # one kernel per step (the decode kernel)
    total_tokens = distributed.sum_over_ranks(n_tokens * K, dev)
    kernel_ms = region_ms / launches

    # ---- end to end through the public API: pinned host inputs copied in and
    # the output copied back every step, inside the timed region. The state
    # pool stays resident on the device, as it does in serving.
    e2e = None
    if with_e2e:
        xd = copies[0]
        out = outs[0]

        def e2e_step(o=out, inputs=None):
            call({**xd, **inputs} if inputs is not None else xd, o)

        e2e = measure_e2e(args, w, x, xd, out, dev, e2e_step, barrier, max_over_ranks, world,
                          n_tokens)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, toks, items, secs = oracle_tokens_per_s(x, gated,
                                                     items_per_call=1 if op == "prefill" else 8,
                                                     budget_s=cpu_seconds)
        cpu = {"value": tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{items} of {w.B} batch items ({toks} tokens) of the same "
                         f"workload, fp64 NumPy, 1 thread, {secs:.1f} s of oracle time"}
    del copies, outs

    peak, peak_kind = measured_hbm_peak()
    achieved = step_bytes / (kernel_ms / 1e3) / 1e9
    value = total_tokens / (region_ms / 1e3)
    l2 = (f"inputs larger than L2: {step_bytes / 1e9:.2f} GB per step vs "
          f"{L2_BYTES / 2**20:.0f} MiB L2, no flush" if n_copies == 1 else
          f"{step_bytes / 1e6:.1f} MB per step: steps rotate over {n_copies} copies of the "
          f"inputs and pool ({n_copies * step_bytes / 1e6:.0f} MB, over 3x the "
          f"{L2_BYTES / 2**20:.0f} MiB L2), no flush")
    return {
        "metric": METRIC if op == "decode" else PREFILL_METRIC,
        "op": op,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": region_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "H_qk": w.H_qk, "H_v": w.H_v, "T": w.T,
            "D_k": w.D_k, "D_v": w.D_v, "pool": w.pool,
            "tokens_per_step": n_tokens,
            "gate": "fused" if gated else "none",
            "storage": "bf16 state/q/k/v/out, fp32 g/gk",
            "state_layout": "[pool, H_v, D_k, D_v]" if args.layout == "kv"
                            else "[pool, H_v, D_v, D_k]",
            "l2": l2,
            "launch": ("one CUDA graph replay of the K steps" if not args.no_graph
                       else "K direct calls through the Python binding"),
            "parallelism": f"one call of {world} x {w.B} items split by item over {world} "
                           f"rank(s), no collective",
        },
        "achieved_hbm_gbs": achieved,
        "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
        "repeat_ms_per_step": {
            "n": len(repeats), "median": float(np.median(repeats)) if repeats else None,
            "min": min(repeats) if repeats else None, "max": max(repeats) if repeats else None,
            "note": f"{len(repeats)} more regions of {K} steps right after the timed one"},
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": f"{peak_kind} copy bandwidth",
            "kernel": ("gdr::prefill_tc_kernel" if op == "prefill"
                       else decode_kernel_name(w, args.layout)), "kernel_ms": kernel_ms,
            "kernel_form": kernel,
            "bytes_per_launch": step_bytes,
            "traffic": recorded_traffic(w.name, args.layout) if n_copies == 1 else None,
        },
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }


def run_gdr(args):
    import torch.distributed as dist

    world, rank, local = distributed.rank_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    from gated_delta_rule_recurrent_b200 import binding

    binding.lib()  # fail loudly now if the library is missing

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    def max_over_ranks(v):
        return distributed.max_over_ranks(v, dev)

    sampler = ClockSampler(local, period_ms=10)
    sampler.wait_first()
    ctx = (world, rank, dev, barrier, max_over_ranks, sampler)
    if args.op == "prefill":
        lines = [bench_decode_workload(args, "prefill", ctx, False, args.cpu_seconds,
                                       op="prefill")]
    else:
        lines = [bench_decode_workload(args, args.workload, ctx, not args.no_e2e,
                                       args.cpu_seconds)]
    if args.all_workloads and args.op == "decode":
        for wk in (1, 2, 3):
            if wk != args.workload:
                lines.append(bench_decode_workload(args, wk, ctx, False,
                                                   min(args.cpu_seconds, 5.0)))
    sampler.stop()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        for line in lines:
            print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- oracle arm

def run_reference(args):
    world, rank, _ = distributed.rank_env()
    if rank != 0:
        return  # rank 0 alone times the CPU oracle
    w = workloads.workload(args.workload)
    if args.batch is not None:
        w = w.replace(name=f"{w.name}_B{args.batch}", B=args.batch, pool=args.batch)
    x = workloads.make_inputs(w)
    n_steps = args.warmup + args.steps
    budget_total = args.reference_seconds
    per_step_budget = budget_total / max(1, n_steps)
    # calibrate: items per step so that every step is a bounded sample
    tps, _, _, _ = oracle_tokens_per_s(x, w.gated, items_per_call=1, budget_s=0.5)
    items_per_step = max(1, int(per_step_budget * tps / max(1, w.T)))
    items_per_step = min(items_per_step, w.B)
    order = np.arange(w.B)
    tokens = 0
    secs = 0.0
    for i in range(n_steps):
        sel = np.roll(order, -i * items_per_step)[:items_per_step]
        _, toks, _, el = oracle_tokens_per_s(x, w.gated, items_per_call=items_per_step,
                                             budget_s=1e-9, items_order=sel)
        if i >= args.warmup:
            tokens += toks
            secs += el
    value = tokens / secs
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H_qk": w.H_qk, "H_v": w.H_v, "T": w.T,
                   "D_k": w.D_k, "D_v": w.D_v, "pool": w.pool,
                   "gate": "fused" if w.gated else "none",
                   "sample_items_per_step": items_per_step},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{items_per_step} of {w.B} batch items per step, "
                                   f"fp64 NumPy oracle, 1 thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_gate(args):
    """The standalone LinearAttentionGate op on one GPU: one JSON line of its own
    (elements per second, and achieved HBM GB/s against the measured copy peak)."""
    import gated_delta_rule_recurrent_b200 as gdr
    from gated_delta_rule_recurrent_b200 import binding

    binding.lib()  # fail loudly now if the library is missing
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dtype = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[args.gate_dtype]
    shape = tuple(int(v) for v in args.gate_shape.split("x"))
    x = workloads.make_gate_inputs(shape, dtype, seed=2024)
    xd = {k: v.to(dev) for k, v in x.items()}
    decay = torch.empty_like(xd["a"])
    beta = torch.empty_like(xd["a"])
    n = xd["a"].numel()
    esize = xd["a"].element_size()
    step_bytes = 4 * n * esize + 2 * 4 * shape[-1]  # a, b in; decay, beta out; per-head vectors

    def step():
        gdr.linear_attention_gate(xd["a"], xd["dt_bias"], xd["decay_scale"], b=xd["b"],
                                  decay=decay, beta=beta)

    sampler = ClockSampler(0)
    sampler.wait_first()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    stream = torch.cuda.current_stream(dev)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    host_t0 = time.time()
    r0.record(stream)
    for i in range(K):  # back to back, events at the region's ends only
        step()
    r1.record(stream)
    torch.cuda.synchronize(dev)
    host_t1 = time.time()
    clocks = sampler.summary(host_t0, host_t1)
    sampler.stop()
    region_ms = r0.elapsed_time(r1)
    kernel_ms = region_ms / K  # per step: the vector launch (and the tail launch, if any)
    peak, peak_src = measured_hbm_peak()
    achieved = step_bytes / (kernel_ms * 1e-3) / 1e9
    # the fp64 oracle on a bounded sample of rows, one thread
    cpu = None
    if not args.no_cpu_baseline:
        from threadpoolctl import threadpool_limits

        from oracle.gdr_oracle import linear_attention_gate as oracle_gate
        a64 = x["a"].reshape(-1, shape[-1]).double().numpy()
        b64 = x["b"].reshape(-1, shape[-1]).double().numpy()
        dtb, dsc = x["dt_bias"].double().numpy(), x["decay_scale"].double().numpy()
        rows = min(a64.shape[0], 4096)
        done, t_cpu = 0, 0.0
        with threadpool_limits(limits=1):
            while t_cpu < args.cpu_seconds:
                lo = (done // shape[-1]) % a64.shape[0]
                t0 = time.perf_counter()
                oracle_gate(a64[lo:lo + rows], dtb, dsc, b64[lo:lo + rows])
                t_cpu += time.perf_counter() - t0
                done += rows * shape[-1]
        cpu = {"value": done / t_cpu, "unit": "elements/s", "cores": 1, "kind": "oracle",
               "sample": f"{rows}-row chunks of the same tensor for {t_cpu:.1f} s"}
    line = {
        "metric": "LinearAttentionGate elements/s (standalone gate op)",
        "op": "gate", "value": n * K / (region_ms * 1e-3), "unit": "elements/s", "n_gpus": 1,
        "steps": K, "warmup": args.warmup, "ms_per_step": region_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": args.gate_dtype, "data": "synthetic",
        "config": {"workload": f"gate_{args.gate_shape}_{args.gate_dtype}", "shape": list(shape),
                   "beta": True,
                   "l2": f"inputs larger than L2: {step_bytes / 1e9:.2f} GB per step vs 126 MiB "
                         "L2, no flush" if step_bytes > 126 * 2**20 else
                         f"{step_bytes / 1e6:.1f} MB per step, within L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": "gdr::gate_vec_kernel", "kernel_ms": kernel_ms,
                     "bytes_per_launch": step_bytes, "traffic": None},
        "e2e": None, "gpu_launches": K, "clocks": clocks, "cpu_baseline": cpu,
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("gdr", "reference"), default="gdr")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    type=lambda s: int(s) if s.isdigit() else s)
    ap.add_argument("--batch", type=int, default=None,
                    help="override B (and the pool size) of the workload, e.g. for a small "
                         "profiling case of the same kernel")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time K direct calls instead of one CUDA-graph replay of them")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    ap.add_argument("--op", choices=("decode", "gate", "prefill"), default="decode",
                    help="decode: the decode step (the default line); gate: the standalone "
                         "LinearAttentionGate op; prefill: the long-prompt recurrence "
                         "(gdr_prefill_gated); each a line of its own")
    ap.add_argument("--gate-shape", default="32768x8x64",
                    help="shape of a and b for --op gate, heads last")
    ap.add_argument("--gate-dtype", choices=("f32", "f16", "bf16"), default="bf16")
    ap.add_argument("--all-workloads", action="store_true",
                    help="after the default line, one line for each of workloads 1-3 (the "
                         "single-sequence, grouped-head and speculative decode workloads)")
    ap.add_argument("--repeats", type=int, default=5,
                    help="extra timed regions after the main one, reported as "
                         "repeat_ms_per_step (the main region alone gives ms_per_step)")
    ap.add_argument("--layout", choices=("kv", "vk"), default="kv",
                    help="state pool layout: kv = [pool, H_v, D_k, D_v] (the op page's), "
                         "vk = [pool, H_v, D_v, D_k]")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "gdr":
        raise SystemExit("--warmup must be >= 3")
    if args.op == "gate":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "op": "gate",
                              "unavailable": "the gate op's reference is the oracle; "
                                             "see the cpu_baseline key of the gate line"}))
        else:
            run_gate(args)
    elif args.impl == "reference" and args.op == "prefill":
        print(json.dumps({"impl": "reference", "op": "prefill",
                          "unavailable": "the prefill op's reference is the oracle; see the "
                                         "cpu_baseline key of the prefill line"}))
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gdr(args)


if __name__ == "__main__":
    main()
