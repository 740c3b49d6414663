"""Benchmark: prefill of the 56-execution looped hybrid stack (9B shape, bf16) on B200.

Workload (default): the full 9B-shape stack with random-init bf16 weights -- vocab
248,320 embedding + LM head, 32 stored layers run as 56 executions (4 + 24x2 + 4),
hidden 4096, FFN 12288, 3:1 GDN/GQA groups, two-stream mHC with FP32 routing --
prefill of batch 1 x 8192 uniform random token ids.  One step = one prefill (all
56 executions, final norm, LM head on the last position) from an empty cache.

`python bench.py [--gpus N --steps K --warmup W]` prints one JSON line.  With
--gpus N > 1 it runs under torchrun as N independent replicas (the forward pass
has no exchange step), one process per GPU; time is the max over ranks.
`--impl reference` times the CPU oracle instead, on a bounded sample.

The same line carries two more legs of the same stack: "decode" (batch 64 over
32,768-token contexts, 256 greedy steps) and "long_prefill" (batch 1, 131,072 tokens).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SEQ, BATCH = 8192, 1
WORKLOAD = "9B-shape looped hybrid stack, 56 executions, prefill B=1 T=8192, bf16, random-init weights"


def load_peaks():
    """Measured B200 peaks of this machine (driver-written), else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device):
        import torch
        try:
            self.index = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.index = str(device.index or 0)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(T=64, seed=0):
    """The CPU oracle on a bounded sample of the workload: one full-width group (3 GDN + 1 GQA
    layers inside the two-stream mHC) on T tokens.  Returns (seconds, tokens, executions)."""
    import numpy as np
    import torch

    import synth
    from oracle import model as omodel
    s = synth.GROUP
    W = omodel.Weights(synth.make_weights(s, seed=seed))
    for name, _, _ in synth.weight_names(s):      # widen the weights before timing (not oracle work)
        W[name]
    h = synth.normal((1, T, s.d), 1.0, seed, "hidden").to(torch.bfloat16)
    t0 = time.perf_counter()
    omodel.forward_hidden(s, W, h)
    dt = time.perf_counter() - t0
    return dt, T, 4


def cpu_cores():
    """Threads the oracle's numpy BLAS uses (what the all-core number ran on)."""
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
        return int(n)
    except Exception:
        return os.cpu_count()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


SAMPLE_CAVEATS = ("scaled from one group's 4 executions to 56 per token: the sample's attention rows are "
                  "64 keys long, so the quadratic attention cost of an 8,192-token prefill is under-counted, "
                  "and the LM head is left out")


def cpu_baseline_entry(T=64):
    """The oracle on the bounded sample, once on all host cores and once on one core."""
    import threadpoolctl
    dt, tokens, execs = oracle_sample(T)
    with threadpoolctl.threadpool_limits(limits=1):
        dt1, _, _ = oracle_sample(T)
    # per-token time of the full stack = (time per execution per token) x 56 executions
    per_token, per_token1 = dt / tokens / execs * 56, dt1 / tokens / execs * 56
    return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "single_core": {"value": 1.0 / per_token1, "unit": "tokens/s", "cores": 1, "sample_s": round(dt1, 3)},
            "sample": f"oracle forward of one full-width group (3 GDN + 1 GQA + mHC, d 4096) on {tokens} tokens "
                      f"({dt:.2f} s on {cpu_cores()} BLAS threads, {dt1:.2f} s on one); " + SAMPLE_CAVEATS}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest of every rank's x (device time is taken as the max over ranks)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, ms):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def run_reference(args, world, rank):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(args.ref_tokens)
    times, sample_s = [], []
    for _ in range(args.steps):
        dt, tokens, execs = oracle_sample(args.ref_tokens)
        sample_s.append(dt)
        times.append(dt / tokens / execs * 56)
    value = 1.0 / (sum(times) / len(times))
    # a step is one bounded sample: ms_per_step is the time actually measured for it; the
    # tokens/s value is extrapolated from it to the 56-execution stack
    line = {"impl": "reference", "metric": "prefill tokens/s (56-execution looped hybrid stack)", "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000.0 * sum(sample_s) / len(sample_s), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": BATCH, "seq_len": SEQ, "parallelism": "cpu oracle"},
            "step": f"one oracle forward of one full-width group (3 GDN + 1 GQA + mHC, d 4096) on "
                    f"{args.ref_tokens} tokens; ms_per_step is that sample's measured time",
            "extrapolated": {"value_from": "seconds per token per execution x 56 executions", "caveats": SAMPLE_CAVEATS,
                             "ms_per_8192_token_prefill": round(1000.0 * sum(times) / len(times) * SEQ, 1)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                             "nproc": os.cpu_count(), "cpu_model": cpu_model(),
                             "sample": f"each step: oracle forward of one full-width group on {args.ref_tokens} "
                                       "tokens, scaled to 56 executions per token; " + SAMPLE_CAVEATS},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when the
    kernel's sources have changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    src = b"".join(open(os.path.join(ROOT, "looped_hybrid_attention_b200", "csrc", n), "rb").read()
                   for n in ("gemm_tc.cu", "gemm_tc2.cu", "tc_common.cuh"))
    if hashlib.sha256(src).hexdigest() != rec.get("kernel_sources_sha256"):
        return None
    return rec.get("traffic_bytes_per_launch_step_average")


def summarize(kernels, steps, peaks, sustained=True, tensor_bound=("gemm", "attention", "gdn_chunk")):
    """Roofline entry for the dominant kernel class and a per-class table.

    Classes in `tensor_bound` are rated in TFLOP/s against the bf16 peak, the rest in
    GB/s against the HBM copy bandwidth (decode passes an empty tuple: every kernel of
    a batch-64 decode step streams weights or caches)."""
    name, k = max(kernels.items(), key=lambda kv: kv[1]["ms"])
    if k["flops"] > 0 and name in tensor_bound:
        achieved = k["flops"] / (k["ms"] / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        roof = {"bound": "tensor", "unit": "TFLOP/s",
                "peak_kind": ("bf16 sustained" if sustained else "bf16 burst") + " (" + peaks["source"] + ")"}
    else:
        achieved = k["bytes"] / (k["ms"] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "unit": "GB/s", "peak_kind": "HBM copy (" + peaks["source"] + ")"}
    roof.update({"kernel": name, "achieved": round(achieved, 2), "peak": peak, "frac": round(achieved / peak, 4),
                 "launches": k["launches"], "ms_per_launch": round(k["ms"] / k["launches"], 4),
                 "algorithmic_per_launch": (k["flops"] if roof["bound"] == "tensor" else k["bytes"]) / k["launches"],
                 "traffic": recorded_traffic(name) if name == "gemm" and tensor_bound else None})
    per_kernel = {}
    total_ms = sum(v["ms"] for v in kernels.values())
    for kname, v in sorted(kernels.items(), key=lambda kv: -kv[1]["ms"]):
        e = {"launches": v["launches"] // steps, "ms_per_step": round(v["ms"] / steps, 3),
             "share": round(v["ms"] / total_ms, 4)}
        if v["flops"]:
            e["tflops"] = round(v["flops"] / (v["ms"] / 1e3) / 1e12, 1)
        if v["bytes"]:
            e["gbs"] = round(v["bytes"] / (v["ms"] / 1e3) / 1e9, 1)
        per_kernel[kname] = e
    return roof, per_kernel


def step_tensor_roofline(kernels, ms_step, peaks):
    """The whole prefill step against the tensor roofline: every kernel's algorithmic FLOPs of
    one step over the step's time, as a fraction of the sustained bf16 peak."""
    flops = sum(v["flops"] for v in kernels.values())
    achieved = flops / (ms_step / 1e3) / 1e12
    return {"bound": "tensor", "algorithmic_flops_per_step": flops, "achieved_tflops": round(achieved, 1),
            "peak": peaks["bf16_tflops_sustained"], "frac": round(achieved / peaks["bf16_tflops_sustained"], 4)}


def profiled(m, fn, n):
    """Per-kernel table from the runtime's CUDA events around every launch, over n more
    calls of fn.  Kept out of the timed regions: an event between two launches costs time
    and stops a programmatic dependent launch from overlapping its predecessor."""
    import torch
    torch.cuda.synchronize()
    m.profile(True)
    for _ in range(n):
        fn()
    torch.cuda.synchronize()
    kernels = m.profile_read()
    m.profile(False)
    return kernels


def run_decode(args, m, s, dev, world, seed):
    """Decode at batch 64 over 32,768-token contexts (the decode configuration), greedy argmax.

    By default the per-execution caches are filled with random values of the real shapes
    (K, V ~ N(0,1) in every slab, states ~ N(0, 0.1^2)) and the cache length set to the
    context length: the decode step's work does not depend on the cache's values.
    --decode-real-prefill fills them with a real prefill of random ids instead.
    """
    import torch

    import looped_hybrid_attention_b200 as L
    import synth
    B, ctx = args.decode_batch, args.decode_context
    steps, warm = args.decode_steps, 3
    c = m.cache(B, ctx + warm + 2 * steps + min(steps, 32))   # warm-up, timed, profiled, end to end
    stream = torch.cuda.current_stream()
    g = torch.Generator(device=dev).manual_seed(seed)
    t0 = time.time()
    if args.decode_real_prefill:
        ids = synth.uniform_ids((B, ctx), s.vocab, seed, "decode_ctx", device=dev)
        lg = torch.empty((B, s.vocab), device=dev)
        seg = 512
        for p0 in range(0, ctx, seg):
            m.prefill(c, ids[:, p0:p0 + seg].contiguous(), lg, stream)
        torch.cuda.synchronize()
    else:
        n_fa, n_gdn = 14, 42
        for slot in range(n_fa):
            kp, vp = c.kv_ptrs(slot)
            for p in (kp, vp):
                slab = L.device_view(p, (B, s.fa_kv_heads, c.max_tokens, s.fa_head_dim), torch.bfloat16)
                slab[:, :, :ctx].normal_(generator=g)
        for slot in range(n_gdn):
            st = L.device_view(c.state_ptr(slot), (B, s.gdn_heads, s.gdn_dv, s.gdn_dk), torch.float32)
            st.normal_(generator=g).mul_(0.1)
        c.length = ctx
        torch.cuda.synchronize()
    setup_s = time.time() - t0
    tok = synth.uniform_ids((B,), s.vocab, seed, "decode_tok", device=dev)
    nxt = torch.empty_like(tok)
    for _ in range(warm):
        m.decode_step(c, tok, None, nxt, stream)
        tok, nxt = nxt, tok
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        ev0.record(stream)
        for _ in range(steps):
            m.decode_step(c, tok, None, nxt, stream)
            tok, nxt = nxt, tok
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    prof_steps = min(steps, 32)
    kernels = profiled(m, lambda: m.decode_step(c, tok, None, nxt, stream), prof_steps)
    # end to end: each step's token ids come from pinned host memory and the next tokens go back
    tok_host = tok.cpu().pin_memory()
    nxt_host = torch.empty_like(tok_host).pin_memory()
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        tok.copy_(tok_host, non_blocking=True)
        m.decode_step(c, tok, None, nxt, stream)
        nxt_host.copy_(nxt, non_blocking=True)
        stream.synchronize()
        tok_host, nxt_host = nxt_host, tok_host
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world)
    peaks = load_peaks()
    roof, per_kernel = summarize(kernels, prof_steps, peaks, tensor_bound=())
    # whole-step HBM roofline: weights per execution + KV read + GDN state read/write
    kv_bytes, st_bytes = c.nbytes()
    ctx_mid = ctx + warm + steps // 2
    step_bytes = (sum(v["bytes"] for v in kernels.values()) / prof_steps)
    out = {"metric": "decode tokens/s (56-execution looped hybrid stack)", "workload":
           f"9B-shape stack, decode B={B} over {ctx}-token contexts, {steps} greedy steps",
           "value": round(B * steps * world / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms / steps, 3),
           "context": "real prefill of random ids" if args.decode_real_prefill else
           "random K/V and GDN states of the real shapes (decode work does not depend on cache values)",
           "setup_s": round(setup_s, 1),
           "e2e": {"value": round(B * steps * world / (ms_e2e / 1e3), 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": B * 4, "d2h_bytes_per_step": B * 4},
           "gpu_launches": sum(v["launches"] for v in kernels.values()) * steps // prof_steps,
           "kernel_table_steps": prof_steps,
           "step_roofline": {"bound": "hbm", "algorithmic_bytes_per_step": step_bytes,
                             "achieved_gbs": round(step_bytes / (ms / steps / 1e3) / 1e9, 1),
                             "peak": peaks["hbm_gbs"],
                             "frac": round(step_bytes / (ms / steps / 1e3) / 1e9 / peaks["hbm_gbs"], 4)},
           "roofline": roof, "kernels": per_kernel, "clocks": clk.summary()}
    del c
    return out


def run_long(args, m, s, dev, world, seed):
    """Long-context prefill: batch 1, 131,072 uniform random ids in one call (14 KV slabs of
    131,072 positions, 42 GDN states).  One step is ~6 s, so this leg runs one warm-up and
    --long-steps timed steps."""
    import torch

    import looped_hybrid_attention_b200 as L
    import synth
    T = args.long_seq
    c = m.cache(1, T)
    ids = synth.uniform_ids((1, T), s.vocab, seed, "long", device=dev)
    logits = torch.empty((1, s.vocab), device=dev)
    stream = torch.cuda.current_stream()
    torch.cuda.reset_peak_memory_stats(dev)
    c.reset()
    m.prefill(c, ids, logits, stream)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert torch.isfinite(logits).all(), "non-finite logits"
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        ev0.record(stream)
        for _ in range(args.long_steps):
            c.reset()
            m.prefill(c, ids, logits, stream)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)

    def one():
        c.reset()
        m.prefill(c, ids, logits, stream)
    kernels = profiled(m, one, 1)
    free, total = torch.cuda.mem_get_info(dev)
    kv_bytes, st_bytes = c.nbytes()
    roof, per_kernel = summarize(kernels, 1, load_peaks())
    out = {"metric": "prefill tokens/s (56-execution looped hybrid stack)",
           "workload": f"9B-shape stack, long-context prefill B=1 T={T}, bf16, random-init weights",
           "value": round(T * args.long_steps * world / (ms / 1e3), 1), "unit": "tokens/s",
           "ms_per_step": round(ms / args.long_steps, 1), "steps": args.long_steps, "warmup": 1,
           "kv_slab_bytes": kv_bytes, "gdn_state_bytes": st_bytes,
           "device_bytes_in_use": total - free,
           "gpu_launches": sum(v["launches"] for v in kernels.values()) * args.long_steps,
           "kernel_table_steps": 1,
           "roofline": roof, "step_roofline": step_tensor_roofline(kernels, ms / args.long_steps, load_peaks()),
           "kernels": per_kernel, "clocks": clk.summary()}
    del c
    return out


def run_ours(args, world, rank, local):
    import torch

    import looped_hybrid_attention_b200 as L
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    s = synth.FULL
    w = synth.make_weights(s, seed=args.seed + rank, device=dev)
    m = L.Model(s, w)
    c = m.cache(BATCH, SEQ)
    ids = synth.uniform_ids((BATCH, SEQ), s.vocab, args.seed + rank, device=dev)
    logits = torch.empty((BATCH, s.vocab), device=dev)
    stream = torch.cuda.current_stream()

    def step():
        c.reset()
        m.prefill(c, ids, logits, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert torch.isfinite(logits).all(), "non-finite logits"

    # ---------------- device-resident timed region
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, world)
    kernels = profiled(m, step, 1)      # per-kernel table from one more step
    tokens = BATCH * SEQ * args.steps * world
    value = weak_scaling_value(BATCH * SEQ * args.steps, world, ms)

    # ---------------- end to end through the public API with host buffers
    ids_host = ids.cpu().pin_memory()
    logits_host = torch.empty((BATCH, s.vocab), pin_memory=True)
    ids_dev = torch.empty_like(ids)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        ids_dev.copy_(ids_host, non_blocking=True)
        c.reset()
        m.prefill(c, ids_dev, logits, stream)
        logits_host.copy_(logits, non_blocking=True)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world)

    peaks = load_peaks()
    roof, per_kernel = summarize(kernels, 1, peaks)
    launches = sum(v["launches"] for v in kernels.values()) * args.steps

    line = {"metric": "prefill tokens/s (56-execution looped hybrid stack)", "value": round(value, 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random-init weights, uniform token ids)",
            "config": {"workload": WORKLOAD, "global_batch": BATCH * world, "seq_len": SEQ,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (16.3 GB of weights streamed per step)"},
            "e2e": {"value": round(tokens / (ms_e2e / 1e3), 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": ids.numel() * 4, "d2h_bytes_per_step": logits.numel() * 4},
            "gpu_launches": launches, "kernel_table_steps": 1, "roofline": roof,
            "step_roofline": step_tensor_roofline(kernels, ms / args.steps, peaks),
            "kernels": per_kernel, "clocks": clk.summary()}
    if not args.no_decode or not args.no_long:
        del c
        torch.cuda.empty_cache()
    if not args.no_decode:
        line["decode"] = run_decode(args, m, s, dev, world, args.seed + rank)
    if not args.no_long:
        line["long_prefill"] = run_long(args, m, s, dev, world, args.seed + rank)
    if rank != 0:
        return
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_entry(args.ref_tokens)
    # compact per-leg summary as the line's last key, so that a reader of the line's tail
    # sees every leg's number after the long per-kernel tables
    legs = {"prefill": {"value": line["value"], "unit": "tokens/s", "ms_per_step": line["ms_per_step"],
                        "roofline_kernel": roof["kernel"], "roofline_frac": roof["frac"],
                        "step_frac_of_tensor_roofline": line["step_roofline"]["frac"],
                        "sm_mhz": line["clocks"]["sm_mhz"]}}
    for key in ("decode", "long_prefill"):
        if key in line:
            leg = line[key]
            legs[key] = {"value": leg["value"], "unit": leg["unit"], "ms_per_step": leg["ms_per_step"],
                         "roofline_kernel": leg["roofline"]["kernel"], "roofline_frac": leg["roofline"]["frac"],
                         "sm_mhz": leg["clocks"]["sm_mhz"]}
            if "step_roofline" in leg:
                sr = leg["step_roofline"]
                legs[key][f"step_frac_of_{sr['bound']}_roofline"] = sr["frac"]
    line["legs"] = legs
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-tokens", type=int, default=64, help="tokens per oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--decode-batch", type=int, default=64)
    ap.add_argument("--decode-context", type=int, default=32768)
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--no-long", action="store_true", help="skip the long-context prefill measurement")
    ap.add_argument("--long-seq", type=int, default=131072)
    ap.add_argument("--long-steps", type=int, default=1)
    ap.add_argument("--decode-real-prefill", action="store_true",
                    help="fill the decode contexts with a real prefill instead of random cache values")
    args = ap.parse_args()
    world, rank, local = 1, int(os.environ.get("RANK", "0")), 0
    if args.impl == "ours":
        world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
