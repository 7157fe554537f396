#!/usr/bin/env python
"""Benchmark of the paged-KV attention hot path on B200.

Default (N=1): one layer of 7B-GQA-shaped decode -- batch 256, context
lengths uniform in [512, 4096], 28 query / 4 KV heads, head_dim 128, block
size 256, shuffled pool sized 1.25x the need (the largest decode
configuration).  One step = store each sequence's new K/V row into the pool +
paged decode attention over the batch (one fused launch, then the split-K
merge).

Metric: decode-step KV GB/s (algorithmic bytes of the step / step time), with
tokens/s (sequences decoded per second for this layer) beside it.  Inputs are
resident in HBM when timing starts; L2 is flushed (a 512 MiB write, then a
512 MiB read so the write's dirty lines are gone too) before every timed step
and each step is bracketed by CUDA events on the launching stream.  With
--gpus N (torchrun, one rank per GPU) every rank runs its own replica of the
workload (no collective on the data path: "scaling": "weak") and the time is
the max over ranks.

Also measured in the same run, at the same --steps / --warmup, and reported
under "workloads": Qwen3-0.6B-shaped decode (batch 32, 16/8 heads), the
7B-GQA decode at block 16, the prefix-cached prefill (TFLOP/s), a large
store_kvcache (GB/s) and the continuous-batching trace replay (tokens/s, with
GPU-busy and host control-plane time).  "cpu_baselines" times the CPU oracle
on every configuration (bounded samples; the trace replay's full-trace figure
is a labelled projection).  ``--impl reference`` times the CPU oracle on a
bounded sample of the headline workload instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": BF16_FALLBACK_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks / throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------- timing
class Timer:
    """Per-step CUDA-event timing on the current stream, L2 flushed before each step.

    The flush writes a 512 MiB buffer (4x the 126 MB L2) and then reads another
    512 MiB buffer: the write evicts every line, the read pushes the write's own
    dirty lines back to HBM before the step starts, so the timed kernels neither
    find their inputs in L2 nor pay for write-backs that are not theirs."""

    def __init__(self, torch, flush_bytes=512 << 20):
        self.torch = torch
        self.flush_buf = torch.empty(flush_bytes, dtype=torch.uint8, device="cuda")
        self.read_buf = torch.zeros(flush_bytes // 4, dtype=torch.float32, device="cuda")

    def flush(self):
        self.flush_buf.fill_(1)
        self.read_buf.sum()

    def time_steps(self, fn, steps, marks=1):
        """Runs `fn(ev)` `steps` times; fn records its own events in `ev` (list of marks+1 events).
        Returns per-step lists of segment durations in ms.  Python's garbage collector
        is paused meanwhile so a collection cannot stall the launches of a step."""
        import gc
        torch = self.torch
        segs = []
        gc_was = gc.isenabled()
        gc.disable()
        try:
            for _ in range(steps):
                self.flush()
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(marks + 1)]
                fn(ev)
                segs.append(ev)
            torch.cuda.synchronize()
        finally:
            if gc_was:
                gc.enable()
        return [[e[i].elapsed_time(e[i + 1]) for i in range(marks)] for e in segs]


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return torch, dist, world, rank, local


def max_over_ranks(torch, dist, world, x: float) -> float:
    """The slowest rank's value (device-timed regions are reported as the max)."""
    if world == 1:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, max_total_ms: float) -> float:
    """Replicas: every rank processes the same per-step work, so the whole job did
    world x units x steps in the slowest rank's time; units per second."""
    return world * units_per_rank_step * steps / (max_total_ms * 1e-3)


def barrier(torch, dist, world):
    """Device work done, then every rank here (the CPU path for gloo ranks)."""
    cuda = torch.cuda.is_available()
    if cuda:
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


# ------------------------------------------------------------ workloads (ours)
def bench_decode(torch, w, steps, warmup, timer, dist=None, world=1, partition=0):
    """Times `steps` decode steps through pa_decode_store (the step's store_kvcache
    fused into the decode launch; one event pair around the step, the merge kernel
    follows by programmatic dependent launch), then `steps` of the same step as
    two launches (store_kvcache, decode) and `steps` decode launches alone.  One
    untimed pass of the fused step runs first: the first timed pass after the
    clock sampler starts showed host stalls between launches inside the timed
    region (3-10 us a step)."""
    from paged_kv_attention_35_b200 import ops
    stream = torch.cuda.current_stream()
    need = ops.decode_workspace_size(w.B, w.hq, w.hkv, w.d, w.max_context_len, partition)
    if need > w.d_ws.numel():
        w.d_ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    def fused():
        ops.decode_store(w.d_q, w.d_new_k, w.d_new_v, w.kc, w.vc, w.d_slots, w.d_bt, w.d_cl,
                         w.max_context_len, out=w.d_out, workspace=w.d_ws, partition_size=partition)

    for _ in range(warmup):
        fused()

    def one(ev):
        ev[0].record(stream)
        fused()
        ev[1].record(stream)

    def two(ev):
        ev[0].record(stream)
        ops.store_kvcache(w.d_new_k, w.d_new_v, w.kc, w.vc, w.d_slots)
        ops.decode(w.d_q, w.kc, w.vc, w.d_bt, w.d_cl, w.max_context_len, out=w.d_out,
                   workspace=w.d_ws, partition_size=partition)
        ev[1].record(stream)

    timer.time_steps(one, steps)                   # untimed settling pass
    barrier(torch, dist, world)

    def dec(ev):
        ev[0].record(stream)
        ops.decode(w.d_q, w.kc, w.vc, w.d_bt, w.d_cl, w.max_context_len, out=w.d_out,
                   workspace=w.d_ws, partition_size=partition)
        ev[1].record(stream)

    segs = np.asarray(timer.time_steps(one, steps))[:, 0]
    barrier(torch, dist, world)
    tsegs = np.asarray(timer.time_steps(two, steps))[:, 0]
    dsegs = np.asarray(timer.time_steps(dec, steps))[:, 0]
    return {"decode_ms": float(dsegs.mean()), "step_ms": float(segs.mean()),
            "two_launch_ms": float(tsegs.mean()), "step_ms_total": float(segs.sum())}


def bench_decode_e2e(torch, w, steps, warmup, timer):
    """Same step through host buffers: H2D of the step's inputs, kernels, D2H of the output.

    The step's inputs (q, new K/V rows, slot_mapping, block tables, context lengths)
    sit in one pinned staging buffer at 256-byte aligned offsets and go up in one
    copy per step into one device buffer whose views the calls take, as an
    engine would stage a step (one DMA instead of six fixed-cost transfers)."""
    from paged_kv_attention_35_b200 import ops
    stream = torch.cuda.current_stream()
    src = {
        "q": w.q, "k": w.new_k, "v": w.new_v,
        "slots": torch.from_numpy(w.decode_slots),
        "bt": torch.from_numpy(w.block_tables),
        "cl": torch.tensor(w.lens, dtype=torch.int32),
    }
    offs, total = {}, 0
    for k, t in src.items():
        offs[k] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_buf = torch.empty(total, dtype=torch.uint8, device="cuda")

    def view(buf, k):
        t = src[k]
        n = t.numel() * t.element_size()
        return buf[offs[k]:offs[k] + n].view(t.dtype).view(t.shape)

    for k, t in src.items():
        view(h_buf, k).copy_(t.contiguous())
    d = {k: view(d_buf, k) for k in src}
    out_h = torch.empty(w.d_out.shape, dtype=torch.bfloat16).pin_memory()
    h2d = total
    d2h = out_h.numel() * out_h.element_size()

    def one(ev):
        ev[0].record(stream)
        d_buf.copy_(h_buf, non_blocking=True)
        ops.decode_store(d["q"], d["k"], d["v"], w.kc, w.vc, d["slots"], d["bt"], d["cl"],
                         w.max_context_len, out=w.d_out, workspace=w.d_ws)
        out_h.copy_(w.d_out, non_blocking=True)
        ev[1].record(stream)

    for _ in range(warmup):
        timer.time_steps(one, 1)
    segs = np.asarray(timer.time_steps(one, steps))
    serial_ms = float(segs.mean())

    # Pipelined, as a serving loop runs it: two staging sets; step i+1's
    # upload (one copy stream) and step i-1's download (another) run while
    # step i's kernels run, each copy ordered after what it depends on by
    # events.  Every step still moves its whole input up and its output down
    # inside the timed region.  No L2 flush between steps: the 1.2 GB of KV
    # read per step is ten times the L2.
    us, ds = torch.cuda.Stream(), torch.cuda.Stream()
    hb = [h_buf, torch.empty_like(h_buf).pin_memory()]
    hb[1].copy_(h_buf)
    db = [d_buf, torch.empty_like(d_buf)]
    dv = [{k: view(db[i], k) for k in src} for i in range(2)]
    od = [w.d_out, torch.empty_like(w.d_out)]
    oh = [out_h, torch.empty_like(out_h).pin_memory()]

    def run(n):
        up = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        down = [torch.cuda.Event() for _ in range(2)]
        started = [False, False]
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(us):
                if started[b]:
                    us.wait_event(done[b])      # step i-2's kernels have read db[b]
                db[b].copy_(hb[b], non_blocking=True)
                up[b].record(us)
            stream.wait_event(up[b])
            if started[b]:
                stream.wait_event(down[b])      # od[b] has gone down before it is rewritten
            d = dv[b]
            ops.decode_store(d["q"], d["k"], d["v"], w.kc, w.vc, d["slots"], d["bt"], d["cl"],
                             w.max_context_len, out=od[b], workspace=w.d_ws)
            done[b].record(stream)
            with torch.cuda.stream(ds):
                ds.wait_event(done[b])
                oh[b].copy_(od[b], non_blocking=True)
                down[b].record(ds)
            started[b] = True
        stream.wait_stream(us)
        stream.wait_stream(ds)

    run(max(warmup, 2))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    us.wait_event(e0)
    ds.wait_event(e0)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, serial_ms, h2d, d2h


def bench_prefill(torch, steps, warmup, timer):
    from paged_kv_attention_35_b200.workloads import PrefixPrefillWorkload
    from paged_kv_attention_35_b200 import synth
    w = PrefixPrefillWorkload(seed=synth.SEED_BASE + 4).upload("cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        w.step()

    def one(ev):
        ev[0].record(stream)
        w.store()
        ev[1].record(stream)
        w.attend()
        ev[2].record(stream)

    segs = np.asarray(timer.time_steps(one, steps, marks=2))
    store_ms, attn_ms = float(segs[:, 0].mean()), float(segs[:, 1].mean())

    # the same step as one launch: the store folded into the prefill (pa_prefill_store)
    for _ in range(warmup):
        w.fused_step()

    def fused(ev):
        ev[0].record(stream)
        w.fused_step()
        ev[1].record(stream)

    w.fused_ms = float(np.asarray(timer.time_steps(fused, steps, marks=1))[:, 0].mean())
    return w, store_ms, attn_ms


def bench_store_large(torch, steps, warmup, timer):
    """N = 65536 new tokens, Hkv 8, D 128, block 256, slots a seeded permutation of the pool."""
    from paged_kv_attention_35_b200 import ops, synth
    n, hkv, d, bs = 65536, 8, 128, 256
    nb = n // bs
    key = synth.bf16_normal((n, hkv, d), 7).cuda()
    val = synth.bf16_normal((n, hkv, d), 8).cuda()
    kc = torch.empty((nb, bs, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    slots = torch.from_numpy(synth.permutation(nb * bs, 9).astype(np.int32)).cuda()
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        ops.store_kvcache(key, val, kc, vc, slots)

    def one(ev):
        ev[0].record(stream)
        ops.store_kvcache(key, val, kc, vc, slots)
        ev[1].record(stream)

    ms = float(np.asarray(timer.time_steps(one, steps)).mean())
    nbytes = 2 * 2 * n * hkv * d * 2
    return nbytes, ms


def decode_config(spec, w, partition, world):
    """The `config` object of a decode bench line (both arms print the same one)."""
    lo, hi = (spec.ctx_lo, spec.ctx_hi) if not spec.fixed_lens else (min(w.lens), max(w.lens))
    return {"workload": spec.name, "num_seqs": w.B, "context_lens": f"U[{lo},{hi}]",
            "sum_context": int(sum(w.lens)), "num_q_heads": w.hq, "num_kv_heads": w.hkv,
            "head_dim": w.d, "block_size": w.bs, "num_blocks": w.nb,
            "partition": partition or "auto",
            "l2": "flushed before every step (512 MiB write, then 512 MiB read)",
            "parallelism": f"replicas x{world}"}


METRIC = "paged decode attention KV GB/s (decode step: store_kvcache + decode)"


def ours(args):
    torch, dist, world, rank, local = dist_setup()
    from paged_kv_attention_35_b200 import ops  # noqa: F401  (fails loudly without the library)
    from paged_kv_attention_35_b200 import synth
    from paged_kv_attention_35_b200.workloads import DecodeWorkload
    pk = peaks()
    timer = Timer(torch)
    spec = synth.WORKLOADS[args.workload]
    w = DecodeWorkload.from_spec(spec).upload("cuda")
    # the fused store + decode kernel, and the merge kernel when contexts are split
    launches_per_step = 1 + (1 if ops.decode_workspace_size(
        w.B, w.hq, w.hkv, w.d, w.max_context_len, args.partition) > 0 else 0)

    with ClockSampler(local) as clk:
        time.sleep(1.5)                            # the sampler's nvidia-smi is up before timing
        r = bench_decode(torch, w, args.steps, args.warmup, timer, dist, world, args.partition)
    # max over ranks of the timed region (sum of the K steps' device time)
    total_ms = max_over_ranks(torch, dist, world, r["step_ms_total"])
    step_ms = total_ms / args.steps
    step_bytes = w.step_bytes()
    value = whole_job_rate(world, step_bytes, args.steps, total_ms) / 1e9
    tokens_s = whole_job_rate(world, w.B, args.steps, total_ms)
    kernel_gbs = step_bytes / (step_ms * 1e-3) / 1e9      # the step is the fused kernel (+ merge)

    e2e_ms, e2e_serial_ms, h2d, d2h = bench_decode_e2e(torch, w, args.steps, args.warmup, timer)
    e2e_ms = max_over_ranks(torch, dist, world, e2e_ms)
    e2e_serial_ms = max_over_ranks(torch, dist, world, e2e_serial_ms)

    extra = {}
    if not args.quick and rank == 0:
        extra = secondary(torch, args, timer, pk)

    cpu, cpus = None, None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_decode(w, budget_s=args.cpu_budget)
        cpus = cpu_baselines(args, w, extra)

    if rank == 0:
        traffic = load_traffic("decode_kernel", args.workload)
        line = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(step_ms, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 K/V/q, seeded context lengths and shuffled pool)",
            "config": decode_config(spec, w, args.partition, world),
            "tokens_per_s": round(tokens_s, 1),
            "breakdown_ms": {"fused_store_decode": round(r["step_ms"], 4),
                             "store_then_decode": round(r["two_launch_ms"], 4),
                             "decode_alone": round(r["decode_ms"], 4)},
            "roofline": {"bound": "hbm",
                         "kernel": "decode_kernel with the fused store (pa_decode_store) + split-K merge",
                         "achieved": round(kernel_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(kernel_gbs / pk["hbm_gbs"], 4),
                         "peak_source": pk["source"], "traffic": traffic,
                         "bytes_per_launch": step_bytes},
            "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                    "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "mode": "pipelined: step i+1's upload and step i-1's download overlap "
                            "step i's kernels (an upload and a download stream, two staging "
                            "sets); serial_*: each step's copies and kernels back to back",
                    "serial_ms_per_step": round(e2e_serial_ms, 4),
                    "serial_value": round(world * step_bytes / (e2e_serial_ms * 1e-3) / 1e9, 1)},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "cpu_baselines": cpus,
            "workloads": extra,
            "pages_context": {"qwen7b_tokens_per_s": {"bs1": 32, "bs8": 215, "bs16": 398},
                              "note": "end-to-end model throughput quoted by the pages, hardware not stated"},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def library_comparison(torch, steps, warmup, timer):
    """FlashAttention-2 (`flash_attn`, installed in the image: the attention library the
    pages' engine calls) on the same inputs, as a black-box comparison, never as the oracle:
    paged decode (`flash_attn_with_kvcache` with the block tables) on the 7B-GQA and Qwen3
    decode workloads, and paged varlen prefill (`flash_attn_varlen_func` with the block
    tables) on the prefix-cached prefill, each beside this library's kernel on the same
    buffers, timed the same way (events, L2 flushed before every launch)."""
    from paged_kv_attention_35_b200 import ops, synth
    from paged_kv_attention_35_b200.workloads import DecodeWorkload, PrefixPrefillWorkload
    try:
        from flash_attn import flash_attn_with_kvcache, flash_attn_varlen_func
    except Exception as e:                         # noqa: BLE001 (any import failure)
        return {"unavailable": f"flash_attn import failed: {e!r}"[:200]}
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(warmup):
            fn()

        def one(ev):
            ev[0].record(stream)
            fn()
            ev[1].record(stream)
        return float(np.asarray(timer.time_steps(one, steps))[:, 0].mean())

    res = {"library": "flash_attn " + getattr(__import__("flash_attn"), "__version__", "?"),
           "note": "black-box comparison on the same buffers; not the oracle, not the product path"}
    for name in ("gqa7b_decode", "qwen3_0p6b_decode"):
        w = DecodeWorkload.from_spec(synth.WORKLOADS[name]).upload("cuda")
        ops.store_kvcache(w.d_new_k, w.d_new_v, w.kc, w.vc, w.d_slots)
        q4 = w.d_q.unsqueeze(1)
        lib = flash_attn_with_kvcache(q4, w.kc, w.vc, cache_seqlens=w.d_cl, block_table=w.d_bt,
                                      causal=True)
        ours = ops.decode(w.d_q, w.kc, w.vc, w.d_bt, w.d_cl, w.max_context_len, out=w.d_out,
                          workspace=w.d_ws)
        torch.cuda.synchronize()
        diff = float((lib[:, 0].float() - ours.float()).abs().max())
        t_lib = timed(lambda: flash_attn_with_kvcache(q4, w.kc, w.vc, cache_seqlens=w.d_cl,
                                                      block_table=w.d_bt, causal=True))
        t_ours = timed(lambda: ops.decode(w.d_q, w.kc, w.vc, w.d_bt, w.d_cl, w.max_context_len,
                                          out=w.d_out, workspace=w.d_ws))
        res[name] = {"flash_attn_ms": round(t_lib, 4), "ours_ms": round(t_ours, 4),
                     "flash_attn_GBs": round(w.kv_bytes() / (t_lib * 1e-3) / 1e9, 1),
                     "ours_GBs": round(w.kv_bytes() / (t_ours * 1e-3) / 1e9, 1),
                     "speedup": round(t_lib / t_ours, 2), "max_abs_diff_outputs": diff}
        del w
        torch.cuda.empty_cache()
    w = PrefixPrefillWorkload(seed=synth.SEED_BASE + 4).upload("cuda")
    w.store()
    ours = w.attend().clone()
    mq, mk = int(w.md.max_seqlen_q), int(w.md.max_seqlen_k)
    lib = flash_attn_varlen_func(w.d_q, w.kc, w.vc, w.d_cu_q, w.d_cu_k, mq, mk, causal=True,
                                 block_table=w.d_bt)
    torch.cuda.synchronize()
    diff = float((lib.float() - ours.float()).abs().max())
    t_lib = timed(lambda: flash_attn_varlen_func(w.d_q, w.kc, w.vc, w.d_cu_q, w.d_cu_k, mq, mk,
                                                 causal=True, block_table=w.d_bt))
    t_ours = timed(lambda: w.attend())
    res["prefix_prefill"] = {"flash_attn_ms": round(t_lib, 4), "ours_ms": round(t_ours, 4),
                             "flash_attn_TFLOPs": round(w.flops() / (t_lib * 1e-3) / 1e12, 1),
                             "ours_TFLOPs": round(w.flops() / (t_ours * 1e-3) / 1e12, 1),
                             "speedup": round(t_lib / t_ours, 2), "max_abs_diff_outputs": diff}
    del w
    torch.cuda.empty_cache()
    return res


def secondary(torch, args, timer, pk):
    """The other workloads, each at its own roofline (rank 0), at the same --steps / --warmup."""
    from paged_kv_attention_35_b200 import synth
    from paged_kv_attention_35_b200.workloads import DecodeWorkload
    out = {}
    steps, warm = args.steps, args.warmup
    others = [("qwen3_0p6b_decode", None), ("gqa7b_decode", 256), ("gqa7b_decode", 16)]
    for name, bs in others:
        spec = synth.WORKLOADS[name]
        if name == args.workload and bs in (None, spec.block_size):
            continue                               # the headline itself
        w = DecodeWorkload.from_spec(spec, block_size=bs).upload("cuda")
        r = bench_decode(torch, w, steps, warm, timer)
        step_gbs = w.step_bytes() / (r["step_ms"] * 1e-3) / 1e9
        gbs = w.kv_bytes() / (r["decode_ms"] * 1e-3) / 1e9
        out[f"{name}_bs{w.bs}"] = {
            "step_ms": round(r["step_ms"], 4), "decode_ms": round(r["decode_ms"], 4),
            "store_then_decode_ms": round(r["two_launch_ms"], 4), "kv_bytes": w.kv_bytes(),
            "step_GBs": round(step_gbs, 1), "frac_hbm_step": round(step_gbs / pk["hbm_gbs"], 4),
            "decode_GBs": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
            "tokens_per_s": round(w.B / (r["step_ms"] * 1e-3), 1)}
        del w
        torch.cuda.empty_cache()
    w, store_ms, attn_ms = bench_prefill(torch, steps, warm, timer)
    tf = w.flops() / (attn_ms * 1e-3) / 1e12
    out["prefix_prefill"] = {
        "attn_ms": round(attn_ms, 4), "store_ms": round(store_ms, 4), "flops": w.flops(),
        "total_q": int(w.md.total_q), "TFLOPs": round(tf, 1),
        "frac_bf16_peak": round(tf / pk["bf16_tflops"], 4),
        "frac_bf16_sustained": round(tf / pk["bf16_tflops_sustained"], 4),
        "peak_source": pk["source"], "traffic": load_traffic("prefill_tc_kernel", "prefix_prefill"),
        "store_GBs": round(w.store_bytes() / (store_ms * 1e-3) / 1e9, 1),
        "fused_store_prefill_ms": round(w.fused_ms, 4),
        "fused_TFLOPs": round(w.flops() / (w.fused_ms * 1e-3) / 1e12, 1)}
    del w
    torch.cuda.empty_cache()
    nbytes, ms = bench_store_large(torch, steps, warm, timer)
    try:
        out["library_comparison"] = library_comparison(torch, steps, warm, timer)
    except Exception as e:                         # noqa: BLE001 (a library failure is reported)
        out["library_comparison"] = {"unavailable": repr(e)[:200]}
        torch.cuda.empty_cache()
    out["store_kvcache_65536"] = {"ms": round(ms, 4), "bytes": nbytes,
                                  "GBs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                                  "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
    torch.cuda.empty_cache()
    if not args.no_replay:
        from paged_kv_attention_35_b200.replay import run_replay_bench
        out["trace_replay"] = run_replay_bench(torch, max_steps=args.replay_steps, graphs=False)
        g = run_replay_bench(torch, max_steps=args.replay_steps, graphs=True)
        out["trace_replay_graphs"] = {k: g[k] for k in (
            "tokens_per_s", "wall_s", "gpu_busy_s", "host_s", "host_wait_s", "steps", "graph_steps",
            "graph_captures", "decode_kv_GBs")}
        torch.cuda.empty_cache()
    return out


def only(args):
    """One secondary workload by itself (profiling aid); prints its JSON object."""
    import torch
    from paged_kv_attention_35_b200 import synth
    from paged_kv_attention_35_b200.workloads import DecodeWorkload
    pk = peaks()
    timer = Timer(torch)
    if args.only == "prefill":
        w, store_ms, attn_ms = bench_prefill(torch, args.steps, args.warmup, timer)
        tf = w.flops() / (attn_ms * 1e-3) / 1e12
        res = {"workload": "prefix_prefill", "attn_ms": round(attn_ms, 4), "TFLOPs": round(tf, 1),
               "frac_bf16_peak": round(tf / pk["bf16_tflops"], 4), "store_ms": round(store_ms, 4),
               "fused_store_prefill_ms": round(w.fused_ms, 4)}
    elif args.only == "decode":
        w = DecodeWorkload.from_spec(synth.WORKLOADS[args.workload],
                                     block_size=args.block_size or None).upload("cuda")
        r = bench_decode(torch, w, args.steps, args.warmup, timer, partition=args.partition)
        gbs = w.kv_bytes() / (r["decode_ms"] * 1e-3) / 1e9
        res = {"workload": args.workload, "block_size": w.bs, "step_ms": round(r["step_ms"], 4),
               "decode_ms": round(r["decode_ms"], 4), "decode_GBs": round(gbs, 1),
               "frac_hbm": round(gbs / pk["hbm_gbs"], 4)}
    elif args.only == "store":
        nbytes, ms = bench_store_large(torch, args.steps, args.warmup, timer)
        res = {"workload": "store_kvcache_65536", "ms": round(ms, 4),
               "GBs": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    else:
        from paged_kv_attention_35_b200.replay import run_replay_bench
        res = run_replay_bench(torch, max_steps=args.replay_steps, graphs=args.graphs)
    print(json.dumps(res), flush=True)


def load_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch from an ncu capture of this kernel and
    workload, or None when there is none or the kernel's source changed since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(f"{kernel}:{workload}")
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src) or \
            hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != e["source_sha256_16"]:
        return None
    return e["bytes"]


# ------------------------------------------------------------ CPU oracle arm
def decode_sample_inputs(w, rows):
    """Oracle inputs (float64) for sequences `rows` of a decode workload: q, and a
    compact pool holding only their blocks (renumbered), built from the logical draws."""
    import oracle
    import torch

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    lens = [w.lens[i] for i in rows]
    nblk = [-(-L // w.bs) for L in lens]
    bt = np.full((len(rows), max(nblk)), -1, np.int32)
    kp = np.zeros((sum(nblk), w.bs, w.hkv, w.d), np.uint16)
    vp = np.zeros_like(kp)
    k = 0
    for j, i in enumerate(rows):
        bt[j, :nblk[j]] = np.arange(k, k + nblk[j])
        flat_k = kp[k:k + nblk[j]].reshape(-1, w.hkv, w.d)
        flat_v = vp[k:k + nblk[j]].reshape(-1, w.hkv, w.d)
        flat_k[:lens[j]] = bits(w.k[i])
        flat_v[:lens[j]] = bits(w.v[i])
        k += nblk[j]
    q = oracle.bf16_bits_to_f64(bits(w.q))[rows]
    return q, oracle.bf16_bits_to_f64(kp), oracle.bf16_bits_to_f64(vp), bt, np.asarray(lens)


def cpu_baseline_decode(w, budget_s=15.0):
    """Time the oracle (as it stands) on a bounded sample of the decode workload."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    done_bytes = 0
    n = 0
    t_or = 0.0
    # cycle through the batch's sequences (all heads each) until the budget is spent
    while t_or < budget_s:
        i = n % w.B
        q, kp, vp, bt, lens = decode_sample_inputs(w, [i])
        t0 = time.perf_counter()
        oracle.ref_decode(q, kp, vp, bt, lens)
        t_or += time.perf_counter() - t0
        done_bytes += w.lens[i] * w.hkv * w.d * 2 * 2
        n += 1
    gbs = done_bytes / t_or / 1e9 if t_or > 0 else None
    return {"value": gbs, "unit": "GB/s", "cores": _blas_threads(cores), "kind": "oracle",
            "sample": f"{n} sequence decodes (all {w.hq} heads each; {n / w.B:.1f} passes over the "
                      f"{w.B}-sequence batch), oracle time {t_or:.2f} s",
            "seconds": round(t_or, 2)}


def _blas_threads(default):
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(int(i.get("num_threads", 1)) for i in info)
    except Exception:
        pass
    return default


def cpu_baselines(args, w3, extra):
    """The oracle (as it stands, never tuned) timed on every configuration on this
    host's cores.  Decode configs: bounded samples with all BLAS threads and with one;
    the prefix-cached prefill: the whole workload once; the trace replay: sampled
    (step, layer) pairs of a recorded replay, projected to the whole trace by the
    number of (query, key) pairs it visits (labelled as a projection)."""
    from threadpoolctl import threadpool_limits
    from paged_kv_attention_35_b200 import synth
    from paged_kv_attention_35_b200.workloads import DecodeWorkload
    budget = max(1.0, args.cpu_budget / 3)
    res = {}
    tiny = DecodeWorkload.from_spec(synth.WORKLOADS["tiny_decode"])
    w2 = DecodeWorkload.from_spec(synth.WORKLOADS["qwen3_0p6b_decode"])
    for name, w, b in (("tiny_decode", tiny, 1.0), ("qwen3_0p6b_decode", w2, budget),
                       ("gqa7b_decode", w3, budget)):
        e = {}
        if name != "gqa7b_decode" or w3.bs != 256:
            e["all_threads"] = cpu_baseline_decode(w, budget_s=b)
        with threadpool_limits(limits=1):
            e["one_thread"] = cpu_baseline_decode(w, budget_s=b)
        e["one_thread"]["cores"] = 1
        res[name] = e
    res["prefix_prefill"] = cpu_baseline_prefill()
    rp = extra.get("trace_replay") if extra else None
    if rp and not args.no_replay:
        res["trace_replay"] = cpu_baseline_replay(rp, budget_s=budget)
    return res


def cpu_baseline_prefill():
    """The oracle on the whole prefix-cached prefill (16 sequences, every head)."""
    import oracle
    from paged_kv_attention_35_b200 import synth
    from paged_kv_attention_35_b200.workloads import PrefixPrefillWorkload
    w = PrefixPrefillWorkload(seed=synth.SEED_BASE + 4)
    q, kp, vp, cu_q, cu_k, bt = prefill_oracle_inputs(w)
    t0 = time.perf_counter()
    oracle.ref_prefill(q, kp, vp, cu_q, cu_k, bt)
    dt = time.perf_counter() - t0
    return {"value": round(w.flops() / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": _blas_threads(len(os.sched_getaffinity(0))), "kind": "oracle",
            "sample": f"the whole workload: {len(w.seqs)} sequences, {int(w.md.total_q)} queries x "
                      f"{w.hq} heads, oracle time {dt:.2f} s", "seconds": round(dt, 2)}


def prefill_oracle_inputs(w, seqs=None):
    """Oracle inputs (float64) of a prefix-cached prefill workload: packed q and a compact
    pool holding the listed sequences' logical K/V (renumbered blocks)."""
    import oracle
    import torch

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    seqs = list(range(len(w.seqs))) if seqs is None else list(seqs)
    k_lens = [w.k_lens[i] for i in seqs]
    nblk = [-(-L // w.bs) for L in k_lens]
    bt = np.full((len(seqs), max(nblk)), -1, np.int32)
    kp = np.zeros((sum(nblk), w.bs, w.hkv, w.d), np.uint16)
    vp = np.zeros_like(kp)
    k = 0
    for j, i in enumerate(seqs):
        bt[j, :nblk[j]] = np.arange(k, k + nblk[j])
        kp[k:k + nblk[j]].reshape(-1, w.hkv, w.d)[:k_lens[j]] = bits(w.k[i])
        vp[k:k + nblk[j]].reshape(-1, w.hkv, w.d)[:k_lens[j]] = bits(w.v[i])
        k += nblk[j]
    cu = w.md.cu_seqlens_q
    qall = oracle.bf16_bits_to_f64(bits(w.q))
    q = np.concatenate([qall[cu[i]:cu[i + 1]] for i in seqs])
    cu_q = np.concatenate([[0], np.cumsum([w.q_lens[i] for i in seqs])])
    cu_k = np.concatenate([[0], np.cumsum(k_lens)])
    return q, oracle.bf16_bits_to_f64(kp), oracle.bf16_bits_to_f64(vp), cu_q, cu_k, bt


def cpu_baseline_replay(stats, budget_s=10.0):
    """Oracle time for sampled sequences of sampled (step, layer) pairs of the trace
    replay, and a projection to the whole trace by visited (query, key) pairs."""
    import oracle
    import torch
    from paged_kv_attention_35_b200.replay import Replay, ReplayConfig

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    cfg = ReplayConfig()
    rp = Replay(cfg, record=True)
    last = cfg.num_layers - 1
    rp.sample_at = {(0, 0), (1, last), (3, 0), (40, last), (120, 0)}
    rp.run(max_steps=121)
    torch.cuda.synchronize()
    f64 = oracle.bf16_bits_to_f64
    spent = {"prefill": [0.0, 0], "decode": [0.0, 0]}      # seconds, visited pairs x heads
    for (step, layer), smp in sorted(rp.samples.items()):
        snap = rp.snap[step]
        md = smp["md"]
        q_all = f64(bits(rp.q_ring_cpu[rp.ring_index(step, layer)]))
        kind = "prefill" if smp["is_prefill"] else "decode"
        for j in range(min(len(smp["lens"]), 4)):
            if spent[kind][0] > budget_s / 2:
                break
            bt, L = smp["block_tables"][j], smp["lens"][j]
            slots = oracle.ref_slot_mapping(bt, range(L), cfg.block_size)
            wr = snap[slots]
            K = f64(np.stack([bits(rp.k_ring_cpu[rp.ring_index(int(a), layer)][int(b)]) for a, b in wr]))
            V = f64(np.stack([bits(rp.v_ring_cpu[rp.ring_index(int(a), layer)][int(b)]) for a, b in wr]))
            kp, vp = K[None], V[None]
            t0 = time.perf_counter()
            if kind == "prefill":
                a, b = int(md.cu_seqlens_q[j]), int(md.cu_seqlens_q[j + 1])
                oracle.ref_prefill(q_all[a:b], kp, vp, [0, b - a], [0, L], np.array([[0]]))
                pairs = (b - a) * (L - (b - a)) + (b - a) * (b - a + 1) // 2
            else:
                oracle.ref_decode(q_all[j:j + 1], kp, vp, np.array([[0]]), [L])
                pairs = L
            spent[kind][0] += time.perf_counter() - t0
            spent[kind][1] += pairs * cfg.num_q_heads
    per = {k: (v[0] / v[1] if v[1] else None) for k, v in spent.items()}
    total_pairs = {"prefill": stats["prefill_pairs"] * cfg.num_layers * cfg.num_q_heads,
                   "decode": stats["decode_context_tokens"] * cfg.num_layers * cfg.num_q_heads}
    proj = sum(per[k] * total_pairs[k] for k in per if per[k] is not None)
    tokens = stats["prefill_tokens"] + stats["decode_tokens"]
    return {"value": round(tokens / proj, 3) if proj else None, "unit": "tokens/s",
            "cores": _blas_threads(len(os.sched_getaffinity(0))), "kind": "oracle",
            "projection": True,
            "sample": (f"sampled sequences of (step, layer) pairs {sorted(rp.samples)} of the "
                       f"replayed trace: prefill {spent['prefill'][0]:.2f} s for "
                       f"{spent['prefill'][1]} (query, key, head) triples, decode "
                       f"{spent['decode'][0]:.2f} s for {spent['decode'][1]}; PROJECTED to the "
                       f"whole trace's {total_pairs['prefill']} + {total_pairs['decode']} triples "
                       f"({proj:.0f} s)" if proj else "no sample")}


def reference(args):
    """The oracle as the reference arm: same metric/config, bounded sample per step."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from paged_kv_attention_35_b200 import synth
    from paged_kv_attention_35_b200.workloads import DecodeWorkload
    spec = synth.WORKLOADS[args.workload]
    w = DecodeWorkload.from_spec(spec)
    budget = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline_decode(w, budget_s=budget)
    vals = []
    last = None
    for _ in range(args.steps):
        last = cpu_baseline_decode(w, budget_s=budget)
        vals.append(last["value"])
    v = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC,
        "value": round(v, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (same seeded workload)",
        "config": decode_config(spec, w, args.partition, world),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "kind": "oracle",
                         "cores": last["cores"], "sample": last["sample"]},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gqa7b_decode")
    ap.add_argument("--partition", type=int, default=0)
    ap.add_argument("--quick", action="store_true", help="primary workload only")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-replay", action="store_true")
    ap.add_argument("--replay-steps", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--graphs", action="store_true", help="--only replay: graph-replayed decode steps")
    ap.add_argument("--block-size", type=int, default=0, help="--only decode: pool block size")
    ap.add_argument("--only", choices=["prefill", "decode", "store", "replay"], default=None,
                    help="time one secondary workload alone (for profiling) and print its JSON")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        reference(args)
    elif args.only:
        only(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
