"""Continuous-batching trace replay: the control plane driving the GPU kernels.

Sources: "Nano-vLLM engine architecture" (intelliparadigm.com) section 2.2 and
"Deep into the Nano-vLLM inference engine" (lnwmold.com), sections on the
producer-consumer step loop, waiting/running queues, preemption, prefix
caching and the preparation of each step's inputs.  The model itself (weights,
projections, sampling) is out of scope: every layer's Q/K/V rows are slices of
a seeded ring of pre-generated buffers and the sampled token of each step is a
seeded random id.

One step: ``Scheduler.schedule()`` -> ``prepare_prefill`` / ``prepare_decode``
-> one pinned host->device copy of the packed int32 metadata -> for every
layer: the store of the step's new K/V rows into that layer's pool and the
attention, one launch (``prefill_store`` / ``decode_store``), into a scratch output -> postprocess
(append tokens, finish, free).  All launches go to the current stream; the
host runs ahead of the GPU except where it reuses a pinned staging buffer.

With ``graphs=True`` a decode step's 28 layers run as one captured CUDA graph
("CUDA Graphs", lnwmold.com item: decode is captured for common batch sizes
to cut launch overhead).  A graph is keyed by the batch size rounded up to a
multiple of 16, the longest context rounded up to 512 and the ring offset of
the step; the metadata goes to fixed device buffers the graph reads (padding
rows: slot -1, context length 0, which the kernels skip / answer with zeros).
On the first step of a key the layers run eagerly and the graph is captured
for the next ones.  Prefill steps always run eagerly.

Timing: ``run`` reports the wall time of the loop, the host time spent inside
the steps (scheduling, preparation, packing, launching, postprocessing) and
how much of it was spent blocked on the GPU (a pinned staging buffer whose
copy has not run yet), and the GPU time of the steps: for each step the device time from its metadata
copy to its last kernel, summed (idle device time between steps, while the
host prepares the next one, is not counted).

``scheduler="priority"`` replays the trace through ``PriorityScheduler``
(each request gets a seeded priority in ``[0, num_priorities)``; waiting
sequences are admitted highest priority first).

``slot_writer`` records, for every pool slot, which (step, packed row) last
wrote it -- the same for every layer, since all layers share the block tables.
With the CPU copy of the ring this lets a checker rebuild exactly what any
sequence's K/V history holds on the GPU.
"""

from __future__ import annotations

import time
from collections import OrderedDict
from dataclasses import dataclass

import numpy as np
import torch

from . import synth
from .host import (PriorityScheduler, Scheduler, SchedulerConfig, Sequence, prepare_decode,
                   prepare_prefill)


@dataclass
class ReplayConfig:
    num_requests: int = 512
    prompt_lo: int = 100
    prompt_hi: int = 1024
    output_lo: int = 100
    output_hi: int = 1024
    max_num_seqs: int = 256
    max_num_batched_tokens: int = 16384
    block_size: int = 256
    num_blocks: int = 768
    num_layers: int = 28
    num_q_heads: int = 16
    num_kv_heads: int = 8
    head_dim: int = 128
    max_model_len: int = 4096
    ring: int = 8
    seed: int = synth.SEED_BASE + 5
    scheduler: str = "fcfs"           # "fcfs" (Scheduler) or "priority" (PriorityScheduler)
    num_priorities: int = 4           # priorities drawn in [0, num_priorities) for "priority"


class Replay:
    def __init__(self, cfg: ReplayConfig, device="cuda", record=False, graphs=False,
                 max_graphs=64):
        from . import ops
        self.ops = ops
        self.cfg = cfg
        self.device = device
        self.record = record
        c = cfg
        rng = np.random.default_rng(c.seed)
        prompts = rng.integers(c.prompt_lo, c.prompt_hi + 1, size=c.num_requests)
        outputs = rng.integers(c.output_lo, c.output_hi + 1, size=c.num_requests)
        if c.scheduler not in ("fcfs", "priority"):
            raise ValueError(f"unknown scheduler {c.scheduler!r}")
        sched_cls = PriorityScheduler if c.scheduler == "priority" else Scheduler
        self.sched = sched_cls(SchedulerConfig(
            max_num_seqs=c.max_num_seqs, max_num_batched_tokens=c.max_num_batched_tokens,
            block_size=c.block_size, num_blocks=c.num_blocks, max_model_len=c.max_model_len,
            seed=c.seed))
        prio = (np.random.default_rng(c.seed + 7).integers(0, c.num_priorities, size=c.num_requests)
                if c.scheduler == "priority" else np.zeros(c.num_requests, dtype=np.int64))
        self.requests = []
        for i in range(c.num_requests):
            s = Sequence(synth.token_ids(int(prompts[i]), c.seed * 1000 + i), max_tokens=int(outputs[i]),
                         priority=int(prio[i]))
            self.requests.append(s)
            self.sched.add(s)
        self.token_rng = np.random.default_rng(c.seed + 1)
        # the largest step: a full prefill budget, or one recomputed sequence
        self.max_tokens = max(c.max_num_batched_tokens, c.prompt_hi + c.output_hi, c.max_num_seqs)
        hq, hkv, d, T = c.num_q_heads, c.num_kv_heads, c.head_dim, self.max_tokens
        # seeded ring of per-layer inputs, drawn on the CPU
        self.q_ring_cpu = [synth.bf16_normal((T, hq, d), c.seed * 10 + 3 * r) for r in range(c.ring)]
        self.k_ring_cpu = [synth.bf16_normal((T, hkv, d), c.seed * 10 + 3 * r + 1) for r in range(c.ring)]
        self.v_ring_cpu = [synth.bf16_normal((T, hkv, d), c.seed * 10 + 3 * r + 2) for r in range(c.ring)]
        self.q_ring = torch.stack(self.q_ring_cpu).to(device)
        self.k_ring = torch.stack(self.k_ring_cpu).to(device)
        self.v_ring = torch.stack(self.v_ring_cpu).to(device)
        shape = (c.num_blocks, c.block_size, hkv, d)
        self.k_pools = [torch.full(shape, synth.NAN_BF16_BITS, dtype=torch.int16, device=device)
                        .view(torch.bfloat16) for _ in range(c.num_layers)]
        self.v_pools = [p.clone() for p in self.k_pools]
        self.out = torch.empty((T, hq, d), dtype=torch.bfloat16, device=device)
        # metadata staging: two pinned buffers (double buffering) and one device buffer
        width = -(-c.max_model_len // c.block_size) + 1
        self.meta_len = T + 3 * (c.max_num_seqs + 1) + c.max_num_seqs * width
        self.pinned = [torch.empty(self.meta_len, dtype=torch.int32).pin_memory() for _ in range(2)]
        self.pinned_ev = [None, None]
        self.d_meta = torch.empty(self.meta_len, dtype=torch.int32, device=device)
        self.ws = torch.empty(1 << 20, dtype=torch.uint8, device=device)
        self.slot_writer = np.full((c.num_blocks * c.block_size, 2), -1, dtype=np.int64)
        self.graphs = graphs
        if graphs:
            # fixed metadata buffers of graph-replayed decode steps: slots [S],
            # context_lens [S], block_tables [S, width] (S = max_num_seqs)
            S = c.max_num_seqs
            self.g_width = width
            self.g_meta = torch.empty(2 * S + S * width, dtype=torch.int32, device=device)
            self.g_pinned = [torch.empty(self.g_meta.numel(), dtype=torch.int32).pin_memory()
                             for _ in range(2)]
            self.g_pinned_ev = [None, None]
            self.graph_cache = OrderedDict()
            self.max_graphs = max_graphs
            need = ops.decode_workspace_size(S, hq, hkv, d, self._ctx_bucket(c.max_model_len))
            self.g_ws = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
        self.step_idx = 0
        self.stats = dict(steps=0, prefill_steps=0, decode_steps=0, prefill_tokens=0,
                          decode_tokens=0, decode_kv_bytes=0, launches=0, graph_steps=0,
                          graph_captures=0, prefill_pairs=0, decode_context_tokens=0)
        self.host_s = 0.0          # host time inside step()
        self.host_wait_s = 0.0     # of which blocked on the GPU (a staging buffer still in use)
        self.step_events = []      # (start, end) CUDA events of each step's device work
        self.samples = {}          # (step, layer) -> captured output and the step's metadata
        self.sample_at = set()     # (step, layer) pairs to capture (needs record=True)
        self.snap = {}             # step -> slot_writer after that step's stores

    # ----------------------------------------------------------------- helpers
    def ring_index(self, step: int, layer: int) -> int:
        return (step * self.cfg.num_layers + layer) % self.cfg.ring

    def _upload(self, parts):
        """Pack int32 arrays into a pinned buffer and copy them to the device in one go."""
        b = self.step_idx & 1
        if self.pinned_ev[b] is not None:
            t0 = time.perf_counter()
            self.pinned_ev[b].synchronize()        # the copy that last used this buffer is done
            self.host_wait_s += time.perf_counter() - t0
        buf = self.pinned[b]
        views, off = [], 0
        host = buf.numpy()
        for a in parts:
            n = a.size
            host[off:off + n] = a.reshape(-1)
            views.append((off, a.shape))
            off += n
        self.d_meta[:off].copy_(buf[:off], non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        self.pinned_ev[b] = ev
        return [self.d_meta[o:o + int(np.prod(sh))].view(*sh) for o, sh in views]

    # ----------------------------------------------------------- graph steps
    def _batch_bucket(self, n: int) -> int:
        return min(-(-n // 16) * 16, self.cfg.max_num_seqs)

    def _ctx_bucket(self, L: int) -> int:
        return min(-(-L // 512) * 512, self.cfg.max_model_len)

    def _graph_views(self, nb: int):
        S, w = self.cfg.max_num_seqs, self.g_width
        m = self.g_meta
        return m[:nb], m[S:S + nb], m[2 * S:2 * S + nb * w].view(nb, w)

    def _decode_layers(self, nb: int, lb: int, step: int, slots, cl, bt, out):
        c, ops = self.cfg, self.ops
        for layer in range(c.num_layers):
            r = self.ring_index(step, layer)
            kc, vc = self.k_pools[layer], self.v_pools[layer]
            ops.decode_store(self.q_ring[r, :nb], self.k_ring[r, :nb], self.v_ring[r, :nb], kc, vc,
                             slots, bt, cl, lb, out=out, workspace=self.g_ws)

    def _decode_graph_step(self, md, n: int):
        """One decode step through a captured graph (see the module docstring)."""
        c = self.cfg
        S, w = c.max_num_seqs, self.g_width
        nb, lb = self._batch_bucket(n), self._ctx_bucket(md.max_context_len)
        b = self.step_idx & 1
        if self.g_pinned_ev[b] is not None:
            t0 = time.perf_counter()
            self.g_pinned_ev[b].synchronize()
            self.host_wait_s += time.perf_counter() - t0
        host = self.g_pinned[b].numpy()
        host[:nb] = -1
        host[:n] = md.slot_mapping
        host[S:S + nb] = 0
        host[S:S + n] = md.context_lens
        btv = host[2 * S:2 * S + nb * w].reshape(nb, w)
        btv[:] = -1
        btv[:n, :md.block_tables.shape[1]] = md.block_tables
        used = 2 * S + nb * w
        self.g_meta[:used].copy_(self.g_pinned[b][:used], non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        self.g_pinned_ev[b] = ev
        slots, cl, bt = self._graph_views(nb)
        out = self.out[:nb]
        key = (nb, lb, (self.step_idx * c.num_layers) % c.ring)
        g = self.graph_cache.get(key)
        if g is None:
            # this step eagerly (also the lazy set-up of every launch), then the capture
            self._decode_layers(nb, lb, self.step_idx, slots, cl, bt, out)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._decode_layers(nb, lb, self.step_idx, slots, cl, bt, out)
            self.graph_cache[key] = g
            self.stats["graph_captures"] += 1
            if len(self.graph_cache) > self.max_graphs:
                self.graph_cache.popitem(last=False)
        else:
            self.graph_cache.move_to_end(key)
            g.replay()
            self.stats["graph_steps"] += 1
        return out[:n]

    # -------------------------------------------------------------------- step
    def step(self) -> bool:
        if self.sched.is_finished():
            return False
        t_host = time.perf_counter()
        c, ops = self.cfg, self.ops
        seqs, is_prefill = self.sched.schedule()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev0.record()
        bs = c.block_size
        if is_prefill:
            md = prepare_prefill(seqs, bs)
            n = md.total_q
            slots, cu_q, cu_k, bt = self._upload([md.slot_mapping, md.cu_seqlens_q,
                                                  md.cu_seqlens_k, md.block_tables])
            self.stats["prefill_steps"] += 1
            self.stats["prefill_tokens"] += n
            ql = np.diff(md.cu_seqlens_q).astype(np.int64)
            kl = np.diff(md.cu_seqlens_k).astype(np.int64)
            self.stats["prefill_pairs"] += int((ql * (kl - ql) + ql * (ql + 1) // 2).sum())
        else:
            md = prepare_decode(seqs, bs)
            n = len(seqs)
            slots, cl, bt = self._upload([md.slot_mapping, md.context_lens, md.block_tables])
            need = ops.decode_workspace_size(n, c.num_q_heads, c.num_kv_heads, c.head_dim,
                                             md.max_context_len)
            if need > self.ws.numel():
                self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            self.stats["decode_steps"] += 1
            self.stats["decode_tokens"] += n
            self.stats["decode_context_tokens"] += int(md.context_lens.sum())
            self.stats["decode_kv_bytes"] += int(md.context_lens.sum()) * c.num_kv_heads * \
                c.head_dim * 4 * c.num_layers
        out = self.out[:n]
        captured = False
        if self.graphs and not is_prefill:
            out = self._decode_graph_step(md, n)
            last = c.num_layers - 1
            if self.record == "all" or (self.step_idx, last) in self.sample_at:
                self.samples[(self.step_idx, last)] = dict(
                    is_prefill=False, md=md, out=out.cpu().clone(),
                    block_tables=[list(s.block_table) for s in seqs], lens=[len(s) for s in seqs])
                captured = True
        for layer in range(0 if (self.graphs and not is_prefill) else c.num_layers):
            r = self.ring_index(self.step_idx, layer)
            kc, vc = self.k_pools[layer], self.v_pools[layer]
            if is_prefill:
                # the step's store fused into the prefill launch (pa_prefill_store)
                ops.prefill_store(self.q_ring[r, :n], self.k_ring[r, :n], self.v_ring[r, :n], kc,
                                  vc, slots, cu_q, cu_k, md.max_seqlen_q, md.max_seqlen_k, bt,
                                  out=out)
            else:
                # the step's store fused into the decode launch (pa_decode_store)
                ops.decode_store(self.q_ring[r, :n], self.k_ring[r, :n], self.v_ring[r, :n], kc, vc,
                                 slots, bt, cl, md.max_context_len, out=out, workspace=self.ws)
            if self.record == "all" or (self.step_idx, layer) in self.sample_at:
                self.samples[(self.step_idx, layer)] = dict(
                    is_prefill=is_prefill, md=md, out=out.cpu().clone(),
                    block_tables=[list(s.block_table) for s in seqs], lens=[len(s) for s in seqs])
                captured = True
        if self.graphs and not is_prefill:
            nb, lb = self._batch_bucket(n), self._ctx_bucket(md.max_context_len)
            split = ops.decode_workspace_size(nb, c.num_q_heads, c.num_kv_heads, c.head_dim, lb) > 0
        else:
            split = not is_prefill and ops.decode_workspace_size(
                n, c.num_q_heads, c.num_kv_heads, c.head_dim, md.max_context_len) > 0
        # prefill: the fused store + attention; decode: the fused store + decode, and the merge
        self.stats["launches"] += c.num_layers * (1 if is_prefill else (2 if split else 1))
        ev1 = torch.cuda.Event(enable_timing=True)
        ev1.record()
        self.step_events.append((ev0, ev1))
        if self.record:
            sm = md.slot_mapping.astype(np.int64)
            self.slot_writer[sm, 0] = self.step_idx
            self.slot_writer[sm, 1] = np.arange(len(sm))
            if captured:
                self.snap[self.step_idx] = self.slot_writer.copy()
        toks = self.token_rng.integers(0, synth.VOCAB, size=len(seqs)).tolist()
        self.sched.postprocess(seqs, toks)
        self.stats["steps"] += 1
        self.step_idx += 1
        self.host_s += time.perf_counter() - t_host
        return True

    def run(self, max_steps=0):
        t0 = time.perf_counter()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        while self.step():
            if max_steps and self.step_idx >= max_steps:
                break
        e1.record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        st = dict(self.stats)
        st["wall_s"] = wall
        st["gpu_s"] = e0.elapsed_time(e1) / 1e3          # span from the first to the last launch
        st["gpu_busy_s"] = sum(a.elapsed_time(b) for a, b in self.step_events) / 1e3
        st["host_s"] = self.host_s
        st["host_wait_s"] = self.host_wait_s
        st["preemptions"] = self.sched.num_preemptions
        st["prefix_hit_tokens"] = self.sched.block_manager.prefix_hit_tokens
        st["finished"] = sum(1 for s in self.requests if s.is_finished)
        return st


def run_replay_bench(torch_mod=None, max_steps=0, cfg: ReplayConfig | None = None, graphs=True):
    """The trace replay as a bench workload: tokens/s over the whole loop."""
    cfg = cfg or ReplayConfig()
    rp = Replay(cfg, graphs=graphs)
    torch.cuda.synchronize()
    st = rp.run(max_steps=max_steps)
    tokens = st["prefill_tokens"] + st["decode_tokens"]
    return {
        "tokens_per_s": round(tokens / st["wall_s"], 1),
        "tokens": tokens, "wall_s": round(st["wall_s"], 3), "gpu_s": round(st["gpu_s"], 3),
        "gpu_busy_s": round(st["gpu_busy_s"], 3), "host_s": round(st["host_s"], 3),
        "host_wait_s": round(st["host_wait_s"], 3),
        "host_work_over_gpu": round((st["host_s"] - st["host_wait_s"]) / st["gpu_busy_s"], 3)
        if st["gpu_busy_s"] else None,
        "prefill_pairs": st["prefill_pairs"], "decode_context_tokens": st["decode_context_tokens"],
        "steps": st["steps"], "prefill_steps": st["prefill_steps"], "decode_steps": st["decode_steps"],
        "prefill_tokens": st["prefill_tokens"], "decode_tokens": st["decode_tokens"],
        "preemptions": st["preemptions"], "prefix_hit_tokens": st["prefix_hit_tokens"],
        "finished": st["finished"], "requests": cfg.num_requests, "launches": st["launches"],
        "graphs": graphs, "graph_steps": st["graph_steps"], "graph_captures": st["graph_captures"],
        "scheduler": cfg.scheduler,
        "decode_kv_GBs": round(st["decode_kv_bytes"] / st["wall_s"] / 1e9, 1),
        "config": {"layers": cfg.num_layers, "heads": f"{cfg.num_q_heads}/{cfg.num_kv_heads}",
                   "head_dim": cfg.head_dim, "block_size": cfg.block_size,
                   "num_blocks": cfg.num_blocks, "max_num_seqs": cfg.max_num_seqs,
                   "max_num_batched_tokens": cfg.max_num_batched_tokens,
                   "prompt": f"U[{cfg.prompt_lo},{cfg.prompt_hi}]",
                   "output": f"U[{cfg.output_lo},{cfg.output_hi}]"},
    }
