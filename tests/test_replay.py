"""Trace replay on the GPU checked against the oracle (``-m gpu``).

A small trace (tiny pool, so preemption fires) is checked at every step and
every layer: the oracle recomputes each sequence's slots from its block table,
rebuilds the sequence's K/V history from the host record of which ring row
last wrote each slot (CPU copies of the ring; nothing read back from the
pool), and runs ``ref_prefill`` / ``ref_decode``.  The full 512-request trace
is checked on sampled steps and layers.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_attention_35_b200.replay import Replay, ReplayConfig
from tests.gpu_cases import TOL_MAX, TOL_MEAN
from tests.problems import to_bits

pytestmark = pytest.mark.gpu
f64 = oracle.bf16_bits_to_f64


_RING_BITS = {}


def _ring_bits(rp, which):
    """The CPU ring of K (or V) rows as one [ring, rows, Hkv, D] uint16 array (cached)."""
    key = (id(rp), which)
    if key not in _RING_BITS:
        ring = rp.k_ring_cpu if which == "k" else rp.v_ring_cpu
        _RING_BITS.clear()
        _RING_BITS[key] = np.stack([to_bits(t) for t in ring])
    return _RING_BITS[key]


def _history(rp, snap, block_table, length, layer, which):
    """[length, Hkv, D] float64 K (or V) rows a sequence's positions hold after a step:
    each position's row is the ring row of the step that last wrote its slot."""
    c = rp.cfg
    slots = oracle.ref_slot_mapping(block_table, range(length), c.block_size)
    writer = snap[slots]
    assert (writer[:, 0] >= 0).all(), "a position was never stored"
    steps, inv = np.unique(writer[:, 0], return_inverse=True)
    ring_idx = np.array([rp.ring_index(int(st), layer) for st in steps])[inv]
    return f64(_ring_bits(rp, which)[ring_idx, writer[:, 1]])


def check_sample(rp, step, layer, max_seqs=None, max_prefill_seqs=None):
    """Every (or an evenly spread max_seqs / max_prefill_seqs of the) sequence(s) of a
    captured (step, layer) against the oracle."""
    c = rp.cfg
    smp = rp.samples[(step, layer)]
    if smp["is_prefill"] and max_prefill_seqs is not None:
        max_seqs = max_prefill_seqs
    snap = rp.snap[step]
    md = smp["md"]
    q_all = f64(to_bits(rp.q_ring_cpu[rp.ring_index(step, layer)]))
    out = smp["out"].double().numpy()
    nseq = len(smp["lens"])
    idx = range(nseq) if max_seqs is None else np.linspace(0, nseq - 1, min(nseq, max_seqs)).astype(int)
    errs = []
    for j in idx:
        bt = smp["block_tables"][j]
        L = smp["lens"][j]
        K = _history(rp, snap, bt, L, layer, "k")
        V = _history(rp, snap, bt, L, layer, "v")
        kp, vp = K[None], V[None]                     # one contiguous block holding the sequence
        if smp["is_prefill"]:
            a, b = int(md.cu_seqlens_q[j]), int(md.cu_seqlens_q[j + 1])
            # the product's slots for the computed positions equal the oracle's
            assert np.array_equal(md.slot_mapping[a:b],
                                  oracle.ref_slot_mapping(bt, range(L - (b - a), L), c.block_size))
            ref = oracle.ref_prefill(q_all[a:b], kp.reshape(1, L, c.num_kv_heads, c.head_dim),
                                     vp.reshape(1, L, c.num_kv_heads, c.head_dim), [0, b - a], [0, L],
                                     np.array([[0]]))
            got = out[a:b]
        else:
            assert md.slot_mapping[j] == oracle.ref_slot_mapping(bt, [L - 1], c.block_size)[0]
            assert md.context_lens[j] == L
            ref = oracle.ref_decode(q_all[j:j + 1], kp.reshape(1, L, c.num_kv_heads, c.head_dim),
                                    vp.reshape(1, L, c.num_kv_heads, c.head_dim), np.array([[0]]),
                                    [L])
            got = out[j:j + 1]
        err = np.abs(got - ref)
        assert np.isfinite(got).all()
        errs.append((float(err.max()), float(err.mean())))
    mx = max(e[0] for e in errs)
    mean = float(np.mean([e[1] for e in errs]))
    assert mx <= TOL_MAX and mean <= TOL_MEAN, (step, layer, mx, mean)


def test_small_trace_every_step(cuda_device):
    cfg = ReplayConfig(num_requests=14, prompt_lo=5, prompt_hi=70, output_lo=3, output_hi=40,
                       max_num_seqs=6, max_num_batched_tokens=160, block_size=16, num_blocks=14,
                       num_layers=2, num_q_heads=8, num_kv_heads=2, head_dim=128, ring=3, seed=4242,
                       max_model_len=128)
    rp = Replay(cfg, record="all")
    st = rp.run()
    assert st["finished"] == cfg.num_requests
    assert st["preemptions"] > 0, "the tiny pool should force preemption"
    assert st["prefill_steps"] > 0 and st["decode_steps"] > 0
    for s in rp.requests:
        assert s.num_completion_tokens == s.max_tokens
    for (step, layer) in sorted(rp.samples):
        check_sample(rp, step, layer)
    rp.sched.block_manager.check_invariants([])
    assert rp.sched.block_manager.num_free_blocks == cfg.num_blocks


def _small_cfg():
    return ReplayConfig(num_requests=14, prompt_lo=5, prompt_hi=70, output_lo=3, output_hi=40,
                        max_num_seqs=6, max_num_batched_tokens=160, block_size=16, num_blocks=14,
                        num_layers=2, num_q_heads=8, num_kv_heads=2, head_dim=128, ring=3, seed=4242,
                        max_model_len=128)


def test_small_trace_graphs_every_step(cuda_device):
    """Decode steps replayed as captured CUDA graphs (padded batch, fixed metadata
    buffers): every prefill layer and every decode step's last layer against the oracle."""
    cfg = _small_cfg()
    rp = Replay(cfg, record="all", graphs=True)
    st = rp.run()
    assert st["finished"] == cfg.num_requests
    assert st["graph_captures"] > 0 and st["graph_steps"] > st["graph_captures"]
    decode_samples = [k for k in rp.samples if not rp.samples[k]["is_prefill"]]
    assert decode_samples and all(l == cfg.num_layers - 1 for _, l in decode_samples)
    for (step, layer) in sorted(rp.samples):
        check_sample(rp, step, layer)
    assert rp.sched.block_manager.num_free_blocks == cfg.num_blocks


def test_graph_replay_pools_equal_eager(cuda_device):
    """The same trace eager and graph-replayed leaves bit-identical K/V pools."""
    cfg = _small_cfg()
    a = Replay(cfg)
    a.run()
    b = Replay(cfg, graphs=True)
    b.run()
    torch.cuda.synchronize()
    for la in range(cfg.num_layers):
        assert torch.equal(a.k_pools[la].view(torch.int16), b.k_pools[la].view(torch.int16))
        assert torch.equal(a.v_pools[la].view(torch.int16), b.v_pools[la].view(torch.int16))


def test_full_trace_sampled(cuda_device):
    """512 requests, prompt/output U[100,1024], 256 seqs, block 256, 768 blocks, 28 layers:
    nine steps across the trace at layers 0 and 27; 32 evenly spread sequences of a sampled
    decode step, 8 of a sampled prefill step (about a minute of oracle time)."""
    cfg = ReplayConfig()
    rp = Replay(cfg, record=True)
    steps = (0, 3, 40, 400, 800, 1100, 1500, 1900, 2200)
    rp.sample_at = {(s, l) for s in steps for l in (0, cfg.num_layers - 1)}
    st = rp.run()
    assert st["finished"] == cfg.num_requests
    assert st["preemptions"] > 0
    checked, kinds = 0, set()
    for key in sorted(rp.samples):
        check_sample(rp, *key, max_seqs=32, max_prefill_seqs=8)
        kinds.add(rp.samples[key]["is_prefill"])
        checked += 1
    assert checked >= 16 and kinds == {True, False}


def test_full_trace_graphs_sampled(cuda_device):
    """The bench's trace with graph-replayed decode steps, last layer sampled."""
    cfg = ReplayConfig()
    rp = Replay(cfg, record=True, graphs=True)
    last = cfg.num_layers - 1
    rp.sample_at = {(s, last) for s in (3, 40, 400, 1100, 1900)}
    st = rp.run()
    assert st["finished"] == cfg.num_requests
    assert st["graph_steps"] > 10 * st["graph_captures"]
    checked = 0
    for key in sorted(rp.samples):
        check_sample(rp, *key, max_seqs=6)
        checked += 1
    assert checked >= 4


def test_small_trace_priority_scheduler(cuda_device):
    """The small trace through PriorityScheduler (seeded priorities 0..3): every step and
    layer against the oracle; admission order follows priority, then arrival."""
    from dataclasses import replace
    cfg = replace(_small_cfg(), scheduler="priority", num_priorities=4)
    rp = Replay(cfg, record="all")
    first_prefill = None
    orig = rp.sched.schedule

    def schedule():
        nonlocal first_prefill
        seqs, is_prefill = orig()
        if is_prefill and first_prefill is None:
            first_prefill = [s.priority for s in seqs]
        return seqs, is_prefill

    rp.sched.schedule = schedule
    st = rp.run()
    assert st["finished"] == cfg.num_requests
    assert len({s.priority for s in rp.requests}) > 1
    # the first batch admits the highest priorities first
    assert first_prefill == sorted(first_prefill, reverse=True)
    assert max(first_prefill) == max(s.priority for s in rp.requests)
    for (step, layer) in sorted(rp.samples):
        check_sample(rp, step, layer)
    assert rp.sched.block_manager.num_free_blocks == cfg.num_blocks
    assert st["gpu_busy_s"] > 0 and st["host_s"] > 0
