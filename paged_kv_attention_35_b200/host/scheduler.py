"""Prefill-first continuous-batching scheduler with preemption.

Sources
-------
* "Nano-vLLM engine architecture" (intelliparadigm.com), section 2.2
  "Continuous Batching": ``schedule()`` returns a prefill batch of new
  sequences whenever the waiting queue yields one, otherwise a decode batch of
  running sequences; the batch is recomposed at every step; requests can be
  preempted when GPU memory runs short.  Section 6.1 shows a priority
  variant that orders waiting sequences by priority, highest first.
* "Deep into the Nano-vLLM inference engine" (lnwmold.com): section "Waiting
  and Running queues" (new sequences enter the waiting queue, move to running
  once the block manager has given them blocks, and batches are taken from
  running with an operation flag); section "Handling resource exhaustion"
  (a running sequence that has no room for its next token's cache is
  preempted back to the *head* of the waiting queue; finished sequences leave
  running and free their blocks); section "Prefill and Decode" (one prefill
  per sequence, then many decode steps).
* "Learning LLM inference with nano-vLLM" (cxy5.com), section 4.1: batches
  are refilled at every token step as requests finish.

Readings: every step is pure prefill or pure decode; the prefill batch is
capped by ``max_num_seqs`` running sequences and ``max_num_batched_tokens``
computed tokens; when the decode batch cannot extend a sequence, the newest
running sequence is preempted (recompute later) until it can, and a sequence
left alone without room preempts itself.
"""

from __future__ import annotations

from collections import deque
from dataclasses import dataclass

from .block_manager import BlockManager, PoolExhausted
from .sequence import Sequence, SequenceStatus


@dataclass
class SchedulerConfig:
    max_num_seqs: int = 32                  # page 2 section 5.2 Config default
    max_num_batched_tokens: int = 16384
    block_size: int = 256                   # page 2 section 3.2 / 5.2 default
    num_blocks: int = 1024
    max_model_len: int = 4096               # page 2 section 5.2 max_seq_len
    eos: int = -1                           # token id that ends a sequence (-1: none)
    seed: int | None = None                 # seeded free-block order


class Scheduler:
    def __init__(self, config: SchedulerConfig, block_manager: BlockManager | None = None):
        self.config = config
        self.block_manager = block_manager or BlockManager(config.num_blocks, config.block_size,
                                                           seed=config.seed)
        self.waiting: deque = deque()
        self.running: deque = deque()
        self.num_preemptions = 0

    # ------------------------------------------------------------------ queue
    def add(self, seq: Sequence) -> None:
        cap = min(self.config.max_model_len,
                  self.block_manager.num_blocks * self.block_manager.block_size)
        if len(seq) + seq.max_tokens > cap + 1:
            raise ValueError(f"sequence of {len(seq)}+{seq.max_tokens} tokens can never fit "
                             f"(limit {cap})")
        seq.status = SequenceStatus.WAITING
        self.waiting.append(seq)

    def is_finished(self) -> bool:
        return not self.waiting and not self.running

    # --------------------------------------------------------------- schedule
    def _prefill_order(self):
        """Waiting sequences in the order they are considered for admission."""
        return list(self.waiting)

    def _admit_prefill(self) -> list:
        bm = self.block_manager
        batch, tokens = [], 0
        for seq in self._prefill_order():
            if len(self.running) + len(batch) >= self.config.max_num_seqs:
                break
            need, cached = bm.blocks_needed(seq)
            cost = len(seq) - cached
            if batch and tokens + cost > self.config.max_num_batched_tokens:
                break
            if need > bm.num_free_blocks:
                break
            bm.allocate(seq)
            tokens += len(seq) - seq.num_cached_tokens
            batch.append(seq)
        for seq in batch:
            self.waiting.remove(seq)
            seq.status = SequenceStatus.RUNNING
            self.running.append(seq)
        return batch

    def _plan_decode(self) -> list:
        bm = self.block_manager
        batch = []
        pending = deque(self.running)
        self.running.clear()
        while pending and len(batch) < self.config.max_num_seqs:
            seq = pending.popleft()
            while not bm.can_append(seq):
                victim = pending.pop() if pending else seq
                self._preempt(victim)
                if victim is seq:
                    break
            else:
                bm.append_slot(seq)
                batch.append(seq)
        # sequences not considered this step keep their order after the batch
        self.running.extend(batch)
        self.running.extend(pending)
        if not batch and not self.waiting and self.running:
            raise PoolExhausted("no running sequence can make progress")
        return batch

    def schedule(self) -> tuple:
        """Return ``(sequences, is_prefill)`` for the next step."""
        if self.waiting:
            batch = self._admit_prefill()
            if batch:
                return batch, True
            if not self.running:
                head = self.waiting[0]
                raise PoolExhausted(f"cannot admit {head!r}: pool too small")
        return self._plan_decode(), False

    def _preempt(self, seq: Sequence) -> None:
        seq.status = SequenceStatus.WAITING
        seq.num_preemptions += 1
        self.num_preemptions += 1
        self.block_manager.deallocate(seq)
        self.waiting.appendleft(seq)

    # ------------------------------------------------------------ postprocess
    def postprocess(self, seqs, token_ids) -> list:
        """Append each sequence's new token; finish and free the completed ones."""
        finished = []
        for seq, tok in zip(seqs, token_ids):
            seq.append_token(tok)
            done = seq.num_completion_tokens >= seq.max_tokens or (
                self.config.eos >= 0 and tok == self.config.eos)
            if done:
                seq.status = SequenceStatus.FINISHED
                self.block_manager.deallocate(seq)
                self.running.remove(seq)
                finished.append(seq)
        return finished


class PriorityScheduler(Scheduler):
    """Admits waiting sequences highest ``priority`` first (page 2, section 6.1)."""

    def _prefill_order(self):
        return sorted(self.waiting, key=lambda s: s.priority, reverse=True)
