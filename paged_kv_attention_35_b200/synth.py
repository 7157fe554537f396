"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and names workload sizes; it holds none
of the attention, store or slot arithmetic.  Values are drawn on the CPU
(device-independent), so the same seed gives the same inputs on every machine.

* ``bf16_normal``      -- N(0, 1) float32 draws from a seeded CPU
  ``torch.Generator``, rounded to bf16 (torch's round-to-nearest-even cast).
* ``uniform_lengths``  -- integers uniform in ``[lo, hi]`` (inclusive) from
  ``numpy.random.default_rng(seed)``.
* ``permutation``      -- a seeded permutation of ``0 .. n-1`` (the shuffled
  free-block order of the pool).
* ``token_ids``        -- seeded token ids in ``[0, vocab)``.

Workload shapes (the five configurations exercised by the tests and the bench)
are in ``WORKLOADS``.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SEED_BASE = 1000
VOCAB = 151_936
NAN_BF16_BITS = 0x7FC0          # quiet NaN, used to poison unused pool rows


def bf16_normal(shape, seed: int) -> torch.Tensor:
    """CPU bf16 tensor of N(0,1) draws (float32 draws rounded to bf16)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(torch.bfloat16)


def uniform_lengths(n: int, lo: int, hi: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(int(seed))
    return rng.integers(lo, hi + 1, size=int(n)).astype(np.int64)


def permutation(n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(int(seed))
    return rng.permutation(int(n)).astype(np.int64)


def token_ids(n: int, seed: int, vocab: int = VOCAB) -> list:
    rng = np.random.default_rng(int(seed))
    return rng.integers(0, vocab, size=int(n)).tolist()


@dataclass(frozen=True)
class Workload:
    """Sizes of one synthetic workload (names follow the pages' engine)."""
    name: str
    kind: str                       # "decode" | "prefill" | "replay"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_seqs: int = 0
    ctx_lo: int = 0
    ctx_hi: int = 0
    fixed_lens: tuple = ()
    pool_factor: float = 1.25       # pool blocks = ceil(factor * blocks needed)
    num_blocks: int = 0             # fixed pool size (when nonzero)
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return SEED_BASE + WORKLOAD_INDEX[self.name]


WORKLOADS = {
    # tiny decode step: 4 seqs, context lens [17,64,100,255], 4 Q / 2 KV heads,
    # head_dim 64, block 16, pool of 64 shuffled blocks, scale 1/sqrt(64)
    "tiny_decode": Workload("tiny_decode", "decode", 4, 2, 64, 16, num_seqs=4,
                            fixed_lens=(17, 64, 100, 255), num_blocks=64),
    # one layer of Qwen3-0.6B-shaped decode: batch 32, ctx U[128,4096], 16/8, D128, block 256
    "qwen3_0p6b_decode": Workload("qwen3_0p6b_decode", "decode", 16, 8, 128, 256,
                                  num_seqs=32, ctx_lo=128, ctx_hi=4096),
    # one layer of 7B-GQA decode: batch 256, ctx U[512,4096], 28/4, D128, block 256 (and 16)
    "gqa7b_decode": Workload("gqa7b_decode", "decode", 28, 4, 128, 256,
                             num_seqs=256, ctx_lo=512, ctx_hi=4096),
    # prefix-cached varlen prefill: 16 seqs, 8 fresh U[256,2048], 8 sharing a
    # 1024-token prefix with totals U[1025,2048]; 28/4, D128, block 256
    "prefix_prefill": Workload("prefix_prefill", "prefill", 28, 4, 128, 256,
                               num_seqs=16, ctx_lo=256, ctx_hi=2048,
                               extra={"shared_prefix": 1024, "num_shared": 8}),
    # continuous-batching trace replay: 512 requests, prompt/output U[100,1024],
    # max_num_seqs 256, block 256, 28 layers of 16/8 x D128, pool of 768 blocks
    "trace_replay": Workload("trace_replay", "replay", 16, 8, 128, 256,
                             num_seqs=512, ctx_lo=100, ctx_hi=1024, num_blocks=768,
                             extra={"num_layers": 28, "max_num_seqs": 256,
                                    "max_num_batched_tokens": 16384,
                                    "max_model_len": 4096}),
}
WORKLOAD_INDEX = {n: i + 1 for i, n in enumerate(WORKLOADS)}   # configs numbered 1..5
