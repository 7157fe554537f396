"""CPU oracle for the paged-KV attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the
``paged_kv_attention_35_b200`` package and its C-ABI library) may import,
call or link anything in this package.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` /
``--impl reference`` legs use it.

What it is: a plain, slow, obviously correct numpy float64 statement of what
the hot path computes, written from the pages' description of the nano-vLLM
engine:

* ``paged``  -- slot assignment, the store (scatter) into the block pool,
  the per-sequence gather through a block table, decode attention and varlen
  causal prefill attention with a cached prefix.
* ``brute``  -- a second, scalar pure-Python formulation (``math.exp`` /
  ``math.fsum`` triple loops) used to pin ``paged`` on tiny inputs.

The pages (three articles on nano-vLLM) never write the attention formula or
the physical cache layout down: the third page ("Deep into the Nano-vLLM
inference engine", lnwmold.com news item, section "What's Next") defers both
to an unpublished second part.  The readings taken here are listed in each
function's docstring: separate K and V pools laid out
``[num_blocks, block_size, num_kv_heads, head_dim]``, a slot is the flat token
row ``block_id * block_size + offset``, negative slots are skipped, the GQA
query head ``h`` reads KV head ``h // (Hq // Hkv)``, softmax scale
``1/sqrt(head_dim)`` unless given, and the causal mask of a prefill with a
cached prefix is bottom-right aligned.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(brute force, closed forms, library special cases, invariants, planted
mistakes).
"""

from .paged import (  # noqa: F401
    bf16_bits_to_f64,
    f64_to_bf16_bits,
    ref_slot_mapping,
    ref_store,
    ref_gather,
    ref_decode,
    ref_prefill,
    ref_prefill_flops,
)
