"""``Sequence``: the unit of work that flows through the engine.

"Deep into the Nano-vLLM inference engine" (lnwmold.com), section "From
Prompts to Sequences": each prompt becomes a sequence, and the sequence is
the core unit the rest of the system handles.  "Nano-vLLM engine
architecture" (intelliparadigm.com) section 1.1 lists ``Sequence`` as the
carrier that tracks one generation task's state.  The pages list no fields;
the ones below are what the scheduler and block manager need.
"""

from __future__ import annotations

import enum
import itertools


class SequenceStatus(enum.Enum):
    WAITING = 0
    RUNNING = 1
    FINISHED = 2


_ids = itertools.count()


class Sequence:
    """Token ids of one request plus its place in the block pool.

    ``token_ids``          prompt followed by the tokens generated so far.
    ``num_prompt_tokens``  length of the original prompt.
    ``max_tokens``         generation budget (tokens after the prompt).
    ``num_cached_tokens``  leading tokens whose K/V were found in the prefix
                           cache at the last allocation (not recomputed).
    ``block_table``        physical block id of each logical block.
    """

    __slots__ = ("seq_id", "token_ids", "num_prompt_tokens", "max_tokens",
                 "num_cached_tokens", "block_table", "status", "priority",
                 "num_preemptions")

    def __init__(self, token_ids, max_tokens: int = 1, priority: int = 0, seq_id=None):
        if len(token_ids) == 0:
            raise ValueError("a sequence needs at least one prompt token")
        self.seq_id = next(_ids) if seq_id is None else seq_id
        self.token_ids = list(token_ids)
        self.num_prompt_tokens = len(self.token_ids)
        self.max_tokens = int(max_tokens)
        self.num_cached_tokens = 0
        self.block_table: list[int] = []
        self.status = SequenceStatus.WAITING
        self.priority = priority
        self.num_preemptions = 0

    def __len__(self) -> int:
        return len(self.token_ids)

    @property
    def num_tokens(self) -> int:
        return len(self.token_ids)

    @property
    def num_completion_tokens(self) -> int:
        return len(self.token_ids) - self.num_prompt_tokens

    @property
    def is_finished(self) -> bool:
        return self.status == SequenceStatus.FINISHED

    def num_blocks(self, block_size: int) -> int:
        return -(-len(self.token_ids) // block_size)

    def block_tokens(self, i: int, block_size: int) -> list:
        """Token ids held by logical block ``i``."""
        return self.token_ids[i * block_size:(i + 1) * block_size]

    def append_token(self, token_id: int) -> None:
        self.token_ids.append(int(token_id))

    def __repr__(self) -> str:
        return (f"Sequence(id={self.seq_id}, len={len(self)}, prompt={self.num_prompt_tokens}, "
                f"cached={self.num_cached_tokens}, blocks={self.block_table}, {self.status.name})")
