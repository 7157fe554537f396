"""Host control plane: sequences, the block manager and the scheduler.

Runs in CPU memory and produces the metadata (block tables, slot mappings,
context lengths, cumulative sequence lengths) that the GPU data plane reads.
"""

from .sequence import Sequence, SequenceStatus  # noqa: F401
from .block_manager import Block, BlockManager, PoolExhausted, chain_hash  # noqa: F401
from .scheduler import Scheduler, SchedulerConfig, PriorityScheduler  # noqa: F401
from .prepare import (  # noqa: F401
    PrefillMetadata, DecodeMetadata, prepare_prefill, prepare_decode, slots_for,
    block_tables_array,
)
