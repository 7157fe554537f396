"""B200-native paged-KV attention: the data-parallel hot path of a nano-vLLM-style engine.

* ``ops``   -- thin ctypes binding over ``libpagedattn.so`` (the C-ABI library
  of hand-written sm_100a kernels): ``store_kvcache``, ``decode``,
  ``prefill_varlen``.  Importing it raises if the library is missing: there is
  no CPU or library fallback.
* ``host``  -- the CPU control plane: ``Sequence``, ``BlockManager`` (hash
  prefix cache, reference counts), ``Scheduler`` (prefill-first continuous
  batching with preemption) and the per-step metadata preparation.
* ``replay`` -- the continuous-batching trace replay that drives the library
  from the control plane.
* ``synth`` -- seeded synthetic inputs.
"""

__all__ = ["ops", "host", "replay", "synth"]
