"""Plain fp64 CPU oracle for the paged decode-attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code
with the CUDA library (no kernels, headers, helpers or generators); inputs
reach it as plain arrays.

Sources (web pages on PagedAttention):
  * "PagedAttention blog" (0539edu.com), section 3(3) "processing a single
    request" and section 4 "parallel sampling" -- logical blocks of B tokens,
    the block table, filled slots, the decode-time gather, copy-on-write.
  * "Month 2 · PagedAttention" study guide (weishuz.com), section 02 (OS to
    vLLM mapping table), section 03 reading 4 (block_table and slot_mapping
    handed to the attention kernel) and section 06 (the kernel is ordinary
    attention that gathers K and V from non-contiguous addresses).

Every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py``; none is "parity unpinned".
"""

from .paged_attention import (  # noqa: F401
    gather_kv,
    decode_attention,
    decode_attention_one,
    prefill_attention,
    reshape_and_cache,
    copy_blocks,
)
