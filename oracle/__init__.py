"""Plain fp64 CPU oracle for attention over a head-split KV cache (DuoAttention).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
legs of ``bench.py`` may use it. It shares no code with the CUDA library in
``head_split_kv_decode_b200/`` and imports nothing from it; both sides receive
the same arrays from the seeded generators in ``head_split_kv_decode_b200/synth.py``,
a module that holds none of the method's arithmetic.

Modules
-------
attention  masked softmax attention (decode rows and prefill rows) with the
           retrieval (causal) and streaming (sink + recent, Lambda-shaped) masks
cache      the scalar ring-buffer append/evict simulation and the expected
           cache contents, plus the kept-KV byte count for a head mask
int4       the fp32 mirror of the asymmetric 4-bit KV quantiser and its
           exact dequantisation

Parity status: every function here is pinned by a ``-m "not gpu"`` test
(``tests/test_oracle_pins.py``); none is "parity unpinned" except the pages'
own memory-reduction figures, which the byte formula does not reproduce (the
pages never state the basis of their ratio).
"""

from . import attention, cache, int4  # noqa: F401
