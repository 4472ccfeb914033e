"""Attention over a head-split KV cache (DuoAttention), B200-native.

Retrieval heads (one 0/1 bit per KV head) keep a full KV page and attend
causally over the whole history; streaming heads keep S attention-sink slots
plus an R-slot ring of recent tokens and attend with a Lambda-shaped mask.  All
arithmetic runs in hand-written CUDA kernels for sm_100a inside ``libduo.so``,
reached through its C ABI (``include/duo.h``); :mod:`.binding` is the thin
ctypes layer over it and :mod:`.cache` a convenience wrapper that allocates the
device buffers with PyTorch.  :mod:`.synth` produces seeded synthetic inputs.

Importing the package loads nothing; :func:`binding.lib` loads the shared
library and raises if it is missing.
"""

__all__ = ["binding", "cache", "synth"]
