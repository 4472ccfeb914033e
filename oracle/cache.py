"""Scalar model of the two KV caches: append/evict and the bytes they keep.

Test infrastructure only (see ``oracle/__init__.py``).

Pages: "What is DuoAttention" (nav.superapi.store), section "Technical
principles of DuoAttention": retrieval heads retain a full KV cache; streaming
heads use a fixed-length KV cache of recent tokens and attention sinks.  The
takechan.xyz re-post of the same article, paragraph "流式头的轻量化 KV 缓存",
says the same (a constant-length cache).  The pages fix no slot order; the
reading used here (and by the CUDA path, independently written) is:

* retrieval KV head: position p lives in row p of its page;
* streaming KV head: W = S + R slots; position p < S lives in sink slot p,
  any later position in slot S + ((p - S) mod R), overwriting (evicting) the
  position R earlier.

The simulation below walks tokens one at a time, which is the plainest form of
that rule; the expected buffers it produces are compared byte for byte with the
device cache.
"""

import numpy as np

__all__ = [
    "ring_slot",
    "simulate_ring",
    "expected_streaming_buffer",
    "kept_tokens",
    "kv_bytes",
    "bytes_per_token_per_head",
]


def ring_slot(p, S, R):
    """Slot of position ``p`` in a streaming head's W = S + R slot buffer."""
    if p < S:
        return p
    return S + (p - S) % R


def simulate_ring(n, S, R):
    """Append positions 0..n-1 one by one; return {slot: position held}."""
    held = {}
    for p in range(n):
        held[ring_slot(p, S, R)] = p
    return held


def expected_streaming_buffer(k_head, S, R):
    """Expected [W, d] contents of one streaming head after appending
    ``k_head`` ([n, d], positions 0..n-1) token by token.

    Returns (buffer, filled): rows never written are zero and ``filled`` is
    False there.
    """
    k_head = np.asarray(k_head)
    n, d = k_head.shape
    W = S + R
    buf = np.zeros((W, d), dtype=k_head.dtype)
    filled = np.zeros(W, dtype=bool)
    for slot, p in simulate_ring(n, S, R).items():
        buf[slot] = k_head[p]
        filled[slot] = True
    return buf, filled


def kept_tokens(n, retrieval, S, R):
    """Tokens a KV head holds after n appends: n (retrieval), min(n, S+R) else."""
    return n if retrieval else min(n, S + R)


def bytes_per_token_per_head(head_dim, kv_dtype):
    """K+V bytes one token occupies in one KV head.

    f32: 8d, bf16: 4d, int4: 2 * (d/2 codes + 2 fp16 scale/zero) = d + 8.
    """
    if kv_dtype == "f32":
        return 8 * head_dim
    if kv_dtype == "bf16":
        return 4 * head_dim
    if kv_dtype == "int4":
        return 2 * (head_dim // 2 + 4)
    raise ValueError(kv_dtype)


def kv_bytes(head_mask, batch, n, S, R, head_dim, kv_dtype):
    """(kept, full): KV bytes the split cache holds after n tokens, and what a
    full cache for every head would hold.  head_mask: [layers][Hkv] of 0/1.
    """
    per = bytes_per_token_per_head(head_dim, kv_dtype)
    mask = np.asarray(head_mask)
    kept = 0
    for layer in mask:
        for bit in layer:
            kept += batch * kept_tokens(n, bool(bit), S, R) * per
    full = mask.size * batch * n * per
    return int(kept), int(full)
