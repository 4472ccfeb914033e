"""Masked softmax attention in float64: the definition the CUDA path must reach.

Test infrastructure only (see ``oracle/__init__.py``).

What the method computes, from the pages:

* "DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
  Streaming Heads" (hotpaper.ai), abstract: retrieval heads need full attention
  across all tokens; streaming heads attend to recent tokens and attention sinks
  through a light-weight, constant-length KV cache; this applies to decoding and
  to pre-filling.  Same page, section "기술적 접근법" (technical approach): each
  Transformer layer holds two KV caches, a full one for retrieval heads and a
  fixed-length one (recent tokens and attention sinks only) for streaming heads;
  MHA and GQA are both supported.
* "韩松团队长上下文LLM推理高效框架" (cn.bg3.co), section "研究背景": under full
  attention every token attends to all preceding tokens (decode cost linear,
  pre-fill cost quadratic in the context).

The method therefore reaches *exactly* masked softmax attention, so the oracle
is that definition written out, evaluated in float64 on the exact stored input
values.  Readings taken where the pages are silent:

* scale: 1/sqrt(d) unless the caller overrides it;
* window: sinks are the absolute positions 0..S-1; "recent R" counts the
  current token, so query i sees key j iff j <= i and (j < S or i - j < R);
* GQA: one mask bit per KV head; query head h uses KV head h // G, G = Hq / Hkv;
* keys and queries arrive post-RoPE at their original positions.
"""

import numpy as np

__all__ = [
    "visible_mask",
    "masked_attention",
    "attend_head",
    "decode_reference",
    "prefill_reference",
    "default_scale",
]


def default_scale(head_dim):
    """Softmax temperature 1/sqrt(d) (the pages give none; standard reading)."""
    return 1.0 / np.sqrt(float(head_dim))


def visible_mask(query_pos, key_pos, retrieval, S, R):
    """Boolean [rows, keys]: may the query at ``query_pos[r]`` see ``key_pos[c]``.

    Retrieval head: the causal set {j <= i}.
    Streaming head: {j <= i : j < S  or  i - j < R} (sinks plus the R most
    recent positions, the current one included).
    """
    qp = np.asarray(query_pos, dtype=np.int64)[:, None]
    kp = np.asarray(key_pos, dtype=np.int64)[None, :]
    causal = kp <= qp
    if retrieval:
        return causal
    return causal & ((kp < S) | ((qp - kp) < R))


def masked_attention(q, k, v, mask, scale):
    """softmax(q k^T * scale, restricted to ``mask``) v, all in float64.

    q: [rows, d], k: [n, d], v: [n, dv], mask: bool [rows, n].  Every row must
    see at least one key (a query always sees itself).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if not np.all(mask.any(axis=1)):
        raise ValueError("a query row sees no key")
    s = (q @ k.T) * float(scale)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def attend_head(q_rows, query_pos, k, v, key_pos, retrieval, S, R, scale):
    """Attention of several query rows of one head against one KV history.

    ``k``/``v`` hold the keys/values at positions ``key_pos`` (the whole history
    of that KV head, or any superset of the visible set).
    """
    mask = visible_mask(query_pos, key_pos, retrieval, S, R)
    return masked_attention(q_rows, k, v, mask, scale)


def decode_reference(q, k_hist, v_hist, head_mask, S, R, scale=None):
    """One decode step: the query at position t = n-1 attends to the history.

    q: [B, Hq, d]; k_hist, v_hist: [B, n, Hkv, d], the full history including the
    token just appended; head_mask: [Hkv] with 1 = retrieval, 0 = streaming.
    Returns float64 [B, Hq, d].
    """
    q = np.asarray(q)
    B, Hq, d = q.shape
    n, Hkv = k_hist.shape[1], k_hist.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    scale = default_scale(d) if scale is None or scale <= 0 else scale
    t = n - 1
    keys = np.arange(n)
    out = np.empty((B, Hq, v_hist.shape[3]), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            rows = q[b, g * G:(g + 1) * G]
            out[b, g * G:(g + 1) * G] = attend_head(
                rows, np.full(G, t), k_hist[b, :, g], v_hist[b, :, g], keys,
                bool(head_mask[g]), S, R, scale)
    return out


def prefill_reference(q, k_hist, v_hist, c0, head_mask, S, R, scale=None,
                      rows=None):
    """Chunked pre-fill: the chunk's queries attend to everything before them.

    q: [B, C, Hq, d], the queries at positions c0..c0+C-1; k_hist, v_hist:
    [B, >= c0+C, Hkv, d], the history up to and including the chunk.
    ``rows`` optionally restricts the computation to those chunk rows.
    Returns float64 [B, len(rows), Hq, d].
    """
    q = np.asarray(q)
    B, C, Hq, d = q.shape
    Hkv = k_hist.shape[2]
    G = Hq // Hkv
    scale = default_scale(d) if scale is None or scale <= 0 else scale
    rows = np.arange(C) if rows is None else np.asarray(rows, dtype=np.int64)
    qpos = c0 + rows
    n = c0 + C
    keys = np.arange(n)
    out = np.empty((B, len(rows), Hq, v_hist.shape[3]), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            out[b, :, h] = attend_head(
                q[b, rows, h], qpos, k_hist[b, :n, g], v_hist[b, :n, g], keys,
                bool(head_mask[g]), S, R, scale)
    return out
