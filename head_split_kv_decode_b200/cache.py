"""PyTorch-facing wrapper of the C ABI: allocates the cache and workspace as
torch tensors, checks tensor arguments and forwards to :mod:`.binding`.

PyTorch is used for device memory and streams only; every byte of K/V/Q/O is
read and written by the library's kernels.
"""

import torch

from . import binding as B

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "int4": torch.bfloat16}
_ALIGN = 256


def _aligned_buffer(nbytes, device, zero):
    buf = (torch.zeros if zero else torch.empty)(nbytes + _ALIGN, dtype=torch.uint8, device=device)
    base = buf.data_ptr()
    off = (-base) % _ALIGN
    return buf, off


def _stream_handle(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


class DuoCache:
    """A head-split KV cache for ``layers`` layers bound to torch-allocated memory.

    head_mask: [layers, n_kv_heads] of 0/1 (1 = retrieval head).
    kv_dtype: "f32", "bf16" or "int4" (K/V given in bf16 and quantised on append).
    pool_blocks: None for the packed layout (``capacity`` tokens reserved per
    batch row), or the block count of the paged layout's retrieval pool
    (blocks of ``binding.PAGE_TOKENS`` tokens taken by rows as they grow;
    ``capacity`` then bounds one row).  Each batch row is a sequence slot with
    its own length; the ``*_rows`` methods act on a list of rows.
    """

    def __init__(self, layers, batch, n_q_heads, n_kv_heads, head_dim, kv_dtype, capacity,
                 head_mask, S, R, device="cuda", pool_blocks=None):
        mask = torch.as_tensor(head_mask).reshape(-1).to(torch.uint8).tolist()
        if pool_blocks is None:
            self.handle = B.duo_cache_create(layers, batch, n_q_heads, n_kv_heads, head_dim,
                                             kv_dtype, capacity, mask, S, R)
        else:
            self.handle = B.duo_cache_create_paged(layers, batch, n_q_heads, n_kv_heads, head_dim,
                                                   kv_dtype, capacity, mask, S, R, pool_blocks)
        self.paged = pool_blocks is not None
        self.layers, self.batch = layers, batch
        self.n_q_heads, self.n_kv_heads, self.head_dim = n_q_heads, n_kv_heads, head_dim
        self.kv_dtype, self.capacity, self.S, self.R = kv_dtype, capacity, S, R
        self.io_dtype = _TORCH_DTYPE[kv_dtype]
        self.out_dtype = self.io_dtype  # decode outputs (see set_decode_output)
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.cache_bytes, self.ws_bytes = B.duo_cache_required_bytes(self.handle)
        self._storage, off = _aligned_buffer(self.cache_bytes, self.device, zero=False)
        self.base_ptr = self._storage.data_ptr() + off
        self.storage = self._storage[off:off + self.cache_bytes]
        B.duo_cache_bind(self.handle, self.base_ptr, self.cache_bytes)
        self._ws, woff = _aligned_buffer(self.ws_bytes, self.device, zero=True)
        self.ws_ptr = self._ws.data_ptr() + woff
        self.prefill_ws_bytes = B.duo_prefill_workspace_bytes(self.handle)
        self._pf_ws, self.pf_ws_ptr = None, None

    def _prefill_ws(self):
        """Pre-fill scratch (4-bit caches only), allocated on first use."""
        if self.prefill_ws_bytes == 0:
            return None, 0
        if self._pf_ws is None:
            self._pf_ws, off = _aligned_buffer(self.prefill_ws_bytes, self.device, zero=False)
            self.pf_ws_ptr = self._pf_ws.data_ptr() + off
        return self.pf_ws_ptr, self.prefill_ws_bytes

    # ------------------------------------------------------------ checks
    def _check(self, t, shape, name, dtype=None):
        if not isinstance(t, torch.Tensor):
            raise TypeError("%s must be a torch tensor" % name)
        if t.device != self.device:
            raise ValueError("%s is on %s, cache on %s" % (name, t.device, self.device))
        if tuple(t.shape) != tuple(shape):
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
        if t.dtype != (dtype or self.io_dtype):
            raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype or self.io_dtype))
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)

    # ------------------------------------------------------------ calls
    def append(self, layer, k, v, stream=None):
        """k, v: [batch, n_tokens, n_kv_heads, head_dim]."""
        n = k.shape[1]
        shape = (self.batch, n, self.n_kv_heads, self.head_dim)
        self._check(k, shape, "k")
        self._check(v, shape, "v")
        B.duo_append_kv(self.handle, layer, k.data_ptr(), v.data_ptr(), n,
                        _stream_handle(stream, self.device))

    def decode(self, layer, q, out=None, scale=0.0, stream=None):
        """q: [batch, n_q_heads, head_dim] at position seq_len-1.  Returns out."""
        shape = (self.batch, self.n_q_heads, self.head_dim)
        self._check(q, shape, "q")
        if out is None:
            out = torch.empty(shape, dtype=self.out_dtype, device=q.device)
        self._check(out, shape, "out", self.out_dtype)
        B.duo_decode_attn(self.handle, layer, q.data_ptr(), out.data_ptr(), float(scale),
                          self.ws_ptr, self.ws_bytes, _stream_handle(stream, self.device))
        return out

    def step(self, layer, q, k_new, v_new, out=None, scale=0.0, stream=None):
        """Append one token (k_new, v_new: [batch, n_kv_heads, head_dim]) and
        attend with q at its position, in one launch where possible."""
        kv_shape = (self.batch, self.n_kv_heads, self.head_dim)
        shape = (self.batch, self.n_q_heads, self.head_dim)
        self._check(q, shape, "q")
        self._check(k_new, kv_shape, "k_new")
        self._check(v_new, kv_shape, "v_new")
        if out is None:
            out = torch.empty(shape, dtype=self.out_dtype, device=q.device)
        self._check(out, shape, "out", self.out_dtype)
        B.duo_decode_step(self.handle, layer, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(),
                          out.data_ptr(), float(scale), self.ws_ptr, self.ws_bytes,
                          _stream_handle(stream, self.device))
        return out

    def prefill(self, layer, q, k, v, out=None, scale=0.0, stream=None):
        """q: [batch, C, n_q_heads, d]; k, v: [batch, C, n_kv_heads, d].  Attends only."""
        C = q.shape[1]
        self._check(q, (self.batch, C, self.n_q_heads, self.head_dim), "q")
        self._check(k, (self.batch, C, self.n_kv_heads, self.head_dim), "k")
        self._check(v, (self.batch, C, self.n_kv_heads, self.head_dim), "v")
        if out is None:
            out = torch.empty_like(q)
        self._check(out, tuple(q.shape), "out")
        ws, wsb = self._prefill_ws()
        B.duo_prefill_attn(self.handle, layer, q.data_ptr(), k.data_ptr(), v.data_ptr(), C,
                           out.data_ptr(), float(scale), ws, wsb,
                           _stream_handle(stream, self.device))
        return out

    # ------------------------------------------------------------ row calls
    def _rows(self, rows):
        rows = [int(r) for r in rows]
        if not rows:
            raise ValueError("empty row list")
        return rows

    def append_rows(self, layer, rows, k, v, stream=None):
        """k, v: [len(rows), n_tokens, n_kv_heads, head_dim] for the listed rows."""
        rows = self._rows(rows)
        n = k.shape[1]
        shape = (len(rows), n, self.n_kv_heads, self.head_dim)
        self._check(k, shape, "k")
        self._check(v, shape, "v")
        B.duo_append_kv_rows(self.handle, layer, rows, k.data_ptr(), v.data_ptr(), n,
                             _stream_handle(stream, self.device))

    def decode_rows(self, layer, rows, q, out=None, scale=0.0, stream=None):
        """q: [len(rows), n_q_heads, head_dim], each row's query at its last position."""
        rows = self._rows(rows)
        shape = (len(rows), self.n_q_heads, self.head_dim)
        self._check(q, shape, "q")
        if out is None:
            out = torch.empty(shape, dtype=self.out_dtype, device=q.device)
        self._check(out, shape, "out", self.out_dtype)
        B.duo_decode_attn_rows(self.handle, layer, rows, q.data_ptr(), out.data_ptr(), float(scale),
                               self.ws_ptr, self.ws_bytes, _stream_handle(stream, self.device))
        return out

    def step_rows(self, layer, rows, q, k_new, v_new, out=None, scale=0.0, stream=None):
        """Append one token to each listed row and attend (see :meth:`step`)."""
        rows = self._rows(rows)
        kv_shape = (len(rows), self.n_kv_heads, self.head_dim)
        shape = (len(rows), self.n_q_heads, self.head_dim)
        self._check(q, shape, "q")
        self._check(k_new, kv_shape, "k_new")
        self._check(v_new, kv_shape, "v_new")
        if out is None:
            out = torch.empty(shape, dtype=self.out_dtype, device=q.device)
        self._check(out, shape, "out", self.out_dtype)
        B.duo_decode_step_rows(self.handle, layer, rows, q.data_ptr(), k_new.data_ptr(),
                               v_new.data_ptr(), out.data_ptr(), float(scale), self.ws_ptr,
                               self.ws_bytes, _stream_handle(stream, self.device))
        return out

    def prefill_rows(self, layer, rows, q, k, v, out=None, scale=0.0, stream=None):
        """q: [len(rows), C, n_q_heads, d]; k, v: [len(rows), C, n_kv_heads, d]."""
        rows = self._rows(rows)
        C = q.shape[1]
        self._check(q, (len(rows), C, self.n_q_heads, self.head_dim), "q")
        self._check(k, (len(rows), C, self.n_kv_heads, self.head_dim), "k")
        self._check(v, (len(rows), C, self.n_kv_heads, self.head_dim), "v")
        if out is None:
            out = torch.empty_like(q)
        self._check(out, tuple(q.shape), "out")
        ws, wsb = self._prefill_ws()
        B.duo_prefill_attn_rows(self.handle, layer, rows, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                C, out.data_ptr(), float(scale), ws, wsb,
                                _stream_handle(stream, self.device))
        return out

    # ------------------------------------------------------------ sequence shards
    def set_retrieval_shard(self, lo, hi):
        """Keep only retrieval positions [lo, hi) (call before any append)."""
        B.duo_set_retrieval_shard(self.handle, int(lo), int(hi))

    def decode_partial(self, layer, q, o_part=None, lse_part=None, owns_streaming=True, scale=0.0,
                       stream=None):
        """This cache's share of the decode: returns (o_part f32 [batch, Hq, d],
        lse_part f32 [batch, Hq]) to merge with :func:`merge_partials`."""
        shape = (self.batch, self.n_q_heads, self.head_dim)
        self._check(q, shape, "q")
        if o_part is None:
            o_part = torch.empty(shape, dtype=torch.float32, device=q.device)
        if lse_part is None:
            lse_part = torch.empty(shape[:2], dtype=torch.float32, device=q.device)
        self._check(o_part, shape, "o_part", torch.float32)
        self._check(lse_part, shape[:2], "lse_part", torch.float32)
        B.duo_decode_attn_partial(self.handle, layer, q.data_ptr(), o_part.data_ptr(),
                                  lse_part.data_ptr(), owns_streaming, float(scale), self.ws_ptr,
                                  self.ws_bytes, _stream_handle(stream, self.device))
        return o_part, lse_part

    def release_rows(self, rows=None):
        B.duo_release_rows(self.handle, None if rows is None else self._rows(rows))

    def row_seq_len(self, layer, row):
        return B.duo_row_seq_len(self.handle, layer, row)

    def row_blocks(self, row):
        return B.duo_row_blocks(self.handle, row)

    def pool_free_blocks(self):
        return B.duo_pool_free_blocks(self.handle)

    # ------------------------------------------------------------ introspection
    def seq_len(self, layer):
        return B.duo_seq_len(self.handle, layer)

    def kv_bytes(self):
        return B.duo_kv_bytes(self.handle)

    def layout(self, layer):
        return B.duo_layout_info(self.handle, layer)

    def set_decode_splits(self, splits):
        B.duo_set_decode_splits(self.handle, splits)

    def set_decode_output(self, dtype):
        """Element type of decode outputs: torch.float32 or torch.bfloat16
        (bf16 and 4-bit caches; an fp32 cache always outputs float32)."""
        name = {torch.float32: "f32", torch.bfloat16: "bf16"}[dtype]
        B.duo_set_decode_output(self.handle, name)
        self.out_dtype = dtype

    def set_decode_reproducible(self, on=True):
        """Fixed key shares per decode split: bit-identical repeated calls."""
        B.duo_set_decode_reproducible(self.handle, on)

    def decode_splits(self, layer):
        return B.duo_decode_splits(self.handle, layer)

    def decode_streaming_pack(self, layer):
        """Streaming heads per streaming CTA of the next decode of `layer`."""
        return B.duo_decode_streaming_pack(self.handle, layer)

    def reset(self):
        B.duo_cache_reset(self.handle)

    def region(self, layer, name):
        """Raw view of one buffer of one layer (for inspection and tests).

        name in ret_k, ret_v, str_k, str_v (rows of K/V elements or int4 codes) and,
        for int4, ret_k_sz, ret_v_sz, str_k_sz, str_v_sz (fp16 scale/zero pairs).
        Returns a uint8 tensor [batch, heads, rows, row_bytes] (or [..., 4]);
        paged retrieval buffers are [pool_blocks, heads, page_tokens, ...].
        """
        lv = self.layout(layer)
        off = getattr(lv, name)
        if off < 0:
            return None
        heads = lv.n_retrieval if name.startswith("ret") else lv.n_streaming
        outer, rows = self.batch, (lv.capacity if name.startswith("ret") else lv.window_stride)
        if self.paged and name.startswith("ret"):
            outer, rows = lv.pool_blocks, lv.page_tokens
        width = 4 if name.endswith("_sz") else lv.row_bytes
        nbytes = outer * heads * rows * width
        return self.storage[off:off + nbytes].view(outer, heads, rows, width)

    def gather_rows(self, layer, name, row, n):
        """The first n retrieval rows of one batch row, in position order, as
        [heads, n, width] (packed: a slice; paged: through the block table)."""
        reg = self.region(layer, name)
        if reg is None:
            return None
        if not self.paged:
            return reg[row, :, :n]
        P = self.layout(layer).page_tokens
        blocks = self.row_blocks(row)
        parts = [reg[blk] for blk in blocks[:(n + P - 1) // P]]
        return torch.cat(parts, dim=1)[:, :n]

    def close(self):
        if getattr(self, "handle", None):
            B.duo_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def merge_partials(o_parts, lse_parts, out, stream=None):
    """o_parts f32 [n, batch, Hq, d], lse_parts f32 [n, batch, Hq] (device,
    contiguous) -> out [batch, Hq, d] (bf16 or f32): the attention over the
    union of the shards' keys."""
    n, rows, d = o_parts.shape[0], o_parts[0].numel() // o_parts.shape[-1], o_parts.shape[-1]
    if tuple(lse_parts.shape) != tuple(o_parts.shape[:-1]) or tuple(out.shape) != tuple(o_parts.shape[1:]):
        raise ValueError("partials and output shapes disagree")
    for t in (o_parts, lse_parts, out):
        if not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError("partials and output must be contiguous device tensors")
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise ValueError("partials must be float32")
    kind = {torch.bfloat16: "bf16", torch.float32: "f32"}.get(out.dtype)
    if kind is None:
        raise ValueError("out must be bfloat16 or float32")
    s = stream if stream is not None else torch.cuda.current_stream(out.device)
    B.duo_merge_partials(n, rows, d, o_parts.data_ptr(), lse_parts.data_ptr(), out.data_ptr(), kind,
                         s.cuda_stream)
    return out
