"""ctypes binding of ``libduo.so``: the C ABI of ``include/duo.h``, same names.

Argument marshalling only: every step of attention, append and merge runs in
the library's CUDA kernels.  Pointers are passed as integers (``tensor.data_ptr()``)
and streams as ``cudaStream_t`` integers.  A non-OK status raises
:class:`DuoError`.  If the library is missing, :func:`lib` raises: there is no
fallback path.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libduo.so")

MAX_KV_HEADS = 64
MAX_SPLITS = 512
DECODE_STATIC_SCRATCH_BYTES = 8 << 20
PAGE_TOKENS = 256
MAX_LAUNCH_ROWS = 128

DUO_OK = 0
STATUS_NAMES = {
    0: "DUO_OK", 1: "DUO_ERR_ARG", 2: "DUO_ERR_CAPACITY", 3: "DUO_ERR_LAYOUT",
    4: "DUO_ERR_WORKSPACE", 5: "DUO_ERR_CUDA", 6: "DUO_ERR_TIMEOUT",
    7: "DUO_ERR_UNSUPPORTED", 8: "DUO_ERR_STATE",
}
DUO_F32, DUO_BF16, DUO_INT4 = 0, 1, 2
DUO_LAYOUT_PACKED = 0
DUO_LAYOUT_PAGED = 1
KV_DTYPES = {"f32": DUO_F32, "bf16": DUO_BF16, "int4": DUO_INT4}


class DuoError(RuntimeError):
    def __init__(self, status, call):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        msg = "%s failed: %s" % (call, self.name)
        if _LIB is not None:
            msg += " (%s)" % _LIB.duo_status_string(status).decode()
        super().__init__(msg)


class duo_cache_desc(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("capacity", ctypes.c_int64)]


class duo_layout_view(ctypes.Structure):
    _fields_ = [("n_retrieval", ctypes.c_int32), ("n_streaming", ctypes.c_int32),
                ("window", ctypes.c_int32), ("window_stride", ctypes.c_int32),
                ("row_bytes", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("seq_len", ctypes.c_int64),
                ("ret_k", ctypes.c_int64), ("ret_v", ctypes.c_int64),
                ("str_k", ctypes.c_int64), ("str_v", ctypes.c_int64),
                ("ret_k_sz", ctypes.c_int64), ("ret_v_sz", ctypes.c_int64),
                ("str_k_sz", ctypes.c_int64), ("str_v_sz", ctypes.c_int64),
                ("kind", ctypes.c_int32 * MAX_KV_HEADS),
                ("packed_index", ctypes.c_int32 * MAX_KV_HEADS),
                ("layout", ctypes.c_int32), ("page_tokens", ctypes.c_int32),
                ("table_stride", ctypes.c_int32),
                ("pool_blocks", ctypes.c_int64), ("block_table", ctypes.c_int64)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float

# name -> (restype, argtypes); every function of include/duo.h
SIGNATURES = {
    "duo_cache_create": (_I32, [ctypes.POINTER(_P), ctypes.POINTER(duo_cache_desc), _P, _I32, _I32, _I32]),
    "duo_cache_create_paged": (_I32, [ctypes.POINTER(_P), ctypes.POINTER(duo_cache_desc), _P, _I32, _I32, _I64]),
    "duo_cache_destroy": (None, [_P]),
    "duo_cache_required_bytes": (_I32, [_P, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]),
    "duo_cache_bind": (_I32, [_P, _P, _SZ]),
    "duo_cache_reset": (_I32, [_P]),
    "duo_release_rows": (_I32, [_P, _P, _I32]),
    "duo_append_kv": (_I32, [_P, _I32, _P, _P, _I32, _P]),
    "duo_append_kv_rows": (_I32, [_P, _I32, _P, _I32, _P, _P, _I32, _P]),
    "duo_decode_attn": (_I32, [_P, _I32, _P, _P, _F, _P, _SZ, _P]),
    "duo_decode_attn_rows": (_I32, [_P, _I32, _P, _I32, _P, _P, _F, _P, _SZ, _P]),
    "duo_decode_step": (_I32, [_P, _I32, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "duo_decode_step_rows": (_I32, [_P, _I32, _P, _I32, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "duo_decode_attn_static": (_I32, [_P, _I32, _P, _P, _F, _P]),
    "duo_prefill_attn": (_I32, [_P, _I32, _P, _P, _P, _I32, _P, _F, _P, _SZ, _P]),
    "duo_prefill_attn_rows": (_I32, [_P, _I32, _P, _I32, _P, _P, _P, _I32, _P, _F, _P, _SZ, _P]),
    "duo_prefill_workspace_bytes": (_I32, [_P, ctypes.POINTER(_SZ)]),
    "duo_set_retrieval_shard": (_I32, [_P, _I64, _I64]),
    "duo_decode_attn_partial": (_I32, [_P, _I32, _P, _P, _P, _I32, _F, _P, _SZ, _P]),
    "duo_merge_partials": (_I32, [_I32, _I64, _I32, _P, _P, _P, _I32, _P]),
    "duo_seq_len": (_I32, [_P, _I32, ctypes.POINTER(_I64)]),
    "duo_row_seq_len": (_I32, [_P, _I32, _I32, ctypes.POINTER(_I64)]),
    "duo_row_blocks": (_I32, [_P, _I32, _P, _I32, ctypes.POINTER(_I32)]),
    "duo_pool_free_blocks": (_I32, [_P, ctypes.POINTER(_I64)]),
    "duo_kv_bytes": (_I32, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "duo_layout_info": (_I32, [_P, _I32, ctypes.POINTER(duo_layout_view)]),
    "duo_set_decode_splits": (_I32, [_P, _I32]),
    "duo_set_decode_reproducible": (_I32, [_P, _I32]),
    "duo_set_decode_output": (_I32, [_P, _I32]),
    "duo_test_stall_next_prefill": (_I32, [_P, _I64]),
    "duo_test_plan_decode": (_I32, [_P, _I32, ctypes.POINTER(_I32), _I32, _I32, _I32,
                                    ctypes.POINTER(_I32), ctypes.POINTER(_I32)]),
    "duo_decode_splits": (_I32, [_P, _I32, ctypes.POINTER(_I32)]),
    "duo_decode_streaming_pack": (_I32, [_P, _I32, ctypes.POINTER(_I32)]),
    "duo_poll_device_error": (_I32, [ctypes.POINTER(_I32)]),
    "duo_status_string": (ctypes.c_char_p, [_I32]),
}

_LIB = None


def lib():
    """Load ``libduo.so`` once and declare its signatures.  Raises if absent."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libduo.so is not built (%s); run `python -m head_split_kv_decode_b200.build`"
                % LIB_PATH)
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def _check(status, call):
    if status != DUO_OK:
        raise DuoError(status, call)


def duo_status_string(status):
    return lib().duo_status_string(status).decode()


def _desc_and_mask(layers, batch, n_q_heads, n_kv_heads, head_dim, kv_dtype, capacity, head_mask):
    desc = duo_cache_desc(layers, batch, n_q_heads, n_kv_heads, head_dim,
                          KV_DTYPES.get(kv_dtype, kv_dtype), capacity)
    vals = [int(x) for x in head_mask]
    if len(vals) != layers * n_kv_heads or any(not 0 <= x <= 255 for x in vals):
        raise ValueError("head_mask must hold layers * n_kv_heads byte values")
    return desc, (ctypes.c_uint8 * len(vals))(*vals)


def duo_cache_create(layers, batch, n_q_heads, n_kv_heads, head_dim, kv_dtype, capacity,
                     head_mask, S, R, layout=DUO_LAYOUT_PACKED):
    """head_mask: bytes-like / array of layers*n_kv_heads 0/1 values.  Returns a handle."""
    desc, mask = _desc_and_mask(layers, batch, n_q_heads, n_kv_heads, head_dim, kv_dtype,
                                capacity, head_mask)
    out = _P()
    _check(lib().duo_cache_create(ctypes.byref(out), ctypes.byref(desc), mask, S, R, layout),
           "duo_cache_create")
    return out.value


def duo_cache_create_paged(layers, batch, n_q_heads, n_kv_heads, head_dim, kv_dtype, capacity,
                           head_mask, S, R, pool_blocks):
    desc, mask = _desc_and_mask(layers, batch, n_q_heads, n_kv_heads, head_dim, kv_dtype,
                                capacity, head_mask)
    out = _P()
    _check(lib().duo_cache_create_paged(ctypes.byref(out), ctypes.byref(desc), mask, S, R,
                                        pool_blocks), "duo_cache_create_paged")
    return out.value


def _rows(rows):
    """(pointer, count) of an int32 row list; (None, 0) for every row."""
    if rows is None:
        return None, 0
    vals = [int(r) for r in rows]
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr, len(vals)


def duo_release_rows(handle, rows=None):
    arr, n = _rows(rows)
    _check(lib().duo_release_rows(handle, arr, n), "duo_release_rows")


def duo_append_kv_rows(handle, layer, rows, k_ptr, v_ptr, n_tokens, stream=0):
    arr, n = _rows(rows)
    _check(lib().duo_append_kv_rows(handle, layer, arr, n, k_ptr, v_ptr, n_tokens, stream),
           "duo_append_kv_rows")


def duo_decode_attn_rows(handle, layer, rows, q_ptr, out_ptr, softmax_scale, ws_ptr, ws_bytes,
                         stream=0):
    arr, n = _rows(rows)
    _check(lib().duo_decode_attn_rows(handle, layer, arr, n, q_ptr, out_ptr, softmax_scale, ws_ptr,
                                      ws_bytes, stream), "duo_decode_attn_rows")


def duo_decode_step_rows(handle, layer, rows, q_ptr, k_new_ptr, v_new_ptr, out_ptr, softmax_scale,
                         ws_ptr, ws_bytes, stream=0):
    arr, n = _rows(rows)
    _check(lib().duo_decode_step_rows(handle, layer, arr, n, q_ptr, k_new_ptr, v_new_ptr, out_ptr,
                                      softmax_scale, ws_ptr, ws_bytes, stream),
           "duo_decode_step_rows")


def duo_prefill_attn_rows(handle, layer, rows, q_ptr, k_ptr, v_ptr, C, out_ptr, softmax_scale,
                          ws_ptr=None, ws_bytes=0, stream=0):
    arr, n = _rows(rows)
    _check(lib().duo_prefill_attn_rows(handle, layer, arr, n, q_ptr, k_ptr, v_ptr, C, out_ptr,
                                       softmax_scale, ws_ptr, ws_bytes, stream),
           "duo_prefill_attn_rows")


def duo_prefill_workspace_bytes(handle):
    n = _SZ()
    _check(lib().duo_prefill_workspace_bytes(handle, ctypes.byref(n)), "duo_prefill_workspace_bytes")
    return n.value


def duo_row_seq_len(handle, layer, row):
    n = _I64()
    _check(lib().duo_row_seq_len(handle, layer, row, ctypes.byref(n)), "duo_row_seq_len")
    return n.value


def duo_row_blocks(handle, row):
    n = _I32()
    _check(lib().duo_row_blocks(handle, row, None, 0, ctypes.byref(n)), "duo_row_blocks")
    arr = (ctypes.c_int32 * max(1, n.value))()
    _check(lib().duo_row_blocks(handle, row, arr, n.value, ctypes.byref(n)), "duo_row_blocks")
    return list(arr[:n.value])


def duo_pool_free_blocks(handle):
    n = _I64()
    _check(lib().duo_pool_free_blocks(handle, ctypes.byref(n)), "duo_pool_free_blocks")
    return n.value


def duo_cache_destroy(handle):
    lib().duo_cache_destroy(handle)


def duo_cache_required_bytes(handle):
    cb, wb = _SZ(), _SZ()
    _check(lib().duo_cache_required_bytes(handle, ctypes.byref(cb), ctypes.byref(wb)),
           "duo_cache_required_bytes")
    return cb.value, wb.value


def duo_cache_bind(handle, ptr, nbytes):
    _check(lib().duo_cache_bind(handle, ptr, nbytes), "duo_cache_bind")


def duo_cache_reset(handle):
    _check(lib().duo_cache_reset(handle), "duo_cache_reset")


def duo_append_kv(handle, layer, k_ptr, v_ptr, n_tokens, stream=0):
    _check(lib().duo_append_kv(handle, layer, k_ptr, v_ptr, n_tokens, stream), "duo_append_kv")


def duo_decode_attn(handle, layer, q_ptr, out_ptr, softmax_scale, ws_ptr, ws_bytes, stream=0):
    _check(lib().duo_decode_attn(handle, layer, q_ptr, out_ptr, softmax_scale, ws_ptr,
                                 ws_bytes, stream), "duo_decode_attn")


def duo_decode_step(handle, layer, q_ptr, k_new_ptr, v_new_ptr, out_ptr, softmax_scale, ws_ptr,
                    ws_bytes, stream=0):
    _check(lib().duo_decode_step(handle, layer, q_ptr, k_new_ptr, v_new_ptr, out_ptr, softmax_scale,
                                 ws_ptr, ws_bytes, stream), "duo_decode_step")


def duo_decode_attn_static(handle, layer, q_ptr, out_ptr, softmax_scale, stream=0):
    """Decode without a workspace: the library's own fixed scratch array is used
    (see include/duo.h for its limit and the serialisation rule)."""
    _check(lib().duo_decode_attn_static(handle, layer, q_ptr, out_ptr, softmax_scale, stream),
           "duo_decode_attn_static")


def duo_prefill_attn(handle, layer, q_ptr, k_ptr, v_ptr, C, out_ptr, softmax_scale,
                     ws_ptr=None, ws_bytes=0, stream=0):
    _check(lib().duo_prefill_attn(handle, layer, q_ptr, k_ptr, v_ptr, C, out_ptr,
                                  softmax_scale, ws_ptr, ws_bytes, stream), "duo_prefill_attn")


def duo_seq_len(handle, layer):
    n = _I64()
    _check(lib().duo_seq_len(handle, layer, ctypes.byref(n)), "duo_seq_len")
    return n.value


def duo_kv_bytes(handle):
    kept, full = _I64(), _I64()
    _check(lib().duo_kv_bytes(handle, ctypes.byref(kept), ctypes.byref(full)), "duo_kv_bytes")
    return kept.value, full.value


def duo_layout_info(handle, layer):
    v = duo_layout_view()
    _check(lib().duo_layout_info(handle, layer, ctypes.byref(v)), "duo_layout_info")
    return v


def duo_set_decode_splits(handle, splits):
    _check(lib().duo_set_decode_splits(handle, splits), "duo_set_decode_splits")


def duo_test_stall_next_prefill(handle, wait_ns):
    """Testing hook: the next pre-fill loads nothing and its waits give up
    after wait_ns (the timeout path, without any fault)."""
    _check(lib().duo_test_stall_next_prefill(handle, int(wait_ns)), "duo_test_stall_next_prefill")


def duo_test_plan_decode(handle, layer, lens, num_sms, ctas_per_sm=1):
    """Testing hook: the tensor-core decode's plan for one launch of rows with
    these lengths (query included) on num_sms SMs, computed on the host.
    Returns (splits per row, streaming heads per streaming CTA)."""
    n = len(lens)
    arr = (_I32 * max(n, 1))(*[int(x) for x in lens])
    out = (_I32 * max(n, 1))()
    pack = _I32()
    _check(lib().duo_test_plan_decode(handle, layer, arr, n, num_sms, ctas_per_sm, out,
                                      ctypes.byref(pack)), "duo_test_plan_decode")
    return list(out)[:n], pack.value


def duo_set_decode_output(handle, dtype):
    """dtype: "f32" or "bf16" (the element type of decode outputs)."""
    _check(lib().duo_set_decode_output(handle, KV_DTYPES[dtype]), "duo_set_decode_output")


def duo_set_decode_reproducible(handle, on):
    _check(lib().duo_set_decode_reproducible(handle, 1 if on else 0), "duo_set_decode_reproducible")


def duo_decode_splits(handle, layer):
    s = _I32()
    _check(lib().duo_decode_splits(handle, layer, ctypes.byref(s)), "duo_decode_splits")
    return s.value


def duo_decode_streaming_pack(handle, layer):
    s = _I32()
    _check(lib().duo_decode_streaming_pack(handle, layer, ctypes.byref(s)), "duo_decode_streaming_pack")
    return s.value


def duo_poll_device_error():
    """Returns the raw device error word (0 = none) and clears it."""
    code = _I32()
    st = lib().duo_poll_device_error(ctypes.byref(code))
    if st not in (DUO_OK, 6):
        raise DuoError(st, "duo_poll_device_error")
    return code.value


def duo_set_retrieval_shard(handle, lo, hi):
    _check(lib().duo_set_retrieval_shard(handle, lo, hi), "duo_set_retrieval_shard")


def duo_decode_attn_partial(handle, layer, q_ptr, o_ptr, lse_ptr, owns_streaming, softmax_scale,
                            ws_ptr, ws_bytes, stream=0):
    _check(lib().duo_decode_attn_partial(handle, layer, q_ptr, o_ptr, lse_ptr,
                                         1 if owns_streaming else 0, softmax_scale, ws_ptr,
                                         ws_bytes, stream), "duo_decode_attn_partial")


def duo_merge_partials(n_parts, rows, head_dim, o_ptr, lse_ptr, out_ptr, out_dtype, stream=0):
    _check(lib().duo_merge_partials(n_parts, rows, head_dim, o_ptr, lse_ptr, out_ptr,
                                    KV_DTYPES.get(out_dtype, out_dtype), stream),
           "duo_merge_partials")
