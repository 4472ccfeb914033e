"""Host-side checks of the C ABI that need no GPU: the library builds and loads,
it exports every function ``include/duo.h`` declares, and the host logic
(argument checks, layout planning, byte accounting) behaves."""

import os
import re

import pytest

from head_split_kv_decode_b200 import binding as B
from head_split_kv_decode_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.lib()


def declared_functions():
    names = []
    for hdr in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(duo_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in B.SIGNATURES, "binding lacks %s" % n


def _create(**kw):
    args = dict(layers=2, batch=2, n_q_heads=8, n_kv_heads=4, head_dim=128, kv_dtype="bf16",
                capacity=1000, head_mask=[1, 0, 0, 1, 0, 0, 0, 0], S=4, R=60)
    args.update(kw)
    return B.duo_cache_create(**args)


def test_create_and_layout(lib):
    h = _create()
    try:
        cb, wb = B.duo_cache_required_bytes(h)
        v0 = B.duo_layout_info(h, 0)
        v1 = B.duo_layout_info(h, 1)
        assert (v0.n_retrieval, v0.n_streaming) == (2, 2)
        assert (v1.n_retrieval, v1.n_streaming) == (0, 4)
        assert v0.window == 64 and v0.row_bytes == 256 and v0.capacity == 1000
        assert list(v0.kind)[:4] == [1, 0, 0, 1]
        assert list(v0.packed_index)[:4] == [0, 0, 1, 1]
        assert v1.ret_k == -1 and v1.ret_v == -1
        assert v0.ret_k_sz == -1  # bf16 has no scale/zero buffers
        regions = [(v0.ret_k, 2 * 2 * 1000 * 256), (v0.ret_v, 2 * 2 * 1000 * 256),
                   (v0.str_k, 2 * 2 * 64 * 256), (v0.str_v, 2 * 2 * 64 * 256),
                   (v1.str_k, 2 * 4 * 64 * 256), (v1.str_v, 2 * 4 * 64 * 256)]
        for off, size in regions:
            assert off % 256 == 0
        regions.sort()
        for (a, sa), (b, _) in zip(regions, regions[1:]):
            assert a + sa <= b, "regions overlap"
        assert regions[-1][0] + regions[-1][1] <= cb
        assert wb > 0
        assert B.duo_kv_bytes(h) == (0, 0)
        assert B.duo_seq_len(h, 1) == 0
    finally:
        B.duo_cache_destroy(h)


def test_int4_layout_has_scale_zero(lib):
    h = _create(kv_dtype="int4")
    try:
        v = B.duo_layout_info(h, 0)
        assert v.row_bytes == 64
        assert min(v.ret_k_sz, v.ret_v_sz, v.str_k_sz, v.str_v_sz) >= 0
    finally:
        B.duo_cache_destroy(h)


@pytest.mark.parametrize("bad", [
    dict(n_kv_heads=3, head_mask=[1, 0, 0, 0, 1, 0]),  # does not divide n_q_heads
    dict(head_dim=96),
    dict(capacity=0),
    dict(R=0),
    dict(S=-1),
    dict(kv_dtype=7),
    dict(head_mask=[2, 0, 0, 0, 0, 0, 0, 0]),
    dict(n_kv_heads=80, n_q_heads=80, head_mask=[0] * 160),
])
def test_create_rejects_bad_arguments(lib, bad):
    with pytest.raises(B.DuoError) as e:
        _create(**bad)
    assert e.value.name in ("DUO_ERR_ARG", "DUO_ERR_LAYOUT")


def test_mask_length_checked_in_binding(lib):
    with pytest.raises(ValueError):
        _create(head_mask=[1, 0, 0])


def test_calls_before_bind_fail_cleanly(lib):
    h = _create()
    try:
        with pytest.raises(B.DuoError) as e:
            B.duo_append_kv(h, 0, 16, 16, 1)
        assert e.value.name == "DUO_ERR_STATE"
        with pytest.raises(B.DuoError) as e:
            B.duo_decode_attn(h, 0, 16, 16, 0.0, None, 0)
        assert e.value.name == "DUO_ERR_STATE"
        with pytest.raises(B.DuoError) as e:
            B.duo_append_kv(h, 5, 16, 16, 1)
        assert e.value.name == "DUO_ERR_ARG"
        with pytest.raises(B.DuoError):
            B.duo_set_decode_splits(h, B.MAX_SPLITS + 1)
        B.duo_set_decode_splits(h, 7)
        B.duo_set_decode_splits(h, 0)
        assert B.STATUS_NAMES[lib.duo_set_decode_reproducible(h, 2)] == "DUO_ERR_ARG"
        assert B.STATUS_NAMES[lib.duo_set_decode_reproducible(None, 1)] == "DUO_ERR_ARG"
        B.duo_set_decode_reproducible(h, True)
        B.duo_set_decode_reproducible(h, False)
    finally:
        B.duo_cache_destroy(h)


def test_status_strings(lib):
    for s in range(9):
        assert B.duo_status_string(s)
    assert "unknown" in B.duo_status_string(99)


def _create_paged(pool_blocks=10, **kw):
    args = dict(layers=2, batch=3, n_q_heads=8, n_kv_heads=4, head_dim=128, kv_dtype="bf16",
                capacity=1000, head_mask=[1, 0, 0, 1, 0, 1, 0, 0], S=4, R=60,
                pool_blocks=pool_blocks)
    args.update(kw)
    return B.duo_cache_create_paged(**args)


def test_paged_layout_plan(lib):
    """Pool buffers [blocks][n_ret][256][row] per layer, then one block table
    [batch][ceil(capacity/256)] of int32; every byte accounted for."""
    h = _create_paged()
    try:
        cb, _ = B.duo_cache_required_bytes(h)
        v0, v1 = B.duo_layout_info(h, 0), B.duo_layout_info(h, 1)
        assert v0.layout == B.DUO_LAYOUT_PAGED and v0.page_tokens == B.PAGE_TOKENS == 256
        assert v0.pool_blocks == 10 and v0.table_stride == 4  # ceil(1000 / 256)
        assert (v0.n_retrieval, v1.n_retrieval) == (2, 1)
        pool0 = 10 * 2 * 256 * 256
        assert v0.ret_k == 0 and v0.ret_v == pool0
        assert v0.str_k == 2 * pool0 and v0.str_v == v0.str_k + 3 * 2 * 64 * 256
        pool1 = 10 * 1 * 256 * 256
        assert v1.ret_v - v1.ret_k == pool1
        assert v0.block_table == v1.str_v + 3 * 3 * 64 * 256
        assert cb == v0.block_table + 3 * 4 * 4 + (-(3 * 4 * 4) % 256)
        assert B.duo_pool_free_blocks(h) == 10
        assert B.duo_row_blocks(h, 0) == []
        assert B.duo_row_seq_len(h, 1, 2) == 0
        B.duo_release_rows(h, [2, 0])
        B.duo_release_rows(h)
        for rows in ([3], [1, 1], [-1]):
            with pytest.raises(B.DuoError) as e:
                B.duo_release_rows(h, rows)
            assert e.value.name == "DUO_ERR_ARG"
        # row calls before bind fail before touching anything
        with pytest.raises(B.DuoError) as e:
            B.duo_append_kv_rows(h, 0, [1], 16, 16, 1)
        assert e.value.name == "DUO_ERR_STATE"
        packed = _create()
        try:
            vp = B.duo_layout_info(packed, 0)
            assert vp.layout == B.DUO_LAYOUT_PACKED and vp.page_tokens == 0
            assert vp.block_table == -1 and B.duo_pool_free_blocks(packed) == 0
        finally:
            B.duo_cache_destroy(packed)
    finally:
        B.duo_cache_destroy(h)


def test_paged_create_rejects(lib):
    with pytest.raises(B.DuoError) as e:
        _create_paged(pool_blocks=0)
    assert e.value.name == "DUO_ERR_ARG"
    for kw in (dict(kv_dtype="f32"), dict(head_dim=64)):
        with pytest.raises(B.DuoError) as e:  # no tensor-core decode for these
            _create_paged(**kw)
        assert e.value.name == "DUO_ERR_UNSUPPORTED"
    with pytest.raises(B.DuoError) as e:  # the paged layout has its own create call
        _create(layout=B.DUO_LAYOUT_PAGED)
    assert e.value.name == "DUO_ERR_ARG"
    h = _create_paged(kv_dtype="int4")
    try:
        v = B.duo_layout_info(h, 0)
        pool = 10 * 2 * 256  # rows of each retrieval buffer
        assert v.ret_v == pool * 64 and v.str_k == 2 * pool * 64
        assert v.ret_k_sz == v.str_v + 3 * 2 * 64 * 64  # after the streaming codes
        assert v.ret_v_sz - v.ret_k_sz == pool * 4
    finally:
        B.duo_cache_destroy(h)


def test_binding_signatures_match_the_header():
    """Every prototype in include/duo.h and the ctypes signature the binding
    declares for it agree on arity and on each argument's kind (pointer,
    32-bit or 64-bit integer, float), so the two cannot drift apart."""
    import ctypes
    import re
    from head_split_kv_decode_b200 import binding as Bd

    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "duo.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    protos = {}
    for m in re.finditer(r"\b(duo_status|void|const char \*)\s*(duo_\w+)\s*\(([^)]*)\)\s*;", hdr):
        args = [a.strip() for a in m.group(3).split(",") if a.strip() and a.strip() != "void"]
        protos[m.group(2)] = args

    def kind_c(decl):
        if "*" in decl or decl.startswith("duo_stream"):
            return "ptr"
        if decl.startswith(("int64_t", "size_t")):
            return "i64"
        if decl.startswith("float"):
            return "f32"
        if decl.startswith(("int32_t", "int ", "duo_status")):
            return "i32"
        raise AssertionError("unknown C type: " + decl)

    def kind_py(t):
        if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and not isinstance(t._type_, str):
            return "ptr"
        if t in (ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64):
            return "i64"
        if t is ctypes.c_float:
            return "f32"
        if t in (ctypes.c_int32, ctypes.c_uint32):
            return "i32"
        raise AssertionError("unknown ctypes type: %r" % (t,))

    assert set(protos) == set(Bd.SIGNATURES), set(protos) ^ set(Bd.SIGNATURES)
    for name, (_, argtypes) in Bd.SIGNATURES.items():
        c_kinds = [kind_c(a) for a in protos[name]]
        py_kinds = [kind_py(t) for t in argtypes]
        assert c_kinds == py_kinds, (name, c_kinds, py_kinds)
