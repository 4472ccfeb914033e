"""Decode parity: CUDA path (through the C ABI) against the fp64 oracle.

Covers the append/evict layouts bit for bit, the split-K retrieval path with
its log-sum-exp merge, the streaming path, MHA and GQA, fp32 and bf16, ragged
tails, context lengths around the streaming window, and every split count.
"""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache as OC
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache

from _util import assert_parity, f64, seeded_mask

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _build(B, Hq, Hkv, D, kind, n, S, R, n_ret, seed, chunks=None, capacity=None):
    """Fill a one-layer cache with n tokens (appended in the given chunk sizes,
    the last token alone) and return (cache, K, V, q, mask) with K/V/q as the
    exact device values."""
    mask = seeded_mask(seed, Hkv, n_ret)
    cache = DuoCache(1, B, Hq, Hkv, D, kind, capacity or n + 8, mask[None], S, R)
    K = synth.kv_field(seed * 10 + 1, range(B), range(n), Hkv, D, device="cuda").to(DT[kind])
    V = synth.kv_field(seed * 10 + 2, range(B), range(n), Hkv, D, device="cuda").to(DT[kind])
    q = synth.kv_field(seed * 10 + 3, range(B), [n - 1], Hq, D, device="cuda")[:, 0].to(DT[kind])
    pos = 0
    sizes = list(chunks or [])
    while pos < n - 1:
        c = sizes.pop(0) if sizes else n - 1 - pos
        c = min(c, n - 1 - pos)
        cache.append(0, K[:, pos:pos + c].contiguous(), V[:, pos:pos + c].contiguous())
        pos += c
    cache.append(0, K[:, n - 1:n].contiguous(), V[:, n - 1:n].contiguous())
    return cache, K, V, q, mask


def _oracle(K, V, q, mask, S, R, scale=None):
    return OA.decode_reference(f64(q), f64(K), f64(V), mask.numpy(), S, R, scale)


def _check_cache_bytes(cache, K, V, mask, S, R):
    """Device cache contents equal the oracle's scalar append model, bit for bit."""
    torch.cuda.synchronize()
    n = K.shape[1]
    lv = cache.layout(0)
    W = S + R
    rows = {name: cache.region(0, name).cpu() for name in ("ret_k", "ret_v", "str_k", "str_v")
            if cache.region(0, name) is not None}
    Kc = K.cpu().contiguous().view(torch.uint8).view(K.shape[0], n, K.shape[2], -1)
    Vc = V.cpu().contiguous().view(torch.uint8).view(V.shape[0], n, V.shape[2], -1)
    for h in range(K.shape[2]):
        idx = lv.packed_index[h]
        for b in range(K.shape[0]):
            if mask[h]:
                assert torch.equal(rows["ret_k"][b, idx, :n], Kc[b, :, h])
                assert torch.equal(rows["ret_v"][b, idx, :n], Vc[b, :, h])
            else:
                for src, name in ((Kc, "str_k"), (Vc, "str_v")):
                    exp, filled = OC.expected_streaming_buffer(src[b, :, h].numpy(), S, R)
                    got = rows[name][b, idx].numpy()
                    assert got.shape[0] == W
                    np.testing.assert_array_equal(got[filled], exp[filled])


def test_tiny_fp32_workload_full():
    """The tiny fp32 MHA workload: 8/8 heads, d 64, 512-token context, S4+R64,
    4 retrieval heads; append one token, then attend."""
    w = synth.WORKLOADS["tiny_mha_f32"]
    mask = synth.workload_mask(w)[0]
    n = w.context + 1
    cache = DuoCache(1, 1, w.n_q_heads, w.n_kv_heads, w.head_dim, "f32", n, mask[None], w.S, w.R)
    K = synth.history(w, 0, "k", [0], range(n), device="cuda", mask_row=mask)
    V = synth.history(w, 0, "v", [0], range(n), device="cuda", mask_row=mask)
    q = synth.queries(w, 0, [0], [n - 1], device="cuda")[:, 0]
    cache.append(0, K[:, :w.context].contiguous(), V[:, :w.context].contiguous())
    cache.append(0, K[:, w.context:].contiguous(), V[:, w.context:].contiguous())
    out = cache.decode(0, q)
    ref = _oracle(K, V, q, mask, w.S, w.R)
    assert_parity(out, ref, "f32", "tiny fp32")
    _check_cache_bytes(cache, K, V, mask, w.S, w.R)
    kept, full = cache.kv_bytes()
    assert (kept, full) == OC.kv_bytes(mask[None].numpy(), 1, n, w.S, w.R, w.head_dim, "f32")


@pytest.mark.parametrize("kind", ["f32", "bf16"])
@pytest.mark.parametrize("B,Hq,Hkv,D", [(1, 8, 8, 128), (2, 8, 2, 128), (1, 4, 4, 64), (3, 8, 4, 64)])
@pytest.mark.parametrize("n", [1, 5, 67, 68, 69, 200, 1031])
def test_decode_parity_small(kind, B, Hq, Hkv, D, n):
    S, R = 4, 64
    cache, K, V, q, mask = _build(B, Hq, Hkv, D, kind, n, S, R, n_ret=max(1, Hkv // 2),
                                  seed=n * 7 + D + Hkv, chunks=[3, 1, 50, 17, 1000])
    out = cache.decode(0, q)
    ref = _oracle(K, V, q, mask, S, R)
    assert_parity(out, ref, kind, "decode %s n=%d" % (kind, n))
    _check_cache_bytes(cache, K, V, mask, S, R)


@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_split_counts_agree(kind):
    B, Hq, Hkv, D, n, S, R = 2, 8, 2, 128, 9000, 64, 256
    cache, K, V, q, mask = _build(B, Hq, Hkv, D, kind, n, S, R, n_ret=1, seed=99,
                                  chunks=[4096, 4096])
    ref = _oracle(K, V, q, mask, S, R)
    outs = {}
    for splits in (1, 2, 7, 64, 512):
        cache.set_decode_splits(splits)
        outs[splits] = cache.decode(0, q).clone()
        assert_parity(outs[splits], ref, kind, "splits=%d" % splits)
    cache.set_decode_splits(0)
    auto = cache.decode(0, q)
    assert cache.decode_splits(0) > 1
    assert_parity(auto, ref, kind, "auto splits")
    for s, o in outs.items():
        assert (o.float() - outs[1].float()).abs().max().item() <= 2e-2


def test_scale_override_and_all_heads_of_one_kind():
    B, Hq, Hkv, D, n, S, R = 1, 8, 4, 128, 700, 4, 64
    for n_ret in (0, 4):
        cache, K, V, q, mask = _build(B, Hq, Hkv, D, "f32", n, S, R, n_ret=n_ret, seed=5 + n_ret)
        out = cache.decode(0, q, scale=0.05)
        ref = _oracle(K, V, q, mask, S, R, scale=0.05)
        assert_parity(out, ref, "f32", "n_ret=%d" % n_ret)


def test_many_decode_steps_wrap_the_ring():
    """Append-then-attend for 3*(S+R) steps: the ring wraps several times."""
    B, Hq, Hkv, D, S, R = 1, 4, 2, 64, 2, 5
    n0 = 3
    total = n0 + 3 * (S + R) + 4
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, D, "f32", total, mask[None], S, R)
    K = synth.kv_field(71, range(B), range(total), Hkv, D, device="cuda")
    V = synth.kv_field(72, range(B), range(total), Hkv, D, device="cuda")
    Q = synth.kv_field(73, range(B), range(total), Hq, D, device="cuda")
    cache.append(0, K[:, :n0].contiguous(), V[:, :n0].contiguous())
    for t in range(n0, total):
        cache.append(0, K[:, t:t + 1].contiguous(), V[:, t:t + 1].contiguous())
        out = cache.decode(0, Q[:, t].contiguous())
        ref = _oracle(K[:, :t + 1], V[:, :t + 1], Q[:, t], mask, S, R)
        assert_parity(out, ref, "f32", "step t=%d" % t)
    _check_cache_bytes(cache, K, V, mask, S, R)


def test_capacity_error_and_no_partial_state():
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, 1, 2, 2, 64, "f32", 10, mask[None], 2, 4)
    K = torch.zeros(1, 11, 2, 64, device="cuda")
    from head_split_kv_decode_b200.binding import DuoError
    with pytest.raises(DuoError) as e:
        cache.append(0, K, K)
    assert e.value.name == "DUO_ERR_CAPACITY"
    assert cache.seq_len(0) == 0
    cache.append(0, K[:, :10].contiguous(), K[:, :10].contiguous())
    assert cache.seq_len(0) == 10


def test_empty_inputs():
    """A zero-token append is a no-op (length, bytes and the next decode are
    unchanged); decoding a layer that holds no token is a state error."""
    from head_split_kv_decode_b200.binding import DuoError
    cache, K, V, q, mask = _build(2, 8, 2, 128, "bf16", 300, 4, 64, n_ret=1, seed=9)
    before = cache.decode(0, q).clone()
    nb = cache.kv_bytes()
    empty = torch.empty(2, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    cache.append(0, empty, empty)
    assert cache.seq_len(0) == 300 and cache.kv_bytes() == nb
    assert torch.equal(cache.decode(0, q), before)
    fresh = DuoCache(1, 2, 8, 2, 128, "bf16", 64, mask[None], 4, 64)
    with pytest.raises(DuoError) as e:
        fresh.decode(0, q)
    assert e.value.name == "DUO_ERR_STATE"


def test_workspace_too_small_is_rejected():
    from head_split_kv_decode_b200 import binding as B
    cache, K, V, q, mask = _build(1, 4, 2, 128, "bf16", 5000, 4, 64, n_ret=1, seed=3)
    out = torch.empty_like(q)
    with pytest.raises(B.DuoError) as e:
        B.duo_decode_attn(cache.handle, 0, q.data_ptr(), out.data_ptr(), 0.0, cache.ws_ptr, 16)
    assert e.value.name == "DUO_ERR_WORKSPACE"
    assert B.duo_poll_device_error() == 0


@pytest.mark.parametrize("kind,D,Hq,Hkv", [("bf16", 128, 8, 2), ("bf16", 128, 4, 4), ("f32", 64, 4, 2)])
def test_decode_step_fused_append(kind, D, Hq, Hkv):
    """duo_decode_step = append one token + attend, in one launch where a fused
    kernel exists; many steps so the ring wraps and the new token lands both in
    the middle of a split and at a split boundary."""
    B, S, R = 2, 3, 40
    n0, steps = 700, 90
    total = n0 + steps
    mask = torch.tensor([1] + [0] * (Hkv - 1), dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, D, kind, total, mask[None], S, R)
    K = synth.kv_field(81, range(B), range(total), Hkv, D, device="cuda").to(DT[kind])
    V = synth.kv_field(82, range(B), range(total), Hkv, D, device="cuda").to(DT[kind])
    Q = synth.kv_field(83, range(B), range(total), Hq, D, device="cuda").to(DT[kind])
    cache.append(0, K[:, :n0].contiguous(), V[:, :n0].contiguous())
    for t in range(n0, total):
        if t == n0 + 40:
            cache.set_decode_splits(3)
        out = cache.step(0, Q[:, t].contiguous(), K[:, t].contiguous(), V[:, t].contiguous())
        assert cache.seq_len(0) == t + 1
        if t % 7 == 0 or t == total - 1:
            ref = _oracle(K[:, :t + 1], V[:, :t + 1], Q[:, t], mask, S, R)
            assert_parity(out, ref, kind, "step t=%d" % t)
    _check_cache_bytes(cache, K, V, mask, S, R)


@pytest.mark.parametrize("kind,D", [("bf16", 128), ("f32", 64)])
@pytest.mark.parametrize("S,R", [(0, 1), (0, 16), (5, 1), (600, 700)])
def test_decode_degenerate_windows(kind, D, S, R):
    """The method's degenerate windows at decode: no sinks, a window of only the
    current token, sinks only plus the current token, and a window longer than
    the context (streaming = full attention).  Plain append + decode after a
    chunked fill, then fused steps that evict from the ring every step."""
    B, Hq, Hkv, n0, steps = 2, 8, 4, 333, 12
    total = n0 + steps
    mask = torch.tensor([1, 0, 0, 1], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, D, kind, total, mask[None], S, R)
    K = synth.kv_field(91 + S, range(B), range(total), Hkv, D, device="cuda").to(DT[kind])
    V = synth.kv_field(92 + R, range(B), range(total), Hkv, D, device="cuda").to(DT[kind])
    Q = synth.kv_field(93, range(B), range(total), Hq, D, device="cuda").to(DT[kind])
    for p0, p1 in ((0, 100), (100, 101), (101, n0)):
        cache.append(0, K[:, p0:p1].contiguous(), V[:, p0:p1].contiguous())
    out = cache.decode(0, Q[:, n0 - 1].contiguous())
    ref = _oracle(K[:, :n0], V[:, :n0], Q[:, n0 - 1], mask, S, R)
    assert_parity(out, ref, kind, "S=%d R=%d decode" % (S, R))
    for t in range(n0, total):
        out = cache.step(0, Q[:, t].contiguous(), K[:, t].contiguous(), V[:, t].contiguous())
        ref = _oracle(K[:, :t + 1], V[:, :t + 1], Q[:, t], mask, S, R)
        assert_parity(out, ref, kind, "S=%d R=%d step t=%d" % (S, R, t))
    _check_cache_bytes(cache, K, V, mask, S, R)


@pytest.mark.parametrize("kind,D,paged", [("bf16", 128, False), ("f32", 64, False), ("bf16", 128, True)])
def test_batch_beyond_one_launch(kind, D, paged):
    """130 batch rows: appends, decodes (automatic and forced split counts) and
    the fused step are issued as launches of at most 128 rows (paged: with
    each launch's rows reading through their own block tables)."""
    B, Hq, Hkv, n, S, R = 130, 4, 2, 45, 3, 8
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    kw = dict(pool_blocks=B + 3) if paged else {}
    cache = DuoCache(1, B, Hq, Hkv, D, kind, n + 4, mask[None], S, R, **kw)
    K = synth.kv_field(71, range(B), range(n + 1), Hkv, D, device="cuda").to(DT[kind])
    V = synth.kv_field(72, range(B), range(n + 1), Hkv, D, device="cuda").to(DT[kind])
    Q = synth.kv_field(73, range(B), range(n + 1), Hq, D, device="cuda").to(DT[kind])
    cache.append(0, K[:, :n - 1].contiguous(), V[:, :n - 1].contiguous())
    cache.append(0, K[:, n - 1:n].contiguous(), V[:, n - 1:n].contiguous())
    ref = _oracle(K[:, :n], V[:, :n], Q[:, n - 1], mask, S, R)
    for splits in (0, 3):
        cache.set_decode_splits(splits)
        out = cache.decode(0, Q[:, n - 1].contiguous())
        assert_parity(out, ref, kind, "130 rows, splits=%d" % splits)
    cache.set_decode_splits(0)
    out = cache.step(0, Q[:, n].contiguous(), K[:, n].contiguous(), V[:, n].contiguous())
    ref = _oracle(K, V, Q[:, n], mask, S, R)
    assert_parity(out, ref, kind, "130 rows, fused step")
    if paged:
        for r in (0, 127, 128, 129):  # retrieval rows through the block table
            got = cache.gather_rows(0, "ret_k", r, n + 1)[0].cpu()
            want = K[r, :, 0].cpu().contiguous().view(torch.uint8)
            assert torch.equal(got, want), r
    else:
        _check_cache_bytes(cache, K, V, mask, S, R)


@pytest.mark.parametrize("kind,D,paged", [("bf16", 128, False), ("f32", 64, False), ("bf16", 128, True)])
def test_layers_with_different_masks(kind, D, paged):
    """Three layers with different head masks (mixed, all streaming, all
    retrieval), filled to different lengths: each layer decodes against the
    oracle with its own mask and holds its own bytes (paged: the layers'
    retrieval rows share block ids but not storage)."""
    B, Hq, Hkv, S, R = 2, 8, 4, 4, 16
    masks = torch.tensor([[1, 0, 0, 1], [0, 0, 0, 0], [1, 1, 1, 1]], dtype=torch.uint8)
    lens = [300, 120, 517]
    kw = dict(pool_blocks=B * 3 + 2) if paged else {}
    cache = DuoCache(3, B, Hq, Hkv, D, kind, 600, masks, S, R, **kw)
    data = []
    for layer, n in enumerate(lens):
        K = synth.kv_field(100 + layer, range(B), range(n), Hkv, D, device="cuda").to(DT[kind])
        V = synth.kv_field(110 + layer, range(B), range(n), Hkv, D, device="cuda").to(DT[kind])
        q = synth.kv_field(120 + layer, range(B), [n - 1], Hq, D, device="cuda")[:, 0].to(DT[kind])
        data.append((K, V, q))
    for layer in (2, 0, 1):  # layers are filled in any order
        K, V, _ = data[layer]
        half = lens[layer] // 2
        cache.append(layer, K[:, :half].contiguous(), V[:, :half].contiguous())
        cache.append(layer, K[:, half:].contiguous(), V[:, half:].contiguous())
    for layer, n in enumerate(lens):
        K, V, q = data[layer]
        assert cache.seq_len(layer) == n
        out = cache.decode(layer, q)
        ref = _oracle(K, V, q, masks[layer], S, R)
        assert_parity(out, ref, kind, "layer %d" % layer)
        if not paged:
            torch.cuda.synchronize()
            lv = cache.layout(layer)
            rows = {nm: cache.region(layer, nm) for nm in ("ret_k", "str_k")}
            for h in range(Hkv):
                idx = lv.packed_index[h]
                want = K[1, :, h].cpu().contiguous().view(torch.uint8)
                if masks[layer][h]:
                    assert torch.equal(rows["ret_k"][1, idx, :n].cpu(), want)
                else:
                    exp, filled = OC.expected_streaming_buffer(want.numpy(), S, R)
                    got = rows["str_k"][1, idx].cpu().numpy()
                    np.testing.assert_array_equal(got[filled], exp[filled])
        elif masks[layer].any():
            got = cache.gather_rows(layer, "ret_k", 1, n)[0].cpu()
            h0 = int(torch.nonzero(masks[layer])[0])
            assert torch.equal(got, K[1, :, h0].cpu().contiguous().view(torch.uint8))


@pytest.mark.parametrize("kind,D", [("bf16", 128), ("f32", 64)])
def test_reproducible_mode(kind, D):
    """Fixed split shares: repeated decodes of one cache state are bit-identical;
    the default (pooled) mode agrees with them within rounding; both match the
    oracle."""
    B, Hq, Hkv, n, S, R = 2, 8, 2, 20000, 16, 128
    cache, K, V, q, mask = _build(B, Hq, Hkv, D, kind, n, S, R, n_ret=1, seed=123,
                                  chunks=[8192, 8192])
    assert cache.decode_splits(0) > 1
    ref = _oracle(K, V, q, mask, S, R)
    cache.set_decode_reproducible(True)
    outs = [cache.decode(0, q).clone() for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert_parity(outs[0], ref, kind, "reproducible")
    cache.set_decode_reproducible(False)
    pooled = cache.decode(0, q)
    assert_parity(pooled, ref, kind, "pooled")
    assert (pooled.float() - outs[0].float()).abs().max().item() <= 2e-2
