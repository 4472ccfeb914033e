"""Chunked pre-fill parity: the tcgen05 kernel (through the C ABI) against the
fp64 oracle, causal for retrieval heads and Lambda-masked for streaming heads.

Covers chunks starting at 0 and in the middle of a prompt, ragged chunk
lengths (not multiples of the 128-row tile), windows smaller and larger than a
tile, the sink edge inside a chunk, MHA and GQA, batch > 1, and a whole prompt
fed chunk by chunk with the append between chunks.
"""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache

from _util import assert_parity, f64, seeded_mask

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


def _prompt(seed, B, n, Hq, Hkv, D=128):
    K = synth.kv_field(seed * 10 + 1, range(B), range(n), Hkv, D, device="cuda").to(BF)
    V = synth.kv_field(seed * 10 + 2, range(B), range(n), Hkv, D, device="cuda").to(BF)
    Q = synth.kv_field(seed * 10 + 3, range(B), range(n), Hq, D, device="cuda").to(BF)
    return Q, K, V


def _run_chunks(cache, Q, K, V, bounds, check_rows=None):
    """Feed [c0, c1) chunks: attend, then append.  Returns [(c0, out)]."""
    outs = []
    for c0, c1 in bounds:
        q = Q[:, c0:c1].contiguous()
        k = K[:, c0:c1].contiguous()
        v = V[:, c0:c1].contiguous()
        assert cache.seq_len(0) == c0
        o = cache.prefill(0, q, k, v)
        cache.append(0, k, v)
        outs.append((c0, o.clone()))
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("B,Hq,Hkv", [(1, 8, 2), (2, 4, 4)])
@pytest.mark.parametrize("S,R", [(4, 64), (64, 256), (0, 1), (200, 50)])
@pytest.mark.parametrize("bounds", [[(0, 128)], [(0, 300)], [(0, 257), (257, 700)],
                                    [(0, 100), (100, 612), (612, 1000)]])
def test_prefill_parity_small(B, Hq, Hkv, S, R, bounds):
    n = bounds[-1][1]
    seed = n + 7 * S + R + Hq
    Q, K, V = _prompt(seed, B, n, Hq, Hkv)
    mask = seeded_mask(seed, Hkv, max(1, Hkv // 2))
    cache = DuoCache(1, B, Hq, Hkv, 128, "bf16", n, mask[None], S, R)
    outs = _run_chunks(cache, Q, K, V, bounds)
    Kd, Vd = f64(K), f64(V)
    for (c0, o), (_, c1) in zip(outs, bounds):
        ref = OA.prefill_reference(f64(Q[:, c0:c1]), Kd, Vd, c0, mask.numpy(), S, R)
        assert_parity(o, ref, "bf16", "chunk [%d,%d) S=%d R=%d" % (c0, c1, S, R))


def test_prefill_batch_beyond_one_launch():
    """130 batch rows: the pre-fill (and the appends between chunks) is issued
    as launches of at most 128 rows; every row matches the oracle."""
    B, Hq, Hkv, n, S, R = 130, 4, 2, 300, 4, 64
    Q, K, V = _prompt(55, B, n, Hq, Hkv)
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, 128, "bf16", n, mask[None], S, R)
    bounds = [(0, 100), (100, 300)]
    outs = _run_chunks(cache, Q, K, V, bounds)
    Kd, Vd = f64(K), f64(V)
    for (c0, o), (_, c1) in zip(outs, bounds):
        ref = OA.prefill_reference(f64(Q[:, c0:c1]), Kd, Vd, c0, mask.numpy(), S, R)
        assert_parity(o, ref, "bf16", "130 rows chunk [%d,%d)" % (c0, c1))


def test_prefill_all_heads_one_kind():
    B, Hq, Hkv, n = 1, 4, 2, 600
    for bits in ([1, 1], [0, 0]):
        Q, K, V = _prompt(31 + bits[0], B, n, Hq, Hkv)
        mask = torch.tensor(bits, dtype=torch.uint8)
        cache = DuoCache(1, B, Hq, Hkv, 128, "bf16", n, mask[None], 64, 256)
        outs = _run_chunks(cache, Q, K, V, [(0, 300), (300, 600)])
        for c0, o in outs:
            ref = OA.prefill_reference(f64(Q[:, c0:c0 + 300]), f64(K), f64(V), c0, mask.numpy(), 64, 256)
            assert_parity(o, ref, "bf16", "mask %s c0=%d" % (bits, c0))


def test_prefill_then_decode_continues_the_same_cache():
    """Pre-fill a prompt in chunks, then decode: the decode sees exactly what the
    pre-fill appended (one consistent cache for both paths)."""
    B, Hq, Hkv, n = 1, 8, 2, 900
    S, R = 16, 128
    Q, K, V = _prompt(77, B, n + 1, Hq, Hkv)
    mask = torch.tensor([0, 1], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, 128, "bf16", n + 1, mask[None], S, R)
    _run_chunks(cache, Q, K, V, [(0, 512), (512, n)])
    cache.append(0, K[:, n:n + 1].contiguous(), V[:, n:n + 1].contiguous())
    out = cache.decode(0, Q[:, n].contiguous())
    ref = OA.decode_reference(f64(Q[:, n]), f64(K), f64(V), mask.numpy(), S, R)
    assert_parity(out, ref, "bf16", "decode after prefill")


def test_prefill_rejects_unsupported_and_capacity():
    from head_split_kv_decode_b200.binding import DuoError
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    c32 = DuoCache(1, 1, 2, 2, 128, "f32", 256, mask[None], 4, 64)
    q = torch.zeros(1, 128, 2, 128, device="cuda")
    with pytest.raises(DuoError) as e:
        c32.prefill(0, q, q, q)
    assert e.value.name == "DUO_ERR_UNSUPPORTED"
    cb = DuoCache(1, 1, 2, 2, 128, "bf16", 100, mask[None], 4, 64)
    qb = torch.zeros(1, 128, 2, 128, device="cuda", dtype=BF)
    with pytest.raises(DuoError) as e:
        cb.prefill(0, qb, qb, qb)
    assert e.value.name == "DUO_ERR_CAPACITY"


def _int4_view(x):
    """What a 4-bit cache holds for bf16 rows x [B, n, H, D]: the exact
    dequantisation of each (token, head) group, float64."""
    from oracle import int4 as OQ
    return OQ.dequantize_int4(*OQ.quantize_int4(x.float().cpu().numpy()))


@pytest.mark.parametrize("B,Hq,Hkv,S,R", [(1, 8, 2, 4, 64), (2, 8, 4, 64, 256)])
@pytest.mark.parametrize("paged", [False, True])
def test_prefill_int4_cache(B, Hq, Hkv, S, R, paged):
    """Chunks attend to a 4-bit cache (expanded to bf16 for the tensor cores)
    plus their own bf16 k/v; the oracle reads the dequantised history exactly.
    The expansion workspace starts full of NaN bytes: the library writes every
    row the tensor-core pass reads (keys, then zeros to the tile's end), so the
    caller needs no zero fill."""
    bounds = [(0, 300), (300, 812), (812, 1500)]
    n = bounds[-1][1]
    seed = 41 + Hkv + S
    Q, K, V = _prompt(seed, B, n, Hq, Hkv)
    mask = seeded_mask(seed, Hkv, max(1, Hkv // 2))
    kw = dict(pool_blocks=B * 8) if paged else {}
    cache = DuoCache(1, B, Hq, Hkv, 128, "int4", n, mask[None], S, R, **kw)
    assert cache.prefill_ws_bytes > 0
    cache._prefill_ws()
    cache._pf_ws.fill_(0xFF)  # every bf16 in it is a NaN
    outs = _run_chunks(cache, Q, K, V, bounds)
    Kq, Vq = _int4_view(K), _int4_view(V)
    for (c0, o), (_, c1) in zip(outs, bounds):
        k_view = np.concatenate([Kq[:, :c0], f64(K[:, c0:c1])], axis=1)
        v_view = np.concatenate([Vq[:, :c0], f64(V[:, c0:c1])], axis=1)
        ref = OA.prefill_reference(f64(Q[:, c0:c1]), k_view, v_view, c0, mask.numpy(), S, R)
        assert_parity(o, ref, "bf16", "int4 prefill chunk at %d" % c0)


def test_prefill_int4_needs_workspace():
    from head_split_kv_decode_b200 import binding as Bd
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    c4 = DuoCache(1, 1, 8, 2, 128, "int4", 512, mask[None], 4, 64)
    qb = torch.zeros(1, 128, 8, 128, device="cuda", dtype=BF)
    kb = torch.zeros(1, 128, 2, 128, device="cuda", dtype=BF)
    with pytest.raises(Bd.DuoError) as e:
        Bd.duo_prefill_attn(c4.handle, 0, qb.data_ptr(), kb.data_ptr(), kb.data_ptr(), 128,
                            qb.data_ptr(), 0.0, None, 0)
    assert e.value.name == "DUO_ERR_WORKSPACE"


def test_prefill_bounded_wait_gives_up_and_recovers():
    """The failure path of the bounded waits, with no fault: the testing hook
    makes the next pre-fill issue no tile loads and shortens its wait limit to
    2 ms, so every wait of the MMA and softmax roles runs out.  Each CTA
    records the timeout, frees its tensor memory and returns; the output is
    left as it was; duo_poll_device_error reports DUO_ERR_TIMEOUT.  The same
    process then runs a normal pre-fill that matches the oracle."""
    from head_split_kv_decode_b200 import binding as Bd
    B, Hq, Hkv, C, S, R = 1, 8, 2, 256, 4, 64
    Q, K, V = _prompt(91, B, C, Hq, Hkv)
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, 128, "bf16", C, mask[None], S, R)
    assert Bd.duo_poll_device_error() == 0
    with pytest.raises(Bd.DuoError):
        Bd.duo_test_stall_next_prefill(cache.handle, 10)  # below the allowed range
    Bd.duo_test_stall_next_prefill(cache.handle, 2_000_000)
    sentinel = torch.full((B, C, Hq, 128), 7.0, dtype=BF, device="cuda")
    cache.prefill(0, Q, K, V, out=sentinel)
    torch.cuda.synchronize()
    code = Bd.duo_poll_device_error()
    assert code != 0, "the stalled pre-fill did not report a timeout"
    assert (code & 2) != 0  # kErrWaitMma: the MMA / softmax waits gave up
    assert torch.all(sentinel == 7.0)  # no CTA wrote its output
    assert Bd.duo_poll_device_error() == 0  # polling clears the word
    out = cache.prefill(0, Q, K, V)  # the hook was one-shot
    torch.cuda.synchronize()
    assert Bd.duo_poll_device_error() == 0
    ref = OA.prefill_reference(f64(Q), f64(K), f64(V), 0, mask.numpy(), S, R)
    assert_parity(out, ref, "bf16", "pre-fill after a stalled call")
