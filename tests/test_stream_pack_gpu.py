"""Streaming heads packed several to a CTA (tensor-core decode, bf16 cache).

When a layer's streaming windows are short next to its retrieval splits, the
planner runs 2, 4 or 8 of a row's streaming heads in one CTA, one group of
warps each, and gives the SMs this frees to retrieval splits.  Each case
checks that packing was chosen and compares the CUDA path with the fp64
oracle: MHA (one query per KV head), a pack whose last CTA has fewer heads
than groups, the fused step (new token written and attended by the head's
group) with float32 output, rows of different lengths (packed and paged
layouts), sequence shards (partial outputs, the streaming heads on one shard
only), and the 4-bit cache.
"""

import pytest
import torch

from oracle import attention as OA
from head_split_kv_decode_b200 import shard, synth
from head_split_kv_decode_b200.binding import duo_poll_device_error
from head_split_kv_decode_b200.cache import DuoCache, merge_partials

from _util import assert_parity, f64
from test_decode_gpu import _check_cache_bytes

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
D = 128


def _mask(Hkv, ret):
    m = torch.zeros(Hkv, dtype=torch.uint8)
    m[list(ret)] = 1
    return m


def _seq(seed, B_, n, heads):
    return synth.kv_field(seed, range(B_), range(n), heads, D, device="cuda").to(BF)


def _filled(B_, Hq, Hkv, n, S, R, mask, seed, cap=None):
    cache = DuoCache(1, B_, Hq, Hkv, D, "bf16", cap or n + 8, mask[None], S, R)
    K, V = _seq(seed * 10 + 1, B_, n, Hkv), _seq(seed * 10 + 2, B_, n, Hkv)
    for p0 in range(0, n, 8192):
        cache.append(0, K[:, p0:p0 + 8192].contiguous(), V[:, p0:p0 + 8192].contiguous())
    return cache, K, V


@pytest.mark.parametrize("Hq,Hkv,ret,n,S,R", [
    (16, 16, (0, 4, 8, 12), 24576, 4, 60),   # MHA: 12 streaming heads
    (32, 8, (0, 5), 60000, 4, 60),           # GQA: 6 streaming heads
    (32, 8, (0, 3, 6), 40000, 4, 28),        # 5 streaming heads: a CTA with idle groups
])
def test_packed_decode_matches_oracle(Hq, Hkv, ret, n, S, R):
    mask = _mask(Hkv, ret)
    cache, K, V = _filled(1, Hq, Hkv, n, S, R, mask, seed=Hkv + n)
    pack = cache.decode_streaming_pack(0)
    assert pack in (2, 4, 8), pack
    q = synth.kv_field(n + 7, [0], [n - 1], Hq, D, device="cuda")[:, 0].to(BF)
    out = cache.decode(0, q)
    torch.cuda.synchronize()
    ref = OA.decode_reference(f64(q), f64(K), f64(V), mask.numpy(), S, R)
    assert_parity(out, ref, "bf16", "pack %d, %d streaming heads" % (pack, Hkv - len(ret)))
    assert duo_poll_device_error() == 0


def test_packed_fused_step_f32():
    """duo_decode_step with packed streaming heads: each group's first warp
    writes its head's new row into the ring and attends to it; outputs in
    float32 against the oracle at every step, then every cache byte."""
    Hq, Hkv, S, R, n0, steps = 16, 16, 4, 60, 24576, 4
    mask = _mask(Hkv, (1, 6, 11, 15))
    n = n0 + steps
    cache, K, V = _filled(1, Hq, Hkv, n0, S, R, mask, seed=5, cap=n)
    Kx, Vx = _seq(51, 1, steps, Hkv), _seq(52, 1, steps, Hkv)
    K, V = torch.cat([K, Kx], 1), torch.cat([V, Vx], 1)
    Q = _seq(53, 1, steps, Hq)
    cache.set_decode_output(torch.float32)
    assert cache.decode_streaming_pack(0) > 1
    for i in range(steps):
        t = n0 + i
        q = Q[:, i].contiguous()
        out = cache.step(0, q, K[:, t].contiguous(), V[:, t].contiguous())
        torch.cuda.synchronize()
        ref = OA.decode_reference(f64(q), f64(K[:, :t + 1]), f64(V[:, :t + 1]), mask.numpy(), S, R)
        assert_parity(out, ref, "bf16", "packed fused step at %d" % t)
    _check_cache_bytes(cache, K, V, mask, S, R)
    assert duo_poll_device_error() == 0


def test_packed_rows_of_different_lengths():
    """Three rows of 30000, 12000 and 700 tokens in one launch; the pack is
    chosen per launch from the longest window and the rows' splits."""
    Hq, Hkv, S, R = 32, 8, 4, 60
    mask = _mask(Hkv, (2, 7))
    lens = [30000, 12000, 700]
    cache = DuoCache(1, 3, Hq, Hkv, D, "bf16", max(lens) + 8, mask[None], S, R)
    K, V = _seq(61, 3, max(lens), Hkv), _seq(62, 3, max(lens), Hkv)
    for r, n in enumerate(lens):
        for p0 in range(0, n, 8192):
            p1 = min(n, p0 + 8192)
            cache.append_rows(0, [r], K[r:r + 1, p0:p1].contiguous(), V[r:r + 1, p0:p1].contiguous())
    assert cache.decode_streaming_pack(0) > 1
    q = synth.kv_field(63, range(3), [0], Hq, D, device="cuda")[:, 0].to(BF)
    out = cache.decode_rows(0, [0, 1, 2], q)
    torch.cuda.synchronize()
    for r, n in enumerate(lens):
        ref = OA.decode_reference(f64(q[r:r + 1]), f64(K[r:r + 1, :n]), f64(V[r:r + 1, :n]),
                                  mask.numpy(), S, R)
        assert_parity(out[r:r + 1], ref, "bf16", "row %d (%d tokens)" % (r, n))
    assert duo_poll_device_error() == 0


def test_packed_sequence_shards():
    """Two shards of an 80000-token sequence: each decodes its retrieval range
    as partials, the streaming heads (packed) on the first shard only; the
    merged output equals the oracle over the whole sequence."""
    Hq, Hkv, S, R, n = 32, 8, 4, 60, 80000
    mask = _mask(Hkv, (0, 4))
    K, V = _seq(71, 1, n, Hkv), _seq(72, 1, n, Hkv)
    caches = []
    for lo, hi in shard.shard_ranges(n, 2):
        c = DuoCache(1, 1, Hq, Hkv, D, "bf16", max(1, min(hi, n) - lo), mask[None], S, R)
        c.set_retrieval_shard(lo, hi)
        for p0 in range(0, n, 8192):
            c.append(0, K[:, p0:p0 + 8192].contiguous(), V[:, p0:p0 + 8192].contiguous())
        caches.append(c)
    assert all(c.decode_streaming_pack(0) > 1 for c in caches)
    q = synth.kv_field(73, [0], [0], Hq, D, device="cuda")[:, 0].to(BF)
    parts = [c.decode_partial(0, q, owns_streaming=shard.owns_streaming(i))
             for i, c in enumerate(caches)]
    o = torch.stack([p[0] for p in parts]).contiguous()
    lse = torch.stack([p[1] for p in parts]).contiguous()
    out = merge_partials(o, lse, torch.empty(q.shape, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    ref = OA.decode_reference(f64(q), f64(K), f64(V), mask.numpy(), S, R)
    assert_parity(out, ref, "bf16", "merged shards")
    assert duo_poll_device_error() == 0


def test_packed_int4_decode_and_step():
    """4-bit cache: three streaming heads packed into one CTA of four warp
    groups (one group idle), each group with its own query fragments in
    shared memory.  A decode and two fused steps against the oracle fed the
    identically dequantised K/V (float32 outputs), then every code and
    (scale, zero) pair in the cache, the new tokens' ring slots included."""
    from test_int4_gpu import _check_cache_bytes as check_int4_bytes
    from test_int4_gpu import _dequant_history, _inputs
    B_, Hq, Hkv, S, R, n0, steps = 1, 24, 6, 4, 60, 52000, 2
    n = n0 + steps
    mask = _mask(Hkv, (0, 2, 4))
    K, V, _ = _inputs(91, B_, n, Hq, Hkv, D)
    Q = synth.kv_field(915, range(B_), range(n0 - 1, n), Hq, D, device="cuda").to(BF)
    cache = DuoCache(1, B_, Hq, Hkv, D, "int4", n, mask[None], S, R)
    cache.set_decode_output(torch.float32)
    for p0 in range(0, n0, 8192):
        p1 = min(n0, p0 + 8192)
        cache.append(0, K[:, p0:p1].contiguous(), V[:, p0:p1].contiguous())
    assert cache.decode_streaming_pack(0) > 1
    Kh, Kc, Ks, Kz = _dequant_history(K)
    Vh, Vc, Vs, Vz = _dequant_history(V)
    out = cache.decode(0, Q[:, 0].contiguous())
    torch.cuda.synchronize()
    ref = OA.decode_reference(f64(Q[:, 0]), Kh[:, :n0], Vh[:, :n0], mask.numpy(), S, R)
    assert_parity(out, ref, "int4", "packed 4-bit decode")
    for i in range(steps):
        t = n0 + i
        q = Q[:, i + 1].contiguous()
        out = cache.step(0, q, K[:, t].contiguous(), V[:, t].contiguous())
        torch.cuda.synchronize()
        ref = OA.decode_reference(f64(q), Kh[:, :t + 1], Vh[:, :t + 1], mask.numpy(), S, R)
        assert_parity(out, ref, "int4", "packed 4-bit step at %d" % t)
    check_int4_bytes(cache, Kc, Ks, Kz, Vc, Vs, Vz, mask, B_, n, Hkv, S, R)
    assert duo_poll_device_error() == 0


def test_packed_paged_rows_and_steps():
    """Paged layout: four rows of 40000, 25000, 9000 and 500 tokens in one
    launch with the streaming heads packed; decode_rows, then two fused steps
    on every row (each at its own position), against the oracle per row."""
    Hq, Hkv, S, R = 32, 8, 4, 60
    mask = _mask(Hkv, (1, 6))
    lens = [40000, 25000, 9000, 500]
    steps = 2
    blocks = sum((n + steps + 255) // 256 for n in lens) + 8
    cache = DuoCache(1, 4, Hq, Hkv, D, "bf16", max(lens) + steps, mask[None], S, R, pool_blocks=blocks)
    top = max(lens) + steps
    K, V = _seq(81, 4, top, Hkv), _seq(82, 4, top, Hkv)
    Q = _seq(83, 4, top, Hq)
    for r, n in enumerate(lens):
        for p0 in range(0, n, 8192):
            p1 = min(n, p0 + 8192)
            cache.append_rows(0, [r], K[r:r + 1, p0:p1].contiguous(), V[r:r + 1, p0:p1].contiguous())
    assert cache.decode_streaming_pack(0) > 1
    rows = [2, 0, 3, 1]  # listed out of order
    q = torch.cat([Q[r:r + 1, lens[r] - 1] for r in rows]).contiguous()
    out = cache.decode_rows(0, rows, q)
    torch.cuda.synchronize()
    for i, r in enumerate(rows):
        n = lens[r]
        ref = OA.decode_reference(f64(q[i:i + 1]), f64(K[r:r + 1, :n]), f64(V[r:r + 1, :n]),
                                  mask.numpy(), S, R)
        assert_parity(out[i:i + 1], ref, "bf16", "paged row %d (%d tokens)" % (r, n))
    rows = [0, 1, 2, 3]
    for s_ in range(steps):
        pos = [lens[r] + s_ for r in rows]
        q = torch.cat([Q[r:r + 1, pos[r]] for r in rows]).contiguous()
        kn = torch.cat([K[r:r + 1, pos[r]] for r in rows]).contiguous()
        vn = torch.cat([V[r:r + 1, pos[r]] for r in rows]).contiguous()
        out = cache.step_rows(0, rows, q, kn, vn)
        torch.cuda.synchronize()
        for r in rows:
            t = pos[r] + 1
            ref = OA.decode_reference(f64(q[r:r + 1]), f64(K[r:r + 1, :t]), f64(V[r:r + 1, :t]),
                                      mask.numpy(), S, R)
            assert_parity(out[r:r + 1], ref, "bf16", "paged step %d row %d" % (s_, r))
    assert duo_poll_device_error() == 0
