"""Sequence-sharded decode, emulated on one GPU: several caches each keep a
contiguous range of the retrieval positions (as one GPU each would), all keep
the streaming state; their decode partials, merged, must equal the oracle's
attention over the whole sequence (and the unsharded cache's decode).  The
exchange between GPUs is an all-gather of the partials (tests of its host side
run on CPU); here the partials are stacked on the one device.
"""

import pytest
import torch

from oracle import attention as OA
from oracle import int4 as OQ
from head_split_kv_decode_b200 import binding as B
from head_split_kv_decode_b200 import shard, synth
from head_split_kv_decode_b200.cache import DuoCache, merge_partials

from _util import assert_parity, f64

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
D = 128


def _seq(seed, B_, n, heads):
    return synth.kv_field(seed, range(B_), range(n), heads, D, device="cuda").to(BF)


def _merged(caches, q, layer=0, out_dtype=BF):
    parts = [c.decode_partial(layer, q, owns_streaming=shard.owns_streaming(i))
             for i, c in enumerate(caches)]
    o = torch.stack([p[0] for p in parts]).contiguous()
    lse = torch.stack([p[1] for p in parts]).contiguous()
    return merge_partials(o, lse, torch.empty(q.shape, dtype=out_dtype, device="cuda")), parts


@pytest.mark.parametrize("world,paged", [(3, False), (2, True), (4, False)])
def test_sharded_decode_matches_whole_sequence(world, paged):
    B_, Hq, Hkv, S, R = 2, 8, 2, 16, 64
    n0, steps, cap = 5000, 4, 5200
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    K, V = _seq(11, B_, n0 + steps, Hkv), _seq(12, B_, n0 + steps, Hkv)
    Q = _seq(13, B_, n0 + steps, Hq)
    ranges = shard.shard_ranges(cap, world) if world < 4 else [(0, 2000), (2000, 4000),
                                                               (4000, 6000), (6000, 1 << 62)]
    caches = []
    for lo, hi in ranges:
        held = min(hi, cap) - lo
        kw = dict(pool_blocks=B_ * (held // 256 + 2)) if paged else {}
        c = DuoCache(1, B_, Hq, Hkv, D, "bf16", max(held, 1), mask[None], S, R, **kw)
        c.set_retrieval_shard(lo, hi)
        caches.append(c)
    whole = DuoCache(1, B_, Hq, Hkv, D, "bf16", cap, mask[None], S, R)
    for p0 in range(0, n0, 1500):  # every cache gets every token
        k = K[:, p0:min(n0, p0 + 1500)].contiguous()
        v = V[:, p0:min(n0, p0 + 1500)].contiguous()
        for c in caches + [whole]:
            c.append(0, k, v)
    if world == 4:  # the last shard holds no retrieval token yet: streaming bytes only
        assert caches[3].kv_bytes()[0] == B_ * 1 * min(n0, S + R) * 4 * D
    for step in range(steps):
        t = n0 + step
        if step:
            for c in caches + [whole]:
                c.append(0, K[:, t - 1:t].contiguous(), V[:, t - 1:t].contiguous())
        q = Q[:, t - 1].contiguous()
        got, parts = _merged(caches, q)
        ref = OA.decode_reference(f64(q), f64(K[:, :t]), f64(V[:, :t]), mask.numpy(), S, R)
        assert_parity(got, ref, "bf16", "world %d step %d" % (world, step))
        assert (got.float() - whole.decode(0, q).float()).abs().max().item() <= 2e-2
        if world == 4:  # an empty shard leaves -inf and zeros
            assert torch.all(parts[3][1][:, :4] == -float("inf"))  # retrieval heads' rows
    assert B.duo_poll_device_error() == 0


def test_sharded_int4_decode():
    B_, Hq, Hkv, S, R, n = 1, 8, 2, 8, 64, 3000
    mask = torch.tensor([0, 1], dtype=torch.uint8)
    K, V, Q = _seq(21, B_, n, Hkv), _seq(22, B_, n, Hkv), _seq(23, B_, n, Hq)
    caches = []
    for lo, hi in shard.shard_ranges(n, 2):
        c = DuoCache(1, B_, Hq, Hkv, D, "int4", min(hi, n) - lo, mask[None], S, R)
        c.set_retrieval_shard(lo, hi)
        c.append(0, K.contiguous(), V.contiguous())
        caches.append(c)
    q = Q[:, n - 1].contiguous()
    got, _ = _merged(caches, q, out_dtype=torch.float32)
    kd = OQ.dequantize_int4(*OQ.quantize_int4(K.float().cpu().numpy()))
    vd = OQ.dequantize_int4(*OQ.quantize_int4(V.float().cpu().numpy()))
    ref = OA.decode_reference(f64(q), kd, vd, mask.numpy(), S, R)
    assert_parity(got, ref, "int4", "int4 shards")


def test_shard_rules():
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    c = DuoCache(1, 1, 8, 2, D, "bf16", 512, mask[None], 4, 16)
    with pytest.raises(B.DuoError) as e:
        c.set_retrieval_shard(10, 10)
    assert e.value.name == "DUO_ERR_ARG"
    c.set_retrieval_shard(256, 768)
    K = _seq(5, 1, 300, 2)
    c.append(0, K, K)
    with pytest.raises(B.DuoError) as e:  # tokens present
        c.set_retrieval_shard(0, 512)
    assert e.value.name == "DUO_ERR_STATE"
    q = _seq(6, 1, 1, 8)[:, 0].contiguous()
    with pytest.raises(B.DuoError) as e:  # a shard only decodes as a partial
        c.decode(0, q)
    assert e.value.name == "DUO_ERR_UNSUPPORTED"
    with pytest.raises(B.DuoError) as e:
        c.prefill(0, _seq(7, 1, 128, 8), _seq(8, 1, 128, 2), _seq(9, 1, 128, 2))
    assert e.value.name == "DUO_ERR_UNSUPPORTED"
    f = DuoCache(1, 1, 4, 2, 64, "f32", 64, mask[None], 4, 16)
    with pytest.raises(B.DuoError) as e:
        f.set_retrieval_shard(0, 32)
    assert e.value.name == "DUO_ERR_UNSUPPORTED"
