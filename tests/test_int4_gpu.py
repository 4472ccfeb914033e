"""INT4 KV cache: quantise-on-append bit for bit, and decode against an oracle
fed the identically dequantised K/V: max |err| <= 2e-2 on float32 outputs, and
on the default bf16 outputs 2e-2 plus half an ulp of bf16 at the element."""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache as OC
from oracle import int4 as OQ
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache

from _util import assert_parity, f64, seeded_mask

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


def _inputs(seed, B, n, Hq, Hkv, D, outliers=True):
    K = synth.kv_field(seed * 10 + 1, range(B), range(n), Hkv, D, device="cuda")
    V = synth.kv_field(seed * 10 + 2, range(B), range(n), Hkv, D, device="cuda")
    if outliers:  # a few channels x10, fixed across tokens (as in the 1M-context workload)
        ch = synth.outlier_channels(seed, D, 0.02).cuda()
        K[..., ch] *= 10.0
        V[..., ch] *= 10.0
    q = synth.kv_field(seed * 10 + 3, range(B), [n - 1], Hq, D, device="cuda")[:, 0]
    return K.to(BF), V.to(BF), q.to(BF)


def _dequant_history(X):
    """Oracle side: fp32 mirror of the encoder on the exact bf16 inputs, then
    the exact dequantisation.  Returns (x_hat float64, codes, sc, zp)."""
    x = X.detach().cpu().float().numpy()
    codes, sc, zp = OQ.quantize_int4(x)
    return OQ.dequantize_int4(codes, sc, zp), codes, sc, zp


def _fill(cache, K, V, chunks):
    n = K.shape[1]
    pos = 0
    sizes = list(chunks)
    while pos < n - 1:
        c = min(sizes.pop(0) if sizes else n - 1 - pos, n - 1 - pos)
        cache.append(0, K[:, pos:pos + c].contiguous(), V[:, pos:pos + c].contiguous())
        pos += c
    cache.append(0, K[:, n - 1:].contiguous(), V[:, n - 1:].contiguous())


def _check_cache_bytes(cache, Kc, Ks, Kz, Vc, Vs, Vz, mask, B, n, Hkv, S, R):
    """Packed codes and (scale, zero) pairs of layer 0, bit for bit against the
    oracle's encoder and its ring model."""
    lv = cache.layout(0)
    for name, codes, sc, zp in (("k", Kc, Ks, Kz), ("v", Vc, Vs, Vz)):
        packed = OQ.pack_nibbles(codes)                                  # [B, n, Hkv, D/2]
        szb = np.stack([sc, zp], axis=-1).view(np.uint8).reshape(B, n, Hkv, 4)
        ret = cache.region(0, "ret_" + name)
        ret_sz = cache.region(0, "ret_%s_sz" % name)
        st = cache.region(0, "str_" + name)
        st_sz = cache.region(0, "str_%s_sz" % name)
        for h in range(Hkv):
            idx = lv.packed_index[h]
            for b in range(B):
                if mask[h]:
                    np.testing.assert_array_equal(ret[b, idx, :n].cpu().numpy(), packed[b, :, h])
                    np.testing.assert_array_equal(ret_sz[b, idx, :n].cpu().numpy(), szb[b, :, h])
                else:
                    exp, filled = OC.expected_streaming_buffer(packed[b, :, h], S, R)
                    np.testing.assert_array_equal(st[b, idx, :S + R].cpu().numpy()[filled], exp[filled])
                    exp, filled = OC.expected_streaming_buffer(szb[b, :, h], S, R)
                    np.testing.assert_array_equal(st_sz[b, idx, :S + R].cpu().numpy()[filled], exp[filled])


@pytest.mark.parametrize("B,Hq,Hkv,D", [(1, 8, 2, 128), (2, 4, 4, 64), (1, 8, 8, 128)])
@pytest.mark.parametrize("n", [1, 3, 70, 333, 2049])
def test_int4_append_bit_exact_and_decode(B, Hq, Hkv, D, n, S=4, R=64):
    seed = n + D + Hkv
    K, V, q = _inputs(seed, B, n, Hq, Hkv, D)
    mask = seeded_mask(seed, Hkv, max(1, Hkv // 2))
    cache = DuoCache(1, B, Hq, Hkv, D, "int4", n, mask[None], S, R)
    _fill(cache, K, V, [2, 31, 500])
    out_bf16 = cache.decode(0, q)
    cache.set_decode_output(torch.float32)
    out = cache.decode(0, q)
    torch.cuda.synchronize()

    Kh, Kc, Ks, Kz = _dequant_history(K)
    Vh, Vc, Vs, Vz = _dequant_history(V)
    ref = OA.decode_reference(f64(q), Kh, Vh, mask.numpy(), S, R)
    assert_parity(out, ref, "int4", "int4 decode n=%d (fp32 output)" % n)
    assert_parity(out_bf16, ref, "int4_bf16", "int4 decode n=%d (bf16 output)" % n)

    _check_cache_bytes(cache, Kc, Ks, Kz, Vc, Vs, Vz, mask, B, n, Hkv, S, R)
    kept, full = cache.kv_bytes()
    assert (kept, full) == OC.kv_bytes(mask[None].numpy(), B, n, S, R, D, "int4")


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("S,R", [(0, 1), (5, 1), (0, 7), (600, 700)])
def test_int4_degenerate_windows(D, S, R):
    """4-bit cache with the degenerate windows (slot buffers padded to a
    multiple of 4 rows when S + R is not): codes, scale/zero and decode."""
    test_int4_append_bit_exact_and_decode(2, 8, 4, D, 333, S=S, R=R)


def test_int4_split_counts_agree():
    B, Hq, Hkv, D, n, S, R = 1, 8, 2, 128, 20000, 64, 256
    K, V, q = _inputs(7, B, n, Hq, Hkv, D)
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, D, "int4", n, mask[None], S, R)
    _fill(cache, K, V, [8192, 8192])
    Kh = _dequant_history(K)[0]
    Vh = _dequant_history(V)[0]
    ref = OA.decode_reference(f64(q), Kh, Vh, mask.numpy(), S, R)
    cache.set_decode_output(torch.float32)
    for splits in (1, 3, 64, 0):
        cache.set_decode_splits(splits)
        assert_parity(cache.decode(0, q), ref, "int4", "splits=%d" % splits)


def test_int4_constant_rows_and_prefill_limits():
    """A (token, head) row of identical values has scale 0: codes 0, x_hat = zp.
    Pre-fill on a 4-bit cache needs room for the chunk and head_dim 128."""
    from head_split_kv_decode_b200.binding import DuoError
    B, Hq, Hkv, D, n = 1, 2, 2, 128, 40
    K = torch.full((B, n, Hkv, D), 0.75, dtype=BF, device="cuda")
    V = synth.kv_field(3, range(B), range(n), Hkv, D, device="cuda").to(BF)
    q = synth.kv_field(4, range(B), [n - 1], Hq, D, device="cuda")[:, 0].to(BF)
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, D, "int4", n, mask[None], 2, 8)
    cache.append(0, K, V)
    cache.set_decode_output(torch.float32)
    out = cache.decode(0, q)
    Kh = _dequant_history(K)[0]
    assert (Kh == 0.75).all()
    ref = OA.decode_reference(f64(q), Kh, _dequant_history(V)[0], mask.numpy(), 2, 8)
    assert_parity(out, ref, "int4", "constant rows")
    cap = cache.layout(0).capacity  # 4-bit caches round capacity up to one 128-key tile
    assert cap == 128
    zeros = torch.zeros(B, cap - n, Hkv, D, dtype=BF, device="cuda")
    cache.append(0, zeros, zeros)
    with pytest.raises(DuoError) as e:  # the cache is full
        cache.prefill(0, torch.zeros(B, 8, Hq, D, dtype=BF, device="cuda"),
                      torch.zeros(B, 8, Hkv, D, dtype=BF, device="cuda"),
                      torch.zeros(B, 8, Hkv, D, dtype=BF, device="cuda"))
    assert e.value.name == "DUO_ERR_CAPACITY"
    c64 = DuoCache(1, B, Hq, Hkv, 64, "int4", 64, mask[None], 2, 8)
    with pytest.raises(DuoError) as e:
        c64.prefill(0, torch.zeros(B, 8, Hq, 64, dtype=BF, device="cuda"),
                    torch.zeros(B, 8, Hkv, 64, dtype=BF, device="cuda"),
                    torch.zeros(B, 8, Hkv, 64, dtype=BF, device="cuda"))
    assert e.value.name == "DUO_ERR_UNSUPPORTED"


@pytest.mark.parametrize("B,Hq,Hkv,n0,S,R", [(2, 8, 2, 3000, 4, 64), (1, 8, 8, 40, 2, 8),
                                             (1, 32, 8, 20000, 64, 256)])
def test_int4_fused_step(B, Hq, Hkv, n0, S, R, steps=5):
    """duo_decode_step on a 4-bit cache: the decode launch quantises the new
    token itself.  Every step's output against the oracle (float32 output,
    absolute 2e-2), then every code and (scale, zero) in the cache bit for bit,
    including ring slots that wrapped during the steps and split heads."""
    D = 128
    seed = n0 + Hkv
    n = n0 + steps
    K, V, _ = _inputs(seed, B, n, Hq, Hkv, D)
    Q = synth.kv_field(seed * 10 + 5, range(B), range(n), Hq, D, device="cuda").to(BF)
    mask = seeded_mask(seed, Hkv, max(1, Hkv // 2))
    cache = DuoCache(1, B, Hq, Hkv, D, "int4", n, mask[None], S, R)
    cache.set_decode_output(torch.float32)
    cache.append(0, K[:, :n0].contiguous(), V[:, :n0].contiguous())
    Kh, Kc, Ks, Kz = _dequant_history(K)
    Vh, Vc, Vs, Vz = _dequant_history(V)
    for t in range(n0, n):
        q = Q[:, t].contiguous()
        out = cache.step(0, q, K[:, t].contiguous(), V[:, t].contiguous())
        torch.cuda.synchronize()
        ref = OA.decode_reference(f64(q), Kh[:, :t + 1], Vh[:, :t + 1], mask.numpy(), S, R)
        assert_parity(out, ref, "int4", "fused int4 step at %d" % t)
    assert cache.seq_len(0) == n
    _check_cache_bytes(cache, Kc, Ks, Kz, Vc, Vs, Vz, mask, B, n, Hkv, S, R)
    from head_split_kv_decode_b200.binding import duo_poll_device_error
    assert duo_poll_device_error() == 0


@pytest.mark.parametrize("fused", [False, True])
def test_int4_extreme_value_ranges(fused):
    """Value ranges far outside the workloads': tokens whose V rows are scaled
    by 3e3 (fp16 scale ~1e3, so p*scale passes f16's 65504 unless the kernel's
    power-of-two headroom shrinks; the zero point, ~-1e4, still fits fp16),
    tokens scaled by 1e-6 (tiny scales), and a query channel of 1e5 (beyond
    f16's range before the kernel's power-of-two prescale).  The output must
    stay finite and match the oracle to a bound relative to the largest
    |value| (the absolute 2e-2 is the bar for the workloads' ranges, where |O|
    stays below ~50)."""
    B, Hq, Hkv, D, n, S, R = 1, 8, 2, 128, 600, 4, 64
    K, V, _ = _inputs(77, B, n, Hq, Hkv, D, outliers=False)
    V = V.float()
    V[:, 100:110] *= 3e3
    V[:, 200:300] *= 1e-6
    V[:, n - 3:] *= 3e3  # big rows inside every streaming window too
    V = V.to(BF)
    q = synth.kv_field(78, range(B), [n - 1], Hq, D, device="cuda")[:, 0]
    q[:, 1, 5] = 1e5
    q[:, 6, 17] = -7e4
    q = q.to(BF)
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, B, Hq, Hkv, D, "int4", n, mask[None], S, R)
    cache.set_decode_output(torch.float32)
    if fused:
        cache.append(0, K[:, :n - 1].contiguous(), V[:, :n - 1].contiguous())
        out = cache.step(0, q, K[:, n - 1].contiguous(), V[:, n - 1].contiguous())
    else:
        cache.append(0, K.contiguous(), V.contiguous())
        out = cache.decode(0, q)
    torch.cuda.synchronize()
    Kh, Vh = _dequant_history(K)[0], _dequant_history(V)[0]
    ref = OA.decode_reference(f64(q), Kh, Vh, mask.numpy(), S, R)
    got = f64(out)
    assert np.isfinite(ref).all()  # the inputs stay inside what fp16 scale/zero can hold
    assert np.isfinite(got).all()
    bound = 2e-2 + 1e-5 * np.abs(Vh).max()
    err = np.abs(got - ref).max()
    assert err <= bound, "max |err| %.3g > %.3g" % (err, bound)
