"""The allocation-free decode entry point (duo_decode_attn_static).

Some callers cannot allocate device memory for a workspace: a serving loop
that must never stall on cudaMalloc/cudaFree (both can synchronise the
device), or a host program whose memory belongs to an allocator it cannot call.
For them the library decodes with a fixed scratch array of its own.  This file
checks, through the C ABI, that two calls in a row give the same result as the
workspace-taking entry point and as the fp64 oracle, on the tensor-core decode
(bf16 and 4-bit caches, head_dim 128) and on the CUDA-core decode (fp32,
head_dim 64), bit for bit with the workspace call when splits are
reproducible; and that a layer needing more scratch than the array holds is
refused before anything runs.  It is collected last so that a failure here
cannot hide another test's result; it passes alone or after the rest of the
suite.
"""

import numpy as np
import pytest
import torch

from head_split_kv_decode_b200 import binding as B
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache
from oracle import attention as OA
from oracle import int4 as OQ

from _util import assert_parity, f64

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
S_, R_ = 64, 256


def _cache(batch, n, seed, kv="bf16", D=128, Hq=8, Hkv=2):
    mask = torch.tensor([1, 0] * (Hkv // 2), dtype=torch.uint8)
    cache = DuoCache(1, batch, Hq, Hkv, D, kv, n + 4, mask[None], S_, R_)
    dt = torch.float32 if kv == "f32" else BF
    K = synth.kv_field(seed + 1, range(batch), range(n + 2), Hkv, D, device="cuda").to(dt)
    V = synth.kv_field(seed + 2, range(batch), range(n + 2), Hkv, D, device="cuda").to(dt)
    Q = synth.kv_field(seed + 3, range(batch), range(n + 2), Hq, D, device="cuda").to(dt)
    cache.append(0, K[:, :n].contiguous(), V[:, :n].contiguous())
    return cache, mask, K, V, Q


def _two_calls(cache, mask, K, V, Q, n, kind, dequant=None, exact=False):
    """Two decode steps in a row; at each, the static call against the
    workspace call and against the oracle."""
    for step in range(2):
        t = n + step
        cache.append(0, K[:, t:t + 1].contiguous(), V[:, t:t + 1].contiguous())
        q = Q[:, t].contiguous()
        ref = torch.empty(q.shape, dtype=cache.out_dtype, device=q.device)
        got = torch.full(q.shape, float("nan"), dtype=cache.out_dtype, device=q.device)
        B.duo_decode_attn(cache.handle, 0, q.data_ptr(), ref.data_ptr(), 0.0,
                          cache.ws_ptr, cache.ws_bytes)
        B.duo_decode_attn_static(cache.handle, 0, q.data_ptr(), got.data_ptr(), 0.0)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        if exact:
            assert torch.equal(got, ref), "step %d: static and workspace calls differ" % step
        else:
            assert_parity(got, f64(ref), "bf16" if kind != "f32" else "f32", "static vs workspace")
        kh, vh = K[:, :t + 1], V[:, :t + 1]
        if dequant is not None:
            kh, vh = dequant(kh), dequant(vh)
        else:
            kh, vh = f64(kh), f64(vh)
        oracle = OA.decode_reference(f64(q), kh, vh, mask.numpy(), S_, R_)
        assert_parity(got, oracle, kind, "static vs oracle, step %d" % step)
    assert B.duo_poll_device_error() == 0


def test_static_decode_matches_workspace_decode_twice():
    batch, n = 2, 20000
    cache, mask, K, V, Q = _cache(batch, n, 500)
    assert cache.decode_splits(0) > 1  # the scratch is really used
    _two_calls(cache, mask, K, V, Q, n, "bf16")


def test_static_decode_bit_equal_when_reproducible():
    batch, n = 2, 20000
    cache, mask, K, V, Q = _cache(batch, n, 520)
    cache.set_decode_reproducible(True)
    assert cache.decode_splits(0) > 1
    _two_calls(cache, mask, K, V, Q, n, "bf16", exact=True)


def test_static_decode_cuda_core_f32_d64():
    """fp32 cache, head_dim 64: the CUDA-core decode and its own scratch
    layout, with a forced split count so that the partials are merged."""
    batch, n = 1, 5000
    cache, mask, K, V, Q = _cache(batch, n, 540, kv="f32", D=64)
    cache.set_decode_splits(7)
    assert cache.decode_splits(0) > 1
    _two_calls(cache, mask, K, V, Q, n, "f32")


def test_static_decode_int4_cache():
    batch, n = 1, 12000
    cache, mask, K, V, Q = _cache(batch, n, 560, kv="int4")
    cache.set_decode_output(torch.float32)  # the 4-bit bound is absolute
    assert cache.decode_splits(0) > 1

    def dequant(x):
        return OQ.dequantize_int4(*OQ.quantize_int4(x.detach().cpu().float().numpy()))

    _two_calls(cache, mask, K, V, Q, n, "int4", dequant=dequant)


def test_static_decode_refuses_oversized_layer():
    # 16 batch rows x 1 retrieval head x 313 splits x G=4 x 129 floats x 4 B
    # = 10.3 MB > 8 MiB (80000 keys in at most 512 splits rounded up to whole
    # tiles of 128 or 256 keys: 313 splits of 256)
    batch, n = 16, 80000
    cache, mask, K, V, Q = _cache(batch, n, 900)
    cache.set_decode_splits(512)
    q = Q[:, n - 1].contiguous()
    out = torch.zeros_like(q)
    with pytest.raises(B.DuoError) as e:
        B.duo_decode_attn_static(cache.handle, 0, q.data_ptr(), out.data_ptr(), 0.0)
    assert e.value.name == "DUO_ERR_WORKSPACE"
    torch.cuda.synchronize()
    assert out.abs().max().item() == 0.0  # nothing was launched
