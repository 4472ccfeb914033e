"""The allocation-free decode entry point (duo_decode_attn_static).

Some callers cannot allocate device memory for a workspace: a serving loop
that must never stall on cudaMalloc/cudaFree (both can synchronise the
device), or a host program whose memory belongs to an allocator it cannot call.
For them the library decodes with a fixed scratch array of its own.  This file
checks, through the C ABI, that two calls in a row give the same result as the
workspace-taking entry point, and that a layer needing more scratch than the
array holds is refused before anything runs.  It is collected last so that a
failure here cannot hide another test's result; it passes alone or after the
rest of the suite.
"""

import pytest
import torch

from head_split_kv_decode_b200 import binding as B
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


def _cache(batch, n, seed):
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, batch, 8, 2, 128, "bf16", n + 4, mask[None], 64, 256)
    K = synth.kv_field(seed + 1, range(batch), range(n + 2), 2, 128, device="cuda").to(BF)
    V = synth.kv_field(seed + 2, range(batch), range(n + 2), 2, 128, device="cuda").to(BF)
    Q = synth.kv_field(seed + 3, range(batch), range(n + 2), 8, 128, device="cuda").to(BF)
    cache.append(0, K[:, :n].contiguous(), V[:, :n].contiguous())
    return cache, K, V, Q


def test_static_decode_matches_workspace_decode_twice():
    batch, n = 2, 20000
    cache, K, V, Q = _cache(batch, n, 500)
    assert cache.decode_splits(0) > 1  # the scratch is really used
    for step in range(2):  # two calls in a row, each after one more append
        t = n + step
        cache.append(0, K[:, t:t + 1].contiguous(), V[:, t:t + 1].contiguous())
        q = Q[:, t].contiguous()
        ref = torch.empty_like(q)
        got = torch.full_like(q, float("nan"))
        B.duo_decode_attn(cache.handle, 0, q.data_ptr(), ref.data_ptr(), 0.0,
                          cache.ws_ptr, cache.ws_bytes)
        B.duo_decode_attn_static(cache.handle, 0, q.data_ptr(), got.data_ptr(), 0.0)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3, (step, err.max().item())
    assert B.duo_poll_device_error() == 0


def test_static_decode_refuses_oversized_layer():
    # 16 batch rows x 1 retrieval head x 313 splits x G=4 x 129 floats x 4 B
    # = 10.3 MB > 8 MiB (80000 keys in at most 512 splits rounded up to whole
    # tiles of 128 or 256 keys: 313 splits of 256)
    batch, n = 16, 80000
    cache, K, V, Q = _cache(batch, n, 900)
    cache.set_decode_splits(512)
    q = Q[:, n - 1].contiguous()
    out = torch.zeros_like(q)
    with pytest.raises(B.DuoError) as e:
        B.duo_decode_attn_static(cache.handle, 0, q.data_ptr(), out.data_ptr(), 0.0)
    assert e.value.name == "DUO_ERR_WORKSPACE"
    torch.cuda.synchronize()
    assert out.abs().max().item() == 0.0  # nothing was launched
