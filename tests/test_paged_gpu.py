"""Sequences of different lengths in one cache: per-row appends, decode and
pre-fill through the *_rows calls, on the paged layout (retrieval K/V in a
shared pool of 256-token blocks found through per-row block tables) and on the
packed layout.  Every result is checked against the fp64 oracle run on that
row's own history; cache bytes are checked bit for bit through the block
table.  Rows are filled in interleaved chunks so that their blocks interleave
in the pool, and a released row is refilled with a new sequence.
"""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache as OC
from oracle import int4 as OQ
from head_split_kv_decode_b200 import binding as B
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache

from _util import assert_parity, f64, seeded_mask

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
D, HQ, HKV = 128, 8, 2


def _seq(seed, n, heads, dtype=BF):
    """One sequence's K (or V, Q) rows [1, n, heads, D] on the device."""
    return synth.kv_field(seed, [0], range(n), heads, D, device="cuda").to(dtype)


class Rows:
    """The host-side truth of each row: its K, V history and query source."""

    def __init__(self, n_rows, max_len, seed):
        self.K = [None] * n_rows
        self.V = [None] * n_rows
        self.Q = [None] * n_rows
        self.len = [0] * n_rows
        self.max_len = max_len
        self.seed = seed

    def start(self, r, seq_id):
        s = self.seed * 100 + seq_id * 3
        self.K[r] = _seq(s + 1, self.max_len, HKV)
        self.V[r] = _seq(s + 2, self.max_len, HKV)
        self.Q[r] = _seq(s + 3, self.max_len, HQ)
        self.len[r] = 0


def _append(cache, rows_state, rows, n_tok):
    k = torch.cat([rows_state.K[r][:, rows_state.len[r]:rows_state.len[r] + n_tok] for r in rows])
    v = torch.cat([rows_state.V[r][:, rows_state.len[r]:rows_state.len[r] + n_tok] for r in rows])
    cache.append_rows(0, rows, k.contiguous(), v.contiguous())
    for r in rows:
        rows_state.len[r] += n_tok


def _oracle_decode(st, r, mask, S, R):
    n = st.len[r]
    q = st.Q[r][:, n - 1]
    return OA.decode_reference(f64(q), f64(st.K[r][:, :n]), f64(st.V[r][:, :n]), mask.numpy(), S, R)


def _check_bytes(cache, st, rows, mask, S, R):
    torch.cuda.synchronize()
    lv = cache.layout(0)
    for r in rows:
        n = st.len[r]
        assert cache.row_seq_len(0, r) == n
        Kc = st.K[r][0, :n].cpu().contiguous().view(torch.uint8).view(n, HKV, -1)
        Vc = st.V[r][0, :n].cpu().contiguous().view(torch.uint8).view(n, HKV, -1)
        for h in range(HKV):
            idx = lv.packed_index[h]
            if mask[h]:
                got_k = cache.gather_rows(0, "ret_k", r, n)[idx].cpu()
                got_v = cache.gather_rows(0, "ret_v", r, n)[idx].cpu()
                assert torch.equal(got_k, Kc[:, h]) and torch.equal(got_v, Vc[:, h])
            else:
                for src, name in ((Kc, "str_k"), (Vc, "str_v")):
                    exp, filled = OC.expected_streaming_buffer(src[:, h].numpy(), S, R)
                    got = cache.region(0, name)[r, idx].cpu().numpy()
                    np.testing.assert_array_equal(got[filled], exp[filled])


@pytest.mark.parametrize("paged", [True, False])
def test_rows_of_different_lengths(paged):
    S, R = 16, 96
    n_rows, max_len = 4, 3200
    mask = seeded_mask(31, HKV, 1)
    kw = dict(pool_blocks=40) if paged else {}
    cache = DuoCache(1, n_rows, HQ, HKV, D, "bf16", max_len, mask[None], S, R, **kw)
    st = Rows(n_rows, max_len, seed=7)
    for r in range(n_rows):
        st.start(r, r)
    # interleaved chunks: rows grow at different rates, blocks interleave in the pool
    for rows, n_tok in [([0, 1, 2, 3], 37), ([3], 700), ([1, 3], 250), ([0], 300), ([3, 0], 1),
                        ([1], 513), ([3], 900), ([2], 3), ([0, 3], 256), ([1], 1)]:
        _append(cache, st, rows, n_tok)
    _check_bytes(cache, st, range(n_rows), mask, S, R)
    if paged:
        held = sum(len(cache.row_blocks(r)) for r in range(n_rows))
        assert held == sum((n + 255) // 256 for n in st.len)
        assert cache.pool_free_blocks() == 40 - held
        assert len({b for r in range(n_rows) for b in cache.row_blocks(r)}) == held

    # decode a subset of rows, listed out of order
    rows = [3, 0, 2]
    q = torch.cat([st.Q[r][:, st.len[r] - 1] for r in rows]).contiguous()
    out = cache.decode_rows(0, rows, q)
    for i, r in enumerate(rows):
        assert_parity(out[i:i + 1], _oracle_decode(st, r, mask, S, R), "bf16", "row %d" % r)

    # fused decode steps on every row (each at its own position)
    rows = [0, 1, 2, 3]
    for step in range(3):
        q = torch.cat([st.Q[r][:, st.len[r]] for r in rows]).contiguous()
        kn = torch.cat([st.K[r][:, st.len[r]] for r in rows]).contiguous()
        vn = torch.cat([st.V[r][:, st.len[r]] for r in rows]).contiguous()
        out = cache.step_rows(0, rows, q, kn, vn)
        for r in rows:
            st.len[r] += 1
        for i, r in enumerate(rows):
            assert_parity(out[i:i + 1], _oracle_decode(st, r, mask, S, R), "bf16",
                          "step %d row %d" % (step, r))
    _check_bytes(cache, st, rows, mask, S, R)

    # a finished sequence leaves; its row takes a new one
    free0 = cache.pool_free_blocks() if paged else 0
    held1 = len(cache.row_blocks(1)) if paged else 0
    cache.release_rows([1])
    assert cache.row_seq_len(0, 1) == 0
    if paged:
        assert cache.pool_free_blocks() == free0 + held1 and cache.row_blocks(1) == []
    st.start(1, 9)
    _append(cache, st, [1], 600)
    _append(cache, st, [1, 2], 44)
    _check_bytes(cache, st, range(n_rows), mask, S, R)
    q = torch.cat([st.Q[r][:, st.len[r] - 1] for r in range(n_rows)]).contiguous()
    out = cache.decode(0, q)  # every row, each at its own length
    for r in range(n_rows):
        assert_parity(out[r:r + 1], _oracle_decode(st, r, mask, S, R), "bf16", "after reuse %d" % r)

    # chunked pre-fill of two rows at their own positions, then the appends
    rows, C = [2, 1], 256
    q = torch.cat([st.Q[r][:, st.len[r]:st.len[r] + C] for r in rows]).contiguous()
    k = torch.cat([st.K[r][:, st.len[r]:st.len[r] + C] for r in rows]).contiguous()
    v = torch.cat([st.V[r][:, st.len[r]:st.len[r] + C] for r in rows]).contiguous()
    out = cache.prefill_rows(0, rows, q, k, v)
    sample = [0, 1, 5, 95, 96, 97, 128, 200, 255]
    for i, r in enumerate(rows):
        c0 = st.len[r]
        ref = OA.prefill_reference(f64(st.Q[r][:, c0:c0 + C]), f64(st.K[r][:, :c0 + C]),
                                   f64(st.V[r][:, :c0 + C]), c0, mask.numpy(), S, R, rows=sample)
        assert_parity(out[i:i + 1, sample].cpu(), ref, "bf16", "prefill row %d" % r)
    cache.append_rows(0, rows, k, v)
    for r in rows:
        st.len[r] += C
    _check_bytes(cache, st, range(n_rows), mask, S, R)
    assert B.duo_poll_device_error() == 0


def test_paged_pool_exhaustion_changes_nothing():
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, 2, HQ, HKV, D, "bf16", 4096, mask[None], 4, 16, pool_blocks=3)
    K = _seq(1, 1024, HKV)
    cache.append_rows(0, [0], K[:, :512].contiguous(), K[:, :512].contiguous())
    assert cache.pool_free_blocks() == 1
    with pytest.raises(B.DuoError) as e:  # needs 2 blocks for row 1, 1 is left
        cache.append_rows(0, [1, 0], torch.cat([K[:, :300], K[:, 512:812]]).contiguous(),
                          torch.cat([K[:, :300], K[:, 512:812]]).contiguous())
    assert e.value.name == "DUO_ERR_CAPACITY"
    assert cache.pool_free_blocks() == 1
    assert cache.row_seq_len(0, 0) == 512 and cache.row_seq_len(0, 1) == 0
    cache.append_rows(0, [1], K[:, :200].contiguous(), K[:, :200].contiguous())
    assert cache.pool_free_blocks() == 0
    cache.reset()
    assert cache.pool_free_blocks() == 3


def test_paged_int4_rows_decode():
    S, R = 8, 64
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    lens = [1500, 260, 777]
    cache = DuoCache(1, 3, HQ, HKV, D, "int4", 2048, mask[None], S, R, pool_blocks=16)
    hist = []
    for r, n in enumerate(lens):
        K, V = _seq(50 + 3 * r, n, HKV), _seq(51 + 3 * r, n, HKV)
        hist.append((K, V))
    # interleave: row 2 first half, row 0, row 1, row 2 rest
    cache.append_rows(0, [2], hist[2][0][:, :400].contiguous(), hist[2][1][:, :400].contiguous())
    cache.append_rows(0, [0], hist[0][0].contiguous(), hist[0][1].contiguous())
    cache.append_rows(0, [1], hist[1][0].contiguous(), hist[1][1].contiguous())
    cache.append_rows(0, [2], hist[2][0][:, 400:].contiguous(), hist[2][1][:, 400:].contiguous())
    rows = [1, 2, 0]
    q = torch.cat([_seq(60 + r, lens[r], HQ)[:, -1] for r in rows]).contiguous()
    cache.set_decode_output(torch.float32)
    out = cache.decode_rows(0, rows, q)
    assert out.dtype == torch.float32
    for i, r in enumerate(rows):
        K, V = hist[r]
        kd = OQ.dequantize_int4(*OQ.quantize_int4(K[0].float().cpu().numpy()))
        vd = OQ.dequantize_int4(*OQ.quantize_int4(V[0].float().cpu().numpy()))
        ref = OA.decode_reference(f64(q[i:i + 1]), kd[None], vd[None], mask.numpy(), S, R)
        assert_parity(out[i:i + 1], ref, "int4", "int4 paged row %d" % r)


def test_row_argument_errors():
    mask = torch.tensor([1, 0], dtype=torch.uint8)
    cache = DuoCache(1, 3, HQ, HKV, D, "bf16", 512, mask[None], 4, 16, pool_blocks=4)
    K = _seq(3, 64, HKV)
    k2 = torch.cat([K, K]).contiguous()
    for rows in ([0, 0], [3, 1], [-1, 0]):
        with pytest.raises(B.DuoError) as e:
            cache.append_rows(0, rows, k2, k2)
        assert e.value.name == "DUO_ERR_ARG"
    q = torch.zeros(1, HQ, D, dtype=BF, device="cuda")
    with pytest.raises(B.DuoError) as e:  # row 2 holds no token yet
        cache.decode_rows(0, [2], q)
    assert e.value.name == "DUO_ERR_STATE"
    # fp32 caches decode on CUDA cores: every row at one length only
    f = DuoCache(1, 2, 4, 2, 64, "f32", 64, mask[None], 4, 16)
    Kf = synth.kv_field(5, [0, 1], range(8), 2, 64, device="cuda")
    f.append_rows(0, [1], Kf[1:, :8].contiguous(), Kf[1:, :8].contiguous())
    with pytest.raises(B.DuoError) as e:
        f.decode(0, torch.zeros(2, 4, 64, device="cuda"))
    assert e.value.name == "DUO_ERR_STATE"  # row 0 is empty
    f.append_rows(0, [0], Kf[:1, :4].contiguous(), Kf[:1, :4].contiguous())
    with pytest.raises(B.DuoError) as e:
        f.decode(0, torch.zeros(2, 4, 64, device="cuda"))
    assert e.value.name == "DUO_ERR_UNSUPPORTED"
    with pytest.raises(B.DuoError) as e:  # no paged layout without the tensor-core decode
        DuoCache(1, 2, 4, 2, 64, "f32", 64, mask[None], 4, 16, pool_blocks=4)
    assert e.value.name == "DUO_ERR_UNSUPPORTED"
