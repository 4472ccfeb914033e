"""Pins of the fp64 oracle to things other than itself (no GPU needed).

Each check is chosen so that a plausible slip in the oracle -- a wrong window
edge, a dropped scale, a transposed operand, a wrong GQA head mapping, a
missing max subtraction, a wrong nibble order -- fails at least one of them;
``test_planted_mistakes_are_caught`` plants such slips and confirms it.
"""

import collections
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as A
from oracle import cache as C
from oracle import int4 as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa_causal(q, k, v, scale=None):
    """Library routine: causal SDPA in float64.  q [Hq, n, d], k/v [Hkv, n, d]."""
    qt = torch.from_numpy(np.ascontiguousarray(q))[None]
    kt = torch.from_numpy(np.ascontiguousarray(k))[None]
    vt = torch.from_numpy(np.ascontiguousarray(v))[None]
    out = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale,
                                         enable_gqa=qt.shape[1] != kt.shape[1])
    return out[0].numpy()


# ---------------------------------------------------------------- retrieval


@pytest.mark.parametrize("Hq,Hkv,n,d", [(4, 4, 37, 16), (8, 2, 50, 32), (6, 3, 1, 8)])
def test_all_retrieval_prefill_equals_causal_sdpa(Hq, Hkv, n, d):
    r = _rng(n * 7 + Hq)
    q = r.standard_normal((1, n, Hq, d))
    k = r.standard_normal((1, n, Hkv, d))
    v = r.standard_normal((1, n, Hkv, d))
    got = A.prefill_reference(q, k, v, 0, np.ones(Hkv), S=2, R=3)
    ref = _sdpa_causal(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                       v[0].transpose(1, 0, 2)).transpose(1, 0, 2)
    np.testing.assert_allclose(got[0], ref, rtol=0, atol=1e-12)


def test_chunk_offset_rows_equal_tail_of_full_causal():
    r = _rng(11)
    n, c0, d, H = 40, 25, 16, 4
    q = r.standard_normal((1, n, H, d))
    k = r.standard_normal((1, n, H, d))
    v = r.standard_normal((1, n, H, d))
    got = A.prefill_reference(q[:, c0:], k, v, c0, np.ones(H), S=1, R=4)
    ref = _sdpa_causal(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                       v[0].transpose(1, 0, 2)).transpose(1, 0, 2)[c0:]
    np.testing.assert_allclose(got[0], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2)])
def test_all_retrieval_decode_equals_last_causal_row(Hq, Hkv):
    r = _rng(5 + Hkv)
    n, d = 33, 16
    q_all = r.standard_normal((1, n, Hq, d))
    k = r.standard_normal((1, n, Hkv, d))
    v = r.standard_normal((1, n, Hkv, d))
    got = A.decode_reference(q_all[:, -1], k, v, np.ones(Hkv), S=4, R=4)
    ref = _sdpa_causal(q_all[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                       v[0].transpose(1, 0, 2))[:, -1]
    np.testing.assert_allclose(got[0], ref, rtol=0, atol=1e-12)


def test_explicit_scale_matches_sdpa_scale():
    r = _rng(3)
    n, d = 20, 8
    q = r.standard_normal((1, n, 2, d))
    k = r.standard_normal((1, n, 2, d))
    v = r.standard_normal((1, n, 2, d))
    got = A.prefill_reference(q, k, v, 0, np.ones(2), 1, 1, scale=0.37)
    ref = _sdpa_causal(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                       v[0].transpose(1, 0, 2), scale=0.37).transpose(1, 0, 2)
    np.testing.assert_allclose(got[0], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- streaming


@pytest.mark.parametrize("S,R,n", [(4, 64, 60), (2, 5, 7), (0, 10, 10)])
def test_streaming_window_covering_context_is_full_attention(S, R, n):
    r = _rng(S * 100 + R)
    d = 8
    q = r.standard_normal((1, n, 2, d))
    k = r.standard_normal((1, n, 2, d))
    v = r.standard_normal((1, n, 2, d))
    got = A.prefill_reference(q, k, v, 0, np.zeros(2), S, R)
    ref = _sdpa_causal(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                       v[0].transpose(1, 0, 2)).transpose(1, 0, 2)
    np.testing.assert_allclose(got[0], ref, rtol=0, atol=1e-12)


class _DequeCache:
    """Independent model of a streaming head's cache: a sink list that fills
    first and a bounded deque of recent positions."""

    def __init__(self, S, R):
        self.S, self.sinks, self.recent = S, [], collections.deque(maxlen=R)

    def append(self, p):
        if len(self.sinks) < self.S:
            self.sinks.append(p)
        else:
            self.recent.append(p)

    def held(self):
        return list(self.sinks) + list(self.recent)


def _python_softmax_attention(q, keys, values, scale):
    logits = [scale * sum(a * b for a, b in zip(q, kk)) for kk in keys]
    m = max(logits)
    w = [math.exp(s - m) for s in logits]
    z = sum(w)
    return [sum(wi * vv[c] for wi, vv in zip(w, values)) / z
            for c in range(len(values[0]))]


@pytest.mark.parametrize("S", [0, 1, 2])
@pytest.mark.parametrize("R", [1, 3, 8])
def test_streaming_bruteforce_tiny(S, R):
    r = _rng(S * 10 + R)
    d = 3
    n = 29
    q = r.standard_normal((n, d))
    k = r.standard_normal((n, d))
    v = r.standard_normal((n, d))
    scale = 1.0 / math.sqrt(d)
    cache = _DequeCache(S, R)
    expect = []
    for p in range(n):
        cache.append(p)
        held = cache.held()
        expect.append(_python_softmax_attention(
            q[p], [k[j] for j in held], [v[j] for j in held], scale))
    expect = np.array(expect)
    # pre-fill rows of one streaming head, whole prompt as one chunk
    got = A.prefill_reference(q[None, :, None], k[None, :, None], v[None, :, None],
                              0, np.zeros(1), S, R)[0, :, 0]
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)
    # the same rows as successive decode steps
    for t in (0, S, S + R - 1, S + R, n - 1):
        if t >= n:
            continue
        dec = A.decode_reference(q[None, t][:, None], k[None, :t + 1, None],
                                 v[None, :t + 1, None], np.zeros(1), S, R)
        np.testing.assert_allclose(dec[0, 0], expect[t], rtol=0, atol=1e-12)


def test_rows_are_probability_vectors():
    r = _rng(9)
    n, d = 24, 24
    q = r.standard_normal((1, n, 1, d))
    k = r.standard_normal((1, n, 1, d))
    eye = np.eye(n)[None, :, None, :]  # v_j = e_j: the output row is p_i
    for retrieval in (0, 1):
        p = A.prefill_reference(q, k, eye, 0, np.array([retrieval]), 2, 5)[0, :, 0]
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert (p >= 0).all()
        vis = A.visible_mask(np.arange(n), np.arange(n), bool(retrieval), 2, 5)
        assert (p[~vis] == 0).all()
        ones = A.prefill_reference(q, k, np.ones((1, n, 1, 5)), 0,
                                   np.array([retrieval]), 2, 5)
        np.testing.assert_allclose(ones, 1.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariances


def test_streaming_decode_depends_only_on_its_window():
    """Changing K/V at a position that is neither a sink nor recent leaves a
    streaming head's output unchanged; changing one inside the window does
    not (the mask definition, checked without the ring)."""
    r = _rng(31)
    n, d, S, R = 40, 8, 3, 5
    q = r.standard_normal((1, 2, d))
    k = r.standard_normal((1, n, 2, d))
    v = r.standard_normal((1, n, 2, d))
    mask = np.array([0, 1])
    base = A.decode_reference(q, k, v, mask, S, R)
    for p in range(n):
        k2, v2 = k.copy(), v.copy()
        k2[0, p, 0] += 3.0
        v2[0, p, 0] -= 2.0
        got = A.decode_reference(q, k2, v2, mask, S, R)
        inside = p < S or n - 1 - p < R
        np.testing.assert_array_equal(got[0, 1], base[0, 1])  # retrieval head untouched
        if inside:
            assert np.abs(got[0, 0] - base[0, 0]).max() > 1e-6, p
        else:
            np.testing.assert_array_equal(got[0, 0], base[0, 0])


def test_value_affine_equivariance():
    """Softmax weights sum to one: O(q, K, a V + b) = a O(q, K, V) + b, for
    both kinds of head, at decode and in pre-fill."""
    r = _rng(32)
    n, d, S, R, a, b = 23, 8, 2, 4, -1.75, 0.625
    q = r.standard_normal((1, n, 4, d))
    k = r.standard_normal((1, n, 2, d))
    v = r.standard_normal((1, n, 2, d))
    mask = np.array([1, 0])
    o = A.prefill_reference(q, k, v, 0, mask, S, R)
    o2 = A.prefill_reference(q, k, a * v + b, 0, mask, S, R)
    np.testing.assert_allclose(o2, a * o + b, rtol=0, atol=1e-12)
    od = A.decode_reference(q[:, -1], k, v, mask, S, R)
    od2 = A.decode_reference(q[:, -1], k, a * v + b, mask, S, R)
    np.testing.assert_allclose(od2, a * od + b, rtol=0, atol=1e-12)


def test_retrieval_decode_ignores_history_order():
    """At decode every earlier key is visible to a retrieval head, so
    reordering the history (K and V together) leaves its output unchanged,
    while a streaming head, which sees positions, changes."""
    r = _rng(33)
    n, d, S, R = 30, 8, 2, 4
    q = r.standard_normal((1, 4, d))
    k = r.standard_normal((1, n, 2, d))
    v = r.standard_normal((1, n, 2, d))
    mask = np.array([1, 0])
    perm = np.concatenate([r.permutation(n - 1), [n - 1]])
    base = A.decode_reference(q, k, v, mask, S, R)
    got = A.decode_reference(q, k[:, perm], v[:, perm], mask, S, R)
    np.testing.assert_allclose(got[0, :2], base[0, :2], rtol=0, atol=1e-12)
    assert np.abs(got[0, 2:] - base[0, 2:]).max() > 1e-6


# ---------------------------------------------------------------- golden


def _golden():
    with open(GOLDEN) as f:
        return {c["name"]: c for c in json.load(f)["cases"]}


def test_golden_equal_logits_decode():
    c = _golden()["equal_logits_decode"]
    n, d = c["n"], c["d"]
    k = np.zeros((1, n, 2, d))
    v = np.zeros((1, n, 2, d))
    v[0, :, :, 0] = np.arange(n)[:, None]
    v[0, :, :, 1] = 1.0
    q = np.zeros((1, 2, d))
    out = A.decode_reference(q, k, v, np.array([1, 0]), c["S"], c["R"])
    np.testing.assert_allclose(out[0, 0], c["expected_retrieval"], atol=1e-12)
    np.testing.assert_allclose(out[0, 1], c["expected_streaming"], atol=1e-12)


def test_golden_equal_logits_prefill():
    c = _golden()["equal_logits_prefill_lambda"]
    C_ = c["C"]
    q = np.zeros((1, C_, 2, 1))
    k = np.zeros((1, C_, 2, 1))
    v = np.broadcast_to(np.arange(C_, dtype=float)[None, :, None, None], (1, C_, 2, 1))
    out = A.prefill_reference(q, k, v, c["c0"], np.array([1, 0]), c["S"], c["R"])
    np.testing.assert_allclose(out[0, :, 0, 0], c["expected_retrieval"], atol=1e-12)
    np.testing.assert_allclose(out[0, :, 1, 0], c["expected_streaming"], atol=1e-12)


def test_golden_heavy_key_default_scale():
    c = _golden()["one_heavy_key_default_scale"]
    n, d = c["n"], c["d"]
    k = np.zeros((1, n, 2, d))
    k[0, c["heavy_key"], :, 0] = c["heavy_logit_component"]
    v = np.zeros((1, n, 2, d))
    v[0, :, :, 0] = np.arange(n)[:, None]
    q = np.tile(np.array(c["q"]), (1, 2, 1))
    out = A.decode_reference(q, k, v, np.array([1, 0]), c["S"], c["R"])
    np.testing.assert_allclose(out[0, 0], c["expected_retrieval"], atol=1e-12)
    np.testing.assert_allclose(out[0, 1], c["expected_streaming"], atol=1e-12)


def test_golden_int4():
    c = _golden()["int4_group_of_four"]
    codes, sc, zp = Q.quantize_int4(np.array([c["x"]], dtype=np.float32))
    assert float(sc[0]) == c["expected_scale"]
    assert float(zp[0]) == c["expected_zero"]
    assert codes[0].tolist() == c["expected_codes"]
    assert Q.pack_nibbles(codes)[0].tolist() == c["expected_packed"]
    np.testing.assert_array_equal(Q.dequantize_int4(codes, sc, zp)[0],
                                  c["expected_dequant"])


def test_golden_ring_and_bytes():
    g = _golden()
    c = g["ring_slots"]
    assert [C.ring_slot(p, c["S"], c["R"]) for p in range(c["n"])] == c["expected_slots"]
    held = C.simulate_ring(c["n"], c["S"], c["R"])
    assert {str(s): p for s, p in held.items()} == c["expected_held"]
    b = g["kv_bytes_one_retrieval_head"]
    kept, full = C.kv_bytes(b["mask"], b["batch"], b["n"], b["S"], b["R"], b["d"], b["dtype"])
    assert (kept, full) == (b["expected_kept"], b["expected_full"])


def _position_rows(n, d=2):
    """Row p = [p, 100 + p, ...]: every position's row is distinct."""
    return np.array([[p + 100 * c for c in range(d)] for p in range(n)], dtype=np.int64)


def test_expected_streaming_buffer_golden_ring():
    """The golden ring case (S=2, R=3, n=10) written out by hand: after ten
    appends slot s holds position expected_held[s], so buffer row s must be
    position expected_held[s]'s row."""
    c = _golden()["ring_slots"]
    S, R, n = c["S"], c["R"], c["n"]
    rows = _position_rows(n)
    buf, filled = C.expected_streaming_buffer(rows, S, R)
    hand = np.array([[0, 100], [1, 101], [8, 108], [9, 109], [7, 107]], dtype=np.int64)
    assert [int(c["expected_held"][str(s)]) for s in range(S + R)] == [0, 1, 8, 9, 7]
    np.testing.assert_array_equal(buf, hand)
    assert filled.all()


def test_expected_streaming_buffer_partial_and_no_sinks():
    """Hand-built buffers where the ring has not wrapped yet (unwritten slots
    stay zero and are marked unfilled), and with no sinks (S=0)."""
    buf, filled = C.expected_streaming_buffer(_position_rows(3), 2, 3)
    np.testing.assert_array_equal(buf, [[0, 100], [1, 101], [2, 102], [0, 0], [0, 0]])
    assert filled.tolist() == [True, True, True, False, False]
    # S=0, R=3, n=7: positions 6, 4, 5 sit in slots 0, 1, 2 (p mod 3)
    buf, filled = C.expected_streaming_buffer(_position_rows(7), 0, 3)
    np.testing.assert_array_equal(buf, [[6, 106], [4, 104], [5, 105]])
    assert filled.all()
    # R=1: only the newest position after the sinks survives
    buf, filled = C.expected_streaming_buffer(_position_rows(9), 4, 1)
    np.testing.assert_array_equal(buf[:, 0], [0, 1, 2, 3, 8])


# ---------------------------------------------------------------- ring + bytes


@pytest.mark.parametrize("S,R", [(0, 1), (1, 1), (2, 3), (4, 64), (64, 256)])
def test_ring_holds_exactly_sinks_and_recent(S, R):
    cache = _DequeCache(S, R)
    for n in range(1, 3 * (S + R) + 7):
        cache.append(n - 1)
        held = C.simulate_ring(n, S, R)
        assert sorted(held.values()) == sorted(cache.held())
        assert all(0 <= s < S + R for s in held)
        for s, p in held.items():
            assert C.ring_slot(p, S, R) == s


def test_kv_bytes_matches_counted_buffers():
    mask = np.array([[1, 0, 1, 0, 0], [0, 0, 0, 0, 1]])
    for dtype, d in (("bf16", 128), ("f32", 64), ("int4", 128)):
        for n in (1, 7, 100, 1000):
            S, R, B = 4, 12, 3
            per = C.bytes_per_token_per_head(d, dtype)
            counted = 0
            for layer in mask:
                for bit in layer:
                    tokens = n if bit else len(C.simulate_ring(n, S, R))
                    counted += B * tokens * per
            kept, full = C.kv_bytes(mask, B, n, S, R, d, dtype)
            assert kept == counted
            assert full == mask.size * B * n * per
    assert C.bytes_per_token_per_head(128, "int4") == 136
    assert C.bytes_per_token_per_head(128, "bf16") == 512


# ---------------------------------------------------------------- int4


def test_int4_error_bound_and_range():
    r = _rng(21)
    x = r.standard_normal((500, 128)).astype(np.float32)
    x[:, ::37] *= 10.0
    codes, sc, zp = Q.quantize_int4(x)
    assert codes.max() <= 15
    xh = Q.dequantize_int4(codes, sc, zp)
    bound = sc.astype(np.float64)[:, None] / 2
    # the fp16 rounding of the scale can push the top of the range past 15*sc
    slack = np.abs(15 * sc.astype(np.float64) - (x.max(1) - zp.astype(np.float64)))[:, None]
    assert (np.abs(x - xh) <= bound + slack + 1e-7).all()
    inner = (x >= zp.astype(np.float32)[:, None]) & (x <= (zp.astype(np.float64) + 15 * sc.astype(np.float64))[:, None])
    assert (np.abs(x - xh)[inner] <= bound.repeat(128, 1)[inner] * (1 + 1e-3)).all()


def test_int4_on_grid_round_trip_and_constant_group():
    sc = np.float16(0.125)
    zp = np.float16(-0.75)
    u = np.arange(16, dtype=np.uint8)
    x = (np.float32(sc) * u + np.float32(zp)).astype(np.float32)
    codes, sc2, zp2 = Q.quantize_int4(x[None])
    assert sc2[0] == sc and zp2[0] == zp
    assert codes[0].tolist() == u.tolist()
    const = np.full((1, 8), 3.25, dtype=np.float32)
    codes, sc3, zp3 = Q.quantize_int4(const)
    assert sc3[0] == 0 and codes.max() == 0
    assert Q.dequantize_int4(codes, sc3, zp3)[0].tolist() == [3.25] * 8


def test_int4_fp32_mirror_matches_float64_away_from_ties():
    r = _rng(4)
    x = r.standard_normal((300, 64)).astype(np.float32)
    codes, sc, zp = Q.quantize_int4(x)
    t64 = (x.astype(np.float64) - zp.astype(np.float64)[:, None]) / sc.astype(np.float64)[:, None]
    frac = np.abs(t64 - np.floor(t64) - 0.5)
    safe = frac > 1e-4
    ref = np.clip(np.rint(t64), 0, 15)
    assert (codes[safe] == ref[safe]).all()
    assert safe.mean() > 0.99


def test_nibble_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert Q.pack_nibbles(codes).tolist() == [[0x21, 0x43]]
    np.testing.assert_array_equal(Q.unpack_nibbles(Q.pack_nibbles(codes)), codes)


# ---------------------------------------------------------------- needle sanity


def test_needle_draws_mass_on_retrieval_only():
    from head_split_kv_decode_b200 import synth
    r = _rng(8)
    n, d, S, R = 2000, 128, 64, 256
    k = 0.5 * r.standard_normal((1, n, 2, d))
    v = r.standard_normal((1, n, 2, d))
    q = r.standard_normal((1, 2, d))
    pos = 700
    for h in range(2):
        k[0, pos, h] = synth.needle_key(torch.from_numpy(q[0, h]), 8.0, 0.5).numpy()
    eye_v = np.zeros((1, n, 2, n))
    eye_v[0, np.arange(n), :, np.arange(n)] = 1.0
    p = A.decode_reference(q, k, eye_v, np.array([1, 0]), S, R)
    assert p[0, 0, pos] > 20.0 / n  # e^4 against ~1.13 per ordinary key
    assert p[0, 1, pos] == 0.0


# ---------------------------------------------------------------- mutation check


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant typical slips in the oracle and confirm a pin above notices."""
    good_mask = A.visible_mask

    def off_by_one_window(qp, kp, retrieval, S, R):
        m = good_mask(qp, kp, retrieval, S, R + 1)
        return m

    def sinks_dropped(qp, kp, retrieval, S, R):
        return good_mask(qp, kp, retrieval, 0, R)

    for bad in (off_by_one_window, sinks_dropped):
        monkeypatch.setattr(A, "visible_mask", bad)
        with pytest.raises(AssertionError):
            test_streaming_bruteforce_tiny(2, 3)
        with pytest.raises(AssertionError):
            test_golden_equal_logits_prefill()
        with pytest.raises(AssertionError):
            test_streaming_decode_depends_only_on_its_window()
        monkeypatch.setattr(A, "visible_mask", good_mask)

    good_attn = A.masked_attention

    def no_scale(q, k, v, mask, scale):
        return good_attn(q, k, v, mask, 1.0)

    def transposed_v(q, k, v, mask, scale):
        vv = np.asarray(v)
        if vv.shape[0] == vv.shape[1]:
            vv = vv.T
        return good_attn(q, k, vv, mask, scale)

    def unnormalised(q, k, v, mask, scale):
        # weights exp(s - max) without dividing by their sum
        s_ = np.where(mask, (np.asarray(q) @ np.asarray(k).T) * scale, -np.inf)
        return np.exp(s_ - s_.max(axis=1, keepdims=True)) @ np.asarray(v)

    monkeypatch.setattr(A, "masked_attention", unnormalised)
    with pytest.raises(AssertionError):
        test_value_affine_equivariance()
    monkeypatch.setattr(A, "masked_attention", no_scale)
    with pytest.raises(AssertionError):
        test_all_retrieval_prefill_equals_causal_sdpa(4, 4, 37, 16)
    monkeypatch.setattr(A, "masked_attention", transposed_v)
    with pytest.raises(AssertionError):
        test_golden_heavy_key_default_scale()
    monkeypatch.setattr(A, "masked_attention", good_attn)

    good_q = Q.quantize_int4

    def floor_not_rint(x):
        codes, sc, zp = good_q(x)
        scf = sc.astype(np.float32)[..., None]
        t = (np.asarray(x, np.float32) - zp.astype(np.float32)[..., None]) / np.where(scf == 0, 1, scf)
        return np.clip(np.floor(t), 0, 15).astype(np.uint8), sc, zp

    monkeypatch.setattr(Q, "quantize_int4", floor_not_rint)
    with pytest.raises(AssertionError):
        test_golden_int4()
    monkeypatch.setattr(Q, "quantize_int4", good_q)

    good_buf = C.expected_streaming_buffer

    def indexed_by_position(k_head, S, R):
        # a slip: row p stored at row p mod W instead of at its ring slot
        k_head = np.asarray(k_head)
        W = S + R
        buf = np.zeros((W,) + k_head.shape[1:], dtype=k_head.dtype)
        filled = np.zeros(W, dtype=bool)
        for p in range(k_head.shape[0]):
            buf[p % W] = k_head[p]
            filled[p % W] = True
        return buf, filled

    monkeypatch.setattr(C, "expected_streaming_buffer", indexed_by_position)
    with pytest.raises(AssertionError):
        test_expected_streaming_buffer_golden_ring()
    monkeypatch.setattr(C, "expected_streaming_buffer", good_buf)
