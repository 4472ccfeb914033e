"""The tensor-core decode's launch planner, on the host (no GPU): split counts
per row and streaming heads per streaming CTA for given lengths and SM
counts, through the C ABI's testing hook.  Checks the plans of the
benchmark's workloads on a 148-SM device and, over seeded random launches,
the rules the planner states: every SM slot used while splits can grow, no
row past its split cap, longer rows never fewer splits, and streaming heads
packed only while a streaming warp's keys stay within 3/4 of a retrieval
warp's in the longest split."""

import math

import numpy as np
import pytest

from head_split_kv_decode_b200 import binding as B
from head_split_kv_decode_b200 import build as BUILD

SMS = 148


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.lib()


def _cache(Hq, Hkv, ret, kv="bf16", S=64, R=256, batch=1, capacity=1 << 20, D=128):
    mask = [1 if h in ret else 0 for h in range(Hkv)]
    return B.duo_cache_create(layers=1, batch=batch, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=D,
                              kv_dtype=kv, capacity=capacity, head_mask=mask, S=S, R=R)


def _ctas(splits, pack, n_ret, n_str):
    return n_ret * sum(splits) + len(splits) * math.ceil(n_str / pack)


def test_benchmark_workloads(lib):
    # 128K GQA, batch 1: 4 retrieval heads split 36 ways; 4 streaming heads,
    # one per CTA (packing frees no split: (148 - 1) // 4 == (148 - 4) // 4)
    h = _cache(32, 8, (0, 2, 4, 6))
    try:
        splits, pack = B.duo_test_plan_decode(h, 0, [131073], SMS)
        assert (splits, pack) == ([36], 1)
        # batch 4: 16 streaming CTAs become 4, which buys 3 more splits
        splits, pack = B.duo_test_plan_decode(h, 0, [131073] * 4, SMS)
        assert pack == 4 and sum(splits) == 36 and _ctas(splits, pack, 4, 4) == 148
    finally:
        B.duo_cache_destroy(h)
    # 32K MHA: 8 retrieval heads, 24 streaming heads two to a CTA
    h = _cache(32, 32, tuple(range(0, 32, 4)))
    try:
        splits, pack = B.duo_test_plan_decode(h, 0, [32769], SMS)
        assert (splits, pack) == ([17], 2) and _ctas(splits, pack, 8, 24) == 148
    finally:
        B.duo_cache_destroy(h)
    # 1M on a 4-bit cache: 2 retrieval heads, 6 streaming heads four to a CTA
    h = _cache(32, 8, (1, 5), kv="int4", capacity=1 << 21)
    try:
        splits, pack = B.duo_test_plan_decode(h, 0, [1048577], SMS)
        assert (splits, pack) == ([73], 4) and _ctas(splits, pack, 2, 6) == 148
    finally:
        B.duo_cache_destroy(h)


def test_short_rows_and_forced_splits(lib):
    h = _cache(32, 8, (0, 2, 4, 6))
    try:
        # a context shorter than two CTA iterations: one split, no packing
        assert B.duo_test_plan_decode(h, 0, [200], SMS) == ([1], 1)
        B.duo_set_decode_splits(h, 5)
        splits, pack = B.duo_test_plan_decode(h, 0, [131073, 100, 3], SMS)
        assert splits == [5, 5, 3] and pack == 1  # forced: every row, capped by its keys
        B.duo_set_decode_splits(h, 0)
        splits, _ = B.duo_test_plan_decode(h, 0, [131073, 100], SMS)
        assert splits[0] > 5 and splits[1] == 1
    finally:
        B.duo_cache_destroy(h)


@pytest.mark.parametrize("seed", range(40))
def test_planner_rules_on_random_launches(lib, seed):
    rng = np.random.default_rng(seed)
    Hkv = int(rng.choice([4, 8, 16, 32]))
    G = int(rng.choice([1, 2, 4, 8])) if Hkv <= 8 else int(rng.choice([1, 2]))
    n_ret = int(rng.integers(1, Hkv + 1))
    ret = tuple(sorted(rng.choice(Hkv, n_ret, replace=False)))
    n_str = Hkv - n_ret
    kv = "int4" if rng.random() < 0.3 else "bf16"
    S, R = int(rng.choice([4, 16, 64])), int(rng.choice([60, 128, 256]))
    W = S + R
    tile_rows = 512 if kv == "int4" else 256
    nrows = int(rng.integers(1, 9))
    lens = [int(x) for x in np.exp(rng.uniform(np.log(2), np.log(600000), nrows))]
    sms = int(rng.choice([132, 148, 160]))
    h = _cache(Hkv * G, Hkv, ret, kv=kv, S=S, R=R, batch=nrows)
    try:
        splits, pack = B.duo_test_plan_decode(h, 0, lens, sms)
    finally:
        B.duo_cache_destroy(h)
    caps = [max(1, min(512, -(-n // (2 * tile_rows)), n)) for n in lens]
    # pack: a power of two, no more groups than the next power of two of the heads
    assert pack in (1, 2, 4, 8)
    assert pack == 1 or pack < 2 * n_str
    # splits within [1, cap]; longer rows never get fewer
    assert all(1 <= s <= c for s, c in zip(splits, caps)), (splits, caps)
    order = np.argsort(lens, kind="stable")
    assert all(splits[order[i]] <= splits[order[i + 1]] for i in range(nrows - 1)), (lens, splits)
    # every SM slot left after the streaming CTAs is used while rows can take more splits
    str_ctas = nrows * math.ceil(n_str / pack)
    budget = max(nrows, (sms - str_ctas) // n_ret)
    assert sum(splits) == min(budget, sum(caps)), (splits, caps, budget)
    # packing only while a streaming warp's keys stay within 3/4 of a retrieval warp's
    if pack > 1:
        win = (min(max(lens), W) + 15) // 16 * 16
        longest = max(n / s for n, s in zip(lens, splits))
        assert pack * win <= 0.75 * longest


def test_plan_hook_arguments(lib):
    h = _cache(32, 8, (0, 2, 4, 6))
    try:
        for bad in ([], [0], [10] * 129):
            with pytest.raises(B.DuoError):
                B.duo_test_plan_decode(h, 0, bad, SMS)
        with pytest.raises(B.DuoError):
            B.duo_test_plan_decode(h, 0, [100], 0)
        with pytest.raises(B.DuoError):
            B.duo_test_plan_decode(h, 1, [100], SMS)
    finally:
        B.duo_cache_destroy(h)
    h = _cache(8, 8, (0, 1), kv="f32", D=64)
    try:
        with pytest.raises(B.DuoError) as e:
            B.duo_test_plan_decode(h, 0, [100], SMS)
        assert e.value.name == "DUO_ERR_UNSUPPORTED"
    finally:
        B.duo_cache_destroy(h)
