"""The library's KV cache manager (C++, hstu_cache_* in include/hstu.h) against the oracle's model.

The manager is host code, so these tests need no GPU: they load libhstu_b200.so and drive the
manager and ``oracle/kv_cache.py`` with the same operations, comparing every output exactly
(integer page ids, pairs, lengths, tiers, dropped users, statistics).  The oracle model itself
is pinned in test_oracle_cache_pins.py.
"""
from __future__ import annotations

import json
import os
import random

import numpy as np
import pytest

import hstu_attention_b200 as hb
from oracle import kv_cache as kc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_cache_scenario.json")


def _lib_or_skip():
    try:
        hb.load()
    except hb.HstuError as e:
        pytest.skip(str(e))


def lib_prepare(c: hb.KVCache, ids, append):
    try:
        r = c.prepare(ids, append)
    except hb.CacheFull:
        return "full"
    except hb.HstuError:
        return "invalid"
    return {"tier_before": r["tier_before"].tolist(), "cached_lens": r["cached_lens"].tolist(),
            "page_rows": r["page_rows"].tolist(), "offload": r["offload"].tolist(),
            "onboard": r["onboard"].tolist(), "dropped": r["dropped"].tolist()}


def oracle_prepare(m: kc.CacheModel, ids, append):
    try:
        r = m.prepare(ids, append)
    except kc.CacheError as e:
        return e.kind
    return {"tier_before": r["tier_before"], "cached_lens": r["cached_lens"], "page_rows": r["page_rows"],
            "offload": [list(p) for p in r["offload"]], "onboard": [list(p) for p in r["onboard"]],
            "dropped": r["dropped"]}


def test_hand_worked_scenario_through_the_library():
    _lib_or_skip()
    spec = json.load(open(GOLDEN))
    cfg = spec["config"]
    c = hb.KVCache(cfg["gpu_pages"], cfg["host_pages"], cfg["page_size"], cfg["max_pages_per_user"])
    for i, st in enumerate(spec["steps"]):
        exp = st["expect"]
        where = f"step {i} ({st['op']})"
        if st["op"] == "prepare":
            got = lib_prepare(c, st["ids"], st["append"])
            if "error" in exp:
                assert got == exp["error"], where
            else:
                for key in exp:
                    assert got[key] == exp[key], f"{where}: {key} {got[key]} != {exp[key]}"
        elif st["op"] == "lookup":
            tiers, lens = c.lookup(st["ids"])
            assert tiers.tolist() == exp["tiers"] and lens.tolist() == exp["lengths"], where
        elif st["op"] == "evict":
            assert c.evict(st["id"]) == exp["tier"], where
        elif st["op"] == "compact":
            assert c.compact().tolist() == exp["moves"], where
        elif st["op"] == "page_rows":
            assert c.page_rows(st["ids"]).tolist() == exp["rows"], where
        elif st["op"] == "stats":
            s = c.stats()
            for key, val in exp.items():
                assert s[key] == val, f"{where}: {key}"


def drive_both(seed: int, steps: int):
    rng = random.Random(seed)
    P = rng.choice([1, 2, 4, 16])
    M = rng.randint(2, 12)
    G = rng.randint(M, 6 * M)
    Hp = rng.choice([0, rng.randint(1, 4 * M)])
    universe = [rng.randint(-(1 << 40), 1 << 40) for _ in range(rng.randint(4, 40))]
    c = hb.KVCache(G, Hp, P, M)
    m = kc.CacheModel(G, Hp, P, M)
    seen = {"full": 0, "invalid": 0, "offload": 0, "onboard": 0, "dropped": 0, "moves": 0}
    for step in range(steps):
        x = rng.random()
        where = f"seed {seed} step {step}"
        if x < 0.05:
            a, b = c.compact().tolist(), [list(p) for p in m.compact()]
            assert a == b, f"{where}: compaction"
            seen["moves"] += len(a)
        elif x < 0.1:
            uid = rng.choice(universe)
            assert c.evict(uid) == m.evict(uid), f"{where}: evict"
        else:
            ids = rng.sample(universe, rng.randint(1, min(6, len(universe))))
            if rng.random() < 0.03:
                ids.append(ids[0])          # a repeated id: rejected by both
            append = [rng.randint(0, 3 * P * rng.choice([1, 1, 2, M])) for _ in ids]
            a, b = lib_prepare(c, ids, append), oracle_prepare(m, ids, append)
            assert a == b, f"{where}: prepare {ids} {append}\nlibrary {a}\noracle  {b}"
            if isinstance(a, str):
                seen[a] += 1
            else:
                seen["offload"] += len(a["offload"])
                seen["onboard"] += len(a["onboard"])
                seen["dropped"] += len(a["dropped"])
        tiers, lens = c.lookup(universe)
        ref = m.lookup(universe)
        assert tiers.tolist() == [t for t, _ in ref] and lens.tolist() == [n for _, n in ref], f"{where}: lookup"
        assert c.stats() == m.stats(), f"{where}: stats"
        assert c.page_rows(universe).tolist() == m.page_rows(universe), f"{where}: page rows"
    return seen


@pytest.mark.parametrize("seed", range(12))
def test_library_matches_the_oracle_on_random_streams(seed):
    _lib_or_skip()
    drive_both(seed, 150)


def test_random_streams_cover_every_path():
    _lib_or_skip()
    total = {}
    for seed in range(12, 20):
        for k, v in drive_both(seed, 150).items():
            total[k] = total.get(k, 0) + v
    for k, v in total.items():
        assert v > 0, f"the random streams never exercised '{k}'"


def test_large_pool_matches_the_oracle():
    # bitmap words past the first, page ids in the hundreds of thousands
    _lib_or_skip()
    rng = random.Random(7)
    G, Hp, P, M = 70000, 30000, 32, 600
    c, m = hb.KVCache(G, Hp, P, M), kc.CacheModel(G, Hp, P, M)
    for step in range(40):
        ids = rng.sample(range(500), 8)
        append = [rng.randint(0, 4000) for _ in ids]
        assert lib_prepare(c, ids, append) == oracle_prepare(m, ids, append), f"step {step}"
        if step % 10 == 9:
            assert c.compact().tolist() == [list(p) for p in m.compact()]
            victim = rng.randrange(500)
            assert c.evict(victim) == m.evict(victim)
    assert c.stats() == m.stats()


def test_argument_errors_change_nothing():
    _lib_or_skip()
    c = hb.KVCache(8, 4, 4, 2)
    c.prepare([1, 2], [8, 4])
    before = (c.stats(), c.page_rows([1, 2]).tolist())
    with pytest.raises(hb.HstuError):
        c.prepare([3], [9])                 # 3 pages > max_pages_per_user
    with pytest.raises(hb.HstuError):
        c.prepare([3, 3], [1, 1])           # repeated id
    with pytest.raises(hb.HstuError):
        c.prepare([3], [-1])                # negative append
    with pytest.raises(hb.CacheFull):
        c.prepare([3, 4, 5, 6, 7], [8, 8, 8, 8, 8])
    assert (c.stats(), c.page_rows([1, 2]).tolist()) == before
    with pytest.raises(hb.HstuError):
        hb.KVCache(8, 4, 1 << 16, 1 << 16)  # stored lengths would overflow int32


def test_output_capacity_is_reported_and_changes_nothing():
    _lib_or_skip()
    import ctypes

    c = hb.KVCache(4, 4, 2, 4)
    c.prepare([1], [8])
    lib = hb.load()
    ids = np.array([2], np.int64)
    app = np.array([8], np.int32)
    tiers, cached = np.zeros(1, np.int32), np.zeros(1, np.int32)
    rows = np.zeros((1, 4), np.int32)
    off, on, drop = np.zeros((1, 2), np.int32), np.zeros((1, 2), np.int32), np.zeros(1, np.int64)
    n_off, n_on, n_drop = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    rc = lib.hstu_cache_prepare(c._h, ids.ctypes.data, app.ctypes.data, 1, tiers.ctypes.data, cached.ctypes.data,
                                rows.ctypes.data, off.ctypes.data, 1, ctypes.byref(n_off), on.ctypes.data, 1,
                                ctypes.byref(n_on), drop.ctypes.data, 1, ctypes.byref(n_drop))
    assert rc == hb.ERR_OUTPUT_CAPACITY
    assert (n_off.value, n_on.value, n_drop.value) == (4, 0, 0)
    assert c.stats()["clock"] == 1 and c.lookup([1])[0].tolist() == [hb.TIER_GPU]
    r = c.prepare([2], [8])                 # the binding retries with room for all four pairs
    assert r["offload"].tolist() == [[0, 0], [1, 1], [2, 2], [3, 3]]
