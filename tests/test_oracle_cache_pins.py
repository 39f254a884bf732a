"""Pins of the oracle's two-tier KV cache model (oracle/kv_cache.py) against facts other than itself.

* A scenario worked out by hand from the cache's definition (tests/golden/kv_cache_scenario.json):
  eviction order, offload and onboard pairs, drops, errors that leave the state unchanged.
* Invariants on seeded random request streams, checked from outside the model:
  - every page belongs to at most one user or to the free list, and together they cover the tier;
  - a user holds ceil(n / P) pages;
  - every batch user is on the GPU afterwards;
  - GPU victims are the oldest residents outside the batch, and no more than the batch needed;
  - host residents are dropped oldest first, and only for a newer victim.
* Data follows each user: tagged tokens are moved by exactly the copies the calls return
  (offload, then onboard, then the append at the returned positions, and compaction moves).
  Reading every resident user's tokens back through its pages must give its tags in order.
* Planted mistakes (MRU order, evicting batch members, swapped pairs, floor instead of ceil,
  stale stamps, ...) are compiled into copies of the model, and each one must fail a pin.

The cache's definition follows the NVIDIA blog "Deploying an HSTU Generative Recommender with
NVIDIA Dynamo-Triton", section "Why serving large sequential recommenders is hard" (paged GPU KV
table: lookup, allocate, append, evict; LRU-like eviction; host tier; onboard and offload).
"""
from __future__ import annotations

import inspect
import json
import os
import random
import types

import numpy as np
import pytest

from oracle import kv_cache as kc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_cache_scenario.json")


def run_scenario(mod):
    spec = json.load(open(GOLDEN))
    cfg = spec["config"]
    m = mod.CacheModel(cfg["gpu_pages"], cfg["host_pages"], cfg["page_size"], cfg["max_pages_per_user"])
    for i, st in enumerate(spec["steps"]):
        exp = st["expect"]
        where = f"step {i} ({st['op']})"
        if st["op"] == "prepare":
            if "error" in exp:
                before = (repr(sorted((k, v.tier, v.n, v.pages, v.stamp) for k, v in m.users.items())),
                          repr(m.free), m.clock)
                with pytest.raises(mod.CacheError) as ei:
                    m.prepare(st["ids"], st["append"])
                assert ei.value.kind == exp["error"], where
                after = (repr(sorted((k, v.tier, v.n, v.pages, v.stamp) for k, v in m.users.items())),
                         repr(m.free), m.clock)
                assert before == after, f"{where}: a rejected call changed the state"
                continue
            r = m.prepare(st["ids"], st["append"])
            for key in ("tier_before", "cached_lens", "page_rows", "dropped"):
                assert r[key] == exp[key], f"{where}: {key} {r[key]} != {exp[key]}"
            for key in ("offload", "onboard"):
                assert [list(p) for p in r[key]] == exp[key], f"{where}: {key} {r[key]} != {exp[key]}"
        elif st["op"] == "lookup":
            got = m.lookup(st["ids"])
            assert [t for t, _ in got] == exp["tiers"], where
            assert [n for _, n in got] == exp["lengths"], where
        elif st["op"] == "evict":
            assert m.evict(st["id"]) == exp["tier"], where
        elif st["op"] == "compact":
            assert [list(p) for p in m.compact()] == exp["moves"], where
        elif st["op"] == "page_rows":
            assert m.page_rows(st["ids"]) == exp["rows"], where
        elif st["op"] == "stats":
            s = m.stats()
            for key, val in exp.items():
                assert s[key] == val, f"{where}: {key} {s[key]} != {val}"


def tag(uid: int, pos: int) -> int:
    return uid * 100000 + pos


class DataSim:
    """Tagged tokens in a GPU pool and a host pool, moved only by the copies the model returns."""

    def __init__(self, mod, G, Hp, P, M):
        self.mod = mod
        self.m = mod.CacheModel(G, Hp, P, M)
        self.G, self.Hp, self.P, self.M = G, Hp, P, M
        self.gpu = np.full((G, P), -1, np.int64)
        self.host = np.full((max(Hp, 1), P), -1, np.int64)

    def snapshot(self):
        return {uid: (u.tier, u.n, list(u.pages), u.stamp) for uid, u in self.m.users.items()}

    def prepare(self, ids, append):
        m, mod = self.m, self.mod
        before = self.snapshot()
        free_gpu_before = len(m.free[mod.GPU])
        r = m.prepare(ids, append)
        # copies in the order the definition prescribes, then the append
        kc.page_copy(self.gpu, self.host, r["offload"])
        kc.page_copy(self.host, self.gpu, r["onboard"])
        for b, uid in enumerate(ids):
            row = r["page_rows"][b]
            for t in range(append[b]):
                pos = r["cached_lens"][b] + t
                self.gpu[row[pos // self.P], pos % self.P] = tag(uid, pos)
        self.check_after_prepare(before, free_gpu_before, ids, append, r)
        self.check_state()
        return r

    def compact(self):
        moves = self.m.compact()
        srcs = {s for s, _ in moves}
        assert not srcs & {d for _, d in moves}, "compaction moves overlap"
        kc.page_copy(self.gpu, self.gpu, moves)
        live = sum(len(u.pages) for u in self.m.users.values() if u.tier == self.mod.GPU)
        for u in self.m.users.values():
            if u.tier == self.mod.GPU:
                assert all(p < live for p in u.pages), "compaction left a page above the live count"
        self.check_state()

    def evict(self, uid):
        self.m.evict(uid)
        self.check_state()

    def check_state(self):
        m, mod = self.m, self.mod
        for tier, size in ((mod.GPU, self.G), (mod.HOST, self.Hp)):
            owned = [p for u in m.users.values() if u.tier == tier for p in u.pages]
            assert len(owned) == len(set(owned)), "a page belongs to two users"
            assert not set(owned) & set(m.free[tier]), "a page is both owned and free"
            assert sorted(owned + m.free[tier]) == list(range(size)), "pages lost or invented"
        for uid, u in m.users.items():
            assert len(u.pages) == -(-u.n // self.P), f"user {uid}: {len(u.pages)} pages for {u.n} tokens"
            assert len(u.pages) <= self.M
            pool = self.gpu if u.tier == mod.GPU else self.host
            got = [int(pool[u.pages[p // self.P], p % self.P]) for p in range(u.n)]
            assert got == [tag(uid, p) for p in range(u.n)], f"user {uid}: its tokens did not follow it"

    def check_after_prepare(self, before, free_gpu_before, ids, append, r):
        mod = self.mod
        after = self.snapshot()
        batch = set(ids)
        for uid in ids:
            assert after[uid][0] == mod.GPU, "a batch user is not on the GPU"
        # the batch's page demand, from the state before the call
        demand = 0
        for uid, a in zip(ids, append):
            n = before[uid][1] if uid in before else 0
            have = len(before[uid][2]) if (uid in before and before[uid][0] == mod.GPU) else 0
            demand += -(-(n + a) // self.P) - have
        key = lambda uid: (before[uid][3], uid)  # noqa: E731
        was_gpu = [u for u in before if before[u][0] == mod.GPU and u not in batch]
        victims = [u for u in was_gpu if after.get(u, (mod.MISS,))[0] != mod.GPU]
        stayed = [u for u in was_gpu if u not in victims]
        if victims and stayed:
            assert max(map(key, victims)) < min(map(key, stayed)), "a newer GPU resident was evicted first"
        if victims:
            oldest_first = sorted(victims, key=key)
            freed_but_last = sum(len(before[u][2]) for u in oldest_first[:-1])
            assert free_gpu_before + freed_but_last < demand, "more GPU users evicted than the batch needed"
        # host residents dropped: oldest first, and only for a newer offloaded victim
        was_host = [u for u in before if before[u][0] == mod.HOST and u not in batch]
        host_dropped = [u for u in was_host if u not in after]
        host_kept = [u for u in was_host if u in after]
        if host_dropped:
            offloaded = [u for u in victims if u in after]
            assert offloaded, "a host resident was dropped with nothing to offload"
            assert max(map(key, host_dropped)) < max(map(key, offloaded)), "a host resident made room for an older user"
            if host_kept:
                assert max(map(key, host_dropped)) < min(map(key, host_kept)), "host residents not dropped oldest first"
        gone = sorted(u for u in before if u not in after)
        assert sorted(r["dropped"]) == gone, "the dropped list does not match the users that left the cache"
        # one copy launch runs the pairs in any order: no page may be written twice, and a user
        # whose pages are offloaded must still be in the host tier afterwards
        for pairs in (r["offload"], r["onboard"]):
            dsts = [d for _, d in pairs]
            assert len(set(dsts)) == len(dsts), "a page is the destination of two copies"
        offloaded_src = {s for s, _ in r["offload"]}
        for u in gone:
            if before[u][0] == mod.GPU:
                assert not offloaded_src & set(before[u][2]), "a user was offloaded and dropped in one call"
        for u in victims:
            if u in after:
                assert after[u][0] == mod.HOST and len(after[u][2]) == len(before[u][2])
        for b, uid in enumerate(ids):
            assert r["cached_lens"][b] == (before[uid][1] if uid in before else 0)


def random_stream(mod, seed: int, steps: int = 120):
    rng = random.Random(seed)
    P = rng.choice([2, 4, 8])
    M = rng.randint(3, 8)
    G = rng.randint(M, 4 * M)
    Hp = rng.randint(0, 3 * M)
    sim = DataSim(mod, G, Hp, P, M)
    universe = list(range(1, rng.randint(6, 24)))
    fulls = 0
    for _ in range(steps):
        x = rng.random()
        if x < 0.06:
            sim.compact()
            continue
        if x < 0.1:
            sim.evict(rng.choice(universe))
            continue
        ids = rng.sample(universe, rng.randint(1, min(4, len(universe))))
        append = []
        for uid in ids:
            n = sim.m.users[uid].n if uid in sim.m.users else 0
            room = M * P - n
            append.append(rng.randint(0, max(0, min(room, 3 * P))))
        before = sim.snapshot()
        free_before = {t: list(v) for t, v in sim.m.free.items()}
        try:
            sim.prepare(ids, append)
        except mod.CacheError as e:
            assert e.kind == "full"
            assert sim.snapshot() == before and sim.m.free == free_before, "a rejected call changed the state"
            fulls += 1
    return fulls


def test_hand_worked_scenario():
    run_scenario(kc)


@pytest.mark.parametrize("seed", range(8))
def test_random_streams_keep_data_and_invariants(seed):
    random_stream(kc, seed)


def test_random_streams_reach_the_full_cache():
    # the streams exercise the rejection path too (else the state-unchanged check proves nothing)
    assert sum(random_stream(kc, s, steps=80) for s in range(8)) > 0


def test_page_copy_moves_whole_pages():
    src = np.arange(12).reshape(4, 3)
    dst = np.zeros((3, 3), np.int64)
    kc.page_copy(src, dst, [(3, 0), (1, 2)])
    assert dst.tolist() == [[9, 10, 11], [0, 0, 0], [3, 4, 5]]


MUTATIONS = {
    "most recently used evicted first": ("if u.tier == GPU and uid not in batch), key=self.key)",
                                         "if u.tier == GPU and uid not in batch), key=self.key, reverse=True)"),
    "batch members can be evicted": ("if u.tier == GPU and uid not in batch), key=self.key)",
                                     "if u.tier == GPU), key=self.key)"),
    "victims offloaded oldest first": ("return sorted(victims, key=self.key, reverse=True)",
                                       "return sorted(victims, key=self.key)"),
    "newer host residents evictable": ("and uid not in batch and self.key(uid) < vk)", "and uid not in batch)"),
    "onboarding users' host pages evictable": ("and uid not in batch and self.key(uid) < vk)",
                                               "and self.key(uid) < vk)"),
    "onboard pairs reversed": ("onboard += list(zip(u.pages, fresh))", "onboard += list(zip(fresh, u.pages))"),
    "offload pairs reversed": ("offload += list(zip(v.pages, hp))", "offload += list(zip(hp, v.pages))"),
    "compaction pairs reversed": ("return list(zip(srcs, dsts))", "return list(zip(dsts, srcs))"),
    "floor instead of ceil": ("return -(-n // self.P)", "return n // self.P"),
    "stamps of hits not refreshed": ("            u.stamp = stamp\n", "            pass\n"),
    "demand ignores pages already held": ("demand += k - have", "demand += k"),
    "cached length reported after the append": ("            cached.append(u.n)\n            u.n += a\n",
                                                "            u.n += a\n            cached.append(u.n)\n"),
    "free list handed out highest first": ("got = self.free[tier][:k]\n        assert len(got) == k\n        del self.free[tier][:k]",
                                           "got = self.free[tier][len(self.free[tier]) - k:][::-1]\n        assert len(got) == k\n        del self.free[tier][len(self.free[tier]) - k:]"),
}


def mutated(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(kc)
    assert src.count(old) == 1, f"mutation '{name}' does not match the oracle source exactly once"
    mod = types.ModuleType(f"kv_cache_mutant_{abs(hash(name))}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


def pins_fail(mod) -> bool:
    try:
        run_scenario(mod)
        for seed in range(8):
            random_stream(mod, seed)
    except (AssertionError, Exception):
        return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name):
    assert pins_fail(mutated(name)), f"planted mistake '{name}' passed every pin"
