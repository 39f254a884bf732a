"""Plain model of the two-tier paged KV cache around append (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module.  It shares no code with ``hstu_attention_b200`` (whose cache manager is C++ in the
library); tests run both on the same operation sequences and compare every output exactly.

What the pages fix (NVIDIA blog "Deploying an HSTU Generative Recommender with NVIDIA
Dynamo-Triton", section "Why serving large sequential recommenders is hard"; the same facts in
the Russian and Vietnamese summaries of that post): the GPU cache is a paged KV table with
lookup, allocate, append and evict; when GPU cache space runs short, old users are evicted by an
LRU-like policy; host storage is a further tier for cached KV; the exported path has cache-aware
operations for lookup, allocate, onboard, append and offload.  The pages give no algorithm
beyond that.  The readings below are this model's definition (the C++ manager implements the
same definition independently):

* Two tiers of pages, GPU (``gpu_pages``) and host (``host_pages``).  A user is resident in at
  most one tier, with a stored length ``n`` (tokens), ``ceil(n / P)`` pages of that tier in
  logical order, and a stamp (the number of the last batch it was in).
* Free pages are handed out lowest id first.
* ``prepare(ids, append)`` serves one batch (ids distinct).  With ``n_b`` the stored length
  (0 on a miss), user b needs ``ceil((n_b + append_b) / P)`` GPU pages (at most
  ``max_pages_per_user``).  The extra GPU pages the batch needs are taken from the free list;
  if it is short, GPU residents outside the batch are evicted oldest first, ordered by
  (stamp, user id), until enough pages are free (if that cannot be done, nothing changes and
  the call fails).  Evicted users are offloaded to the host tier newest first: a victim that
  does not fit in the free host pages may take the pages of host residents outside the batch
  that are older than itself (oldest first); if even all of those would not make room, the
  victim is dropped.  Then, in batch order, GPU residents get their extra pages, host
  residents of the batch are onboarded into fresh GPU pages (their host pages are freed at the
  end of the call, after the offloads took theirs), and misses get fresh pages.  Every batch
  user's stamp becomes the new batch number and its stored length becomes ``n_b + append_b``:
  the caller appends those tokens right after the call.
* Copies the caller must run, in this order, before it writes any of the batch's pages:
  ``offload`` pairs (GPU page -> host page), then ``onboard`` pairs (host page -> GPU page).
* ``compact()`` moves GPU pages so that the resident users occupy pages ``[0, live)``: the live
  pages at ids >= live, ascending, go to the free ids < live, ascending.

Pins: ``tests/test_oracle_cache_pins.py`` (a scenario worked by hand in
``tests/golden/kv_cache_scenario.json``; structural and LRU invariants; data that follows each
user through offload, onboard, append and compaction; planted mistakes).
"""
from __future__ import annotations

import copy

MISS, GPU, HOST = 0, 1, 2


class CacheError(Exception):
    """Raised for a request the cache rejects; the state is left as it was."""

    def __init__(self, kind: str, msg: str = ""):
        super().__init__(f"{kind}: {msg}" if msg else kind)
        self.kind = kind  # "invalid" | "full"


class User:
    def __init__(self, tier: int, n: int, pages: list, stamp: int):
        self.tier = tier
        self.n = n
        self.pages = pages
        self.stamp = stamp


class CacheModel:
    def __init__(self, gpu_pages: int, host_pages: int, page_size: int, max_pages_per_user: int):
        self.G = gpu_pages
        self.Hp = host_pages
        self.P = page_size
        self.M = max_pages_per_user
        self.users = {}
        self.free = {GPU: list(range(gpu_pages)), HOST: list(range(host_pages))}
        self.clock = 0

    # ---- small steps (each one line of the definition above) ----
    def pages_for(self, n: int) -> int:
        return -(-n // self.P)

    def take(self, tier: int, k: int) -> list:
        got = self.free[tier][:k]
        assert len(got) == k
        del self.free[tier][:k]
        return got

    def give(self, tier: int, pages: list):
        self.free[tier] = sorted(self.free[tier] + list(pages))

    def key(self, uid: int):
        return (self.users[uid].stamp, uid)

    def gpu_victim_order(self, batch: set) -> list:
        """GPU residents outside the batch, oldest first."""
        return sorted((uid for uid, u in self.users.items() if u.tier == GPU and uid not in batch), key=self.key)

    def offload_order(self, victims: list) -> list:
        """Victims are placed in the host tier newest first."""
        return sorted(victims, key=self.key, reverse=True)

    def host_evictable(self, batch: set, victim: int) -> list:
        """Host residents outside the batch that are older than the victim, oldest first."""
        vk = self.key(victim)
        return sorted((uid for uid, u in self.users.items()
                       if u.tier == HOST and uid not in batch and self.key(uid) < vk), key=self.key)

    # ---- operations ----
    def lookup(self, ids) -> list:
        """(tier, stored length) per id; no state changes."""
        out = []
        for uid in ids:
            u = self.users.get(int(uid))
            out.append((u.tier, u.n) if u is not None else (MISS, 0))
        return out

    def prepare(self, ids, append) -> dict:
        saved = copy.deepcopy((self.users, self.free, self.clock))
        try:
            return self._prepare([int(x) for x in ids], [int(x) for x in append])
        except CacheError:
            self.users, self.free, self.clock = saved
            raise

    def _prepare(self, ids: list, append: list) -> dict:
        if len(ids) != len(append) or len(set(ids)) != len(ids):
            raise CacheError("invalid", "ids must be distinct, one append length each")
        if any(a < 0 for a in append):
            raise CacheError("invalid", "negative append length")
        batch = set(ids)
        need = []
        demand = 0
        for uid, a in zip(ids, append):
            u = self.users.get(uid)
            n = u.n if u is not None else 0
            k = self.pages_for(n + a)
            if k > self.M:
                raise CacheError("invalid", f"user {uid} needs {k} pages > max_pages_per_user")
            need.append(k)
            have = len(u.pages) if (u is not None and u.tier == GPU) else 0
            demand += k - have

        # GPU victims, oldest first, until the demand fits
        victims = []
        free_gpu = len(self.free[GPU])
        for uid in self.gpu_victim_order(batch):
            if free_gpu >= demand:
                break
            victims.append(uid)
            free_gpu += len(self.users[uid].pages)
        if free_gpu < demand:
            raise CacheError("full", f"{demand} pages needed, {free_gpu} obtainable")

        self.clock += 1
        stamp = self.clock
        offload, onboard, dropped = [], [], []

        # offload the victims into the host tier, newest first
        gpu_freed = []
        for uid in self.offload_order(victims):
            v = self.users[uid]
            k = len(v.pages)
            gpu_freed += v.pages
            older = self.host_evictable(batch, uid)
            if len(self.free[HOST]) + sum(len(self.users[h].pages) for h in older) < k:
                del self.users[uid]
                dropped.append(uid)
                continue
            for h in older:
                if len(self.free[HOST]) >= k:
                    break
                self.give(HOST, self.users[h].pages)
                del self.users[h]
                dropped.append(h)
            hp = self.take(HOST, k)
            offload += list(zip(v.pages, hp))
            v.tier, v.pages = HOST, hp
        self.give(GPU, gpu_freed)

        # allocate the batch in batch order
        tier_before, cached = [], []
        host_to_free = []
        for uid, a, k in zip(ids, append, need):
            u = self.users.get(uid)
            if u is None:
                tier_before.append(MISS)
                u = User(GPU, 0, self.take(GPU, k), stamp)
                self.users[uid] = u
            elif u.tier == GPU:
                tier_before.append(GPU)
                u.pages = u.pages + self.take(GPU, k - len(u.pages))
            else:
                tier_before.append(HOST)
                fresh = self.take(GPU, k)
                onboard += list(zip(u.pages, fresh))
                host_to_free += u.pages
                u.tier, u.pages = GPU, fresh
            cached.append(u.n)
            u.n += a
            u.stamp = stamp
        self.give(HOST, host_to_free)

        rows = [self.users[uid].pages + [-1] * (self.M - len(self.users[uid].pages)) for uid in ids]
        return {"tier_before": tier_before, "cached_lens": cached, "page_rows": rows,
                "offload": offload, "onboard": onboard, "dropped": dropped}

    def evict(self, uid: int) -> int:
        """Drop a user from whichever tier holds it; returns that tier (MISS if none)."""
        u = self.users.pop(int(uid), None)
        if u is None:
            return MISS
        self.give(u.tier, u.pages)
        return u.tier

    def compact(self) -> list:
        """Move the GPU residents' pages into [0, live); returns (from, to) pairs."""
        live = sorted(p for u in self.users.values() if u.tier == GPU for p in u.pages)
        n_live = len(live)
        srcs = [p for p in live if p >= n_live]
        dsts = [p for p in self.free[GPU] if p < n_live]
        assert len(srcs) == len(dsts)
        move = dict(zip(srcs, dsts))
        for u in self.users.values():
            if u.tier == GPU:
                u.pages = [move.get(p, p) for p in u.pages]
        self.free[GPU] = list(range(n_live, self.G))
        return list(zip(srcs, dsts))

    def page_rows(self, ids) -> list:
        """GPU page rows (padded with -1 to max_pages_per_user); all -1 for a user not on the GPU."""
        rows = []
        for uid in ids:
            u = self.users.get(int(uid))
            pages = u.pages if (u is not None and u.tier == GPU) else []
            rows.append(pages + [-1] * (self.M - len(pages)))
        return rows

    def stats(self) -> dict:
        return {"free_gpu": len(self.free[GPU]), "free_host": len(self.free[HOST]),
                "gpu_users": sum(u.tier == GPU for u in self.users.values()),
                "host_users": sum(u.tier == HOST for u in self.users.values()),
                "clock": self.clock}


def page_copy(src, dst, pairs):
    """The copy the pairs describe: dst[to] = src[from] for every (from, to), whole pages."""
    for s, d in pairs:
        dst[d] = src[s]
