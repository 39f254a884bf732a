"""KV cache management on the GPU: page copies (onboard, offload, compaction) bit-exact against
the oracle's copy, and a serving loop through the cache whose attention outputs match the oracle's
full recompute of every user's whole sequence.

The cache (NVIDIA blog "Deploying an HSTU Generative Recommender with NVIDIA Dynamo-Triton",
section "Why serving large sequential recommenders is hard"): a paged GPU KV table with lookup,
allocate, append, evict and LRU-like eviction, a host tier, onboard and offload.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen
from oracle import kv_cache as kc

from .helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import hstu_attention_b200 as hb

    hb.load()
    return hb


def _pool(rng, pages, H, P, D, dtype, pinned=False):
    import torch

    x = gen._values(rng, (pages, H, P, D), 1.0, dtype)
    t = torch.from_numpy(x.view(np.int16) if dtype == "bf16" else x)
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.pin_memory() if pinned else t.cuda()


def _bits(t):
    return host(t).copy()


@pytest.mark.parametrize("dtype,H,P,D", [("bf16", 4, 32, 128), ("fp32", 2, 16, 32), ("bf16", 8, 64, 128)])
def test_page_copy_bit_exact(hb, dtype, H, P, D):
    import torch

    rng = np.random.default_rng(11)
    G, Hp = 48, 40
    p = hb.params(H, D, dtype, 32, 1024, page_size=P, num_pages=G, max_pages_per_user=8)
    ws = hb.Workspace(p, 1, 1, 1)
    gk, gv = _pool(rng, G, H, P, D, dtype), _pool(rng, G, H, P, D, dtype)
    hk, hv = _pool(rng, Hp, H, P, D, dtype, pinned=True), _pool(rng, Hp, H, P, D, dtype, pinned=True)
    ref = {n: _bits(t) for n, t in (("gk", gk), ("gv", gv), ("hk", hk), ("hv", hv))}

    def pairs(n, src_n, dst_n):
        return np.stack([rng.choice(src_n, n, replace=False), rng.choice(dst_n, n, replace=False)], 1).astype(np.int32)

    # offload (GPU -> pinned host), pairs in device memory
    off = pairs(17, G, Hp)
    hb.kv_page_copy(p, gk, gv, hk, hv, dev(off), workspace=ws)
    kc.page_copy(ref["gk"], ref["hk"], off.tolist())
    kc.page_copy(ref["gv"], ref["hv"], off.tolist())
    # onboard (pinned host -> GPU), pairs in pinned host memory
    on = pairs(23, Hp, G)
    hb.kv_page_copy(p, hk, hv, gk, gv, torch.from_numpy(on).pin_memory(), workspace=ws)
    kc.page_copy(ref["hk"], ref["gk"], on.tolist())
    kc.page_copy(ref["hv"], ref["gv"], on.tolist())
    # compaction-style move within the GPU pool: disjoint sources and destinations
    ids = rng.permutation(G)
    mv = np.stack([ids[:20], ids[20:40]], 1).astype(np.int32)
    hb.kv_page_copy(p, gk, gv, gk, gv, dev(mv), workspace=ws)
    kc.page_copy(ref["gk"], ref["gk"], mv.tolist())
    kc.page_copy(ref["gv"], ref["gv"], mv.tolist())
    torch.cuda.synchronize()
    assert ws.status() == 0
    for n, t in (("gk", gk), ("gv", gv), ("hk", hk), ("hv", hv)):
        assert np.array_equal(_bits(t), ref[n]), f"{n} differs from the oracle's copy"


def test_page_copy_flags_bad_pages_and_copies_the_rest(hb):
    import torch

    rng = np.random.default_rng(12)
    H, P, D, G = 2, 16, 64, 16
    p = hb.params(H, D, "bf16", 32, 1024, page_size=P, num_pages=G, max_pages_per_user=4)
    ws = hb.Workspace(p, 1, 1, 1)
    k, v = _pool(rng, G, H, P, D, "bf16"), _pool(rng, G, H, P, D, "bf16")
    dk, dv = _pool(rng, 8, H, P, D, "bf16"), _pool(rng, 8, H, P, D, "bf16")
    ref_k, ref_v = _bits(dk), _bits(dv)
    pairs = np.array([[3, 0], [G, 1], [-1, 2], [5, 8], [7, 4]], np.int32)
    hb.kv_page_copy(p, k, v, dk, dv, dev(pairs), workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == hb.DEV_BAD_PAGE
    good = [(3, 0), (7, 4)]
    kc.page_copy(_bits(k), ref_k, good)
    kc.page_copy(_bits(v), ref_v, good)
    assert np.array_equal(_bits(dk), ref_k) and np.array_equal(_bits(dv), ref_v)


def test_page_copy_rejects_memory_the_device_cannot_address(hb):
    import ctypes

    import torch

    H, P, D = 2, 16, 64
    p = hb.params(H, D, "bf16", 32, 1024, page_size=P, num_pages=4, max_pages_per_user=4)
    ws = hb.Workspace(p, 1, 1, 1)
    g = torch.zeros(4, H, P, D, dtype=torch.bfloat16, device="cuda")
    pageable = np.zeros((4, H, P, D), np.uint16)          # ordinary host memory, never registered
    pairs = dev(np.array([[0, 1]], np.int32))
    lib = hb.load()
    rc = lib.hstu_kv_page_copy(ctypes.byref(p), pageable.ctypes.data, pageable.ctypes.data, 4, g.data_ptr(),
                               g.data_ptr(), 4, pairs.data_ptr(), 1, ws.ptr, ws.nbytes,
                               torch.cuda.current_stream().cuda_stream)
    assert rc == -1
    # a pool shorter than the page count it claims (the far end falls outside the allocation)
    small = torch.zeros(1, H, P, D, dtype=torch.bfloat16).pin_memory()
    rc = lib.hstu_kv_page_copy(ctypes.byref(p), small.data_ptr(), small.data_ptr(), 1 << 20, g.data_ptr(),
                               g.data_ptr(), 4, pairs.data_ptr(), 1, ws.ptr, ws.nbytes,
                               torch.cuda.current_stream().cuda_stream)
    assert rc == -1
    with pytest.raises(hb.HstuError):
        hb.kv_page_copy(p, torch.zeros(4, H, P, D, dtype=torch.bfloat16), g, g, g, pairs, workspace=ws)
    torch.cuda.synchronize()


class Users:
    """Each user's token stream (history positions 0, 1, ...): q, k, v, u rows drawn once, seeded."""

    def __init__(self, rng, n_users, max_hist, H, D):
        self.ids = [int(x) for x in rng.choice(1 << 40, n_users, replace=False)]
        self.stream = {uid: [gen._values(rng, (max_hist, H, D), 0.5, "bf16") for _ in range(4)] for uid in self.ids}
        self.length = {uid: 0 for uid in self.ids}   # history the user has produced so far


def _serving_loop(hb, seed, steps, G, Hp, compact_every, evict_every):
    import torch

    rng = np.random.default_rng(seed)
    H, D, P, NB, n_max, M = 2, 128, 16, 32, 600, 24
    max_hist = M * P - 16
    users = Users(rng, 12, max_hist, H, D)
    rab = gen._values(rng, (H, NB), 0.3, "fp32").astype(np.float32)
    p = hb.params(H, D, "bf16", NB, n_max, page_size=P, num_pages=G, max_pages_per_user=M)
    cache = hb.KVCache(G, Hp, P, M)
    gk = torch.zeros(G, H, P, D, dtype=torch.bfloat16, device="cuda")
    gv = torch.zeros_like(gk)
    hk = torch.zeros(max(Hp, 1), H, P, D, dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    ws = hb.Workspace(p, 8, 8 * (max_hist + 16), max_hist + 16)
    d_rab = dev(rab)
    stats = {"miss": 0, "gpu": 0, "host": 0, "offload": 0, "onboard": 0, "moves": 0, "dropped": 0}
    for step in range(steps):
        if evict_every and step % evict_every == evict_every - 1:
            cache.evict(users.ids[int(rng.integers(len(users.ids)))])
        batch = [users.ids[i] for i in rng.choice(len(users.ids), int(rng.integers(1, 5)), replace=False)]
        tiers, stored = cache.lookup(batch)
        grow = {uid: int(rng.integers(1, 40)) for uid in batch}
        for uid in batch:
            grow[uid] = min(grow[uid], max_hist - users.length[uid])
        # a miss re-sends the user's whole history; a hit (either tier) only the new part
        append = [users.length[uid] + grow[uid] if t == hb.TIER_MISS else grow[uid] for uid, t in zip(batch, tiers)]
        for uid, t, n in zip(batch, tiers, stored):
            assert t == hb.TIER_MISS or n == users.length[uid], "the cache lost track of a stored length"
        try:
            r = cache.prepare(batch, append)
        except hb.CacheFull:
            continue
        assert r["cached_lens"].tolist() == [0 if t == hb.TIER_MISS else users.length[u] for u, t in zip(batch, tiers)]
        for key, name in ((hb.TIER_MISS, "miss"), (hb.TIER_GPU, "gpu"), (hb.TIER_HOST, "host")):
            stats[name] += int(np.sum(r["tier_before"] == key))
        stats["offload"] += len(r["offload"])
        stats["onboard"] += len(r["onboard"])
        stats["dropped"] += len(r["dropped"])
        # copies in the order the cache prescribes, then the append and the attention
        if len(r["offload"]):
            hb.kv_page_copy(p, gk, gv, hk, hv, dev(r["offload"]), workspace=ws)
        if len(r["onboard"]):
            hb.kv_page_copy(p, hk, hv, gk, gv, dev(r["onboard"]), workspace=ws)
        cands = {uid: int(rng.integers(1, 9)) for uid in batch}
        new_rows = {n: [] for n in "qkvu"}
        cand_rows = {}
        for b, uid in enumerate(batch):
            c0 = int(r["cached_lens"][b])
            end = users.length[uid] + grow[uid]
            cand_rows[uid] = [gen._values(rng, (cands[uid], H, D), 0.5, "bf16") for _ in range(4)]
            for i, n in enumerate("qkvu"):
                new_rows[n].append(users.stream[uid][i][c0:end])
                new_rows[n].append(cand_rows[uid][i])
        qn, kn, vn, un = (np.concatenate(new_rows[n]) for n in "qkvu")
        new_lens = np.array([append[b] + cands[uid] for b, uid in enumerate(batch)], np.int32)
        nt = np.array([cands[uid] for uid in batch], np.int32)
        t = dict(q=dev(qn), k=dev(kn), v=dev(vn), u=dev(un), pt=dev(r["page_rows"]), cl=dev(r["cached_lens"]),
                 nl=dev(new_lens), nt=dev(nt))
        out = hb.paged_fwd(p, t["q"], t["k"], t["v"], t["u"], gk, gv, t["pt"], t["cl"], t["nl"], t["nt"], d_rab,
                           max_new=int(new_lens.max()), workspace=ws)
        hb.kv_append(p, gk, gv, t["pt"], t["k"], t["v"], t["cl"], t["nl"], t["nt"], max_new=int(new_lens.max()),
                     workspace=ws)
        torch.cuda.synchronize()
        assert ws.status() == 0
        got = host(out)
        # oracle: every batch user's whole sequence (full history + candidates), recomputed
        row0 = 0
        for b, uid in enumerate(batch):
            c0 = int(r["cached_lens"][b])
            end = users.length[uid] + grow[uid]
            seq = [np.concatenate([users.stream[uid][i][:end], cand_rows[uid][i]]) for i in range(4)]
            L = end + cands[uid]
            ref = oracle.hstu_jagged(*seq, np.array([0, L], np.int64), np.array([cands[uid]], np.int64), rab, n_max)
            nrows = L - c0
            assert_close(got[row0:row0 + nrows], ref[c0:], "bf16", f"step {step} user {uid}")
            row0 += nrows
            users.length[uid] = end
        if compact_every and step % compact_every == compact_every - 1:
            mv = cache.compact()
            stats["moves"] += len(mv)
            if len(mv):
                hb.kv_page_copy(p, gk, gv, gk, gv, dev(mv), workspace=ws)
        # every user on the GPU holds exactly its stream in its pages, bit for bit
        torch.cuda.synchronize()
        tiers_all, lens_all = cache.lookup(users.ids)
        rows_all = cache.page_rows(users.ids)
        kb, vb = _bits(gk), _bits(gv)
        for uid, tier, n, row in zip(users.ids, tiers_all, lens_all, rows_all):
            if tier != hb.TIER_GPU:
                continue
            assert n == users.length[uid]
            pos = np.arange(n)
            kk = kb[row[pos // P], :, pos % P, :]
            vv = vb[row[pos // P], :, pos % P, :]
            assert np.array_equal(kk, users.stream[uid][1][:n]), f"step {step}: K pages of user {uid}"
            assert np.array_equal(vv, users.stream[uid][2][:n]), f"step {step}: V pages of user {uid}"
    cache.close()
    return stats


def test_serving_loop_through_the_cache(hb):
    stats = _serving_loop(hb, seed=21, steps=40, G=64, Hp=48, compact_every=7, evict_every=11)
    for key in ("miss", "gpu", "host", "offload", "onboard", "moves"):
        assert stats[key] > 0, f"the loop never exercised '{key}': {stats}"


def test_serving_loop_without_a_host_tier(hb):
    stats = _serving_loop(hb, seed=22, steps=25, G=56, Hp=0, compact_every=0, evict_every=0)
    assert stats["dropped"] > 0 and stats["host"] == 0


@pytest.mark.parametrize("nbytes", [16, 4096 + 7, 3 * 1024 * 1024 + 48, 41 * 1024 * 1024 + 5])
def test_host_copy_bit_exact(hb, nbytes):
    """hstu_host_copy moves pinned host bytes to the device and back, bit for bit, tails included."""
    import torch

    rng = np.random.default_rng(nbytes)
    src = torch.from_numpy(rng.integers(0, 256, nbytes, dtype=np.uint8)).pin_memory()
    mid = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    back = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    hb.host_copy(mid, src)
    hb.host_copy(back, mid)
    torch.cuda.synchronize()
    assert torch.equal(mid.cpu(), src) and torch.equal(back, src)
    with pytest.raises(hb.HstuError):
        hb.host_copy(mid[:16], torch.zeros(16, dtype=torch.uint8))   # pageable host memory
    with pytest.raises(hb.HstuError):
        hb.host_copy(mid[16:32], mid[8:24])                           # overlapping ranges (and misaligned)
