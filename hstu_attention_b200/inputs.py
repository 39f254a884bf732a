"""Seeded synthetic workloads for HSTU attention (jagged prefill, paged cache hit, append).

This module only draws random numbers and builds lengths, offsets and page tables.  It
holds none of the attention arithmetic, so both the CUDA library's tests/benchmark and the
float64 oracle can be fed from it without sharing any of the method's code.

Shapes follow the serving workload the HSTU deployment pages describe (NVIDIA blog
"Deploying an HSTU Generative Recommender with NVIDIA Dynamo-Triton", section "HSTU serving
latency benchmark": hidden size 512 over 4 heads, BF16 KV cache, long user histories,
up to about a hundred candidates, dynamic batch 8, 100% GPU KV-cache hit).  The KuaiRand-1K
data used there is not available here; these seeded tensors stand in for it.

Conventions
-----------
* Token rows are ``[tokens, H, D]`` with D contiguous.
* Pages are ``[num_pages, H, P, D]``; ``page_table[b, p]`` is the physical page holding
  logical positions ``p*P .. p*P+P-1`` of user b, ``-1`` where the user has no page.
* bf16 tensors are carried as ``uint16`` bit patterns (drawn in fp32, rounded once to
  nearest-even), so the GPU and the oracle see identical bytes.
* Random generator: NumPy PCG64, seed chosen by the caller (1000 + config number for the
  named workloads).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

# ----------------------------------------------------------------------------- bf16 bits


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


BF16_NAN_BITS = 0x7FC0


def _values(rng: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


def as_f32(x: np.ndarray) -> np.ndarray:
    """View a generated tensor as float32 values (bf16 bits are widened exactly)."""
    return bf16_bits_to_f32(x) if x.dtype == np.uint16 else np.asarray(x, dtype=np.float32)


# ----------------------------------------------------------------------------- cases


@dataclasses.dataclass
class JaggedCase:
    """Inputs of one jagged prefill call: every token of every user is a query."""

    H: int
    D: int
    NB: int
    n_max: int
    dtype: str                  # "bf16" or "fp32"
    seq_offsets: np.ndarray     # int64 [B+1]
    num_targets: np.ndarray     # int64 [B]
    q: np.ndarray               # [T, H, D]
    k: np.ndarray
    v: np.ndarray
    u: np.ndarray
    rab: np.ndarray             # float32 [H, NB]
    eps: float = 1e-5

    @property
    def B(self) -> int:
        return int(self.seq_offsets.shape[0] - 1)

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets)

    @property
    def max_seqlen(self) -> int:
        return int(self.lengths.max()) if self.B else 0


@dataclasses.dataclass
class PagedCase:
    """Inputs of one paged cache-hit call (plus the append of its new history tokens).

    The pool content of the cached history is given only for the pages in use:
    ``pool_k[i]`` / ``pool_v[i]`` hold physical page ``page_ids[i]``.  Pages that the user
    owns but whose positions are not yet cached (room for appends) are listed in
    ``page_table`` but have no content here.
    """

    H: int
    D: int
    P: int
    NB: int
    n_max: int
    dtype: str
    num_pages: int              # physical pool size
    page_table: np.ndarray      # int32 [B, max_pages], -1 = none
    cached_lens: np.ndarray     # int64 [B]
    new_lens: np.ndarray        # int64 [B]  (append + candidates)
    num_targets: np.ndarray     # int64 [B]  (candidates: the last num_targets new tokens)
    append_lens: np.ndarray     # int64 [B]  (new history tokens to write into pages)
    page_ids: np.ndarray        # int32 [n_used] physical ids holding cached history
    pool_k: np.ndarray          # [n_used, H, P, D]
    pool_v: np.ndarray
    q_new: np.ndarray           # [Tn, H, D]
    k_new: np.ndarray
    v_new: np.ndarray
    u_new: np.ndarray
    rab: np.ndarray             # float32 [H, NB]
    eps: float = 1e-5

    @property
    def B(self) -> int:
        return int(self.cached_lens.shape[0])

    @property
    def new_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.new_lens)]).astype(np.int64)

    @property
    def Tn(self) -> int:
        return int(self.new_lens.sum())

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def max_new(self) -> int:
        return int(self.new_lens.max()) if self.B else 0

    def compact_pool(self):
        """(pool_k, pool_v, page_table) with pages renumbered 0..n_used-1 (same content)."""
        remap = np.full(self.num_pages, -1, dtype=np.int64)
        remap[self.page_ids] = np.arange(self.page_ids.shape[0])
        pt = self.page_table.astype(np.int64)
        compact = np.where(pt >= 0, remap[np.clip(pt, 0, None)], -1).astype(np.int32)
        return self.pool_k, self.pool_v, compact


# ----------------------------------------------------------------------------- builders


def jagged_case(lengths, num_targets, H, D, NB, n_max, dtype="bf16", seed=0, std=0.5,
                rab_std=math.sqrt(0.1)) -> JaggedCase:
    rng = np.random.Generator(np.random.PCG64(seed))
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    q = _values(rng, (T, H, D), std, dtype)
    k = _values(rng, (T, H, D), std, dtype)
    v = _values(rng, (T, H, D), std, dtype)
    u = _values(rng, (T, H, D), std, dtype)
    rab = (rng.standard_normal((H, NB), dtype=np.float32) * np.float32(rab_std)).astype(np.float32)
    return JaggedCase(H=H, D=D, NB=NB, n_max=int(n_max), dtype=dtype, seq_offsets=off,
                      num_targets=np.asarray(num_targets, dtype=np.int64), q=q, k=k, v=v, u=u, rab=rab)


def paged_case(cached_lens, append_lens, num_targets, H, D, P, NB, n_max, num_pages, dtype="bf16",
               seed=0, std=0.5, rab_std=math.sqrt(0.1), page_perm: Optional[np.ndarray] = None,
               perm_start: int = 0, extra_pages: int = 0) -> PagedCase:
    """Build a cache-hit call.  Each user owns ceil((cached + append) / P) pages, dealt out
    as consecutive chunks of a seeded permutation of the pool (``page_perm`` if given,
    starting at ``perm_start``, so several layers can share one pool with disjoint pages).
    ``extra_pages`` adds that many spare columns of -1 to the page table."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cl = np.asarray(cached_lens, dtype=np.int64)
    al = np.asarray(append_lens, dtype=np.int64)
    nt = np.asarray(num_targets, dtype=np.int64)
    B = cl.shape[0]
    nl = al + nt
    need = [(int(c + a) + P - 1) // P for c, a in zip(cl, al)]
    max_pages = max(need + [1]) + extra_pages
    if page_perm is None:
        page_perm = rng.permutation(num_pages).astype(np.int32)
    if perm_start + sum(need) > page_perm.shape[0]:
        raise ValueError("page pool too small for this batch")
    pt = np.full((B, max_pages), -1, dtype=np.int32)
    used = []
    cur = perm_start
    for b in range(B):
        pages = page_perm[cur:cur + need[b]]
        cur += need[b]
        pt[b, :need[b]] = pages
        used.extend(pages[: (int(cl[b]) + P - 1) // P])   # pages holding cached positions
    page_ids = np.asarray(used, dtype=np.int32)
    pool_k = _values(rng, (page_ids.shape[0], H, P, D), std, dtype)
    pool_v = _values(rng, (page_ids.shape[0], H, P, D), std, dtype)
    Tn = int(nl.sum())
    q = _values(rng, (Tn, H, D), std, dtype)
    k = _values(rng, (Tn, H, D), std, dtype)
    v = _values(rng, (Tn, H, D), std, dtype)
    u = _values(rng, (Tn, H, D), std, dtype)
    rab = (rng.standard_normal((H, NB), dtype=np.float32) * np.float32(rab_std)).astype(np.float32)
    case = PagedCase(H=H, D=D, P=P, NB=NB, n_max=int(n_max), dtype=dtype, num_pages=int(num_pages),
                     page_table=pt, cached_lens=cl, new_lens=nl, num_targets=nt, append_lens=al,
                     page_ids=page_ids, pool_k=pool_k, pool_v=pool_v, q_new=q, k_new=k, v_new=v,
                     u_new=u, rab=rab)
    case.perm_end = cur  # type: ignore[attr-defined]
    return case


# ----------------------------------------------------------------------------- named workloads
#
# Config numbers follow the five workloads of the specification:
#   1 tiny fp32, 2 jagged prefill, 3 paged cache hit x 8 layers, 4 long history, 5 mixed.


def config1_tiny(seed: int = 1001):
    """Tiny fp32: 2 users, cached {37, 64}, 4 candidates each, H=2, D=32, P=16, pool 32
    (seeded permutation), 32 log-spaced buckets, n_max = 64 + 4 = 68, values ~N(0, 1)."""
    cached, cand = [37, 64], [4, 4]
    paged = paged_case(cached, [0, 0], cand, H=2, D=32, P=16, NB=32, n_max=68, num_pages=32,
                       dtype="fp32", seed=seed, std=1.0)
    return paged


def config2_prefill(seed: int = 1002) -> JaggedCase:
    """Jagged prefill: 8 users, lengths ~U[256, 4096], last 64 tokens are candidates, H=4,
    D=128, values ~N(0, 0.5^2), rab 128 buckets, n_max = 4096."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lengths = rng.integers(256, 4096, size=8, endpoint=True)
    return jagged_case(lengths, [64] * 8, H=4, D=128, NB=128, n_max=4096, dtype="bf16",
                       seed=seed + 7919, std=0.5)


CONFIG3 = dict(B=8, H=4, D=128, P=32, NB=128, n_max=4096 + 16 + 64, num_pages=65536, layers=8,
               append=16, targets=64, cmin=1024, cmax=4096)


def config3_paged_layers(seed: int = 1003, layers: int = 8) -> List[PagedCase]:
    """Paged cache hit, 8 layers: batch 8, cached ~U[1024, 4096], 16 appended + 64 candidates
    per user, H=4, D=128, P=32, 65,536-page pool shared by all layers, each layer's pages
    disjoint (one seeded permutation dealt out layer by layer)."""
    c = CONFIG3
    rng = np.random.Generator(np.random.PCG64(seed))
    cached = rng.integers(c["cmin"], c["cmax"], size=c["B"], endpoint=True)
    perm = rng.permutation(c["num_pages"]).astype(np.int32)
    out, start = [], 0
    for layer in range(layers):
        case = paged_case(cached, [c["append"]] * c["B"], [c["targets"]] * c["B"], H=c["H"], D=c["D"],
                          P=c["P"], NB=c["NB"], n_max=c["n_max"], num_pages=c["num_pages"],
                          dtype="bf16", seed=seed * 100 + layer, std=0.5, page_perm=perm,
                          perm_start=start)
        start = case.perm_end  # type: ignore[attr-defined]
        out.append(case)
    return out


def config4_long(seed: int = 1004) -> PagedCase:
    """Long-history cache hit: 32 users, cached ~U[8192, 16384], 256 candidates, no appends,
    H=8, D=128, P=64, 256 buckets, n_max = 16640, pool = exactly the pages needed."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cached = rng.integers(8192, 16384, size=32, endpoint=True)
    need = int(sum((int(c) + 63) // 64 for c in cached))
    return paged_case(cached, [0] * 32, [256] * 32, H=8, D=128, P=64, NB=256, n_max=16640,
                      num_pages=need, dtype="bf16", seed=seed + 7919, std=0.5)


CONFIG5 = dict(B=128, H=4, D=128, P=32, NB=128, n_max=32768 + 32 + 512, num_pages=262144)


def config5_mixed(seed: int = 1005):
    """Mixed serving batch: 128 users, history ~lognormal(ln 2000, 1) clipped to [64, 32768];
    the first 64 are cache hits (append 8..32 new tokens, paged attention), the last 64 are
    misses (jagged prefill of history + candidates, then append of the history into pages).
    Candidates ~U[16, 512].  H=4, D=128, P=32, 262,144-page pool.

    Returns (hits: PagedCase, misses: JaggedCase, miss_pages: PagedCase-like page table for
    the misses' appends, sharing the pool with the hits)."""
    c = CONFIG5
    rng = np.random.Generator(np.random.PCG64(seed))
    hist = np.clip(np.round(rng.lognormal(math.log(2000.0), 1.0, size=c["B"])), 64, 32768).astype(np.int64)
    cand = rng.integers(16, 512, size=c["B"], endpoint=True)
    appends = rng.integers(8, 32, size=64, endpoint=True)
    perm = rng.permutation(c["num_pages"]).astype(np.int32)
    hits = paged_case(hist[:64], appends, cand[:64], H=c["H"], D=c["D"], P=c["P"], NB=c["NB"],
                      n_max=c["n_max"], num_pages=c["num_pages"], dtype="bf16", seed=seed + 1,
                      std=0.5, page_perm=perm, perm_start=0)
    misses = jagged_case(hist[64:] + cand[64:], cand[64:], H=c["H"], D=c["D"], NB=c["NB"],
                         n_max=c["n_max"], dtype="bf16", seed=seed + 2, std=0.5)
    # Pages for the misses' history (cached_len 0, append = history length), disjoint from hits.
    start = hits.perm_end  # type: ignore[attr-defined]
    need = [(int(h) + c["P"] - 1) // c["P"] for h in hist[64:]]
    miss_pt = np.full((64, max(need)), -1, dtype=np.int32)
    for b in range(64):
        miss_pt[b, :need[b]] = perm[start:start + need[b]]
        start += need[b]
    return hits, misses, miss_pt, hist[64:].astype(np.int64)
