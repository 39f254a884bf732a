"""GPU parity: the CUDA library against the float64 oracle, through the C ABI.

Tolerances: bf16 inputs with fp32 accumulation must satisfy
max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3; the fp32 path <= 1e-4 * max|oracle|;
kv_append and page indexing are compared bit for bit.
"""
import math

import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen
from tests.helpers import (assert_close, dev, device_pool, gpu_jagged, gpu_paged, host, oracle_jagged,
                           oracle_paged, paged_params)

pytestmark = pytest.mark.gpu


# --------------------------------------------------------------------------- bucket table


@pytest.mark.parametrize("n_max,nb", [(68, 32), (4096, 128), (4176, 128), (16640, 256), (33312, 128), (20, 6)])
def test_bucket_table_matches_oracle(cuda_lib, n_max, nb):
    hb = cuda_lib
    import torch

    p = hb.params(2, 32, torch.float32, nb, n_max)
    got = hb.bucket_table(p, n_max).cpu().numpy()
    assert np.array_equal(got, oracle.bucket_table(n_max, n_max, nb))


# --------------------------------------------------------------------------- kv_append


def _append_check(hb, c: gen.PagedCase):
    """GPU append into a pool, compared byte for byte with the oracle's scatter."""
    import torch

    p = paged_params(hb, c)
    kp, vp = device_pool(c)
    ws = hb.Workspace(p, c.B, max(c.Tn, 1), max(c.max_new, 1))
    ref_k, ref_v = host(kp).copy(), host(vp).copy()
    skipped = oracle.kv_append(ref_k, ref_v, c.page_table, c.k_new, c.v_new, c.cached_lens, c.new_offsets,
                               c.new_lens - c.num_targets)
    assert skipped == 0
    hb.kv_append(p, kp, vp, dev(c.page_table), dev(c.k_new), dev(c.v_new), dev(c.cached_lens), dev(c.new_lens),
                 dev(c.num_targets), max_new=max(c.max_new, 1), workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert np.array_equal(host(kp).view(np.uint8), ref_k.view(np.uint8))
    assert np.array_equal(host(vp).view(np.uint8), ref_v.view(np.uint8))


def test_append_tiny_fp32_from_empty(cuda_lib):
    """The tiny fp32 workload's pages filled by appending each user's whole history."""
    c = gen.config1_tiny()
    rng = np.random.default_rng(5)
    k_hist = rng.standard_normal((101, 2, 32)).astype(np.float32)
    v_hist = rng.standard_normal((101, 2, 32)).astype(np.float32)
    fill = gen.PagedCase(H=2, D=32, P=16, NB=32, n_max=68, dtype="fp32", num_pages=32, page_table=c.page_table,
                         cached_lens=np.array([0, 0]), new_lens=np.array([37, 64]), num_targets=np.array([0, 0]),
                         append_lens=np.array([37, 64]), page_ids=np.zeros(0, np.int32),
                         pool_k=np.zeros((0, 2, 16, 32), np.float32), pool_v=np.zeros((0, 2, 16, 32), np.float32),
                         q_new=k_hist, k_new=k_hist, v_new=v_hist, u_new=v_hist, rab=c.rab)
    _append_check(cuda_lib, fill)


@pytest.mark.parametrize("P", [8, 16, 32, 64])
def test_append_bf16_ragged(cuda_lib, P):
    c = gen.paged_case([0, 5, 37, 64, 200, 1], [0, 3, 40, 1, 17, 70], [0, 2, 0, 3, 5, 1], H=4, D=128, P=P, NB=16,
                       n_max=512, num_pages=400, dtype="bf16", seed=P)
    _append_check(cuda_lib, c)


def test_append_flags_bad_pages(cuda_lib):
    hb = cuda_lib
    import torch

    c = gen.paged_case([3, 10], [20, 4], [1, 1], H=2, D=64, P=8, NB=8, n_max=64, num_pages=12, dtype="bf16", seed=3)
    pt = c.page_table.copy()
    pt[0, 2] = 999                     # logical page 2 of user 0 (positions 16..23) is invalid
    p = paged_params(hb, c)
    kp, vp = device_pool(c)
    before = host(kp).copy()
    ws = hb.Workspace(p, c.B, c.Tn, c.max_new)
    hb.kv_append(p, kp, vp, dev(pt), dev(c.k_new), dev(c.v_new), dev(c.cached_lens), dev(c.new_lens),
                 dev(c.num_targets), max_new=c.max_new, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() & hb.DEV_BAD_PAGE
    ref_k, ref_v = before.copy(), before.copy()
    assert oracle.kv_append(ref_k, ref_v, pt, c.k_new, c.v_new, c.cached_lens, c.new_offsets,
                            c.new_lens - c.num_targets) > 0
    assert np.array_equal(host(kp).view(np.uint8), ref_k.view(np.uint8))   # valid tokens written, bad skipped


# --------------------------------------------------------------------------- tiny fp32 workload


def test_tiny_fp32_paged(cuda_lib):
    c = gen.config1_tiny()
    o, ws, _, _ = gpu_paged(cuda_lib, c)
    assert ws.status() == 0
    assert_close(host(o), oracle_paged(c), "fp32", "tiny paged")


def test_tiny_fp32_jagged(cuda_lib):
    """The tiny workload as jagged prefill: history {37, 64} plus 4 candidates each."""
    jc = gen.jagged_case([41, 68], [4, 4], H=2, D=32, NB=32, n_max=68, dtype="fp32", seed=1001, std=1.0)
    o, ws, _ = gpu_jagged(cuda_lib, jc)
    assert ws.status() == 0
    assert_close(host(o), oracle_jagged(jc), "fp32", "tiny jagged")


def test_tiny_fp32_paged_equals_jagged_recompute(cuda_lib):
    """Invariant (a) at fp32 on the GPU."""
    from tests.test_oracle_pins import _concatenate, _full_pool

    c = gen.config1_tiny()
    paged = host(gpu_paged(cuda_lib, c)[0])
    pk, pv = _full_pool(c)
    jc, rows = _concatenate(c, pk, pv)
    jag = host(gpu_jagged(cuda_lib, jc)[0])
    assert_close(paged, jag[rows].astype(np.float64), "fp32", "tiny paged vs jagged")


# --------------------------------------------------------------------------- bf16 jagged (tensor cores)


JAGGED_CASES = {
    "ragged_tiles": ([1, 127, 128, 129, 300, 700], [1, 0, 64, 64, 3, 100]),
    "all_candidates": ([5, 130], [5, 130]),
    "no_candidates": ([255, 256, 257], [0, 0, 0]),
    "with_empty_users": ([0, 40, 0, 513, 0], [0, 7, 0, 64, 0]),
}


@pytest.mark.parametrize("name", sorted(JAGGED_CASES))
def test_jagged_bf16(cuda_lib, name):
    lengths, targets = JAGGED_CASES[name]
    c = gen.jagged_case(lengths, targets, H=4, D=128, NB=128, n_max=1024, dtype="bf16", seed=hash(name) % 1000)
    o, ws, _ = gpu_jagged(cuda_lib, c)
    assert ws.status() == 0
    assert_close(host(o), oracle_jagged(c), "bf16", name)


@pytest.mark.parametrize("D", [32, 64])
def test_jagged_bf16_small_head_dims(cuda_lib, D):
    c = gen.jagged_case([50, 200, 3], [10, 64, 1], H=2, D=D, NB=32, n_max=256, dtype="bf16", seed=D)
    o, ws, _ = gpu_jagged(cuda_lib, c)
    assert_close(host(o), oracle_jagged(c), "bf16", f"D={D}")


def test_jagged_batch_equals_per_user_runs(cuda_lib):
    """Invariant (c): each CTA's work depends only on its own user, so a batch run is
    bit-identical to running the users one at a time."""
    lengths, targets = [200, 129, 64], [20, 1, 64]
    c = gen.jagged_case(lengths, targets, H=4, D=128, NB=128, n_max=512, dtype="bf16", seed=8)
    full = host(gpu_jagged(cuda_lib, c, max_seqlen=512)[0])
    off = c.seq_offsets
    for b in range(c.B):
        s0, s1 = int(off[b]), int(off[b + 1])
        one = gen.JaggedCase(H=c.H, D=c.D, NB=c.NB, n_max=c.n_max, dtype=c.dtype, seq_offsets=np.array([0, s1 - s0]),
                             num_targets=c.num_targets[b:b + 1], q=c.q[s0:s1], k=c.k[s0:s1], v=c.v[s0:s1],
                             u=c.u[s0:s1], rab=c.rab)
        part = host(gpu_jagged(cuda_lib, one, max_seqlen=512)[0])
        assert np.array_equal(part, full[s0:s1]), b


def test_jagged_padding_rows_poisoned(cuda_lib):
    """Rows of the buffers past the last token hold NaN: outputs stay finite and unchanged."""
    import torch

    hb = cuda_lib
    c = gen.jagged_case([90, 33], [5, 2], H=4, D=128, NB=64, n_max=256, dtype="bf16", seed=12)
    ref = host(gpu_jagged(hb, c)[0])
    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max)
    T = c.T
    big = {}
    for name in "qkvu":
        arr = getattr(c, name)
        t = torch.full((T + 200, c.H, c.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        t[:T] = dev(arr)
        big[name] = t
    ws = hb.Workspace(p, c.B, T, 256)
    out = torch.empty((T, c.H, c.D), dtype=torch.bfloat16, device="cuda")
    hb.jagged_fwd(p, big["q"][:T], big["k"][:T], big["v"][:T], big["u"][:T], dev(c.seq_offsets),
                  dev(c.num_targets), dev(c.rab), max_seqlen=256, workspace=ws, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(host(out), ref)


# --------------------------------------------------------------------------- bf16 paged (tensor cores)


def _paged_small(P, seed, extra_pages=0):
    return gen.paged_case([0, 31, 129, 300, 1000, 77], [3, 16, 0, 16, 5, 16], [1, 64, 2, 64, 130, 4], H=4, D=128,
                          P=P, NB=128, n_max=1400, num_pages=300, dtype="bf16", seed=seed, extra_pages=extra_pages)


@pytest.mark.parametrize("P", [16, 32, 64, 128])
def test_paged_bf16(cuda_lib, P):
    c = _paged_small(P, seed=P)
    o, ws, _, _ = gpu_paged(cuda_lib, c)
    assert ws.status() == 0
    assert_close(host(o), oracle_paged(c), "bf16", f"P={P}")


def test_paged_bf16_small_head_dim(cuda_lib):
    c = gen.paged_case([40, 3], [5, 0], [8, 2], H=2, D=64, P=16, NB=32, n_max=128, num_pages=20, dtype="bf16", seed=4)
    o, ws, _, _ = gpu_paged(cuda_lib, c)
    assert_close(host(o), oracle_paged(c), "bf16", "paged D=64")


def test_paged_page_permutation_bit_identical(cuda_lib):
    """Invariant (b): moving pages to other physical slots leaves the output bit-identical."""
    import torch

    c = _paged_small(32, seed=77)
    o1, _, _, (kp, vp) = gpu_paged(cuda_lib, c)
    perm = np.random.default_rng(1).permutation(c.num_pages)
    permt = torch.from_numpy(perm).cuda()
    kp2 = torch.empty_like(kp)
    vp2 = torch.empty_like(vp)
    kp2[permt] = kp
    vp2[permt] = vp
    pt2 = np.where(c.page_table >= 0, perm[np.clip(c.page_table, 0, None)], -1).astype(np.int32)
    o2, _, _, _ = gpu_paged(cuda_lib, c, pool=(kp2, vp2), page_table=pt2)
    assert np.array_equal(host(o1), host(o2))


def test_paged_poisoned_pool_bit_identical(cuda_lib):
    """Invariant (e): NaN in every page the call must not read (unused pages, slots past each
    user's cached length, spare page-table columns) leaves the output finite and unchanged."""
    c = _paged_small(32, seed=78, extra_pages=2)
    clean = host(gpu_paged(cuda_lib, c)[0])
    poisoned = host(gpu_paged(cuda_lib, c, poison=True)[0])
    assert np.all(np.isfinite(gen.as_f32(poisoned)))
    assert np.array_equal(clean, poisoned)


def test_paged_equals_jagged_recompute(cuda_lib):
    """Invariant (a) on the GPU: the cache hit matches jagged prefill of the concatenation."""
    c = _paged_small(32, seed=79)
    paged = host(gpu_paged(cuda_lib, c)[0])
    from tests.test_oracle_pins import _concatenate, _full_pool

    pk, pv = _full_pool(c)
    jc, rows = _concatenate(c, pk, pv)
    jag = host(gpu_jagged(cuda_lib, jc, max_seqlen=int(jc.max_seqlen))[0])
    assert_close(paged, gen.as_f32(jag[rows]).astype(np.float64), "bf16", "paged vs jagged")


def test_paged_independent_of_append(cuda_lib):
    """The cache-hit result is the same whether or not the new history tokens were appended."""
    import torch

    hb = cuda_lib
    c = _paged_small(32, seed=80)
    o1, ws, p, (kp, vp) = gpu_paged(hb, c)
    hb.kv_append(p, kp, vp, dev(c.page_table), dev(c.k_new), dev(c.v_new), dev(c.cached_lens), dev(c.new_lens),
                 dev(c.num_targets), max_new=c.max_new, workspace=ws)
    torch.cuda.synchronize()
    o2, _, _, _ = gpu_paged(hb, c, pool=(kp, vp), ws=ws)
    assert np.array_equal(host(o1), host(o2))


# --------------------------------------------------------------------------- device-side errors


def test_device_flags_bad_page_and_lengths(cuda_lib):
    hb = cuda_lib
    c = _paged_small(32, seed=81)
    pt = c.page_table.copy()
    pt[4, 3] = c.num_pages + 5                      # user 4 reads an invalid page
    o, ws, _, _ = gpu_paged(hb, c, page_table=pt)
    assert ws.status() & hb.DEV_BAD_PAGE
    # over-long user: total length above n_max
    c2 = gen.paged_case([100], [0], [10], H=4, D=128, P=32, NB=16, n_max=64, num_pages=8, dtype="bf16", seed=2)
    o2, ws2, _, _ = gpu_paged(hb, c2)
    assert ws2.status() & hb.DEV_BAD_NMAX
    assert np.all(gen.as_f32(host(o2)) == 0.0)       # rows of a rejected user are zeros
    # num_targets larger than the sequence (jagged)
    jc = gen.jagged_case([10, 20], [11, 2], H=4, D=128, NB=16, n_max=64, dtype="bf16", seed=3)
    o3, ws3, _ = gpu_jagged(hb, jc)
    assert ws3.status() & hb.DEV_BAD_LENGTH
    ref = oracle.hstu_jagged(jc.q[10:], jc.k[10:], jc.v[10:], jc.u[10:], [0, 20], [2], jc.rab, 64)
    assert_close(host(o3)[10:], ref, "bf16", "valid user next to a rejected one")


def test_user_longer_than_the_host_bound_is_zeroed(cuda_lib):
    """A user longer than max_seqlen (jagged) or with more than max_new new tokens (paged) is
    rejected: BAD_LENGTH, and every one of its output rows is zero -- also the rows past the
    query blocks the host bound sized the grid for.  The other users are unaffected."""
    hb = cuda_lib
    jc = gen.jagged_case([60, 300, 45], [4, 64, 5], H=4, D=128, NB=64, n_max=512, dtype="bf16", seed=21)
    o, ws, _ = gpu_jagged(hb, jc, max_seqlen=129)          # user 1 (300 tokens) is over the bound
    assert ws.status() & hb.DEV_BAD_LENGTH
    out = gen.as_f32(host(o))
    assert np.all(out[60:360] == 0.0)
    for b in (0, 2):
        s0, s1 = int(jc.seq_offsets[b]), int(jc.seq_offsets[b + 1])
        ref = oracle.hstu_jagged(jc.q[s0:s1], jc.k[s0:s1], jc.v[s0:s1], jc.u[s0:s1], [0, s1 - s0],
                                 jc.num_targets[b:b + 1], jc.rab, jc.n_max)
        assert_close(host(o)[s0:s1], ref, "bf16", f"jagged user {b} next to a rejected one")
    # paged: user 1 has 300 new tokens against max_new = 129
    c = gen.paged_case([40, 100, 7], [0, 236, 3], [5, 64, 2], H=4, D=128, P=32, NB=64, n_max=512, num_pages=40,
                       dtype="bf16", seed=22)
    o2, ws2, _, _ = gpu_paged(hb, c, max_new=129)
    assert ws2.status() & hb.DEV_BAD_LENGTH
    out2 = gen.as_f32(host(o2))
    off = c.new_offsets
    assert np.all(out2[off[1]:off[2]] == 0.0)
    ref = oracle_paged(c)
    keep = np.r_[off[0]:off[1], off[2]:off[3]]
    assert_close(host(o2)[keep], ref[keep], "bf16", "paged users next to a rejected one")


def test_empty_calls_are_noops(cuda_lib):
    hb = cuda_lib
    import torch

    p = hb.params(4, 128, torch.bfloat16, 16, 64)
    ws = hb.Workspace(p, 1, 1, 1)
    z = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    off = torch.zeros(1, dtype=torch.int32, device="cuda")
    hb.jagged_fwd(p, z, z, z, z, off, None, torch.zeros((4, 16), device="cuda"), max_seqlen=0, workspace=ws, out=z)
    assert ws.status() == 0


# --------------------------------------------------------------------------- full-size workloads (sampled)


def _sample_rows(n, k, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n, size=min(k, n), replace=False).tolist())
    rows |= {0, n - 1}
    return np.array(sorted(rows), dtype=np.int64)


def test_prefill_full_size_sampled(cuda_lib):
    """Jagged prefill workload (8 users, lengths U[256,4096], 64 candidates, H=4, D=128)."""
    c = gen.config2_prefill()
    o, ws, _ = gpu_jagged(cuda_lib, c, max_seqlen=4096)
    assert ws.status() == 0
    # every user's first, last, first-candidate rows plus random ones
    rows = set(_sample_rows(c.T, 96, 2).tolist())
    for b in range(c.B):
        s0, s1 = int(c.seq_offsets[b]), int(c.seq_offsets[b + 1])
        rows |= {s0, s1 - 1, s1 - 64, s1 - 65, s0 + 127, s0 + 128}
    rows = np.array(sorted(rows), dtype=np.int64)
    assert_close(host(o)[rows], oracle_jagged(c, rows=rows), "bf16", "prefill sampled")


def test_paged_full_size_one_layer(cuda_lib):
    """Paged cache-hit workload, one layer (8 users, cached U[1024,4096], 16 + 64 new, P=32,
    65,536-page pool): every output row."""
    c = gen.config3_paged_layers(layers=1)[0]
    o, ws, _, _ = gpu_paged(cuda_lib, c)
    assert ws.status() == 0
    assert_close(host(o), oracle_paged(c), "bf16", "paged layer 0")


def test_long_history(cuda_lib):
    """Long-history cache hit (32 users, cached U[8192,16384], 256 candidates, H=8, P=64): every
    row of the shortest and of the longest user, plus rows sampled over the whole batch."""
    c = gen.config4_long()
    o, ws, _, _ = gpu_paged(cuda_lib, c)
    assert ws.status() == 0
    off = np.concatenate([[0], np.cumsum(c.new_lens)])
    rows = set(_sample_rows(c.Tn, 64, 4).tolist())
    for b in (int(np.argmin(c.cached_lens)), int(np.argmax(c.cached_lens))):
        rows |= set(range(int(off[b]), int(off[b + 1])))
    rows = np.array(sorted(rows), dtype=np.int64)
    assert_close(host(o)[rows], oracle_paged(c, rows=rows), "bf16", "long history")


def _pages_to_host(kp, vp, ids):
    """The listed physical pages of the pool, copied to the host (renumbered 0..len-1)."""
    import torch

    idx = torch.from_numpy(np.asarray(ids, dtype=np.int64)).cuda()
    return host(kp.index_select(0, idx)).copy(), host(vp.index_select(0, idx)).copy()


def _renumber(pt, ids):
    """Page table over the compact host copy made by _pages_to_host(ids)."""
    where = {int(x): i for i, x in enumerate(ids)}
    return np.vectorize(lambda x: where.get(int(x), -1))(pt).astype(np.int32)


def test_mixed_batch(cuda_lib):
    """Mixed serving batch.  Hits: append of their new history tokens (byte-exact over every page
    they touch) and paged attention (every output row).  Misses: jagged prefill (every row of the
    smaller half of the users, sampled rows of the rest), then the append of their history into
    pages (byte-exact over every page the misses own)."""
    import torch

    hb = cuda_lib
    hits, misses, miss_pt, miss_hist = gen.config5_mixed()
    p = paged_params(hb, hits)
    kp, vp = device_pool(hits)
    ws = hb.Workspace(p, max(hits.B, misses.B), max(hits.Tn, misses.T), int(misses.max_seqlen))
    hit_ids = np.unique(hits.page_table[hits.page_table >= 0])
    before_k, before_v = _pages_to_host(kp, vp, hit_ids)

    o_hit, _, _, _ = gpu_paged(hb, hits, pool=(kp, vp), ws=ws)
    assert ws.status() == 0
    assert_close(host(o_hit), oracle_paged(hits), "bf16", "mixed hits")

    hb.kv_append(p, kp, vp, dev(hits.page_table), dev(hits.k_new), dev(hits.v_new), dev(hits.cached_lens),
                 dev(hits.new_lens), dev(hits.num_targets), max_new=hits.max_new, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    got_k, got_v = _pages_to_host(kp, vp, hit_ids)
    cpt = _renumber(hits.page_table, hit_ids)
    assert oracle.kv_append(before_k, before_v, cpt, hits.k_new, hits.v_new, hits.cached_lens, hits.new_offsets,
                            hits.new_lens - hits.num_targets) == 0
    assert np.array_equal(got_k.view(np.uint8), before_k.view(np.uint8))
    assert np.array_equal(got_v.view(np.uint8), before_v.view(np.uint8))

    o_miss, _, _ = gpu_jagged(hb, misses, ws=ws, max_seqlen=int(misses.max_seqlen))
    assert ws.status() == 0
    lens = misses.lengths
    small = np.argsort(lens, kind="stable")[: misses.B // 2]
    rows = np.concatenate([np.arange(misses.seq_offsets[b], misses.seq_offsets[b + 1]) for b in sorted(small)])
    big = np.argsort(lens, kind="stable")[misses.B // 2:]
    for b in big:                                    # first, last, first candidate of each big user
        s0, s1 = int(misses.seq_offsets[b]), int(misses.seq_offsets[b + 1])
        rows = np.concatenate([rows, [s0, s0 + 127, s1 - int(misses.num_targets[b]), s1 - 1]])
    rows = np.unique(np.concatenate([rows, _sample_rows(misses.T, 64, 6)]))
    assert_close(host(o_miss)[rows], oracle_jagged(misses, rows=rows), "bf16", "mixed misses")

    # misses populate pages: append each miss's whole history (cached 0; candidates not appended)
    miss_ids = np.unique(miss_pt[miss_pt >= 0])
    assert not np.intersect1d(miss_ids, hit_ids).size
    mk, mv = _pages_to_host(kp, vp, miss_ids)
    pm = hb.params(4, 128, torch.bfloat16, 128, hits.n_max, page_size=32, num_pages=hits.num_pages,
                   max_pages_per_user=miss_pt.shape[1])
    zeros = np.zeros(misses.B, dtype=np.int32)
    hb.kv_append(pm, kp, vp, dev(miss_pt), dev(misses.k), dev(misses.v), dev(zeros), dev(misses.lengths),
                 dev(misses.num_targets), max_new=int(misses.max_seqlen), workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    got_k, got_v = _pages_to_host(kp, vp, miss_ids)
    assert oracle.kv_append(mk, mv, _renumber(miss_pt, miss_ids), misses.k, misses.v, zeros, misses.seq_offsets,
                            misses.lengths - misses.num_targets) == 0
    assert np.array_equal(got_k.view(np.uint8), mk.view(np.uint8))
    assert np.array_equal(got_v.view(np.uint8), mv.view(np.uint8))
    # the hits' pages were not touched by the misses' append
    again_k, _ = _pages_to_host(kp, vp, hit_ids)
    assert np.array_equal(again_k.view(np.uint8), before_k.view(np.uint8))


# --------------------------------------------------------------------------- launch overlap flag


def test_overlap_previous_flag_is_bit_identical(cuda_lib):
    """HSTU_FLAG_OVERLAP_PREVIOUS only changes when the kernel may start: back-to-back paged calls
    sharing one workspace (each call's set-up overlapping the previous call's LayerNorm kernel)
    give the same bytes as calls without the flag."""
    import torch

    hb = cuda_lib
    cases = [_paged_small(32, seed=s) for s in (101, 102, 103)]
    c0 = cases[0]
    pools = [device_pool(c) for c in cases]

    def run(flags):
        p = hb.params(c0.H, c0.D, c0.dtype, c0.NB, c0.n_max, page_size=c0.P, num_pages=c0.num_pages,
                      max_pages_per_user=c0.max_pages, ln_eps=c0.eps, flags=flags)
        ws = hb.Workspace(p, c0.B, max(c.Tn for c in cases), max(c.max_new for c in cases))
        outs = []
        for _ in range(2):
            for c, (kp, vp) in zip(cases, pools):
                outs.append(hb.paged_fwd(p, dev(c.q_new), dev(c.k_new), dev(c.v_new), dev(c.u_new), kp, vp,
                                         dev(c.page_table), dev(c.cached_lens), dev(c.new_lens), dev(c.num_targets),
                                         dev(c.rab), max_new=c.max_new, workspace=ws))
        torch.cuda.synchronize()
        assert ws.status() == 0
        return outs

    plain, overlapped = run(0), run(hb.FLAG_OVERLAP_PREVIOUS)
    for a, b in zip(plain, overlapped):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert_close(host(overlapped[0]), oracle_paged(cases[0]), "bf16", "overlapped call vs oracle")

    # jagged prefill calls back to back on one workspace
    jcs = [gen.jagged_case([300, 5, 129], [64, 1, 8], H=4, D=128, NB=128, n_max=512, dtype="bf16", seed=s)
           for s in (111, 112)]

    def run_j(flags):
        p = hb.params(4, 128, torch.bfloat16, 128, 512, flags=flags)
        ws = hb.Workspace(p, 3, max(c.T for c in jcs), 512)
        outs = [hb.jagged_fwd(p, dev(c.q), dev(c.k), dev(c.v), dev(c.u), dev(c.seq_offsets), dev(c.num_targets),
                              dev(c.rab), max_seqlen=512, workspace=ws) for _ in range(2) for c in jcs]
        torch.cuda.synchronize()
        assert ws.status() == 0
        return outs

    for a, b in zip(run_j(0), run_j(hb.FLAG_OVERLAP_PREVIOUS)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
