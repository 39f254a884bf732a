"""Pins for the float64 oracle: closed forms, library routines, brute force and invariants.

Each test ties the oracle to something other than itself, so that a plausible slip in it
(a dropped term, a sign, an off-by-one in the mask or the page index, a transposed operand,
the wrong LayerNorm axis) fails at least one of them.  No GPU is used here.

Sources for what is computed: SiLU weighting instead of softmax, a relative attention bias
and elementwise gating (aitrends.kr summary, section "HSTU의 순차 모델링"; news.bpdata.com,
section "HSTU"); jagged inputs and a paged KV cache holding the user's history with only the
new tokens computed (NVIDIA blog "Deploying an HSTU Generative Recommender with NVIDIA
Dynamo-Triton", sections on why serving is hard and on the benefits of the cache).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from hstu_attention_b200 import inputs as gen

# --------------------------------------------------------------------------- bucket table


def test_bucket_hand_values():
    # n_max = 68, NB = 32 (tiny workload):
    #   bucket(2)  = 1 + floor(31 * ln 2 / ln 68)  = 1 + floor(31 * 0.693147 / 4.219508) = 1 + 5 = 6
    #   bucket(67) = 1 + floor(31 * ln 67 / ln 68) = 1 + floor(30.891)                 = 31 (= NB-1)
    assert oracle.bucket(0, 68, 32) == 0
    assert oracle.bucket(1, 68, 32) == 1
    assert oracle.bucket(2, 68, 32) == 6
    assert oracle.bucket(67, 68, 32) == 31
    # n_max = 4096 = 2^12, NB = 128: ln(2^a) / ln(2^12) = a / 12
    #   bucket(2) = 1 + floor(127/12) = 11; bucket(8) = 1 + floor(127*3/12) = 32;
    #   bucket(64) = 1 + floor(63.5) = 64; bucket(4095) = 1 + floor(126.99..) = 127
    assert oracle.bucket(2, 4096, 128) == 11
    assert oracle.bucket(8, 4096, 128) == 32
    assert oracle.bucket(64, 4096, 128) == 64
    assert oracle.bucket(4095, 4096, 128) == 127
    # degenerate: a single bucket
    assert oracle.bucket(5, 4096, 1) == 0


@pytest.mark.parametrize("n_max,nb", [(68, 32), (4096, 128), (4176, 128), (16640, 256), (33312, 128)])
def test_bucket_table_shape(n_max, nb):
    t = oracle.bucket_table(n_max, n_max, nb)
    assert t[0] == 0 and t[1] == 1
    assert t.min() >= 0 and t.max() == nb - 1
    assert np.all(np.diff(t) >= 0)                      # monotone in distance
    # log spacing: the bucket of 2^a moves by (NB-1)/log2(n_max) per doubling (within 1)
    for a in range(1, int(math.log2(n_max))):
        expect = 1 + (nb - 1) * a / math.log2(n_max)
        assert abs(t[2 ** a] - expect) < 1.0 + 1e-9


def test_bucket_boundaries_not_razor_thin():
    """The GPU library computes its own table; a boundary flip between two correct log()
    implementations needs (NB-1)*ln(d)/ln(n_max) within rounding of an integer.  Check the
    named workloads keep every value at least 1e-9 away from an integer (d >= 2)."""
    for n_max, nb in [(68, 32), (4096, 128), (4176, 128), (16640, 256), (33312, 128)]:
        d = np.arange(2, n_max, dtype=np.float64)
        x = (nb - 1) * np.log(d) / math.log(n_max)
        frac = np.abs(x - np.round(x))
        # exact integers only where d is a power hitting a bucket edge exactly (n_max=4096)
        exact = frac < 1e-12
        assert np.all(frac[~exact] > 1e-9), (n_max, nb)
        # exact edges land on the same integer either way the rounding goes only if the
        # table treats them identically; list them so the GPU test can check those entries.
        if n_max == 4096:
            assert set(d[exact].astype(int)) <= {2 ** a for a in range(13)}


# --------------------------------------------------------------------------- helpers


def _jagged(lengths, targets, H=2, D=16, NB=8, n_max=None, seed=0, dtype="fp32", std=1.0):
    n_max = n_max or int(max(lengths))
    return gen.jagged_case(lengths, targets, H=H, D=D, NB=NB, n_max=n_max, dtype=dtype, seed=seed, std=std)


def _run_jagged(c, rows=None, return_o=False, nthreads=2):
    return oracle.hstu_jagged(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max,
                              c.eps, rows=rows, nthreads=nthreads, return_o=return_o)


def _silu(x):
    return x / (1.0 + np.exp(-x))


# --------------------------------------------------------------------------- closed forms


def test_single_key_sigmoid_direction():
    """One token, q = 0: s = rab[h][0].  With rab = +ln 3, sigmoid = 3/4; with -ln 3, 1/4.
    rab is stored in fp32, so ln 3 carries a relative rounding of ~3e-8: compare at 1e-7,
    far tighter than the factor 3 between sigmoid(s) and sigmoid(-s)."""
    c = _jagged([1], [0], H=2, D=4, NB=4, n_max=8)
    c.q[:] = 0.0
    c.rab[:] = 0.0
    c.rab[0, 0] = math.log(3.0)
    c.rab[1, 0] = -math.log(3.0)
    out, o = _run_jagged(c, return_o=True)
    v = c.v.astype(np.float64)
    w0 = math.log(3.0) * 0.75 / 8.0
    w1 = -math.log(3.0) * 0.25 / 8.0
    np.testing.assert_allclose(o[0, 0], w0 * v[0, 0], rtol=1e-7, atol=0)
    np.testing.assert_allclose(o[0, 1], w1 * v[0, 1], rtol=1e-7, atol=0)


def test_q_zero_one_hot_v_reads_weight_matrix():
    """Q = 0 and V[j,h,:] = e_j make o[i,h,j] = w(i,j) = allowed(i,j) * SiLU(rab[h][b(i-j)]) / n_max.
    This reads out the whole weight matrix, including the target-aware mask."""
    L, T, D = 12, 3, 16          # 9 history tokens, 3 candidates; D >= L
    c = _jagged([L], [T], H=2, D=D, NB=6, n_max=20, seed=3)
    c.q[:] = 0.0
    c.v[:] = 0.0
    for j in range(L):
        c.v[j, :, j] = 1.0
    _, o = _run_jagged(c, return_o=True)
    hist = L - T
    for h in range(2):
        for i in range(L):
            for j in range(D):
                if j >= L:
                    expect = 0.0
                else:
                    candidate_i = i >= hist
                    if j < hist:
                        ok = j <= i          # history keys: causal (candidates see all history)
                    else:
                        ok = (j == i)        # a candidate key is seen only by itself
                    b = 0 if i == j else min(5, 1 + math.floor(5 * math.log(max(i - j, 1)) / math.log(20)))
                    expect = _silu(float(c.rab[h, b])) / 20.0 if ok else 0.0
                    if candidate_i and j < hist:
                        assert ok
                assert o[i, h, j] == pytest.approx(expect, rel=1e-13, abs=1e-16), (h, i, j)


def test_k_zero_rab_zero_gives_zero():
    c = _jagged([7, 5], [2, 0], seed=4)
    c.k[:] = 0.0
    c.rab[:] = 0.0
    out, o = _run_jagged(c, return_o=True)
    assert np.all(o == 0.0)
    assert np.all(out == 0.0)


def test_layernorm_closed_form_one_hot():
    """q = 0 and rab = a at bucket 0, 0 elsewhere: every off-diagonal weight is SiLU(0) = 0,
    so o[i] = SiLU(a)/n_max * v[i].  With v[i] = e_k (one entry 1 over the whole H*D vector)
    LayerNorm over the H*D axis has the closed form below; per-head normalisation would
    give a different value on the other head."""
    H, D = 2, 8
    HD = H * D
    c = _jagged([3], [0], H=H, D=D, NB=4, n_max=10, seed=5)
    c.q[:] = 0.0
    c.rab[:] = 0.0
    a = 1.5
    c.rab[:, 0] = a
    c.v[:] = 0.0
    c.v[2, 0, 3] = 1.0                                        # token 2, head 0, channel 3
    out, o = _run_jagged(c, rows=[2], return_o=True)
    cval = _silu(a) / 10.0
    mean = cval / HD
    var = cval * cval * (HD - 1) / (HD * HD)
    rstd = 1.0 / math.sqrt(var + c.eps)
    u = c.u[2].astype(np.float64)
    expect = np.full((H, D), -mean * rstd) * u
    expect[0, 3] = (cval - mean) * rstd * u[0, 3]
    np.testing.assert_allclose(out[0], expect, rtol=1e-12, atol=1e-14)


def test_layernorm_unit_gate_moments():
    """With u = 1 each output row has mean 0 and biased variance var/(var + eps)."""
    c = _jagged([40, 17], [5, 3], H=4, D=8, seed=6)
    c.u[:] = 1.0
    out, o = _run_jagged(c, return_o=True)
    T = out.shape[0]
    flat = out.reshape(T, -1)
    of = o.reshape(T, -1)
    var = of.var(axis=1)
    np.testing.assert_allclose(flat.mean(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(flat.var(axis=1), var / (var + c.eps), rtol=1e-10)


# --------------------------------------------------------------------------- library routines


def _torch_reference(c):
    """The same operation from torch CPU library routines in float64: matmul, silu, tril,
    layer_norm.  The mask is built from set logic (history block lower-triangular,
    candidate block the identity), a different construction from the oracle's predicate."""
    outs = []
    off = c.seq_offsets
    for b in range(c.B):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        hist = L - int(c.num_targets[b])
        q = torch.from_numpy(gen.as_f32(c.q[s0:s1]).astype(np.float64)).permute(1, 0, 2)  # [H,L,D]
        k = torch.from_numpy(gen.as_f32(c.k[s0:s1]).astype(np.float64)).permute(1, 0, 2)
        v = torch.from_numpy(gen.as_f32(c.v[s0:s1]).astype(np.float64)).permute(1, 0, 2)
        u = torch.from_numpy(gen.as_f32(c.u[s0:s1]).astype(np.float64))                    # [L,H,D]
        idx = torch.arange(L)
        delta = (idx[:, None] - idx[None, :]).clamp(min=0)
        table = torch.from_numpy(oracle.bucket_table(max(L, 1), c.n_max, c.NB).astype(np.int64))
        bias = torch.from_numpy(c.rab.astype(np.float64))[:, table[delta]]                # [H,L,L]
        mask = torch.zeros(L, L, dtype=torch.bool)
        mask[:, :hist] = torch.tril(torch.ones(L, hist, dtype=torch.bool))
        mask[hist:, hist:] = torch.eye(L - hist, dtype=torch.bool)
        s = q @ k.transpose(1, 2) + bias
        w = torch.where(mask, torch.nn.functional.silu(s), torch.zeros_like(s)) / c.n_max
        o = (w @ v).permute(1, 0, 2).reshape(L, -1)
        y = torch.nn.functional.layer_norm(o, (o.shape[1],), eps=c.eps).reshape(L, c.H, c.D) * u
        outs.append(y.numpy())
    return np.concatenate(outs, axis=0)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_against_torch_library_routines(seed):
    rng = np.random.default_rng(100 + seed)
    B = 3
    lengths = rng.integers(1, 40, size=B)
    targets = [int(rng.integers(0, l + 1)) for l in lengths]
    c = _jagged(lengths, targets, H=3, D=8, NB=7, n_max=48, seed=seed)
    got = _run_jagged(c)
    ref = _torch_reference(c)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_against_torch_bf16_inputs():
    c = _jagged([33, 70], [8, 16], H=4, D=32, NB=16, n_max=90, seed=9, dtype="bf16", std=0.5)
    np.testing.assert_allclose(_run_jagged(c), _torch_reference(c), rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------- invariants


def test_jagged_batch_equals_per_user_runs():
    c = _jagged([9, 1, 0, 25, 4], [2, 1, 0, 6, 4], seed=11)
    full = _run_jagged(c)
    off = c.seq_offsets
    for b in range(c.B):
        s0, s1 = int(off[b]), int(off[b + 1])
        if s1 == s0:
            continue
        one = gen.JaggedCase(H=c.H, D=c.D, NB=c.NB, n_max=c.n_max, dtype=c.dtype,
                             seq_offsets=np.array([0, s1 - s0]), num_targets=c.num_targets[b:b + 1],
                             q=c.q[s0:s1], k=c.k[s0:s1], v=c.v[s0:s1], u=c.u[s0:s1], rab=c.rab)
        assert np.array_equal(_run_jagged(one), full[s0:s1])


def test_rows_subset_matches_full():
    c = _jagged([30, 11], [4, 2], seed=12)
    full = _run_jagged(c)
    rows = np.array([40, 0, 29, 31, 15])
    assert np.array_equal(_run_jagged(c, rows=rows), full[rows])


def _paged_case(seed=21, dtype="fp32", extra_pages=0):
    return gen.paged_case([37, 64, 5, 0], [3, 0, 2, 0], [4, 4, 1, 2], H=2, D=16, P=16, NB=8,
                          n_max=80, num_pages=40, dtype=dtype, seed=seed, std=1.0,
                          extra_pages=extra_pages)


def _full_pool(pc, fill=0.0):
    shape = (pc.num_pages, pc.H, pc.P, pc.D)
    if pc.pool_k.dtype == np.uint16:
        bits = np.uint16(gen.BF16_NAN_BITS) if isinstance(fill, float) and math.isnan(fill) else np.uint16(0)
        pk = np.full(shape, bits, dtype=np.uint16)
        pv = np.full(shape, bits, dtype=np.uint16)
    else:
        pk = np.full(shape, fill, dtype=np.float32)
        pv = np.full(shape, fill, dtype=np.float32)
    pk[pc.page_ids] = pc.pool_k
    pv[pc.page_ids] = pc.pool_v
    return pk, pv


def _run_paged(pc, pk, pv, pt=None, rows=None, return_o=False):
    return oracle.hstu_paged(pc.q_new, pc.k_new, pc.v_new, pc.u_new, pk, pv,
                             pc.page_table if pt is None else pt, pc.cached_lens, pc.new_lens,
                             pc.num_targets, pc.rab, pc.n_max, pc.eps, rows=rows, nthreads=2,
                             return_o=return_o)


def _concatenate(pc, pk, pv):
    """Build the jagged equivalent of a paged call by plain gathering (test-side numpy)."""
    ks, vs, qs, us, lens, tg = [], [], [], [], [], []
    no = pc.new_offsets
    for b in range(pc.B):
        C = int(pc.cached_lens[b])
        pos = np.arange(C)
        pages = pc.page_table[b, pos // pc.P]
        kc = pk[pages, :, pos % pc.P, :]                  # [C, H, D]
        vc = pv[pages, :, pos % pc.P, :]
        s0, s1 = int(no[b]), int(no[b + 1])
        ks.append(np.concatenate([kc, pc.k_new[s0:s1]]))
        vs.append(np.concatenate([vc, pc.v_new[s0:s1]]))
        filler = np.zeros((C,) + pc.q_new.shape[1:], dtype=pc.q_new.dtype)
        qs.append(np.concatenate([filler, pc.q_new[s0:s1]]))
        us.append(np.concatenate([filler, pc.u_new[s0:s1]]))
        lens.append(C + s1 - s0)
        tg.append(int(pc.num_targets[b]))
    cat = lambda xs: np.ascontiguousarray(np.concatenate(xs))  # noqa: E731
    jc = gen.JaggedCase(H=pc.H, D=pc.D, NB=pc.NB, n_max=pc.n_max, dtype=pc.dtype,
                        seq_offsets=np.concatenate([[0], np.cumsum(lens)]).astype(np.int64),
                        num_targets=np.array(tg), q=cat(qs), k=cat(ks), v=cat(vs), u=cat(us),
                        rab=pc.rab)
    rows = np.concatenate([jc.seq_offsets[b] + int(pc.cached_lens[b]) + np.arange(int(pc.new_lens[b]))
                           for b in range(pc.B)]).astype(np.int64)
    return jc, rows


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_paged_equals_full_recompute(dtype):
    """Invariant (a): the cache-hit result equals recomputing the concatenated sequence."""
    pc = _paged_case(dtype=dtype)
    pk, pv = _full_pool(pc)
    got = _run_paged(pc, pk, pv)
    jc, rows = _concatenate(pc, pk, pv)
    ref = _run_jagged(jc, rows=rows)
    assert np.array_equal(got, ref)


def test_paged_invariant_to_page_permutation():
    """Invariant (b): moving pages to other physical slots (table updated) changes nothing."""
    pc = _paged_case()
    pk, pv = _full_pool(pc)
    base = _run_paged(pc, pk, pv)
    perm = np.random.default_rng(5).permutation(pc.num_pages)   # new slot of old page p = perm[p]
    pk2 = np.empty_like(pk)
    pv2 = np.empty_like(pv)
    pk2[perm] = pk
    pv2[perm] = pv
    pt2 = np.where(pc.page_table >= 0, perm[np.clip(pc.page_table, 0, None)], -1).astype(np.int32)
    assert np.array_equal(_run_paged(pc, pk2, pv2, pt=pt2), base)


def test_paged_compact_pool_same_result():
    pc = _paged_case()
    pk, pv = _full_pool(pc)
    ck, cv, cpt = pc.compact_pool()
    assert np.array_equal(_run_paged(pc, ck, cv, pt=cpt), _run_paged(pc, pk, pv))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_masked_positions_contribute_exactly_zero_paged(dtype):
    """Invariant (e): NaN in every pool page the call may not read (unreferenced pages and
    the slots past each user's cached length) and spare page-table columns of -1 leave
    the output finite and bit-identical."""
    pc = _paged_case(dtype=dtype, extra_pages=2)
    pk, pv = _full_pool(pc, fill=0.0)
    clean = _run_paged(pc, pk, pv)
    pk_nan, pv_nan = _full_pool(pc, fill=float("nan"))
    for b in range(pc.B):        # tail slots past cached_len inside owned pages -> NaN too
        C = int(pc.cached_lens[b])
        for pos in range(C, int(np.sum(pc.page_table[b] >= 0)) * pc.P):
            page = pc.page_table[b, pos // pc.P]
            nanv = np.uint16(gen.BF16_NAN_BITS) if dtype == "bf16" else np.float32("nan")
            pk_nan[page, :, pos % pc.P, :] = nanv
            pv_nan[page, :, pos % pc.P, :] = nanv
    poisoned = _run_paged(pc, pk_nan, pv_nan)
    assert np.all(np.isfinite(poisoned))
    assert np.array_equal(poisoned, clean)


def test_masked_positions_contribute_exactly_zero_jagged():
    """Invariant (e) on the jagged layout: for history queries i < m, keys j >= m are in the
    future; for one candidate query, the other candidates' keys are masked.  NaN there
    must not reach those outputs."""
    c = _jagged([30], [6], seed=13)
    m = 12
    rows = np.arange(m)
    clean = _run_jagged(c, rows=rows)
    c.k[m:] = np.nan
    c.v[m:] = np.nan
    assert np.array_equal(_run_jagged(c, rows=rows), clean)
    c2 = _jagged([30], [6], seed=13)
    i = 26                                   # a candidate (history length 24)
    clean = _run_jagged(c2, rows=[i])
    for j in range(24, 30):
        if j != i:
            c2.k[j] = np.nan
            c2.v[j] = np.nan
    assert np.array_equal(_run_jagged(c2, rows=[i]), clean)


def test_candidates_do_not_see_each_other():
    """Changing one candidate's K/V changes only that candidate's own output row."""
    c = _jagged([20], [5], seed=14)
    base = _run_jagged(c)
    c.k[17] += 1.0
    c.v[17] += 1.0
    new = _run_jagged(c)
    changed = np.where(np.any(new != base, axis=(1, 2)))[0]
    assert list(changed) == [17]


def test_history_change_reaches_later_tokens_only():
    c = _jagged([20], [5], seed=15)
    base = _run_jagged(c)
    c.v[7] += 1.0
    new = _run_jagged(c)
    changed = np.where(np.any(new != base, axis=(1, 2)))[0]
    assert list(changed) == list(range(7, 20))      # history 7..14 causally, and all candidates


# --------------------------------------------------------------------------- append


def test_append_scatter_and_roundtrip():
    pc = _paged_case(seed=31)
    pk, pv = _full_pool(pc)
    pk0, pv0 = pk.copy(), pv.copy()
    no = pc.new_offsets
    skipped = oracle.kv_append(pk, pv, pc.page_table, pc.k_new, pc.v_new, pc.cached_lens, no,
                               pc.append_lens)
    assert skipped == 0
    touched = np.zeros(pk.shape[:1] + pk.shape[2:3], dtype=bool)   # [page, slot]
    for b in range(pc.B):
        for t in range(int(pc.append_lens[b])):
            pos = int(pc.cached_lens[b]) + t
            page = pc.page_table[b, pos // pc.P]
            slot = pos % pc.P
            touched[page, slot] = True
            assert np.array_equal(pk[page, :, slot, :], pc.k_new[no[b] + t])
            assert np.array_equal(pv[page, :, slot, :], pc.v_new[no[b] + t])
    # nothing else moved
    mask = ~touched[:, None, :, None] * np.ones_like(pk, dtype=bool)
    assert np.array_equal(pk[mask], pk0[mask]) and np.array_equal(pv[mask], pv0[mask])


def test_append_from_empty_then_paged_equals_jagged():
    """Pages filled by appending a user's whole history from cached_len 0, then a cache hit
    on the candidates, equals jagged prefill over history + candidates."""
    H, D, P = 2, 8, 4
    hist = [7, 12]
    cand = [3, 2]
    jc = _jagged([h + c for h, c in zip(hist, cand)], cand, H=H, D=D, NB=6, n_max=16, seed=41)
    ref = _run_jagged(jc)
    num_pages = 12
    perm = np.random.default_rng(0).permutation(num_pages).astype(np.int32)
    need = [(h + P - 1) // P for h in hist]
    pt = np.full((2, max(need)), -1, dtype=np.int32)
    pt[0, :need[0]] = perm[:need[0]]
    pt[1, :need[1]] = perm[need[0]:need[0] + need[1]]
    pk = np.zeros((num_pages, H, P, D), dtype=np.float32)
    pv = np.zeros_like(pk)
    hist_rows = np.concatenate([np.arange(jc.seq_offsets[b], jc.seq_offsets[b] + hist[b]) for b in range(2)])
    assert oracle.kv_append(pk, pv, pt, jc.k[hist_rows], jc.v[hist_rows], [0, 0],
                            [0, hist[0]], hist) == 0
    cand_rows = np.concatenate([np.arange(jc.seq_offsets[b] + hist[b], jc.seq_offsets[b + 1]) for b in range(2)])
    got = oracle.hstu_paged(jc.q[cand_rows], jc.k[cand_rows], jc.v[cand_rows], jc.u[cand_rows], pk, pv, pt,
                            hist, cand, cand, jc.rab, jc.n_max, jc.eps, nthreads=1)
    assert np.array_equal(got, ref[cand_rows])


def test_append_rejects_out_of_range_pages():
    pk = np.zeros((4, 1, 4, 8), dtype=np.float32)
    pv = np.zeros_like(pk)
    pt = np.array([[0, 9]], dtype=np.int32)          # logical page 1 -> invalid id 9
    kn = np.ones((6, 1, 8), dtype=np.float32)
    skipped = oracle.kv_append(pk, pv, pt, kn, kn, [0], [0], [6])
    assert skipped == 2                              # positions 4, 5
    assert np.all(pk[0] == 1.0) and np.all(pk[1:] == 0.0)
