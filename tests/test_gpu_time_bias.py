"""The second (time-bucketed) bias on the GPU: jagged forward on the tensor-core path against the
dense float64 oracle with the same bias (oracle/time_bias.py)."""
from __future__ import annotations

import numpy as np
import pytest

from hstu_attention_b200 import inputs as gen
from oracle import time_bias as tb

from .helpers import assert_close, dev, device_pool, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import hstu_attention_b200 as hb

    hb.load()
    return hb


def _timestamps(rng, lengths, gap):
    return np.concatenate([1_000_000 + np.cumsum(rng.integers(0, gap, n)) for n in lengths]).astype(np.int32)


@pytest.mark.parametrize("lengths,targets,gap,nbt", [([300, 5, 129], [64, 1, 8], 5000, 24),
                                                     ([700, 256, 1], [16, 0, 1], 2, 8),
                                                     ([1000, 130], [64, 64], 1 << 20, 40)])
def test_time_bias_jagged(hb, lengths, targets, gap, nbt):
    import torch

    c = gen.jagged_case(lengths, targets, H=4, D=128, NB=64, n_max=1100, dtype="bf16", seed=len(lengths) * nbt)
    rng = np.random.default_rng(nbt)
    ts = _timestamps(rng, lengths, gap)
    rabt = (rng.standard_normal((c.H, nbt)) * 0.4).astype(np.float32)
    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, ln_eps=c.eps, rab_time=dev(rabt), timestamps=dev(ts))
    ws = hb.Workspace(p, c.B, c.T, c.max_seqlen)
    out = hb.jagged_fwd(p, dev(c.q), dev(c.k), dev(c.v), dev(c.u), dev(c.seq_offsets), dev(c.num_targets),
                        dev(c.rab), max_seqlen=c.max_seqlen, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = tb.jagged_fwd_dense(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps,
                              rab_time=rabt, timestamps=ts)
    assert_close(host(out), ref, "bf16", f"time bias gap={gap} nbt={nbt}")


def test_time_bias_is_rejected_where_it_is_not_implemented(hb):
    import torch

    c = gen.jagged_case([20], [2], H=2, D=64, NB=8, n_max=64, dtype="bf16", seed=3)
    ts = dev(np.arange(20, dtype=np.int32))
    rabt = torch.zeros((2, 4), device="cuda")
    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, rab_time=rabt, timestamps=ts)    # D = 64: CUDA-core path
    ws = hb.Workspace(p, 1, 20, 20)
    with pytest.raises(hb.HstuError):
        hb.jagged_fwd(p, dev(c.q), dev(c.k), dev(c.v), dev(c.u), dev(c.seq_offsets), dev(c.num_targets),
                      dev(c.rab), max_seqlen=20, workspace=ws)


def _full_sequence_rows(c, b, ck, cv, cpt):
    """User b's cached K and V in logical order (from the case's compact pool), [C, H, D] bits."""
    C = int(c.cached_lens[b])
    npg = (C + c.P - 1) // c.P
    pages = cpt[b, :npg]
    k = ck[pages].transpose(0, 2, 1, 3).reshape(npg * c.P, c.H, c.D)[:C]
    v = cv[pages].transpose(0, 2, 1, 3).reshape(npg * c.P, c.H, c.D)[:C]
    return k, v


@pytest.mark.parametrize("gap,nbt", [(3000, 24), (1, 6)])
def test_time_bias_paged(hb, gap, nbt):
    """Paged cache hit with the time bias = the jagged definition over each user's whole sequence
    (cached history + new tokens), read at the new rows: timestamps of cached tokens come from
    the timestamp pages, those of new tokens from the call."""
    import torch

    c = gen.paged_case([700, 37, 0, 1500], [16, 5, 3, 0], [64, 2, 1, 30], H=4, D=128, P=32, NB=64, n_max=1700,
                       num_pages=160, dtype="bf16", seed=gap + nbt)
    rng = np.random.default_rng(nbt)
    rabt = (rng.standard_normal((c.H, nbt)) * 0.4).astype(np.float32)
    ts_pages = np.zeros((c.num_pages, c.P), np.int32)
    ts_new = np.zeros(int(c.Tn), np.int32)
    ts_user = []
    off = 0
    for b in range(c.B):
        C, N = int(c.cached_lens[b]), int(c.new_lens[b])
        ts = (10_000 + np.cumsum(rng.integers(0, gap + 1, C + N))).astype(np.int32)
        ts_user.append(ts)
        for pos in range(C):
            ts_pages[c.page_table[b, pos // c.P], pos % c.P] = ts[pos]
        ts_new[off:off + N] = ts[C:]
        off += N
    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                  max_pages_per_user=c.max_pages, ln_eps=c.eps, rab_time=dev(rabt), timestamps=dev(ts_new),
                  ts_pages=dev(ts_pages))
    kp, vp = device_pool(c)
    ws = hb.Workspace(p, c.B, c.Tn, c.max_new)
    out = hb.paged_fwd(p, dev(c.q_new), dev(c.k_new), dev(c.v_new), dev(c.u_new), kp, vp, dev(c.page_table),
                       dev(c.cached_lens), dev(c.new_lens), dev(c.num_targets), dev(c.rab), max_new=c.max_new,
                       workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    got = host(out)
    ck, cv, cpt = c.compact_pool()
    off = 0
    for b in range(c.B):
        C, N = int(c.cached_lens[b]), int(c.new_lens[b])
        if N == 0:
            continue
        kc, vc = _full_sequence_rows(c, b, ck, cv, cpt)
        zeros = np.zeros((C, c.H, c.D), np.uint16)
        q = np.concatenate([zeros, c.q_new[off:off + N]])
        k = np.concatenate([kc, c.k_new[off:off + N]])
        v = np.concatenate([vc, c.v_new[off:off + N]])
        u = np.concatenate([zeros, c.u_new[off:off + N]])
        ref = tb.jagged_fwd_dense(q, k, v, u, [0, C + N], c.num_targets[b:b + 1], c.rab, c.n_max, c.eps,
                                  rab_time=rabt, timestamps=ts_user[b])
        assert_close(got[off:off + N], ref[C:], "bf16", f"paged time bias user {b}")
        off += N


def test_append_writes_timestamps_and_ts_pages_copy(hb):
    import torch

    c = gen.paged_case([5, 40, 0], [20, 3, 9], [2, 1, 0], H=2, D=64, P=16, NB=8, n_max=128, num_pages=24,
                       dtype="bf16", seed=5)
    rng = np.random.default_rng(6)
    ts_new = rng.integers(1, 1 << 30, int(c.Tn)).astype(np.int32)
    ts0 = rng.integers(-5, 5, (c.num_pages, c.P)).astype(np.int32)
    ts_pages = dev(ts0.copy())
    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                  max_pages_per_user=c.max_pages, timestamps=dev(ts_new), ts_pages=ts_pages)
    kp, vp = device_pool(c)
    ws = hb.Workspace(p, c.B, c.Tn, c.max_new)
    hb.kv_append(p, kp, vp, dev(c.page_table), dev(c.k_new), dev(c.v_new), dev(c.cached_lens), dev(c.new_lens),
                 dev(c.num_targets), max_new=c.max_new, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    want = ts0.copy()
    off = 0
    for b in range(c.B):
        C, N, T = int(c.cached_lens[b]), int(c.new_lens[b]), int(c.num_targets[b])
        for t in range(N - T):
            pos = C + t
            want[c.page_table[b, pos // c.P], pos % c.P] = ts_new[off + t]
        off += N
    assert np.array_equal(ts_pages.cpu().numpy(), want)
    # the timestamp side of onboard / offload / compaction moves, bit for bit
    host_ts = torch.zeros((10, c.P), dtype=torch.int32).pin_memory()
    pairs = np.array([[3, 0], [7, 9], [0, 4]], np.int32)
    hb.ts_page_copy(ts_pages, host_ts, dev(pairs), workspace=ws)
    back = torch.zeros_like(ts_pages)
    hb.ts_page_copy(host_ts, back, dev(pairs[:, ::-1].copy()), workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    h = host_ts.numpy()
    for s_, d_ in pairs:
        assert np.array_equal(h[d_], want[s_])
        assert np.array_equal(back.cpu().numpy()[s_], want[s_])
