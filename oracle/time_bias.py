"""Jagged HSTU attention with a second, time-bucketed relative bias (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module; it shares no code with ``hstu_attention_b200``.

HSTU's input is a timestamp-sorted stream of items and actions, and its attention adds a relative
attention bias (aitrends.kr summary, section "HSTU의 순차 모델링"); the pages do not give the
bias's form.  The library's base bias depends on the position difference (hstu_oracle.c); this
module adds the reading of a time-based second bias:

    s_ij = q_i . k_j + rab[h][bucket(i - j)] + rab_time[h][tbucket(ts_i - ts_j)]
    tbucket(d) = 0 for d <= 0, else min(NBT - 1, bit length of d)

with everything else as in the base definition (mask, SiLU weight / n_max, LayerNorm over H*D,
gate u).  Written with dense per-user matrices and library matmuls in float64.  Pins:
tests/test_oracle_time_bias_pins.py.
"""
from __future__ import annotations

import numpy as np

import oracle


def time_bucket(d, nbt):
    """tbucket(d) elementwise for an integer array d: the bit length of d (0 for d <= 0), capped."""
    d = np.asarray(d, dtype=np.int64)
    bits = np.zeros_like(d)
    x = np.where(d > 0, d, 0)
    while np.any(x > 0):
        bits += (x > 0)
        x = x >> 1
    return np.minimum(bits, nbt - 1)


def _f64(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def jagged_fwd_dense(q, k, v, u, seq_offsets, num_targets, rab, n_max, eps=1e-5, rab_time=None, timestamps=None):
    """float64 out [T, H, D]; rab_time [H, NBT] and timestamps [T] add the time bias."""
    q, k, v, u = (_f64(x) for x in (q, k, v, u))
    rab = np.asarray(rab, dtype=np.float64)
    T, H, D = q.shape
    NB = rab.shape[1]
    off = np.asarray(seq_offsets, dtype=np.int64)
    nt = np.zeros(len(off) - 1, np.int64) if num_targets is None else np.asarray(num_targets, np.int64)
    out = np.zeros((T, H, D))
    Lmax = int(np.max(np.diff(off))) if len(off) > 1 else 0
    table = oracle.bucket_table(max(Lmax, 1), n_max, NB).astype(np.int64)
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L <= 0:
            continue
        hist = L - int(nt[b])
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        M = ((j <= i) & (j < hist)) | (j == i)
        bidx = table[np.clip(i - j, 0, None)]
        if rab_time is not None:
            ts = np.asarray(timestamps[s0:s1], dtype=np.int64)
            tidx = time_bucket(ts[:, None] - ts[None, :], np.asarray(rab_time).shape[1])
        O = np.zeros((L, H, D))
        for h in range(H):
            S = q[s0:s1, h] @ k[s0:s1, h].T + rab[h][bidx]
            if rab_time is not None:
                S = S + np.asarray(rab_time, dtype=np.float64)[h][tidx]
            P = np.where(M, S / (1.0 + np.exp(-S)) / n_max, 0.0)
            O[:, h] = P @ v[s0:s1, h]
        x = O.reshape(L, H * D)
        mean = x.mean(axis=1, keepdims=True)
        var = ((x - mean) ** 2).mean(axis=1, keepdims=True)
        out[s0:s1] = ((x - mean) / np.sqrt(var + eps)).reshape(L, H, D) * u[s0:s1]
    return out
