"""The backward pass of jagged HSTU attention with dense per-user matrices (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module; it shares no code with ``hstu_attention_b200``.

The same definition as ``oracle_hstu_jagged_bwd`` in hstu_oracle.c (the chain rule through the
forward: SiLU weighting with the relative attention bias, LayerNorm over each token's H*D vector,
the gate u; aitrends.kr summary, section "HSTU의 순차 모델링"; news.bpdata.com, section "HSTU"),
written with whole [L, L] matrices per user and head and library matmuls instead of pair loops, in
float64, so that a batch of thousands of tokens per user takes seconds instead of minutes:

  S    = Q K^T + rab[h][bucket(i - j)]        M = allowed(i, j)
  sig  = sigmoid(S),  P = M S sig / n_max,    O = P V
  out  = LayerNorm(O over H*D) * u            (forward, for the gradient through the norm)
  du   = xhat * dout;  do = rstd (dy - mean(dy) - xhat mean(dy xhat)),  dy = dout * u
  dP   = do V^T,  dS = M dP sig (1 + S (1 - sig)) / n_max
  dq   = dS K,  dk = dS^T Q,  dv = P^T do,  drab[h][b] = sum of dS over the pairs in bucket b

Pinned against the C oracle's backward (itself pinned by finite differences) in
tests/test_oracle_bwd_pins.py.
"""
from __future__ import annotations

import numpy as np

import oracle


def _f64(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def jagged_bwd_dense(q, k, v, u, dout, seq_offsets, num_targets, rab, n_max, eps=1e-5):
    """Returns float64 dq, dk, dv, du [T, H, D] and drab [H, NB]."""
    q, k, v, u, dout = (_f64(x) for x in (q, k, v, u, dout))
    rab = np.asarray(rab, dtype=np.float64)
    T, H, D = q.shape
    NB = rab.shape[1]
    off = np.asarray(seq_offsets, dtype=np.int64)
    nt = np.zeros(len(off) - 1, np.int64) if num_targets is None else np.asarray(num_targets, np.int64)
    dq, dk, dv, du = (np.zeros((T, H, D)) for _ in range(4))
    drab = np.zeros((H, NB))
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
        O = np.zeros((L, H, D))
        cache = []
        for h in range(H):
            S = q[s0:s1, h] @ k[s0:s1, h].T + rab[h][bidx]
            sig = 1.0 / (1.0 + np.exp(-S))
            P = np.where(M, S * sig / n_max, 0.0)
            O[:, h] = P @ v[s0:s1, h]
            cache.append((S, sig, P))
        x = O.reshape(L, H * D)
        mean = x.mean(axis=1, keepdims=True)
        var = ((x - mean) ** 2).mean(axis=1, keepdims=True)
        rstd = 1.0 / np.sqrt(var + eps)
        xhat = (x - mean) * rstd
        g = dout[s0:s1].reshape(L, H * D)
        du[s0:s1] = (xhat * g).reshape(L, H, D)
        dy = g * u[s0:s1].reshape(L, H * D)
        do = rstd * (dy - dy.mean(axis=1, keepdims=True) - xhat * (dy * xhat).mean(axis=1, keepdims=True))
        do = do.reshape(L, H, D)
        for h in range(H):
            S, sig, P = cache[h]
            dP = do[:, h] @ v[s0:s1, h].T
            dS = np.where(M, dP * sig * (1.0 + S * (1.0 - sig)) / n_max, 0.0)
            dq[s0:s1, h] = dS @ k[s0:s1, h]
            dk[s0:s1, h] = dS.T @ q[s0:s1, h]
            dv[s0:s1, h] = P.T @ do[:, h]
            drab[h] += np.bincount(bidx[M], weights=dS[M], minlength=NB)[:NB]
    return dq, dk, dv, du, drab
