"""LayerNorm-gate epilogue with its variants, in float64 numpy (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module; it shares no code with ``hstu_attention_b200``.

HSTU gates elementwise before the output projection (aitrends.kr summary, section "HSTU의 순차
모델링"; news.bpdata.com, section "HSTU"); the pages fix neither the normalisation axis nor an
affine transform.  The library's base reading normalises a token's whole H*D vector with no
affine (oracle/hstu_oracle.c); the variants, a reading of this library as well:

  per_head = False:  mean, var (biased) over the token's H*D values of o
  per_head = True:   mean, var over each head's D values separately
  xhat = (o - mean) / sqrt(var + eps)
  out  = (xhat * gamma + beta) * u        gamma, beta: [H, D] (None = 1 and 0)

So gamma and beta act before the gate, as the affine part of the LayerNorm itself.  Pins:
tests/test_oracle_ln_pins.py.
"""
from __future__ import annotations

import numpy as np


def ln_gate(o, u, eps, per_head=False, gamma=None, beta=None):
    """o: [T, H, D] float64 (pre-LayerNorm attention output); u: [T, H, D]; returns float64 [T, H, D]."""
    o = np.asarray(o, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    T, H, D = o.shape
    if per_head:
        groups = o                                     # [T, H, D]: one group per (token, head)
    else:
        groups = o.reshape(T, 1, H * D)                # one group per token
    mean = groups.mean(axis=-1, keepdims=True)
    var = ((groups - mean) ** 2).mean(axis=-1, keepdims=True)
    xhat = ((groups - mean) / np.sqrt(var + eps)).reshape(T, H, D)
    g = np.ones((H, D)) if gamma is None else np.asarray(gamma, dtype=np.float64).reshape(H, D)
    b = np.zeros((H, D)) if beta is None else np.asarray(beta, dtype=np.float64).reshape(H, D)
    return (xhat * g[None] + b[None]) * u
