"""One HSTU layer around the paged cache hit, in float64 (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module; it shares no code with ``hstu_attention_b200``.

What the pages fix (aitrends.kr summary, section "HSTU의 순차 모델링"; news.bpdata.com, section
"HSTU"): HSTU replaces softmax attention with SiLU weighting, adds a relative attention bias, and
gates elementwise before the output projection.  The projections themselves are not written out.
This module's reading, the plainest one that fits (no bias vectors, no residual, no input norm):

  h          = SiLU(x_new W_qkvu^T)                 x_new [Tn, d_model], W_qkvu [4*H*D, d_model]
  q, k, v, u = the four consecutive H*D-column blocks of h, in that order, each rounded to bf16
               (the layer hands bf16 tensors to the attention, as a bf16 model does)
  g          = LayerNorm(attention(q, k, v; cached pages)) * u      (oracle.hstu_paged)
  y          = bf16(g) W_out^T                      W_out [d_model, H*D]

k and v of the new history tokens are also what the layer appends to the user's pages.
Pins: tests/test_oracle_layer_pins.py.
"""
from __future__ import annotations

import numpy as np

import oracle


def bf16_round(x):
    """float64 -> nearest bf16 value (via float32; ties to even), returned as float64."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    b = f.view(np.uint32)
    r = ((b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)) << np.uint32(16)
    return r.view(np.float32).astype(np.float64)


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def bf16_bits(x):
    """float64 values that are exact bf16 numbers -> uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def qkvu(x_new, w_qkvu, H, D):
    """SiLU projection, split into q, k, v, u (float64 values of bf16 numbers, [Tn, H, D] each)."""
    h = silu(np.asarray(x_new, np.float64) @ np.asarray(w_qkvu, np.float64).T)
    Tn = h.shape[0]
    HD = H * D
    assert h.shape[1] == 4 * HD
    return [bf16_round(h[:, i * HD:(i + 1) * HD]).reshape(Tn, H, D) for i in range(4)]


def layer_paged(x_new, w_qkvu, w_out, k_pages, v_pages, page_table, cached_lens, new_lens, num_targets, rab,
                n_max, eps=1e-5, rows=None):
    """x_new [Tn, d_model] and weights as float64 values (bf16 numbers); pages as bf16 bits
    [num_pages, H, P, D].  Returns y [Tn, d_model] float64 (or the listed rows)."""
    H, D = k_pages.shape[1], k_pages.shape[3]
    q, k, v, u = (bf16_bits(t) for t in qkvu(x_new, w_qkvu, H, D))
    g = oracle.hstu_paged(q, k, v, u, k_pages, v_pages, page_table, cached_lens, new_lens, num_targets, rab,
                          n_max, eps, rows=rows)
    Tg = g.shape[0]
    return bf16_round(g).reshape(Tg, H * D) @ np.asarray(w_out, np.float64).T
