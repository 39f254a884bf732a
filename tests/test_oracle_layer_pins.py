"""Pins of the HSTU layer oracle (oracle/hstu_layer.py) against facts other than itself.

* The projection step equals torch's float64 linear + SiLU (a library routine), up to the bf16
  rounding the layer applies.
* The split order is fixed by construction: with W_qkvu = [1*I; 2*I; 3*I; 4*I] (d_model = H*D),
  block b of h is SiLU((b + 1) x), so q, k, v, u are told apart by their scale.
* The output projection is checked element by element against a brute-force sum on a tiny case,
  which fixes its orientation (y = g W_out^T, W_out [d_model, H*D]).
* With W_out = I the layer equals the attention of its own q, k, v, u, rounded to bf16.
* Planted mistakes (split order swapped, SiLU dropped, u taken from the wrong block, the output
  projection transposed) each fail a pin.
"""
from __future__ import annotations

import inspect
import types

import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen
from oracle import hstu_layer as hl


def _case(seed, H=2, D=32, d_model=None, P=8):
    c = gen.paged_case([13, 0, 30], [4, 3, 5], [2, 1, 3], H=H, D=D, P=P, NB=16, n_max=64, num_pages=24, dtype="bf16",
                       seed=seed)
    d_model = d_model or 2 * H * D
    rng = np.random.default_rng(seed)
    x = hl.bf16_round(rng.standard_normal((c.Tn, d_model)))
    w1 = hl.bf16_round(rng.standard_normal((4 * H * D, d_model)) / np.sqrt(d_model))
    w2 = hl.bf16_round(rng.standard_normal((d_model, H * D)) / np.sqrt(H * D))
    return c, x, w1, w2


def pin_projection_matches_torch(mod):
    import torch
    import torch.nn.functional as F

    c, x, w1, _ = _case(1)
    parts = mod.qkvu(x, w1, c.H, c.D)
    ref = F.silu(F.linear(torch.from_numpy(x), torch.from_numpy(w1))).numpy()
    HD = c.H * c.D
    for b in range(4):
        want = ref[:, b * HD:(b + 1) * HD].reshape(-1, c.H, c.D)
        assert np.allclose(parts[b], want, rtol=2 ** -8, atol=1e-30)


def pin_split_order(mod):
    H, D = 2, 16
    HD = H * D
    rng = np.random.default_rng(2)
    x = hl.bf16_round(rng.standard_normal((7, HD)))
    w1 = np.concatenate([(b + 1) * np.eye(HD) for b in range(4)])
    parts = mod.qkvu(x, w1, H, D)
    for b in range(4):
        want = hl.bf16_round(x * (b + 1) / (1 + np.exp(-(b + 1) * x))).reshape(7, H, D)
        assert np.array_equal(parts[b], want), f"block {b} is not SiLU({b + 1} x)"


def pin_output_projection_brute_force(mod):
    c, x, w1, w2 = _case(3, d_model=24)
    y = mod.layer_paged(x, w1, w2, c.pool_k_full(), c.pool_v_full(), c.page_table, c.cached_lens, c.new_lens,
                        c.num_targets, c.rab, c.n_max)
    q, k, v, u = (hl.bf16_bits(t) for t in hl.qkvu(x, w1, c.H, c.D))
    g = hl.bf16_round(oracle.hstu_paged(q, k, v, u, c.pool_k_full(), c.pool_v_full(), c.page_table, c.cached_lens,
                                        c.new_lens, c.num_targets, c.rab, c.n_max)).reshape(c.Tn, -1)
    for t in range(c.Tn):
        for j in range(w2.shape[0]):
            s = 0.0
            for col in range(g.shape[1]):
                s += g[t, col] * w2[j, col]
            assert abs(y[t, j] - s) <= 1e-12 * (1 + abs(s))


def pin_identity_output_is_the_attention(mod):
    c, x, w1, _ = _case(4)
    HD = c.H * c.D
    x = x[:, :HD] if x.shape[1] >= HD else x
    w1 = w1[:, :HD]
    y = mod.layer_paged(x, w1, np.eye(HD), c.pool_k_full(), c.pool_v_full(), c.page_table, c.cached_lens, c.new_lens,
                        c.num_targets, c.rab, c.n_max)
    q, k, v, u = (hl.bf16_bits(t) for t in hl.qkvu(x, w1, c.H, c.D))
    att = oracle.hstu_paged(q, k, v, u, c.pool_k_full(), c.pool_v_full(), c.page_table, c.cached_lens, c.new_lens,
                            c.num_targets, c.rab, c.n_max)
    assert np.array_equal(y, hl.bf16_round(att).reshape(c.Tn, HD))


PINS = [pin_projection_matches_torch, pin_split_order, pin_output_projection_brute_force,
        pin_identity_output_is_the_attention]


@pytest.fixture(autouse=True)
def _full_pools(monkeypatch):
    # the oracle reads whole pools: expose the case's pages as full [num_pages, H, P, D] arrays
    def full(c, which):
        pool = np.zeros((c.num_pages, c.H, c.P, c.D), np.uint16)
        src = c.pool_k if which == "k" else c.pool_v
        if c.page_ids.shape[0]:
            pool[c.page_ids] = src
        return pool

    monkeypatch.setattr(gen.PagedCase, "pool_k_full", lambda c: full(c, "k"), raising=False)
    monkeypatch.setattr(gen.PagedCase, "pool_v_full", lambda c: full(c, "v"), raising=False)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(hl)


MUTATIONS = {
    "q and k swapped": ("    q, k, v, u = (bf16_bits(t) for t in qkvu(x_new, w_qkvu, H, D))",
                        "    k, q, v, u = (bf16_bits(t) for t in qkvu(x_new, w_qkvu, H, D))"),
    "SiLU dropped": ("    h = silu(np.asarray(x_new, np.float64) @ np.asarray(w_qkvu, np.float64).T)",
                     "    h = np.asarray(x_new, np.float64) @ np.asarray(w_qkvu, np.float64).T"),
    "u from the v block": ("    q, k, v, u = (bf16_bits(t) for t in qkvu(x_new, w_qkvu, H, D))",
                           "    q, k, v, u = (bf16_bits(t) for t in [qkvu(x_new, w_qkvu, H, D)[i] for i in (0, 1, 2, 2)])"),
    "blocks taken in reverse": ("    return [bf16_round(h[:, i * HD:(i + 1) * HD]).reshape(Tn, H, D) for i in range(4)]",
                                "    return [bf16_round(h[:, i * HD:(i + 1) * HD]).reshape(Tn, H, D) for i in range(3, -1, -1)]"),
    "output projection transposed": ("    return bf16_round(g).reshape(Tg, H * D) @ np.asarray(w_out, np.float64).T",
                                     "    return bf16_round(g).reshape(Tg, H * D) @ np.asarray(w_out, np.float64).reshape(-1, w_out.shape[0])"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(hl)
    assert src.count(old) == 1, f"mutation '{name}' does not match the oracle source exactly once"
    mod = types.ModuleType(f"layer_mutant_{abs(hash(name))}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name):
    mod = _mutant(name)
    for pin in PINS:
        try:
            pin(mod)
        except Exception:
            return
    raise AssertionError(f"planted mistake '{name}' passed every pin")
