"""Pins of the LayerNorm-gate variants (oracle/ln_variants.py) against facts other than itself.

* The base reading (whole H*D vector, no affine) equals the C oracle's own epilogue, which is pinned
  separately (an independent implementation of the same definition).
* Closed forms with eps = 0: a head vector c + b*e_k normalises to sqrt(D-1) at k and
  -1/sqrt(D-1) elsewhere, whatever c and b; a token whose o is constant gives out = beta * u.
* torch.nn.functional.layer_norm in float64 (a library routine): over [H*D] with weight/bias,
  and per head over [D] with that head's weight/bias, then times u.
* Invariances: per-head output is unchanged when one head is scaled and shifted; the whole-vector
  output is not (the heads share one mean), which separates the two axes.
* Planted mistakes (beta after the gate, gamma before the normalisation, unbiased variance, the
  wrong axis, eps outside the square root) each fail a pin.
"""
from __future__ import annotations

import inspect
import types

import numpy as np
import pytest

import oracle
from oracle import ln_variants as lv


def _rand(seed, T=5, H=3, D=32):
    rng = np.random.default_rng(seed)
    o = rng.standard_normal((T, H, D)) * rng.uniform(0.5, 3, (T, H, 1)) + rng.standard_normal((T, H, 1))
    u = rng.standard_normal((T, H, D))
    g = rng.uniform(0.5, 1.5, (H, D))
    b = rng.standard_normal((H, D)) * 0.3
    return o, u, g, b


def pin_base_matches_c_oracle(mod):
    # jagged case through the C oracle: its out is LN(o) * u over H*D, no affine
    rng = np.random.default_rng(5)
    T, H, D = 40, 2, 32
    q, k, v, u = (rng.standard_normal((T, H, D)).astype(np.float32) for _ in range(4))
    rab = (rng.standard_normal((H, 8)) * 0.3).astype(np.float32)
    out, o = oracle.hstu_jagged(q, k, v, u, np.array([0, 17, T]), np.array([2, 3]), rab, 64, 1e-5, return_o=True)
    got = mod.ln_gate(o, u.astype(np.float64), 1e-5)
    assert np.allclose(got, out, rtol=1e-12, atol=1e-12)


def pin_closed_form_one_hot_per_head(mod):
    T, H, D = 2, 3, 32
    o = np.zeros((T, H, D))
    rng = np.random.default_rng(6)
    ks = rng.integers(0, D, (T, H))
    for t in range(T):
        for h in range(H):
            o[t, h, :] = rng.uniform(-5, 5)
            o[t, h, ks[t, h]] += rng.uniform(1, 4) * rng.choice([-1, 1])
    got = mod.ln_gate(o, np.ones_like(o), 0.0, per_head=True)
    for t in range(T):
        for h in range(H):
            sign = np.sign(o[t, h, ks[t, h]] - o[t, h, (ks[t, h] + 1) % D])
            want = np.full(D, -1.0 / np.sqrt(D - 1)) * sign
            want[ks[t, h]] = np.sqrt(D - 1) * sign
            assert np.allclose(got[t, h], want, rtol=1e-12, atol=1e-12)


def pin_constant_token_gives_beta_times_u(mod):
    T, H, D = 3, 2, 32
    o = np.ones((T, H, D)) * np.arange(1, T + 1)[:, None, None]
    _, u, g, b = _rand(7, T, H, D)
    for per_head in (False, True):
        got = mod.ln_gate(o, u, 1e-5, per_head=per_head, gamma=g, beta=b)
        assert np.allclose(got, b[None] * u, rtol=0, atol=1e-15)


def pin_torch_layer_norm(mod):
    import torch
    import torch.nn.functional as F

    for seed in range(3):
        o, u, g, b = _rand(10 + seed)
        T, H, D = o.shape
        ot, ut = torch.from_numpy(o), torch.from_numpy(u)
        full = F.layer_norm(ot.reshape(T, H * D), [H * D], torch.from_numpy(g).reshape(-1),
                            torch.from_numpy(b).reshape(-1), 1e-5).reshape(T, H, D) * ut
        assert np.allclose(mod.ln_gate(o, u, 1e-5, gamma=g, beta=b), full.numpy(), rtol=1e-12, atol=1e-12)
        per = torch.stack([F.layer_norm(ot[:, h], [D], torch.from_numpy(g[h]), torch.from_numpy(b[h]), 1e-5)
                           for h in range(H)], 1) * ut
        assert np.allclose(mod.ln_gate(o, u, 1e-5, per_head=True, gamma=g, beta=b), per.numpy(),
                           rtol=1e-12, atol=1e-12)
        plain = F.layer_norm(ot.reshape(T, H * D), [H * D], eps=1e-3).reshape(T, H, D) * ut
        assert np.allclose(mod.ln_gate(o, u, 1e-3), plain.numpy(), rtol=1e-12, atol=1e-12)


def pin_axis_invariance(mod):
    o, u, g, b = _rand(20)
    o2 = o.copy()
    o2[:, 1] = 7.0 * o2[:, 1] - 3.0                  # one head scaled and shifted
    ph = mod.ln_gate(o, u, 0.0, per_head=True, gamma=g, beta=b)
    ph2 = mod.ln_gate(o2, u, 0.0, per_head=True, gamma=g, beta=b)
    assert np.allclose(ph, ph2, rtol=1e-10, atol=1e-10)
    full = mod.ln_gate(o, u, 0.0, gamma=g, beta=b)
    full2 = mod.ln_gate(o2, u, 0.0, gamma=g, beta=b)
    assert not np.allclose(full[:, 0], full2[:, 0], rtol=1e-6, atol=1e-6)


PINS = [pin_base_matches_c_oracle, pin_closed_form_one_hot_per_head, pin_constant_token_gives_beta_times_u,
        pin_torch_layer_norm, pin_axis_invariance]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(lv)


MUTATIONS = {
    "beta added after the gate": ("return (xhat * g[None] + b[None]) * u", "return xhat * g[None] * u + b[None]"),
    "gamma before the normalisation": ("return (xhat * g[None] + b[None]) * u",
                                       "return (((groups * g.reshape(groups.shape[1:]) if per_head else groups) - mean) "
                                       "/ np.sqrt(var + eps)).reshape(T, H, D) * u + b[None] * u"),
    "unbiased variance": ("var = ((groups - mean) ** 2).mean(axis=-1, keepdims=True)",
                          "var = ((groups - mean) ** 2).sum(axis=-1, keepdims=True) / (groups.shape[-1] - 1)"),
    "per-head flag ignored": ("    if per_head:\n        groups = o ", "    if False:\n        groups = o "),
    "normalised over heads instead of D": ("        groups = o                                     # [T, H, D]",
                                           "        groups = o.transpose(0, 2, 1)                  # [T, H, D]"),
    "eps outside the square root": ("np.sqrt(var + eps)", "(np.sqrt(var) + eps)"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(lv)
    assert src.count(old) == 1, f"mutation '{name}' does not match the oracle source exactly once"
    mod = types.ModuleType(f"ln_mutant_{abs(hash(name))}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name):
    mod = _mutant(name)
    failed = False
    for pin in PINS:
        try:
            pin(mod)
        except Exception:
            failed = True
            break
    assert failed, f"planted mistake '{name}' passed every pin"
