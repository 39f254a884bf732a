"""Pins of the time-bias oracle (oracle/time_bias.py) against facts other than itself.

* The bucket function on hand-computed values (bit lengths, the cap, d <= 0).
* Without the time bias it equals the pair-loop C oracle's forward (pinned separately).
* With equal timestamps every pair falls in time bucket 0, so the time bias is a constant shift of
  the position bias: it equals the C oracle run with rab + rab_time[:, 0].
* A brute-force Python loop over the pairs of a tiny case (scores, mask, SiLU weight, LayerNorm,
  gate) agrees with the dense form.
* Planted mistakes (the time difference reversed, the bucket one lower, the time bias left out)
  each fail a pin.
"""
from __future__ import annotations

import inspect
import math
import types

import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen
from oracle import time_bias as tb


def _case(seed, lengths=(23, 1, 40), targets=(3, 1, 5), H=2, D=32, NBT=12):
    c = gen.jagged_case(list(lengths), list(targets), H=H, D=D, NB=16, n_max=64, dtype="fp32", seed=seed, std=1.0)
    rng = np.random.default_rng(seed)
    ts = np.concatenate([np.cumsum(rng.integers(0, 500, n)) for n in lengths]).astype(np.int32)
    rabt = (rng.standard_normal((H, NBT)) * 0.5).astype(np.float32)
    return c, ts, rabt


def pin_bucket_values(mod):
    d = np.array([-5, 0, 1, 2, 3, 4, 7, 8, 1000, 1023, 1024, 2 ** 31 - 1])
    want = [0, 0, 1, 2, 2, 3, 3, 4, 10, 10, 11, 31]
    assert mod.time_bucket(d, 64).tolist() == want
    assert mod.time_bucket(d, 8).tolist() == [min(w, 7) for w in want]


def pin_no_time_bias_is_the_c_oracle(mod):
    c, _, _ = _case(1)
    ref = oracle.hstu_jagged(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    got = mod.jagged_fwd_dense(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))


def pin_equal_timestamps_shift_the_bias(mod):
    c, _, rabt = _case(2)
    ts = np.full(c.q.shape[0], 777, np.int32)
    got = mod.jagged_fwd_dense(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps,
                               rab_time=rabt, timestamps=ts)
    shifted = (c.rab.astype(np.float64) + rabt[:, :1].astype(np.float64)).astype(np.float32)
    ref = oracle.hstu_jagged(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, shifted, c.n_max, c.eps)
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))


def pin_brute_force_pairs(mod):
    c, ts, rabt = _case(3, lengths=(9, 6), targets=(2, 1), H=2, D=8, NBT=6)
    got = mod.jagged_fwd_dense(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps,
                               rab_time=rabt, timestamps=ts)
    H, D = c.H, c.D
    q, k, v, u = (np.asarray(x, np.float64) for x in (c.q, c.k, c.v, c.u))
    for b in range(len(c.seq_offsets) - 1):
        s0, s1 = int(c.seq_offsets[b]), int(c.seq_offsets[b + 1])
        L, hist = s1 - s0, s1 - s0 - int(c.num_targets[b])
        for i in range(L):
            o = np.zeros((H, D))
            for h in range(H):
                for j in range(L):
                    if not ((j <= i and j < hist) or j == i):
                        continue
                    dt = int(ts[s0 + i]) - int(ts[s0 + j])
                    tbk = 0 if dt <= 0 else min(rabt.shape[1] - 1, dt.bit_length())
                    s = float(q[s0 + i, h] @ k[s0 + j, h]) + float(c.rab[h, oracle.bucket(i - j, c.n_max, c.rab.shape[1])]) \
                        + float(rabt[h, tbk])
                    w = s / (1.0 + math.exp(-s)) / c.n_max
                    o[h] += w * v[s0 + j, h]
            x = o.reshape(-1)
            xh = (x - x.mean()) / math.sqrt(((x - x.mean()) ** 2).mean() + c.eps)
            want = xh.reshape(H, D) * u[s0 + i]
            assert np.max(np.abs(got[s0 + i] - want)) <= 1e-9 * (1 + np.max(np.abs(want))), (b, i)


PINS = [pin_bucket_values, pin_no_time_bias_is_the_c_oracle, pin_equal_timestamps_shift_the_bias, pin_brute_force_pairs]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(tb)


MUTATIONS = {
    "time difference reversed": ("tidx = time_bucket(ts[:, None] - ts[None, :]", "tidx = time_bucket(ts[None, :] - ts[:, None]"),
    "bucket one lower": ("    return np.minimum(bits, nbt - 1)", "    return np.minimum(np.maximum(bits - 1, 0), nbt - 1)"),
    "time bias left out": ("                S = S + np.asarray(rab_time, dtype=np.float64)[h][tidx]", "                S = S"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(tb)
    assert src.count(old) == 1, f"mutation '{name}' does not match the oracle source exactly once"
    mod = types.ModuleType(f"tb_mutant_{abs(hash(name))}")
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
