"""Pins of the oracle's backward pass (oracle_hstu_jagged_bwd) against things other than itself:
central finite differences of the forward oracle, closed forms and invariants."""
import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen


def _case(seed=3, lengths=(9, 6, 1), targets=(3, 2, 1), H=2, D=4, NB=8, n_max=16):
    return gen.jagged_case(list(lengths), list(targets), H=H, D=D, NB=NB, n_max=n_max, dtype="fp32", seed=seed,
                           std=1.0)


def _loss(c, dout, q=None, k=None, v=None, u=None, rab=None):
    out = oracle.hstu_jagged(c.q if q is None else q, c.k if k is None else k, c.v if v is None else v,
                             c.u if u is None else u, c.seq_offsets, c.num_targets, c.rab if rab is None else rab,
                             c.n_max, nthreads=1)
    return float(np.sum(out * dout.astype(np.float64)))


def _fd(c, dout, name, idx, h=2e-3):
    """Central difference of sum(dout * out) with respect to one fp32 input element."""
    base = getattr(c, name).copy()
    plus, minus = base.copy(), base.copy()
    plus[idx] = np.float32(base[idx] + h)
    minus[idx] = np.float32(base[idx] - h)
    step = float(plus[idx]) - float(minus[idx])
    return (_loss(c, dout, **{name: plus}) - _loss(c, dout, **{name: minus})) / step


@pytest.mark.parametrize("seed", [3, 4])
def test_gradients_match_finite_differences(seed):
    c = _case(seed=seed)
    rng = np.random.default_rng(100 + seed)
    dout = rng.standard_normal(c.q.shape).astype(np.float32)
    dq, dk, dv, du, drab = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab,
                                                  c.n_max)
    grads = {"q": dq, "k": dk, "v": dv, "u": du, "rab": drab}
    for name, g in grads.items():
        flat = [tuple(ix) for ix in np.ndindex(g.shape)]
        picks = [flat[i] for i in rng.choice(len(flat), size=min(12, len(flat)), replace=False)]
        for ix in picks:
            fd = _fd(c, dout, name, ix)
            assert abs(fd - g[ix]) <= 2e-4 * max(1.0, abs(fd)), (name, ix, fd, g[ix])


def test_zero_upstream_gives_zero_gradients():
    c = _case()
    dout = np.zeros_like(c.q)
    for g in oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max):
        assert not np.any(g)


def test_zero_gate_blocks_attention_gradients():
    """u = 0: out does not depend on q, k, v or rab, and du = LayerNorm(o) * dout exactly."""
    c = _case()
    rng = np.random.default_rng(7)
    dout = rng.standard_normal(c.q.shape).astype(np.float32)
    zero_u = np.zeros_like(c.u)
    dq, dk, dv, du, drab = oracle.hstu_jagged_bwd(c.q, c.k, c.v, zero_u, dout, c.seq_offsets, c.num_targets,
                                                  c.rab, c.n_max)
    assert not np.any(dq) and not np.any(dk) and not np.any(dv) and not np.any(drab)
    # with u = 1 the forward output is LayerNorm(o) itself
    ones = np.ones_like(c.u)
    ln = oracle.hstu_jagged(c.q, c.k, c.v, ones, c.seq_offsets, c.num_targets, c.rab, c.n_max)
    np.testing.assert_allclose(du, ln * dout.astype(np.float64), rtol=1e-12, atol=1e-14)


def test_batch_equals_per_user_runs():
    """Users do not interact: the batched backward equals the per-user ones (bit-equal)."""
    c = _case()
    rng = np.random.default_rng(8)
    dout = rng.standard_normal(c.q.shape).astype(np.float32)
    full = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max)
    off = c.seq_offsets
    drab_sum = np.zeros_like(full[4])
    for b in range(c.B):
        s0, s1 = int(off[b]), int(off[b + 1])
        part = oracle.hstu_jagged_bwd(c.q[s0:s1], c.k[s0:s1], c.v[s0:s1], c.u[s0:s1], dout[s0:s1], [0, s1 - s0],
                                      c.num_targets[b:b + 1], c.rab, c.n_max)
        for g_full, g_part in zip(full[:4], part[:4]):
            assert np.array_equal(g_full[s0:s1], g_part)
        drab_sum += part[4]
    np.testing.assert_allclose(full[4], drab_sum, rtol=1e-12, atol=1e-15)


def test_candidates_only_reach_themselves():
    """A candidate's key and value receive gradient only from the candidate's own query."""
    c = _case(lengths=(8,), targets=(3,))
    rng = np.random.default_rng(9)
    dout = rng.standard_normal(c.q.shape).astype(np.float32)
    j = 6                                   # a candidate (history length 5)
    only = np.zeros_like(dout)
    only[j] = dout[j]
    g_all = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max)
    g_own = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, only, c.seq_offsets, c.num_targets, c.rab, c.n_max)
    np.testing.assert_allclose(g_all[1][j], g_own[1][j], rtol=1e-12, atol=1e-15)   # dk
    np.testing.assert_allclose(g_all[2][j], g_own[2][j], rtol=1e-12, atol=1e-15)   # dv


@pytest.mark.parametrize("seed,dtype", [(31, "fp32"), (32, "bf16"), (33, "bf16")])
def test_dense_backward_equals_the_pair_loop_oracle(seed, dtype):
    """oracle/dense_bwd.py (whole per-user matrices, library matmuls) restates the same backward as
    the C oracle's pair loops, which finite differences pin; the two must agree to float64
    rounding on ragged batches with candidates, including a single-token user."""
    from oracle.dense_bwd import jagged_bwd_dense

    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(1, 90, 3)] + [1]
    targets = [min(int(rng.integers(0, 6)), n) for n in lengths]
    c = gen.jagged_case(lengths, targets, H=2, D=32, NB=16, n_max=128, dtype=dtype, seed=seed, std=1.0)
    g = rng.standard_normal(c.q.shape).astype(np.float32)
    dout = gen.f32_to_bf16_bits(g) if dtype == "bf16" else g
    ref = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    got = jagged_bwd_dense(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    for name, a, b in zip(("dq", "dk", "dv", "du", "drab"), got, ref):
        scale = float(np.max(np.abs(b))) + 1e-30
        assert np.max(np.abs(a - b)) <= 1e-10 * scale, name
