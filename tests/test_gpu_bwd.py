"""Backward pass of jagged HSTU attention on the GPU against the float64 oracle backward."""
import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen
from tests.helpers import dev, host

pytestmark = pytest.mark.gpu


def _dout(c, seed):
    g = np.random.default_rng(seed).standard_normal(c.q.shape).astype(np.float32)
    return gen.f32_to_bf16_bits(g) if c.dtype == "bf16" else g


def _run(hb, c, dout, max_seqlen):
    import torch

    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, ln_eps=c.eps)
    ws = hb.BwdWorkspace(p, c.T)
    grads = hb.jagged_bwd(p, dev(c.q), dev(c.k), dev(c.v), dev(c.u), dev(c.seq_offsets), dev(c.num_targets),
                          dev(c.rab), dev(dout), max_seqlen=max_seqlen, workspace=ws)
    torch.cuda.synchronize()
    return [host(g).astype(np.float64) for g in grads], ws.status()


def _close(got, ref, rel, what):
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert np.all(np.isfinite(got)), what
    assert err <= rel * scale + 1e-6, f"{what}: max err {err:.3e} > {rel:.0e} * {scale:.3e}"


NAMES = ("dq", "dk", "dv", "du", "drab")


def test_bwd_fp32_tiny(cuda_lib):
    c = gen.jagged_case([41, 68, 1], [4, 4, 1], H=2, D=32, NB=32, n_max=68, dtype="fp32", seed=1001, std=1.0)
    dout = _dout(c, 5)
    got, status = _run(cuda_lib, c, dout, 128)
    assert status == 0
    ref = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    for name, g, r in zip(NAMES, got, ref):
        _close(g, r, 1e-3, f"fp32 {name}")


@pytest.mark.parametrize("D", [64, 128])
def test_bwd_bf16(cuda_lib, D):
    """D = 128 recomputes o on the tensor-core path, D = 64 on the CUDA-core path."""
    c = gen.jagged_case([300, 5, 129], [64, 1, 8], H=4, D=D, NB=128, n_max=512, dtype="bf16", seed=7 + D)
    dout = _dout(c, 6)
    got, status = _run(cuda_lib, c, dout, 512)
    assert status == 0
    ref = oracle.hstu_jagged_bwd(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    for name, g, r in zip(NAMES, got, ref):
        _close(g, r, 1e-2, f"bf16 D={D} {name}")


def test_bwd_rejected_user_has_zero_gradients(cuda_lib):
    hb = cuda_lib
    c = gen.jagged_case([10, 20], [11, 2], H=4, D=128, NB=16, n_max=64, dtype="bf16", seed=3)
    dout = _dout(c, 7)
    got, status = _run(hb, c, dout, 64)
    assert status & hb.DEV_BAD_LENGTH
    for g in got[:3]:
        assert not np.any(g[:10])                 # dq, dk, dv of the rejected user
    ref = oracle.hstu_jagged_bwd(c.q[10:], c.k[10:], c.v[10:], c.u[10:], dout[10:], [0, 20], [2], c.rab, 64, c.eps)
    for name, g, r in zip(NAMES[:4], got[:4], ref[:4]):
        _close(g[10:], r, 1e-2, f"valid user {name}")


def test_bwd_user_longer_than_max_seqlen(cuda_lib):
    """The forward rejects a user longer than max_seqlen (its o is zero); the backward must too:
    zero dq/dk/dv/du for that user and a drab that holds only the valid users' pairs."""
    hb = cuda_lib
    c = gen.jagged_case([60, 300, 45], [4, 64, 5], H=4, D=128, NB=64, n_max=512, dtype="bf16", seed=23)
    dout = _dout(c, 8)
    got, status = _run(hb, c, dout, 129)
    assert status & hb.DEV_BAD_LENGTH
    for g in got[:4]:
        assert not np.any(g[60:360])                  # dq, dk, dv, du of the rejected user
    keep = np.r_[0:60, 360:405]
    off = np.array([0, 60, 105])
    ref = oracle.hstu_jagged_bwd(c.q[keep], c.k[keep], c.v[keep], c.u[keep], dout[keep], off, c.num_targets[[0, 2]],
                                 c.rab, c.n_max, c.eps)
    for name, g, r in zip(NAMES[:4], got[:4], ref[:4]):
        _close(g[keep], r, 1e-2, f"valid users {name}")
    _close(got[4], ref[4], 1e-2, "drab of the valid users only")


def test_bwd_empty_batch_zeroes_drab(cuda_lib):
    import torch

    hb = cuda_lib
    p = hb.params(4, 128, torch.bfloat16, 16, 64)
    ws = hb.BwdWorkspace(p, 1)
    z = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    off = torch.zeros(1, dtype=torch.int32, device="cuda")
    rab = torch.zeros((4, 16), device="cuda")
    grads = hb.jagged_bwd(p, z, z, z, z, off, None, rab, z, max_seqlen=0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.all(grads[4] == 0) and ws.status() == 0


def test_bwd_full_prefill_batch(cuda_lib):
    """The prefill benchmark batch (8 users, lengths U[256, 4096], 64 candidates, H=4, D=128,
    NB=128) on the tensor-core backward, every row of dq/dk/dv/du and every drab bucket against
    the dense float64 oracle (oracle/dense_bwd.py, pinned against the pair-loop oracle)."""
    from oracle.dense_bwd import jagged_bwd_dense

    c = gen.config2_prefill()
    dout = _dout(c, 9)
    got, status = _run(cuda_lib, c, dout, int(c.max_seqlen))
    assert status == 0
    ref = jagged_bwd_dense(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
    for name, g, r in zip(NAMES, got, ref):
        _close(g, r, 1e-2, f"full prefill batch {name}")
