"""The second (time-bucketed) bias on the GPU: jagged forward on the tensor-core path against the
dense float64 oracle with the same bias (oracle/time_bias.py)."""
from __future__ import annotations

import numpy as np
import pytest

from hstu_attention_b200 import inputs as gen
from oracle import time_bias as tb

from .helpers import assert_close, dev, host

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
