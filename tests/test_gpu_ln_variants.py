"""LayerNorm-gate variants on the GPU (per-head statistics, affine gamma/beta before the gate)
against the oracle's float64 epilogue applied to the oracle's own attention output o."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from hstu_attention_b200 import inputs as gen
from oracle import ln_variants as lv

from .helpers import assert_close, dev, device_pool, host

pytestmark = pytest.mark.gpu

VARIANTS = [(False, "gamma"), (False, "affine"), (True, None), (True, "affine")]


@pytest.fixture(scope="module")
def hb():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import hstu_attention_b200 as hb

    hb.load()
    return hb


def _affine(rng, H, D, kind):
    g = b = None
    if kind in ("gamma", "affine"):
        g = rng.uniform(0.5, 1.5, (H, D)).astype(np.float32)
    if kind == "affine":
        b = (rng.standard_normal((H, D)) * 0.2).astype(np.float32)
    return g, b


def _params(hb, c, per_head, g, b, paged=False):
    kw = dict(ln_eps=c.eps, ln_per_head=per_head, ln_weight=dev(g.reshape(-1)) if g is not None else None,
              ln_bias=dev(b.reshape(-1)) if b is not None else None)
    if paged:
        kw.update(page_size=c.P, num_pages=c.num_pages, max_pages_per_user=c.max_pages)
    return hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, **kw)


@pytest.mark.parametrize("per_head,affine", VARIANTS)
@pytest.mark.parametrize("dtype,H,D", [("bf16", 4, 128), ("bf16", 2, 64), ("fp32", 2, 32)])
def test_jagged_variants(hb, per_head, affine, dtype, H, D):
    import torch

    c = gen.jagged_case([300, 17, 129], [16, 1, 8], H=H, D=D, NB=32, n_max=512, dtype=dtype, seed=H * D,
                        std=1.0 if dtype == "fp32" else 0.5)
    rng = np.random.default_rng(D)
    g, b = _affine(rng, H, D, affine)
    p = _params(hb, c, per_head, g, b)
    ws = hb.Workspace(p, c.B, c.T, c.max_seqlen)
    out = hb.jagged_fwd(p, dev(c.q), dev(c.k), dev(c.v), dev(c.u), dev(c.seq_offsets), dev(c.num_targets),
                        dev(c.rab), max_seqlen=c.max_seqlen, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    _, o = oracle.hstu_jagged(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps,
                              return_o=True)
    ref = lv.ln_gate(o, gen.as_f32(c.u), c.eps, per_head=per_head, gamma=g, beta=b)
    assert_close(host(out), ref, dtype, f"jagged {dtype} per_head={per_head} {affine}")


@pytest.mark.parametrize("per_head,affine", VARIANTS)
def test_paged_variants_with_split_keys(hb, per_head, affine):
    import torch

    # long cached histories: the tensor-core paged path splits keys across CTAs (several planes)
    c = gen.paged_case([2000, 37, 900], [16, 3, 0], [64, 2, 8], H=4, D=128, P=32, NB=64, n_max=2100,
                       num_pages=128, dtype="bf16", seed=41)
    rng = np.random.default_rng(42)
    g, b = _affine(rng, c.H, c.D, affine)
    p = _params(hb, c, per_head, g, b, paged=True)
    kp, vp = device_pool(c)
    ws = hb.Workspace(p, c.B, c.Tn, c.max_new)
    out = hb.paged_fwd(p, dev(c.q_new), dev(c.k_new), dev(c.v_new), dev(c.u_new), kp, vp, dev(c.page_table),
                       dev(c.cached_lens), dev(c.new_lens), dev(c.num_targets), dev(c.rab), max_new=c.max_new,
                       workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ck, cv, cpt = c.compact_pool()
    _, o = oracle.hstu_paged(c.q_new, c.k_new, c.v_new, c.u_new, ck, cv, cpt, c.cached_lens, c.new_lens,
                             c.num_targets, c.rab, c.n_max, c.eps, return_o=True)
    ref = lv.ln_gate(o, gen.as_f32(c.u_new), c.eps, per_head=per_head, gamma=g, beta=b)
    assert_close(host(out), ref, "bf16", f"paged per_head={per_head} {affine}")


def test_backward_rejects_the_variants(hb):
    import torch

    c = gen.jagged_case([20], [2], H=2, D=64, NB=8, n_max=64, dtype="bf16", seed=3)
    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, ln_per_head=True)
    ws = hb.BwdWorkspace(p, c.T)
    with pytest.raises(hb.HstuError):
        hb.jagged_bwd(p, dev(c.q), dev(c.k), dev(c.v), dev(c.u), dev(c.seq_offsets), dev(c.num_targets),
                      dev(c.rab), dev(c.u), max_seqlen=c.max_seqlen, workspace=ws)
    torch.cuda.synchronize()
