"""The HSTU layer around the paged cache hit on the GPU (tensor-core projections, append, paged
attention, LayerNorm gate) against the float64 layer oracle (oracle/hstu_layer.py)."""
from __future__ import annotations

import numpy as np
import pytest

from hstu_attention_b200 import inputs as gen
from oracle import hstu_layer as hl

from .helpers import assert_close, dev, device_pool, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hb():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import hstu_attention_b200 as hb

    hb.load()
    return hb


def _f64(bits):
    return gen.as_f32(bits).astype(np.float64)


@pytest.mark.parametrize("M,N,K,act", [(300, 384, 512, 0), (300, 384, 512, 1), (1, 128, 64, 1), (640, 2048, 512, 1),
                                       (129, 512, 128, 0)])
def test_linear_matches_the_oracle(hb, M, N, K, act):
    import torch

    rng = np.random.default_rng(M + N + K)
    x = gen._values(rng, (M, K), 1.0, "bf16")
    w = gen._values(rng, (N, K), 1.0 / np.sqrt(K), "bf16")
    p = hb.params(1, 128, "bf16", 1, 1)
    ws = hb.Workspace(p, 1, 1, 1)
    y = hb.linear_fwd(dev(x), dev(w), activation=act, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = _f64(x) @ _f64(w).T
    if act:
        ref = hl.silu(ref)
    assert_close(host(y), ref, "bf16", f"linear {M}x{N}x{K} act={act}")


def _layer_case(seed, cached, append, targets, H=4, D=128, d_model=256, P=32, num_pages=None):
    need = sum(-(-(c + a) // P) for c, a in zip(cached, append))
    c = gen.paged_case(cached, append, targets, H=H, D=D, P=P, NB=64, n_max=max(cached) + max(append) + max(targets) + 8,
                       num_pages=num_pages or need + 16, dtype="bf16", seed=seed)
    rng = np.random.default_rng(seed + 100)
    x = gen._values(rng, (c.Tn, d_model), 1.0, "bf16")
    w1 = gen._values(rng, (4 * H * D, d_model), 1.0 / np.sqrt(d_model), "bf16")
    w2 = gen._values(rng, (d_model, H * D), 1.0 / np.sqrt(H * D), "bf16")
    return c, x, w1, w2, d_model


def _run_layer(hb, c, x, w1, w2, d_model):
    import torch

    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                  max_pages_per_user=c.max_pages, ln_eps=c.eps)
    kp, vp = device_pool(c)
    ws = hb.LayerWorkspace(p, d_model, c.B, c.Tn, c.max_new)
    y = hb.layer_paged_fwd(p, d_model, dev(x), dev(w1), dev(w2), kp, vp, dev(c.page_table), dev(c.cached_lens),
                           dev(c.new_lens), dev(c.num_targets), dev(c.rab), max_new=c.max_new, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    return host(y), kp, vp


def _oracle_layer(c, x, w1, w2, rows=None):
    ck, cv, cpt = c.compact_pool()
    return hl.layer_paged(_f64(x), _f64(w1), _f64(w2), ck, cv, cpt, c.cached_lens, c.new_lens, c.num_targets, c.rab,
                          c.n_max, c.eps, rows=rows)


def test_layer_small_matches_the_oracle(hb):
    c, x, w1, w2, d_model = _layer_case(5, [0, 37, 300, 129], [5, 16, 0, 40], [3, 64, 8, 1])
    y, kp, vp = _run_layer(hb, c, x, w1, w2, d_model)
    assert_close(y, _oracle_layer(c, x, w1, w2), "bf16", "layer output")
    # the new history tokens' k and v went into the pages (within bf16 rounding of the projection)
    q, k, v, u = hl.qkvu(_f64(x), _f64(w1), c.H, c.D)
    kb, vb = host(kp), host(vp)
    off = 0
    for b in range(c.B):
        n_app = int(c.new_lens[b] - c.num_targets[b])
        for t in range(n_app):
            pos = int(c.cached_lens[b]) + t
            pg = int(c.page_table[b, pos // c.P])
            assert_close(kb[pg, :, pos % c.P, :], k[off + t], "bf16", f"appended k of user {b} token {t}")
            assert_close(vb[pg, :, pos % c.P, :], v[off + t], "bf16", f"appended v of user {b} token {t}")
        off += int(c.new_lens[b])


def test_layer_benchmark_shape_sampled_rows(hb):
    # the paged benchmark's shape (8 users, cached U[1024, 4096], 16 appended + 64 candidates,
    # H=4, D=128, P=32) with d_model = 512; every 7th row against the oracle
    rng = np.random.default_rng(1003)
    cached = [int(x) for x in rng.integers(1024, 4097, 8)]
    c, x, w1, w2, d_model = _layer_case(6, cached, [16] * 8, [64] * 8, d_model=512)
    y, _, _ = _run_layer(hb, c, x, w1, w2, d_model)
    rows = np.arange(0, c.Tn, 7)
    assert_close(y[rows], _oracle_layer(c, x, w1, w2, rows=rows), "bf16", "layer output (sampled rows)")
