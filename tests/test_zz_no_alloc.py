"""hstu_attn_paged_fwd_noalloc: the paged forward on the library's built-in scratch array.

Compared with hstu_attn_paged_fwd (caller workspace) on the same inputs, within the parity
tolerance of the suite: the built-in 8 MiB scratch may hold fewer fp32 partial planes than a full
workspace, so the key range can be split differently and only the summation order changes.
This file is named to be collected last; it also passes on its own.
"""
import dataclasses

import numpy as np
import pytest

from hstu_attention_b200 import inputs as gen
from tests.helpers import (BF16_TOL, FP32_TOL, assert_close, dev, device_pool, gpu_paged, host, oracle_paged,
                           paged_params, values)

pytestmark = pytest.mark.gpu


def _compact(c):
    """The same case over a pool holding only its own pages (renumbered; same content)."""
    ck, cv, cpt = c.compact_pool()
    return dataclasses.replace(c, num_pages=int(ck.shape[0]), page_table=cpt,
                               page_ids=np.arange(ck.shape[0], dtype=np.int32))


def _noalloc(hb, c, pool, flags, page_table=None):
    p = paged_params(hb, c)
    kp, vp = pool
    pt = dev(c.page_table if page_table is None else page_table)
    return hb.paged_fwd_noalloc(p, dev(c.q_new), dev(c.k_new), dev(c.v_new), dev(c.u_new), kp, vp, pt,
                                dev(c.cached_lens), dev(c.new_lens), dev(c.num_targets), dev(c.rab),
                                max_new=max(c.max_new, 1), flags=flags)


def _close(a, b, dtype, what):
    a, b = values(host(a)), values(host(b))
    assert np.all(np.isfinite(a)), what
    err = float(np.max(np.abs(a - b)))
    scale = float(np.max(np.abs(b)))
    tol = BF16_TOL[0] * scale + BF16_TOL[1] if dtype == "bf16" else FP32_TOL * scale
    assert err <= tol, f"{what}: max err {err:.3e} > tol {tol:.3e}"


def _flags(torch):
    return torch.full((1,), -1, dtype=torch.int32, device="cuda")   # poisoned: the call must overwrite


def test_two_calls_in_a_row_match_the_workspace_entry(cuda_lib):
    import torch

    hb = cuda_lib
    # one layer of the 8-user cache-hit batch (640 new tokens at H*D = 512: the scratch holds 6
    # partial planes, a full workspace 8) and a small ragged batch with an empty history
    a = _compact(gen.config3_paged_layers(layers=1)[0])
    b = gen.paged_case([0, 31, 129, 300, 1000, 77], [3, 16, 0, 16, 5, 16], [1, 64, 2, 64, 130, 4], H=4, D=128,
                       P=32, NB=128, n_max=1400, num_pages=300, dtype="bf16", seed=91)
    pa, pb = device_pool(a), device_pool(b)
    ref_a, ws_a, _, _ = gpu_paged(hb, a, pool=pa)
    ref_b, ws_b, _, _ = gpu_paged(hb, b, pool=pb)
    assert ws_a.status() == 0 and ws_b.status() == 0

    fa, fb, fa2 = _flags(torch), _flags(torch), _flags(torch)
    out_a = _noalloc(hb, a, pa, fa)
    out_b = _noalloc(hb, b, pb, fb)          # second call right behind the first, same stream
    out_a2 = _noalloc(hb, a, pa, fa2)
    torch.cuda.synchronize()
    assert int(fa.item()) == 0 and int(fb.item()) == 0 and int(fa2.item()) == 0
    _close(out_a, ref_a, "bf16", "cache-hit layer")
    _close(out_b, ref_b, "bf16", "small ragged batch")
    assert torch.equal(out_a.view(torch.int16), out_a2.view(torch.int16))   # deterministic on repeat
    # and against the float64 oracle directly
    assert_close(host(out_a), oracle_paged(a), "bf16", "no-alloc cache-hit layer vs oracle")
    assert_close(host(out_b), oracle_paged(b), "bf16", "no-alloc ragged batch vs oracle")


def test_fp32_path_matches_the_workspace_entry(cuda_lib):
    import torch

    hb = cuda_lib
    c = gen.config1_tiny()
    pool = device_pool(c)
    ref, ws, _, _ = gpu_paged(hb, c, pool=pool)
    assert ws.status() == 0
    f1, f2 = _flags(torch), _flags(torch)
    o1 = _noalloc(hb, c, pool, f1)
    o2 = _noalloc(hb, c, pool, f2)
    torch.cuda.synchronize()
    assert int(f1.item()) == 0 and int(f2.item()) == 0
    _close(o1, ref, "fp32", "tiny fp32, first call")
    _close(o2, ref, "fp32", "tiny fp32, second call")
    assert_close(host(o2), oracle_paged(c), "fp32", "no-alloc tiny fp32 vs oracle")


def test_flags_are_per_call(cuda_lib):
    """A bad page id is reported to that call's flags only: the status word is cleared per call."""
    import torch

    hb = cuda_lib
    c = gen.paged_case([0, 31, 129, 300], [3, 16, 0, 16], [1, 64, 2, 64], H=4, D=128, P=32, NB=128, n_max=1400,
                       num_pages=64, dtype="bf16", seed=92)
    pool = device_pool(c)
    bad = c.page_table.copy()
    bad[3, 2] = c.num_pages + 7
    f_bad, f_ok = _flags(torch), _flags(torch)
    _noalloc(hb, c, pool, f_bad, page_table=bad)
    out = _noalloc(hb, c, pool, f_ok)
    torch.cuda.synchronize()
    assert int(f_bad.item()) & hb.DEV_BAD_PAGE
    assert int(f_ok.item()) == 0
    ref, _, _, _ = gpu_paged(hb, c, pool=pool)
    _close(out, ref, "bf16", "clean call after a flagged one")


def test_request_beyond_the_scratch_is_rejected(cuda_lib):
    """4,088 new tokens at H*D = 512 need more than 8 MiB: rejected on the host, nothing launched."""
    import torch

    hb = cuda_lib
    p = hb.params(4, 128, torch.bfloat16, 128, 8192, page_size=32, num_pages=4, max_pages_per_user=4)
    t = torch.zeros((4088, 4, 128), dtype=torch.bfloat16, device="cuda")
    pages = torch.zeros((4, 4, 32, 128), dtype=torch.bfloat16, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    with pytest.raises(hb.HstuError, match=r"8 MiB .*\(-5\)"):
        hb.paged_fwd_noalloc(p, t, t, t, t, pages, pages, torch.zeros((1, 4), **i32), torch.zeros(1, **i32),
                             torch.full((1,), 4088, **i32), torch.zeros(1, **i32),
                             torch.zeros((4, 128), dtype=torch.float32, device="cuda"), max_new=4088)
    # one token fewer than the limit at this width still runs (4,087 fits)
    t2 = t[:4087]
    out = hb.paged_fwd_noalloc(p, t2, t2, t2, t2, pages, pages, torch.zeros((1, 4), **i32), torch.zeros(1, **i32),
                               torch.full((1,), 4087, **i32), torch.zeros(1, **i32),
                               torch.zeros((4, 128), dtype=torch.float32, device="cuda"), max_new=4087)
    torch.cuda.synchronize()
    assert torch.all(out == 0)          # q = k = v = u = 0: LayerNorm of zeros gated by zeros
