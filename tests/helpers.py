"""Shared test plumbing: move generated inputs to the GPU, call the library, call the oracle."""
from __future__ import annotations

import numpy as np

import oracle
from hstu_attention_b200 import inputs as gen

BF16_TOL = (1e-2, 1e-3)     # max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3  (bf16 in, fp32 accumulate)
FP32_TOL = 1e-4             # max|gpu - oracle| <= 1e-4 * max|oracle|           (fp32 path)


def dev(x, dtype=None):
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    import torch

    if x is None:
        return None
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    if dtype is not None:
        x = x.astype(dtype)
    if x.dtype == np.int64:
        x = x.astype(np.int32)
    return torch.from_numpy(x).cuda()


def host(t):
    """CUDA tensor -> numpy (bf16 as uint16 bits, widened to float32 with as_f32)."""
    import torch

    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def values(x):
    return gen.as_f32(x).astype(np.float64)


def assert_close(gpu, ref, dtype: str, what: str = ""):
    g = values(gpu)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = float(np.max(np.abs(g - ref))) if g.size else 0.0
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if dtype == "bf16":
        tol = BF16_TOL[0] * scale + BF16_TOL[1]
    else:
        tol = FP32_TOL * scale
    assert err <= tol, f"{what}: max err {err:.3e} > tol {tol:.3e} (max|ref| {scale:.3e})"
    return err, tol


# --------------------------------------------------------------------------- jagged


def gpu_jagged(hb, c: gen.JaggedCase, ws=None, max_seqlen=None, out=None):
    import torch

    p = hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, ln_eps=c.eps)
    ms = int(max_seqlen if max_seqlen is not None else max(c.max_seqlen, 1))
    if ws is None:
        ws = hb.Workspace(p, c.B, max(c.T, 1), ms)
    t = dict(q=dev(c.q), k=dev(c.k), v=dev(c.v), u=dev(c.u), off=dev(c.seq_offsets), nt=dev(c.num_targets),
             rab=dev(c.rab))
    o = hb.jagged_fwd(p, t["q"], t["k"], t["v"], t["u"], t["off"], t["nt"], t["rab"], max_seqlen=ms, workspace=ws,
                      out=out)
    torch.cuda.synchronize()
    return o, ws, p


def oracle_jagged(c: gen.JaggedCase, rows=None):
    return oracle.hstu_jagged(c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps, rows=rows)


# --------------------------------------------------------------------------- paged


def device_pool(c: gen.PagedCase, poison: bool = False):
    """Full physical pool on the GPU: used pages from the case, the rest zero (or NaN)."""
    import torch

    tdt = torch.bfloat16 if c.dtype == "bf16" else torch.float32
    shape = (c.num_pages, c.H, c.P, c.D)
    fill = float("nan") if poison else 0.0
    kp = torch.full(shape, fill, dtype=tdt, device="cuda")
    vp = torch.full(shape, fill, dtype=tdt, device="cuda")
    if c.page_ids.shape[0]:
        ids = torch.from_numpy(c.page_ids.astype(np.int64)).cuda()
        kp[ids] = dev(c.pool_k)
        vp[ids] = dev(c.pool_v)
    return kp, vp


def paged_params(hb, c: gen.PagedCase):
    return hb.params(c.H, c.D, c.dtype, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                     max_pages_per_user=c.max_pages, ln_eps=c.eps)


def gpu_paged(hb, c: gen.PagedCase, pool=None, ws=None, page_table=None, poison=False, max_new=None):
    import torch

    p = paged_params(hb, c)
    kp, vp = pool if pool is not None else device_pool(c, poison=poison)
    mn = int(max_new if max_new is not None else max(c.max_new, 1))
    if ws is None:
        ws = hb.Workspace(p, c.B, max(c.Tn, 1), mn)
    pt = dev(c.page_table if page_table is None else page_table)
    o = hb.paged_fwd(p, dev(c.q_new), dev(c.k_new), dev(c.v_new), dev(c.u_new), kp, vp, pt, dev(c.cached_lens),
                     dev(c.new_lens), dev(c.num_targets), dev(c.rab), max_new=mn, workspace=ws)
    torch.cuda.synchronize()
    return o, ws, p, (kp, vp)


def oracle_paged(c: gen.PagedCase, rows=None):
    ck, cv, cpt = c.compact_pool()
    return oracle.hstu_paged(c.q_new, c.k_new, c.v_new, c.u_new, ck, cv, cpt, c.cached_lens, c.new_lens,
                             c.num_targets, c.rab, c.n_max, c.eps, rows=rows)
