"""The C-ABI library loads on a machine without a GPU, exports every symbol include/hstu.h
declares, and rejects bad host-side arguments before touching the device."""
import ctypes
import os
import re

import pytest

import hstu_attention_b200 as hb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hstu.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from hstu_attention_b200 import build

    build.build()
    return hb.load()


def test_header_declares_the_api():
    names = _declared()
    assert "hstu_attn_jagged_fwd" in names and "hstu_attn_paged_fwd" in names and "hstu_kv_append" in names
    assert set(names) == set(hb.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_version_and_error_strings(lib):
    assert "sm_100a" in hb.version()
    for code, text in [(0, "ok"), (-1, "invalid"), (-2, "unsupported"), (-3, "workspace"), (-4, "CUDA")]:
        assert text in lib.hstu_error_string(code).decode()


def _p(**kw):
    base = dict(num_heads=4, head_dim=128, dtype="bf16", num_buckets=128, n_max=4096, page_size=32,
                num_pages=64, max_pages_per_user=8)
    base.update(kw)
    return hb.params(**base)


def test_workspace_size(lib):
    p = _p()
    n = hb.workspace_size(p, 8, 1000, 256)
    assert n % 256 == 0 and n >= 256 + 1000 * 4 * 128 * 4
    assert lib.hstu_workspace_size(None, 1, 1, 1) == 0
    bad = _p(head_dim=96)
    assert lib.hstu_workspace_size(ctypes.byref(bad), 1, 1, 1) == 0


def test_host_validation_without_gpu(lib):
    """Every call here fails host-side validation, so nothing reaches the device."""
    p = _p()
    fake = 1 << 20                      # aligned, never dereferenced
    ws = 1 << 24
    J = lib.hstu_attn_jagged_fwd
    args = [fake, fake, fake, fake, fake, None, fake, fake, 2, 100, 64, ws, 1 << 30, None]
    assert J(None, *args) == -1                                          # INVALID_ARG
    assert J(ctypes.byref(_p(head_dim=96)), *args) == -2                  # UNSUPPORTED
    assert J(ctypes.byref(_p(dtype="fp32", num_buckets=0)), *args) == -1
    mis = list(args)
    mis[0] = fake + 2                                                     # misaligned q
    assert J(ctypes.byref(p), *mis) == -1
    small = list(args)
    small[-2] = 100                                                       # workspace too small
    assert J(ctypes.byref(p), *small) == -3
    unal = list(args)
    unal[-3] = ws + 8                                                     # misaligned workspace
    assert J(ctypes.byref(p), *unal) == -3
    neg = list(args)
    neg[8] = -1
    assert J(ctypes.byref(p), *neg) == -1
    # empty batch is a no-op success
    empty = list(args)
    empty[8] = 0
    assert J(ctypes.byref(p), *empty) == 0

    P = lib.hstu_attn_paged_fwd
    pargs = [fake] * 6 + [fake, fake, fake, None, fake, fake, 2, 100, 64, ws, 1 << 30, None]
    assert P(ctypes.byref(_p(page_size=24)), *pargs) == -2
    assert P(ctypes.byref(_p(num_pages=0)), *pargs) == -1
    nul = list(pargs)
    nul[6] = None                                                         # page_table
    assert P(ctypes.byref(p), *nul) == -1

    A = lib.hstu_kv_append
    aargs = [fake, fake, fake, fake, fake, fake, fake, None, 2, 100, 64, ws, 1 << 20, None]
    assert A(ctypes.byref(_p(page_size=12)), *aargs) == -2
    bad_ws = list(aargs)
    bad_ws[-3] = None
    assert A(ctypes.byref(p), *bad_ws) == -3
    assert lib.hstu_bucket_table(ctypes.byref(p), -1, None, None) == -1


def test_flags_and_noalloc_limit_without_gpu(lib):
    """Unknown flag bits are rejected; the allocation-free entry rejects a request larger than its
    built-in 8 MiB scratch before it touches the device."""
    bad = _p(flags=1 << 7)
    assert lib.hstu_workspace_size(ctypes.byref(bad), 1, 1, 1) == 0
    ok = _p(flags=hb.FLAG_OVERLAP_PREVIOUS)
    assert lib.hstu_workspace_size(ctypes.byref(ok), 1, 1, 1) > 0
    fake = 1 << 20
    N = lib.hstu_attn_paged_fwd_noalloc
    # 4,088 new tokens at H*D = 512 need 256 + 16,384 + 8,372,224 bytes > 8 MiB
    args = [fake] * 6 + [fake, fake, fake, None, fake, fake, 1, 4088, 4088, None, None]
    assert N(ctypes.byref(_p(n_max=8192)), *args) == hb.ERR_SCRATCH_LIMIT
    assert "8 MiB" in lib.hstu_error_string(hb.ERR_SCRATCH_LIMIT).decode()
    assert N(ctypes.byref(bad), *args) == -1
    misaligned_flags = list(args)
    misaligned_flags[-2] = fake + 2                                       # flags_out not 4-byte aligned
    assert N(ctypes.byref(_p(n_max=8192)), *misaligned_flags) == -1


def test_page_copy_host_validation_without_gpu(lib):
    """The page-copy entry rejects bad arguments before it touches the device; on a machine
    without a GPU no pointer is device-addressable, so even well-formed calls are refused."""
    p = _p()
    fake = 1 << 20
    C = lib.hstu_kv_page_copy
    good = [fake, fake, 8, fake, fake, 8, fake, 4, fake, 4096, None]
    assert C(None, *good) == -1
    bad = list(good)
    bad[7] = -1                                   # n_pairs < 0
    assert C(ctypes.byref(p), *bad) == -1
    bad = list(good)
    bad[8] = fake + 8                             # workspace not 256-byte aligned
    assert C(ctypes.byref(p), *bad) == -3
    bad = list(good)
    bad[0] = fake + 4                             # source pool not 16-byte aligned
    assert C(ctypes.byref(p), *bad) == -1
    zero = list(good)
    zero[7] = 0
    assert C(ctypes.byref(p), *zero) == 0         # nothing to copy
    assert C(ctypes.byref(p), *good) == -1        # not addressable by any device here
    for code in (hb.ERR_CACHE_FULL, hb.ERR_OUTPUT_CAPACITY):
        assert lib.hstu_error_string(code).decode() != "unknown error"


def test_backward_host_validation_without_gpu(lib):
    """The backward entry rejects bad arguments before it enqueues anything."""
    p = _p()
    fake = 1 << 20
    ws = 1 << 24
    n = lib.hstu_workspace_size_bwd(ctypes.byref(p), 1000)
    assert n % 256 == 0 and n >= 256 + 2 * 1000 * 4 * 128 * 4
    assert lib.hstu_workspace_size_bwd(None, 10) == 0
    Bw = lib.hstu_attn_jagged_bwd
    args = [fake] * 4 + [fake, None, fake, fake] + [fake] * 5 + [2, 100, 64, ws, 1 << 30, None]
    assert Bw(None, *args) == -1
    assert Bw(ctypes.byref(_p(head_dim=96)), *args) == -2
    no_drab = list(args)
    no_drab[12] = None
    assert Bw(ctypes.byref(p), *no_drab) == -1
    no_dout = list(args)
    no_dout[7] = None
    assert Bw(ctypes.byref(p), *no_dout) == -1
    mis = list(args)
    mis[8] = fake + 4                                                     # dq not 16-byte aligned
    assert Bw(ctypes.byref(p), *mis) == -1
    small = list(args)
    small[-2] = 1000                                                      # workspace too small
    assert Bw(ctypes.byref(p), *small) == -3
    unal = list(args)
    unal[-3] = ws + 8
    assert Bw(ctypes.byref(p), *unal) == -3
    # the LayerNorm variants exist in the forward calls only
    assert Bw(ctypes.byref(_p(flags=hb.FLAG_LN_PER_HEAD)), *args) == -2
    affine = _p()
    affine.ln_weight = fake
    assert Bw(ctypes.byref(affine), *args) == -2
    odd = _p()
    odd.ln_bias = fake + 2                                                # not 4-byte aligned
    assert lib.hstu_workspace_size(ctypes.byref(odd), 1, 1, 1) == 0
    # the time bias: argument checks, and the calls that do not implement it
    tbias = _p()
    tbias.rab_time, tbias.timestamps, tbias.num_time_buckets = fake, fake, 16
    assert lib.hstu_workspace_size(ctypes.byref(tbias), 1, 1, 1) > 0
    assert Bw(ctypes.byref(tbias), *args) == -2
    for bad in ((fake, None, 16), (fake, fake, 0), (fake, fake, 65), (fake + 2, fake, 16)):
        tb = _p()
        tb.rab_time, tb.timestamps, tb.num_time_buckets = bad
        assert lib.hstu_workspace_size(ctypes.byref(tb), 1, 1, 1) == 0


def test_binding_checks_types_before_any_call():
    """The binding refuses tensors of the wrong element type or shape (the C ABI takes bare
    pointers) before it touches the library or the device."""
    import torch

    p = hb.params(4, 128, torch.bfloat16, 16, 64)
    t = torch.zeros((8, 4, 128), dtype=torch.bfloat16)
    off = torch.tensor([0, 8], dtype=torch.int32)
    rab = torch.zeros((4, 16))
    with pytest.raises(hb.HstuError, match="q must be torch.bfloat16"):
        hb.jagged_fwd(p, t.float(), t, t, t, off, None, rab, max_seqlen=8, workspace=None)
    with pytest.raises(hb.HstuError, match="seq_offsets must be int32"):
        hb.jagged_fwd(p, t, t, t, t, off.long(), None, rab, max_seqlen=8, workspace=None)
    with pytest.raises(hb.HstuError, match="rab must be float32"):
        hb.jagged_fwd(p, t, t, t, t, off, None, rab.double(), max_seqlen=8, workspace=None)
    with pytest.raises(hb.HstuError, match="expected"):
        hb.jagged_fwd(p, t[:, :2], t, t, t, off, None, rab, max_seqlen=8, workspace=None)
    with pytest.raises(hb.HstuError, match="dout must be torch.bfloat16"):
        hb.jagged_bwd(p, t, t, t, t, off, None, rab, t.float(), max_seqlen=8, workspace=None)
