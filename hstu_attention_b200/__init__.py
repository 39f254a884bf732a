"""Python binding of the HSTU B200 attention library (libhstu_b200.so, C ABI in include/hstu.h).

This module only marshals arguments: it turns torch tensors into device pointers and host
sizes and calls the C entry points of the same names.  Every step of the computation runs
in the library's CUDA kernels.  There is no CPU fallback: if the shared library is missing
or no GPU is present, the calls raise.

    import hstu_attention_b200 as hb
    p = hb.params(num_heads=4, head_dim=128, dtype=torch.bfloat16, num_buckets=128, n_max=4096)
    ws = hb.Workspace(p, max_batch=8, max_tokens=20000, max_new=4096)
    out = hb.jagged_fwd(p, q, k, v, u, seq_offsets, num_targets, rab, max_seqlen=4096, workspace=ws)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhstu_b200.so")
_lib = None
_lock = threading.Lock()

HSTU_DTYPE_BF16 = 0
HSTU_DTYPE_FP32 = 1

DEV_BAD_PAGE = 1 << 0
DEV_BAD_LENGTH = 1 << 1
DEV_BAD_NMAX = 1 << 2
DEV_TIMEOUT = 1 << 3

ERR_SCRATCH_LIMIT = -5
ERR_CACHE_FULL = -6
ERR_OUTPUT_CAPACITY = -7

TIER_MISS = 0
TIER_GPU = 1
TIER_HOST = 2

FLAG_OVERLAP_PREVIOUS = 1 << 0
FLAG_LN_PER_HEAD = 1 << 1

INJECT_STALL_V = 1

EXPORTED = (
    "hstu_version",
    "hstu_error_string",
    "hstu_workspace_size",
    "hstu_workspace_init",
    "hstu_read_status",
    "hstu_attn_jagged_fwd",
    "hstu_attn_jagged_bwd",
    "hstu_workspace_size_bwd",
    "hstu_attn_paged_fwd",
    "hstu_attn_paged_fwd_noalloc",
    "hstu_kv_append",
    "hstu_bucket_table",
    "hstu_cache_create",
    "hstu_cache_destroy",
    "hstu_cache_lookup",
    "hstu_cache_prepare",
    "hstu_cache_evict",
    "hstu_cache_compact",
    "hstu_cache_page_rows",
    "hstu_cache_stats",
    "hstu_kv_page_copy",
    "hstu_host_copy",
    "hstu_test_inject",
    "hstu_linear_fwd",
    "hstu_workspace_size_layer",
    "hstu_layer_paged_fwd",
    "hstu_ts_page_copy",
)


class HstuParams(ctypes.Structure):
    """Mirror of ``hstu_attn_params`` in include/hstu.h."""

    _fields_ = [
        ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("num_buckets", ctypes.c_int32),
        ("n_max", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages_per_user", ctypes.c_int32),
        ("ln_eps", ctypes.c_float),
        ("flags", ctypes.c_uint32),
        ("ln_weight", ctypes.c_void_p),
        ("ln_bias", ctypes.c_void_p),
        ("rab_time", ctypes.c_void_p),
        ("timestamps", ctypes.c_void_p),
        ("num_time_buckets", ctypes.c_int32),
        ("ts_pages", ctypes.c_void_p),
    ]


class HstuError(RuntimeError):
    pass


def load(path: Optional[str] = None):
    """Load the shared library (raises HstuError if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise HstuError(f"{p} not found: build it with `python -m hstu_attention_b200.build`")
            lib = ctypes.CDLL(p)
            i32, i64, sz, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
            pp = ctypes.POINTER(HstuParams)
            lib.hstu_version.restype = ctypes.c_char_p
            lib.hstu_version.argtypes = []
            lib.hstu_error_string.restype = ctypes.c_char_p
            lib.hstu_error_string.argtypes = [ctypes.c_int]
            lib.hstu_workspace_size.restype = sz
            lib.hstu_workspace_size.argtypes = [pp, i32, i64, i32]
            lib.hstu_workspace_init.restype = ctypes.c_int
            lib.hstu_workspace_init.argtypes = [vp, sz, vp]
            lib.hstu_read_status.restype = ctypes.c_int
            lib.hstu_read_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
            lib.hstu_attn_jagged_fwd.restype = ctypes.c_int
            lib.hstu_attn_jagged_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, sz, vp]
            lib.hstu_workspace_size_bwd.restype = sz
            lib.hstu_workspace_size_bwd.argtypes = [pp, i64]
            lib.hstu_attn_jagged_bwd.restype = ctypes.c_int
            lib.hstu_attn_jagged_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64,
                                                 i32, vp, sz, vp]
            lib.hstu_attn_paged_fwd.restype = ctypes.c_int
            lib.hstu_attn_paged_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32,
                                                vp, sz, vp]
            lib.hstu_attn_paged_fwd_noalloc.restype = ctypes.c_int
            lib.hstu_attn_paged_fwd_noalloc.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64,
                                                        i32, vp, vp]
            lib.hstu_kv_append.restype = ctypes.c_int
            lib.hstu_kv_append.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, sz, vp]
            lib.hstu_bucket_table.restype = ctypes.c_int
            lib.hstu_bucket_table.argtypes = [pp, i32, vp, vp]
            lib.hstu_cache_create.restype = ctypes.c_int
            lib.hstu_cache_create.argtypes = [i32, i32, i32, i32, ctypes.POINTER(vp)]
            lib.hstu_cache_destroy.restype = None
            lib.hstu_cache_destroy.argtypes = [vp]
            lib.hstu_cache_lookup.restype = ctypes.c_int
            lib.hstu_cache_lookup.argtypes = [vp, vp, i32, vp, vp]
            lib.hstu_cache_prepare.restype = ctypes.c_int
            lib.hstu_cache_prepare.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, i32, vp]
            lib.hstu_cache_evict.restype = ctypes.c_int
            lib.hstu_cache_evict.argtypes = [vp, i64, vp]
            lib.hstu_cache_compact.restype = ctypes.c_int
            lib.hstu_cache_compact.argtypes = [vp, vp, i32, vp]
            lib.hstu_cache_page_rows.restype = ctypes.c_int
            lib.hstu_cache_page_rows.argtypes = [vp, vp, i32, vp]
            lib.hstu_cache_stats.restype = ctypes.c_int
            lib.hstu_cache_stats.argtypes = [vp, vp]
            lib.hstu_kv_page_copy.restype = ctypes.c_int
            lib.hstu_kv_page_copy.argtypes = [pp, vp, vp, i32, vp, vp, i32, vp, i32, vp, sz, vp]
            lib.hstu_host_copy.restype = ctypes.c_int
            lib.hstu_host_copy.argtypes = [vp, vp, sz, vp]
            lib.hstu_linear_fwd.restype = ctypes.c_int
            lib.hstu_linear_fwd.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, sz, vp]
            lib.hstu_workspace_size_layer.restype = sz
            lib.hstu_workspace_size_layer.argtypes = [pp, i32, i32, i64, i32]
            lib.hstu_layer_paged_fwd.restype = ctypes.c_int
            lib.hstu_layer_paged_fwd.argtypes = [pp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32,
                                                 vp, sz, vp]
            lib.hstu_ts_page_copy.restype = ctypes.c_int
            lib.hstu_ts_page_copy.argtypes = [vp, i32, vp, i32, i32, vp, i32, vp, sz, vp]
            lib.hstu_test_inject.restype = ctypes.c_int
            lib.hstu_test_inject.argtypes = [ctypes.c_uint32, ctypes.c_uint64]
            _lib = lib
    return _lib


def version() -> str:
    return load().hstu_version().decode()


def _check(rc: int, what: str):
    if rc != 0:
        msg = load().hstu_error_string(rc).decode()
        raise HstuError(f"{what} failed: {msg} ({rc})")


def params(num_heads: int, head_dim: int, dtype, num_buckets: int, n_max: int, page_size: int = 0,
           num_pages: int = 0, max_pages_per_user: int = 0, ln_eps: float = 1e-5, flags: int = 0,
           ln_per_head: bool = False, ln_weight=None, ln_bias=None, rab_time=None, timestamps=None,
           ts_pages=None) -> HstuParams:
    """Mirror of hstu_attn_params.  ln_per_head / ln_weight / ln_bias select the LayerNorm-gate
    variants (fp32 CUDA tensors of H*D elements for gamma and beta; the params object keeps them
    alive)."""
    import torch

    for name, t in (("ln_weight", ln_weight), ("ln_bias", ln_bias)):
        if t is not None and (not t.is_cuda or t.dtype != torch.float32 or t.numel() != num_heads * head_dim
                              or not t.is_contiguous()):
            raise HstuError(f"{name} must be a contiguous fp32 CUDA tensor of H*D = {num_heads * head_dim} elements")
    if ln_per_head:
        flags |= FLAG_LN_PER_HEAD
    if rab_time is not None and timestamps is None:
        raise HstuError("rab_time needs timestamps")
    if ts_pages is not None and (not ts_pages.is_cuda or ts_pages.dtype != torch.int32 or not ts_pages.is_contiguous()):
        raise HstuError("ts_pages must be a contiguous int32 CUDA tensor [num_pages, page_size]")
    if timestamps is not None and (not timestamps.is_cuda or timestamps.dtype != torch.int32
                                   or not timestamps.is_contiguous()):
        raise HstuError("timestamps must be a contiguous int32 CUDA tensor, one per token")
    if rab_time is not None:
        if (not rab_time.is_cuda or rab_time.dtype != torch.float32 or rab_time.dim() != 2
                or rab_time.shape[0] != num_heads or not rab_time.is_contiguous()):
            raise HstuError("rab_time must be a contiguous fp32 CUDA tensor [H, num_time_buckets]")

    if dtype in (torch.bfloat16, "bf16"):
        dt = HSTU_DTYPE_BF16
    elif dtype in (torch.float32, "fp32"):
        dt = HSTU_DTYPE_FP32
    else:
        raise HstuError(f"unsupported dtype {dtype}")
    p = HstuParams(num_heads, head_dim, dt, num_buckets, n_max, page_size, num_pages, max_pages_per_user,
                   ln_eps, flags, ln_weight.data_ptr() if ln_weight is not None else None,
                   ln_bias.data_ptr() if ln_bias is not None else None,
                   rab_time.data_ptr() if rab_time is not None else None,
                   timestamps.data_ptr() if timestamps is not None else None,
                   int(rab_time.shape[1]) if rab_time is not None else 0,
                   ts_pages.data_ptr() if ts_pages is not None else None)
    p._keep = (ln_weight, ln_bias, rab_time, timestamps, ts_pages)
    return p


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise HstuError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise HstuError("tensor arguments must be contiguous")
    return t.data_ptr()


def _check_args(p: HstuParams, elems=(), ints=(), floats=()):
    """Element types and shapes the C ABI expects (it receives bare pointers and cannot tell):
    token tensors [T, H, D] and pages of the params dtype, index arrays int32, rab fp32."""
    import torch

    want = torch.bfloat16 if p.dtype == HSTU_DTYPE_BF16 else torch.float32
    for name, t in elems:
        if t is None:
            continue
        if t.dtype != want:
            raise HstuError(f"{name} must be {want}, got {t.dtype}")
        if t.dim() < 3 or t.shape[-1] != p.head_dim or (t.dim() == 3 and t.shape[1] != p.num_heads):
            raise HstuError(f"{name} has shape {tuple(t.shape)}; expected [..., H={p.num_heads}, D={p.head_dim}]")
    for name, t in ints:
        if t is not None and t.dtype != torch.int32:
            raise HstuError(f"{name} must be int32, got {t.dtype}")
    for name, t in floats:
        if t is not None and t.dtype != torch.float32:
            raise HstuError(f"{name} must be float32, got {t.dtype}")


def _stream(stream) -> int:
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def workspace_size(p: HstuParams, max_batch: int, max_tokens: int, max_new: int) -> int:
    n = load().hstu_workspace_size(ctypes.byref(p), int(max_batch), int(max_tokens), int(max_new))
    if n == 0:
        raise HstuError("hstu_workspace_size: invalid parameters")
    return int(n)


class Workspace:
    """Device scratch for the calls (status word + fp32 partial outputs), zeroed once."""

    def __init__(self, p: HstuParams, max_batch: int, max_tokens: int, max_new: int, device=None, stream=None):
        import torch

        self.nbytes = workspace_size(p, max_batch, max_tokens, max_new)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buf.data_ptr()
        self.offset = (-base) % 256
        self.ptr = base + self.offset
        _check(load().hstu_workspace_init(self.ptr, self.nbytes, _stream(stream)), "hstu_workspace_init")

    def status(self, clear: bool = True, stream=None) -> int:
        flags = ctypes.c_uint32(0)
        _check(load().hstu_read_status(self.ptr, _stream(stream), ctypes.byref(flags), int(clear)), "hstu_read_status")
        return int(flags.value)


class BwdWorkspace(Workspace):
    """Device scratch of the backward pass (status word + the recomputed o and its gradient)."""

    def __init__(self, p: HstuParams, max_tokens: int, device=None, stream=None):
        import torch

        n = load().hstu_workspace_size_bwd(ctypes.byref(p), int(max_tokens))
        if n == 0:
            raise HstuError("hstu_workspace_size_bwd: invalid parameters")
        self.nbytes = int(n)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buf.data_ptr()
        self.offset = (-base) % 256
        self.ptr = base + self.offset
        _check(load().hstu_workspace_init(self.ptr, self.nbytes, _stream(stream)), "hstu_workspace_init")


def jagged_bwd(p: HstuParams, q, k, v, u, seq_offsets, num_targets, rab, dout, *, max_seqlen: int,
               workspace: BwdWorkspace, stream=None):
    """hstu_attn_jagged_bwd: gradients of sum(dout * out) of jagged_fwd.  Returns fp32
    (dq, dk, dv, du) [T, H, D] and drab [H, NB]."""
    import torch

    _check_args(p, elems=(("q", q), ("k", k), ("v", v), ("u", u), ("dout", dout)),
                ints=(("seq_offsets", seq_offsets), ("num_targets", num_targets)), floats=(("rab", rab),))
    dq, dk, dv, du = (torch.empty(q.shape, dtype=torch.float32, device=q.device) for _ in range(4))
    drab = torch.empty(rab.shape, dtype=torch.float32, device=q.device)
    B = seq_offsets.shape[0] - 1
    rc = load().hstu_attn_jagged_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(seq_offsets),
                                     _ptr(num_targets), _ptr(rab), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(du),
                                     _ptr(drab), B, q.shape[0], int(max_seqlen), workspace.ptr, workspace.nbytes,
                                     _stream(stream))
    _check(rc, "hstu_attn_jagged_bwd")
    return dq, dk, dv, du, drab


def jagged_fwd(p: HstuParams, q, k, v, u, seq_offsets, num_targets, rab, *, max_seqlen: int, workspace: Workspace,
               out=None, stream=None):
    """hstu_attn_jagged_fwd: q/k/v/u [T, H, D]; seq_offsets [B+1] int32; num_targets [B] int32 or None;
    rab [H, NB] fp32.  Returns out [T, H, D]."""
    import torch

    _check_args(p, elems=(("q", q), ("k", k), ("v", v), ("u", u), ("out", out)),
                ints=(("seq_offsets", seq_offsets), ("num_targets", num_targets)), floats=(("rab", rab),))
    if out is None:
        out = torch.empty_like(q)
    B = seq_offsets.shape[0] - 1
    rc = load().hstu_attn_jagged_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(seq_offsets),
                                     _ptr(num_targets), _ptr(rab), _ptr(out), B, q.shape[0], int(max_seqlen),
                                     workspace.ptr, workspace.nbytes, _stream(stream))
    _check(rc, "hstu_attn_jagged_fwd")
    return out


def paged_fwd(p: HstuParams, q_new, k_new, v_new, u_new, k_pages, v_pages, page_table, cached_lens, new_lens,
              num_targets, rab, *, max_new: int, workspace: Workspace, out=None, stream=None):
    """hstu_attn_paged_fwd: new-token tensors [Tn, H, D]; pages [num_pages, H, P, D];
    page_table [B, max_pages] int32; cached_lens/new_lens/num_targets [B] int32."""
    import torch

    _check_args(p, elems=(("q_new", q_new), ("k_new", k_new), ("v_new", v_new), ("u_new", u_new),
                          ("k_pages", k_pages), ("v_pages", v_pages), ("out", out)),
                ints=(("page_table", page_table), ("cached_lens", cached_lens), ("new_lens", new_lens),
                      ("num_targets", num_targets)), floats=(("rab", rab),))
    if out is None:
        out = torch.empty_like(q_new)
    B = cached_lens.shape[0]
    rc = load().hstu_attn_paged_fwd(ctypes.byref(p), _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(u_new),
                                    _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(cached_lens),
                                    _ptr(new_lens), _ptr(num_targets), _ptr(rab), _ptr(out), B, q_new.shape[0],
                                    int(max_new), workspace.ptr, workspace.nbytes, _stream(stream))
    _check(rc, "hstu_attn_paged_fwd")
    return out


def paged_fwd_noalloc(p: HstuParams, q_new, k_new, v_new, u_new, k_pages, v_pages, page_table, cached_lens,
                      new_lens, num_targets, rab, *, max_new: int, out=None, flags=None, stream=None):
    """hstu_attn_paged_fwd_noalloc: paged_fwd on the library's built-in 8 MiB scratch instead of a
    workspace.  ``flags``: optional 1-element int32 CUDA tensor that receives this call's device
    status bits.  All calls on a device share the scratch: do not overlap them across streams."""
    import torch

    _check_args(p, elems=(("q_new", q_new), ("k_new", k_new), ("v_new", v_new), ("u_new", u_new),
                          ("k_pages", k_pages), ("v_pages", v_pages), ("out", out)),
                ints=(("page_table", page_table), ("cached_lens", cached_lens), ("new_lens", new_lens),
                      ("num_targets", num_targets), ("flags", flags)), floats=(("rab", rab),))
    if out is None:
        out = torch.empty_like(q_new)
    B = cached_lens.shape[0]
    rc = load().hstu_attn_paged_fwd_noalloc(ctypes.byref(p), _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(u_new),
                                            _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(cached_lens),
                                            _ptr(new_lens), _ptr(num_targets), _ptr(rab), _ptr(out), B,
                                            q_new.shape[0], int(max_new), _ptr(flags), _stream(stream))
    _check(rc, "hstu_attn_paged_fwd_noalloc")
    return out


def kv_append(p: HstuParams, k_pages, v_pages, page_table, k_new, v_new, cached_lens, new_lens, num_targets, *,
              max_new: int, workspace: Workspace, stream=None):
    """hstu_kv_append: copy the first new_lens[b] - num_targets[b] new rows of each user into its pages."""
    _check_args(p, elems=(("k_pages", k_pages), ("v_pages", v_pages), ("k_new", k_new), ("v_new", v_new)),
                ints=(("page_table", page_table), ("cached_lens", cached_lens), ("new_lens", new_lens),
                      ("num_targets", num_targets)))
    B = cached_lens.shape[0]
    rc = load().hstu_kv_append(ctypes.byref(p), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(k_new),
                               _ptr(v_new), _ptr(cached_lens), _ptr(new_lens), _ptr(num_targets), B,
                               k_new.shape[0], int(max_new), workspace.ptr, workspace.nbytes, _stream(stream))
    _check(rc, "hstu_kv_append")


def bucket_table(p: HstuParams, n: int, stream=None):
    """hstu_bucket_table: the library's bucket(d) for d in [0, n) as a device int32 tensor."""
    import torch

    out = torch.empty(int(n), dtype=torch.int32, device="cuda")
    _check(load().hstu_bucket_table(ctypes.byref(p), int(n), _ptr(out), _stream(stream)), "hstu_bucket_table")
    return out


class CacheFull(HstuError):
    """hstu_cache_prepare: the batch does not fit in the GPU tier even with every other user evicted."""


class KVCache:
    """Host-side manager of the two-tier paged KV cache (hstu_cache_* in include/hstu.h).

    It owns no device memory: it hands out page ids of a GPU pool and a pinned host pool that
    the caller allocates ([pages, H, P, D] for K and for V), and returns the page copies that
    ``kv_page_copy`` performs.  Arrays come back as numpy int32/int64 arrays.
    """

    def __init__(self, gpu_pages: int, host_pages: int, page_size: int, max_pages_per_user: int):
        import numpy as np  # noqa: F401  (numpy is what the results are returned in)

        self.gpu_pages, self.host_pages = int(gpu_pages), int(host_pages)
        self.page_size, self.max_pages_per_user = int(page_size), int(max_pages_per_user)
        h = ctypes.c_void_p()
        _check(load().hstu_cache_create(self.gpu_pages, self.host_pages, self.page_size, self.max_pages_per_user,
                                        ctypes.byref(h)), "hstu_cache_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            load().hstu_cache_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _ids(ids):
        import numpy as np

        return np.ascontiguousarray(np.asarray(ids, dtype=np.int64).reshape(-1))

    def lookup(self, ids):
        """(tiers, stored lengths) of the users; changes nothing."""
        import numpy as np

        ids = self._ids(ids)
        tiers = np.zeros(len(ids), np.int32)
        lens = np.zeros(len(ids), np.int32)
        _check(load().hstu_cache_lookup(self._h, ids.ctypes.data, len(ids), tiers.ctypes.data, lens.ctypes.data),
               "hstu_cache_lookup")
        return tiers, lens

    def prepare(self, ids, append_lens) -> dict:
        """Allocate for one batch: returns tier_before, cached_lens, page_rows [B, max_pages],
        offload [n, 2] (GPU page, host page), onboard [n, 2] (host page, GPU page), dropped ids."""
        import numpy as np

        ids = self._ids(ids)
        app = np.ascontiguousarray(np.asarray(append_lens, dtype=np.int32).reshape(-1))
        if len(app) != len(ids):
            raise HstuError("one append length per user id")
        B = len(ids)
        tiers = np.zeros(B, np.int32)
        cached = np.zeros(B, np.int32)
        rows = np.zeros((B, self.max_pages_per_user), np.int32)
        cap_off = cap_on = cap_drop = 64
        while True:
            off = np.zeros((cap_off, 2), np.int32)
            on = np.zeros((cap_on, 2), np.int32)
            drop = np.zeros(cap_drop, np.int64)
            n_off, n_on, n_drop = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
            rc = load().hstu_cache_prepare(self._h, ids.ctypes.data, app.ctypes.data, B, tiers.ctypes.data,
                                           cached.ctypes.data, rows.ctypes.data, off.ctypes.data, cap_off,
                                           ctypes.byref(n_off), on.ctypes.data, cap_on, ctypes.byref(n_on),
                                           drop.ctypes.data, cap_drop, ctypes.byref(n_drop))
            if rc == ERR_OUTPUT_CAPACITY:
                cap_off, cap_on, cap_drop = (max(cap_off, n_off.value), max(cap_on, n_on.value),
                                             max(cap_drop, n_drop.value))
                continue
            if rc == ERR_CACHE_FULL:
                raise CacheFull(load().hstu_error_string(rc).decode())
            _check(rc, "hstu_cache_prepare")
            return {"tier_before": tiers, "cached_lens": cached, "page_rows": rows,
                    "offload": off[:n_off.value].copy(), "onboard": on[:n_on.value].copy(),
                    "dropped": drop[:n_drop.value].copy()}

    def evict(self, uid: int) -> int:
        tier = ctypes.c_int32()
        _check(load().hstu_cache_evict(self._h, int(uid), ctypes.byref(tier)), "hstu_cache_evict")
        return int(tier.value)

    def compact(self):
        """(from, to) GPU page moves [n, 2] that pack the residents into pages [0, live)."""
        import numpy as np

        moves = np.zeros((max(self.gpu_pages, 1), 2), np.int32)
        n = ctypes.c_int32()
        _check(load().hstu_cache_compact(self._h, moves.ctypes.data, self.gpu_pages, ctypes.byref(n)),
               "hstu_cache_compact")
        return moves[:n.value].copy()

    def page_rows(self, ids):
        import numpy as np

        ids = self._ids(ids)
        rows = np.zeros((len(ids), self.max_pages_per_user), np.int32)
        _check(load().hstu_cache_page_rows(self._h, ids.ctypes.data, len(ids), rows.ctypes.data),
               "hstu_cache_page_rows")
        return rows

    def stats(self) -> dict:
        import numpy as np

        s = np.zeros(5, np.int64)
        _check(load().hstu_cache_stats(self._h, s.ctypes.data), "hstu_cache_stats")
        return {"free_gpu": int(s[0]), "free_host": int(s[1]), "gpu_users": int(s[2]), "host_users": int(s[3]),
                "clock": int(s[4])}


def _ptr_addressable(t, name):
    """Pointer of a CUDA tensor or of a pinned host tensor (which the device addresses directly)."""
    if t is None:
        raise HstuError(f"{name} is required")
    if not t.is_contiguous():
        raise HstuError(f"{name} must be contiguous")
    if not t.is_cuda and not t.is_pinned():
        raise HstuError(f"{name} must be a CUDA tensor or pinned host memory")
    return t.data_ptr()


def kv_page_copy(p: HstuParams, src_k, src_v, dst_k, dst_v, pairs, *, workspace: Workspace, stream=None):
    """hstu_kv_page_copy: for each (from, to) row of ``pairs`` ([n, 2] int32, CUDA or pinned),
    copy page ``from`` of (src_k, src_v) to page ``to`` of (dst_k, dst_v).  Pools are
    [pages, H, P, D] CUDA tensors or pinned host tensors (onboard: host -> GPU, offload:
    GPU -> host, compaction: within the GPU pool)."""
    import torch

    want = torch.bfloat16 if p.dtype == HSTU_DTYPE_BF16 else torch.float32
    for name, t in (("src_k", src_k), ("src_v", src_v), ("dst_k", dst_k), ("dst_v", dst_v)):
        if t.dtype != want or t.dim() != 4 or tuple(t.shape[1:]) != (p.num_heads, p.page_size, p.head_dim):
            raise HstuError(f"{name} must be {want} [pages, {p.num_heads}, {p.page_size}, {p.head_dim}], "
                            f"got {t.dtype} {tuple(t.shape)}")
    if src_k.shape != src_v.shape or dst_k.shape != dst_v.shape:
        raise HstuError("K and V pools must have the same shape")
    if pairs.dtype != torch.int32 or pairs.dim() != 2 or pairs.shape[1] != 2:
        raise HstuError("pairs must be int32 [n, 2]")
    n = pairs.shape[0]
    if n == 0:
        return
    rc = load().hstu_kv_page_copy(ctypes.byref(p), _ptr_addressable(src_k, "src_k"), _ptr_addressable(src_v, "src_v"),
                                  src_k.shape[0], _ptr_addressable(dst_k, "dst_k"), _ptr_addressable(dst_v, "dst_v"),
                                  dst_k.shape[0], _ptr_addressable(pairs, "pairs"), n, workspace.ptr,
                                  workspace.nbytes, _stream(stream))
    _check(rc, "hstu_kv_page_copy")


def host_copy(dst, src, stream=None):
    """hstu_host_copy: copy src into dst (same number of bytes; CUDA or pinned host tensors) with
    the GPU's SMs, asynchronously on ``stream``."""
    n = dst.numel() * dst.element_size()
    if src.numel() * src.element_size() != n:
        raise HstuError("host_copy: src and dst differ in size")
    _check(load().hstu_host_copy(_ptr_addressable(dst, "dst"), _ptr_addressable(src, "src"), n, _stream(stream)),
           "hstu_host_copy")


def test_inject(kind: int, wait_limit_ns: int = 0):
    """hstu_test_inject: test-only fault injection of the time-out path (INJECT_STALL_V: the V
    producer issues nothing and role waits give up after wait_limit_ns); kind 0 restores normal calls."""
    _check(load().hstu_test_inject(int(kind), int(wait_limit_ns)), "hstu_test_inject")


def linear_fwd(x, w, *, activation: int = 0, workspace: Workspace, out=None, stream=None):
    """hstu_linear_fwd: act(x w^T) for bf16 CUDA tensors x [M, K], w [N, K]; activation 1 = SiLU."""
    import torch

    for name, t in (("x", x), ("w", w)):
        if t.dtype != torch.bfloat16 or t.dim() != 2:
            raise HstuError(f"{name} must be a 2-D bf16 tensor")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise HstuError("x and w disagree on K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(load().hstu_linear_fwd(_ptr(x), _ptr(w), _ptr(out), M, N, K, int(activation), workspace.ptr,
                                  workspace.nbytes, _stream(stream)), "hstu_linear_fwd")
    return out


class LayerWorkspace(Workspace):
    """Device scratch of hstu_layer_paged_fwd (the paged call's workspace plus q, k, v, u and the gate)."""

    def __init__(self, p: HstuParams, d_model: int, max_batch: int, max_tokens: int, max_new: int, device=None,
                 stream=None):
        import torch

        n = load().hstu_workspace_size_layer(ctypes.byref(p), int(d_model), int(max_batch), int(max_tokens),
                                             int(max_new))
        if n == 0:
            raise HstuError("hstu_workspace_size_layer: unsupported parameters")
        self.nbytes = int(n)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buf.data_ptr()
        self.offset = (-base) % 256
        self.ptr = base + self.offset
        _check(load().hstu_workspace_init(self.ptr, self.nbytes, _stream(stream)), "hstu_workspace_init")


def layer_paged_fwd(p: HstuParams, d_model: int, x_new, w_qkvu, w_out, k_pages, v_pages, page_table, cached_lens,
                    new_lens, num_targets, rab, *, max_new: int, workspace: LayerWorkspace, out=None, stream=None):
    """hstu_layer_paged_fwd: one HSTU layer (SiLU QKVU projection, append, paged attention with its
    LayerNorm gate, output projection) for the new tokens.  Returns y [Tn, d_model] bf16."""
    import torch

    _check_args(p, elems=(("k_pages", k_pages), ("v_pages", v_pages)),
                ints=(("page_table", page_table), ("cached_lens", cached_lens), ("new_lens", new_lens),
                      ("num_targets", num_targets)), floats=(("rab", rab),))
    for name, t, shape in (("x_new", x_new, (x_new.shape[0], d_model)),
                           ("w_qkvu", w_qkvu, (4 * p.num_heads * p.head_dim, d_model)),
                           ("w_out", w_out, (d_model, p.num_heads * p.head_dim))):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape:
            raise HstuError(f"{name} must be bf16 {shape}, got {t.dtype} {tuple(t.shape)}")
    if out is None:
        out = torch.empty((x_new.shape[0], d_model), dtype=torch.bfloat16, device=x_new.device)
    B = cached_lens.shape[0]
    rc = load().hstu_layer_paged_fwd(ctypes.byref(p), int(d_model), _ptr(x_new), _ptr(w_qkvu), _ptr(w_out),
                                     _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(cached_lens),
                                     _ptr(new_lens), _ptr(num_targets), _ptr(rab), _ptr(out), B, x_new.shape[0],
                                     int(max_new), workspace.ptr, workspace.nbytes, _stream(stream))
    _check(rc, "hstu_layer_paged_fwd")
    return out


def ts_page_copy(src, dst, pairs, *, workspace: Workspace, stream=None):
    """hstu_ts_page_copy: timestamp pages [pages, P] int32 (CUDA or pinned host), page pairs[i, 0] of
    src to page pairs[i, 1] of dst -- the timestamp side of kv_page_copy's moves."""
    import torch

    for name, t in (("src", src), ("dst", dst)):
        if t.dtype != torch.int32 or t.dim() != 2:
            raise HstuError(f"{name} must be int32 [pages, page_size]")
    if src.shape[1] != dst.shape[1]:
        raise HstuError("src and dst page sizes differ")
    n = pairs.shape[0]
    if n == 0:
        return
    _check(load().hstu_ts_page_copy(_ptr_addressable(src, "src"), src.shape[0], _ptr_addressable(dst, "dst"),
                                    dst.shape[0], src.shape[1], _ptr_addressable(pairs, "pairs"), n, workspace.ptr,
                                    workspace.nbytes, _stream(stream)), "hstu_ts_page_copy")
