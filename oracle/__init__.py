"""Float64 CPU oracle for HSTU pointwise-aggregated attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (``hstu_attention_b200``) never does: the oracle
and the CUDA library share no code, and neither imports the other.

The arithmetic lives in ``hstu_oracle.c`` (plain loops in double precision); this module
only builds it with gcc and marshals numpy arrays through ctypes.  What the oracle
computes, and the passages it follows, are written at the top of ``hstu_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_hstu.so")
_lock = threading.Lock()
_lib = None

F32 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compile hstu_oracle.c into liboracle_hstu.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def bind(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    i32, i64, dbl, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_bucket.restype = ctypes.c_int
    lib.oracle_bucket.argtypes = [i64, i64, i32]
    lib.oracle_bucket_table.restype = None
    lib.oracle_bucket_table.argtypes = [i64, i64, i32, vp]
    lib.oracle_hstu_jagged.restype = ctypes.c_int
    lib.oracle_hstu_jagged.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, i32,
                                       i64, dbl, vp, i64, vp, vp, i32]
    lib.oracle_hstu_paged.restype = ctypes.c_int
    lib.oracle_hstu_paged.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                      vp, vp, vp, vp, i32, vp, i32, i64, dbl, vp, i64, vp, vp, i32]
    lib.oracle_hstu_jagged_bwd.restype = ctypes.c_int
    lib.oracle_hstu_jagged_bwd.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i64,
                                           ctypes.c_double, vp, vp, vp, vp, vp]
    lib.oracle_kv_append.restype = ctypes.c_int64
    lib.oracle_kv_append.argtypes = [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp,
                                     vp, vp, vp]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(ctypes.CDLL(build()))
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _elems(x: np.ndarray):
    """Return (contiguous array, elem_type): float32 as is; bf16 given as uint16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle inputs must be float32 or bf16 bits (uint16), got {x.dtype}")


def _same_type(*arrs):
    out, kinds = [], set()
    for a in arrs:
        c, k = _elems(a)
        out.append(c)
        kinds.add(k)
    if len(kinds) != 1:
        raise TypeError("all tensor inputs must share one element type")
    return out, kinds.pop()


def bucket(delta: int, n_max: int, num_buckets: int) -> int:
    return int(_load().oracle_bucket(int(delta), int(n_max), int(num_buckets)))


def bucket_table(n: int, n_max: int, num_buckets: int) -> np.ndarray:
    out = np.empty(int(n), dtype=np.int32)
    _load().oracle_bucket_table(int(n), int(n_max), int(num_buckets), _ptr(out))
    return out


def hstu_jagged(q, k, v, u, seq_offsets, num_targets, rab, n_max, eps=1e-5, rows=None,
                nthreads=None, return_o=False):
    """Jagged prefill.  q/k/v/u: [T, H, D] float32 or bf16 bits; returns float64 [rows, H, D]
    (and the pre-LayerNorm o rows too when ``return_o``)."""
    (q, k, v, u), et = _same_type(q, k, v, u)
    T, H, D = q.shape
    off = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    nt = np.ascontiguousarray(num_targets, dtype=np.int64)
    B = off.shape[0] - 1
    rab = np.ascontiguousarray(rab, dtype=np.float32)
    assert rab.shape[0] == H
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = T if r is None else r.shape[0]
    out = np.zeros((n_rows, H, D), dtype=np.float64)
    o = np.zeros((n_rows, H, D), dtype=np.float64) if return_o else None
    rc = _load().oracle_hstu_jagged(B, H, D, _ptr(off), _ptr(nt), _ptr(q), _ptr(k), _ptr(v), _ptr(u),
                                    et, _ptr(rab), rab.shape[1], int(n_max), float(eps), _ptr(r),
                                    n_rows, _ptr(out), _ptr(o), nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_hstu_jagged: inconsistent inputs (rc={rc})")
    return (out, o) if return_o else out


def hstu_jagged_bwd(q, k, v, u, dout, seq_offsets, num_targets, rab, n_max, eps=1e-5):
    """Gradients of the jagged prefill for upstream gradient ``dout`` (same shape and element
    type as q).  Returns float64 (dq, dk, dv, du) [T, H, D] and drab [H, NB]."""
    (q, k, v, u, dout), et = _same_type(q, k, v, u, dout)
    T, H, D = q.shape
    off = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    nt = np.ascontiguousarray(num_targets, dtype=np.int64)
    B = off.shape[0] - 1
    rab = np.ascontiguousarray(rab, dtype=np.float32)
    assert rab.shape[0] == H
    dq, dk, dv, du = (np.zeros((T, H, D), dtype=np.float64) for _ in range(4))
    drab = np.zeros(rab.shape, dtype=np.float64)
    rc = _load().oracle_hstu_jagged_bwd(B, H, D, _ptr(off), _ptr(nt), _ptr(q), _ptr(k), _ptr(v), _ptr(u),
                                        _ptr(dout), et, _ptr(rab), rab.shape[1], int(n_max), float(eps),
                                        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(du), _ptr(drab))
    if rc != 0:
        raise ValueError(f"oracle_hstu_jagged_bwd: inconsistent inputs (rc={rc})")
    return dq, dk, dv, du, drab


def hstu_paged(q_new, k_new, v_new, u_new, k_pages, v_pages, page_table, cached_lens, new_lens,
               num_targets, rab, n_max, eps=1e-5, rows=None, nthreads=None, return_o=False):
    """Paged cache hit.  Pages: [num_pages, H, P, D]; new tokens: [Tn, H, D]; float64 out
    (and the pre-LayerNorm o rows too when ``return_o``)."""
    (q_new, k_new, v_new, u_new, k_pages, v_pages), et = _same_type(
        q_new, k_new, v_new, u_new, k_pages, v_pages)
    Tn, H, D = q_new.shape
    num_pages, H2, P, D2 = k_pages.shape
    assert H2 == H and D2 == D
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    B, max_pages = pt.shape
    cl = np.ascontiguousarray(cached_lens, dtype=np.int64)
    nl = np.ascontiguousarray(new_lens, dtype=np.int64)
    nt = np.ascontiguousarray(num_targets, dtype=np.int64)
    rab = np.ascontiguousarray(rab, dtype=np.float32)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = Tn if r is None else r.shape[0]
    out = np.zeros((n_rows, H, D), dtype=np.float64)
    o = np.zeros((n_rows, H, D), dtype=np.float64) if return_o else None
    rc = _load().oracle_hstu_paged(B, H, D, P, num_pages, max_pages, _ptr(pt), _ptr(cl), _ptr(nl),
                                   _ptr(nt), _ptr(k_pages), _ptr(v_pages), _ptr(q_new), _ptr(k_new),
                                   _ptr(v_new), _ptr(u_new), et, _ptr(rab), rab.shape[1], int(n_max),
                                   float(eps), _ptr(r), n_rows, _ptr(out), _ptr(o),
                                   nthreads or default_threads())
    if rc == -2:
        raise ValueError("oracle_hstu_paged: page id out of range")
    if rc != 0:
        raise ValueError(f"oracle_hstu_paged: inconsistent inputs (rc={rc})")
    return (out, o) if return_o else out


def kv_append(k_pages, v_pages, page_table, k_new, v_new, cached_lens, new_offsets, append_lens) -> int:
    """In-place scatter of new K/V rows into the pages (raw bytes).  Returns skipped count."""
    assert k_pages.flags.c_contiguous and v_pages.flags.c_contiguous
    assert k_pages.dtype == k_new.dtype == v_new.dtype == v_pages.dtype
    num_pages, H, P, D = k_pages.shape
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    B, max_pages = pt.shape
    kn = np.ascontiguousarray(k_new)
    vn = np.ascontiguousarray(v_new)
    cl = np.ascontiguousarray(cached_lens, dtype=np.int64)
    no = np.ascontiguousarray(new_offsets, dtype=np.int64)
    al = np.ascontiguousarray(append_lens, dtype=np.int64)
    rc = _load().oracle_kv_append(B, H, D, P, num_pages, max_pages, k_pages.dtype.itemsize,
                                  _ptr(k_pages), _ptr(v_pages), _ptr(pt), _ptr(kn), _ptr(vn),
                                  _ptr(cl), _ptr(no), _ptr(al))
    return int(-rc)
