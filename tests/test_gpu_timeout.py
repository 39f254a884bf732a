"""The in-kernel time-out path of the tensor-core attention kernels, made to run out on purpose.

A test-only injection (hstu_test_inject) stops the V-tile producer from issuing its loads, so the
first wait on a V tile can never complete.  With a 20 ms limit on the waits between roles, the
kernel must give up, set HSTU_DEV_TIMEOUT, let every role drain its own copies and products,
release tensor memory and return -- well inside a second.  The next call, without the injection,
must be clean and correct.  Nothing faults, traps or waits without a limit: every wait in the
kernels is bounded (2 s for a CTA's own copies and products in flight).
"""
from __future__ import annotations

import time

import numpy as np
import pytest

from hstu_attention_b200 import inputs as gen

from .helpers import assert_close, gpu_jagged, gpu_paged, oracle_jagged, oracle_paged

LIMIT_NS = 20_000_000


@pytest.fixture(scope="module")
def hb():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import hstu_attention_b200 as hb

    hb.load()
    yield hb
    hb.test_inject(0)


def _paged_case():
    return gen.paged_case([300, 40, 1000], [16, 5, 16], [64, 3, 64], H=4, D=128, P=32, NB=64, n_max=1200,
                          num_pages=64, dtype="bf16", seed=77)


@pytest.mark.gpu
def test_paged_stalled_v_times_out_and_the_next_call_is_clean(hb):
    import torch

    c = _paged_case()
    _, ws, _, pool = gpu_paged(hb, c)              # warm: module load, descriptors
    assert ws.status() == 0
    hb.test_inject(hb.INJECT_STALL_V, LIMIT_NS)
    try:
        t0 = time.perf_counter()
        gpu_paged(hb, c, pool=pool, ws=ws)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        hb.test_inject(0)
    assert ws.status() & hb.DEV_TIMEOUT, "the stalled wait did not report a time-out"
    assert dt < 1.0, f"the aborted call took {dt:.2f} s (role limit 20 ms)"
    out, ws, _, _ = gpu_paged(hb, c, pool=pool, ws=ws)
    assert ws.status() == 0
    assert_close(out.cpu().view(torch.int16).numpy().view(np.uint16), oracle_paged(c), "bf16", "after the time-out")


@pytest.mark.gpu
def test_jagged_stalled_v_times_out_and_the_next_call_is_clean(hb):
    import torch

    c = gen.jagged_case([700, 90, 260], [64, 4, 16], H=2, D=128, NB=64, n_max=1024, dtype="bf16", seed=78)
    _, ws, _ = gpu_jagged(hb, c)
    assert ws.status() == 0
    hb.test_inject(hb.INJECT_STALL_V, LIMIT_NS)
    try:
        t0 = time.perf_counter()
        gpu_jagged(hb, c, ws=ws)
        dt = time.perf_counter() - t0
    finally:
        hb.test_inject(0)
    assert ws.status() & hb.DEV_TIMEOUT
    assert dt < 1.0, f"the aborted call took {dt:.2f} s (role limit 20 ms)"
    out, ws, _ = gpu_jagged(hb, c, ws=ws)
    assert ws.status() == 0
    assert_close(out.cpu().view(torch.int16).numpy().view(np.uint16), oracle_jagged(c), "bf16", "after the time-out")


def test_injection_arguments_are_checked():
    import ctypes

    import hstu_attention_b200 as hb

    lib = hb.load()
    assert lib.hstu_test_inject(2, LIMIT_NS) == -1                      # unknown kind
    assert lib.hstu_test_inject(hb.INJECT_STALL_V, 10) == -1            # limit below 1 ms
    assert lib.hstu_test_inject(hb.INJECT_STALL_V, 5_000_000_000) == -1  # above the 2 s drain limit
    assert lib.hstu_test_inject(0, 0) == 0
    assert ctypes.c_int(lib.hstu_test_inject(0, 123)).value == 0
