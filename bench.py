"""Benchmark: HSTU paged cache-hit attention, new tokens/s on B200.

Workload (one "step"): the paged cache-hit ranking batch -- 8 users, cached histories
U[1024, 4096] tokens, 16 new action tokens + 64 candidates per user, 4 heads x 128, page
size 32, a 65,536-page bf16 KV pool -- through an 8-layer stack, each layer with its own
pages: per layer hstu_kv_append (16 tokens/user) then hstu_attn_paged_fwd (80 tokens/user).
Inputs are seeded synthetic tensors shaped like the serving benchmark of the NVIDIA HSTU
deployment blog (KuaiRand-1K itself is not available here).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own replica of the batch
on its own GPU (weak scaling, no collective on the data path); the time is the max over
ranks.  The step is captured in one CUDA graph and timed with CUDA events; the 8 layers
read ~340 MB of distinct pages and tokens per step, more than the 126 MB L2, so no flush is needed.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hstu_attention_b200 import inputs as gen  # noqa: E402

METRIC = "HSTU paged-attn new tokens/s per B200; % of BF16 tensor / HBM roofline"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per paged call on one layer of this
# batch, from one `ncu --set full` capture of the attention and LayerNorm kernels (ncu flushes
# caches, so the LayerNorm kernel's partial-plane reads show up as DRAM reads).  Valid only for
# the kernel sources they were taken from (hash below); otherwise the bench reports traffic as null.
PAGED_TRAFFIC_BYTES = 41.913088e6 + 4.096e3 + 6.407e6
PAGED_FILES = ("attn_paged.cu", "combine.cu")
PAGED_TRAFFIC_SOURCES = "6ba38f878f0500ea"
# the same kind of capture for the jagged prefill attention kernel
PREFILL_TRAFFIC_BYTES = 63.091712e6 + 11.832832e6
PREFILL_TRAFFIC_SOURCES = "b12b4d1a3bd60a89"
# long-history attention kernel: DRAM bytes of one call on the batch's first 8 users (the capture
# size rule), 381.17 MB against 371.60 MB of algorithmic bytes; the full call's traffic is scaled
# by that ratio (traffic grows with the pages read)
LONG_TRAFFIC_RATIO = 381.17e6 / 371602680
# backward dQ/drab kernel (the call's dominant kernel) on the prefill batch, per launch
BWD_DQ_TRAFFIC_BYTES = 85.852928e6 + 13.68832e6
BWD_TRAFFIC_SOURCES = "59548f9c264f2571"       # hash of attn_bwd_tc.cu
# projection GEMM (640 x 2048 x 512, SiLU) per launch
GEMM_TRAFFIC_BYTES = 2.769e6
GEMM_TRAFFIC_SOURCES = "65ee9d0fc18e6424"      # hash of gemm.cu


# headers every kernel includes (wait loops, descriptors, argument blocks)
SHARED_KERNEL_HEADERS = ("sm100.cuh", "common.cuh", "kernels.cuh")


def kernel_sources_hash(files) -> str:
    """Hash of the kernels' source code (the listed files and the shared headers) with comments
    and blank space removed (editing a comment does not change the kernel the counters were
    taken from)."""
    import hashlib
    import re

    h = hashlib.sha256()
    for f in tuple(files) + SHARED_KERNEL_HEADERS:
        with open(os.path.join(ROOT, "hstu_attention_b200", "csrc", f), encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", " ", src).strip().encode())
    return h.hexdigest()[:16]
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------------------- replicas


def max_over_ranks(x: float, device=None) -> float:
    """The largest of every rank's x (the job time of weak-scaled replicas); x itself when the
    process group is not initialised.  NCCL ranks pass their CUDA device, gloo ranks the CPU."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, ms_per_step: float, world: int) -> float:
    """Whole-job units/s of `world` replicas that each process units_per_rank_step per step,
    with ms_per_step the max over ranks."""
    return units_per_rank_step * world / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons (every 100 ms, into a file) while the
    timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        import tempfile

        self.path = os.path.join(tempfile.gettempdir(), f"hstu_bench_clocks_gpu{index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.remove(self.path)
        except OSError:
            pass

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [v for v in (num(r[1]) for r in rows) if v is not None]
        mx = [v for v in (num(r[2]) for r in rows) if v is not None]
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "timed steps plus >= 0.3 s of identical graph replays before and after"}


# ----------------------------------------------------------------------------- workload


def workload_stats(layers):
    """Algorithmic bytes and FLOPs of the paged calls, and the new-token count."""
    tokens = int(layers[0].Tn)
    per_layer_bytes, per_layer_flops = [], []
    for c in layers:
        HD = c.H * c.D
        cached = int(np.sum(c.cached_lens))
        # cached K and V read once; q, k, v, u of new tokens read; out written (all bf16);
        # the page-table entries of the cached pages (int32)
        pages = int(np.sum((c.cached_lens + c.P - 1) // c.P))
        nbytes = cached * HD * 2 * 2 + c.Tn * HD * 2 * 5 + pages * 4
        pairs = 0
        for C, N, T in zip(c.cached_lens, c.new_lens, c.num_targets):
            C, N, T = int(C), int(N), int(T)
            hist = C + N - T
            for r in range(N):
                i = C + r
                pairs += (i + 1) if i < hist else (hist + 1)
        per_layer_bytes.append(nbytes)
        per_layer_flops.append(4 * c.D * pairs * c.H)
    return tokens, per_layer_bytes, per_layer_flops


def setup_device(layers, device):
    import torch

    import hstu_attention_b200 as hb

    c0 = layers[0]
    num_pages = c0.num_pages
    shape = (num_pages, c0.H, c0.P, c0.D)
    kp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    vp = torch.zeros(shape, dtype=torch.bfloat16, device=device)

    def d(x):
        x = np.ascontiguousarray(x)
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        if x.dtype == np.int64:
            x = x.astype(np.int32)
        return torch.from_numpy(x).to(device)

    L = []
    max_pages = max(c.max_pages for c in layers)
    for c in layers:
        ids = torch.from_numpy(c.page_ids.astype(np.int64)).to(device)
        kp[ids] = d(c.pool_k)
        vp[ids] = d(c.pool_v)
        pt = np.full((c.B, max_pages), -1, dtype=np.int32)
        pt[:, :c.max_pages] = c.page_table
        L.append(dict(q=d(c.q_new), k=d(c.k_new), v=d(c.v_new), u=d(c.u_new), pt=d(pt), cl=d(c.cached_lens),
                      nl=d(c.new_lens), nt=d(c.num_targets), rab=d(c.rab), out=torch.empty_like(d(c.q_new))))
    # nothing in the step writes the page tables or the lengths, so each layer's attention may
    # start its set-up while the previous layer's LayerNorm kernel finishes
    p = hb.params(c0.H, c0.D, torch.bfloat16, c0.NB, c0.n_max, page_size=c0.P, num_pages=num_pages,
                  max_pages_per_user=max_pages, flags=hb.FLAG_OVERLAP_PREVIOUS)
    ws = hb.Workspace(p, c0.B, c0.Tn, c0.max_new, device=device)
    return p, ws, kp, vp, L


def run_step(hb, p, ws, kp, vp, L, max_new, events=None, side=None):
    """One step: per layer kv_append of the 16 new history tokens and paged attention of all
    80 new tokens.  The attention reads the new keys from k_new/v_new, not from the pages, so
    the appends do not feed it: with a side stream they run concurrently (fork at the start of
    the step, join at the end)."""
    import torch

    main = torch.cuda.current_stream()
    if side is not None:
        side.wait_stream(main)
    for li, t in enumerate(L):
        if side is not None:
            with torch.cuda.stream(side):
                hb.kv_append(p, kp, vp, t["pt"], t["k"], t["v"], t["cl"], t["nl"], t["nt"], max_new=max_new,
                             workspace=ws, stream=side)
        else:
            hb.kv_append(p, kp, vp, t["pt"], t["k"], t["v"], t["cl"], t["nl"], t["nt"], max_new=max_new,
                         workspace=ws)
        if events is not None:
            events[li][0].record()
        hb.paged_fwd(p, t["q"], t["k"], t["v"], t["u"], kp, vp, t["pt"], t["cl"], t["nl"], t["nt"], t["rab"],
                     max_new=max_new, workspace=ws, out=t["out"])
        if events is not None:
            events[li][1].record()
    if side is not None:
        main.wait_stream(side)


def bench_prefill(hb, device, steps, warmup, peaks):
    """Secondary line: jagged prefill (8 users, lengths U[256, 4096]) against the tensor peak."""
    import torch

    c = gen.config2_prefill()
    d = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)  # noqa
    q, k, v, u = d(c.q), d(c.k), d(c.v), d(c.u)
    off = torch.from_numpy(c.seq_offsets.astype(np.int32)).to(device)
    nt = torch.from_numpy(c.num_targets.astype(np.int32)).to(device)
    rab = torch.from_numpy(c.rab).to(device)
    # nothing between the calls writes seq_offsets / num_targets: each call's set-up may overlap
    # the previous call's LayerNorm kernel
    p = hb.params(c.H, c.D, torch.bfloat16, c.NB, c.n_max, flags=hb.FLAG_OVERLAP_PREVIOUS)
    ws = hb.Workspace(p, c.B, c.T, 4096, device=device)
    out = torch.empty_like(q)
    # rotate three copies of q/k/v/u (3 x 83 MB, more than the 126 MB L2) so that each timed call
    # reads its inputs from HBM
    sets = [(q, k, v, u)] + [(q.clone(), k.clone(), v.clone(), u.clone()) for _ in range(2)]
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        a = sets[i % len(sets)]
        hb.jagged_fwd(p, *a, off, nt, rab, max_seqlen=4096, workspace=ws, out=out)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for a in sets:
            hb.jagged_fwd(p, *a, off, nt, rab, max_seqlen=4096, workspace=ws, out=out)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (len(sets) * steps)
    pairs = 0
    for L, T in zip(c.lengths, c.num_targets):
        hist = int(L - T)
        pairs += hist * (hist + 1) // 2 + int(T) * (hist + 1)
    flops = 4 * c.D * pairs * c.H
    tf = flops / (ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    assert ws.status() == 0
    return {"workload": "jagged prefill: 8 users, lengths U[256,4096] (seed 1002), 64 candidates, H=4, D=128",
            "tokens": int(c.T), "ms_per_call": ms, "tokens_per_s": c.T / (ms * 1e-3), "tflops": tf,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "traffic": (PREFILL_TRAFFIC_BYTES if kernel_sources_hash(("attn_tc.cu",)) ==
                                     PREFILL_TRAFFIC_SOURCES else None),
                         "traffic_kernel": "attn_tc_kernel (jagged) per launch"},
            "launches_per_call": 2}


def _to_dev(x, device):
    import torch

    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    if x.dtype == np.int64:
        x = x.astype(np.int32)
    return torch.from_numpy(x).to(device)


def paged_pairs(c) -> int:
    """Unmasked (query, key) pairs per head of a paged call."""
    pairs = 0
    for C, N, T in zip(c.cached_lens, c.new_lens, c.num_targets):
        C, N, T = int(C), int(N), int(T)
        hist = C + N - T
        q = np.arange(C, C + N)
        pairs += int(np.sum(np.where(q < hist, q + 1, hist + 1)))
    return pairs


def jagged_pairs(lengths, targets) -> int:
    pairs = 0
    for L, T in zip(lengths, targets):
        hist = int(L) - int(T)
        pairs += hist * (hist + 1) // 2 + int(T) * (hist + 1)
    return pairs


def graph_ms(graph, steps, stream) -> float:
    """Mean ms per replay of `graph` over `steps` replays (CUDA events on `stream`)."""
    import torch

    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def bench_long_history(hb, device, steps, warmup, peaks, with_cpu):
    """Sub-line: the long-history cache hit (32 users, cached U[8192,16384], 256 candidates,
    H=8, P=64): one paged call per step, 1.69 GB of distinct pages (more than L2)."""
    import torch

    c = gen.config4_long()
    p = hb.params(c.H, c.D, torch.bfloat16, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                  max_pages_per_user=c.max_pages, flags=hb.FLAG_OVERLAP_PREVIOUS)
    shape = (c.num_pages, c.H, c.P, c.D)
    kp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    vp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    ids = torch.from_numpy(c.page_ids.astype(np.int64)).to(device)
    kp[ids] = _to_dev(c.pool_k, device)
    vp[ids] = _to_dev(c.pool_v, device)
    t = [_to_dev(x, device) for x in (c.q_new, c.k_new, c.v_new, c.u_new)]
    meta = [_to_dev(x, device) for x in (c.page_table, c.cached_lens, c.new_lens, c.num_targets, c.rab)]
    ws = hb.Workspace(p, c.B, c.Tn, c.max_new, device=device)
    out = torch.empty_like(t[0])
    for _ in range(warmup):
        hb.paged_fwd(p, *t, kp, vp, *meta, max_new=c.max_new, workspace=ws, out=out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hb.paged_fwd(p, *t, kp, vp, *meta, max_new=c.max_new, workspace=ws, out=out)
    ms = graph_ms(g, steps, torch.cuda.current_stream())
    assert ws.status() == 0
    HD = c.H * c.D
    pages = int(np.sum((c.cached_lens + c.P - 1) // c.P))
    nbytes = int(np.sum(c.cached_lens)) * HD * 2 * 2 + c.Tn * HD * 2 * 5 + pages * 4
    flops = 4 * c.D * c.H * paged_pairs(c)
    gbs = nbytes / (ms * 1e-3) / 1e9
    tf = flops / (ms * 1e-3) / 1e12
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    bf16 = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    line = {"workload": "long-history cache hit: 32 users, cached U[8192,16384] (seed 1004), 256 candidates, "
                        "H=8, D=128, P=64, NB=256, n_max=16640; one paged call per step",
            "new_tokens": int(c.Tn), "ms_per_call": ms, "new_tokens_per_s": c.Tn / (ms * 1e-3),
            "algorithmic_bytes_per_call": nbytes, "flops_per_call": flops,
            "roofline": {"bound": "hbm and tensor (at the ridge)", "achieved_gbs": gbs, "hbm_peak_gbs": hbm,
                         "hbm_frac": gbs / hbm, "achieved_tflops": tf, "bf16_peak_tflops": bf16,
                         "tensor_frac": tf / bf16, "frac": max(gbs / hbm, tf / bf16),
                         "traffic": (LONG_TRAFFIC_RATIO * nbytes
                                     if kernel_sources_hash(PAGED_FILES) == PAGED_TRAFFIC_SOURCES else None),
                         "traffic_note": "ncu DRAM bytes of the attention kernel on the first 8 users, scaled to "
                                         "the full call by algorithmic bytes (1.03x algorithmic)"},
            "l2": "inputs larger than L2 (1.69 GB of distinct pages per call)"}
    if with_cpu:
        import oracle

        # seeded subset: the first user's 256 rows, extrapolated by unmasked pairs
        sub = dataclasses.replace(c, cached_lens=c.cached_lens[:1], new_lens=c.new_lens[:1],
                                  num_targets=c.num_targets[:1], page_table=c.page_table[:1])
        ck, cv, cpt = sub.compact_pool()
        nthreads = oracle.default_threads()
        t0 = time.perf_counter()
        oracle.hstu_paged(sub.q_new[:int(sub.Tn)], sub.k_new[:int(sub.Tn)], sub.v_new[:int(sub.Tn)],
                          sub.u_new[:int(sub.Tn)], ck, cv, cpt, sub.cached_lens, sub.new_lens, sub.num_targets,
                          sub.rab, sub.n_max, sub.eps, nthreads=nthreads)
        dt = time.perf_counter() - t0
        scale = paged_pairs(c) / max(1, paged_pairs(sub))
        line["cpu_baseline"] = {"value": c.Tn / (dt * scale), "unit": "new tokens/s", "cores": nthreads,
                                "kind": "oracle", "sample": f"user 0 only (256 rows, {dt:.2f} s), extrapolated "
                                                            f"to the whole call by unmasked pairs (x{scale:.1f})"}
    del kp, vp, ws, g
    torch.cuda.empty_cache()
    return line


def bench_mixed(hb, device, steps, warmup, peaks, with_cpu):
    """Sub-line: the mixed serving batch as one step -- the 64 hits append their new history
    tokens and run the paged cache hit; the 64 misses run jagged prefill of history plus
    candidates and then append their history into pages (one shared 262,144-page pool)."""
    import torch

    hits, misses, miss_pt, miss_hist = gen.config5_mixed()
    flags = hb.FLAG_OVERLAP_PREVIOUS
    ph = hb.params(hits.H, hits.D, torch.bfloat16, hits.NB, hits.n_max, page_size=hits.P, num_pages=hits.num_pages,
                   max_pages_per_user=hits.max_pages, flags=flags)
    pm = hb.params(hits.H, hits.D, torch.bfloat16, hits.NB, hits.n_max, page_size=hits.P, num_pages=hits.num_pages,
                   max_pages_per_user=int(miss_pt.shape[1]), flags=flags)
    pj = hb.params(misses.H, misses.D, torch.bfloat16, misses.NB, misses.n_max, flags=flags)
    shape = (hits.num_pages, hits.H, hits.P, hits.D)
    kp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    vp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    ids = torch.from_numpy(hits.page_ids.astype(np.int64)).to(device)
    kp[ids] = _to_dev(hits.pool_k, device)
    vp[ids] = _to_dev(hits.pool_v, device)
    ht = [_to_dev(x, device) for x in (hits.q_new, hits.k_new, hits.v_new, hits.u_new)]
    hmeta = [_to_dev(x, device) for x in (hits.page_table, hits.cached_lens, hits.new_lens, hits.num_targets)]
    hrab = _to_dev(hits.rab, device)
    mt = [_to_dev(x, device) for x in (misses.q, misses.k, misses.v, misses.u)]
    moff, mnt, mrab = (_to_dev(x, device) for x in (misses.seq_offsets, misses.num_targets, misses.rab))
    mpt, mzero, mlen = (_to_dev(x, device) for x in (miss_pt, np.zeros(misses.B, np.int32), misses.lengths))
    max_seq = int(misses.max_seqlen)
    ws = hb.Workspace(ph, max(hits.B, misses.B), max(hits.Tn, misses.T), max(hits.max_new, max_seq), device=device)
    hout, mout = torch.empty_like(ht[0]), torch.empty_like(mt[0])

    def step():
        hb.kv_append(ph, kp, vp, hmeta[0], ht[1], ht[2], hmeta[1], hmeta[2], hmeta[3], max_new=hits.max_new,
                     workspace=ws)
        hb.paged_fwd(ph, *ht, kp, vp, *hmeta, hrab, max_new=hits.max_new, workspace=ws, out=hout)
        hb.jagged_fwd(pj, *mt, moff, mnt, mrab, max_seqlen=max_seq, workspace=ws, out=mout)
        hb.kv_append(pm, kp, vp, mpt, mt[1], mt[2], mzero, mlen, mnt, max_new=max_seq, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert ws.status() == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    ms = graph_ms(g, steps, torch.cuda.current_stream())
    assert ws.status() == 0
    tokens = int(hits.Tn + misses.T)
    hit_flops = 4 * hits.D * hits.H * paged_pairs(hits)
    miss_flops = 4 * misses.D * misses.H * jagged_pairs(misses.lengths, misses.num_targets)
    tf = (hit_flops + miss_flops) / (ms * 1e-3) / 1e12
    bf16 = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    line = {"workload": "mixed serving batch (seed 1005): 128 users, history lognormal(ln 2000, 1) clipped "
                        "[64, 32768], candidates U[16,512]; 64 hits (append 8-32 + paged attention), 64 misses "
                        "(jagged prefill + append of the history), H=4, D=128, P=32, 262,144-page pool",
            "tokens": tokens, "hit_new_tokens": int(hits.Tn), "miss_tokens": int(misses.T), "ms_per_step": ms,
            "tokens_per_s": tokens / (ms * 1e-3), "flops_per_step": hit_flops + miss_flops, "tflops": tf,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16},
            "launches_per_step": 6, "l2": "inputs larger than L2 (about 2.1 GB of pages and tokens per step)"}
    if with_cpu:
        import oracle

        # seeded subset: the two shortest hits (paged oracle) and the two shortest misses (prefill
        # oracle), extrapolated to the whole step by unmasked pairs
        nthreads = oracle.default_threads()
        # the 3 hits and 3 misses closest to the median length: a representative sample of a few s
        hsel = np.argsort(np.abs(hits.cached_lens - np.median(hits.cached_lens)), kind="stable")[:3]
        msel = np.argsort(np.abs(misses.lengths - np.median(misses.lengths)), kind="stable")[:3]
        t0 = time.perf_counter()
        pairs_done = 0
        for b in hsel:
            o0, o1 = int(hits.new_offsets[b]), int(hits.new_offsets[b + 1])
            sub = dataclasses.replace(hits, cached_lens=hits.cached_lens[b:b + 1], new_lens=hits.new_lens[b:b + 1],
                                      num_targets=hits.num_targets[b:b + 1], page_table=hits.page_table[b:b + 1])
            ck, cv, cpt = sub.compact_pool()
            oracle.hstu_paged(hits.q_new[o0:o1], hits.k_new[o0:o1], hits.v_new[o0:o1], hits.u_new[o0:o1], ck, cv,
                              cpt, sub.cached_lens, sub.new_lens, sub.num_targets, hits.rab, hits.n_max, hits.eps,
                              nthreads=nthreads)
            pairs_done += paged_pairs(sub) * hits.H
        for b in msel:
            s0, s1 = int(misses.seq_offsets[b]), int(misses.seq_offsets[b + 1])
            oracle.hstu_jagged(misses.q[s0:s1], misses.k[s0:s1], misses.v[s0:s1], misses.u[s0:s1], [0, s1 - s0],
                               misses.num_targets[b:b + 1], misses.rab, misses.n_max, misses.eps)
            pairs_done += jagged_pairs([s1 - s0], [misses.num_targets[b]]) * misses.H
        dt = time.perf_counter() - t0
        scale = (hit_flops + miss_flops) / (4 * hits.D) / max(1, pairs_done)
        line["cpu_baseline"] = {"value": tokens / (dt * scale), "unit": "tokens/s", "cores": nthreads,
                                "kind": "oracle", "sample": f"the 3 hits and 3 misses nearest the median length "
                                                            f"({dt:.2f} s), extrapolated by unmasked pairs "
                                                            f"(x{scale:.0f})"}
    del kp, vp, ws, g
    torch.cuda.empty_cache()
    return line


def bench_backward(hb, device, steps, warmup, peaks, with_cpu):
    """Sub-line: the backward pass of jagged attention on the prefill batch (8 users, lengths
    U[256,4096], 64 candidates, H=4, D=128, NB=128): o recomputed by the forward kernels, the
    LayerNorm-gate backward, then the tensor-core dQ/drab and dK/dV kernels.  Three seeded input
    sets rotate so consecutive calls do not find their inputs in L2."""
    import torch

    sets = []
    for seed in (1002, 2002, 3002):
        c = gen.config2_prefill(seed=seed)
        dout = gen._values(np.random.default_rng(seed + 7), c.q.shape, 1.0, "bf16")
        sets.append((c, [_to_dev(x, device) for x in (c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab,
                                                       dout)]))
    c0 = sets[0][0]
    T = max(int(c.T) for c, _ in sets)
    ms_len = max(int(c.max_seqlen) for c, _ in sets)
    p = hb.params(c0.H, c0.D, torch.bfloat16, c0.NB, c0.n_max, ln_eps=c0.eps)
    ws = hb.BwdWorkspace(p, T, device=device)
    for i in range(warmup):
        hb.jagged_bwd(p, *sets[i % 3][1], max_seqlen=ms_len, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        hb.jagged_bwd(p, *sets[i % 3][1], max_seqlen=ms_len, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ms = e0.elapsed_time(e1) / steps
    flops = float(np.mean([10 * c.D * c.H * jagged_pairs(np.diff(c.seq_offsets), c.num_targets) for c, _ in sets]))
    tf = flops / (ms * 1e-3) / 1e12
    bf16 = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    line = {"workload": "backward of jagged attention on the prefill batch (seeds 1002/2002/3002 rotated): 8 users, "
                        "lengths U[256,4096], 64 candidates, H=4, D=128, NB=128; dq, dk, dv, du (fp32) and drab",
            "tokens": int(np.mean([c.T for c, _ in sets])), "ms_per_call": ms,
            "algorithmic_flops_per_call": flops,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16,
                         "note": "algorithmic FLOPs = 10 D H pairs (S recomputed, dP, dQ, dK, dV: 2.5x the forward); "
                                 "the call also recomputes o with the forward kernels and runs the LayerNorm backward",
                         "traffic": (BWD_DQ_TRAFFIC_BYTES if kernel_sources_hash(("attn_bwd_tc.cu",)) ==
                                     BWD_TRAFFIC_SOURCES else None),
                         "traffic_kernel": "bwd_dq_kernel (48 % of the call in the ncu launch list) per launch"},
            "launches_per_call": 5}
    if with_cpu:
        from oracle.dense_bwd import jagged_bwd_dense

        c, _ = sets[0]
        dout = gen._values(np.random.default_rng(1009), c.q.shape, 1.0, "bf16")
        t0 = time.perf_counter()
        jagged_bwd_dense(c.q, c.k, c.v, c.u, dout, c.seq_offsets, c.num_targets, c.rab, c.n_max, c.eps)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": c.T / dt, "unit": "tokens/s", "kind": "oracle",
                                "cores": os.cpu_count(),
                                "sample": f"the whole first batch ({dt:.1f} s) on the dense float64 restatement of the "
                                          "oracle backward (numpy matmuls on all host cores)"}
    del ws
    torch.cuda.empty_cache()
    return line


def bench_layer_stack(hb, device, steps, warmup, peaks, with_cpu):
    """Sub-line: 8 whole HSTU layers on the paged cache hit, chained (layer l's output is layer
    l+1's input): per layer the SiLU QKVU projection, the append, the paged attention with its
    LayerNorm gate and the output projection, d_model = 512, seeded random weights per layer, each
    layer with its own pages (the benchmark batch: 8 users, cached U[1024,4096], 16 appended +
    64 candidates, H=4, D=128, P=32)."""
    import torch

    layers = gen.config3_paged_layers()
    d_model = 512
    c0 = layers[0]
    HD = c0.H * c0.D
    p = hb.params(c0.H, c0.D, torch.bfloat16, c0.NB, c0.n_max, page_size=c0.P, num_pages=c0.num_pages,
                  max_pages_per_user=max(c.max_pages for c in layers), flags=hb.FLAG_OVERLAP_PREVIOUS)
    shape = (c0.num_pages, c0.H, c0.P, c0.D)
    kp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    vp = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    rng = np.random.default_rng(2024)
    meta, weights = [], []
    for c in layers:
        ids = torch.from_numpy(c.page_ids.astype(np.int64)).to(device)
        kp[ids] = _to_dev(c.pool_k, device)
        vp[ids] = _to_dev(c.pool_v, device)
        pt = np.full((c.B, p.max_pages_per_user), -1, np.int32)
        pt[:, :c.page_table.shape[1]] = c.page_table
        meta.append([_to_dev(x, device) for x in (pt, c.cached_lens, c.new_lens, c.num_targets, c.rab)])
        weights.append([_to_dev(gen._values(rng, (4 * HD, d_model), 1.0 / np.sqrt(d_model), "bf16"), device),
                        _to_dev(gen._values(rng, (d_model, HD), 1.0 / np.sqrt(HD), "bf16"), device)])
    Tn = int(c0.Tn)
    max_new = max(c.max_new for c in layers)
    x0 = _to_dev(gen._values(rng, (Tn, d_model), 1.0, "bf16"), device)
    acts = [torch.empty((Tn, d_model), dtype=torch.bfloat16, device=device) for _ in layers]
    ws = hb.LayerWorkspace(p, d_model, c0.B, Tn, max_new, device=device)

    def step():
        x = x0
        for li in range(len(layers)):
            hb.layer_paged_fwd(p, d_model, x, weights[li][0], weights[li][1], kp, vp, *meta[li][:4], meta[li][4],
                               max_new=max_new, workspace=ws, out=acts[li])
            x = acts[li]

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert ws.status() == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    ms = graph_ms(g, steps, torch.cuda.current_stream())
    assert ws.status() == 0
    # the projection GEMM alone, at the layer's shapes (tensor bound)
    lw = hb.Workspace(p, 1, 1, 1, device=device)
    xq = acts[0]
    qkvu_out = torch.empty((Tn, 4 * HD), dtype=torch.bfloat16, device=device)
    gq = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gq):
        for _ in range(8):
            hb.linear_fwd(xq, weights[0][0], activation=1, workspace=lw, out=qkvu_out)
    ms_gemm = graph_ms(gq, steps, torch.cuda.current_stream()) / 8
    proj_flops = 2 * Tn * d_model * 4 * HD + 2 * Tn * HD * d_model
    attn_flops = sum(4 * c.D * c.H * paged_pairs(c) for c in layers)
    flops = proj_flops * len(layers) + attn_flops
    bf16 = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    gemm_tf = 2 * Tn * d_model * 4 * HD / (ms_gemm * 1e-3) / 1e12
    line = {"workload": "8 chained HSTU layers on the paged cache hit (seed 1003): per layer SiLU QKVU projection "
                        "(d_model 512 -> 4 x 512), append, paged attention + LayerNorm gate, output projection "
                        "(512 -> 512); 8 users, cached U[1024,4096], 16 appended + 64 candidates, H=4, D=128, P=32; "
                        "seeded random weights",
            "new_tokens": Tn, "ms_per_step": ms, "new_tokens_per_s": Tn / (ms * 1e-3), "ms_per_layer": ms / len(layers),
            "flops_per_step": flops, "tflops": flops / (ms * 1e-3) / 1e12,
            "projection_gemm": {"shape": f"{Tn} x {4 * HD} x {d_model}, SiLU epilogue", "ms": ms_gemm,
                                "roofline": {"bound": "tensor", "achieved": gemm_tf, "peak": bf16, "unit": "TFLOP/s",
                                             "frac": gemm_tf / bf16,
                                             "traffic": (GEMM_TRAFFIC_BYTES if kernel_sources_hash(("gemm.cu",)) ==
                                                         GEMM_TRAFFIC_SOURCES else None),
                                             "note": "5 x 16 output tiles on 148 SMs: a latency-bound small GEMM"}},
            "launches_per_step": 6 * len(layers)}
    if with_cpu:
        from oracle import hstu_layer as hl

        c = layers[0]
        sub = dataclasses.replace(c, cached_lens=c.cached_lens[:1], new_lens=c.new_lens[:1],
                                  num_targets=c.num_targets[:1], page_table=c.page_table[:1])
        ck, cv, cpt = sub.compact_pool()
        n0 = int(c.new_lens[0])
        xs = gen.as_f32(gen._values(np.random.default_rng(5), (n0, d_model), 1.0, "bf16")).astype(np.float64)
        w1 = gen.as_f32(host_bits(weights[0][0])).astype(np.float64)
        w2 = gen.as_f32(host_bits(weights[0][1])).astype(np.float64)
        t0 = time.perf_counter()
        hl.layer_paged(xs, w1, w2, ck, cv, cpt, sub.cached_lens, sub.new_lens, sub.num_targets, c.rab, c.n_max)
        dt = time.perf_counter() - t0
        scale = len(layers) * c.B
        line["cpu_baseline"] = {"value": Tn / (dt * scale), "unit": "new tokens/s", "kind": "oracle",
                                "cores": __import__("oracle").default_threads(),
                                "sample": f"one user of layer 0 ({n0} rows, {dt:.2f} s), scaled by 8 users x 8 layers"}
    del kp, vp, ws, g, gq
    torch.cuda.empty_cache()
    return line


def host_bits(t):
    """A bf16 CUDA tensor as uint16 bit patterns on the host."""
    import torch

    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bench_cache_ops(hb, device, steps, warmup, peaks):
    """Sub-line: the cache-management copies at the paged configuration's page shape (H=4, D=128,
    P=32, bf16: 32 KB of K and 32 KB of V per page) and the host manager's prepare latency.
      onboard -- the cached pages of layer 0's 8 users (seed 1003, 640 pages) from a pinned host
                 pool into their scattered GPU pages, one kv_page_copy;
      offload -- the same pages from the GPU pool back to the host pool;
      compact -- 16,384 scattered pages moved within the 65,536-page GPU pool (disjoint sets).
    The host-link copies are set against one contiguous cudaMemcpyAsync of the same number of
    bytes between the same pinned buffer and device memory (the DMA engines' rate on this machine);
    the in-pool move against HBM bandwidth."""
    import torch

    layer = gen.config3_paged_layers(layers=1)[0]
    H, D, P, G = layer.H, layer.D, layer.P, layer.num_pages
    p = hb.params(H, D, torch.bfloat16, layer.NB, layer.n_max, page_size=P, num_pages=G,
                  max_pages_per_user=layer.max_pages)
    ws = hb.Workspace(p, 1, 1, 1, device=device)
    gk = torch.zeros((G, H, P, D), dtype=torch.bfloat16, device=device)
    gv = torch.zeros_like(gk)
    gpu_pages = np.concatenate([layer.page_table[b, :(int(layer.cached_lens[b]) + P - 1) // P]
                                for b in range(layer.B)]).astype(np.int32)
    n = len(gpu_pages)
    hk = torch.zeros((n, H, P, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros((n, H, P, D), dtype=torch.bfloat16).pin_memory()
    on = torch.from_numpy(np.stack([np.arange(n, dtype=np.int32), gpu_pages], 1)).to(device)
    off = torch.from_numpy(np.stack([gpu_pages, np.arange(n, dtype=np.int32)], 1)).to(device)
    rng = np.random.default_rng(7)
    perm = rng.permutation(G).astype(np.int32)
    moves = torch.from_numpy(np.stack([perm[:16384], perm[16384:32768]], 1)).to(device)
    page_bytes = H * P * D * 2 * 2
    stream = torch.cuda.current_stream()

    def timed(fn, reps):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ms_on = timed(lambda: hb.kv_page_copy(p, hk, hv, gk, gv, on, workspace=ws), steps)
    ms_off = timed(lambda: hb.kv_page_copy(p, gk, gv, hk, hv, off, workspace=ws), steps)
    ms_mv = timed(lambda: hb.kv_page_copy(p, gk, gv, gk, gv, moves, workspace=ws), steps)
    assert ws.status() == 0
    # the DMA reference: the same bytes as one contiguous copy each way
    dflat = torch.empty(n * page_bytes // 2, dtype=torch.bfloat16, device=device)
    hflat = torch.cat([hk.reshape(-1), hv.reshape(-1)]).pin_memory()
    ms_h2d = timed(lambda: dflat.copy_(hflat, non_blocking=True), steps)
    ms_d2h = timed(lambda: hflat.copy_(dflat, non_blocking=True), steps)
    nb = n * page_bytes

    def gbs(nbytes, ms):
        return nbytes / (ms * 1e-3) / 1e9

    # the host manager: a 65,536-page GPU tier and a 16,384-page host tier kept full by misses
    cache = hb.KVCache(G, 16384, P, 256)
    lat = []
    uid = 0
    for i in range(3000):
        ids = list(range(uid, uid + layer.B))
        uid += layer.B
        t0 = time.perf_counter()
        cache.prepare(ids, [int(x) for x in rng.integers(1024, 4096, layer.B)])
        lat.append(time.perf_counter() - t0)
    st = cache.stats()
    cache.close()
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    line = {"workload": "cache copies at H=4, D=128, P=32 bf16 (64 KB of K+V per page): onboard/offload of layer "
                        f"0's {n} cached pages (seed 1003) between a pinned host pool and the 65,536-page GPU pool; "
                        "compaction move of 16,384 scattered pages within the GPU pool",
            "onboard": {"pages": n, "bytes": nb, "ms": ms_on, "gbs": gbs(nb, ms_on),
                        "dma_contiguous_gbs": gbs(nb, ms_h2d), "frac_of_dma": ms_h2d / ms_on},
            "offload": {"pages": n, "bytes": nb, "ms": ms_off, "gbs": gbs(nb, ms_off),
                        "dma_contiguous_gbs": gbs(nb, ms_d2h), "frac_of_dma": ms_d2h / ms_off},
            "compact": {"pages": 16384, "bytes_moved": 16384 * page_bytes, "ms": ms_mv,
                        "roofline": {"bound": "hbm", "achieved": gbs(2 * 16384 * page_bytes, ms_mv), "peak": hbm,
                                     "unit": "GB/s", "frac": gbs(2 * 16384 * page_bytes, ms_mv) / hbm,
                                     "note": "read + write bytes"}},
            "prepare": {"calls": len(lat), "batch": layer.B, "median_us": statistics.median(lat) * 1e6,
                        "p99_us": float(np.percentile(lat, 99)) * 1e6,
                        "pool": "65,536 GPU pages + 16,384 host pages, every batch 8 new users of U[1024,4096) "
                                "tokens, so each call evicts and offloads (the host tier drops the oldest)",
                        "final_stats": st},
            "launches": 3}
    del gk, gv, hk, hv, dflat, hflat
    torch.cuda.empty_cache()
    return line


def cpu_oracle_layer(layer, nthreads=None):
    """Oracle time for one layer (append + paged attention of all new tokens)."""
    import oracle

    ck, cv, cpt = layer.compact_pool()
    ck, cv = ck.copy(), cv.copy()
    t0 = time.perf_counter()
    oracle.kv_append(ck, cv, cpt, layer.k_new, layer.v_new, layer.cached_lens, layer.new_offsets,
                     layer.new_lens - layer.num_targets)
    oracle.hstu_paged(layer.q_new, layer.k_new, layer.v_new, layer.u_new, ck, cv, cpt, layer.cached_lens,
                      layer.new_lens, layer.num_targets, layer.rab, layer.n_max, layer.eps, nthreads=nthreads)
    return time.perf_counter() - t0


def profile_case(case, calls):
    """A small case for ncu: `calls` launches of one layer of the paged batch (its own pages
    only, ~0.4 GB on the device) or of the jagged prefill batch."""
    import torch

    import hstu_attention_b200 as hb

    torch.cuda.set_device(0)
    if case == "paged":
        c = gen.config3_paged_layers(layers=1)[0]
        ck, cv, cpt = c.compact_pool()

        compact = dataclasses.replace(c, num_pages=int(ck.shape[0]), page_table=cpt,
                                      page_ids=np.arange(ck.shape[0], dtype=np.int32))
        p, ws, kp, vp, L = setup_device([compact], torch.device("cuda", 0))
        t = L[0]
        for _ in range(calls):
            hb.paged_fwd(p, t["q"], t["k"], t["v"], t["u"], kp, vp, t["pt"], t["cl"], t["nl"], t["nt"], t["rab"],
                         max_new=c.max_new, workspace=ws, out=t["out"])
    elif case == "long":
        # the first 8 users of the long-history batch (about 0.4 GB of pages)
        c = gen.config4_long()
        c = dataclasses.replace(c, cached_lens=c.cached_lens[:8], new_lens=c.new_lens[:8], num_targets=c.num_targets[:8],
                                append_lens=c.append_lens[:8], page_table=c.page_table[:8],
                                q_new=c.q_new[:2048], k_new=c.k_new[:2048], v_new=c.v_new[:2048], u_new=c.u_new[:2048])
        dev = torch.device("cuda", 0)
        p = hb.params(c.H, c.D, torch.bfloat16, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                      max_pages_per_user=c.max_pages)
        kp = torch.zeros((c.num_pages, c.H, c.P, c.D), dtype=torch.bfloat16, device=dev)
        vp = torch.zeros_like(kp)
        used = np.unique(c.page_table[c.page_table >= 0])
        where = np.full(c.num_pages, -1, dtype=np.int64)
        where[c.page_ids] = np.arange(c.page_ids.shape[0])
        used = used[where[used] >= 0]
        pos = where[used]
        ids = torch.from_numpy(used.astype(np.int64)).to(dev)
        kp[ids] = _to_dev(c.pool_k[pos], dev)
        vp[ids] = _to_dev(c.pool_v[pos], dev)
        t = [_to_dev(x, dev) for x in (c.q_new, c.k_new, c.v_new, c.u_new)]
        meta = [_to_dev(x, dev) for x in (c.page_table, c.cached_lens, c.new_lens, c.num_targets, c.rab)]
        ws = hb.Workspace(p, c.B, c.Tn, c.max_new)
        for _ in range(calls):
            hb.paged_fwd(p, *t, kp, vp, *meta, max_new=c.max_new, workspace=ws)
    elif case == "backward":
        # the backward of the prefill batch (about 0.6 GB with its workspace)
        c = gen.config2_prefill()
        dev = torch.device("cuda", 0)
        dout = gen._values(np.random.default_rng(9), c.q.shape, 1.0, "bf16")
        args = [_to_dev(x, dev) for x in (c.q, c.k, c.v, c.u, c.seq_offsets, c.num_targets, c.rab, dout)]
        p = hb.params(c.H, c.D, torch.bfloat16, c.NB, c.n_max)
        ws = hb.BwdWorkspace(p, c.T)
        for _ in range(calls):
            hb.jagged_bwd(p, *args, max_seqlen=int(c.max_seqlen), workspace=ws)
    elif case == "layer":
        # one HSTU layer on layer 0 of the paged batch (d_model 512): projection GEMMs + attention;
        # the pool is compacted to the layer's pages, the appended tokens' pages included
        c = gen.config3_paged_layers(layers=1)[0]
        used = np.unique(c.page_table[c.page_table >= 0])
        remap = np.full(c.num_pages, -1, dtype=np.int64)
        remap[c.page_ids] = np.arange(c.page_ids.shape[0])
        extra = used[remap[used] < 0]
        remap[extra] = c.page_ids.shape[0] + np.arange(extra.shape[0])
        pt = np.where(c.page_table >= 0, remap[np.clip(c.page_table, 0, None)], -1).astype(np.int32)
        compact = dataclasses.replace(c, num_pages=int(c.page_ids.shape[0] + extra.shape[0]), page_table=pt,
                                      page_ids=np.arange(c.page_ids.shape[0], dtype=np.int32))
        dev = torch.device("cuda", 0)
        p, _, kp, vp, L = setup_device([compact], dev)
        t = L[0]
        rng = np.random.default_rng(2024)
        HD = c.H * c.D
        w1 = _to_dev(gen._values(rng, (4 * HD, 512), 1.0 / np.sqrt(512), "bf16"), dev)
        w2 = _to_dev(gen._values(rng, (512, HD), 1.0 / np.sqrt(HD), "bf16"), dev)
        x = _to_dev(gen._values(rng, (int(c.Tn), 512), 1.0, "bf16"), dev)
        ws = hb.LayerWorkspace(p, 512, c.B, int(c.Tn), c.max_new)
        for _ in range(calls):
            hb.layer_paged_fwd(p, 512, x, w1, w2, kp, vp, t["pt"], t["cl"], t["nl"], t["nt"], t["rab"],
                               max_new=c.max_new, workspace=ws)
    elif case == "cache":
        # onboard of layer 0's cached pages from pinned host pages, and a 16,384-page in-pool move
        c = gen.config3_paged_layers(layers=1)[0]
        dev = torch.device("cuda", 0)
        p = hb.params(c.H, c.D, torch.bfloat16, c.NB, c.n_max, page_size=c.P, num_pages=c.num_pages,
                      max_pages_per_user=c.max_pages)
        ws = hb.Workspace(p, 1, 1, 1)
        gk = torch.zeros((c.num_pages, c.H, c.P, c.D), dtype=torch.bfloat16, device=dev)
        gv = torch.zeros_like(gk)
        pages = np.concatenate([c.page_table[b, :(int(c.cached_lens[b]) + c.P - 1) // c.P] for b in range(c.B)])
        n = len(pages)
        hk = torch.zeros((n, c.H, c.P, c.D), dtype=torch.bfloat16).pin_memory()
        hv = torch.zeros((n, c.H, c.P, c.D), dtype=torch.bfloat16).pin_memory()
        on = torch.from_numpy(np.stack([np.arange(n), pages], 1).astype(np.int32)).to(dev)
        perm = np.random.default_rng(7).permutation(c.num_pages).astype(np.int32)
        mv = torch.from_numpy(np.stack([perm[:16384], perm[16384:32768]], 1)).to(dev)
        for _ in range(calls):
            hb.kv_page_copy(p, hk, hv, gk, gv, on, workspace=ws)
            hb.kv_page_copy(p, gk, gv, gk, gv, mv, workspace=ws)
    else:
        c = gen.config2_prefill()
        d = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)  # noqa
        p = hb.params(c.H, c.D, torch.bfloat16, c.NB, c.n_max)
        ws = hb.Workspace(p, c.B, c.T, 4096)
        args = (d(c.q), d(c.k), d(c.v), d(c.u), torch.from_numpy(c.seq_offsets.astype(np.int32)).cuda(),
                torch.from_numpy(c.num_targets.astype(np.int32)).cuda(), torch.from_numpy(c.rab).cuda())
        for _ in range(calls):
            hb.jagged_fwd(p, *args, max_seqlen=4096, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the long-history sub-line")
    ap.add_argument("--no-mixed", action="store_true", help="skip the mixed-batch sub-line")
    ap.add_argument("--no-cache-ops", action="store_true", help="skip the cache-management sub-line")
    ap.add_argument("--no-layer", action="store_true", help="skip the 8-layer HSTU stack sub-line")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward sub-line")
    ap.add_argument("--e2e-upload", choices=("sm", "dma"), default="dma",
                    help="e2e uploads: a DMA cudaMemcpyAsync per layer (default) or hstu_host_copy (the SMs read "
                         "pinned host memory; slower here because it competes with the attention kernels)")
    ap.add_argument("--e2e-upload-streams", type=int, default=1, choices=(1, 2, 4),
                    help="copy streams the e2e uploads alternate between (more than one measured no faster)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["paged", "prefill", "long", "backward", "layer", "cache"], default=None,
                    help="run a few calls of one workload for an ncu capture and exit (no JSON line)")
    ap.add_argument("--calls", type=int, default=3)
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case, args.calls)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    peaks, peaks_kind = load_peaks()
    layers_cfg = gen.CONFIG3

    if args.impl == "reference":
        if rank != 0:
            return
        import oracle

        layer = gen.config3_paged_layers(layers=1)[0]
        nthreads = oracle.default_threads()
        for _ in range(args.warmup):
            cpu_oracle_layer(layer, nthreads)
        times = [cpu_oracle_layer(layer, nthreads) for _ in range(args.steps)]
        t_layer = statistics.median(times)
        value = layer.Tn / (t_layer * args.layers)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value, "unit": "new tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_layer * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "paged cache hit x 8 layers: 8 users, cached U[1024,4096], 16 appended + 64 "
                                   "candidates each, H=4, D=128, P=32, 65,536-page pool; per layer kv_append + "
                                   "paged attention",
                       "step": "one layer (layer 0) of the stack per step; ms_per_step is that layer's median time, "
                               "value = 640 new tokens / (8 x layer time)",
                       "layers_per_step": 1, "global_batch": layer.B, "seq_len": int(layer.cached_lens.max()),
                       "parallelism": "none"},
            "cpu_baseline": {"value": value, "unit": "new tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": "layer 0 of the 8-layer stack: append + paged attention of all 640 new "
                                       "tokens; new tokens/s of the stack = 640 / (8 x layer time)"},
            "e2e": {"value": value, "unit": "new tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    import torch

    import hstu_attention_b200 as hb

    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    hb.load()

    layers = gen.config3_paged_layers(seed=1003 + rank, layers=args.layers)
    tokens, lbytes, lflops = workload_stats(layers)
    p, ws, kp, vp, L = setup_device(layers, device)
    max_new = max(c.max_new for c in layers)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        run_step(hb, p, ws, kp, vp, L, max_new)
    torch.cuda.synchronize()
    assert ws.status() == 0, "device status flags set during warm-up"

    # capture one step (8 x append + paged attention) in a graph.  No timing events inside it:
    # an event node between two calls would stop the next call's set-up from overlapping the
    # previous call's LayerNorm kernel (programmatic dependent launch), so per-call figures come
    # from the step time (calls run back to back) and, separately, from an instrumented copy
    side = torch.cuda.Stream(device=device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_step(hb, p, ws, kp, vp, L, max_new, side=side)
    graph.replay()
    torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    call_ms = []
    def roll(seconds):
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            for _ in range(20):
                graph.replay()
            torch.cuda.synchronize()

    with ClockSampler(local_rank) as clk:
        roll(0.3)                      # clocks are sampled every 100 ms: keep the GPU busy around
        if world > 1:                  # the timed window so samples land while it runs
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        roll(0.3)
    elapsed_ms = e0.elapsed_time(e1)
    elapsed_ms = max_over_ranks(elapsed_ms, device)
    if world > 1:
        dist.barrier()
    ms_step = elapsed_ms / args.steps
    value = job_throughput(tokens, ms_step, world)
    assert ws.status() == 0, "device status flags set during the timed region"

    # one call in isolation: the same step with CUDA events around every paged call (the events
    # serialise the calls), replayed a few times after the timed region
    events = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
              for _ in L]
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev):
        run_step(hb, p, ws, kp, vp, L, max_new, events=events, side=side)
    for _ in range(5):
        graph_ev.replay()
        torch.cuda.synchronize()
        call_ms.extend(a.elapsed_time(b) for a, b in events)
    del graph_ev

    # e2e through the public API with host buffers: per step, H2D of every layer's new-token
    # q/k/v/u and metadata from pinned memory, the step, and D2H of every layer's output.  Each
    # layer's inputs live in one pinned host buffer and one device buffer (256-byte aligned
    # views), so a layer uploads with a single copy.  Layers are pipelined (layer l's upload on
    # one copy stream overlaps layer l-1's kernels, one small graph per layer; its download on a
    # second copy stream overlaps layer l+1), and steps are double-buffered: step s+1 uploads into
    # the other set of device buffers while step s computes.
    names = ("q", "k", "v", "u", "pt", "cl", "nl", "nt")
    nsets = 2
    host_in, dev_in, L_e2e = [], [[] for _ in range(nsets)], [[] for _ in range(nsets)]
    for t in L:
        offs, total = [], 0
        for k in names:
            offs.append(total)
            total += (t[k].numel() * t[k].element_size() + 255) // 256 * 256
        hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
        for k, o in zip(names, offs):
            n = t[k].numel() * t[k].element_size()
            hbuf[o:o + n].copy_(t[k].contiguous().view(torch.uint8).view(-1).cpu())
        host_in.append(hbuf)
        for si in range(nsets):
            dbuf = torch.empty(total, dtype=torch.uint8, device=device)
            t2 = dict(t)
            t2["out"] = torch.empty_like(t["out"])
            for k, o in zip(names, offs):
                n = t[k].numel() * t[k].element_size()
                t2[k] = dbuf[o:o + n].view(t[k].dtype).view(t[k].shape)
            dev_in[si].append(dbuf)
            L_e2e[si].append(t2)
    host_out = [[t["out"].cpu().pin_memory() for t in L_e2e[si]] for si in range(nsets)]
    h2d = sum(x.numel() for x in host_in)
    d2h = sum(x.numel() * x.element_size() for x in host_out[0])
    e_steps = max(4, args.steps // 5)
    layer_graphs = [[] for _ in range(nsets)]
    for si in range(nsets):
        for t in L_e2e[si]:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run_step(hb, p, ws, kp, vp, [t], max_new, side=side)
            layer_graphs[si].append(g)
    # uploads may alternate between copy streams (measured: no faster than one on this host link)
    ups = [torch.cuda.Stream(device=device) for _ in range(args.e2e_upload_streams)]
    down = torch.cuda.Stream(device=device)
    ev_up = [[torch.cuda.Event() for _ in L] for _ in range(nsets)]
    ev_done = [[torch.cuda.Event() for _ in L] for _ in range(nsets)]
    ev_computed = [torch.cuda.Event() for _ in range(nsets)]     # a step's kernels on set si done
    ev_fetched = [torch.cuda.Event() for _ in range(nsets)]      # a step's downloads from set si done
    for si in range(nsets):
        ev_computed[si].record(stream)
        ev_fetched[si].record(down)

    def e2e_step(step):
        si = step % nsets
        # the step that last used this set has consumed its inputs and shipped its outputs
        for up in ups:
            up.wait_event(ev_computed[si])
            up.wait_event(ev_fetched[si])
        for li in range(len(L)):
            up = ups[li % len(ups)]
            with torch.cuda.stream(up):
                if args.e2e_upload == "sm":
                    hb.host_copy(dev_in[si][li], host_in[li], stream=up)
                else:
                    dev_in[si][li].copy_(host_in[li], non_blocking=True)
                ev_up[si][li].record(up)
        for li, t in enumerate(L_e2e[si]):
            stream.wait_event(ev_up[si][li])
            layer_graphs[si][li].replay()
            ev_done[si][li].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[si][li])
                host_out[si][li].copy_(t["out"], non_blocking=True)
        ev_computed[si].record(stream)
        ev_fetched[si].record(down)

    for s_ in range(2):
        e2e_step(s_)
    stream.wait_stream(down)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for up in ups:
        up.wait_stream(stream)                  # the first uploads start after the start event
    for s_ in range(e_steps):
        e2e_step(s_)
    stream.wait_stream(down)                    # every step's results are on the host
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / e_steps, device)
    assert ws.status() == 0, "device status flags set during the e2e steps"
    # the e2e results are the device results: the outputs that reached the host are the step's
    for si in range(nsets):
        for t, te, hdst in zip(L, L_e2e[si], host_out[si]):
            assert torch.equal(hdst.view(torch.int16), te["out"].cpu().view(torch.int16))
            assert torch.equal(te["out"].view(torch.int16), t["out"].view(torch.int16))

    prefill = long_history = mixed = cache_ops = layer_stack = backward = None
    if rank == 0 and not args.no_prefill:
        prefill = bench_prefill(hb, device, max(5, args.steps // 2), 3, peaks)
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    if rank == 0 and not args.no_long:
        long_history = bench_long_history(hb, device, max(5, args.steps // 2), 3, peaks, with_cpu)
    if rank == 0 and not args.no_mixed:
        mixed = bench_mixed(hb, device, max(3, args.steps // 4), 3, peaks, with_cpu)
    if rank == 0 and not args.no_backward:
        backward = bench_backward(hb, device, max(5, args.steps // 2), 3, peaks, with_cpu)
    if rank == 0 and not args.no_layer:
        layer_stack = bench_layer_stack(hb, device, max(5, args.steps // 2), 3, peaks, with_cpu)
    if rank == 0 and not args.no_cache_ops:
        cache_ops = bench_cache_ops(hb, device, max(5, args.steps // 2), 3, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        nthreads = oracle.default_threads()
        samples = [cpu_oracle_layer(layers[0], nthreads) for _ in range(3)]
        t_layer = statistics.median(samples)
        cpu = {"value": tokens / (t_layer * len(layers)), "unit": "new tokens/s", "cores": nthreads, "kind": "oracle",
               "sample": "layer 0 of the 8-layer stack (append + paged attention of all 640 new tokens), median of "
                         f"3 runs ({', '.join(f'{x:.2f}' for x in samples)} s); scaled as 640 / (8 x layer time)"}

    if world > 1:
        graph.reset() if hasattr(graph, "reset") else None
        del graph
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    isolated_call_ms = float(np.mean(call_ms))
    mean_call_ms = ms_step / len(L)                 # calls back to back in the timed step
    mean_bytes = float(np.mean(lbytes))
    achieved = mean_bytes / (mean_call_ms * 1e-3) / 1e9
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "new tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, shaped like the KuaiRand-1K serving config)",
        "config": {"workload": "paged cache hit x 8 layers: 8 users, cached U[1024,4096], 16 appended + 64 "
                               "candidates each, H=4, D=128, P=32, 65,536-page pool; per layer kv_append + "
                               "paged attention",
                   "global_batch": layers_cfg["B"] * world, "seq_len": int(max(int(c.cached_lens.max()) for c in layers)),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (8 layers of distinct pages, ~343 MB per step)",
                   "graph": "one CUDA graph per step; appends on a forked stream (they do not feed "
                            "the attention, which reads new keys from k_new)"},
        "roofline": {"bound": "hbm", "kernel": "hstu_attn_paged_fwd (attention kernel + LayerNorm-gate kernel)",
                     "timing": "CUDA events around the timed step replays / 8 calls per step (the appends run "
                               "concurrently on a forked stream and are not subtracted)",
                     "ms_per_call_isolated": isolated_call_ms,
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": PAGED_TRAFFIC_BYTES if kernel_sources_hash(PAGED_FILES) == PAGED_TRAFFIC_SOURCES else None,
                     "peak_kind": peaks_kind, "algorithmic_bytes_per_call": mean_bytes,
                     "ms_per_call": mean_call_ms,
                     "tflops": float(np.mean(lflops)) / (mean_call_ms * 1e-3) / 1e12},
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(tokens, e2e_ms, world), "unit": "new tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "upload": ("hstu_host_copy (SM copy kernel reading pinned host memory)" if args.e2e_upload == "sm"
                           else "cudaMemcpyAsync (DMA)") + f", alternating over {args.e2e_upload_streams} copy streams",
                "mode": "one graph per layer; each layer's inputs in one pinned buffer (one upload per layer); "
                        "uploads and downloads overlap the neighbouring layers' kernels on two copy streams; "
                        "two sets of device buffers, so a step's uploads overlap the previous step"},
        "gpu_launches": 3 * len(L),
        "clocks": clocks,
        "prefill": prefill,
        "long_history": long_history,
        "mixed": mixed,
        "cache_ops": cache_ops,
        "layer_stack": layer_stack,
        "backward": backward,
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
