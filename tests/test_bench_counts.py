"""The numerators of the bench's roofline figures, checked against brute force.

Every TFLOP/s figure `bench.py` reports divides 4 * D * H * (visible query-key pairs) by a time,
so the pair counts must equal the number of pairs the attention mask lets through: query i sees
key j when j <= i and j is a history token (j < L - targets), and always itself (aitrends.kr
summary, section "HSTU의 순차 모델링": causal attention over the user's stream, candidates
attending to the history and not to each other).  The counts here are taken element by element
over small seeded batches.  Also pinned: the kernel-source hash that guards the bench's DRAM
traffic figures ignores comments and blank space but not code.
"""
import os

import numpy as np
import pytest

import bench
from hstu_attention_b200 import inputs as gen


def _visible_pairs(C, N, T):
    """Queries C..C+N-1 of one user with C cached and N new tokens (T of them candidates)."""
    hist = C + N - T
    count = 0
    for i in range(C, C + N):
        for j in range(C + N):
            if (j <= i and j < hist) or j == i:
                count += 1
    return count


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_jagged_pair_count_equals_brute_force(seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    lengths = rng.integers(1, 90, size=6)
    targets = np.array([rng.integers(0, L + 1) for L in lengths])
    want = sum(_visible_pairs(0, int(L), int(T)) for L, T in zip(lengths, targets))
    assert bench.jagged_pairs(lengths, targets) == want


def test_jagged_pair_count_special_cases():
    # no candidates: the full lower triangle; all candidates: each token sees only itself
    assert bench.jagged_pairs([5], [0]) == 15
    assert bench.jagged_pairs([5], [5]) == 5
    assert bench.jagged_pairs([0], [0]) == 0


@pytest.mark.parametrize("seed", [3, 4])
def test_paged_pair_counts_equal_brute_force(seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    cached = rng.integers(0, 70, size=5)
    append = rng.integers(0, 9, size=5)
    targets = rng.integers(0, 9, size=5)
    c = gen.paged_case(cached, append, targets, H=2, D=32, P=8, NB=16, n_max=200, num_pages=128,
                       dtype="fp32", seed=seed)
    want = sum(_visible_pairs(int(C), int(N), int(T))
               for C, N, T in zip(c.cached_lens, c.new_lens, c.num_targets))
    assert bench.paged_pairs(c) == want
    # the per-layer FLOPs of the step's workload statistics use the same pairs
    tokens, nbytes, flops = bench.workload_stats([c])
    assert tokens == int(c.Tn)
    assert flops[0] == 4 * c.D * c.H * want
    # bytes: cached K and V once, q/k/v/u read and out written, page-table entries of cached pages
    HD = c.H * c.D
    pages = sum((int(C) + c.P - 1) // c.P for C in c.cached_lens)
    assert nbytes[0] == int(np.sum(c.cached_lens)) * HD * 4 + int(c.Tn) * HD * 10 + pages * 4


def test_kernel_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "hstu_attention_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("k.cu",) + bench.SHARED_KERNEL_HEADERS:
        (csrc / f).write_text("int f(int x) { return x + 1; }  // one\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_sources_hash(("k.cu",))
    (csrc / "k.cu").write_text("/* a block */\nint f(int x)  {\n  return x + 1;   // two\n}\n")
    assert bench.kernel_sources_hash(("k.cu",)) == h0
    (csrc / "k.cu").write_text("int f(int x) { return x + 2; }\n")
    assert bench.kernel_sources_hash(("k.cu",)) != h0
    # a shared header counts too
    (csrc / "k.cu").write_text("int f(int x) { return x + 1; }\n")
    assert bench.kernel_sources_hash(("k.cu",)) == h0
    (csrc / bench.SHARED_KERNEL_HEADERS[0]).write_text("int g;\n")
    assert bench.kernel_sources_hash(("k.cu",)) != h0
    assert os.path.isdir(csrc)
