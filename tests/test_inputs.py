"""The seeded workload generators: deterministic, shaped as the benchmark states, and the
structure the benchmark relies on (disjoint pages per layer, page tables that cover every
cached and appended position)."""
import numpy as np

from hstu_attention_b200 import inputs as gen


def test_generators_are_deterministic():
    a, b = gen.config1_tiny(), gen.config1_tiny()
    for name in ("q_new", "k_new", "pool_k", "page_table", "rab"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], dtype=np.float32)
    bits = gen.f32_to_bf16_bits(x)
    back = gen.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); 1 + 3 * 2^-8 ties up to 1 + 2^-6
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0]


def test_paged_layers_use_disjoint_pages_and_cover_their_positions():
    layers = gen.config3_paged_layers(layers=8)
    seen = set()
    for c in layers:
        assert c.B == 8 and c.H == 4 and c.D == 128 and c.P == 32
        assert np.all((c.cached_lens >= 1024) & (c.cached_lens <= 4096))
        assert np.all(c.new_lens == 80) and np.all(c.num_targets == 64)
        ids = set(int(x) for x in c.page_ids)
        assert not (ids & seen), "layers share a physical page"
        seen |= ids
        for b in range(c.B):
            need = (int(c.cached_lens[b]) + int(c.new_lens[b] - c.num_targets[b]) + c.P - 1) // c.P
            row = c.page_table[b, :need]
            assert np.all(row >= 0) and np.all(row < c.num_pages)
            assert len(set(row.tolist())) == need
    # the 8 layers' cached K and V (~317 MB) exceed the 126 MB L2 more than twice over
    total = sum(int(c.cached_lens.sum()) for c in layers) * 4 * 128 * 2 * 2
    assert total > 2 * 126e6


def test_prefill_workload_shape():
    c = gen.config2_prefill()
    L = np.diff(c.seq_offsets)
    assert c.B == 8 and np.all((L >= 256) & (L <= 4096)) and np.all(c.num_targets == 64)
    assert c.q.shape == (int(L.sum()), 4, 128) and c.q.dtype == np.uint16
