"""The seeded generators: determinism, layout, canaries, block-table structure."""
import numpy as np

from paged_kv_cache_380_b200 import workloads as W


def test_deterministic_and_seeded_per_config():
    a = W.tiny_decode_f32()
    b = W.tiny_decode_f32()
    assert np.array_equal(a.q, b.q) and np.array_equal(a.block_tables, b.block_tables)
    assert np.array_equal(a.k_pages, b.k_pages, equal_nan=True)


def test_tiny_decode_layout_and_canaries():
    c = W.tiny_decode_f32()
    assert c.k_pages.shape == (16, 16, 2, 64) and c.q.shape == (2, 4, 64)
    assert c.context_lens.tolist() == [37, 100]
    used = set()
    for b, ctx in enumerate(c.context_lens):
        n = -(-int(ctx) // 16)
        row = c.block_tables[b]
        assert (row[:n] >= 0).all() and (row[n:] == -1).all()
        used |= set(row[:n].tolist())
        last = row[n - 1]
        tail = int(ctx) - (n - 1) * 16
        assert np.isnan(c.k_pages[last, tail:]).all()          # tail rows are canary
        assert not np.isnan(c.k_pages[row[:n - 1]]).any()
    assert len(used) == 10
    free = [p for p in range(16) if p not in used]
    assert np.isnan(c.v_pages[free]).all()


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -3.5, 1e-3], dtype=np.float32)
    bits = W.to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-8 -> 1 + 2^-6
    assert W.bf16_bits_to_f32(bits).tolist()[:4] == [1.0, 1.0, 1.015625, -3.5]


def test_prefill_shared_prefix_structure():
    c = W.chunked_prefill_shared_prefix(num_seqs=3, prefix=32, chunk=20)
    assert (c.block_tables[:, :2] == c.block_tables[0, :2]).all()     # shared pages
    assert c.q_start.tolist() == [0, 20, 40, 60] and c.context_lens.tolist() == [52] * 3
    assert len(set(c.slot_mapping.tolist())) == 60
    own = set(c.block_tables[:, 2:].ravel().tolist()) - {-1}
    assert not own & set(c.block_tables[0, :2].tolist())
    # the chunk's slots are the sequence's logical positions 32..51
    b = 1
    i = np.arange(32, 52)
    want = c.block_tables[b, i // 16].astype(np.int64) * 16 + i % 16
    assert np.array_equal(c.slot_mapping[20:40], want)


def test_decode_random_slots_distinct_and_in_range():
    c = W.decode_case(name="t", config_index=9, batch=5, num_q_heads=4, num_kv_heads=4,
                      head_dim=16, page_size=16, dtype="bf16", context_lens=np.array([3, 40, 16, 17, 1]),
                      new_tokens="random", num_new=7)
    s = c.slot_mapping
    assert len(set(s.tolist())) == 7 and (s >= 0).all() and (s < c.num_pages * 16).all()


def test_decode_append_slots_point_at_last_position():
    c = W.decode_case(name="t", config_index=9, batch=3, num_q_heads=2, num_kv_heads=1,
                      head_dim=8, page_size=4, dtype="bf16", context_lens=np.array([5, 8, 1]),
                      new_tokens="append")
    for b, ctx in enumerate(c.context_lens):
        p = c.block_tables[b, (ctx - 1) // 4]
        assert c.slot_mapping[b] == p * 4 + (ctx - 1) % 4
        flat = c.k_pages.reshape(-1, 1, 8)
        assert (flat[c.slot_mapping[b]] == W.CANARY_BITS["bf16"]).all()   # not yet written


def test_full_cache_scatter_covers_every_cached_token_once():
    c = W.decode_case(name="fc", config_index=77, batch=5, num_q_heads=4, num_kv_heads=2, head_dim=64,
                      page_size=16, dtype="bf16", context_lens=np.array([0, 1, 16, 17, 100]))
    src, dst = W.full_cache_scatter(c)
    # brute force over the block tables: sequence by sequence, position by position
    want = [int(c.block_tables[b, i // 16]) * 16 + i % 16
            for b in range(c.batch) for i in range(int(c.context_lens[b]))]
    assert src.tolist() == want
    n_slots = c.k_pages.shape[0] * 16
    assert dst.shape == src.shape and len(set(dst.tolist())) == dst.shape[0]
    assert dst.min() >= 0 and dst.max() < n_slots
    src2, dst2 = W.full_cache_scatter(c)                  # seeded: same draw every time
    assert (src2 == src).all() and (dst2 == dst).all()
