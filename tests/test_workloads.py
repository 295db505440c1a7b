"""Host-side checks of the seeded workloads (block tables, slots, fragmentation). CPU only."""
import numpy as np
import pytest
import torch

from paged_kv_cache_390_b200.workloads import (WORKLOADS, SeededBlockAllocator, logical_kv_bytes,
                                               make_problem, unique_kv_bytes)


@pytest.mark.parametrize("name", ["tiny_f32", "qwen3_32b_f16", "quant_fp8"])
def test_tables_slots_and_fragmentation(name):
    p = make_problem(name, 0)
    b = p.batch
    bs = p.wl.block_size
    used = set()
    for s in range(p.wl.num_seqs):
        n = int(b.seq_lens[s])
        nb = -(-n // bs)
        row = b.block_tables[s].tolist()
        assert all(x >= 0 for x in row[:nb]) and all(x == -1 for x in row[nb:])
        # only the last block is partly filled: waste < one block (the "<4%" claim of
        # KV Cache 与 PagedAttention §二 rests on this)
        assert nb * bs - n <= bs - 1
        assert not used & set(row[:nb])           # private blocks are never shared here
        used |= set(row[:nb])
        slot = int(b.new_slots[s])
        assert slot == row[(n - 1) // bs] * bs + (n - 1) % bs
    assert max(used) < p.num_blocks
    # every history slot is distinct and none is a new-token slot
    hs = p.hist_slots.tolist()
    assert len(set(hs)) == len(hs) and not set(hs) & set(b.new_slots.tolist())
    assert len(hs) == int(b.seq_lens.sum()) - p.wl.num_seqs


def test_shared_prefix_tables():
    p = make_problem("mixed_f16", 0, num_seqs=16)
    b = p.batch
    pre = p.wl.shared_prefix_tokens // p.wl.block_size
    first = b.block_tables[0, :pre]
    assert (b.block_tables[:, :pre] == first).all()
    lens = b.seq_lens.numpy()
    assert (lens > p.wl.shared_prefix_tokens).all() and (lens <= 8192 * 2).all()
    assert unique_kv_bytes(p.wl, lens) < logical_kv_bytes(p.wl, lens)


def test_block_size_variants_keep_pool_tokens():
    for bs in (8, 16, 32):
        p = make_problem("qwen3_32b_f16", 0, block_size=bs, num_seqs=4)
        assert p.num_blocks * bs == 12480 * 16
        assert p.k_cache.shape == (p.num_blocks, bs, 8, 128)


def test_allocator_is_a_seeded_permutation():
    a = SeededBlockAllocator(64, np.random.default_rng(0))
    ids = a.take(10) + a.take(54)
    assert sorted(ids) == list(range(64)) and a.num_free == 0
    with pytest.raises(MemoryError):
        a.take(1)
    b = SeededBlockAllocator(64, np.random.default_rng(0))
    assert b.take(10) == ids[:10]


def test_seeded_inputs_are_reproducible():
    a, b = make_problem("tiny_f32", 3), make_problem("tiny_f32", 3)
    assert torch.equal(a.batch.q, b.batch.q) and torch.equal(a.hist_key, b.hist_key)
    assert torch.equal(a.batch.block_tables, b.batch.block_tables)
    c = make_problem("tiny_f32", 4)
    assert not torch.equal(a.batch.q, c.batch.q)


def test_rotating_batches_use_disjoint_blocks():
    p = make_problem("qwen3_32b_f16", 0, num_batches=4)
    seen = set()
    for b in p.batches:
        ids = set(b.block_tables[b.block_tables >= 0].tolist())
        assert not ids & seen
        seen |= ids


def test_workload_catalogue_shapes():
    w = WORKLOADS["qwen3_32b_f16"]
    assert (w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks) == \
        (32, 64, 8, 128, 16, 12480)
    w = WORKLOADS["long_ctx_bf16"]
    assert w.num_blocks * w.block_size == w.num_seqs * w.len_lo
