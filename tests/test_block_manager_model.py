"""Pins for the oracle's block-manager model (CPU only): the pages' worked figures,
published FNV-1a test vectors, and invariants that any correct block manager keeps."""
import random

import pytest

from oracle.block_manager import BlockManagerModel, NoSpace, block_key, fnv1a64


def test_fnv1a64_published_vectors():
    # test vectors of the FNV reference (Fowler, Noll, Vo)
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


def test_block_key_chains_the_parent():
    a = block_key(block_key(0xCBF29CE484222325, list(range(16))), [7] * 16)
    b = block_key(block_key(0xCBF29CE484222325, list(range(1, 17))), [7] * 16)
    assert a != b                      # same tokens after a different prefix: another key


def test_worked_block_count_and_lifo_order():
    """A 40-token sequence takes ceil(40/16) = 3 blocks, the last 8/16 full; blocks
    come from the end of list(range(num_blocks)) (pop())."""
    m = BlockManagerModel(100, 0, 16, False)
    slots, cached = m.add_sequence(1, list(range(40)))
    blocks, n = m.block_table(1)
    assert blocks == [99, 98, 97] and n == 40 and cached == 0
    assert slots[:2] == [99 * 16, 99 * 16 + 1] and slots[39] == 97 * 16 + 7
    m.free_sequence(1)
    m.add_sequence(2, list(range(20)))
    assert m.block_table(2)[0] == [97, 98]          # freed blocks are reused last-in first


def test_concurrency_figure_of_the_pages():
    """12480 blocks of 16 tokens hold 48 sequences of 4096 tokens (12480*16/4096 = 48.75)."""
    m = BlockManagerModel(12480, 0, 16, False)
    for s in range(48):
        m.add_sequence(s, [1] * 4096)
    with pytest.raises(NoSpace):
        m.add_sequence(48, [1] * 4096)
    assert m.free_gpu_blocks() == 12480 - 48 * 256 == 192


def test_append_takes_a_block_only_when_the_last_is_full():
    m = BlockManagerModel(10, 0, 4, False)
    m.add_sequence(0, [5, 6, 7])
    assert m.append_token(0, 8) == (9 * 4 + 3, -1, -1)
    slot, src, dst = m.append_token(0, 9)
    assert slot == 8 * 4 and (src, dst) == (-1, -1)
    assert m.block_table(0) == ([9, 8], 5)


def test_copy_on_write_after_fork():
    m = BlockManagerModel(10, 0, 4, False)
    m.add_sequence(0, [1, 2, 3, 4, 5, 6])            # blocks 9 (full), 8 (2 of 4)
    m.fork(0, 1)
    slot, src, dst = m.append_token(1, 7)
    assert (src, dst) == (8, 7) and slot == 7 * 4 + 2
    assert m.block_table(0)[0] == [9, 8] and m.block_table(1)[0] == [9, 7]
    # the parent now owns block 8 alone: its append writes in place
    assert m.append_token(0, 9) == (8 * 4 + 2, -1, -1)


def test_prefix_cache_reuses_full_blocks_and_keeps_the_last_token():
    m = BlockManagerModel(20, 0, 4, True)
    p = [3, 1, 4, 1, 5, 9, 2, 6, 5, 3]
    s0, c0 = m.add_sequence(0, p)
    assert c0 == 0
    s1, c1 = m.add_sequence(1, p[:8] + [7, 7])       # two full blocks in common
    assert c1 == 8 and s1[:8] == [-1] * 8
    assert m.block_table(1)[0][:2] == m.block_table(0)[0][:2]
    s2, c2 = m.add_sequence(2, p[:8])                # whole prompt cached: last block redone
    assert c2 == 4 and m.block_table(2)[0][0] == m.block_table(0)[0][0]
    assert m.block_table(2)[0][1] != m.block_table(0)[0][1]


def test_freed_cached_blocks_are_evicted_oldest_first():
    m = BlockManagerModel(3, 0, 2, True)
    m.add_sequence(0, [1, 2, 3])                     # blocks 2 (cached), 1
    m.free_sequence(0)                               # 2 -> evictable, 1 -> free
    assert m.free_gpu_blocks() == 3
    _, c = m.add_sequence(1, [1, 2, 9])              # hit on block 2
    assert c == 2 and m.block_table(1)[0][0] == 2
    m.free_sequence(1)
    m.add_sequence(2, [4, 4, 4, 4, 4, 4])            # needs all 3: evicts block 2
    assert sorted(m.block_table(2)[0]) == [0, 1, 2]
    m.free_sequence(2)
    _, c = m.add_sequence(3, [1, 2, 0])              # block 2's key is gone: a miss
    assert c == 0


def test_swap_out_and_in_keeps_sharing():
    m = BlockManagerModel(8, 8, 4, False)
    m.add_sequence(0, list(range(6)))
    m.fork(0, 1)
    out = m.swap_out([0, 1])
    assert [g for g, _ in out] == [7, 6] and len(out) == 2    # shared blocks move once
    assert m.free_gpu_blocks() == 8 and m.free_cpu_blocks() == 6
    back = m.swap_in([0, 1])
    assert [c for c, _ in back] == [c for _, c in out]
    assert m.block_table(0)[0] == m.block_table(1)[0]
    m.swap_out([1])
    with pytest.raises(ValueError):                  # a swapped-out sequence cannot grow
        m.append_token(1, 1)


def _invariants(m, total_gpu, total_cpu):
    ref_gpu = [0] * total_gpu
    ref_cpu = [0] * total_cpu
    for s in m.seqs.values():
        n = len(s["tokens"])
        assert len(s["blocks"]) == -(-n // m.bs)     # waste is only the last block's tail
        for b in s["blocks"]:
            (ref_gpu if s["on_gpu"] else ref_cpu)[b] += 1
    assert ref_gpu == m.gpu.ref and ref_cpu == m.cpu.ref
    free = set(m.gpu.free) | set(m.evictable)
    assert len(free) == len(m.gpu.free) + len(m.evictable)
    assert all(ref_gpu[b] == 0 for b in free)
    assert all(ref_gpu[b] > 0 for b in range(total_gpu) if b not in free)
    assert sorted(m.cpu.free) == [b for b in range(total_cpu) if ref_cpu[b] == 0]


@pytest.mark.parametrize("prefix", [False, True])
def test_random_operations_keep_the_invariants(prefix):
    rng = random.Random(5)
    G, C, bs = 64, 32, 4
    m = BlockManagerModel(G, C, bs, prefix)
    nxt = 0
    for _ in range(3000):
        op = rng.random()
        live = [i for i, s in m.seqs.items() if s["on_gpu"]]
        out = [i for i, s in m.seqs.items() if not s["on_gpu"]]
        try:
            if op < 0.25 or not m.seqs:
                toks = [rng.randrange(3) for _ in range(rng.randrange(1, 20))]
                m.add_sequence(nxt, toks)
                nxt += 1
            elif op < 0.6 and live:
                m.append_token(rng.choice(live), rng.randrange(3))
            elif op < 0.7 and live:
                m.fork(rng.choice(live), nxt)
                nxt += 1
            elif op < 0.8 and live:
                m.swap_out([rng.choice(live)])
            elif op < 0.85 and out:
                m.swap_in([rng.choice(out)])
            else:
                m.free_sequence(rng.choice(list(m.seqs)))
        except NoSpace:
            pass
        _invariants(m, G, C)
