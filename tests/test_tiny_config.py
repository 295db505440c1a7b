"""The tiny fp32 configuration exactly as stated -- 4 sequences, 4 query heads and 4 kv
heads (G = 1, plain multi-head attention), head_dim 64, block 16, a 64-block pool,
lengths U{1..100}, scale 1/8, tables cut from a shuffled pool -- on every decode entry
point, each output element against the oracle at the fp32 tolerance.

Pages: the attention formula of "LLM推理优化：vLLM PagedAttention深度解析与工程实践" §二
and its statement (§九) that paging changes no computation; the v2 partition and
merge of the same page, §4.1."""
import pytest
import torch

from _helpers import TOL32, CpuCaches, GpuProblem, bytes_equal, compare
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu

SEEDS = [0, 1, 2, 3]


def _problem(seed):
    p = make_problem("tiny_f32", seed)
    wl = p.wl
    assert (wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
            p.num_blocks, wl.scale) == (4, 4, 4, 64, 16, 64, 0.125)
    assert p.k_cache.dtype == torch.float32 and p.batch.q.dtype == torch.float32
    return p


@pytest.mark.parametrize("seed", SEEDS)
def test_tiny_f32_every_entry_point_matches_the_oracle(pa, orc, seed):
    p = _problem(seed)
    ref = CpuCaches(p, orc).decode(orc)
    g = GpuProblem(p).fill(pa)
    outs = {"v1": g.v1(pa)}
    for P in (16, 64):
        outs[f"v2 P={P}"] = g.v2(pa, partition_size=P)
    outs["fused"] = g.fused(pa)
    # the one-launch step: history in the cache, the new token written by the call
    a = GpuProblem(p).fill(pa, include_new=False)
    outs["append"] = pa.append_decode_v1(a.q, a.new_key, a.new_value, a.new_slots, a.kc, a.vc,
                                         a.tables, a.lens, p.wl.scale)
    torch.cuda.synchronize()
    assert bytes_equal(a.kc, g.kc) and bytes_equal(a.vc, g.vc)
    for name, out in outs.items():
        info = compare(out, ref, f"tiny_f32 seed {seed} {name}")
        assert info["rel_l2"] <= TOL32


def test_tiny_f32_cache_write_is_bit_exact(pa, orc):
    p = _problem(0)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)


def test_tiny_f32_with_an_empty_and_a_one_token_sequence(pa, orc):
    p = _problem(1)
    g = GpuProblem(p).fill(pa)
    lens = p.batch.seq_lens.clone()
    lens[0], lens[3] = 1, 0
    g.lens.copy_(lens)
    ref = CpuCaches(p, orc).decode(orc, lens=lens)
    for name, out in (("v1", g.v1(pa)), ("v2 P=16", g.v2(pa, partition_size=16)),
                      ("fused", g.fused(pa))):
        torch.cuda.synchronize()
        assert not out[3].any(), name
        compare(out, ref, f"tiny_f32 empty/one-token {name}")
        # one token: each head's output is that token's V row (G = 1: head h reads kv head h)
        blk = int(p.batch.block_tables[0, 0])
        assert torch.equal(out[0], g.vc[blk, 0]), name
