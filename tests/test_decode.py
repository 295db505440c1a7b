"""GPU paged decode (v1, v2 partition + merge) against the oracle, plus the
invariants the pages fix: physical relabelling, shared prefix blocks, CoW."""
import numpy as np
import pytest
import torch

from _helpers import (CpuCaches, GpuProblem, compare, partition_sizes, sample_pairs,
                      small_problem)
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu

DTYPE_COMBOS = [("f16", "f16"), ("bf16", "bf16"), ("f32", "f32"), ("f16", "int8"),
                ("f16", "fp8"), ("bf16", "int8"), ("bf16", "fp8")]


@pytest.mark.parametrize("dt,cd", DTYPE_COMBOS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_decode_matches_oracle(pa, orc, dt, cd, D, bs):
    p = small_problem(cache_dtype=cd, dtype=dt, D=D, bs=bs, seed=7 * D + bs)
    g = GpuProblem(p).fill(pa)
    ref = CpuCaches(p, orc).decode(orc)
    compare(g.v1(pa), ref, f"v1 {dt}/{cd} D{D} bs{bs}")
    for P in partition_sizes(bs):
        compare(g.v2(pa, partition_size=P), ref, f"v2 P{P} {dt}/{cd} D{D} bs{bs}")


@pytest.mark.parametrize("H,Hkv", [(8, 8), (8, 4), (16, 4), (12, 3), (14, 2), (64, 8)])
def test_gqa_group_sizes(pa, orc, H, Hkv):
    p = small_problem(cache_dtype="f16", H=H, Hkv=Hkv, seed=H * 31 + Hkv)
    g = GpuProblem(p).fill(pa)
    ref = CpuCaches(p, orc).decode(orc)
    compare(g.v1(pa), ref, f"v1 G{H // Hkv}")
    compare(g.v2(pa, partition_size=32), ref, f"v2 G{H // Hkv}")


def test_v2_partials_match_oracle_partials(pa, orc):
    p = small_problem(cache_dtype="bf16", lens=(1, 40, 129, 300), seed=11)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    P = 64
    maxp = -(-300 // P)
    S, H, D = g.q.shape
    tmp = torch.full((S, H, maxp, D), float("nan"), device="cuda")
    ml = torch.full((S, H, maxp), float("nan"), device="cuda")
    es = torch.full((S, H, maxp), float("nan"), device="cuda")
    pa.decode_v2_partition(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, P, tmp, ml, es)
    torch.cuda.synchronize()
    t_ref, m_ref, l_ref = orc.paged_decode_partition(c.b.q, c.kc, c.vc, c.b.block_tables,
                                                     c.b.seq_lens, p.wl.scale, P, maxp)
    for s in range(S):
        n = int(p.batch.seq_lens[s])
        npart = -(-n // P)
        np.testing.assert_allclose(ml[s, :, :npart].cpu().numpy(), m_ref[s, :, :npart],
                                   rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(es[s, :, :npart].cpu().numpy(), l_ref[s, :, :npart],
                                   rtol=1e-4)
        np.testing.assert_allclose(tmp[s, :, :npart].cpu().numpy(), t_ref[s, :, :npart],
                                   rtol=0, atol=2e-4)
        # partitions past the sequence are left untouched
        assert torch.isnan(ml[s, :, npart:]).all() and torch.isnan(tmp[s, :, npart:]).all()


def test_single_partition_v2_equals_v1(pa, orc):
    p = small_problem(cache_dtype="f32", D=128, seed=13)
    g = GpuProblem(p).fill(pa)
    a = g.v1(pa)
    b = g.v2(pa, partition_size=512)
    torch.cuda.synchronize()
    rel = (a - b).norm() / a.norm()
    assert float(rel) <= 1e-6


def test_empty_and_single_token_sequences(pa, orc):
    p = small_problem(cache_dtype="f16", lens=(1, 5, 1, 64), seed=17)
    g = GpuProblem(p).fill(pa)
    g.lens[2] = 0
    lens_cpu = p.batch.seq_lens.clone()
    lens_cpu[2] = 0
    ref = CpuCaches(p, orc).decode(orc, lens=lens_cpu)
    for out in (g.v1(pa), g.v2(pa, partition_size=16)):
        torch.cuda.synchronize()
        assert not out[2].any()
        compare(out, ref, "empty/single")
        # seq_len 1: each head's output is exactly its kv head's single V row
        G = out.shape[1] // g.new_value.shape[1]
        for h in range(out.shape[1]):
            assert torch.equal(out[0, h], g.new_value[0, h // G])


def test_many_partitions(pa, orc):
    p = small_problem(cache_dtype="f16", lens=(4096, 3000), seed=19)
    g = GpuProblem(p).fill(pa)
    ref = CpuCaches(p, orc).decode(orc)
    compare(g.v2(pa, partition_size=16), ref, "P=16, 256 partitions")
    compare(g.v1(pa), ref, "v1 4096 tokens")


@pytest.mark.parametrize("dt,D", [("f16", 64), ("bf16", 64), ("bf16", 128)])
def test_many_partitions_every_merge_path(pa, orc, dt, D):
    """The split-K merge streams partition rows four at a time per row group (two rows a
    warp step at head_dim 64): hundreds of partitions run its unrolled loop and its
    tail, beside sequences of 1, 17 and 500 tokens and an empty one."""
    p = small_problem(cache_dtype=dt, D=D, lens=(3000, 1, 17, 1, 500, 2049), seed=23 + D)
    g = GpuProblem(p).fill(pa)
    lens = p.batch.seq_lens.clone()
    lens[3] = 0
    g.lens.copy_(lens)
    ref = CpuCaches(p, orc).decode(orc, lens=lens)
    for P in (16, 32):
        out = g.v2(pa, partition_size=P)
        torch.cuda.synchronize()
        assert not out[3].any()
        compare(out, ref, f"v2 {dt} D{D} P={P}, up to {-(-3000 // P)} partitions")


def test_many_sequences(pa, orc):
    lens = tuple(int(x) for x in np.random.default_rng(0).integers(1, 40, 3000))
    p = small_problem(cache_dtype="f16", H=8, Hkv=8, D=64, lens=lens, seed=23)
    g = GpuProblem(p).fill(pa)
    out = g.v1(pa)
    out2 = g.v2(pa, partition_size=16)
    pairs = sample_pairs(len(lens), 8, 64)
    ref = CpuCaches(p, orc).decode_pairs(orc, pairs)
    compare(out[pairs[:, 0], pairs[:, 1]], ref, "3000 seqs v1")
    compare(out2[pairs[:, 0], pairs[:, 1]], ref, "3000 seqs v2")


# ---------------------------------------------------------------------------
# Invariants fixed by the pages (physical relabelling, shared prefix, CoW).
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("cd", ["f16", "int8"])
def test_physical_relabelling_is_bit_identical(pa, cd):
    p = small_problem(cache_dtype=cd, seed=29)
    g = GpuProblem(p).fill(pa)
    a1, a2 = g.v1(pa), g.v2(pa, partition_size=32)
    nb = g.kc.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(1)).cuda()
    for name in ("kc", "vc", "ks", "vs"):
        t = getattr(g, name)
        if t is None:
            continue
        t2 = torch.empty_like(t)
        t2[perm] = t
        setattr(g, name, t2)
    live = g.tables >= 0
    t2 = g.tables.clone()
    t2[live] = perm[g.tables[live].long()].to(torch.int32)
    g.tables = t2
    b1, b2 = g.v1(pa), g.v2(pa, partition_size=32)
    torch.cuda.synchronize()
    assert torch.equal(a1, b1) and torch.equal(a2, b2)


def _private_copy_of_prefix(g, prefix_blocks):
    """Give every sequence private copies of the shared prefix blocks."""
    S = g.tables.shape[0]
    nb = g.kc.shape[0]
    extra = S * prefix_blocks
    for name in ("kc", "vc", "ks", "vs"):
        t = getattr(g, name)
        if t is None:
            continue
        src = t[g.tables[:, :prefix_blocks].reshape(-1).long()]
        setattr(g, name, torch.cat([t, src], dim=0))
    t2 = g.tables.clone()
    t2[:, :prefix_blocks] = (nb + torch.arange(extra, device="cuda").view(S, prefix_blocks)).to(
        torch.int32)
    g.tables = t2
    return g


@pytest.mark.parametrize("cd", ["f16", "fp8"])
def test_shared_prefix_equals_private_copies(pa, orc, cd):
    p = make_problem("mixed_f16", 3, num_seqs=6, cache_dtype=cd)
    g = GpuProblem(p).fill(pa)
    a1, a2 = g.v1(pa), g.v2(pa, partition_size=256)
    _private_copy_of_prefix(g, p.wl.shared_prefix_tokens // p.wl.block_size)
    b1, b2 = g.v1(pa), g.v2(pa, partition_size=256)
    torch.cuda.synchronize()
    assert torch.equal(a1, b1) and torch.equal(a2, b2)
    pairs = sample_pairs(6, 64, 6, seed=3)
    ref = CpuCaches(p, orc).decode_pairs(orc, pairs)
    compare(a1[pairs[:, 0], pairs[:, 1]], ref, "shared prefix")


def test_copy_on_write_leaves_the_other_sequence_unchanged(pa, orc):
    """Two sequences share all blocks of a 40-token prefix (last block partly full).
    Sequence 0 appends a token: its shared last block is copied to a free block,
    its table repointed, and the token written there; sequence 1 must not change."""
    bs, Hkv, D, H = 16, 2, 128, 16
    p = make_problem("qwen3_32b_f16", 31, num_seqs=2, seq_lens=[40, 40], num_heads=H,
                     num_kv_heads=Hkv, head_dim=D, num_blocks=16)
    g = GpuProblem(p)
    g.tables[1] = g.tables[0]                       # seq 1 shares seq 0's blocks
    g.q[1] = g.q[0]                                 # ... and asks the same question
    g.hist_slots = g.hist_slots[:39]
    g.hist_key, g.hist_value = g.hist_key[:39], g.hist_value[:39]
    g.fill(pa, include_new=False)
    # both have 39 tokens so far; write token 39 of the shared prefix once
    g.new_slots[1] = -1
    g.new_slots[0] = int(g.tables[0, 2]) * bs + 7
    g.write_new(pa)
    before = g.v1(pa)
    torch.cuda.synchronize()
    assert torch.equal(before[0], before[1])
    # CoW: seq 0 appends token 40 -> copy its last block to a free block first
    used = set(g.tables[0, :3].tolist())
    fresh = next(b for b in range(16) if b not in used)
    g.kc[fresh] = g.kc[g.tables[0, 2]]
    g.vc[fresh] = g.vc[g.tables[0, 2]]
    g.tables[0, 2] = fresh
    newk = torch.randn((2, Hkv, D), device="cuda").half()
    g.new_key, g.new_value = newk, newk.flip(0)
    g.new_slots = torch.tensor([fresh * bs + 8, -1], device="cuda")
    g.write_new(pa)
    g.lens[0] = 41
    after = g.v1(pa)
    torch.cuda.synchronize()
    assert torch.equal(after[1], before[1])
    assert not torch.equal(after[0], before[0])


# ---------------------------------------------------------------------------
# The workloads at full size, on sampled outputs.
# ---------------------------------------------------------------------------

def _full_size(pa, orc, name, P=None, npairs=48, **kw):
    p = make_problem(name, 0, **kw)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    S, H = p.wl.num_seqs, p.wl.num_heads
    pairs = sample_pairs(S, H, npairs, seed=1)
    ref = c.decode_pairs(orc, pairs)
    out1 = g.v1(pa)
    out2 = g.v2(pa, partition_size=P or p.wl.partition_size or None)
    torch.cuda.synchronize()
    i1 = compare(out1[pairs[:, 0], pairs[:, 1]], ref, f"{name} v1")
    i2 = compare(out2[pairs[:, 0], pairs[:, 1]], ref, f"{name} v2")
    assert torch.isfinite(out1).all() and torch.isfinite(out2).all()
    return i1, i2


def test_qwen3_32b_layer_fp16_full_size(pa, orc):
    _full_size(pa, orc, "qwen3_32b_f16")


def test_long_context_bf16_full_size(pa, orc):
    _full_size(pa, orc, "long_ctx_bf16", P=512, npairs=8)


@pytest.mark.parametrize("name", ["quant_int8", "quant_fp8"])
def test_quantised_full_size(pa, orc, name):
    _full_size(pa, orc, name)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_mixed_batch_shared_prefix(pa, orc, bs):
    _full_size(pa, orc, "mixed_f16", npairs=12, block_size=bs,
               num_seqs=256 if bs == 16 else 48)
