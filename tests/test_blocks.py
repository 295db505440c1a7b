"""GPU block copy (pa_copy_blocks) against the oracle's: copy-on-write inside one pool and
swap between the device pool and a pinned host pool, bit-exact over the whole pools."""
import numpy as np
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, bytes_equal, compare, small_problem
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu


def _live_and_free(p):
    live = sorted({int(x) for x in p.batch.block_tables.flatten() if x >= 0})
    used = set(live) | {int(s) // p.wl.block_size for s in p.hist_slots.tolist() if s >= 0}
    free = [b for b in range(p.num_blocks) if b not in used]
    return live, free


def _pairs(p, n, seed):
    live, free = _live_and_free(p)
    g = torch.Generator().manual_seed(seed)
    src = [live[i] for i in torch.randint(0, len(live), (n,), generator=g).tolist()]
    dst = [free[i] for i in torch.randperm(len(free), generator=g)[:n].tolist()]
    return torch.tensor(list(zip(src, dst)), dtype=torch.int64)


@pytest.mark.parametrize("cd", ["f32", "f16", "bf16", "int8", "fp8"])
@pytest.mark.parametrize("D,bs", [(64, 8), (128, 16), (128, 32), (64, 32)])
def test_copy_within_pool_bit_exact(pa, orc, cd, D, bs):
    p = small_problem(cache_dtype=cd, D=D, bs=bs, seed=D + bs)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    pairs = _pairs(p, 6, seed=bs)
    pa.copy_blocks(g.kc, g.vc, g.kc, g.vc, pairs.cuda(), cache_dtype=cd, src_k_scale=g.ks,
                   src_v_scale=g.vs, dst_k_scale=g.ks, dst_v_scale=g.vs)
    orc.copy_blocks(c.kc, c.vc, c.kc, c.vc, pairs, cache_dtype=cd, src_k_scale=c.ks,
                    src_v_scale=c.vs, dst_k_scale=c.ks, dst_v_scale=c.vs)
    torch.cuda.synchronize()
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)
    if c.ks is not None:
        assert bytes_equal(g.ks, c.ks) and bytes_equal(g.vs, c.vs)


@pytest.mark.parametrize("cd", ["bf16", "fp8"])
def test_swap_out_to_pinned_host_and_back_in(pa, orc, cd):
    p = small_problem(cache_dtype=cd, seed=5)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    before = g.v1(pa)
    live, free = _live_and_free(p)
    n = len(live)
    # swap out: every live block to a pinned host pool of n blocks
    shape = (n,) + tuple(g.kc.shape[1:])
    hk = torch.zeros(shape, dtype=g.kc.dtype).pin_memory()
    hv = torch.zeros(shape, dtype=g.kc.dtype).pin_memory()
    hks = hvs = None
    if g.ks is not None:
        hks = torch.zeros((n,) + tuple(g.ks.shape[1:])).pin_memory()
        hvs = torch.zeros((n,) + tuple(g.ks.shape[1:])).pin_memory()
    out_pairs = torch.tensor([[b, i] for i, b in enumerate(live)], dtype=torch.int64)
    pa.copy_blocks(g.kc, g.vc, hk, hv, out_pairs.cuda(), cache_dtype=cd, src_k_scale=g.ks,
                   src_v_scale=g.vs, dst_k_scale=hks, dst_v_scale=hvs)
    torch.cuda.synchronize()
    ck, cv = torch.zeros(shape, dtype=g.kc.dtype), torch.zeros(shape, dtype=g.kc.dtype)
    cks = torch.zeros_like(hks) if hks is not None else None
    cvs = torch.zeros_like(hvs) if hvs is not None else None
    orc.copy_blocks(c.kc, c.vc, ck, cv, out_pairs, cache_dtype=cd, src_k_scale=c.ks,
                    src_v_scale=c.vs, dst_k_scale=cks, dst_v_scale=cvs)
    assert bytes_equal(hk, ck) and bytes_equal(hv, cv)
    if hks is not None:
        assert bytes_equal(hks, cks) and bytes_equal(hvs, cvs)
    # swap in: back into a fresh device pool at relabelled ids; the decode with the
    # relabelled tables is bit-identical (tokens are visited in logical order)
    kc2 = torch.full_like(g.kc, 0)
    vc2 = torch.full_like(g.vc, 0)
    ks2 = torch.full_like(g.ks, float("nan")) if g.ks is not None else None
    vs2 = torch.full_like(g.vs, float("nan")) if g.vs is not None else None
    perm = torch.randperm(p.num_blocks, generator=torch.Generator().manual_seed(3))[:n]
    in_pairs = torch.tensor([[i, int(perm[i])] for i in range(n)], dtype=torch.int64)
    pa.copy_blocks(hk, hv, kc2, vc2, in_pairs.cuda(), cache_dtype=cd, src_k_scale=hks,
                   src_v_scale=hvs, dst_k_scale=ks2, dst_v_scale=vs2)
    remap = {b: int(perm[i]) for i, b in enumerate(live)}
    t2 = p.batch.block_tables.clone()
    for idx, x in np.ndenumerate(t2.numpy()):
        if x >= 0:
            t2[idx] = remap[int(x)]
    after = pa.decode_v1(g.q, kc2, vc2, t2.cuda(), g.lens, p.wl.scale, cache_dtype=cd,
                         k_scale=ks2, v_scale=vs2)
    torch.cuda.synchronize()
    assert bytes_equal(after, before)


def test_copy_on_write_then_decode(pa, orc):
    """Every sequence's table points at the same blocks; sequence 1 then appends a
    token: its last block is copied to a free id, its table repointed and the token
    written there.  Sequence 0's output is unchanged (bit-identical) and both match
    the oracle run through the same steps."""
    p = make_problem("qwen3_32b_f16", 4, num_seqs=2, seq_lens=[200, 200], num_heads=16,
                     num_kv_heads=2, num_blocks=40)
    bs = p.wl.block_size
    g = GpuProblem(p).fill(pa, include_new=False)
    c = CpuCaches(p, orc, include_new=False)
    # both sequences share sequence 0's blocks and its 199 cached tokens
    shared = p.batch.block_tables.clone()
    shared[1] = shared[0]
    lens = torch.tensor([199, 199], dtype=torch.int32)
    before = pa.decode_v1(g.q, g.kc, g.vc, shared.cuda(), lens.cuda(), p.wl.scale)
    _, free = _live_and_free(p)
    last = int(shared[0, 199 // bs])
    fresh = free[0]
    pair = torch.tensor([[last, fresh]], dtype=torch.int64)
    own = shared.clone()
    own[1, 199 // bs] = fresh
    slot = torch.tensor([fresh * bs + 199 % bs], dtype=torch.int64)
    nk, nv = p.batch.new_key[1:2], p.batch.new_value[1:2]
    pa.copy_blocks(g.kc, g.vc, g.kc, g.vc, pair.cuda())
    pa.reshape_and_cache(nk.cuda(), nv.cuda(), g.kc, g.vc, slot.cuda())
    lens2 = torch.tensor([199, 200], dtype=torch.int32)
    after = pa.decode_v1(g.q, g.kc, g.vc, own.cuda(), lens2.cuda(), p.wl.scale)
    torch.cuda.synchronize()
    assert bytes_equal(after[0], before[0])
    orc.copy_blocks(c.kc, c.vc, c.kc, c.vc, pair)
    orc.reshape_and_cache(nk, nv, c.kc, c.vc, slot)
    ref = orc.paged_decode(p.batch.q, c.kc, c.vc, own, lens2, p.wl.scale)
    compare(after, ref, "decode after copy-on-write")
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)


def test_out_of_range_pair_is_skipped_and_flagged(pa, orc):
    p = small_problem(cache_dtype="f16", seed=2)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    good = _pairs(p, 3, seed=1)
    bad = torch.tensor([[0, p.num_blocks], [-1, int(good[0, 1]) + 0]], dtype=torch.int64)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.get_device_error(clear=True)
    pa.copy_blocks(g.kc, g.vc, g.kc, g.vc, torch.cat([good, bad]).cuda(), err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == pa.DEVERR_BLOCK_ID
    assert pa.get_device_error(clear=True) & pa.DEVERR_BLOCK_ID
    orc.copy_blocks(c.kc, c.vc, c.kc, c.vc, good)
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)


def test_many_pairs_at_the_qwen3_32b_block_shape(pa, orc):
    """1500 pairs of 16 x 8 x 128 fp16 blocks (64 KB of K+V each), one launch."""
    nb, bs, Hkv, D, n = 4096, 16, 8, 128, 1500
    gen = torch.Generator().manual_seed(0)
    kc = torch.randn((nb, bs, Hkv, D), generator=gen).half()
    vc = torch.randn((nb, bs, Hkv, D), generator=gen).half()
    ids = torch.randperm(nb, generator=gen)
    pairs = torch.stack([ids[:n], ids[n:2 * n]], 1).to(torch.int64)
    gk, gv = kc.cuda(), vc.cuda()
    pa.copy_blocks(gk, gv, gk, gv, pairs.cuda())
    orc.copy_blocks(kc, vc, kc, vc, pairs)
    torch.cuda.synchronize()
    assert bytes_equal(gk, kc) and bytes_equal(gv, vc)
