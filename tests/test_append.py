"""pa_append_decode_v1 -- the cache write of each sequence's new token fused into the
v1 decode (one launch) -- against the two separate calls (bit-identical caches and
output) and against the oracle's cache write followed by its decode."""
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, bytes_equal, compare, sample_pairs, small_problem
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu

CACHES = ["f32", "f16", "bf16", "int8", "fp8"]


def _append(pa, g, **kw):
    return pa.append_decode_v1(g.q, g.new_key, g.new_value, g.new_slots, g.kc, g.vc, g.tables,
                               g.lens, g.p.wl.scale, cache_dtype=g.cd, k_scale=g.ks,
                               v_scale=g.vs, **kw)


@pytest.mark.parametrize("cd", CACHES)
@pytest.mark.parametrize("D,bs", [(128, 16), (64, 8), (128, 32), (64, 16)])
def test_append_equals_write_then_decode(pa, cd, D, bs):
    p = small_problem(cache_dtype=cd, D=D, bs=bs, seed=3 * D + bs)
    two = GpuProblem(p).fill(pa)                  # history + new token, separate write
    ref = two.v1(pa)
    one = GpuProblem(p).fill(pa, include_new=False)
    out = _append(pa, one)
    torch.cuda.synchronize()
    assert bytes_equal(one.kc, two.kc) and bytes_equal(one.vc, two.vc)
    if one.ks is not None:
        assert bytes_equal(one.ks, two.ks) and bytes_equal(one.vs, two.vs)
    assert bytes_equal(out, ref)


@pytest.mark.parametrize("cd", CACHES)
def test_append_against_the_oracle(pa, orc, cd):
    p = small_problem(cache_dtype=cd, seed=11)
    g = GpuProblem(p).fill(pa, include_new=False)
    out = _append(pa, g)
    torch.cuda.synchronize()
    c = CpuCaches(p, orc)                         # the oracle writes history + new token
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)
    compare(out, c.decode(orc), f"append + decode, {cd} cache")


@pytest.mark.parametrize("name", ["qwen3_32b_f16", "quant_int8", "quant_fp8"])
def test_append_at_full_size_sampled(pa, orc, name):
    """The full batch in one launch; sampled (sequence, head) outputs against the
    oracle over the oracle's own caches."""
    p = make_problem(name, 21)
    g = GpuProblem(p).fill(pa, include_new=False)
    out = _append(pa, g)
    torch.cuda.synchronize()
    c = CpuCaches(p, orc)
    pairs = sample_pairs(p.wl.num_seqs, p.wl.num_heads, 48, seed=2)
    ref = c.decode_pairs(orc, pairs)
    got = torch.stack([out[s, h] for s, h in pairs.tolist()])
    compare(got, ref, f"append + decode sampled, {name}")


def test_negative_slot_writes_nothing(pa):
    p = small_problem(cache_dtype="f16", seed=4)
    g = GpuProblem(p).fill(pa, include_new=False)
    before_k = g.kc.clone()
    g.new_slots[:] = -1
    out = _append(pa, g)
    ref = g.v1(pa)                                # the cache as it was
    torch.cuda.synchronize()
    assert bytes_equal(g.kc, before_k)
    assert bytes_equal(out, ref)


def test_slot_past_the_pool_is_flagged(pa):
    p = small_problem(cache_dtype="bf16", seed=6)
    g = GpuProblem(p).fill(pa, include_new=False)
    before_k = g.kc.clone()
    g.new_slots[0] = p.num_blocks * p.wl.block_size
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    _append(pa, g, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_SLOT
    pa.get_device_error(clear=True)
    changed = (g.kc.view(torch.int16) != before_k.view(torch.int16)).flatten(1).any(1)
    written = {int(s) // p.wl.block_size for s in g.new_slots[1:].tolist()}
    assert set(torch.nonzero(changed).flatten().tolist()) <= written


@pytest.mark.parametrize("tiles", [0, 1, 8])
def test_prefetch_depth_does_not_change_results(pa, tiles):
    p = small_problem(cache_dtype="f16", seed=8)
    g = GpuProblem(p).fill(pa)
    ref = g.v1(pa)
    try:
        pa.set_pdl(2)
        pa.set_prefetch_tiles(tiles)
        out = g.v1(pa)
        torch.cuda.synchronize()
    finally:
        pa.set_prefetch_tiles(-1)
        pa.set_pdl(1)
    assert bytes_equal(out, ref)
