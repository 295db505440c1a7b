"""GPU single-launch persistent decode (pa_decode_fused) against the oracle, and its
workspace contract (counters left at zero, deterministic results)."""
import numpy as np
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, compare, sample_pairs, small_problem
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu

DTYPE_COMBOS = [("f16", "f16"), ("bf16", "bf16"), ("f32", "f32"), ("f16", "int8"),
                ("f16", "fp8"), ("bf16", "int8"), ("bf16", "fp8")]


@pytest.mark.parametrize("dt,cd", DTYPE_COMBOS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fused_matches_oracle(pa, orc, dt, cd, D, bs):
    p = small_problem(cache_dtype=cd, dtype=dt, D=D, bs=bs, seed=11 * D + bs)
    g = GpuProblem(p).fill(pa)
    ref = CpuCaches(p, orc).decode(orc)
    ws = pa.FusedWorkspace(g.q.shape[0], g.kc.shape[2], D)
    compare(g.fused(pa, ws), ref, f"fused {dt}/{cd} D{D} bs{bs}")
    compare(g.fused(pa, ws), ref, f"fused again {dt}/{cd} D{D} bs{bs}")
    torch.cuda.synchronize()
    if cd != "f32":
        assert not ws.counters().any()          # every split unit was merged and reset


@pytest.mark.parametrize("H,Hkv", [(8, 8), (8, 4), (16, 4), (12, 3), (14, 2), (64, 8)])
def test_fused_gqa_group_sizes(pa, orc, H, Hkv):
    p = small_problem(cache_dtype="f16", H=H, Hkv=Hkv, seed=H * 37 + Hkv)
    g = GpuProblem(p).fill(pa)
    ref = CpuCaches(p, orc).decode(orc)
    compare(g.fused(pa), ref, f"fused G{H // Hkv}")


def test_fused_is_deterministic_and_matches_v1_closely(pa, orc):
    p = small_problem(cache_dtype="bf16", lens=(3000, 17, 1, 900, 64, 4096), seed=3)
    g = GpuProblem(p).fill(pa)
    ws = pa.FusedWorkspace(6, 2, 128)
    a = g.fused(pa, ws)
    b = g.fused(pa, ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    compare(a, CpuCaches(p, orc).decode(orc), "fused long/short mix")


def test_fused_empty_and_single_token(pa, orc):
    p = small_problem(cache_dtype="f16", lens=(1, 5, 1, 64), seed=17)
    g = GpuProblem(p).fill(pa)
    g.lens[2] = 0
    lens_cpu = p.batch.seq_lens.clone()
    lens_cpu[2] = 0
    out = g.fused(pa)
    torch.cuda.synchronize()
    assert not out[2].any()
    compare(out, CpuCaches(p, orc).decode(orc, lens=lens_cpu), "fused empty/single")
    G = out.shape[1] // g.new_value.shape[1]
    for h in range(out.shape[1]):
        assert torch.equal(out[0, h], g.new_value[0, h // G])


def test_fused_all_sequences_empty(pa):
    p = small_problem(cache_dtype="f16", lens=(3, 4), seed=19)
    g = GpuProblem(p).fill(pa)
    g.lens.zero_()
    out = g.fused(pa, out=torch.full_like(g.q, 7.0))
    torch.cuda.synchronize()
    assert not out.any()


def test_fused_many_sequences(pa, orc):
    lens = tuple(int(x) for x in np.random.default_rng(1).integers(1, 60, 3000))
    p = small_problem(cache_dtype="f16", H=8, Hkv=8, D=64, lens=lens, seed=23)
    g = GpuProblem(p).fill(pa)
    out = g.fused(pa)
    pairs = sample_pairs(len(lens), 8, 96)
    ref = CpuCaches(p, orc).decode_pairs(orc, pairs)
    compare(out[pairs[:, 0], pairs[:, 1]], ref, "fused 3000 seqs")


@pytest.mark.parametrize("cd", ["f16", "fp8"])
def test_fused_relabelling_and_shared_prefix(pa, orc, cd):
    p = make_problem("mixed_f16", 5, num_seqs=6, cache_dtype=cd)
    g = GpuProblem(p).fill(pa)
    a = g.fused(pa)
    # private copies of the shared prefix: bit-identical
    S = g.tables.shape[0]
    pre = p.wl.shared_prefix_tokens // p.wl.block_size
    nb = g.kc.shape[0]
    for name in ("kc", "vc", "ks", "vs"):
        t = getattr(g, name)
        if t is not None:
            setattr(g, name, torch.cat([t, t[g.tables[:, :pre].reshape(-1).long()]], dim=0))
    t2 = g.tables.clone()
    t2[:, :pre] = (nb + torch.arange(S * pre, device="cuda").view(S, pre)).to(torch.int32)
    g.tables = t2
    b = g.fused(pa)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    pairs = sample_pairs(6, 64, 6, seed=4)
    ref = CpuCaches(p, orc).decode_pairs(orc, pairs)
    compare(a[pairs[:, 0], pairs[:, 1]], ref, "fused shared prefix")


def test_fused_workspace_checks(pa):
    p = small_problem(cache_dtype="f16", seed=29)
    g = GpuProblem(p).fill(pa)
    ws = pa.FusedWorkspace(g.q.shape[0], 2, 128)
    ws.nbytes = 1024                              # claims to be too small
    with pytest.raises(pa.PAError):
        g.fused(pa, ws)


@pytest.mark.parametrize("name,npairs", [("qwen3_32b_f16", 48), ("long_ctx_bf16", 8),
                                         ("quant_int8", 48), ("quant_fp8", 48),
                                         ("mixed_f16", 12)])
def test_fused_full_size(pa, orc, name, npairs):
    p = make_problem(name, 0)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    pairs = sample_pairs(p.wl.num_seqs, p.wl.num_heads, npairs, seed=2)
    ref = c.decode_pairs(orc, pairs)
    ws = pa.FusedWorkspace(p.wl.num_seqs, p.wl.num_kv_heads, p.wl.head_dim)
    out = g.fused(pa, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    compare(out[pairs[:, 0], pairs[:, 1]], ref, f"fused {name}")
    assert not ws.counters().any()


def test_fused_bounds_flag_and_time_out(pa, orc):
    p = small_problem(cache_dtype="f16", lens=(2000, 1800, 1900, 2100), seed=31)
    g = GpuProblem(p).fill(pa)
    f = torch.zeros(1, dtype=torch.int32, device="cuda")
    g2 = GpuProblem(p).fill(pa)
    g2.tables[1, 3] = g2.kc.shape[0] + 9
    g2.lens[2] = g2.tables.shape[1] * 16 + 50
    out = g2.fused(pa, err_flag=f)
    torch.cuda.synchronize()
    assert int(f.item()) & pa.DEVERR_BLOCK_ID and int(f.item()) & pa.DEVERR_SEQ_LEN
    assert torch.isfinite(out).all() and not out[2].any()
    pa.get_device_error(clear=True)
    f.zero_()
    try:
        pa.set_wait_limit_ns(1_000_000)
        pa.set_fault_injection(1)
        out = g.fused(pa, err_flag=f)
        torch.cuda.synchronize()
    finally:
        pa.set_fault_injection(0)
        pa.set_wait_limit_ns(0)
    assert int(f.item()) & pa.DEVERR_TIMEOUT
    assert pa.get_device_error(clear=True) & pa.DEVERR_TIMEOUT
    compare(g.fused(pa), CpuCaches(p, orc).decode(orc), "fused after time-out")
