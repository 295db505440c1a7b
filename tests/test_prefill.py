"""pa_prefill -- causal multi-token query over the paged cache on the tcgen05 tensor
cores -- against the oracle's prefill (small cases, every output) and, at full size,
on sampled rows through the oracle's single-query decode (a query row at position p is
the decode over the first p + 1 tokens)."""
import numpy as np
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, compare
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu


def _setup(pa, orc, lens, qlens, dt="bf16", bs=16, H=16, Hkv=2, seed=0, cpu=True):
    p = make_problem("qwen3_32b_f16", seed, num_seqs=len(lens), seq_lens=list(lens),
                     num_heads=H, num_kv_heads=Hkv, head_dim=128, block_size=bs, dtype=dt,
                     cache_dtype=dt, num_blocks=sum(-(-n // bs) for n in lens) + 5)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc) if cpu else None
    gen = torch.Generator().manual_seed(seed + 1)
    qs = torch.tensor([0] + list(np.cumsum(qlens)), dtype=torch.int32)
    q = torch.randn((int(qs[-1]), H, 128), generator=gen).to(g.q.dtype)
    return p, g, c, q, qs


def _run(pa, p, g, q, qs, **kw):
    out = pa.prefill(q.cuda(), g.kc, g.vc, g.tables, g.lens, qs.cuda(), p.wl.scale, **kw)
    if "err_flag" not in kw:                         # no device error on a good problem
        torch.cuda.synchronize()
        assert pa.get_device_error(clear=True) == 0
    return out


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("bs", [16, 32, 8])
def test_prefill_matches_the_oracle(pa, orc, dt, bs):
    lens = [1, 17, 130, 300, 257, 64]
    qlens = [1, 17, 30, 300, 129, 1]                 # whole prompts, chunks after a prefix
    p, g, c, q, qs = _setup(pa, orc, lens, qlens, dt=dt, bs=bs, seed=bs)
    out = _run(pa, p, g, q, qs)
    torch.cuda.synchronize()
    ref = orc.paged_prefill(q, c.kc, c.vc, p.batch.block_tables, p.batch.seq_lens, qs,
                            p.wl.scale)
    compare(out, ref, f"prefill {dt} bs{bs}")


@pytest.mark.parametrize("H,Hkv", [(64, 8), (8, 8), (32, 8), (16, 1)])
def test_prefill_gqa_groups(pa, orc, H, Hkv):
    lens, qlens = [200, 45], [70, 45]
    p, g, c, q, qs = _setup(pa, orc, lens, qlens, H=H, Hkv=Hkv, seed=H + Hkv)
    out = _run(pa, p, g, q, qs)
    torch.cuda.synchronize()
    ref = orc.paged_prefill(q, c.kc, c.vc, p.batch.block_tables, p.batch.seq_lens, qs,
                            p.wl.scale)
    compare(out, ref, f"prefill G={H // Hkv}")


def test_prefill_of_one_token_matches_the_decode(pa, orc):
    lens = [5, 77, 300]
    p, g, c, q, qs = _setup(pa, orc, lens, [1, 1, 1], dt="f16", seed=4)
    out = _run(pa, p, g, q, qs)
    dec = pa.decode_v1(q.cuda(), g.kc, g.vc, g.tables, g.lens, p.wl.scale)
    torch.cuda.synchronize()
    ref = orc.paged_decode(q, c.kc, c.vc, p.batch.block_tables, p.batch.seq_lens, p.wl.scale)
    compare(out, ref, "prefill q_len 1")
    compare(dec, ref, "decode")


def test_prefill_over_a_shared_prefix(pa, orc):
    """Three requests share a cached 512-token prompt (the same physical blocks) and
    each computes only its own new tokens."""
    bs, prefix = 16, 512
    news = [40, 1, 129]
    lens = [prefix + n for n in news]
    p = make_problem("qwen3_32b_f16", 9, num_seqs=3, seq_lens=lens, num_heads=16,
                     num_kv_heads=2, dtype="bf16", cache_dtype="bf16",
                     num_blocks=sum(-(-n // bs) for n in lens) + 5)
    # point every table's first 32 blocks at sequence 0's prompt blocks
    tables = p.batch.block_tables.clone()
    tables[1:, :prefix // bs] = tables[0, :prefix // bs]
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    gen = torch.Generator().manual_seed(3)
    qs = torch.tensor([0] + list(np.cumsum(news)), dtype=torch.int32)
    q = torch.randn((int(qs[-1]), 16, 128), generator=gen).to(torch.bfloat16)
    out = pa.prefill(q.cuda(), g.kc, g.vc, tables.cuda(), g.lens, qs.cuda(), p.wl.scale)
    torch.cuda.synchronize()
    ref = orc.paged_prefill(q, c.kc, c.vc, tables, p.batch.seq_lens, qs, p.wl.scale)
    compare(out, ref, "prefill over a shared prefix")


def test_prefill_full_size_sampled(pa, orc):
    """8 sequences, 4096 cached tokens + a 512-token chunk each, 64 q / 8 kv heads:
    sampled (row, head) outputs against the oracle's decode of that row."""
    lens = [4096 + 512] * 8
    qlens = [512] * 8
    p, g, _, q, qs = _setup(pa, orc, lens, qlens, H=64, Hkv=8, seed=12, cpu=False)
    out = _run(pa, p, g, q, qs)
    torch.cuda.synchronize()
    c = CpuCaches(p, orc)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, int(qs[-1]), 24)
    heads = rng.integers(0, 64, 24)
    seq_of = np.searchsorted(qs.numpy(), rows, side="right") - 1
    pos = np.array([lens[s] - qlens[s] + (r - int(qs[s])) for r, s in zip(rows, seq_of)])
    # each sampled row as its own decode over the first pos + 1 tokens
    qd = q[torch.from_numpy(rows)]
    tables = p.batch.block_tables[torch.from_numpy(seq_of)]
    dlens = torch.from_numpy(pos + 1).to(torch.int32)
    pairs = np.stack([np.arange(24), heads], 1).astype(np.int32)
    ref = orc.paged_decode_pairs(qd, c.kc, c.vc, tables, dlens, p.wl.scale, pairs)
    got = torch.stack([out[int(r), int(h)] for r, h in zip(rows, heads)])
    compare(got, ref, "prefill full size, sampled")


def test_prefill_flags_a_bad_sequence_and_keeps_the_others(pa, orc):
    lens, qlens = [100, 60], [20, 60]
    p, g, c, q, qs = _setup(pa, orc, lens, qlens, seed=21)
    bad = g.lens.clone()
    bad[0] = 10                                      # shorter than its chunk
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros((int(qs[-1]), 16, 128), dtype=torch.bfloat16, device="cuda")
    pa.prefill(q.cuda(), g.kc, g.vc, g.tables, bad, qs.cuda(), p.wl.scale, out=out,
               err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pa.DEVERR_SEQ_LEN
    pa.get_device_error(clear=True)
    ref = orc.paged_prefill(q[20:], c.kc, c.vc, p.batch.block_tables[1:], p.batch.seq_lens[1:],
                            torch.tensor([0, 60], dtype=torch.int32), p.wl.scale)
    compare(out[20:], ref, "prefill, the good sequence")


def test_prefill_wait_timeout_is_reported(pa, orc):
    lens, qlens = [300], [40]
    p, g, _, q, qs = _setup(pa, orc, lens, qlens, seed=5, cpu=False)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        pa.set_wait_limit_ns(1_000_000)
        pa.set_fault_injection(1)
        pa.prefill(q.cuda(), g.kc, g.vc, g.tables, g.lens, qs.cuda(), p.wl.scale, err_flag=flag)
        torch.cuda.synchronize()
    finally:
        pa.set_fault_injection(0)
        pa.set_wait_limit_ns(0)
    assert int(flag.item()) & pa.DEVERR_TIMEOUT
    pa.get_device_error(clear=True)
    out = _run(pa, p, g, q, qs)                      # the context still computes
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
