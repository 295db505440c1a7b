"""pa_decode_cascade -- decode of sequences that share a cached prefix: the prefix on the
tcgen05 tensor cores once per kv head, each sequence's own tokens on the persistent decode
(or, as the second form, the v1 decode), merged by log-sum-exp -- against the oracle's
decode (the same attention, computed plainly)."""
import numpy as np
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, compare, sample_pairs
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_error(pa):
    """Every case here is a good problem: no kernel may report a device error."""
    pa.get_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert pa.get_device_error(clear=True) == 0


@pytest.fixture(params=[0, 1], ids=["persistent-suffix", "v1-suffix"])
def form(request, pa):
    """Both forms of the suffix launch (pa_set_cascade_config)."""
    pa.set_cascade_config(0, request.param)
    yield request.param
    pa.set_cascade_config(0, 0)


@pytest.fixture(params=[0, -1], ids=["auto", "side-by-side"])
def placement(request, pa, form):
    """The automatic placement (on these small batches: the prefix split to fill the GPU,
    then the suffix) and side by side forced (split count -1: the unsplit prefix on its
    own SMs, the suffix's capped build on all the others)."""
    pa.set_cascade_config(request.param, form)
    yield request.param
    pa.set_cascade_config(0, form)


def _problem(lens, prefix, dt="f16", H=64, Hkv=8, bs=16, seed=0, S=None):
    return make_problem("mixed_f16", seed, num_seqs=S or len(lens), seq_lens=lens,
                        shared_prefix_tokens=prefix, dtype=dt, cache_dtype=dt, num_heads=H,
                        num_kv_heads=Hkv, block_size=bs)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [16, 32, 8])
def test_cascade_matches_the_oracle(pa, orc, dt, bs, form, placement):
    prefix = 256
    lens = [prefix + n for n in (1, 17, 130, 300, 0 + 1, 64, 257, 5, 96, 33, 2, 200)]
    p = _problem(lens, prefix, dt=dt, bs=bs, seed=bs)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    out = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, prefix)
    torch.cuda.synchronize()
    compare(out, c.decode(orc), f"cascade {dt} bs{bs}")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_cascade_prefix_split_over_ctas(pa, orc, dt, form):
    """A long prefix and few sequences: the prefix kernel splits the prefix over up to
    4 CTAs per query tile and the decode merges every split's partial."""
    prefix = 2048 + 512
    lens = [prefix + n for n in (1, 50, 300, 17, 129, 2)]
    p = _problem(lens, prefix, dt=dt, seed=31)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    pa.set_cascade_config(4, form)                    # four splits of the prefix
    out = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, prefix)
    torch.cuda.synchronize()
    compare(out, c.decode(orc), f"cascade with prefix splits, {dt}")


@pytest.mark.parametrize("H,Hkv", [(64, 8), (8, 8), (32, 8), (8, 1)])
def test_cascade_gqa_groups(pa, orc, H, Hkv, form, placement):
    prefix = 384
    lens = [prefix + n for n in (40, 1, 129, 7, 300)]
    p = _problem(lens, prefix, H=H, Hkv=Hkv, seed=H + Hkv)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    out = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, prefix)
    torch.cuda.synchronize()
    compare(out, c.decode(orc), f"cascade G={H // Hkv}")


def test_cascade_edge_lengths_and_plain_decode(pa, orc, form):
    """Sequences that end exactly at the prefix; prefix_len 0 is pa_decode_v1."""
    prefix = 128
    lens = [prefix + 1, prefix + 1, prefix + 16, prefix + 1]
    p = _problem(lens, prefix, seed=3)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    short = g.lens.clone()
    short[:] = prefix                                   # only the prefix left to attend to
    out = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, short, p.wl.scale, prefix)
    torch.cuda.synchronize()
    compare(out, c.decode(orc, lens=short.cpu()), "cascade, prefix only")
    zero = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, 0)
    v1 = g.v1(pa)
    torch.cuda.synchronize()
    assert torch.equal(zero, v1)


def test_cascade_full_mixed_workload_sampled(pa, orc, form):
    """The mixed serving batch: 256 sequences after an 8192-token shared prompt."""
    p = make_problem("mixed_f16", 0)
    g = GpuProblem(p).fill(pa)
    out = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale,
                            p.wl.shared_prefix_tokens)
    torch.cuda.synchronize()
    c = CpuCaches(p, orc)
    pairs = sample_pairs(p.wl.num_seqs, p.wl.num_heads, 40, seed=5)
    ref = c.decode_pairs(orc, pairs)
    got = torch.stack([out[s, h] for s, h in pairs.tolist()])
    compare(got, ref, "cascade, mixed workload sampled")


def test_cascade_workspace_checks(pa):
    p = _problem([160, 170], 128, seed=1)
    g = GpuProblem(p).fill(pa)
    p16 = _problem([160, 170], 128, seed=1, H=16, Hkv=1)
    g16 = GpuProblem(p16).fill(pa)
    with pytest.raises(pa.PAError) as e:               # the v1 decode takes groups <= 8
        pa.decode_cascade(g16.q, g16.kc, g16.vc, g16.tables, g16.lens, p.wl.scale, 128)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PAError):
        pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, 128, workspace=small)
    with pytest.raises(pa.PAError):                    # not whole blocks
        pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, 100)


@pytest.mark.parametrize("splits", [-1, 0, 1, 2, 4])
def test_cascade_repeated_calls_share_one_workspace(pa, orc, splits):
    """The counters inside the workspace start at zero and every call leaves them so:
    three calls in a row on one workspace give the same bits, and match the oracle;
    every prefix split count gives a correct result (-1: side by side, the prefix
    unsplit on its own SMs and the suffix's capped build on the others; 0: the
    automatic placement)."""
    prefix = 1024
    lens = [prefix + n for n in (1, 300, 17, 129, 64, 2, 555, 40)]
    p = _problem(lens, prefix, seed=41)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    n = pa.lib().pa_decode_cascade_workspace_bytes(g.q.shape[0], g.q.shape[1], g.q.shape[2])
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    try:
        pa.set_cascade_config(splits, 0)
        outs = [pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, prefix,
                                  workspace=ws).clone() for _ in range(3)]
    finally:
        pa.set_cascade_config(0, 0)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    compare(outs[0], c.decode(orc), f"cascade, {splits} prefix splits")


@pytest.mark.parametrize("splits", [0, -1])
@pytest.mark.parametrize("pdl", [0, 1, 2])
def test_cascade_every_pdl_mode(pa, orc, pdl, splits):
    """Side by side needs PDL: without it even split count -1 falls back to the split
    prefix followed by the suffix on every SM.  Every combination matches the oracle."""
    prefix = 512
    lens = [prefix + n for n in (3, 200, 1, 77, 130, 16)]
    p = _problem(lens, prefix, seed=53)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    try:
        pa.set_pdl(pdl)
        pa.set_cascade_config(splits, 0)
        out = pa.decode_cascade(g.q, g.kc, g.vc, g.tables, g.lens, p.wl.scale, prefix)
        torch.cuda.synchronize()
    finally:
        pa.set_pdl(1)
        pa.set_cascade_config(0, 0)
    compare(out, c.decode(orc), f"cascade, PDL mode {pdl}")
