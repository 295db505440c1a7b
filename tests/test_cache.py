"""GPU cache write (reshape_and_cache) against the oracle's: bit-exact caches and scales."""
import numpy as np
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, bytes_equal, small_problem
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu

COMBOS = [("f32", "f32"), ("f16", "f16"), ("bf16", "bf16"), ("f16", "int8"), ("bf16", "int8"),
          ("f32", "int8"), ("f16", "fp8"), ("bf16", "fp8"), ("f32", "fp8")]


@pytest.mark.parametrize("src,cd", COMBOS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_cache_write_bit_exact(pa, orc, src, cd, D, bs):
    p = small_problem(cache_dtype=cd, dtype=src, D=D, bs=bs, seed=D + bs)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)
    if c.ks is not None:
        assert bytes_equal(g.ks, c.ks) and bytes_equal(g.vs, c.vs)


@pytest.mark.parametrize("cd", ["int8", "fp8"])
def test_quantised_write_wide_range_and_ties(pa, orc, cd):
    """Rows with wide dynamic range, exact ties and an all-zero row."""
    nb, bs, Hkv, D = 8, 16, 2, 128
    gen = torch.Generator().manual_seed(3)
    n = 40
    x = torch.randn((n, Hkv, D), generator=gen) * torch.logspace(-6, 4, n).view(n, 1, 1)
    x[5] = 0.0
    # a row whose absmax is 127 so s = 1 and many x/s land exactly on k + 0.5
    x[6, 0] = torch.arange(D, dtype=torch.float32) / 2 - 31.5
    x[6, 0, 0] = 127.0
    storage = torch.int8 if cd == "int8" else torch.uint8
    kc = torch.zeros((nb, bs, Hkv, D), dtype=storage)
    ks = torch.full((nb, Hkv, bs), float("nan"))
    slots = torch.randperm(nb * bs, generator=gen)[:n]
    kc_o, vc_o, ks_o, vs_o = kc.clone(), kc.clone(), ks.clone(), ks.clone()
    orc.reshape_and_cache(x, x, kc_o, vc_o, slots, cache_dtype=cd, k_scale=ks_o, v_scale=vs_o)
    kc_g, vc_g, ks_g, vs_g = kc.cuda(), kc.cuda(), ks.cuda(), ks.cuda()
    pa.reshape_and_cache(x.cuda(), x.cuda(), kc_g, vc_g, slots.cuda(), cache_dtype=cd,
                         k_scale=ks_g, v_scale=vs_g)
    torch.cuda.synchronize()
    assert bytes_equal(kc_g, kc_o) and bytes_equal(vc_g, vc_o)
    assert bytes_equal(ks_g, ks_o) and bytes_equal(vs_g, vs_o)


def test_negative_slots_skip_and_untouched_slots_keep_poison(pa, orc):
    p = small_problem(cache_dtype="f16", seed=5)
    g = GpuProblem(p)
    g.new_slots[::2] = -1
    p.batch.new_slots[::2] = -1
    g.fill(pa)
    c = CpuCaches(p, orc)
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)


def test_zero_tokens_is_a_no_op(pa):
    kc = torch.zeros((4, 16, 1, 64), dtype=torch.float16, device="cuda")
    e = torch.empty((0, 1, 64), dtype=torch.float16, device="cuda")
    pa.reshape_and_cache(e, e, kc, kc.clone(), torch.empty((0,), dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert not kc.any()


@pytest.mark.parametrize("name", ["quant_int8", "quant_fp8"])
def test_quantised_full_pool_bit_exact(pa, orc, name):
    """Config-4 scale: every history token of 32 seqs (len 512..768) into a 12480-block pool."""
    p = make_problem(name, 0)
    g = GpuProblem(p).fill(pa)
    c = CpuCaches(p, orc)
    assert bytes_equal(g.kc, c.kc) and bytes_equal(g.vc, c.vc)
    assert bytes_equal(g.ks, c.ks) and bytes_equal(g.vs, c.vs)


def _near_boundaries(cd, n_rows, D, seed):
    """fp32 rows whose quotients x / s sit on and within a few ulps of the points where
    the code changes (half-integers for INT8, midpoints between E4M3 values for FP8)."""
    rng = np.random.default_rng(seed)
    qmax = 127.0 if cd == "int8" else 448.0
    if cd == "int8":
        bounds = np.arange(-126.5, 127.0, 1.0)
    else:
        vals = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
        v = np.unique(vals.to(torch.float64).numpy())
        v = v[np.isfinite(v)]
        bounds = (v[:-1] + v[1:]) / 2
    rows = np.empty((n_rows, D), dtype=np.float32)
    for i in range(n_rows):
        amax = np.float32(rng.uniform(0.01, 50.0))
        s = np.float32(amax / np.float32(qmax))
        b = rng.choice(bounds, D - 1)
        x = (b * np.float64(s)).astype(np.float32)
        steps = rng.integers(-3, 4, D - 1)
        for k in range(D - 1):
            for _ in range(abs(int(steps[k]))):
                x[k] = np.nextafter(x[k], np.float32(np.inf if steps[k] > 0 else -np.inf))
        x = np.clip(x, -amax, amax)
        rows[i, 0] = amax * (1 if rng.random() < 0.5 else -1)
        rows[i, 1:] = x
    return torch.from_numpy(rows)


@pytest.mark.parametrize("cd", ["int8", "fp8"])
@pytest.mark.parametrize("D", [64, 128])
def test_quantised_write_near_code_boundaries(pa, orc, cd, D):
    """Quotients on and next to every rounding boundary: the codes still equal those
    of the IEEE fp32 division bit for bit."""
    Hkv, bs = 2, 16
    n = 512
    x = _near_boundaries(cd, n * Hkv, D, seed=D + len(cd)).view(n, Hkv, D)
    nb = n // bs + 1
    storage = torch.int8 if cd == "int8" else torch.uint8
    kc = torch.zeros((nb, bs, Hkv, D), dtype=storage)
    ks = torch.full((nb, Hkv, bs), float("nan"))
    slots = torch.randperm(nb * bs, generator=torch.Generator().manual_seed(1))[:n]
    kc_o, vc_o, ks_o, vs_o = kc.clone(), kc.clone(), ks.clone(), ks.clone()
    xv = -x
    orc.reshape_and_cache(x, xv, kc_o, vc_o, slots, cache_dtype=cd, k_scale=ks_o, v_scale=vs_o)
    kc_g, vc_g, ks_g, vs_g = kc.cuda(), kc.cuda(), ks.cuda(), ks.cuda()
    pa.reshape_and_cache(x.cuda(), xv.cuda(), kc_g, vc_g, slots.cuda(), cache_dtype=cd,
                         k_scale=ks_g, v_scale=vs_g)
    torch.cuda.synchronize()
    assert bytes_equal(ks_g, ks_o) and bytes_equal(vs_g, vs_o)
    assert bytes_equal(kc_g, kc_o) and bytes_equal(vc_g, vc_o)
