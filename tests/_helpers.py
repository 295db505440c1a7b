"""Shared helpers for the GPU parity tests: move a seeded problem to the GPU,
fill its caches on both sides (each with its own cache write), and compare a
GPU result with the oracle under the tolerances of the comparison rule."""
from __future__ import annotations

import math

import numpy as np
import torch

from paged_kv_cache_390_b200.workloads import FLOAT_DTYPES, Problem, make_problem

# Comparison rule: the GPU output is compared with the oracle's binary64 result
# rounded (nearest-even) to the output dtype.  16-bit outputs: relative L2 <= 1e-3,
# and each element within max(2e-3, one ulp of the output dtype at the reference)
# -- rounding is discontinuous, so any fp32 difference can put the GPU value one
# ulp away from the rounded reference, and for |out| >= 0.5 a bf16 ulp (2^-8) is
# already above 2e-3.  fp32 outputs: relative L2 <= 1e-5 and max abs <= 1e-5
# (scaled by the largest |reference| when that exceeds 1).
TOL16_MAX_ABS = 2e-3
TOL16_REL_L2 = 1e-3
TOL32 = 1e-5
_MANT_BITS = {torch.float16: 10, torch.bfloat16: 7}
_MIN_EXP = {torch.float16: -14, torch.bfloat16: -126}


def ulp(x: np.ndarray, dt) -> np.ndarray:
    """Spacing of the dtype's representable numbers at |x| (binade-wise)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, _MIN_EXP[dt])
    return np.ldexp(1.0, (e - _MANT_BITS[dt]).astype(np.int64))


def small_problem(cache_dtype="f16", dtype=None, D=128, bs=16, H=16, Hkv=2,
                  lens=(1, 15, 16, 17, 33, 100, 255, 300), seed=0) -> Problem:
    if dtype is None:
        dtype = cache_dtype if cache_dtype in ("f32", "f16", "bf16") else "f16"
    need = sum(-(-n // bs) for n in lens)
    return make_problem("qwen3_32b_f16", seed, num_seqs=len(lens), seq_lens=list(lens),
                        num_heads=H, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                        dtype=dtype, cache_dtype=cache_dtype, num_blocks=2 * need + 3)


class GpuProblem:
    """Device copies of a problem's caches and batch tensors."""

    def __init__(self, p: Problem, batch_index: int = 0):
        dev = "cuda"
        self.p = p
        self.kc = p.k_cache.to(dev)
        self.vc = p.v_cache.to(dev)
        self.ks = p.k_scale.to(dev) if p.k_scale is not None else None
        self.vs = p.v_scale.to(dev) if p.v_scale is not None else None
        b = p.batches[batch_index]
        self.q = b.q.to(dev)
        self.tables = b.block_tables.to(dev)
        self.lens = b.seq_lens.to(dev)
        self.new_key = b.new_key.to(dev)
        self.new_value = b.new_value.to(dev)
        self.new_slots = b.new_slots.to(dev)
        self.hist_key = p.hist_key.to(dev)
        self.hist_value = p.hist_value.to(dev)
        self.hist_slots = p.hist_slots.to(dev)

    @property
    def cd(self):
        return self.p.wl.cache_dtype

    def fill(self, pa, include_new=True, err_flag=None):
        if self.hist_slots.numel():
            pa.reshape_and_cache(self.hist_key, self.hist_value, self.kc, self.vc, self.hist_slots,
                                 cache_dtype=self.cd, k_scale=self.ks, v_scale=self.vs,
                                 err_flag=err_flag)
        if include_new:
            self.write_new(pa, err_flag)
        torch.cuda.synchronize()
        return self

    def write_new(self, pa, err_flag=None):
        pa.reshape_and_cache(self.new_key, self.new_value, self.kc, self.vc, self.new_slots,
                             cache_dtype=self.cd, k_scale=self.ks, v_scale=self.vs,
                             err_flag=err_flag)

    def v1(self, pa, **kw):
        return pa.decode_v1(self.q, self.kc, self.vc, self.tables, self.lens, self.p.wl.scale,
                            cache_dtype=self.cd, k_scale=self.ks, v_scale=self.vs, **kw)

    def fused(self, pa, workspace=None, **kw):
        return pa.decode_fused(self.q, self.kc, self.vc, self.tables, self.lens, self.p.wl.scale,
                               workspace=workspace, cache_dtype=self.cd, k_scale=self.ks,
                               v_scale=self.vs, **kw)

    def v2(self, pa, partition_size=None, **kw):
        return pa.decode_v2(self.q, self.kc, self.vc, self.tables, self.lens, self.p.wl.scale,
                            partition_size=partition_size, cache_dtype=self.cd, k_scale=self.ks,
                            v_scale=self.vs, **kw)


class CpuCaches:
    """The oracle's own copies of the caches, written by the oracle's cache write."""

    def __init__(self, p: Problem, orc, batch_index: int = 0, include_new=True):
        self.p = p
        self.kc, self.vc = p.k_cache.clone(), p.v_cache.clone()
        self.ks = p.k_scale.clone() if p.k_scale is not None else None
        self.vs = p.v_scale.clone() if p.v_scale is not None else None
        cd = p.wl.cache_dtype
        if p.hist_slots.numel():
            orc.reshape_and_cache(p.hist_key, p.hist_value, self.kc, self.vc, p.hist_slots,
                                  cache_dtype=cd, k_scale=self.ks, v_scale=self.vs)
        b = p.batches[batch_index]
        self.b = b
        if include_new:
            orc.reshape_and_cache(b.new_key, b.new_value, self.kc, self.vc, b.new_slots,
                                  cache_dtype=cd, k_scale=self.ks, v_scale=self.vs)

    def decode(self, orc, q=None, tables=None, lens=None):
        b = self.b
        return orc.paged_decode(b.q if q is None else q, self.kc, self.vc,
                                b.block_tables if tables is None else tables,
                                b.seq_lens if lens is None else lens, self.p.wl.scale,
                                cache_dtype=self.p.wl.cache_dtype, k_scale=self.ks,
                                v_scale=self.vs)

    def decode_pairs(self, orc, pairs):
        b = self.b
        return orc.paged_decode_pairs(b.q, self.kc, self.vc, b.block_tables, b.seq_lens,
                                      self.p.wl.scale, pairs, cache_dtype=self.p.wl.cache_dtype,
                                      k_scale=self.ks, v_scale=self.vs)


def bytes_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.contiguous().view(torch.uint8).cpu(), b.contiguous().view(torch.uint8).cpu())


def compare(gpu_out: torch.Tensor, ref: np.ndarray, what: str = "") -> dict:
    """Assert the comparison rule; returns the error figures."""
    out = gpu_out.detach().to(torch.float64).cpu().numpy()
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite GPU output"
    dt = gpu_out.dtype
    if dt == torch.float32:
        ref_r = ref
    else:
        ref_r = torch.from_numpy(ref).to(dt).to(torch.float64).numpy()
    diff = out - ref_r
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref_r))
    rel_l2 = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    rel_l2_unrounded = (float(np.linalg.norm(out - ref) / np.linalg.norm(ref))
                        if np.linalg.norm(ref) > 0 else 0.0)
    info = dict(max_abs=max_abs, rel_l2=rel_l2, rel_l2_vs_fp64=rel_l2_unrounded)
    if dt == torch.float32:
        scale = max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
        assert rel_l2 <= TOL32 and max_abs <= TOL32 * scale, f"{what}: {info}"
    else:
        bound = np.maximum(TOL16_MAX_ABS, ulp(ref_r, dt))
        worst = float((np.abs(diff) / bound).max()) if diff.size else 0.0
        info["max_abs_over_bound"] = worst
        assert worst <= 1.0 and rel_l2 <= TOL16_REL_L2, f"{what}: {info}"
    return info


def compare_tensors(out: torch.Tensor, ref: torch.Tensor, what: str = "") -> dict:
    """The comparison rule with another GPU result (already in the output dtype) as
    the reference."""
    assert out.dtype == ref.dtype
    return compare(out, ref.detach().to(torch.float64).cpu().numpy(), what)


def sample_pairs(num_seqs, num_heads, n, seed=0):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, num_seqs, n)
    h = rng.integers(0, num_heads, n)
    return np.stack([s, h], axis=1).astype(np.int32)


def partition_sizes(bs):
    tt = max(16, bs)
    return sorted({tt, 2 * tt, 4 * tt, 128 if 128 % tt == 0 else 4 * tt, 512})


def dtype_of(name):
    return FLOAT_DTYPES[name]


def math_isclose(a, b, rel):
    return math.isclose(a, b, rel_tol=rel)
