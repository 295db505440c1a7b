"""pa_decode_fused_noalloc: the single-launch decode for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).  Called through the C
ABI on two calls in a row: each output is bit-identical to pa_decode_fused's (the same
kernel, grid and merge order) and matches the oracle under the comparison rule.  Kept
in its own file, collected last, so a run that stops at the first failure has run
everything else."""
import ctypes

import pytest
import torch

from _helpers import (CpuCaches, GpuProblem, bytes_equal, compare, compare_tensors,
                      sample_pairs, small_problem)
from paged_kv_cache_390_b200.workloads import make_problem

pytestmark = pytest.mark.gpu


def _call_noalloc(pa, g, out, err_flag=None):
    lib = pa.lib()
    kc = g.kc
    num_blocks, block_size, num_kv_heads, head_dim = kc.shape
    num_seqs, num_heads, _ = g.q.shape
    P = ctypes.c_void_p
    ptr = lambda t: None if t is None else P(t.data_ptr())
    return lib.pa_decode_fused_noalloc(
        ptr(out), ptr(g.q), pa._FLOAT_CODES[g.q.dtype], ptr(kc), ptr(g.vc),
        pa.cache_code(kc, g.cd), ptr(g.ks), ptr(g.vs), ptr(g.tables), g.tables.shape[1],
        ptr(g.lens), num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
        float(g.p.wl.scale), ptr(err_flag), P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,kw", [
    ("qwen3_32b_f16", dict(num_seqs=12)),
    ("quant_int8", dict(num_seqs=6)),
])
def test_noalloc_matches_fused_on_two_calls(pa, orc, name, kw):
    p = make_problem(name, 7, **kw)
    g = GpuProblem(p).fill(pa)
    ref = g.fused(pa)                              # the existing entry point, own workspace
    torch.cuda.synchronize()
    pairs = sample_pairs(p.wl.num_seqs, p.wl.num_heads, 24, seed=4)
    want = CpuCaches(p, orc).decode_pairs(orc, pairs)
    for _ in range(2):
        out = torch.full_like(g.q, float("nan"))
        assert _call_noalloc(pa, g, out) == pa.PA_OK
        torch.cuda.synchronize()
        compare_tensors(out, ref, f"no-alloc vs fused, {name}")
        assert bytes_equal(out, ref), f"no-alloc differs from fused, {name}"
        compare(torch.stack([out[s, h] for s, h in pairs.tolist()]), want,
                f"no-alloc vs oracle, {name}")


def test_noalloc_small_ragged_batch(pa, orc):
    p = small_problem(cache_dtype="bf16", seed=3)
    g = GpuProblem(p).fill(pa)
    ref = g.fused(pa)
    want = CpuCaches(p, orc).decode(orc)
    out = torch.empty_like(g.q)
    for _ in range(2):
        assert _call_noalloc(pa, g, out) == pa.PA_OK
        torch.cuda.synchronize()
        compare_tensors(out, ref, "no-alloc vs fused, ragged bf16")
        assert bytes_equal(out, ref), "no-alloc differs from fused, ragged bf16"
        compare(out, want, "no-alloc vs oracle, ragged bf16")


def test_noalloc_rejected_call_leaves_the_scratch_alone(pa):
    """A call its host checks reject (here: head_dim 96) returns before any GPU work,
    so the array keeps what the last good call left; the next good call is still
    bit-identical to pa_decode_fused."""
    p = small_problem(cache_dtype="f16", seed=9)
    g = GpuProblem(p).fill(pa)
    ref = g.fused(pa)
    out = torch.empty_like(g.q)
    assert _call_noalloc(pa, g, out) == pa.PA_OK
    lib = pa.lib()
    P = ctypes.c_void_p
    rc = lib.pa_decode_fused_noalloc(P(out.data_ptr()), P(g.q.data_ptr()), pa.PA_F16,
                                     P(g.kc.data_ptr()), P(g.vc.data_ptr()), pa.PA_F16, None, None,
                                     P(g.tables.data_ptr()), g.tables.shape[1],
                                     P(g.lens.data_ptr()), g.q.shape[0], g.q.shape[1], 2, 96, 16,
                                     g.kc.shape[0], 0.1, None, None)
    assert rc == pa.PA_ERR_UNSUPPORTED
    out2 = torch.full_like(g.q, float("nan"))
    assert _call_noalloc(pa, g, out2) == pa.PA_OK
    torch.cuda.synchronize()
    assert bytes_equal(out2, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch(pa):
    lib = pa.lib()
    limit = lib.pa_decode_fused_noalloc_scratch_bytes()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert lib.pa_decode_fused_workspace_bytes(8192, 256, 128, sms) > limit
    fake = ctypes.c_void_p(1 << 20)                # never dereferenced: rejected on the host
    rc = lib.pa_decode_fused_noalloc(fake, fake, pa.PA_F16, fake, fake, pa.PA_F16, None, None,
                                     fake, 4, fake, 8192, 2048, 256, 128, 16, 100, 0.1, None,
                                     None)
    assert rc == pa.PA_ERR_UNSUPPORTED
