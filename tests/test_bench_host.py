"""Host-side arithmetic of bench.py (CPU only): the algorithmic bytes and flops the
rooflines divide by, against brute-force counts."""
import numpy as np

import bench
from paged_kv_cache_390_b200 import workloads as W


def test_prefill_flops_brute_force():
    lens, qlens, H, D = [10, 7, 300], [3, 7, 129], 8, 128
    rows = sum(n - q + r + 1 for n, q in zip(lens, qlens) for r in range(q))
    assert bench.prefill_flops(lens, qlens, H, D) == 4 * D * H * rows


def test_step_bytes_count_exact_tokens():
    p = W.make_problem("qwen3_32b_f16", 0)
    wl, b = p.wl, p.batch
    decode, step, unique = bench.step_bytes(wl, b)
    kv = int(b.seq_lens.sum()) * wl.num_kv_heads * wl.head_dim * 2 * 2
    qo = 2 * wl.num_seqs * wl.num_heads * wl.head_dim * 2
    assert decode == kv + qo and unique == decode
    rows = wl.num_seqs * wl.num_kv_heads * wl.head_dim * 2
    assert step == decode + 2 * 2 * rows          # new K and V rows read and written


def test_unique_bytes_count_the_shared_prefix_once():
    p = W.make_problem("mixed_f16", 0, num_seqs=4, seq_lens=[8192 + n for n in (5, 40, 1, 300)])
    wl, b = p.wl, p.batch
    _, _, unique = bench.step_bytes(wl, b)
    per_tok = wl.num_kv_heads * wl.head_dim * 2 * 2
    private = int((b.seq_lens - 8192).sum())
    qo = 2 * wl.num_seqs * wl.num_heads * wl.head_dim * 2
    assert unique == (8192 + private) * per_tok + qo


def test_block_size_override_keeps_the_pool_and_the_tokens():
    class A:
        block_size = 8
    base = W.WORKLOADS["qwen3_32b_f16"]
    over = bench.workload_overrides(A, base)
    assert over == {"block_size": 8, "num_blocks": base.num_blocks * 2}
    A.block_size = 0
    assert bench.workload_overrides(A, base) == {}
    A.block_size = base.block_size
    assert bench.workload_overrides(A, base) == {}
    # --num-seqs scales the pool with the batch (and leaves an auto-sized pool alone)
    A.num_seqs = 64
    assert bench.workload_overrides(A, base) == {"num_seqs": 64, "num_blocks": base.num_blocks * 2}
    assert bench.workload_overrides(A, W.WORKLOADS["mixed_f16"]) == {"num_seqs": 64}
    # the mixed batch at block 8 and 32: the same lengths, the same shared prefix
    ref = W.make_problem("mixed_f16", 0, num_seqs=4)
    for bs in (8, 32):
        p = W.make_problem("mixed_f16", 0, num_seqs=4, block_size=bs)
        assert p.wl.block_size == bs
        assert np.array_equal(p.batch.seq_lens.numpy(), ref.batch.seq_lens.numpy())
        n_pref = p.wl.shared_prefix_tokens // bs
        t = p.batch.block_tables.numpy()
        assert (t[:, :n_pref] == t[0, :n_pref]).all()


def test_all_cores_oracle_baseline_counts_every_thread():
    p = W.make_problem("tiny_f32", 0)
    caches = bench.oracle_caches(p, p.wl)
    one = bench.cpu_baseline(p, p.wl, budget_s=0.3, caches=caches)
    many = bench.cpu_baseline_all_cores(p, p.wl, budget_s=0.3, threads=2, caches=caches)
    assert one["cores"] == 1 and many["cores"] == 2
    assert one["value"] > 0 and many["value"] > 0 and many["kind"] == "oracle"
