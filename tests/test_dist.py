"""Host-side multi-process logic of bench.py, world size 2 on gloo (CPU only): each rank
decodes its own batch (replicas, no data exchange); the timed result is the max over
ranks and the whole-job rate counts every rank's bytes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from paged_kv_cache_390_b200.workloads import make_problem
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        seed = bench.rank_seed(r)
        p = make_problem("tiny_f32", seed)
        elapsed = 10.0 + 5.0 * rank                      # per-rank "times"
        mx = bench.max_over_ranks(elapsed, torch.device("cpu"))
        dist.barrier()
        q.put((rank, r, w, lr, seed, p.batch.q.sum().item(), mx))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_replicas_take_distinct_batches_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for pr in procs:
        pr.join(timeout=30)
        assert pr.exitcode == 0
    (r0, rr0, w0, l0, s0, q0, m0), (r1, rr1, w1, l1, s1, q1, m1) = res
    assert (rr0, rr1) == (0, 1) and w0 == w1 == 2 and (l0, l1) == (0, 1)
    assert s0 != s1 and q0 != q1                         # independent inputs per rank
    assert m0 == m1 == 15.0                              # slowest rank decides


def test_whole_job_rate_counts_every_rank():
    import bench
    assert bench.whole_job_rate(100.0, 4, 2.0) == 200.0
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5   # no process group


@pytest.mark.timeout(240)
def test_bench_gpus_2_starts_two_ranks_itself():
    """`bench.py --gpus 2` with no launcher around it runs two ranks (torch.distributed.run
    on 127.0.0.1) and rank 0 alone prints one line with n_gpus 2.  The oracle arm is the
    one that runs on a CPU-only host."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "2", "--warmup", "0", "--workload", "tiny_f32",
                        "--reference-seconds", "2"],
                       capture_output=True, text=True, timeout=220, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2 and res["value"] > 0
