"""Debug bounds flag and bounded waits: bad inputs are reported through err_flag,
the access is skipped, nothing traps; a run-out wait reports a time-out and the
context stays usable."""
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, compare, small_problem

pytestmark = pytest.mark.gpu


def _flag():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("cd", ["f16", "int8", "f32"])
def test_valid_inputs_raise_no_flag(pa, orc, cd):
    p = small_problem(cache_dtype=cd, seed=41)
    f = _flag()
    g = GpuProblem(p).fill(pa, err_flag=f)
    ref = CpuCaches(p, orc).decode(orc)
    compare(g.v1(pa, err_flag=f), ref, "checked v1")
    compare(g.v2(pa, partition_size=32, err_flag=f), ref, "checked v2")
    assert int(f.item()) == 0


@pytest.mark.parametrize("cd", ["f16", "fp8", "f32"])
def test_bad_block_id_is_flagged_and_skipped(pa, cd):
    p = small_problem(cache_dtype=cd, seed=43)
    g = GpuProblem(p).fill(pa)
    g.tables[3, 1] = g.kc.shape[0] + 5            # past the pool
    g.tables[5, 0] = -7
    for run in (lambda f: g.v1(pa, err_flag=f), lambda f: g.v2(pa, partition_size=32, err_flag=f)):
        f = _flag()
        out = run(f)
        torch.cuda.synchronize()
        assert int(f.item()) & pa.DEVERR_BLOCK_ID
        assert torch.isfinite(out).all()
    pa.get_device_error(clear=True)


def test_seq_len_past_table_is_flagged(pa):
    p = small_problem(cache_dtype="bf16", seed=47)
    g = GpuProblem(p).fill(pa)
    g.lens[0] = g.tables.shape[1] * 16 + 100
    g.lens[1] = -3
    for run in (lambda f: g.v1(pa, err_flag=f), lambda f: g.v2(pa, partition_size=32, err_flag=f)):
        f = _flag()
        out = run(f)
        torch.cuda.synchronize()
        assert int(f.item()) & pa.DEVERR_SEQ_LEN
        assert torch.isfinite(out).all()
        assert not out[0].any() and not out[1].any()     # the bad sequences are skipped
    pa.get_device_error(clear=True)


def test_slot_past_pool_is_flagged(pa):
    p = small_problem(cache_dtype="int8", seed=53)
    g = GpuProblem(p)
    g.new_slots[2] = g.kc.shape[0] * g.kc.shape[1] + 3
    f = _flag()
    g.fill(pa, err_flag=f)
    assert int(f.item()) & pa.DEVERR_SLOT
    pa.get_device_error(clear=True)


def test_wait_time_out_reports_and_context_survives(pa, orc):
    p = small_problem(cache_dtype="f16", lens=(2000, 1800, 1900, 2100), seed=59)
    g = GpuProblem(p).fill(pa)
    pa.get_device_error(clear=True)
    outs = []
    try:
        # every warp's first stage is never armed: its wait can only run out (1 ms)
        pa.set_wait_limit_ns(1_000_000)
        pa.set_fault_injection(1)
        for run in (lambda f: g.v1(pa, err_flag=f), lambda f: g.v2(pa, partition_size=256,
                                                                    err_flag=f)):
            f = _flag()
            outs.append((f, run(f)))
        torch.cuda.synchronize()
    finally:
        pa.set_fault_injection(0)
        pa.set_wait_limit_ns(0)
    for f, out in outs:
        assert int(f.item()) & pa.DEVERR_TIMEOUT
        assert torch.isfinite(out).all()
    assert pa.get_device_error(clear=True) & pa.DEVERR_TIMEOUT
    # the context is intact: a normal run matches the oracle
    ref = CpuCaches(p, orc).decode(orc)
    compare(g.v1(pa), ref, "after time-out")
    assert pa.get_device_error(clear=True) == 0
