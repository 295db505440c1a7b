"""Debug bounds flag and bounded waits: bad inputs are reported through err_flag,
the access is skipped, nothing traps; a run-out wait reports a time-out and the
context stays usable."""
import pytest
import torch

from _helpers import CpuCaches, GpuProblem, bytes_equal, compare, small_problem

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


@pytest.mark.parametrize("cd", ["f16", "int8"])
def test_slot_past_pool_without_flag_writes_nothing(pa, cd):
    """No err_flag: a slot at or past the pool end is still skipped.  The pool is a
    view of a larger buffer whose extra blocks hold a sentinel that must survive."""
    p = small_problem(cache_dtype=cd, seed=55)
    g = GpuProblem(p)
    nb, extra = g.kc.shape[0], 2
    for name in ("kc", "vc"):
        big = torch.empty((nb + extra,) + tuple(g.kc.shape[1:]), dtype=g.kc.dtype, device="cuda")
        big.view(torch.uint8).fill_(0x5A)
        big[:nb].copy_(getattr(g, name))
        setattr(g, name + "_big", big)
        setattr(g, name, big[:nb])
    sentinel_k, sentinel_v = g.kc_big[nb:].clone(), g.vc_big[nb:].clone()
    bs = g.kc.shape[1]
    g.new_slots[1] = nb * bs                          # first slot past the pool
    g.new_slots[4] = (nb + 1) * bs + 3
    g.fill(pa)                                        # no err_flag
    assert bytes_equal(g.kc_big[nb:], sentinel_k) and bytes_equal(g.vc_big[nb:], sentinel_v)
    pa.get_device_error(clear=True)


@pytest.mark.parametrize("cd", ["f16", "int8"])
def test_append_slot_off_the_table_is_flagged_and_not_written(pa, cd):
    """With err_flag, the fused write checks that the slot is the table's slot for
    the sequence's last token; another slot is flagged and left unwritten."""
    p = small_problem(cache_dtype=cd, seed=57)
    g = GpuProblem(p).fill(pa, include_new=False)
    bs = g.kc.shape[1]
    s = 5                                             # a sequence of 100 tokens
    assert int(g.lens[s]) == 100
    earlier = int(g.tables[s, 0]) * bs + 3            # token 3's slot: inside the pool
    good = int(g.new_slots[s])
    g.new_slots[s] = earlier
    before_k, before_v = g.kc.clone(), g.vc.clone()
    f = _flag()
    pa.append_decode_v1(g.q, g.new_key, g.new_value, g.new_slots, g.kc, g.vc, g.tables, g.lens,
                        p.wl.scale, cache_dtype=g.cd, k_scale=g.ks, v_scale=g.vs, err_flag=f)
    torch.cuda.synchronize()
    assert int(f.item()) & pa.DEVERR_SLOT
    blk, off = divmod(earlier, bs)
    gb, go = divmod(good, bs)
    assert bytes_equal(g.kc[blk, off], before_k[blk, off])
    assert bytes_equal(g.vc[blk, off], before_v[blk, off])
    assert bytes_equal(g.kc[gb, go], before_k[gb, go])
    # every other sequence's row was written
    other = int(g.new_slots[0])
    ob, oo = divmod(other, bs)
    assert not bytes_equal(g.kc[ob, oo], before_k[ob, oo])
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
