"""The library's C++ block manager against the oracle's model, operation for operation:
identical block ids, slots, cached-prefix lengths, copy-on-write pairs, swap mappings
and free counts; failed calls change nothing on either side.  CPU only."""
import random

import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, NoSpace


@pytest.fixture(scope="module")
def bm_cls():
    from paged_kv_cache_390_b200 import build
    build.build()
    from paged_kv_cache_390_b200.block_manager import BlockManager
    return BlockManager


def _same_state(cpp, model):
    assert cpp.free_gpu_blocks == model.free_gpu_blocks()
    assert cpp.free_cpu_blocks == model.free_cpu_blocks()
    for sid in model.seqs:
        blocks, n = cpp.block_table(sid)
        mb, mn = model.block_table(sid)
        assert blocks.tolist() == mb and n == mn


def _both(cpp_call, model_call):
    """Run both; they must both succeed with equal results or both refuse alike."""
    from paged_kv_cache_390_b200 import pa
    try:
        want = model_call()
        err = None
    except NoSpace:
        err = pa.PA_ERR_NO_SPACE
    except ValueError:
        err = pa.PA_ERR_INVALID_ARG
    if err is None:
        return cpp_call(), want
    with pytest.raises(pa.PAError) as e:
        cpp_call()
    assert e.value.status == err
    return None, None


@pytest.mark.parametrize("prefix,bs,seed", [(False, 16, 0), (True, 16, 1), (True, 4, 2),
                                            (False, 8, 3), (True, 2, 4)])
def test_random_operations_match_the_model(bm_cls, prefix, bs, seed):
    rng = random.Random(seed)
    G, C = 96, 48
    cpp = bm_cls(G, bs, C, prefix)
    model = BlockManagerModel(G, C, bs, prefix)
    nxt = 0
    vocab = 1000
    # prompts start with one of a few shared system prompts, so prefixes repeat
    templates = [[rng.randrange(vocab) for _ in range(4 * bs)] for _ in range(3)]
    for step in range(2500):
        op = rng.random()
        ids = list(model.seqs)
        live = [i for i in ids if model.seqs[i]["on_gpu"]]
        out = [i for i in ids if not model.seqs[i]["on_gpu"]]
        if op < 0.2 or not ids:
            toks = rng.choice(templates)[:rng.randrange(0, 4 * bs + 1)] + [
                rng.randrange(vocab) for _ in range(rng.randrange(1, 2 * bs))]
            got, want = _both(lambda: cpp.add_sequence(nxt, toks),
                              lambda: model.add_sequence(nxt, toks))
            if want is not None:
                assert got[0].tolist() == want[0] and got[1] == want[1]
            nxt += 1
        elif op < 0.45 and live:
            sid, tok = rng.choice(live), rng.randrange(vocab)
            got, want = _both(lambda: cpp.append_token(sid, tok),
                              lambda: model.append_token(sid, tok))
            assert got == want
        elif op < 0.6 and live:
            group = rng.sample(live, min(len(live), rng.randrange(1, 5)))
            toks = [rng.randrange(vocab) for _ in group]
            got, want = _both(lambda: cpp.append_batch(group, toks),
                              lambda: model.append_batch(group, toks))
            if want is not None:
                assert got[0].tolist() == want[0]
                assert [tuple(p) for p in got[1].tolist()] == want[1]
        elif op < 0.68 and live:
            sid = rng.choice(live)
            got, want = _both(lambda: cpp.fork(sid, nxt), lambda: model.fork(sid, nxt))
            nxt += 1
        elif op < 0.76 and live:
            group = rng.sample(live, min(len(live), rng.randrange(1, 4)))
            got, want = _both(lambda: cpp.swap_out(group), lambda: model.swap_out(group))
            if want is not None:
                assert [tuple(p) for p in got.tolist()] == want
        elif op < 0.84 and out:
            group = rng.sample(out, min(len(out), rng.randrange(1, 4)))
            got, want = _both(lambda: cpp.swap_in(group), lambda: model.swap_in(group))
            if want is not None:
                assert [tuple(p) for p in got.tolist()] == want
        elif op < 0.81:
            bogus = nxt + 1000                         # unknown sequence: refused alike
            _both(lambda: cpp.append_token(bogus, 1), lambda: model.append_token(bogus, 1))
        else:
            sid = rng.choice(ids)
            _both(lambda: cpp.free_sequence(sid), lambda: model.free_sequence(sid))
        if step % 25 == 0:
            _same_state(cpp, model)
    _same_state(cpp, model)
    cpp.close()


def test_build_batch_pads_with_minus_one(bm_cls):
    with bm_cls(32, 16) as bm:
        bm.add_sequence(7, list(range(40)))
        bm.add_sequence(9, list(range(5)))
        tables, lens = bm.build_batch([9, 7])
        assert tables.shape == (2, 3) and lens.tolist() == [5, 40]
        assert tables[0].tolist() == [bm.block_table(9)[0][0], -1, -1]
        assert tables[1].tolist() == bm.block_table(7)[0].tolist()


def test_bad_handles_and_arguments(bm_cls):
    from paged_kv_cache_390_b200 import pa
    L = pa.lib()
    assert not L.pa_bm_create(0, 0, 16, 0)
    assert not L.pa_bm_create(4, -1, 16, 0)
    assert L.pa_bm_free_gpu_blocks(None) == -1
    with bm_cls(4, 16) as bm:
        with pytest.raises(pa.PAError):
            bm.add_sequence(1, [])
        bm.add_sequence(1, [1, 2])
        with pytest.raises(pa.PAError):
            bm.add_sequence(1, [3])                    # duplicate id
        with pytest.raises(pa.PAError):
            bm.fork(1, 1)
        with pytest.raises(pa.PAError) as e:
            bm.add_sequence(2, [0] * 100)              # 7 blocks > 3 free
        assert e.value.status == pa.PA_ERR_NO_SPACE
        assert bm.free_gpu_blocks == 3                 # nothing changed


@pytest.mark.parametrize("bs", [4, 16])
def test_blocks_filled_by_appends_are_found_by_a_later_prompt(bm_cls, bs):
    """The keys of blocks that appends fill (also after a fork) chain like the keys of
    prompt blocks: a later prompt that repeats the whole history hits every full block."""
    rng = random.Random(bs)
    cpp = bm_cls(64, bs, 0, True)
    model = BlockManagerModel(64, 0, bs, True)
    prompt = [rng.randrange(1000) for _ in range(2 * bs + 3)]
    for m in (cpp, model):
        m.add_sequence(0, prompt)
    hist = list(prompt)
    for _ in range(3 * bs):                       # fills three more blocks
        t = rng.randrange(1000)
        assert cpp.append_token(0, t) == model.append_token(0, t)
        hist.append(t)
    cpp.fork(0, 1)
    model.fork(0, 1)
    for _ in range(bs):                           # the child fills one block of its own
        t = rng.randrange(1000)
        assert cpp.append_token(1, t) == model.append_token(1, t)
        hist.append(t)
    probe = hist + [7]
    got = cpp.add_sequence(2, probe)
    want = model.add_sequence(2, probe)
    assert got[1] == want[1] == (len(probe) - 1) // bs * bs   # every full block is a hit
    assert got[0].tolist() == want[0]
    _same_state(cpp, model)
