"""The host block manager driving the kernels: a seeded run of add / decode-step /
fork / swap / free operations.  The C++ manager's block tables, slots, copy-on-write
pairs and swap mappings feed pa_reshape_and_cache, pa_copy_blocks and
pa_append_decode_v1 on the GPU; the oracle's block-manager model feeds the oracle's
cache write, block copy and decode on the CPU.  After every operation the two pools
are bit-identical, and every decode step's output matches the oracle.

Pages: the BlockManager of "大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置"
(allocate on a full last block, append_token) and "KVcache-learning" s05 / s06
(copy-on-write of a shared block, swap to host memory, free-list reuse)."""
import numpy as np
import pytest
import torch

from _helpers import compare

pytestmark = pytest.mark.gpu

H, HKV, D, BS = 16, 2, 128, 16
NUM_GPU, NUM_CPU = 56, 24
SCALE = 1.0 / np.sqrt(D)
MASK = (1 << 64) - 1


def _row_seed(h_prev, token):
    """Rolling 64-bit hash of a token prefix: the K/V rows of position t are a seeded
    function of tokens[0..t], so equal prefixes have equal rows (what makes a cached
    block reusable)."""
    return ((h_prev ^ (token & 0xFFFFFFFF)) * 0x100000001B3) & MASK


def _rows(seeds):
    out = np.empty((len(seeds), 2, HKV, D), dtype=np.float32)
    for i, s in enumerate(seeds):
        out[i] = np.random.default_rng(s).standard_normal((2, HKV, D))
    t = torch.from_numpy(out).half()
    return t[:, 0].contiguous(), t[:, 1].contiguous()


class Side:
    """One side's pools: GPU caches + pinned host pool (product), or CPU tensors (oracle)."""

    def __init__(self, cd, device):
        quant = cd in ("int8", "fp8")
        store = {"f16": torch.float16, "int8": torch.int8, "fp8": torch.uint8}[cd]
        pin = device == "cuda"

        def pool(n, host):
            t = torch.zeros((n, BS, HKV, D), dtype=store)
            if host and pin:
                return t.pin_memory()
            return t.to(device) if not host else t

        def scales(n, host):
            if not quant:
                return None
            t = torch.zeros((n, HKV, BS))
            if host and pin:
                return t.pin_memory()
            return t.to(device) if not host else t

        self.kc, self.vc = pool(NUM_GPU, False), pool(NUM_GPU, False)
        self.ks, self.vs = scales(NUM_GPU, False), scales(NUM_GPU, False)
        self.hk, self.hv = pool(NUM_CPU, True), pool(NUM_CPU, True)
        self.hks, self.hvs = scales(NUM_CPU, True), scales(NUM_CPU, True)


def _same_pools(g, c):
    for a, b in ((g.kc, c.kc), (g.vc, c.vc), (g.hk, c.hk), (g.hv, c.hv), (g.ks, c.ks),
                 (g.vs, c.vs), (g.hks, c.hks), (g.hvs, c.hvs)):
        if a is None:
            continue
        if not torch.equal(a.cpu().contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)):
            return False
    return True


@pytest.mark.parametrize("cd", ["f16", "int8", "fp8"])
def test_block_manager_drives_the_kernels(pa, orc, cd):
    from oracle.block_manager import BlockManagerModel, NoSpace
    from paged_kv_cache_390_b200.block_manager import BlockManager

    rng = np.random.default_rng({"f16": 1, "int8": 2, "fp8": 3}[cd])
    bm = BlockManager(NUM_GPU, BS, NUM_CPU, prefix_caching=True)
    model = BlockManagerModel(NUM_GPU, NUM_CPU, BS, True)
    g, c = Side(cd, "cuda"), Side(cd, "cpu")
    qd = dict(cache_dtype=cd)
    seqs = {}                        # id -> (tokens, prefix hashes) while alive
    on_gpu = {}
    next_id = [0]
    stats = dict(decodes=0, cow=0, swaps=0, forks=0, hits=0, frees=0)

    def both(fn_prod, fn_model):
        """Run one manager call on both; both succeed or both run out of space."""
        try:
            a = fn_prod()
        except pa.PAError as e:
            assert e.status == pa.PA_ERR_NO_SPACE, e
            with pytest.raises(NoSpace):
                fn_model()
            return None, None
        return a, fn_model()

    def new_sequence(prompt):
        sid = next_id[0]
        a, m = both(lambda: bm.add_sequence(sid, prompt), lambda: model.add_sequence(sid, prompt))
        if a is None:
            return
        next_id[0] += 1
        (slots, cached), (mslots, mcached) = a, m
        assert cached == mcached and list(slots) == list(mslots)
        stats["hits"] += cached > 0
        hs, h = [], 0xCBF29CE484222325
        for t in prompt:
            h = _row_seed(h, t)
            hs.append(h)
        seqs[sid] = (list(prompt), hs)
        on_gpu[sid] = True
        # rows of the tokens not served from the cache
        k, v = _rows(hs[cached:])
        sl = torch.from_numpy(np.asarray(slots[cached:], dtype=np.int64))
        pa.reshape_and_cache(k.cuda(), v.cuda(), g.kc, g.vc, sl.cuda(), k_scale=g.ks,
                             v_scale=g.vs, **qd)
        orc.reshape_and_cache(k, v, c.kc, c.vc, sl, k_scale=c.ks, v_scale=c.vs, **qd)

    def decode_step():
        ids = [i for i in seqs if on_gpu[i]]
        if not ids:
            return
        toks = [int(x) for x in rng.integers(0, 50, len(ids))]
        a, m = both(lambda: bm.append_batch(ids, toks), lambda: model.append_batch(ids, toks))
        if a is None:
            return
        (slots, pairs), (mslots, mpairs) = a, m
        assert list(slots) == list(mslots)
        assert [tuple(p) for p in pairs.tolist()] == [tuple(p) for p in mpairs]
        if len(pairs):
            stats["cow"] += len(pairs)
            pt = torch.from_numpy(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
            pa.copy_blocks(g.kc, g.vc, g.kc, g.vc, pt.cuda(), src_k_scale=g.ks,
                           src_v_scale=g.vs, dst_k_scale=g.ks, dst_v_scale=g.vs, **qd)
            orc.copy_blocks(c.kc, c.vc, c.kc, c.vc, pt, src_k_scale=c.ks, src_v_scale=c.vs,
                            dst_k_scale=c.ks, dst_v_scale=c.vs, **qd)
        seeds = []
        for i, t in zip(ids, toks):
            tokens, hs = seqs[i]
            tokens.append(t)
            hs.append(_row_seed(hs[-1], t))
            seeds.append(hs[-1])
        nk, nv = _rows(seeds)
        q = torch.randn((len(ids), H, D), generator=torch.Generator().manual_seed(
            int(rng.integers(1 << 30)))).half()
        tables, lens = bm.build_batch(ids)
        mt = [model.block_table(i) for i in ids]
        width = tables.shape[1]
        mtab = np.full((len(ids), width), -1, dtype=np.int32)
        for r, (blocks, n) in enumerate(mt):
            mtab[r, :len(blocks)] = blocks
            assert n == lens[r]
        assert np.array_equal(tables, mtab)
        sl = torch.from_numpy(np.asarray(slots, dtype=np.int64))
        out = pa.append_decode_v1(q.cuda(), nk.cuda(), nv.cuda(), sl.cuda(), g.kc, g.vc,
                                  torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                                  SCALE, k_scale=g.ks, v_scale=g.vs, **qd)
        orc.reshape_and_cache(nk, nv, c.kc, c.vc, sl, k_scale=c.ks, v_scale=c.vs, **qd)
        ref = orc.paged_decode(q, c.kc, c.vc, torch.from_numpy(mtab), torch.from_numpy(lens),
                               SCALE, k_scale=c.ks, v_scale=c.vs, **qd)
        torch.cuda.synchronize()
        compare(out, ref, f"{cd} decode step {stats['decodes']}")
        stats["decodes"] += 1

    def fork():
        ids = [i for i in seqs if on_gpu[i]]
        if not ids:
            return
        parent = int(rng.choice(ids))
        child = next_id[0]
        next_id[0] += 1
        bm.fork(parent, child)
        model.fork(parent, child)
        tokens, hs = seqs[parent]
        seqs[child] = (list(tokens), list(hs))
        on_gpu[child] = True
        stats["forks"] += 1

    def swap(to_cpu):
        ids = [i for i in seqs if on_gpu[i] == to_cpu]
        if not ids:
            return
        sid = int(rng.choice(ids))
        if to_cpu:
            a, m = both(lambda: bm.swap_out([sid]), lambda: model.swap_out([sid]))
        else:
            a, m = both(lambda: bm.swap_in([sid]), lambda: model.swap_in([sid]))
        if a is None:
            return
        assert [tuple(p) for p in a.tolist()] == [tuple(p) for p in m]
        pt = torch.from_numpy(np.asarray(a, dtype=np.int64).reshape(-1, 2))
        if to_cpu:
            src_g, dst_g = (g.kc, g.vc, g.ks, g.vs), (g.hk, g.hv, g.hks, g.hvs)
            src_c, dst_c = (c.kc, c.vc, c.ks, c.vs), (c.hk, c.hv, c.hks, c.hvs)
        else:
            src_g, dst_g = (g.hk, g.hv, g.hks, g.hvs), (g.kc, g.vc, g.ks, g.vs)
            src_c, dst_c = (c.hk, c.hv, c.hks, c.hvs), (c.kc, c.vc, c.ks, c.vs)
        pa.copy_blocks(src_g[0], src_g[1], dst_g[0], dst_g[1], pt.cuda(), src_k_scale=src_g[2],
                       src_v_scale=src_g[3], dst_k_scale=dst_g[2], dst_v_scale=dst_g[3], **qd)
        orc.copy_blocks(src_c[0], src_c[1], dst_c[0], dst_c[1], pt, src_k_scale=src_c[2],
                        src_v_scale=src_c[3], dst_k_scale=dst_c[2], dst_v_scale=dst_c[3], **qd)
        on_gpu[sid] = not to_cpu
        stats["swaps"] += 1

    def free():
        if len(seqs) <= 1:
            return
        sid = int(rng.choice(list(seqs)))
        bm.free_sequence(sid)
        model.free_sequence(sid)
        del seqs[sid], on_gpu[sid]
        stats["frees"] += 1

    # a shared system prompt: later prompts repeat it, so their full blocks are hits
    system = [int(x) for x in rng.integers(0, 50, 40)]
    new_sequence(system + [1, 2, 3])
    new_sequence(system + [7])
    new_sequence([int(x) for x in rng.integers(0, 50, 23)])
    for step in range(60):
        r = rng.random()
        if r < 0.55:
            decode_step()
        elif r < 0.65:
            fork()
        elif r < 0.75:
            swap(True)
        elif r < 0.85:
            swap(False)
        elif r < 0.93:
            new_sequence(system + [int(x) for x in rng.integers(0, 50, int(rng.integers(1, 20)))])
        else:
            free()
        torch.cuda.synchronize()
        assert _same_pools(g, c), f"{cd}: pools differ after operation {step}"
    assert pa.get_device_error() == 0
    # the run exercised what it is about
    assert stats["decodes"] >= 20 and stats["cow"] > 0 and stats["swaps"] > 0, stats
    assert stats["forks"] > 0 and stats["hits"] > 0, stats
