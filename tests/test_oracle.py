"""Pins for the oracle: each test checks it against something other than itself --
values the pages print, closed forms, invariants, special cases that reduce to a
library routine, or brute force on tiny inputs.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from paged_kv_cache_390_b200.workloads import make_problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# KV-size arithmetic: the pages' worked numbers.
# --------------------------------------------------------------------------

def test_kv_bytes_per_token_matches_pages(orc):
    g = _golden("kv_size.json")
    for c in g["cases"]:
        got = orc.kv_bytes_per_token(c["num_layers"], c["num_kv_heads"], c["head_dim"],
                                     c["dtype_bytes"])
        assert got == c["bytes_per_token"], c["source"]
    cc = g["concurrency"]
    assert cc["num_gpu_blocks"] * cc["block_size"] / cc["tokens_per_request"] == cc["printed"]


def test_kv_total_formula_closed_form(orc):
    # KVcache-learning s11: 2 x L x H_kv x D x S x B x bytes with L=80, H_kv=8, D=128,
    # S=8192, B=16, FP16.  The page prints 4,294,967,296 and calls it one layer; the
    # product of the factors it lists is ten times that and already covers 80 layers.
    per_tok = orc.kv_bytes_per_token(80, 8, 128, 2)
    assert per_tok * 8192 * 16 == 42_949_672_960
    assert per_tok * 8192 * 16 != 4_294_967_296


# --------------------------------------------------------------------------
# Storage formats.
# --------------------------------------------------------------------------

def test_f16_decode_all_codes_match_numpy(orc):
    codes = np.arange(65536, dtype=np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_double(int(c)) for c in codes[::7]])
    r = ref[::7]
    nan = np.isnan(r)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], r[~nan])


def test_bf16_decode_matches_torch(orc):
    codes = torch.arange(0, 65536, 13, dtype=torch.int32).to(torch.int16)
    ref = codes.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.bf16_to_double(int(c) & 0xFFFF) for c in codes.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_points_from_the_format_definition(orc):
    g = _golden("e4m3_points.json")
    for row in g["decode"]:
        v = orc.e4m3_to_double(row["code"])
        assert v == row["value"] and math.copysign(1, v) == math.copysign(1, row["value"])
    for row in g["encode_rne"]:
        assert orc.e4m3_from_float(row["x"]) == row["code"], row["why"]
    assert math.isnan(orc.e4m3_to_double(0x7F)) and math.isnan(orc.e4m3_to_double(0xFF))
    assert orc.e4m3_from_float(float("nan")) & 0x7F == 0x7F
    assert orc.e4m3_from_float(float("inf")) == 0x7E
    assert orc.e4m3_from_float(float("-inf")) == 0xFE


def test_e4m3_decode_encode_identity_all_codes(orc):
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert orc.e4m3_from_float(orc.e4m3_to_double(c)) == c, hex(c)


def test_e4m3_decode_matches_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_to_double(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_rne_in_range(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * 50,
        rng.standard_normal(1000).astype(np.float32) * 0.01,
        (rng.integers(-3584, 3585, 1000) / 8.0).astype(np.float32),   # many exact ties
        np.float32(2.0) ** rng.integers(-12, 9, 500).astype(np.float32) * np.float32(1.0625),
    ])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_from_float(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------
# Quantisation of one (token, head) row.
# --------------------------------------------------------------------------

def test_int8_row_against_numpy(orc):
    rng = np.random.default_rng(2)
    for _ in range(200):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 10)).astype(np.float32)
        codes, s = orc.quant_int8_row(x)
        s_ref = np.float32(np.abs(x).max()) / np.float32(127.0)
        assert np.float32(s) == s_ref
        ref = np.clip(np.rint(x / s_ref), -127, 127).astype(np.int8)   # np.rint: ties to even
        assert np.array_equal(codes, ref)
        # round trip: |x - c s| <= s / 2
        assert np.all(np.abs(x.astype(np.float64) - codes * np.float64(s)) <= s * 0.5 * (1 + 1e-6))


def test_int8_ties_and_zero_row(orc):
    x = np.array([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5], dtype=np.float32)  # s = 1 exactly
    codes, s = orc.quant_int8_row(x)
    assert s == 1.0
    assert codes.tolist() == [127, 2, 4, -2, -4, 0, 0, 2]
    codes, s = orc.quant_int8_row(np.zeros(64, dtype=np.float32))
    assert s == 0.0 and not codes.any()


def test_fp8_row_against_torch(orc):
    rng = np.random.default_rng(3)
    for _ in range(100):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 10)).astype(np.float32)
        codes, s = orc.quant_fp8_row(x)
        s_ref = np.float32(np.abs(x).max()) / np.float32(448.0)
        assert np.float32(s) == s_ref
        y = x / s_ref                                   # float32 division
        y = np.clip(y, -448, 448)                       # satfinite (only rounding excess)
        ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes, ref)
        # the largest |x| lands on +-448 or within one E4M3 step of it
        i = int(np.abs(x).argmax())
        assert abs(orc.e4m3_to_double(int(codes[i]))) >= 416


# --------------------------------------------------------------------------
# Attention: closed forms and special cases.
# --------------------------------------------------------------------------

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_single_token_returns_its_value(orc):
    q, k, v = _rand((4, 16), 0), _rand((1, 2, 16), 1), _rand((1, 2, 16), 2)
    out = orc.attention_contiguous(q, k, v, 0.25)
    for h in range(4):
        assert np.array_equal(out[h], v[0, h // 2])


def test_zero_query_or_zero_scale_gives_mean_of_values(orc):
    k, v = _rand((37, 2, 16), 3), _rand((37, 2, 16), 4)
    mean = v.mean(axis=0)
    out = orc.attention_contiguous(np.zeros((2, 16)), k, v, 0.5)
    np.testing.assert_allclose(out, mean, rtol=0, atol=1e-13)
    out = orc.attention_contiguous(_rand((2, 16), 5), k, v, 0.0)
    np.testing.assert_allclose(out, mean, rtol=0, atol=1e-13)


def test_equal_keys_give_mean_of_values(orc):
    k = np.repeat(_rand((1, 1, 16), 6), 50, axis=0)
    v = _rand((50, 1, 16), 7)
    out = orc.attention_contiguous(_rand((3, 16), 8), k, v, 1.0)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0), (3, 16)), atol=1e-13)


def test_two_tokens_logistic_closed_form(orc):
    q, k, v = _rand((1, 8), 9), _rand((2, 1, 8), 10), _rand((2, 1, 8), 11)
    scale = 0.7
    x0 = scale * sum(q[0, d] * k[0, 0, d] for d in range(8))
    x1 = scale * sum(q[0, d] * k[1, 0, d] for d in range(8))
    w1 = 1.0 / (1.0 + math.exp(x0 - x1))
    expect = w1 * v[1, 0] + (1 - w1) * v[0, 0]
    np.testing.assert_allclose(orc.attention_contiguous(q, k, v, scale)[0], expect, atol=1e-14)


def test_value_affine_equivariance_and_key_shift_invariance(orc):
    q, k, v = _rand((4, 32), 12), _rand((29, 4, 32), 13), _rand((29, 4, 32), 14)
    base = orc.attention_contiguous(q, k, v, 0.3)
    np.testing.assert_allclose(orc.attention_contiguous(q, k, 3 * v - 2, 0.3), 3 * base - 2,
                               atol=1e-12)
    shift = _rand((1, 4, 32), 15)
    np.testing.assert_allclose(orc.attention_contiguous(q, k + shift, v, 0.3), base, atol=1e-12)


def test_dominant_key_selects_its_value(orc):
    q = _rand((1, 16), 16)
    k = _rand((20, 1, 16), 17) * 0.01
    k[13, 0] = 50.0 * q[0]
    v = _rand((20, 1, 16), 18)
    np.testing.assert_allclose(orc.attention_contiguous(q, k, v, 1.0)[0], v[13, 0], atol=1e-12)


def test_softmax_is_global_not_per_block(orc):
    # Per-block softmax summed over blocks (one reading of the s05 pseudo-code) would
    # give sum_b mean(V_b) for q = 0; the oracle gives the mean over all tokens.
    v = _rand((32, 1, 4), 19)
    k = _rand((32, 1, 4), 20)
    out = orc.attention_contiguous(np.zeros((1, 4)), k, v, 1.0)[0]
    per_block = v[:16, 0].mean(0) + v[16:, 0].mean(0)
    np.testing.assert_allclose(out, v[:, 0].mean(0), atol=1e-14)
    assert np.abs(out - per_block).max() > 0.1


def test_gqa_maps_head_to_group(orc):
    H, Hkv, D, T = 8, 2, 16, 23
    q, k, v = _rand((H, D), 21), _rand((T, Hkv, D), 22), _rand((T, Hkv, D), 23)
    out = orc.attention_contiguous(q, k, v, 0.5)
    for h in range(H):
        kvh = h // (H // Hkv)
        one = orc.attention_contiguous(q[h:h + 1], k[:, kvh:kvh + 1], v[:, kvh:kvh + 1], 0.5)
        assert np.array_equal(out[h], one[0])


# --------------------------------------------------------------------------
# Paged attention == contiguous attention on the same tokens; block tables.
# --------------------------------------------------------------------------

def _filled(p, orc):
    """Write the problem's history and new rows into CPU caches with the oracle."""
    kc, vc = p.k_cache.clone(), p.v_cache.clone()
    ks = p.k_scale.clone() if p.k_scale is not None else None
    vs = p.v_scale.clone() if p.v_scale is not None else None
    cd = p.wl.cache_dtype
    orc.reshape_and_cache(p.hist_key, p.hist_value, kc, vc, p.hist_slots, cache_dtype=cd,
                          k_scale=ks, v_scale=vs)
    b = p.batch
    orc.reshape_and_cache(b.new_key, b.new_value, kc, vc, b.new_slots, cache_dtype=cd,
                          k_scale=ks, v_scale=vs)
    return kc, vc, ks, vs


def _gather_contiguous(cache, table, n, bs):
    """Independent statement of the lookup: token t is cache[table[t // bs], t % bs]."""
    idx = [(int(table[t // bs]), t % bs) for t in range(n)]
    return torch.stack([cache[b, o] for b, o in idx]).to(torch.float64).numpy()


def test_paged_equals_contiguous_tiny(orc):
    p = make_problem("tiny_f32", 0)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    out = orc.paged_decode(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale)
    for s in range(p.wl.num_seqs):
        n = int(b.seq_lens[s])
        k = _gather_contiguous(kc, b.block_tables[s], n, p.wl.block_size)
        v = _gather_contiguous(vc, b.block_tables[s], n, p.wl.block_size)
        ref = orc.attention_contiguous(b.q[s].double().numpy(), k, v, p.wl.scale)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-13)
    assert np.isfinite(out).all()        # poisoned slots never read


def test_worked_block_table_from_the_pages(orc):
    g = _golden("worked_block_table.json")
    bs, n = g["block_size"], g["seq_len"]
    table = [r["physical"] for r in g["rows"]]
    assert sum(r["used"] for r in g["rows"]) == n
    assert g["rows"][-1]["used"] < bs                 # only the last block is partly used
    nb, Hkv, D, H = 96, 2, 16, 4
    gen = torch.Generator().manual_seed(0)
    kc = torch.full((nb, bs, Hkv, D), float("nan"))
    vc = torch.full((nb, bs, Hkv, D), float("nan"))
    k = torch.randn((n, Hkv, D), generator=gen)
    v = torch.randn((n, Hkv, D), generator=gen)
    slots = torch.tensor([table[t // bs] * bs + t % bs for t in range(n)])
    orc.reshape_and_cache(k, v, kc, vc, slots)
    q = torch.randn((1, H, D), generator=gen)
    tables = torch.tensor([table + [-1]], dtype=torch.int32)
    out = orc.paged_decode(q, kc, vc, tables, torch.tensor([n], dtype=torch.int32), 0.25)
    ref = orc.attention_contiguous(q[0].double().numpy(), k.double().numpy(),
                                   v.double().numpy(), 0.25)
    np.testing.assert_allclose(out[0], ref, atol=1e-13)


def test_physical_relabelling_is_bit_identical(orc):
    p = make_problem("tiny_f32", 1)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    out = orc.paged_decode(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale)
    perm = torch.randperm(p.num_blocks, generator=torch.Generator().manual_seed(5))
    # new id perm[i] holds old block i
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = b.block_tables.clone()
    live = t2 >= 0
    t2[live] = perm[t2[live].long()].to(torch.int32)
    out2 = orc.paged_decode(b.q, kc2, vc2, t2, b.seq_lens, p.wl.scale)
    assert np.array_equal(out, out2)


def test_shared_prefix_equals_private_copies(orc):
    bs, Hkv, D, H = 16, 2, 32, 8
    gen = torch.Generator().manual_seed(7)
    prefix, lens = 48, [60, 75, 49]
    nb = 40
    kc = torch.full((nb, bs, Hkv, D), float("nan"), dtype=torch.float16)
    vc = kc.clone()
    rows_k = torch.randn((200, Hkv, D), generator=gen).half()
    rows_v = torch.randn((200, Hkv, D), generator=gen).half()
    # shared layout: prefix in blocks 0..2 referenced by all; private blocks after
    shared_tables, private_tables, slots_sh, slots_pr, src = [], [], [], [], []
    nxt = 3
    for s, n in enumerate(lens):
        tbl = [0, 1, 2]
        for _ in range(-(-(n - prefix) // bs)):
            tbl.append(nxt); nxt += 1
        shared_tables.append(tbl)
    for s, n in enumerate(lens):
        tbl = []
        for _ in range(-(-n // bs)):
            tbl.append(nxt); nxt += 1
        private_tables.append(tbl)
    ci = 0
    for t in range(prefix):
        slots_sh.append(t); src.append(t)
    ci = prefix
    for s, n in enumerate(lens):
        for t in range(prefix, n):
            slots_sh.append(shared_tables[s][t // bs] * bs + t % bs); src.append(ci + t - prefix)
        ci += n - prefix
    idx = torch.tensor(src)
    orc.reshape_and_cache(rows_k[idx], rows_v[idx], kc, vc, torch.tensor(slots_sh))
    # private copies: the same rows at private slots
    src_p, slots_p = [], []
    ci = prefix
    for s, n in enumerate(lens):
        for t in range(n):
            slots_p.append(private_tables[s][t // bs] * bs + t % bs)
            src_p.append(t if t < prefix else ci + t - prefix)
        ci += n - prefix
    idx = torch.tensor(src_p)
    orc.reshape_and_cache(rows_k[idx], rows_v[idx], kc, vc, torch.tensor(slots_p))
    W = max(len(t) for t in shared_tables + private_tables)
    pad = lambda ts: torch.tensor([t + [-1] * (W - len(t)) for t in ts], dtype=torch.int32)
    q = torch.randn((3, H, D), generator=gen).half()
    sl = torch.tensor(lens, dtype=torch.int32)
    a = orc.paged_decode(q, kc, vc, pad(shared_tables), sl, 0.2)
    b = orc.paged_decode(q, kc, vc, pad(private_tables), sl, 0.2)
    assert np.array_equal(a, b)


def test_empty_sequence_gives_zero(orc):
    p = make_problem("tiny_f32", 0)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    sl = b.seq_lens.clone()
    sl[1] = 0
    out = orc.paged_decode(b.q, kc, vc, b.block_tables, sl, p.wl.scale)
    assert not out[1].any()


def test_out_of_range_block_id_is_rejected(orc):
    p = make_problem("tiny_f32", 0)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    t = b.block_tables.clone()
    t[0, 0] = p.num_blocks
    with pytest.raises(orc.OracleError):
        orc.paged_decode(b.q, kc, vc, t, b.seq_lens, p.wl.scale)


# --------------------------------------------------------------------------
# v2 split-K: partitions and the log-sum-exp merge.
# --------------------------------------------------------------------------

def test_merge_hand_example(orc):
    # two partitions: (m, l, o) = (0, 1, [1, 0]) and (ln 3, 1, [0, 1]).
    # M = ln 3, weights 1/3 and 1 -> out = ([1/3, 0] + [0, 1]) / (4/3) = [1/4, 3/4].
    tmp = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    ml = np.array([[[0.0, math.log(3.0)]]])
    es = np.array([[[1.0, 1.0]]])
    out = orc.merge(tmp, ml, es, np.array([20]), 10)
    np.testing.assert_allclose(out[0, 0], [0.25, 0.75], atol=1e-15)
    # an empty partition (l = 0, m = -inf) is skipped
    tmp2 = np.concatenate([tmp, np.zeros((1, 1, 1, 2))], axis=2)
    out2 = orc.merge(tmp2, np.concatenate([ml, [[[-np.inf]]]], axis=2),
                     np.concatenate([es, [[[0.0]]]], axis=2), np.array([30]), 10)
    np.testing.assert_allclose(out2[0, 0], [0.25, 0.75], atol=1e-15)


@pytest.mark.parametrize("P", [16, 32, 48, 64, 512])
def test_partition_then_merge_equals_single_pass(orc, P):
    p = make_problem("tiny_f32", 2)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    v1 = orc.paged_decode(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale)
    maxp = -(-int(b.seq_lens.max()) // P)
    tmp, ml, es = orc.paged_decode_partition(b.q, kc, vc, b.block_tables, b.seq_lens,
                                             p.wl.scale, P, maxp)
    out = orc.merge(tmp, ml, es, b.seq_lens.numpy(), P)
    np.testing.assert_allclose(out, v1, rtol=0, atol=1e-13)
    for s in range(p.wl.num_seqs):
        n = int(b.seq_lens[s])
        for part in range(maxp):
            if part * P >= n:
                assert ml[s, :, part].tolist() == [-np.inf] * p.wl.num_heads
                assert not es[s, :, part].any()
            else:
                # l_p >= 1: the max token contributes exp(0)
                assert (es[s, :, part] >= 1.0).all()


def test_single_partition_partials_are_the_softmax_statistics(orc):
    p = make_problem("tiny_f32", 3)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    tmp, ml, es = orc.paged_decode_partition(b.q, kc, vc, b.block_tables, b.seq_lens,
                                             p.wl.scale, 128, 1)
    v1 = orc.paged_decode(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale)
    np.testing.assert_allclose(tmp[:, :, 0], v1, atol=1e-13)
    # m and l against an independent gather of the logits
    s, h = 0, 2
    n = int(b.seq_lens[s])
    k = _gather_contiguous(kc, b.block_tables[s], n, 16)[:, h]
    x = p.wl.scale * (k @ b.q[s, h].double().numpy())
    assert ml[s, h, 0] == pytest.approx(x.max(), abs=1e-13)
    assert es[s, h, 0] == pytest.approx(np.exp(x - x.max()).sum(), rel=1e-13)


# --------------------------------------------------------------------------
# Cache write.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dt", [torch.float32, torch.float16, torch.bfloat16])
def test_cache_write_scatter_matches_indexing(orc, dt):
    nb, bs, Hkv, D, n = 12, 8, 3, 64, 30
    gen = torch.Generator().manual_seed(0)
    kc = torch.full((nb, bs, Hkv, D), 7.0, dtype=dt)
    vc = kc.clone()
    key = torch.randn((n, Hkv, D), generator=gen).to(dt)
    val = torch.randn((n, Hkv, D), generator=gen).to(dt)
    slots = torch.randperm(nb * bs, generator=gen)[:n]
    slots[3] = -1
    orc.reshape_and_cache(key, val, kc, vc, slots)
    ek, ev = torch.full_like(kc, 7.0), torch.full_like(vc, 7.0)
    keep = slots >= 0
    ek.view(-1, Hkv, D)[slots[keep]] = key[keep]
    ev.view(-1, Hkv, D)[slots[keep]] = val[keep]
    assert torch.equal(kc, ek) and torch.equal(vc, ev)


@pytest.mark.parametrize("cd", ["int8", "fp8"])
def test_quantised_cache_write_rows(orc, cd):
    nb, bs, Hkv, D, n = 10, 16, 2, 128, 25
    gen = torch.Generator().manual_seed(1)
    storage = torch.int8 if cd == "int8" else torch.uint8
    kc = torch.zeros((nb, bs, Hkv, D), dtype=storage)
    vc = kc.clone()
    ks = torch.full((nb, Hkv, bs), float("nan"))
    vs = ks.clone()
    key = torch.randn((n, Hkv, D), generator=gen).half()
    val = torch.randn((n, Hkv, D), generator=gen).half()
    val[4, 1] = 0.0
    slots = torch.randperm(nb * bs, generator=gen)[:n]
    orc.reshape_and_cache(key, val, kc, vc, slots, cache_dtype=cd, k_scale=ks, v_scale=vs)
    rowq = orc.quant_int8_row if cd == "int8" else orc.quant_fp8_row
    for i in range(n):
        blk, off = int(slots[i]) // bs, int(slots[i]) % bs
        for h in range(Hkv):
            for src, cache, sc in ((key, kc, ks), (val, vc, vs)):
                codes, s = rowq(src[i, h].float().numpy())
                assert np.array_equal(cache[blk, off, h].numpy().view(codes.dtype), codes)
                assert np.float32(sc[blk, h, off]) == np.float32(s)
    assert vs[int(slots[4]) // bs, 1, int(slots[4]) % bs] == 0.0


def test_cache_write_rejects_slot_past_the_pool(orc):
    kc = torch.zeros((2, 4, 1, 64))
    with pytest.raises(orc.OracleError):
        orc.reshape_and_cache(torch.zeros((1, 1, 64)), torch.zeros((1, 1, 64)), kc, kc.clone(),
                              torch.tensor([8]))


# --------------------------------------------------------------------------
# Quantised decode is attention over the dequantised values c * s.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("cd", ["int8", "fp8"])
def test_quantised_decode_equals_decode_of_dequantised_cache(orc, cd):
    p = make_problem("quant_int8", 4, num_seqs=3, cache_dtype=cd, seq_lens=[37, 16, 70],
                     num_blocks=20, num_heads=8, num_kv_heads=2, head_dim=64)
    kc, vc, ks, vs = _filled(p, orc)
    b = p.batch
    out = orc.paged_decode(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale,
                           cache_dtype=cd, k_scale=ks, v_scale=vs)
    dec = (lambda c: c.to(torch.float64)) if cd == "int8" else (
        lambda c: c.view(torch.float8_e4m3fn).to(torch.float64))
    kd = dec(kc) * ks.double().permute(0, 2, 1).unsqueeze(-1)
    vd = dec(vc) * vs.double().permute(0, 2, 1).unsqueeze(-1)
    ref = orc.paged_decode(b.q, kd, vd, b.block_tables, b.seq_lens, p.wl.scale)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# The sampled-pairs decode (the reference of every full-size parity test) is
# row for row the full decode: same (sequence, head) -> same bits.
# --------------------------------------------------------------------------

_PAIRS_CASES = {
    # the tiny fp32 multi-head configuration exactly (G = 1)
    "tiny_f32": dict(name="tiny_f32"),
    # GQA, group of 8, fp16, lengths across block edges
    "gqa_f16": dict(name="qwen3_32b_f16", num_seqs=5, seq_lens=[1, 16, 17, 40, 3],
                    num_heads=16, num_kv_heads=2, head_dim=64, num_blocks=16),
    "int8": dict(name="quant_int8", num_seqs=4, seq_lens=[1, 33, 16, 50], num_heads=8,
                 num_kv_heads=2, head_dim=64, num_blocks=12),
    "fp8": dict(name="quant_fp8", num_seqs=4, seq_lens=[2, 17, 31, 48], num_heads=12,
                num_kv_heads=3, head_dim=64, num_blocks=12),
}


@pytest.mark.parametrize("case", sorted(_PAIRS_CASES))
def test_decode_pairs_equals_rows_of_the_full_decode(orc, case):
    kw = dict(_PAIRS_CASES[case])
    p = make_problem(kw.pop("name"), 5, **kw)
    kc, vc, ks, vs = _filled(p, orc)
    b = p.batch
    sl = b.seq_lens.clone()
    sl[0] = 1                                     # a single-token sequence (its first row)
    sl[-1] = 0                                    # and an empty one
    S, H = b.q.shape[0], b.q.shape[1]
    cd = p.wl.cache_dtype
    full = orc.paged_decode(b.q, kc, vc, b.block_tables, sl, p.wl.scale, cache_dtype=cd,
                            k_scale=ks, v_scale=vs)
    # every pair once, shuffled, then some repeated: the i-th output row belongs to the
    # i-th pair whatever the order
    every = np.array([(s, h) for s in range(S) for h in range(H)], dtype=np.int32)
    rng = np.random.default_rng(len(case))
    pairs = np.concatenate([every[rng.permutation(len(every))], every[rng.integers(0, len(every), 7)]])
    got = orc.paged_decode_pairs(b.q, kc, vc, b.block_tables, sl, p.wl.scale, pairs,
                                 cache_dtype=cd, k_scale=ks, v_scale=vs)
    assert got.shape == (len(pairs), b.q.shape[2])
    want = full[pairs[:, 0], pairs[:, 1]]
    assert np.array_equal(got, want), case
    assert not got[pairs[:, 0] == S - 1].any()    # the empty sequence's rows are zero
    # a single-token sequence returns its one V row, in the pair form as well
    ones = [s for s in range(S) if int(sl[s]) == 1]
    G = H // p.wl.num_kv_heads
    for s in ones:
        for h in range(H):
            row = got[np.flatnonzero((pairs[:, 0] == s) & (pairs[:, 1] == h))[0]]
            blk, off = int(b.block_tables[s, 0]), 0
            if cd in ("int8", "fp8"):
                codes = vc[blk, off, h // G]
                val = (codes.to(torch.float64) if cd == "int8" else
                       codes.view(torch.float8_e4m3fn).to(torch.float64)) * float(vs[blk, h // G, off])
            else:
                val = vc[blk, off, h // G].to(torch.float64)
            np.testing.assert_allclose(row, val.numpy(), rtol=0, atol=1e-12)


def test_decode_pairs_rejects_a_pair_outside_the_batch(orc):
    p = make_problem("tiny_f32", 0)
    kc, vc, _, _ = _filled(p, orc)
    b = p.batch
    for bad in ([4, 0], [0, 4], [-1, 0]):
        with pytest.raises(Exception):
            orc.paged_decode_pairs(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale,
                                   np.array([[0, 0], bad], dtype=np.int32))


# --------------------------------------------------------------------------
# Block copy: copy-on-write of a shared block and swap between block pools.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("cd", ["f16", "int8"])
def test_copy_blocks_matches_indexing(orc, cd):
    nb, bs, Hkv, D = 12, 16, 2, 64
    gen = torch.Generator().manual_seed(3)
    if cd == "int8":
        kc = torch.randint(-127, 128, (nb, bs, Hkv, D), generator=gen, dtype=torch.int8)
        ks = torch.rand((nb, Hkv, bs), generator=gen)
    else:
        kc = torch.randn((nb, bs, Hkv, D), generator=gen).half()
        ks = None
    vc = kc.flip(0).clone()
    vs = ks.flip(0).clone() if ks is not None else None
    pairs = torch.tensor([[1, 7], [4, 2], [1, 9], [10, 0]])
    ek, ev = kc.clone(), vc.clone()
    ek[pairs[:, 1]] = kc[pairs[:, 0]]
    ev[pairs[:, 1]] = vc[pairs[:, 0]]
    if ks is not None:
        eks, evs = ks.clone(), vs.clone()
        eks[pairs[:, 1]] = ks[pairs[:, 0]]
        evs[pairs[:, 1]] = vs[pairs[:, 0]]
    orc.copy_blocks(kc, vc, kc, vc, pairs, cache_dtype=cd, src_k_scale=ks, src_v_scale=vs,
                    dst_k_scale=ks, dst_v_scale=vs)
    assert torch.equal(kc, ek) and torch.equal(vc, ev)
    if ks is not None:
        assert torch.equal(ks, eks) and torch.equal(vs, evs)


def test_copy_on_write_keeps_the_other_sequence(orc):
    """Two sequences share 40 tokens (the last block half full).  The second appends
    a token: its shared last block is copied to a fresh id, its table repointed and
    the token written into the copy.  The first sequence's output does not change
    and the second's is attention over its own 41 tokens."""
    bs, Hkv, D, H, nb = 16, 2, 32, 4, 8
    gen = torch.Generator().manual_seed(11)
    kc = torch.full((nb, bs, Hkv, D), float("nan"), dtype=torch.float16)
    vc = kc.clone()
    k = torch.randn((41, Hkv, D), generator=gen).half()
    v = torch.randn((41, Hkv, D), generator=gen).half()
    table = [5, 1, 6]
    orc.reshape_and_cache(k[:40], v[:40], kc, vc,
                          torch.tensor([table[t // bs] * bs + t % bs for t in range(40)]))
    q = torch.randn((2, H, D), generator=gen).half()
    shared = torch.tensor([table, table], dtype=torch.int32)
    lens = torch.tensor([40, 40], dtype=torch.int32)
    before = orc.paged_decode(q, kc, vc, shared, lens, 0.3)
    orc.copy_blocks(kc, vc, kc, vc, torch.tensor([[6, 3]]))
    own = torch.tensor([table, [5, 1, 3]], dtype=torch.int32)
    orc.reshape_and_cache(k[40:], v[40:], kc, vc, torch.tensor([3 * bs + 40 % bs]))
    after = orc.paged_decode(q, kc, vc, own, torch.tensor([40, 41], dtype=torch.int32), 0.3)
    assert np.array_equal(after[0], before[0])
    ref = orc.attention_contiguous(q[1].double().numpy(), k.double().numpy(),
                                   v.double().numpy(), 0.3)
    np.testing.assert_allclose(after[1], ref, rtol=0, atol=1e-13)


def test_swap_out_and_back_in_is_bit_identical(orc):
    p = make_problem("quant_fp8", 2, num_seqs=3, seq_lens=[33, 17, 50], num_blocks=16,
                     num_heads=4, num_kv_heads=2, head_dim=64)
    kc, vc, ks, vs = _filled(p, orc)
    b = p.batch
    out = orc.paged_decode(b.q, kc, vc, b.block_tables, b.seq_lens, p.wl.scale,
                           cache_dtype="fp8", k_scale=ks, v_scale=vs)
    live = sorted({int(x) for x in b.block_tables.flatten() if x >= 0})
    # swap out into a separate (host) pool, then back in at other device ids
    hk, hv = torch.zeros((len(live),) + kc.shape[1:], dtype=kc.dtype), None
    hv = torch.zeros_like(hk)
    hks = torch.zeros((len(live),) + ks.shape[1:])
    hvs = torch.zeros_like(hks)
    out_pairs = torch.tensor([[blk, i] for i, blk in enumerate(live)])
    orc.copy_blocks(kc, vc, hk, hv, out_pairs, cache_dtype="fp8", src_k_scale=ks,
                    src_v_scale=vs, dst_k_scale=hks, dst_v_scale=hvs)
    kc2, vc2 = torch.zeros_like(kc), torch.zeros_like(vc)
    ks2, vs2 = torch.full_like(ks, float("nan")), torch.full_like(vs, float("nan"))
    new_ids = torch.randperm(kc.shape[0], generator=torch.Generator().manual_seed(9))[:len(live)]
    in_pairs = torch.tensor([[i, int(new_ids[i])] for i in range(len(live))])
    orc.copy_blocks(hk, hv, kc2, vc2, in_pairs, cache_dtype="fp8", src_k_scale=hks,
                    src_v_scale=hvs, dst_k_scale=ks2, dst_v_scale=vs2)
    remap = {blk: int(new_ids[i]) for i, blk in enumerate(live)}
    t2 = b.block_tables.clone()
    for idx, x in np.ndenumerate(t2.numpy()):
        if x >= 0:
            t2[idx] = remap[int(x)]
    out2 = orc.paged_decode(b.q, kc2, vc2, t2, b.seq_lens, p.wl.scale, cache_dtype="fp8",
                            k_scale=ks2, v_scale=vs2)
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("pairs", [[[0, 2], [1, 2]],      # two writes to block 2
                                   [[0, 1], [1, 3]],      # block 1 both written and read
                                   [[0, 4]]])             # past the pool
def test_copy_blocks_rejects_ambiguous_or_out_of_range(orc, pairs):
    kc = torch.zeros((4, 16, 1, 64), dtype=torch.float16)
    with pytest.raises(orc.OracleError):
        orc.copy_blocks(kc, kc.clone(), kc, kc.clone(), torch.tensor(pairs))


# --------------------------------------------------------------------------
# Multi-token query (prefix-cached prefill chunk) over the paged cache.
# --------------------------------------------------------------------------

def _prefill_problem(orc, lens, qlens, seed, dt=torch.float16, bs=16, H=8, Hkv=2, D=64):
    gen = torch.Generator().manual_seed(seed)
    nb = sum(-(-n // bs) for n in lens) + 4
    kc = torch.full((nb, bs, Hkv, D), float("nan"), dtype=dt)
    vc = kc.clone()
    perm = torch.randperm(nb, generator=gen).tolist()
    tables, slots, rows_k, rows_v = [], [], [], []
    W = max(-(-n // bs) for n in lens)
    for n in lens:
        t = [perm.pop() for _ in range(-(-n // bs))]
        tables.append(t + [-1] * (W - len(t)))
        k = torch.randn((n, Hkv, D), generator=gen).to(dt)
        v = torch.randn((n, Hkv, D), generator=gen).to(dt)
        rows_k.append(k)
        rows_v.append(v)
        slots += [t[i // bs] * bs + i % bs for i in range(n)]
    orc.reshape_and_cache(torch.cat(rows_k), torch.cat(rows_v), kc, vc, torch.tensor(slots))
    qs = torch.tensor([0] + list(np.cumsum(qlens)), dtype=torch.int32)
    q = torch.randn((int(qs[-1]), H, D), generator=gen).to(dt)
    return q, kc, vc, torch.tensor(tables, dtype=torch.int32), torch.tensor(lens, dtype=torch.int32), \
        qs, rows_k, rows_v


def test_prefill_equals_causal_contiguous_attention(orc):
    lens, qlens = [37, 16, 50], [5, 16, 1]
    q, kc, vc, tables, sl, qs, rk, rv = _prefill_problem(orc, lens, qlens, 0)
    out = orc.paged_prefill(q, kc, vc, tables, sl, qs, 0.2)
    for s, (n, ql) in enumerate(zip(lens, qlens)):
        for r in range(ql):
            pos = n - ql + r
            row = int(qs[s]) + r
            G = q.shape[1] // kc.shape[2]
            for h in range(q.shape[1]):
                k = rk[s][:pos + 1, h // G].double().numpy()[:, None, :]
                v = rv[s][:pos + 1, h // G].double().numpy()[:, None, :]
                ref = orc.attention_contiguous(q[row, h:h + 1].double().numpy(), k, v, 0.2)
                np.testing.assert_allclose(out[row, h], ref[0], rtol=0, atol=1e-13)


def test_prefill_of_one_token_is_the_decode(orc):
    lens = [37, 16, 50, 1]
    q, kc, vc, tables, sl, qs, _, _ = _prefill_problem(orc, lens, [1, 1, 1, 1], 1)
    pre = orc.paged_prefill(q, kc, vc, tables, sl, qs, 0.125)
    dec = orc.paged_decode(q, kc, vc, tables, sl, 0.125)
    assert np.array_equal(pre, dec)


def test_prefill_chunks_compose(orc):
    """A 24-token chunk computed at once equals the same rows computed as two chunks
    (the first with the sequence cut after its own last token)."""
    q, kc, vc, tables, sl, qs, _, _ = _prefill_problem(orc, [60], [24], 2)
    full = orc.paged_prefill(q, kc, vc, tables, sl, qs, 0.3)
    a = orc.paged_prefill(q[:10], kc, vc, tables, torch.tensor([46], dtype=torch.int32),
                          torch.tensor([0, 10], dtype=torch.int32), 0.3)
    b = orc.paged_prefill(q[10:], kc, vc, tables, sl, torch.tensor([0, 14], dtype=torch.int32),
                          0.3)
    assert np.array_equal(full, np.concatenate([a, b]))


def test_prefill_rejects_a_chunk_longer_than_the_sequence(orc):
    q, kc, vc, tables, sl, qs, _, _ = _prefill_problem(orc, [8], [8], 3)
    with pytest.raises(orc.OracleError):
        orc.paged_prefill(torch.cat([q, q]), kc, vc, tables, sl,
                          torch.tensor([0, 16], dtype=torch.int32), 0.3)
