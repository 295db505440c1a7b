"""The C-ABI library: it loads, exports every symbol include/pa.h declares, and its
host-side helpers and argument checks behave (no kernel launches).  CPU only."""
import ctypes
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_390_b200 import build, pa
    build.build()
    return pa.lib()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", src)
    return names


def test_header_declares_the_path(lib):
    names = set(_declared())
    for n in ("pa_reshape_and_cache", "pa_decode_v1", "pa_decode_v2_partition",
              "pa_decode_v2_merge", "pa_decode_v2_workspace_bytes", "pa_choose_partition_size",
              "pa_kv_bytes_per_token", "pa_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "pa_bm_create" in names and "pa_copy_blocks" in names and len(names) >= 30
    for n in names:
        assert hasattr(lib, n), n


def test_no_oracle_symbols_in_the_library(lib):
    assert not hasattr(lib, "orc_paged_decode")


def test_status_strings(lib):
    assert lib.pa_status_string(0) == b"PA_OK"
    assert lib.pa_status_string(1) == b"PA_ERR_INVALID_ARG"
    assert lib.pa_status_string(2) == b"PA_ERR_UNSUPPORTED"
    assert lib.pa_status_string(3) == b"PA_ERR_CUDA"


def test_kv_bytes_per_token_page_figures(lib):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "kv_size.json")))
    for c in g["cases"]:
        assert lib.pa_kv_bytes_per_token(c["num_layers"], c["num_kv_heads"], c["head_dim"],
                                         c["dtype_bytes"]) == c["bytes_per_token"]


def test_workspace_bytes(lib):
    assert lib.pa_decode_v2_workspace_bytes(8, 64, 128, 64) == 8 * 64 * 64 * 130 * 4
    assert lib.pa_decode_v2_workspace_bytes(0, 64, 128, 64) == 0


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("max_len,S,Hkv", [(768, 32, 8), (32768, 8, 8), (16384, 256, 8),
                                          (1, 1, 1), (100, 4, 4)])
def test_partition_size_properties(lib, bs, max_len, S, Hkv):
    P = lib.pa_choose_partition_size(max_len, S, Hkv, 148, bs)
    tt = max(16, bs)
    assert P % (6 * tt) == 0          # whole tiles for each of the 6 warps
    assert P >= 24 * tt               # at least 4 tiles per warp


def _null_decode_call(lib, **over):
    P = ctypes.c_void_p
    fake = P(1 << 20)                 # aligned non-null pointer, never dereferenced
    args = dict(out=fake, q=fake, q_dtype=1, k=fake, v=fake, cd=1, ks=None, vs=None, bt=fake,
                mb=4, sl=fake, S=2, H=8, Hkv=2, D=128, bs=16, nb=10, scale=0.1)
    args.update(over)
    return lib.pa_decode_v1(args["out"], args["q"], args["q_dtype"], args["k"], args["v"],
                            args["cd"], args["ks"], args["vs"], args["bt"], args["mb"],
                            args["sl"], args["S"], args["H"], args["Hkv"], args["D"], args["bs"],
                            args["nb"], args["scale"], None, None)


@pytest.mark.parametrize("over,status", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(H=7), 1), (dict(bs=12), 1),
    (dict(D=96), 2), (dict(H=32, Hkv=2), 2), (dict(q_dtype=0, cd=1), 2),
    (dict(cd=3), 1),                      # quantised cache without scales
    (dict(q_dtype=2, cd=1), 2), (dict(scale=float("inf")), 1),
    (dict(q=ctypes.c_void_p((1 << 20) + 4)), 1),   # misaligned q
])
def test_decode_host_checks(lib, over, status):
    assert _null_decode_call(lib, **over) == status


def test_zero_sequences_is_a_no_op(lib):
    assert _null_decode_call(lib, S=0) == 0


def test_v2_partition_size_must_be_whole_tiles(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    rc = lib.pa_decode_v2_partition(fake, fake, fake, fake, 1, fake, fake, 1, None, None, fake, 4,
                                    fake, 2, 8, 2, 128, 16, 10, 0.1, 24, 4, None, None)
    assert rc == 1
    rc = lib.pa_decode_v2_partition(fake, fake, fake, fake, 1, fake, fake, 1, None, None, fake, 4,
                                    fake, 2, 8, 2, 128, 32, 10, 0.1, 48, 4, None, None)
    assert rc == 1


def test_cache_write_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    # fp16 rows into a bf16 cache: unsupported; block size 12: invalid
    assert lib.pa_reshape_and_cache(fake, fake, 1, fake, fake, 2, None, None, fake, 4, 2, 128,
                                    16, 10, None, None) == 2
    assert lib.pa_reshape_and_cache(fake, fake, 1, fake, fake, 1, None, None, fake, 4, 2, 128,
                                    12, 10, None, None) == 1
    assert lib.pa_reshape_and_cache(fake, fake, 1, fake, fake, 3, None, None, fake, 4, 2, 128,
                                    16, 10, None, None) == 1
    assert lib.pa_reshape_and_cache(None, None, 1, None, None, 1, None, None, None, 0, 2, 128,
                                    16, 10, None, None) == 0


def test_copy_blocks_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    args = lambda **kw: [kw.get("sk", fake), fake, kw.get("sks", None), None, 8,
                         fake, fake, None, None, 8, kw.get("dt", 1), kw.get("bm", fake),
                         kw.get("n", 3), 2, kw.get("D", 128), kw.get("bs", 16), None, None]
    assert lib.pa_copy_blocks(*args(n=0, bm=None, sk=None)) == 0     # nothing to copy
    assert lib.pa_copy_blocks(*args(n=-1)) == 1
    assert lib.pa_copy_blocks(*args(bs=12)) == 1
    assert lib.pa_copy_blocks(*args(D=96)) == 2
    assert lib.pa_copy_blocks(*args(sk=None)) == 1
    assert lib.pa_copy_blocks(*args(bm=None)) == 1
    assert lib.pa_copy_blocks(*args(sk=P((1 << 20) + 8))) == 1     # misaligned pool
    assert lib.pa_copy_blocks(*args(dt=3)) == 1                     # int8 without scales
    assert lib.pa_copy_blocks(*args(dt=7)) == 1


def test_append_decode_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    args = lambda **kw: [fake, fake, 1, kw.get("key", fake), fake, kw.get("slots", fake), fake,
                         fake, 1, None, None, fake, 4, fake, kw.get("S", 2), 16, 2, 128,
                         kw.get("bs", 16), 10, 0.1, None, None]
    assert lib.pa_append_decode_v1(*args(S=0)) == 0
    assert lib.pa_append_decode_v1(*args(key=None)) == 1
    assert lib.pa_append_decode_v1(*args(slots=None)) == 1
    assert lib.pa_append_decode_v1(*args(slots=P((1 << 20) + 4))) == 1
    assert lib.pa_append_decode_v1(*args(bs=12)) == 1


def test_prefill_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    args = lambda **kw: [fake, fake, kw.get("qd", 2), fake, 10, 5, fake, fake, kw.get("cd", 2),
                         fake, 4, fake, 2, kw.get("H", 16), 2, kw.get("D", 128), 16, 10, 0.1,
                         None, None]
    assert lib.pa_prefill(*args(D=64)) == 2
    assert lib.pa_prefill(*args(qd=1, cd=2)) == 2          # fp16 q over a bf16 cache
    assert lib.pa_prefill(*args(qd=4, cd=4)) == 2          # fp8 not supported here
    assert lib.pa_prefill(*args(H=15)) == 1


def test_config_knobs(lib):
    assert lib.pa_set_decode_config(9, 0) == 1
    assert lib.pa_set_fault_injection(2) == 1
    assert lib.pa_set_fault_injection(0) == 0
    assert lib.pa_set_decode_config(0, 9) == 1
    assert lib.pa_set_decode_config(2, 3) == 0
    assert lib.pa_set_decode_config(0, 0) == 0
    assert lib.pa_set_pdl(3) == 1 and lib.pa_set_pdl(-1) == 1
    assert lib.pa_set_pdl(2) == 0 and lib.pa_set_pdl(1) == 0
    assert lib.pa_set_prefetch_tiles(-2) == 1 and lib.pa_set_prefetch_tiles(33) == 1
    assert lib.pa_set_prefetch_tiles(4) == 0 and lib.pa_set_prefetch_tiles(-1) == 0
    # cascade: split counts -1 (side by side) .. 4, suffix forms 0 and 1
    assert lib.pa_set_cascade_config(-2, 0) == 1 and lib.pa_set_cascade_config(5, 0) == 1
    assert lib.pa_set_cascade_config(0, 2) == 1 and lib.pa_set_cascade_config(0, -1) == 1
    assert lib.pa_set_cascade_config(-1, 1) == 0 and lib.pa_set_cascade_config(4, 0) == 0
    assert lib.pa_set_cascade_config(0, 0) == 0


def test_product_path_does_not_touch_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_390_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in txt.lower() or f == "workloads.py", f
