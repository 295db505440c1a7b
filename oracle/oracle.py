"""ctypes wrapper around the C oracle (``pa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only users.  The product path never
imports this module.  It marshals torch CPU tensors / numpy arrays into the
C functions and shares nothing with the CUDA library.

Every function here restates one routine of ``pa_oracle.c``; see that file for
the page and section each follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, F16, BF16, INT8, FP8E4M3, F64 = 0, 1, 2, 3, 4, 5
DTYPE_CODES = {"f32": F32, "f16": F16, "bf16": BF16, "int8": INT8, "fp8": FP8E4M3}
_TORCH_CODES = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16, torch.float64: F64}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C11, no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared",
           "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        sig = {
            "orc_f16_to_double": (D, [ctypes.c_uint16]),
            "orc_bf16_to_double": (D, [ctypes.c_uint16]),
            "orc_e4m3_to_double": (D, [ctypes.c_uint8]),
            "orc_e4m3_from_float": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_quant_int8_row": (ctypes.c_float, [P, I, P]),
            "orc_quant_fp8_row": (ctypes.c_float, [P, I, P]),
            "orc_kv_bytes_per_token": (D, [I, I, I, I]),
            "orc_attention_contiguous": (I, [P, P, P, P, I, I, I, I, D]),
            "orc_paged_decode": (I, [P, P, I, P, P, I, P, P, P, I, P, I, I, I, I, I, I, D]),
            "orc_paged_decode_pairs": (I, [P, P, I, P, I, P, P, I, P, P, P, I, P, I, I, I, I,
                                           I, I, D]),
            "orc_paged_decode_partition":(I, [P, P, P, P, I, P, P, I, P, P, P, I, P,
                                               I, I, I, I, I, I, D, I, I]),
            "orc_merge": (I, [P, P, P, P, P, I, I, I, I, I]),
            "orc_reshape_and_cache": (I, [P, P, I, P, P, I, P, P, P, I, I, I, I, I]),
            "orc_copy_blocks": (I, [P, P, P, P, I, P, P, P, P, I, I, P, I, I, I, I]),
            "orc_paged_prefill": (I, [P, P, I, P, P, P, I, P, P, P, I, P, I, I, I, I, I, I, D]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        assert t.flags["C_CONTIGUOUS"]
        return t.ctypes.data
    assert t.device.type == "cpu" and t.is_contiguous()
    return t.data_ptr()


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc}")


def _dtype_code(t: torch.Tensor, cache_dtype: str | None = None) -> int:
    if cache_dtype is not None:
        return DTYPE_CODES[cache_dtype]
    return _TORCH_CODES[t.dtype]


# --- storage formats --------------------------------------------------------

def f16_to_double(bits: int) -> float:
    return _load().orc_f16_to_double(bits)


def bf16_to_double(bits: int) -> float:
    return _load().orc_bf16_to_double(bits)


def e4m3_to_double(code: int) -> float:
    return _load().orc_e4m3_to_double(code)


def e4m3_from_float(x: float) -> int:
    return _load().orc_e4m3_from_float(float(np.float32(x)))


# --- quantisation -------------------------------------------------------------

def quant_int8_row(x) -> tuple[np.ndarray, float]:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    codes = np.zeros(x.shape[0], dtype=np.int8)
    s = _load().orc_quant_int8_row(_ptr(x), x.shape[0], _ptr(codes))
    return codes, float(np.float32(s))


def quant_fp8_row(x) -> tuple[np.ndarray, float]:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    codes = np.zeros(x.shape[0], dtype=np.uint8)
    s = _load().orc_quant_fp8_row(_ptr(x), x.shape[0], _ptr(codes))
    return codes, float(np.float32(s))


def kv_bytes_per_token(num_layers, num_kv_heads, head_dim, dtype_bytes) -> float:
    return _load().orc_kv_bytes_per_token(num_layers, num_kv_heads, head_dim, dtype_bytes)


# --- attention ----------------------------------------------------------------

def attention_contiguous(q, k, v, scale: float) -> np.ndarray:
    """q [H, D], k/v [T, H_kv, D] (any float arrays) -> out [H, D] float64."""
    q = np.ascontiguousarray(np.asarray(q, dtype=np.float64))
    k = np.ascontiguousarray(np.asarray(k, dtype=np.float64))
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    H, D = q.shape
    T, Hkv, _ = k.shape
    out = np.zeros((H, D), dtype=np.float64)
    rc = _load().orc_attention_contiguous(_ptr(out), _ptr(q), _ptr(k) if T else None,
                                          _ptr(v) if T else None, T, H, Hkv, D, float(scale))
    _check(rc, "attention_contiguous")
    return out


def _decode_common(q, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables, seq_lens):
    q = q.contiguous()
    k_cache = k_cache.contiguous()
    v_cache = v_cache.contiguous()
    bt = block_tables.to(torch.int32).contiguous()
    sl = seq_lens.to(torch.int32).contiguous()
    num_blocks, bs, Hkv, D = k_cache.shape
    S, H, _ = q.shape
    cd = _dtype_code(k_cache, cache_dtype)
    ks = k_scale.contiguous() if k_scale is not None else None
    vs = v_scale.contiguous() if v_scale is not None else None
    return q, k_cache, v_cache, cd, ks, vs, bt, sl, num_blocks, bs, Hkv, D, S, H


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, *,
                 cache_dtype=None, k_scale=None, v_scale=None) -> np.ndarray:
    """Paged decode attention in binary64 -> out [S, H, D] float64."""
    (q, k_cache, v_cache, cd, ks, vs, bt, sl, nb, bs, Hkv, D, S, H) = _decode_common(
        q, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables, seq_lens)
    out = np.zeros((S, H, D), dtype=np.float64)
    rc = _load().orc_paged_decode(_ptr(out), _ptr(q), _dtype_code(q), _ptr(k_cache),
                                  _ptr(v_cache), cd, _ptr(ks), _ptr(vs), _ptr(bt),
                                  bt.shape[1], _ptr(sl), S, H, Hkv, D, bs, nb, float(scale))
    _check(rc, "paged_decode")
    return out


def paged_decode_pairs(q, k_cache, v_cache, block_tables, seq_lens, scale, pairs, *,
                       cache_dtype=None, k_scale=None, v_scale=None) -> np.ndarray:
    """Paged decode attention for chosen (seq, head) pairs -> out [n, D] float64."""
    (q, k_cache, v_cache, cd, ks, vs, bt, sl, nb, bs, Hkv, D, S, H) = _decode_common(
        q, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables, seq_lens)
    pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    out = np.zeros((pr.shape[0], D), dtype=np.float64)
    rc = _load().orc_paged_decode_pairs(_ptr(out), _ptr(pr), pr.shape[0], _ptr(q), _dtype_code(q),
                                        _ptr(k_cache), _ptr(v_cache), cd, _ptr(ks), _ptr(vs),
                                        _ptr(bt), bt.shape[1], _ptr(sl), S, H, Hkv, D, bs, nb,
                                        float(scale))
    _check(rc, "paged_decode_pairs")
    return out


def paged_decode_partition(q, k_cache, v_cache, block_tables, seq_lens, scale,
                           partition_size, max_parts, *, cache_dtype=None,
                           k_scale=None, v_scale=None):
    """v2 partition step in binary64 -> (tmp_out [S,H,P,D], max_logits, exp_sums [S,H,P])."""
    (q, k_cache, v_cache, cd, ks, vs, bt, sl, nb, bs, Hkv, D, S, H) = _decode_common(
        q, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables, seq_lens)
    tmp = np.zeros((S, H, max_parts, D), dtype=np.float64)
    ml = np.zeros((S, H, max_parts), dtype=np.float64)
    es = np.zeros((S, H, max_parts), dtype=np.float64)
    rc = _load().orc_paged_decode_partition(
        _ptr(tmp), _ptr(ml), _ptr(es), _ptr(q), _dtype_code(q), _ptr(k_cache), _ptr(v_cache),
        cd, _ptr(ks), _ptr(vs), _ptr(bt), bt.shape[1], _ptr(sl), S, H, Hkv, D, bs, nb,
        float(scale), int(partition_size), int(max_parts))
    _check(rc, "paged_decode_partition")
    return tmp, ml, es


def merge(tmp_out, max_logits, exp_sums, seq_lens, partition_size) -> np.ndarray:
    """LSE merge of v2 partials in binary64 -> out [S, H, D] float64."""
    tmp = np.ascontiguousarray(np.asarray(tmp_out, dtype=np.float64))
    ml = np.ascontiguousarray(np.asarray(max_logits, dtype=np.float64))
    es = np.ascontiguousarray(np.asarray(exp_sums, dtype=np.float64))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    S, H, P, D = tmp.shape
    out = np.zeros((S, H, D), dtype=np.float64)
    rc = _load().orc_merge(_ptr(out), _ptr(tmp), _ptr(ml), _ptr(es), _ptr(sl), S, H, D,
                           int(partition_size), P)
    _check(rc, "merge")
    return out


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, *, cache_dtype=None,
                      k_scale=None, v_scale=None) -> None:
    """Cache write, in place on CPU tensors (caches in their storage dtype)."""
    key = key.contiguous()
    value = value.contiguous()
    assert k_cache.is_contiguous() and v_cache.is_contiguous()
    sm = slot_mapping.to(torch.int64).contiguous()
    num_blocks, bs, Hkv, D = k_cache.shape
    cd = _dtype_code(k_cache, cache_dtype)
    rc = _load().orc_reshape_and_cache(
        _ptr(key), _ptr(value), _dtype_code(key), _ptr(k_cache), _ptr(v_cache), cd,
        _ptr(k_scale), _ptr(v_scale), _ptr(sm), key.shape[0], Hkv, D, bs, num_blocks)
    _check(rc, "reshape_and_cache")


def copy_blocks(src_k, src_v, dst_k, dst_v, block_mapping, *, cache_dtype=None,
                src_k_scale=None, src_v_scale=None, dst_k_scale=None, dst_v_scale=None) -> None:
    """Block copy (copy-on-write or swap), in place on CPU tensors: for each row
    (src, dst) of block_mapping [num_pairs, 2], destination block dst becomes a copy
    of source block src (K, V and, for quantised caches, the scales)."""
    for t in (src_k, src_v, dst_k, dst_v):
        assert t.is_contiguous()
    bm = block_mapping.to(torch.int64).contiguous()
    nb_src, bs, Hkv, D = src_k.shape
    nb_dst = dst_k.shape[0]
    rc = _load().orc_copy_blocks(
        _ptr(src_k), _ptr(src_v), _ptr(src_k_scale), _ptr(src_v_scale), nb_src,
        _ptr(dst_k), _ptr(dst_v), _ptr(dst_k_scale), _ptr(dst_v_scale), nb_dst,
        _dtype_code(src_k, cache_dtype), _ptr(bm), bm.shape[0] if bm.numel() else 0, Hkv, D, bs)
    _check(rc, "copy_blocks")


def paged_prefill(q, k_cache, v_cache, block_tables, seq_lens, query_start, scale, *,
                  cache_dtype=None, k_scale=None, v_scale=None) -> np.ndarray:
    """Causal multi-token query: rows [query_start[s], query_start[s+1]) of q are the last
    tokens of sequence s (already in the cache); returns binary64 [total_q, H, D]."""
    q = q.contiguous()
    tq, H, D = q.shape
    num_blocks, bs, Hkv, _ = k_cache.shape
    qs = query_start.to(torch.int32).contiguous()
    bt = block_tables.to(torch.int32).contiguous()
    sl = seq_lens.to(torch.int32).contiguous()
    out = np.zeros((tq, H, D), dtype=np.float64)
    rc = _load().orc_paged_prefill(
        _ptr(out), _ptr(q), _dtype_code(q), _ptr(qs), _ptr(k_cache.contiguous()),
        _ptr(v_cache.contiguous()), _dtype_code(k_cache, cache_dtype), _ptr(k_scale),
        _ptr(v_scale), _ptr(bt), bt.shape[1], _ptr(sl), sl.shape[0], H, Hkv, D, bs,
        num_blocks, float(scale))
    _check(rc, "paged_prefill")
    return out
