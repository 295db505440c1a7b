"""Python binding of ``libpa.so`` (the C ABI in ``include/pa.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors must be CUDA tensors, contiguous, in the layouts of
``pa.h``; work is enqueued on the current torch stream (or ``stream``).  There
is no fallback: if the library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_F32, PA_F16, PA_BF16, PA_INT8, PA_FP8E4M3 = 0, 1, 2, 3, 4
PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_NO_SPACE = 0, 1, 2, 3, 4
DEVERR_BLOCK_ID, DEVERR_SEQ_LEN, DEVERR_SLOT, DEVERR_TIMEOUT = 1, 2, 4, 8

_FLOAT_CODES = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}
CACHE_CODES = {"f32": PA_F32, "f16": PA_F16, "bf16": PA_BF16, "int8": PA_INT8, "fp8": PA_FP8E4M3}

_lock = threading.Lock()
_lib = None


class PAError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_name(status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libpa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_390_b200.build`"
                " (there is no fallback path)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sigs = {
            "pa_reshape_and_cache": (I, [P, P, I, P, P, I, P, P, P, I, I, I, I, I, P, P]),
            "pa_decode_v1": (I, [P, P, I, P, P, I, P, P, P, I, P, I, I, I, I, I, I, F, P, P]),
            "pa_decode_v2_partition": (I, [P, P, P, P, I, P, P, I, P, P, P, I, P, I, I, I, I,
                                           I, I, F, I, I, P, P]),
            "pa_decode_v2_merge": (I, [P, I, P, P, P, P, I, I, I, I, I, P]),
            "pa_decode_v2_workspace_bytes": (S, [I, I, I, I]),
            "pa_decode_fused": (I, [P, P, I, P, P, I, P, P, P, I, P, I, I, I, I, I, I, F, P, S,
                                    P, P]),
            "pa_decode_fused_workspace_bytes": (S, [I, I, I, I]),
            "pa_decode_fused_noalloc": (I, [P, P, I, P, P, I, P, P, P, I, P, I, I, I, I, I, I, F,
                                            P, P]),
            "pa_decode_fused_noalloc_scratch_bytes": (S, []),
            "pa_choose_partition_size": (I, [I, I, I, I, I]),
            "pa_kv_bytes_per_token": (ctypes.c_double, [I, I, I, I]),
            "pa_status_string": (ctypes.c_char_p, [I]),
            "pa_last_cuda_error_string": (ctypes.c_char_p, []),
            "pa_get_device_error": (I, [ctypes.POINTER(ctypes.c_int), I]),
            "pa_set_decode_config": (I, [I, I]),
            "pa_set_wait_limit_ns": (I, [ctypes.c_ulonglong]),
            "pa_set_fault_injection": (I, [I]),
            "pa_set_pdl": (I, [I]),
            "pa_copy_blocks": (I, [P, P, P, P, I, P, P, P, P, I, I, P, I, I, I, I, P, P]),
            "pa_append_decode_v1": (I, [P, P, I, P, P, P, P, P, I, P, P, P, I, P, I, I, I, I, I,
                                        I, F, P, P]),
            "pa_set_prefetch_tiles": (I, [I]),
            "pa_decode_cascade": (I, [P, P, I, P, P, I, P, I, P, I, I, I, I, I, I, F, I, P, S, P,
                                      P]),
            "pa_decode_cascade_workspace_bytes": (S, [I, I, I]),
            "pa_set_cascade_config": (I, [I, I]),
            "pa_prefill": (I, [P, P, I, P, I, I, P, P, I, P, I, P, I, I, I, I, I, I, F, P, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
        return L


def status_name(status: int) -> str:
    try:
        return lib().pa_status_string(int(status)).decode()
    except Exception:                                   # library not loadable
        return f"status {status}"


def _check(rc: int, what: str) -> None:
    if rc == PA_ERR_CUDA:
        raise PAError(f"{what} ({lib().pa_last_cuda_error_string().decode()})", rc)
    if rc != PA_OK:
        raise PAError(what, rc)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libpa must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def cache_code(cache: torch.Tensor, cache_dtype: str | None = None) -> int:
    if cache_dtype is not None:
        return CACHE_CODES[cache_dtype]
    if cache.dtype in _FLOAT_CODES:
        return _FLOAT_CODES[cache.dtype]
    if cache.dtype == torch.int8:
        return PA_INT8
    if cache.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PA_FP8E4M3
    raise TypeError(f"unsupported cache dtype {cache.dtype}")


# ----------------------------------------------------------------------------------

def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, *, cache_dtype=None,
                      k_scale=None, v_scale=None, err_flag=None, stream=None) -> None:
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    rc = lib().pa_reshape_and_cache(
        _ptr(key), _ptr(value), _FLOAT_CODES[key.dtype], _ptr(k_cache), _ptr(v_cache),
        cache_code(k_cache, cache_dtype), _ptr(k_scale), _ptr(v_scale), _ptr(slot_mapping),
        key.shape[0], num_kv_heads, head_dim, block_size, num_blocks, _ptr(err_flag),
        _stream(stream))
    _check(rc, "pa_reshape_and_cache")


def copy_blocks(src_k, src_v, dst_k, dst_v, block_mapping, *, cache_dtype=None,
                src_k_scale=None, src_v_scale=None, dst_k_scale=None, dst_v_scale=None,
                err_flag=None, stream=None) -> None:
    """Copy whole blocks: row p of block_mapping (int64 [num_pairs, 2], on the device)
    makes destination block [p, 1] a copy of source block [p, 0].  Source and
    destination pools may be the same tensors (copy-on-write) or a device pool and a
    pinned host pool (swap out / swap in)."""
    nb_src, block_size, num_kv_heads, head_dim = src_k.shape
    if dst_k.shape[1:] != src_k.shape[1:] or dst_k.dtype != src_k.dtype:
        raise ValueError("source and destination pools must have the same block shape and dtype")
    for t in (src_k, src_v, dst_k, dst_v, src_k_scale, src_v_scale, dst_k_scale, dst_v_scale):
        if t is not None and not (t.is_cuda or t.is_pinned()):
            raise ValueError("pools must be CUDA tensors or pinned host tensors")
    if not block_mapping.is_cuda or block_mapping.dtype != torch.int64:
        raise ValueError("block_mapping must be an int64 CUDA tensor [num_pairs, 2]")
    rc = lib().pa_copy_blocks(
        _ptr(src_k), _ptr(src_v), _ptr(src_k_scale), _ptr(src_v_scale), nb_src,
        _ptr(dst_k), _ptr(dst_v), _ptr(dst_k_scale), _ptr(dst_v_scale), dst_k.shape[0],
        cache_code(src_k, cache_dtype), _ptr(block_mapping),
        block_mapping.shape[0] if block_mapping.numel() else 0, num_kv_heads, head_dim,
        block_size, _ptr(err_flag), _stream(stream))
    _check(rc, "pa_copy_blocks")


def decode_v1(q, k_cache, v_cache, block_tables, seq_lens, scale, *, out=None, cache_dtype=None,
              k_scale=None, v_scale=None, err_flag=None, stream=None) -> torch.Tensor:
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    if out is None:
        out = torch.empty_like(q)
    rc = lib().pa_decode_v1(
        _ptr(out), _ptr(q), _FLOAT_CODES[q.dtype], _ptr(k_cache), _ptr(v_cache),
        cache_code(k_cache, cache_dtype), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), num_seqs, num_heads, num_kv_heads, head_dim,
        block_size, num_blocks, float(scale), _ptr(err_flag), _stream(stream))
    _check(rc, "pa_decode_v1")
    return out


def append_decode_v1(q, key, value, slot_mapping, k_cache, v_cache, block_tables, seq_lens,
                     scale, *, out=None, cache_dtype=None, k_scale=None, v_scale=None,
                     err_flag=None, stream=None) -> torch.Tensor:
    """One decode step in one launch: writes each sequence's new token (key, value
    [num_seqs, num_kv_heads, head_dim] at slot_mapping [num_seqs]) into the cache and
    decodes over every cached token, the new one included."""
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    if out is None:
        out = torch.empty_like(q)
    if key.dtype != q.dtype or value.dtype != q.dtype:
        raise ValueError("key and value must have q's dtype")
    rc = lib().pa_append_decode_v1(
        _ptr(out), _ptr(q), _FLOAT_CODES[q.dtype], _ptr(key), _ptr(value), _ptr(slot_mapping),
        _ptr(k_cache), _ptr(v_cache), cache_code(k_cache, cache_dtype), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), num_seqs,
        num_heads, num_kv_heads, head_dim, block_size, num_blocks, float(scale), _ptr(err_flag),
        _stream(stream))
    _check(rc, "pa_append_decode_v1")
    return out


def prefill(q, k_cache, v_cache, block_tables, seq_lens, query_start, scale, *,
            max_query_len=None, out=None, err_flag=None, stream=None) -> torch.Tensor:
    """Causal multi-token query: rows [query_start[s], query_start[s+1]) of q are the last
    tokens of sequence s, already in the cache; returns out [total_q, H, D]."""
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    total_q, num_heads, _ = q.shape
    if max_query_len is None:
        max_query_len = int((query_start[1:] - query_start[:-1]).max()) if query_start.numel() > 1 else 0
    if out is None:
        out = torch.empty_like(q)
    rc = lib().pa_prefill(
        _ptr(out), _ptr(q), _FLOAT_CODES[q.dtype], _ptr(query_start), total_q, int(max_query_len),
        _ptr(k_cache), _ptr(v_cache), cache_code(k_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), seq_lens.shape[0], num_heads, num_kv_heads,
        head_dim, block_size, num_blocks, float(scale), _ptr(err_flag), _stream(stream))
    _check(rc, "pa_prefill")
    return out


def decode_cascade(q, k_cache, v_cache, block_tables, seq_lens, scale, prefix_len, *,
                   out=None, workspace=None, err_flag=None, stream=None) -> torch.Tensor:
    """pa_decode_v1 for sequences that share their first prefix_len tokens (the same
    blocks): the prefix on the tensor cores once per kv head, each sequence's own tokens
    on the persistent decode, the partials merged.  A caller-provided workspace must be
    zero-filled before its first use."""
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    if out is None:
        out = torch.empty_like(q)
    need = lib().pa_decode_cascade_workspace_bytes(num_seqs, num_heads, head_dim)
    if workspace is None:       # zero-filled once; every complete call leaves it that way
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=q.device)
    rc = lib().pa_decode_cascade(
        _ptr(out), _ptr(q), _FLOAT_CODES[q.dtype], _ptr(k_cache), _ptr(v_cache),
        cache_code(k_cache), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), num_seqs,
        num_heads, num_kv_heads, head_dim, block_size, num_blocks, float(scale), int(prefix_len),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(err_flag),
        _stream(stream))
    _check(rc, "pa_decode_cascade")
    return out


def decode_v2_partition(q, k_cache, v_cache, block_tables, seq_lens, scale, partition_size,
                        tmp_out, max_logits, exp_sums, *, cache_dtype=None, k_scale=None,
                        v_scale=None, err_flag=None, stream=None) -> None:
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    max_parts = tmp_out.shape[2]
    rc = lib().pa_decode_v2_partition(
        _ptr(tmp_out), _ptr(max_logits), _ptr(exp_sums), _ptr(q), _FLOAT_CODES[q.dtype],
        _ptr(k_cache), _ptr(v_cache), cache_code(k_cache, cache_dtype), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), num_seqs,
        num_heads, num_kv_heads, head_dim, block_size, num_blocks, float(scale),
        int(partition_size), max_parts, _ptr(err_flag), _stream(stream))
    _check(rc, "pa_decode_v2_partition")


def decode_v2_merge(out, tmp_out, max_logits, exp_sums, seq_lens, partition_size, *,
                    stream=None) -> None:
    num_seqs, num_heads, max_parts, head_dim = tmp_out.shape
    rc = lib().pa_decode_v2_merge(
        _ptr(out), _FLOAT_CODES[out.dtype], _ptr(tmp_out), _ptr(max_logits), _ptr(exp_sums),
        _ptr(seq_lens), num_seqs, num_heads, head_dim, int(partition_size), max_parts,
        _stream(stream))
    _check(rc, "pa_decode_v2_merge")


class V2Workspace:
    """tmp_out / max_logits / exp_sums for pa_decode_v2_partition, allocated by torch."""

    def __init__(self, num_seqs, num_heads, head_dim, max_parts, device="cuda"):
        self.tmp_out = torch.empty((num_seqs, num_heads, max_parts, head_dim),
                                   dtype=torch.float32, device=device)
        self.max_logits = torch.empty((num_seqs, num_heads, max_parts), dtype=torch.float32,
                                      device=device)
        self.exp_sums = torch.empty_like(self.max_logits)
        self.max_parts = max_parts


def decode_v2(q, k_cache, v_cache, block_tables, seq_lens, scale, *, max_seq_len=None,
              partition_size=None, out=None, workspace: V2Workspace | None = None,
              cache_dtype=None, k_scale=None, v_scale=None, err_flag=None,
              stream=None) -> torch.Tensor:
    """Partition step then merge.  ``max_seq_len`` (if not given) is read from
    ``block_tables``' capacity, which never needs a device->host copy."""
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    if max_seq_len is None:
        max_seq_len = block_tables.shape[1] * block_size
    if partition_size is None:
        partition_size = choose_partition_size(max_seq_len, num_seqs, num_kv_heads,
                                               block_size=block_size)
    max_parts = max(1, -(-max_seq_len // partition_size))
    if workspace is None or workspace.max_parts < max_parts:
        workspace = V2Workspace(num_seqs, num_heads, head_dim, max_parts, q.device)
    if out is None:
        out = torch.empty_like(q)
    decode_v2_partition(q, k_cache, v_cache, block_tables, seq_lens, scale, partition_size,
                        workspace.tmp_out, workspace.max_logits, workspace.exp_sums,
                        cache_dtype=cache_dtype, k_scale=k_scale, v_scale=v_scale,
                        err_flag=err_flag, stream=stream)
    decode_v2_merge(out, workspace.tmp_out, workspace.max_logits, workspace.exp_sums, seq_lens,
                    partition_size, stream=stream)
    return out


class FusedWorkspace:
    """Workspace of pa_decode_fused (arrival counters + partial records), zeroed once;
    the kernel leaves the counters at zero after every complete call."""

    def __init__(self, num_seqs, num_kv_heads, head_dim, device="cuda"):
        dev = torch.device(device)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.nbytes = int(lib().pa_decode_fused_workspace_bytes(num_seqs, num_kv_heads,
                                                               head_dim, sms))
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=dev)
        self.num_seqs, self.num_kv_heads, self.head_dim = num_seqs, num_kv_heads, head_dim

    def fits(self, num_seqs, num_kv_heads, head_dim) -> bool:
        return (num_seqs <= self.num_seqs and num_kv_heads == self.num_kv_heads
                and head_dim == self.head_dim)

    def counters(self) -> torch.Tensor:
        return self.buf[: self.num_seqs * self.num_kv_heads * 4].view(torch.int32)


def decode_fused(q, k_cache, v_cache, block_tables, seq_lens, scale, *, out=None,
                 workspace: FusedWorkspace | None = None, cache_dtype=None, k_scale=None,
                 v_scale=None, err_flag=None, stream=None) -> torch.Tensor:
    """Single-launch persistent decode (pa_decode_fused)."""
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    if workspace is None or not workspace.fits(num_seqs, num_kv_heads, head_dim):
        workspace = FusedWorkspace(num_seqs, num_kv_heads, head_dim, q.device)
    if out is None:
        out = torch.empty_like(q)
    rc = lib().pa_decode_fused(
        _ptr(out), _ptr(q), _FLOAT_CODES[q.dtype], _ptr(k_cache), _ptr(v_cache),
        cache_code(k_cache, cache_dtype), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), num_seqs, num_heads, num_kv_heads, head_dim,
        block_size, num_blocks, float(scale), _ptr(workspace.buf), workspace.nbytes,
        _ptr(err_flag), _stream(stream))
    _check(rc, "pa_decode_fused")
    return out


def decode_fused_noalloc(q, k_cache, v_cache, block_tables, seq_lens, scale, out, *,
                         cache_dtype=None, k_scale=None, v_scale=None, err_flag=None,
                         stream=None) -> torch.Tensor:
    """pa_decode_fused on the library's fixed scratch array: the caller passes only
    inputs and the output, nothing is allocated.  Calls must not overlap on the GPU."""
    num_blocks, block_size, num_kv_heads, head_dim = k_cache.shape
    num_seqs, num_heads, _ = q.shape
    rc = lib().pa_decode_fused_noalloc(
        _ptr(out), _ptr(q), _FLOAT_CODES[q.dtype], _ptr(k_cache), _ptr(v_cache),
        cache_code(k_cache, cache_dtype), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), num_seqs, num_heads, num_kv_heads, head_dim,
        block_size, num_blocks, float(scale), _ptr(err_flag), _stream(stream))
    _check(rc, "pa_decode_fused_noalloc")
    return out


def pick_decode_variant(num_seqs, num_kv_heads, max_seq_len, num_sms=None) -> str:
    """'v1' when one CTA per (sequence, kv head) already fills the GPU with short units
    (it needs no merge), else 'fused' (balances long or few sequences over every SM)."""
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    units = num_seqs * num_kv_heads
    tiles_per_unit = -(-int(max_seq_len) // 16)
    return "v1" if units >= num_sms and tiles_per_unit <= 256 else "fused"


def choose_partition_size(max_seq_len, num_seqs, num_kv_heads, num_sms=None, block_size=16) -> int:
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(lib().pa_choose_partition_size(int(max_seq_len), int(num_seqs), int(num_kv_heads),
                                              int(num_sms), int(block_size)))


def workspace_bytes(num_seqs, num_heads, head_dim, max_parts) -> int:
    return int(lib().pa_decode_v2_workspace_bytes(num_seqs, num_heads, head_dim, max_parts))


def kv_bytes_per_token(num_layers, num_kv_heads, head_dim, dtype_bytes) -> float:
    return float(lib().pa_kv_bytes_per_token(num_layers, num_kv_heads, head_dim, dtype_bytes))


def get_device_error(clear: bool = True) -> int:
    v = ctypes.c_int(0)
    _check(lib().pa_get_device_error(ctypes.byref(v), int(clear)), "pa_get_device_error")
    return v.value


def set_decode_config(warps: int = 0, stages: int = 0) -> None:
    _check(lib().pa_set_decode_config(int(warps), int(stages)), "pa_set_decode_config")


def set_prefetch_tiles(tiles_per_warp: int = -1) -> None:
    """L2 prefetch depth per decode warp before the PDL wait (PDL mode 2); -1 = default."""
    _check(lib().pa_set_prefetch_tiles(int(tiles_per_warp)), "pa_set_prefetch_tiles")


def set_wait_limit_ns(limit_ns: int = 0) -> None:
    """Per-wait time limit inside the decode kernels (0: the default, 2 s)."""
    _check(lib().pa_set_wait_limit_ns(int(limit_ns)), "pa_set_wait_limit_ns")


def set_cascade_config(prefix_splits: int = 0, suffix_form: int = 0) -> None:
    """pa_decode_cascade knobs: KV splits of the prefix launch (1..4; 0 = automatic
    placement; -1 = side by side with the suffix whenever it fits) and the suffix form
    (0 persistent decode + merge, 1 v1 decode merging in its epilogue)."""
    _check(lib().pa_set_cascade_config(int(prefix_splits), int(suffix_form)),
           "pa_set_cascade_config")


def set_pdl(mode: int = 1) -> None:
    """Programmatic dependent launch mode (0 off, 1 default, 2 early table reads)."""
    _check(lib().pa_set_pdl(int(mode)), "pa_set_pdl")


def set_fault_injection(mode: int = 0) -> None:
    """Test hook: mode 1 withholds each decode warp's first stage so its bounded
    wait runs out (reported as DEVERR_TIMEOUT); 0 turns it off."""
    _check(lib().pa_set_fault_injection(int(mode)), "pa_set_fault_injection")
