"""Python binding of the host block manager in ``libpa.so`` (``include/pa_block_manager.h``).

Argument marshalling only; the allocator itself is C++ in the library.  Methods raise
``pa.PAError`` with the library's status (``PA_ERR_NO_SPACE`` when the pool is full,
``PA_ERR_INVALID_ARG`` for an unknown sequence); a failed call changes nothing.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import pa

_P, _I, _L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
_SIGS = {
    "pa_bm_create": (_P, [_I, _I, _I, _I]),
    "pa_bm_destroy": (None, [_P]),
    "pa_bm_free_gpu_blocks": (_I, [_P]),
    "pa_bm_free_cpu_blocks": (_I, [_P]),
    "pa_bm_add_sequence": (_I, [_P, _L, _P, _I, _P, _P]),
    "pa_bm_append_token": (_I, [_P, _L, ctypes.c_int32, _P, _P, _P]),
    "pa_bm_append_batch": (_I, [_P, _P, _P, _I, _P, _P, _P]),
    "pa_bm_fork": (_I, [_P, _L, _L]),
    "pa_bm_free_sequence": (_I, [_P, _L]),
    "pa_bm_swap_out": (_I, [_P, _P, _I, _P, _I, _P]),
    "pa_bm_swap_in": (_I, [_P, _P, _I, _P, _I, _P]),
    "pa_bm_block_table": (_I, [_P, _L, _P, _I, _P, _P]),
    "pa_bm_build_batch": (_I, [_P, _P, _I, _P, _I, _P]),
}
_ready = False


def _lib():
    global _ready
    L = pa.lib()
    if not _ready:
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _ready = True
    return L


def _arr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class BlockManager:
    """Allocator of physical KV blocks: block tables, slot mappings, copy-on-write and
    swap pairs (for ``pa.copy_blocks``), optional prefix caching."""

    def __init__(self, num_gpu_blocks: int, block_size: int = 16, num_cpu_blocks: int = 0,
                 prefix_caching: bool = False):
        self.block_size = block_size
        self._h = _lib().pa_bm_create(num_gpu_blocks, num_cpu_blocks, block_size,
                                      int(prefix_caching))
        if not self._h:
            raise ValueError("pa_bm_create failed (bad sizes or out of host memory)")

    def close(self):
        if self._h:
            _lib().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def free_gpu_blocks(self) -> int:
        return _lib().pa_bm_free_gpu_blocks(self._h)

    @property
    def free_cpu_blocks(self) -> int:
        return _lib().pa_bm_free_cpu_blocks(self._h)

    def add_sequence(self, seq_id: int, tokens):
        """Returns (slot_mapping int64 [n], num_cached)."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(len(t), dtype=np.int64)
        cached = ctypes.c_int(0)
        rc = _lib().pa_bm_add_sequence(self._h, seq_id, _arr(t), len(t), _arr(slots),
                                       ctypes.byref(cached))
        pa._check(rc, "pa_bm_add_sequence")
        return slots, cached.value

    def append_token(self, seq_id: int, token: int):
        """Returns (slot, cow_src, cow_dst); -1 when no copy is needed."""
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        rc = _lib().pa_bm_append_token(self._h, seq_id, token, ctypes.byref(slot),
                                       ctypes.byref(src), ctypes.byref(dst))
        pa._check(rc, "pa_bm_append_token")
        return slot.value, src.value, dst.value

    def append_batch(self, seq_ids, tokens):
        """Returns (slot_mapping int64 [n], cow_pairs int64 [k, 2])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(len(ids), dtype=np.int64)
        pairs = np.empty((max(1, len(ids)), 2), dtype=np.int64)
        k = ctypes.c_int(0)
        rc = _lib().pa_bm_append_batch(self._h, _arr(ids), _arr(tok), len(ids), _arr(slots),
                                       _arr(pairs), ctypes.byref(k))
        pa._check(rc, "pa_bm_append_batch")
        return slots, pairs[:k.value].copy()

    def fork(self, parent_id: int, child_id: int) -> None:
        pa._check(_lib().pa_bm_fork(self._h, parent_id, child_id), "pa_bm_fork")

    def free_sequence(self, seq_id: int) -> None:
        pa._check(_lib().pa_bm_free_sequence(self._h, seq_id), "pa_bm_free_sequence")

    def _swap(self, fn, seq_ids):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        cap = sum(self.block_table(i)[0].size for i in ids) or 1
        mapping = np.empty((cap, 2), dtype=np.int64)
        n = ctypes.c_int(0)
        rc = fn(self._h, _arr(ids), len(ids), _arr(mapping), cap, ctypes.byref(n))
        pa._check(rc, fn.__name__)
        return mapping[:n.value].copy()

    def swap_out(self, seq_ids):
        """Returns the (gpu block, cpu block) pairs to copy."""
        return self._swap(_lib().pa_bm_swap_out, seq_ids)

    def swap_in(self, seq_ids):
        """Returns the (cpu block, gpu block) pairs to copy."""
        return self._swap(_lib().pa_bm_swap_in, seq_ids)

    def block_table(self, seq_id: int):
        """Returns (block ids int32 [num_blocks], num_tokens)."""
        nb, nt = ctypes.c_int(-1), ctypes.c_int(0)
        rc = _lib().pa_bm_block_table(self._h, seq_id, None, 0, ctypes.byref(nb),
                                      ctypes.byref(nt))
        if nb.value < 0:                           # unknown sequence
            pa._check(rc, "pa_bm_block_table")
        table = np.empty(max(1, nb.value), dtype=np.int32)
        rc = _lib().pa_bm_block_table(self._h, seq_id, _arr(table), table.size,
                                      ctypes.byref(nb), ctypes.byref(nt))
        pa._check(rc, "pa_bm_block_table")
        return table[:nb.value].copy(), nt.value

    def build_batch(self, seq_ids, max_blocks: int | None = None):
        """Returns (block_tables int32 [n, max_blocks] padded with -1, seq_lens int32 [n])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        if max_blocks is None:
            max_blocks = max([self.block_table(i)[0].size for i in ids] + [1])
        tables = np.empty((len(ids), max_blocks), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        rc = _lib().pa_bm_build_batch(self._h, _arr(ids), len(ids), _arr(tables), max_blocks,
                                      _arr(lens))
        pa._check(rc, "pa_bm_build_batch")
        return tables, lens
