"""Seeded synthetic inputs for paged decode attention.

This module is shared by the tests, the bench and the oracle-side checks.  It
draws random numbers and lays out the host-side bookkeeping a block manager
would produce (a free pool of physical block ids, per-sequence block tables,
the slot each new token is written to).  It holds none of the method's
arithmetic: no attention, no quantisation and no cache write -- each side
performs those with its own code on the rows and slots returned here.

Workloads (all values N(0, 1), tables padded with -1, caches poisoned so a
stray read shows up):

* ``tiny_f32``      4 seqs, 4 q / 4 kv heads, head_dim 64, block 16, 64 blocks,
                    len ~ U{1..100}, scale 1/8, fp32.
* ``qwen3_32b_f16`` one Qwen3-32B layer: 32 seqs, 64 q / 8 kv heads, head_dim
                    128, block 16, a 12480-block pool (the pool the vllm-musa
                    lesson logs, §3.2), len ~ U{512..768}, scale 1/sqrt(128).
* ``long_ctx_bf16`` 8 seqs x 32768 tokens, 64 / 8 heads, head_dim 128, block 16,
                    16384-block pool, bf16, partition 512.
* ``quant_int8`` / ``quant_fp8``  the qwen3_32b shapes with fp16 K/V rows to be
                    quantised into an INT8 or FP8 E4M3 cache by the cache write.
* ``mixed_f16``     256 seqs; private length clamp(round(lognormal(ln 600, 1)),
                    1, 8192) after an 8192-token prefix shared by every table.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

FLOAT_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
CACHE_STORAGE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16,
                 "int8": torch.int8, "fp8": torch.uint8}
CACHE_ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "int8": 1, "fp8": 1}


@dataclass
class Workload:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: str                      # q / new-row / output dtype
    cache_dtype: str                # f32 | f16 | bf16 | int8 | fp8
    scale: float
    lens: str                       # length distribution tag
    len_lo: int = 0
    len_hi: int = 0
    shared_prefix_tokens: int = 0
    partition_size: int = 0         # 0: let the library choose


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 4, 4, 4, 64, 16, 64, "f32", "f32", 1.0 / 8,
                         "uniform", 1, 100),
    "qwen3_32b_f16": Workload("qwen3_32b_f16", 32, 64, 8, 128, 16, 12480, "f16", "f16",
                              1.0 / math.sqrt(128), "uniform", 512, 768),
    "long_ctx_bf16": Workload("long_ctx_bf16", 8, 64, 8, 128, 16, 16384, "bf16", "bf16",
                              1.0 / math.sqrt(128), "fixed", 32768, 32768, partition_size=512),
    "quant_int8": Workload("quant_int8", 32, 64, 8, 128, 16, 12480, "f16", "int8",
                           1.0 / math.sqrt(128), "uniform", 512, 768),
    "quant_fp8": Workload("quant_fp8", 32, 64, 8, 128, 16, 12480, "f16", "fp8",
                          1.0 / math.sqrt(128), "uniform", 512, 768),
    "mixed_f16": Workload("mixed_f16", 256, 64, 8, 128, 16, 0, "f16", "f16",
                          1.0 / math.sqrt(128), "lognormal", 1, 8192,
                          shared_prefix_tokens=8192),
}


@dataclass
class Batch:
    """One decode step's per-sequence inputs over a shared block pool."""
    q: torch.Tensor                  # [S, H, D] dtype
    block_tables: torch.Tensor       # int32 [S, max_blocks], padding -1
    seq_lens: torch.Tensor           # int32 [S], length INCLUDING the new token
    new_key: torch.Tensor            # [S, H_kv, D] row of the token appended this step
    new_value: torch.Tensor
    new_slots: torch.Tensor          # int64 [S] slot of the appended token


@dataclass
class Problem:
    wl: Workload
    num_blocks: int
    k_cache: torch.Tensor            # [num_blocks, bs, H_kv, D] storage dtype, poisoned
    v_cache: torch.Tensor
    k_scale: torch.Tensor | None     # fp32 [num_blocks, H_kv, bs], poisoned with NaN
    v_scale: torch.Tensor | None
    hist_key: torch.Tensor           # [T_hist, H_kv, D] rows already in the cache
    hist_value: torch.Tensor
    hist_slots: torch.Tensor         # int64 [T_hist]
    batches: list[Batch] = field(default_factory=list)

    @property
    def batch(self) -> Batch:
        return self.batches[0]


class SeededBlockAllocator:
    """Free pool of physical block ids in a seeded random order; ``take(n)`` pops n ids.

    Tables are cut in order from one seeded permutation of the pool: the first
    ceil(len/bs) ids go to sequence 0, the next ones to sequence 1, and so on.

    Stands in for the host block manager (free list, pop on allocate) of the
    pages' BlockManager sketches; no reference counting or eviction.
    """

    def __init__(self, num_blocks: int, rng: np.random.Generator, shuffle: bool = True):
        ids = np.arange(num_blocks, dtype=np.int64)
        if shuffle:
            ids = rng.permutation(ids)
        self._free = list(ids.tolist())
        self.num_blocks = num_blocks

    def take(self, n: int) -> list[int]:
        if n > len(self._free):
            raise MemoryError(f"pool exhausted: need {n}, have {len(self._free)}")
        out, self._free = self._free[:n], self._free[n:]
        return out

    @property
    def num_free(self) -> int:
        return len(self._free)


def _draw_lengths(wl: Workload, rng: np.random.Generator, n: int) -> np.ndarray:
    if wl.lens == "uniform":
        return rng.integers(wl.len_lo, wl.len_hi + 1, size=n)
    if wl.lens == "fixed":
        return np.full(n, wl.len_lo, dtype=np.int64)
    if wl.lens == "lognormal":
        priv = np.rint(rng.lognormal(mean=math.log(600.0), sigma=1.0, size=n))
        priv = np.clip(priv, wl.len_lo, wl.len_hi).astype(np.int64)
        return priv + wl.shared_prefix_tokens
    raise ValueError(wl.lens)


def _poison(storage: torch.dtype, shape) -> torch.Tensor:
    if storage.is_floating_point:
        return torch.full(shape, float("nan"), dtype=storage)
    if storage == torch.int8:
        return torch.full(shape, 127, dtype=storage)
    return torch.full(shape, 0x7F, dtype=storage)      # E4M3 NaN code


def _randn(gen: torch.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(dtype)


def make_problem(name: str, seed: int = 0, *, num_batches: int = 1,
                 block_size: int | None = None, num_seqs: int | None = None,
                 cache_dtype: str | None = None, dtype: str | None = None,
                 seq_lens: list[int] | None = None, num_blocks: int | None = None,
                 head_dim: int | None = None, num_heads: int | None = None,
                 num_kv_heads: int | None = None,
                 shared_prefix_tokens: int | None = None) -> Problem:
    """Build one seeded problem; keyword overrides give variants of a workload.

    ``num_batches`` independent batches share one pool (their blocks are
    disjoint, apart from a shared prefix), so a bench can rotate over inputs
    whose union is larger than L2.
    """
    base = WORKLOADS[name]
    wl = Workload(**{**base.__dict__})
    if block_size is not None:
        wl.block_size = block_size
    if num_seqs is not None:
        wl.num_seqs = num_seqs
    if cache_dtype is not None:
        wl.cache_dtype = cache_dtype
    if dtype is not None:
        wl.dtype = dtype
    if head_dim is not None:
        wl.head_dim = head_dim
    if num_heads is not None:
        wl.num_heads = num_heads
    if num_kv_heads is not None:
        wl.num_kv_heads = num_kv_heads
    if shared_prefix_tokens is not None:
        wl.shared_prefix_tokens = shared_prefix_tokens
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    S, H, Hkv, D, bs = wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size

    all_lens = []
    for _ in range(num_batches):
        lens = np.asarray(seq_lens if seq_lens is not None else _draw_lengths(wl, rng, S),
                          dtype=np.int64)
        assert lens.shape[0] == S and (lens >= 1).all()
        all_lens.append(lens)

    prefix_blocks = -(-wl.shared_prefix_tokens // bs) if wl.shared_prefix_tokens else 0
    need = prefix_blocks + sum(int(sum(-(-(int(n) - wl.shared_prefix_tokens) // bs)
                                       for n in lens)) for lens in all_lens)
    if num_blocks is not None:
        nb = num_blocks
    else:   # the workload's pool, holding the same number of tokens at any block size
        nb = wl.num_blocks * base.block_size // wl.block_size if wl.num_blocks else need
    if nb < need:
        raise ValueError(f"{name}: {need} blocks needed, pool has {nb}")
    alloc = SeededBlockAllocator(nb, rng)

    storage = CACHE_STORAGE[wl.cache_dtype]
    k_cache = _poison(storage, (nb, bs, Hkv, D))
    v_cache = _poison(storage, (nb, bs, Hkv, D))
    quant = wl.cache_dtype in ("int8", "fp8")
    k_scale = torch.full((nb, Hkv, bs), float("nan")) if quant else None
    v_scale = torch.full((nb, Hkv, bs), float("nan")) if quant else None
    row_dtype = FLOAT_DTYPES[wl.dtype]

    prefix_ids = alloc.take(prefix_blocks) if prefix_blocks else []
    hist_slots = []
    if prefix_blocks:
        for t in range(wl.shared_prefix_tokens):
            hist_slots.append(prefix_ids[t // bs] * bs + t % bs)

    batches = []
    for lens in all_lens:
        max_blocks = int(max(-(-int(n) // bs) for n in lens))
        tables = np.full((S, max_blocks), -1, dtype=np.int32)
        new_slots = np.zeros(S, dtype=np.int64)
        for s, n in enumerate(lens.tolist()):
            priv_tokens = n - wl.shared_prefix_tokens
            ids = prefix_ids + alloc.take(-(-priv_tokens // bs))
            tables[s, :len(ids)] = ids
            for t in range(wl.shared_prefix_tokens, n - 1):       # history rows
                hist_slots.append(ids[t // bs] * bs + t % bs)
            new_slots[s] = ids[(n - 1) // bs] * bs + (n - 1) % bs
        q = _randn(gen, (S, H, D), row_dtype)
        nk = _randn(gen, (S, Hkv, D), row_dtype)
        nv = _randn(gen, (S, Hkv, D), row_dtype)
        batches.append(Batch(q, torch.from_numpy(tables), torch.from_numpy(lens.astype(np.int32)),
                             nk, nv, torch.from_numpy(new_slots)))

    T = len(hist_slots)
    hist_key = _randn(gen, (T, Hkv, D), row_dtype)
    hist_value = _randn(gen, (T, Hkv, D), row_dtype)
    return Problem(wl, nb, k_cache, v_cache, k_scale, v_scale, hist_key, hist_value,
                   torch.tensor(hist_slots, dtype=torch.int64), batches)


def logical_kv_bytes(wl: Workload, seq_lens) -> int:
    """Bytes of K and V (and scales) a decode pass must read: exact tokens, not blocks."""
    tokens = int(np.asarray(seq_lens, dtype=np.int64).sum())
    per_tok = wl.num_kv_heads * wl.head_dim * 2 * CACHE_ELEM_BYTES[wl.cache_dtype]
    if wl.cache_dtype in ("int8", "fp8"):
        per_tok += wl.num_kv_heads * 2 * 4
    return tokens * per_tok


def unique_kv_bytes(wl: Workload, seq_lens) -> int:
    """Like ``logical_kv_bytes`` but a shared prefix counts once."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    tokens = int((lens - wl.shared_prefix_tokens).sum()) + (wl.shared_prefix_tokens if len(lens) else 0)
    per_tok = wl.num_kv_heads * wl.head_dim * 2 * CACHE_ELEM_BYTES[wl.cache_dtype]
    if wl.cache_dtype in ("int8", "fp8"):
        per_tok += wl.num_kv_heads * 2 * 4
    return tokens * per_tok


def qo_bytes(wl: Workload, num_seqs: int) -> int:
    """Bytes of q read and out written by one decode pass."""
    eb = {"f32": 4, "f16": 2, "bf16": 2}[wl.dtype]
    return 2 * num_seqs * wl.num_heads * wl.head_dim * eb
