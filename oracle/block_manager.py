"""Oracle model of the host block manager -- TEST INFRASTRUCTURE ONLY.

A plain Python statement of the block manager the pages describe, used by the tests
to check the C++ block manager of the library step for step (same block ids, slots,
copy-on-write pairs and swap mappings).  Nothing in the product path imports it.

Pages (by title, then section):
  [KV量化]  "大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置", the
            BlockManager pseudo-code: free_blocks = list(range(num_blocks)), allocate()
            takes ceil(num_tokens / block_size) blocks, append_token() takes a new
            block when the last one is full, blocks come from free_blocks.pop().
  [深度解析] "LLM推理优化：vLLM PagedAttention深度解析与工程实践" §3.2 (free() gives
            the blocks back) and §4.2 (automatic prefix caching).
  [KVcache-learning] "KVcache-learning" s05 (copy-on-write of shared blocks), s06
            (allocation, copy-on-write, swap_out / swap_in, free), s08 (prefix cache:
            hash of a block's tokens -> physical block).

Readings of what the pages leave open or contradict:
  B1  Free list order: [KV量化] and s06 pop from the end of free_blocks, [深度解析] §3.2
      pops from the front.  Reading: the end (LIFO); freed blocks are appended.
  B2  The prefix-cache key: s08 hashes a block's own tokens, but a block's K/V depend on
      every token before it.  Reading: block i's key chains block i-1's key with block
      i's tokens; the key is FNV-1a 64 over the parent key (8 bytes, little endian)
      followed by the tokens (4 bytes each, little endian), starting from the FNV
      offset basis; a hit also compares the stored parent key and tokens.
  B3  Only full blocks are cached.  A prompt keeps its last token uncomputed: the
      cached prefix of an n-token prompt is at most n - 1 tokens, so if every block of
      the prompt hits, the last one is allocated afresh.
  B4  A cached block whose reference count falls to 0 stays cached (evictable); a new
      block comes from the free list first, then the evictable block freed longest ago
      (its key is dropped).
  B5  Copy-on-write happens on append: if the sequence's last block is partly filled
      and shared, the token goes to a fresh block and (old, fresh) is returned for the
      caller to copy ([KVcache-learning] s05/s06).
  B6  free() releases a sequence's blocks in table order.  swap_out / swap_in move a
      group of sequences: each distinct block moves once, and blocks shared inside
      the group stay shared on the other side.  All checks happen before any change: a
      call that lacks space changes nothing.
"""
from __future__ import annotations

FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3
MASK64 = (1 << 64) - 1


class NoSpace(Exception):
    pass


def fnv1a64(data: bytes) -> int:
    """FNV-1a, 64-bit: for each byte, xor it in, then multiply by the FNV prime."""
    h = FNV_OFFSET
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & MASK64
    return h


def block_key(parent: int, tokens) -> int:
    """FNV-1a 64 over parent (8 bytes LE) then each token (4 bytes LE, two's complement)."""
    return fnv1a64(parent.to_bytes(8, "little") + b"".join(
        (t & 0xFFFFFFFF).to_bytes(4, "little") for t in tokens))


class Pool:
    def __init__(self, n: int):
        self.free = list(range(n))
        self.ref = [0] * n


class BlockManagerModel:
    def __init__(self, num_gpu_blocks: int, num_cpu_blocks: int, block_size: int,
                 prefix_caching: bool):
        self.bs = block_size
        self.gpu = Pool(num_gpu_blocks)
        self.cpu = Pool(num_cpu_blocks)
        self.prefix = prefix_caching
        self.seqs = {}            # id -> dict(blocks, tokens, on_gpu)
        self.key_of = {}          # gpu block -> (key, parent, tokens) while cached
        self.by_key = {}          # key -> gpu block
        self.evictable = []       # cached gpu blocks with ref 0, oldest first

    # ---------------------------------------------------------------- blocks
    def free_gpu_blocks(self) -> int:
        return len(self.gpu.free) + len(self.evictable)

    def free_cpu_blocks(self) -> int:
        return len(self.cpu.free)

    def _take_gpu(self) -> int:
        if self.gpu.free:
            b = self.gpu.free.pop()
        elif self.evictable:
            b = self.evictable.pop(0)
            key = self.key_of.pop(b)[0]
            del self.by_key[key]
        else:
            raise NoSpace
        self.gpu.ref[b] = 1
        return b

    def _release_gpu(self, b: int) -> None:
        self.gpu.ref[b] -= 1
        if self.gpu.ref[b] == 0:
            if b in self.key_of:
                self.evictable.append(b)
            else:
                self.gpu.free.append(b)

    def _release_cpu(self, b: int) -> None:
        self.cpu.ref[b] -= 1
        if self.cpu.ref[b] == 0:
            self.cpu.free.append(b)

    def _register(self, b: int, parent: int, tokens) -> int:
        key = block_key(parent, tokens)
        if key not in self.by_key:
            self.by_key[key] = b
            self.key_of[b] = (key, parent, tuple(tokens))
        return key

    def _lookup(self, parent: int, tokens):
        key = block_key(parent, tokens)
        b = self.by_key.get(key)
        if b is None:
            return None, key
        _, p, t = self.key_of[b]
        if p != parent or t != tuple(tokens):
            return None, key
        return b, key

    # ---------------------------------------------------------------- sequences
    def add_sequence(self, seq_id: int, tokens):
        """Returns (slot_mapping, num_cached); raises NoSpace (nothing changed)."""
        if seq_id in self.seqs or len(tokens) == 0:
            raise ValueError("bad sequence")
        bs, n = self.bs, len(tokens)
        nblocks = -(-n // bs)
        hits, parent = [], FNV_OFFSET
        if self.prefix:
            for i in range((n - 1) // bs):         # full blocks wholly before the last token
                b, key = self._lookup(parent, tokens[i * bs:(i + 1) * bs])
                if b is None:
                    break
                hits.append(b)
                parent = key
        revived = sum(1 for b in hits if self.gpu.ref[b] == 0)
        if len(self.gpu.free) + len(self.evictable) - revived < nblocks - len(hits):
            raise NoSpace
        for b in hits:
            if self.gpu.ref[b] == 0:
                self.evictable.remove(b)
            self.gpu.ref[b] += 1
        blocks = list(hits)
        for i in range(len(hits), nblocks):
            b = self._take_gpu()
            blocks.append(b)
            if self.prefix and (i + 1) * bs <= n:
                parent = self._register(b, parent, tokens[i * bs:(i + 1) * bs])
        cached = len(hits) * bs
        slots = [-1 if t < cached else blocks[t // bs] * bs + t % bs for t in range(n)]
        self.seqs[seq_id] = dict(blocks=blocks, tokens=list(tokens), on_gpu=True)
        return slots, cached

    def append_token(self, seq_id: int, token: int):
        """Returns (slot, cow_src, cow_dst) with -1 for no copy; raises NoSpace."""
        s = self._gpu_seq(seq_id)
        bs, n = self.bs, len(s["tokens"])
        src = dst = -1
        if n % bs == 0:
            b = self._take_gpu()
            s["blocks"].append(b)
        else:
            b = s["blocks"][-1]
            if self.gpu.ref[b] > 1:
                nb = self._take_gpu()
                self.gpu.ref[b] -= 1
                s["blocks"][-1] = nb
                src, dst, b = b, nb, nb
        s["tokens"].append(token)
        if self.prefix and (n + 1) % bs == 0:
            i = n // bs
            parent = self._chain_key(s["tokens"], i)
            self._register(b, parent, s["tokens"][i * bs:(i + 1) * bs])
        return b * bs + n % bs, src, dst

    def append_batch(self, seq_ids, tokens):
        """One decode step: returns (slots, cow pairs).  The space check counts a block
        for every sequence whose last block is full or shared before any append."""
        if len(set(seq_ids)) != len(seq_ids):
            raise ValueError("duplicate sequence")
        seqs = [self._gpu_seq(i) for i in seq_ids]
        need = sum(1 for s in seqs
                   if len(s["tokens"]) % self.bs == 0 or self.gpu.ref[s["blocks"][-1]] > 1)
        if self.free_gpu_blocks() < need:
            raise NoSpace
        slots, pairs = [], []
        for i, t in zip(seq_ids, tokens):
            slot, src, dst = self.append_token(i, t)
            slots.append(slot)
            if src >= 0:
                pairs.append((src, dst))
        return slots, pairs

    def _chain_key(self, tokens, i):
        parent = FNV_OFFSET
        for j in range(i):
            parent = block_key(parent, tokens[j * self.bs:(j + 1) * self.bs])
        return parent

    def fork(self, parent_id: int, child_id: int) -> None:
        p = self._gpu_seq(parent_id)
        if child_id in self.seqs:
            raise ValueError("child exists")
        for b in p["blocks"]:
            self.gpu.ref[b] += 1
        self.seqs[child_id] = dict(blocks=list(p["blocks"]), tokens=list(p["tokens"]),
                                   on_gpu=True)

    def free_sequence(self, seq_id: int) -> None:
        if seq_id not in self.seqs:
            raise ValueError("unknown sequence")
        s = self.seqs.pop(seq_id)
        for b in s["blocks"]:
            (self._release_gpu if s["on_gpu"] else self._release_cpu)(b)

    def _gpu_seq(self, seq_id):
        s = self.seqs.get(seq_id)
        if s is None:
            raise ValueError("unknown sequence")
        if not s["on_gpu"]:
            raise ValueError("sequence is swapped out")
        return s

    def swap_out(self, seq_ids):
        """Returns [(gpu block, cpu block)] in first-seen order; raises NoSpace."""
        return self._swap(seq_ids, to_cpu=True)

    def swap_in(self, seq_ids):
        """Returns [(cpu block, gpu block)] in first-seen order; raises NoSpace."""
        return self._swap(seq_ids, to_cpu=False)

    def _swap(self, seq_ids, to_cpu):
        if any(i not in self.seqs for i in seq_ids):
            raise ValueError("unknown sequence")
        seqs = [self.seqs[i] for i in seq_ids]
        if len(set(seq_ids)) != len(seq_ids) or any(s["on_gpu"] != to_cpu for s in seqs):
            raise ValueError("bad swap group")
        distinct = list(dict.fromkeys(b for s in seqs for b in s["blocks"]))
        room = len(self.cpu.free) if to_cpu else self.free_gpu_blocks()
        if room < len(distinct):
            raise NoSpace
        mapping = {}
        for s in seqs:
            moved = []
            for b in s["blocks"]:
                if b in mapping:
                    nb = mapping[b]
                    (self.cpu if to_cpu else self.gpu).ref[nb] += 1
                else:
                    if to_cpu:
                        nb = self.cpu.free.pop()
                        self.cpu.ref[nb] = 1
                    else:
                        nb = self._take_gpu()
                    mapping[b] = nb
                moved.append(nb)
                (self._release_gpu if to_cpu else self._release_cpu)(b)
            s["blocks"] = moved
            s["on_gpu"] = not to_cpu
        return list(mapping.items())

    # ---------------------------------------------------------------- views
    def block_table(self, seq_id):
        if seq_id not in self.seqs:
            raise ValueError("unknown sequence")
        s = self.seqs[seq_id]
        return list(s["blocks"]), len(s["tokens"])
