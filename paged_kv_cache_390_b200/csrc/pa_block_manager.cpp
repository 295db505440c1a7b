// pa_block_manager.cpp -- the host block manager: the allocator that hands out
// the physical blocks the kernels read through block_tables and write through
// slot_mapping.
//
// What it does follows the pages' block manager: a free list of block ids
// taken from its end and given back at its end ("大模型推理优化实战：KV Cache
// 量化与PagedAttention显存管理配置", BlockManager; "KVcache-learning" s06),
// ceil(tokens / block_size) blocks per sequence and a new block only when the
// last one is full (append_token), reference counts so that forked sequences
// share blocks, copy-on-write of a shared, partly filled last block before a
// token is appended ("KVcache-learning" s05/s06), swap of sequences between the
// GPU pool and a CPU pool (s06 swap_out / swap_in), and automatic prefix
// caching ("LLM推理优化：vLLM PagedAttention深度解析与工程实践" §4.2;
// "KVcache-learning" s08): full blocks are indexed by a key that chains the
// previous block's key with the block's tokens (FNV-1a, 64 bit), a new prompt
// reuses the cached blocks its prefix matches, and a cached block whose last
// user leaves stays cached (evictable) until a block is needed and the free
// list is empty, oldest first.
//
// Every call checks its preconditions first: a call that fails (unknown
// sequence, not enough free blocks, output buffer too small) changes nothing.
// One manager is not thread-safe: calls on it must not overlap.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"
#include "pa_block_manager.h"

namespace {

constexpr uint64_t kFnvOffset = 0xCBF29CE484222325ull;
constexpr uint64_t kFnvPrime = 0x100000001B3ull;

uint64_t fnv_bytes(uint64_t h, const unsigned char* p, size_t n) {
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= kFnvPrime;
  }
  return h;
}

// Key of a full block: FNV-1a over the parent key (8 bytes, little endian) and
// the block's tokens (4 bytes each, little endian).
uint64_t block_key(uint64_t parent, const int32_t* tokens, int n) {
  unsigned char b[8];
  for (int i = 0; i < 8; ++i) b[i] = static_cast<unsigned char>(parent >> (8 * i));
  uint64_t h = fnv_bytes(kFnvOffset, b, 8);
  for (int t = 0; t < n; ++t) {
    const uint32_t v = static_cast<uint32_t>(tokens[t]);
    for (int i = 0; i < 4; ++i) b[i] = static_cast<unsigned char>(v >> (8 * i));
    h = fnv_bytes(h, b, 4);
  }
  return h;
}

struct Pool {
  std::vector<int32_t> free_ids;   // taken from and given back at the end
  std::vector<int32_t> ref;
  explicit Pool(int n) : ref(n, 0) {
    free_ids.reserve(n);
    for (int i = 0; i < n; ++i) free_ids.push_back(i);
  }
};

struct Seq {
  std::vector<int32_t> blocks;
  std::vector<int32_t> tokens;
  bool on_gpu = true;
  uint64_t chain = 0;   // prefix caching: the key of the sequence's last full block
};

struct Cached {
  bool valid = false;
  uint64_t key = 0, parent = 0;
  std::vector<int32_t> tokens;
  bool evictable = false;
  std::list<int32_t>::iterator pos;
};

}  // namespace

struct pa_block_manager {
  int bs;
  bool prefix;
  Pool gpu, cpu;
  std::unordered_map<int64_t, Seq> seqs;
  std::vector<Cached> cached;                    // per GPU block
  std::unordered_map<uint64_t, int32_t> by_key;
  std::list<int32_t> evictable;                  // oldest first

  pa_block_manager(int g, int c, int block_size, bool prefix_caching)
      : bs(block_size), prefix(prefix_caching), gpu(g), cpu(c), cached(g) {}

  int free_gpu() const { return static_cast<int>(gpu.free_ids.size() + evictable.size()); }

  int32_t take_gpu() {                           // caller has checked there is room
    int32_t b;
    if (!gpu.free_ids.empty()) {
      b = gpu.free_ids.back();
      gpu.free_ids.pop_back();
    } else {
      b = evictable.front();
      evictable.pop_front();
      Cached& c = cached[b];
      by_key.erase(c.key);
      c = Cached{};
    }
    gpu.ref[b] = 1;
    return b;
  }

  void release_gpu(int32_t b) {
    if (--gpu.ref[b] == 0) {
      Cached& c = cached[b];
      if (c.valid) {
        c.evictable = true;
        c.pos = evictable.insert(evictable.end(), b);
      } else {
        gpu.free_ids.push_back(b);
      }
    }
  }

  void release_cpu(int32_t b) {
    if (--cpu.ref[b] == 0) cpu.free_ids.push_back(b);
  }

  uint64_t register_block(int32_t b, uint64_t parent, const int32_t* toks) {
    const uint64_t key = block_key(parent, toks, bs);
    if (by_key.find(key) == by_key.end()) {
      by_key.emplace(key, b);
      Cached& c = cached[b];
      c.valid = true;
      c.key = key;
      c.parent = parent;
      c.tokens.assign(toks, toks + bs);
    }
    return key;
  }

  // The cached block for (parent, tokens), or -1.
  int32_t lookup(uint64_t parent, const int32_t* toks, uint64_t* key_out) const {
    const uint64_t key = block_key(parent, toks, bs);
    *key_out = key;
    auto it = by_key.find(key);
    if (it == by_key.end()) return -1;
    const Cached& c = cached[it->second];
    if (c.parent != parent || std::memcmp(c.tokens.data(), toks, sizeof(int32_t) * bs) != 0)
      return -1;
    return it->second;
  }

};

extern "C" {

PA_API pa_block_manager* pa_bm_create(int num_gpu_blocks, int num_cpu_blocks, int block_size,
                                      int prefix_caching) {
  if (num_gpu_blocks <= 0 || num_cpu_blocks < 0 || block_size <= 0) return nullptr;
  return new (std::nothrow) pa_block_manager(num_gpu_blocks, num_cpu_blocks, block_size,
                                             prefix_caching != 0);
}

PA_API void pa_bm_destroy(pa_block_manager* m) { delete m; }

PA_API int pa_bm_free_gpu_blocks(const pa_block_manager* m) { return m ? m->free_gpu() : -1; }

PA_API int pa_bm_free_cpu_blocks(const pa_block_manager* m) {
  return m ? static_cast<int>(m->cpu.free_ids.size()) : -1;
}

PA_API int pa_bm_add_sequence(pa_block_manager* m, int64_t seq_id, const int32_t* tokens,
                              int num_tokens, int64_t* slot_mapping, int* num_cached) {
  if (!m || !tokens || num_tokens <= 0 || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (m->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  const int bs = m->bs, n = num_tokens;
  const int nblocks = (n + bs - 1) / bs;
  std::vector<int32_t> hits;
  uint64_t parent = kFnvOffset;
  if (m->prefix) {
    for (int i = 0; i < (n - 1) / bs; ++i) {     // full blocks wholly before the last token
      uint64_t key;
      const int32_t b = m->lookup(parent, tokens + i * bs, &key);
      if (b < 0) break;
      hits.push_back(b);
      parent = key;
    }
  }
  int revived = 0;
  for (int32_t b : hits) revived += m->gpu.ref[b] == 0;
  if (m->free_gpu() - revived < nblocks - static_cast<int>(hits.size())) return PA_ERR_NO_SPACE;
  for (int32_t b : hits) {
    Cached& c = m->cached[b];
    if (m->gpu.ref[b] == 0 && c.evictable) {
      m->evictable.erase(c.pos);
      c.evictable = false;
    }
    ++m->gpu.ref[b];
  }
  Seq s;
  s.blocks = hits;
  for (int i = static_cast<int>(hits.size()); i < nblocks; ++i) {
    const int32_t b = m->take_gpu();
    s.blocks.push_back(b);
    if (m->prefix && (i + 1) * bs <= n) parent = m->register_block(b, parent, tokens + i * bs);
  }
  const int cached = static_cast<int>(hits.size()) * bs;
  for (int t = 0; t < n; ++t)
    slot_mapping[t] = t < cached ? -1 : static_cast<int64_t>(s.blocks[t / bs]) * bs + t % bs;
  s.tokens.assign(tokens, tokens + n);
  s.chain = parent;                              // every full block is registered or a hit
  m->seqs.emplace(seq_id, std::move(s));
  if (num_cached) *num_cached = cached;
  return PA_OK;
}

PA_API int pa_bm_append_token(pa_block_manager* m, int64_t seq_id, int32_t token, int64_t* slot,
                              int64_t* cow_src, int64_t* cow_dst) {
  if (!m || !slot) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end() || !it->second.on_gpu) return PA_ERR_INVALID_ARG;
  Seq& s = it->second;
  const int bs = m->bs;
  const int n = static_cast<int>(s.tokens.size());
  int64_t src = -1, dst = -1;
  int32_t b;
  if (n % bs == 0) {
    if (m->free_gpu() < 1) return PA_ERR_NO_SPACE;
    b = m->take_gpu();
    s.blocks.push_back(b);
  } else {
    b = s.blocks.back();
    if (m->gpu.ref[b] > 1) {                     // shared, partly filled: copy on write
      if (m->free_gpu() < 1) return PA_ERR_NO_SPACE;
      const int32_t nb = m->take_gpu();
      --m->gpu.ref[b];
      s.blocks.back() = nb;
      src = b;
      dst = nb;
      b = nb;
    }
  }
  s.tokens.push_back(token);
  if (m->prefix && (n + 1) % bs == 0)          // block n / bs is full: key it off the chain
    s.chain = m->register_block(b, s.chain, s.tokens.data() + (n / bs) * bs);
  *slot = static_cast<int64_t>(b) * bs + n % bs;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_OK;
}

PA_API int pa_bm_fork(pa_block_manager* m, int64_t parent_id, int64_t child_id) {
  if (!m) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(parent_id);
  if (it == m->seqs.end() || !it->second.on_gpu || m->seqs.count(child_id))
    return PA_ERR_INVALID_ARG;
  for (int32_t b : it->second.blocks) ++m->gpu.ref[b];
  Seq child = it->second;
  m->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

PA_API int pa_bm_free_sequence(pa_block_manager* m, int64_t seq_id) {
  if (!m) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
  for (int32_t b : it->second.blocks) {
    if (it->second.on_gpu) m->release_gpu(b);
    else m->release_cpu(b);
  }
  m->seqs.erase(it);
  return PA_OK;
}

namespace {

int swap_group(pa_block_manager* m, const int64_t* seq_ids, int n, int64_t* mapping, int capacity,
               int* num_pairs, bool to_cpu) {
  if (!m || n < 0 || (n > 0 && !seq_ids) || !num_pairs || capacity < 0) return PA_ERR_INVALID_ARG;
  std::vector<Seq*> group;
  for (int i = 0; i < n; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end() || it->second.on_gpu != to_cpu) return PA_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (seq_ids[j] == seq_ids[i]) return PA_ERR_INVALID_ARG;
    group.push_back(&it->second);
  }
  std::vector<int32_t> order;                    // distinct blocks, first-seen order
  std::unordered_map<int32_t, int32_t> moved;
  for (Seq* s : group)
    for (int32_t b : s->blocks)
      if (moved.emplace(b, -1).second) order.push_back(b);
  const int need = static_cast<int>(order.size());
  if (need > capacity || (need > 0 && !mapping)) return PA_ERR_INVALID_ARG;
  const int room = to_cpu ? static_cast<int>(m->cpu.free_ids.size()) : m->free_gpu();
  if (room < need) return PA_ERR_NO_SPACE;
  int pairs = 0;
  for (Seq* s : group) {
    for (int32_t& b : s->blocks) {
      int32_t& nb = moved[b];
      if (nb >= 0) {
        ++(to_cpu ? m->cpu.ref[nb] : m->gpu.ref[nb]);
      } else {
        if (to_cpu) {
          nb = m->cpu.free_ids.back();
          m->cpu.free_ids.pop_back();
          m->cpu.ref[nb] = 1;
        } else {
          nb = m->take_gpu();
        }
        mapping[2 * pairs] = b;
        mapping[2 * pairs + 1] = nb;
        ++pairs;
      }
      if (to_cpu) m->release_gpu(b);
      else m->release_cpu(b);
      b = nb;
    }
    s->on_gpu = !to_cpu;
  }
  *num_pairs = pairs;
  return PA_OK;
}

}  // namespace

PA_API int pa_bm_swap_out(pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                          int64_t* mapping, int capacity, int* num_pairs) {
  return swap_group(m, seq_ids, num_seqs, mapping, capacity, num_pairs, true);
}

PA_API int pa_bm_swap_in(pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                         int64_t* mapping, int capacity, int* num_pairs) {
  return swap_group(m, seq_ids, num_seqs, mapping, capacity, num_pairs, false);
}

PA_API int pa_bm_block_table(const pa_block_manager* m, int64_t seq_id, int32_t* table,
                             int capacity, int* num_blocks, int* num_tokens) {
  if (!m || capacity < 0) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
  const Seq& s = it->second;
  const int nb = static_cast<int>(s.blocks.size());
  if (num_blocks) *num_blocks = nb;             // reported even when table is too small
  if (num_tokens) *num_tokens = static_cast<int>(s.tokens.size());
  if (nb > capacity || (nb > 0 && !table)) return PA_ERR_INVALID_ARG;
  for (int i = 0; i < nb; ++i) table[i] = s.blocks[i];
  return PA_OK;
}

PA_API int pa_bm_build_batch(const pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                             int32_t* block_tables, int max_blocks, int32_t* seq_lens) {
  if (!m || num_seqs < 0 || max_blocks <= 0 || (num_seqs > 0 && (!seq_ids || !block_tables ||
                                                                  !seq_lens)))
    return PA_ERR_INVALID_ARG;
  for (int i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end() || !it->second.on_gpu ||
        static_cast<int>(it->second.blocks.size()) > max_blocks)
      return PA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < num_seqs; ++i) {
    const Seq& s = m->seqs.find(seq_ids[i])->second;
    int32_t* row = block_tables + static_cast<size_t>(i) * max_blocks;
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    std::fill(row + s.blocks.size(), row + max_blocks, -1);
    seq_lens[i] = static_cast<int32_t>(s.tokens.size());
  }
  return PA_OK;
}

PA_API int pa_bm_append_batch(pa_block_manager* m, const int64_t* seq_ids, const int32_t* tokens,
                              int num_seqs, int64_t* slot_mapping, int64_t* cow_pairs,
                              int* num_cow) {
  if (!m || num_seqs < 0 || (num_seqs > 0 && (!seq_ids || !tokens || !slot_mapping)) || !num_cow)
    return PA_ERR_INVALID_ARG;
  std::vector<int64_t> sorted(seq_ids, seq_ids + num_seqs);   // no sequence twice
  std::sort(sorted.begin(), sorted.end());
  if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end()) return PA_ERR_INVALID_ARG;
  int need = 0;
  for (int i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end() || !it->second.on_gpu) return PA_ERR_INVALID_ARG;
    const Seq& s = it->second;
    // a new block when the last is full, or a copy when it is shared (counted
    // before any of this batch's own copies, so the check may be conservative)
    if (s.tokens.size() % m->bs == 0 || m->gpu.ref[s.blocks.back()] > 1) ++need;
  }
  if (m->free_gpu() < need) return PA_ERR_NO_SPACE;
  int cows = 0;
  for (int i = 0; i < num_seqs; ++i) {
    int64_t src, dst;
    pa_bm_append_token(m, seq_ids[i], tokens[i], &slot_mapping[i], &src, &dst);
    if (src >= 0) {
      if (cow_pairs) {
        cow_pairs[2 * cows] = src;
        cow_pairs[2 * cows + 1] = dst;
      }
      ++cows;
    }
  }
  *num_cow = cows;
  return PA_OK;
}

}  // extern "C"
