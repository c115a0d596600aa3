// block_manager.cpp — host-side KV block manager (part of libpa.so, C ABI in
// include/pa.h): the allocator whose block tables, slot mappings and
// copy-on-write pairs the paged-attention kernels consume.
//
// What it does ("PagedAttention: KV cache as virtual memory", "Deep dive";
// "vLLM PagedAttention Deep Dive", "Virtual Memory Paging Analogy" and
// "Automatic Prefix Caching"; "PagedAttention: Why Static Batching Wastes Your
// KV Cache", "How does copy-on-write eliminate duplicate prompt KV cache?"):
//  * a pool of num_blocks fixed-size physical blocks; free blocks sit in a
//    doubly-linked queue in eviction order: allocation pops the front, a
//    freed block is pushed at the back, a cached block revived by a prefix
//    hit is unlinked from the middle — all O(1);
//  * every block has a reference count; a sequence's block table lists its
//    physical blocks in logical order; a block returns to the free queue when
//    its count drops to zero;
//  * prefix caching: a FULL block is keyed by a hash of (parent block's key,
//    its tokens); a new sequence whose leading full blocks have keys already
//    in the map points its table at those blocks (count + 1) instead of
//    taking new ones.  Freed blocks keep their key until the block is handed
//    out again, so a later request can still hit them (least recently freed
//    blocks are reused first);
//  * decode appends tokens: a new block is taken when the last one is full;
//    appending into a partially filled block that is shared (count > 1, e.g.
//    after fork) first copies it to a fresh block — copy-on-write — and
//    queues the (src, dst) pair for pa_copy_blocks.
// A hit also compares the block's stored tokens, so two prefixes can share a
// block only if that block's tokens are equal and the 64-bit keys of their
// parents collide.
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pa.h"

namespace {

constexpr int32_t kNil = -1;

uint64_t mix64(uint64_t x) {  // splitmix64 finaliser
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

struct Block {
  int32_t ref = 0;
  int32_t prev = kNil, next = kNil;  // free-queue links
  bool in_free = false;
  bool cached = false;  // key registered in the prefix map
  uint64_t key = 0;
};

struct Seq {
  std::vector<int32_t> table;   // physical blocks in logical order
  std::vector<int32_t> tokens;  // all token ids (for prefix keys of full blocks)
  std::vector<uint64_t> keys;   // key of each full block
};

}  // namespace

struct pa_block_manager {
  int num_blocks = 0, block_size = 0;
  bool prefix = false;
  std::vector<Block> blocks;
  std::vector<int32_t> cached_tokens;  // [num_blocks][block_size], tokens of cached blocks
  int32_t head = kNil, tail = kNil;
  int num_free = 0;
  std::unordered_map<uint64_t, int32_t> key_to_block;
  std::unordered_map<int64_t, Seq> seqs;
  std::vector<int64_t> pending_copies;  // flattened (src, dst)

  // ----------------------------------------------------------- free queue
  void push_back(int32_t b) {
    Block& x = blocks[b];
    x.prev = tail;
    x.next = kNil;
    if (tail != kNil) blocks[tail].next = b; else head = b;
    tail = b;
    x.in_free = true;
    ++num_free;
  }
  void unlink(int32_t b) {
    Block& x = blocks[b];
    if (x.prev != kNil) blocks[x.prev].next = x.next; else head = x.next;
    if (x.next != kNil) blocks[x.next].prev = x.prev; else tail = x.prev;
    x.prev = x.next = kNil;
    x.in_free = false;
    --num_free;
  }
  // Pop the least recently freed block; drop its old prefix key (eviction).
  int32_t pop_front() {
    const int32_t b = head;
    unlink(b);
    Block& x = blocks[b];
    if (x.cached) {
      auto it = key_to_block.find(x.key);
      if (it != key_to_block.end() && it->second == b) key_to_block.erase(it);
      x.cached = false;
    }
    x.ref = 1;
    return b;
  }
  void release(int32_t b) {
    if (--blocks[b].ref == 0) push_back(b);
  }

  // ----------------------------------------------------------- prefix keys
  uint64_t key_of(uint64_t parent, const int32_t* toks) const {
    uint64_t h = mix64(parent ^ 0xC2B2AE3D27D4EB4Full);
    for (int i = 0; i < block_size; ++i) h = mix64(h ^ (uint64_t)(uint32_t)toks[i]);
    return h;
  }
  bool tokens_match(int32_t b, const int32_t* toks) const {
    return std::memcmp(&cached_tokens[(size_t)b * block_size], toks,
                       sizeof(int32_t) * block_size) == 0;
  }
  // Register block b (now full) under `key` unless that key already maps to
  // a block (the first owner stays canonical).
  void register_full(int32_t b, uint64_t key, const int32_t* toks) {
    if (!prefix || blocks[b].cached) return;
    if (key_to_block.count(key)) return;
    key_to_block.emplace(key, b);
    blocks[b].cached = true;
    blocks[b].key = key;
    std::memcpy(&cached_tokens[(size_t)b * block_size], toks, sizeof(int32_t) * block_size);
  }
  // Blocks of `seq` that just became full get keys (and prefix entries).
  void seal_full_blocks(Seq& q) {
    const int full = (int)q.tokens.size() / block_size;
    while ((int)q.keys.size() < full) {
      const int i = (int)q.keys.size();
      const uint64_t parent = i == 0 ? 0 : q.keys[i - 1];
      const int32_t* toks = &q.tokens[(size_t)i * block_size];
      const uint64_t k = key_of(parent, toks);
      q.keys.push_back(k);
      register_full(q.table[i], k, toks);
    }
  }
};

extern "C" {

pa_status pa_bm_create(int num_blocks, int block_size, int enable_prefix_caching,
                       pa_block_manager** out) {
  if (!out || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  // token counts and positions are int throughout the ABI
  if ((int64_t)num_blocks * block_size > INT32_MAX) return PA_ERR_INVALID_ARG;
  auto* m = new (std::nothrow) pa_block_manager();
  if (!m) return PA_ERR_INVALID_ARG;
  m->num_blocks = num_blocks;
  m->block_size = block_size;
  m->prefix = enable_prefix_caching != 0;
  try {
    m->blocks.resize(num_blocks);
    if (m->prefix) m->cached_tokens.resize((size_t)num_blocks * block_size);
  } catch (const std::bad_alloc&) {
    delete m;
    return PA_ERR_INVALID_ARG;
  }
  for (int b = 0; b < num_blocks; ++b) m->push_back(b);  // ids in order: 0 is handed out first
  *out = m;
  return PA_OK;
}

void pa_bm_destroy(pa_block_manager* m) { delete m; }

int pa_bm_num_free_blocks(const pa_block_manager* m) { return m ? m->num_free : -1; }

int pa_bm_ref_count(const pa_block_manager* m, int block) {
  if (!m || block < 0 || block >= m->num_blocks) return -1;
  return m->blocks[block].ref;
}

int pa_bm_num_tokens(const pa_block_manager* m, int64_t seq_id) {
  if (!m) return -1;
  auto it = m->seqs.find(seq_id);
  return it == m->seqs.end() ? -1 : (int)it->second.tokens.size();
}

pa_status pa_bm_add_sequence(pa_block_manager* m, int64_t seq_id, const int32_t* tokens,
                             int num_tokens, int* num_cached_tokens) {
  if (!m || num_tokens < 0 || (num_tokens > 0 && !tokens)) return PA_ERR_INVALID_ARG;
  if (m->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  const int B = m->block_size;
  const int64_t need = ((int64_t)num_tokens + B - 1) / B;
  if (need > m->num_blocks) return PA_ERR_OUT_OF_RANGE;  // can never fit
  // leading full blocks already cached (prefix hits stop at the first miss)
  std::vector<int32_t> hits;
  std::vector<uint64_t> keys;
  if (m->prefix) {
    uint64_t parent = 0;
    for (int i = 0; i < num_tokens / B; ++i) {
      const int32_t* toks = tokens + (size_t)i * B;
      const uint64_t k = m->key_of(parent, toks);
      auto it = m->key_to_block.find(k);
      if (it == m->key_to_block.end() || !m->tokens_match(it->second, toks)) break;
      hits.push_back(it->second);
      keys.push_back(k);
      parent = k;
    }
  }
  // hits that sit in the free queue leave it, so count what must come from it
  int revived = 0;
  for (int32_t b : hits) revived += m->blocks[b].in_free ? 1 : 0;
  const int fresh = (int)need - (int)hits.size();
  if (fresh + revived > m->num_free) return PA_ERR_OUT_OF_RANGE;  // nothing changed
  Seq q;
  q.tokens.assign(tokens, tokens + num_tokens);
  for (int32_t b : hits) {
    if (m->blocks[b].in_free) {
      m->unlink(b);
      m->blocks[b].ref = 1;
    } else {
      ++m->blocks[b].ref;
    }
    q.table.push_back(b);
  }
  q.keys = keys;
  for (int i = 0; i < fresh; ++i) q.table.push_back(m->pop_front());
  m->seal_full_blocks(q);
  if (num_cached_tokens) *num_cached_tokens = (int)hits.size() * B;
  m->seqs.emplace(seq_id, std::move(q));
  return PA_OK;
}

pa_status pa_bm_append(pa_block_manager* m, int64_t seq_id, const int32_t* tokens,
                       int num_tokens) {
  if (!m || num_tokens < 0 || (num_tokens > 0 && !tokens)) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
  Seq& q = it->second;
  const int B = m->block_size;
  const int64_t L = (int64_t)q.tokens.size();
  // blocks needed: a copy of a shared partial last block, plus new blocks
  const bool partial = L % B != 0;
  const bool cow = num_tokens > 0 && partial && m->blocks[q.table.back()].ref > 1;
  const int64_t new_blocks = (L + num_tokens + B - 1) / B - (L + B - 1) / B;
  if ((cow ? 1 : 0) + new_blocks > m->num_free) return PA_ERR_OUT_OF_RANGE;
  if (cow) {
    const int32_t src = q.table.back();
    const int32_t dst = m->pop_front();
    m->release(src);  // still referenced by the other sharers
    q.table.back() = dst;
    m->pending_copies.push_back(src);
    m->pending_copies.push_back(dst);
  }
  for (int i = 0; i < new_blocks; ++i) q.table.push_back(m->pop_front());
  q.tokens.insert(q.tokens.end(), tokens, tokens + num_tokens);
  m->seal_full_blocks(q);
  return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager* m, int64_t parent_id, int64_t child_id) {
  if (!m) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(parent_id);
  if (it == m->seqs.end() || m->seqs.count(child_id)) return PA_ERR_INVALID_ARG;
  Seq child = it->second;
  for (int32_t b : child.table) ++m->blocks[b].ref;
  m->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

pa_status pa_bm_free(pa_block_manager* m, int64_t seq_id) {
  if (!m) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
  // tail first, so a sequence's last (least shareable) blocks are reused first
  const std::vector<int32_t>& t = it->second.table;
  for (auto b = t.rbegin(); b != t.rend(); ++b) m->release(*b);
  m->seqs.erase(it);
  return PA_OK;
}

pa_status pa_bm_block_table(const pa_block_manager* m, int64_t seq_id, int32_t* out,
                            int capacity, int* num_blocks) {
  if (!m || capacity < 0 || (capacity > 0 && !out)) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
  const std::vector<int32_t>& t = it->second.table;
  if (num_blocks) *num_blocks = (int)t.size();
  if ((int)t.size() > capacity) return PA_ERR_WORKSPACE;
  if (!t.empty()) std::memcpy(out, t.data(), sizeof(int32_t) * t.size());
  for (int i = (int)t.size(); i < capacity; ++i) out[i] = -1;
  return PA_OK;
}

pa_status pa_bm_slots(const pa_block_manager* m, int64_t seq_id, int start, int count,
                      int64_t* out) {
  if (!m || start < 0 || count < 0 || (count > 0 && !out)) return PA_ERR_INVALID_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
  const Seq& q = it->second;
  if ((int64_t)start + count > (int64_t)q.table.size() * m->block_size) return PA_ERR_OUT_OF_RANGE;
  for (int i = 0; i < count; ++i) {
    const int p = start + i;
    out[i] = (int64_t)q.table[p / m->block_size] * m->block_size + p % m->block_size;
  }
  return PA_OK;
}

int pa_bm_take_copies(pa_block_manager* m, int64_t* pairs, int capacity) {
  if (!m || capacity < 0 || (capacity > 0 && !pairs)) return -1;
  const int n = (int)m->pending_copies.size() / 2;
  if (n > capacity) return -n;  // too small: nothing taken
  if (n > 0) std::memcpy(pairs, m->pending_copies.data(), sizeof(int64_t) * 2 * n);
  m->pending_copies.clear();
  return n;
}

}  // extern "C"
