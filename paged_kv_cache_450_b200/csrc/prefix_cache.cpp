// prefix_cache.cpp -- host-side prefix caching by hash chain.
//
// "vLLM KV Cache 实现机制", 4.2: a full block is identified by a hash of
// (the parent block's hash, the exact tokens of the block, an extra hash for
// multimodal inputs); requests whose prompts share a prefix reuse the cached
// blocks.  3.2: blocks carry reference counts, shared blocks are never
// evicted, and eviction is least-recently-used.  The hash function is
// FNV-1a 64 over the little-endian bytes of parent, tokens, extra (this
// library's choice; the page names none).  Every hit compares the stored
// tokens, parent and extra hash, so a hash collision never shares a block.
#include <cstdint>
#include <cstring>
#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/pagedkv.h"

namespace {

constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

uint64_t fnv_bytes(uint64_t h, const uint8_t* p, size_t n) {
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= kFnvPrime;
  }
  return h;
}

uint64_t fnv_u64(uint64_t h, uint64_t v) {
  uint8_t b[8];
  for (int i = 0; i < 8; ++i) b[i] = static_cast<uint8_t>(v >> (8 * i));
  return fnv_bytes(h, b, 8);
}

uint64_t block_hash(uint64_t parent, const int32_t* tokens, int n, uint64_t extra) {
  uint64_t h = fnv_u64(kFnvOffset, parent);
  for (int i = 0; i < n; ++i) {
    const uint32_t t = static_cast<uint32_t>(tokens[i]);
    uint8_t b[4] = {static_cast<uint8_t>(t), static_cast<uint8_t>(t >> 8), static_cast<uint8_t>(t >> 16),
                    static_cast<uint8_t>(t >> 24)};
    h = fnv_bytes(h, b, 4);
  }
  return fnv_u64(h, extra);
}

struct Entry {
  uint64_t parent;
  uint64_t extra;
  std::vector<int32_t> tokens;
  int32_t block_id;
  int64_t refs;
  std::list<uint64_t>::iterator lru_pos;  // position in the LRU list (front = least recent)
};

struct PrefixCache {
  int block_size;
  int64_t capacity;
  std::unordered_map<uint64_t, Entry> map;
  std::list<uint64_t> lru;  // every cached hash, least recently used first
  std::mutex mu;

  void touch(Entry& e, uint64_t h) {
    lru.erase(e.lru_pos);
    e.lru_pos = lru.insert(lru.end(), h);
  }
  Entry* find(uint64_t h, uint64_t parent, const int32_t* toks, uint64_t extra) {
    auto it = map.find(h);
    if (it == map.end()) return nullptr;
    Entry& e = it->second;
    if (e.parent != parent || e.extra != extra ||
        std::memcmp(e.tokens.data(), toks, sizeof(int32_t) * static_cast<size_t>(block_size)) != 0)
      return nullptr;  // a different block with the same hash: never shared
    return &e;
  }
};

}  // namespace

extern "C" {

int64_t pkv_prefix_block_hashes(const int32_t* tokens, int64_t num_tokens, int block_size, uint64_t parent_hash,
                                uint64_t extra_hash, uint64_t* hashes_out) {
  if (num_tokens < 0 || block_size <= 0) return PKV_ERR_BAD_SHAPE;
  const int64_t n = num_tokens / block_size;
  if (n > 0 && (!tokens || !hashes_out)) return PKV_ERR_NULL_POINTER;
  uint64_t h = parent_hash;
  for (int64_t i = 0; i < n; ++i) {
    h = block_hash(h, tokens + i * block_size, block_size, extra_hash);
    hashes_out[i] = h;
  }
  return n;
}

void* pkv_prefix_cache_create(int block_size, int64_t capacity_blocks) {
  if (block_size <= 0 || capacity_blocks < 0) return nullptr;
  PrefixCache* c = new PrefixCache();
  c->block_size = block_size;
  c->capacity = capacity_blocks;
  return c;
}

void pkv_prefix_cache_destroy(void* cache) { delete static_cast<PrefixCache*>(cache); }

int64_t pkv_prefix_cache_size(void* cache) {
  if (!cache) return PKV_ERR_NULL_POINTER;
  PrefixCache* c = static_cast<PrefixCache*>(cache);
  std::lock_guard<std::mutex> lk(c->mu);
  return static_cast<int64_t>(c->map.size());
}

int64_t pkv_prefix_cache_match(void* cache, const int32_t* tokens, int64_t num_tokens, uint64_t extra_hash,
                               int32_t* block_ids_out, int64_t max_blocks) {
  if (!cache) return PKV_ERR_NULL_POINTER;
  PrefixCache* c = static_cast<PrefixCache*>(cache);
  if (num_tokens < 0 || max_blocks < 0) return PKV_ERR_BAD_SHAPE;
  std::lock_guard<std::mutex> lk(c->mu);
  const int bs = c->block_size;
  int64_t n = num_tokens / bs;
  if (n > max_blocks) n = max_blocks;
  if (n > 0 && (!tokens || !block_ids_out)) return PKV_ERR_NULL_POINTER;
  uint64_t parent = 0;
  int64_t hit = 0;
  for (; hit < n; ++hit) {
    const int32_t* t = tokens + hit * bs;
    const uint64_t h = block_hash(parent, t, bs, extra_hash);
    Entry* e = c->find(h, parent, t, extra_hash);
    if (!e) break;
    e->refs += 1;
    c->touch(*e, h);
    block_ids_out[hit] = e->block_id;
    parent = h;
  }
  return hit;
}

int64_t pkv_prefix_cache_insert(void* cache, const int32_t* tokens, int64_t num_tokens, uint64_t extra_hash,
                                const int32_t* block_ids, int64_t num_blocks) {
  if (!cache) return PKV_ERR_NULL_POINTER;
  PrefixCache* c = static_cast<PrefixCache*>(cache);
  const int bs = c->block_size;
  if (num_tokens < 0 || num_blocks < 0 || num_blocks > num_tokens / bs) return PKV_ERR_BAD_SHAPE;
  if (num_blocks > 0 && (!tokens || !block_ids)) return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> lk(c->mu);
  // How many are new?  All or nothing: a full cache inserts none.
  uint64_t parent = 0;
  int64_t fresh = 0;
  for (int64_t i = 0; i < num_blocks; ++i) {
    const uint64_t h = block_hash(parent, tokens + i * bs, bs, extra_hash);
    if (!c->map.count(h)) ++fresh;
    parent = h;
  }
  if (static_cast<int64_t>(c->map.size()) + fresh > c->capacity) return PKV_ERR_OUT_OF_RANGE;
  parent = 0;
  int64_t added = 0;
  for (int64_t i = 0; i < num_blocks; ++i) {
    const int32_t* t = tokens + i * bs;
    const uint64_t h = block_hash(parent, t, bs, extra_hash);
    auto it = c->map.find(h);
    if (it == c->map.end()) {
      Entry e;
      e.parent = parent;
      e.extra = extra_hash;
      e.tokens.assign(t, t + bs);
      e.block_id = block_ids[i];
      e.refs = 1;  // the inserting sequence holds the block
      e.lru_pos = c->lru.insert(c->lru.end(), h);
      c->map.emplace(h, std::move(e));
      ++added;
    } else if (Entry* e = c->find(h, parent, t, extra_hash)) {
      e->refs += 1;  // already cached (the caller keeps its own copy): count the holder
      c->touch(*e, h);
    }
    // (a collision with a different block is left uncached)
    parent = h;
  }
  return added;
}

int64_t pkv_prefix_cache_release(void* cache, const int32_t* tokens, int64_t num_tokens, uint64_t extra_hash,
                                 int64_t num_blocks) {
  if (!cache) return PKV_ERR_NULL_POINTER;
  PrefixCache* c = static_cast<PrefixCache*>(cache);
  const int bs = c->block_size;
  if (num_tokens < 0 || num_blocks < 0 || num_blocks > num_tokens / bs) return PKV_ERR_BAD_SHAPE;
  if (num_blocks > 0 && !tokens) return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> lk(c->mu);
  uint64_t parent = 0;
  int64_t released = 0;
  for (int64_t i = 0; i < num_blocks; ++i) {
    const int32_t* t = tokens + i * bs;
    const uint64_t h = block_hash(parent, t, bs, extra_hash);
    Entry* e = c->find(h, parent, t, extra_hash);
    if (e && e->refs > 0) {
      e->refs -= 1;
      ++released;
    }
    parent = h;
  }
  return released;
}

int64_t pkv_prefix_cache_evict(void* cache, int64_t max_evict, int32_t* evicted_ids_out) {
  if (!cache) return PKV_ERR_NULL_POINTER;
  PrefixCache* c = static_cast<PrefixCache*>(cache);
  if (max_evict < 0) return PKV_ERR_BAD_SHAPE;
  if (max_evict > 0 && !evicted_ids_out) return PKV_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> lk(c->mu);
  int64_t n = 0;
  for (auto it = c->lru.begin(); it != c->lru.end() && n < max_evict;) {
    auto e = c->map.find(*it);
    if (e->second.refs == 0) {  // shared (referenced) blocks are never evicted
      evicted_ids_out[n++] = e->second.block_id;
      c->map.erase(e);
      it = c->lru.erase(it);
    } else {
      ++it;
    }
  }
  return n;
}

}  // extern "C"
