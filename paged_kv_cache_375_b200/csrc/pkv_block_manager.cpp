// pkv_block_manager.cpp -- host-side KV-block bookkeeping behind the C ABI of
// include/pkv_block_manager.h: a scattered free list, reference counts,
// fork / copy-on-write, and automatic prefix caching (hash-chained full
// blocks, exact matching, least-recently-used eviction).
#include "pkv_block_manager.h"

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <random>
#include <unordered_map>
#include <utility>
#include <vector>

namespace {

struct Block {
  int32_t ref = 0;
  bool cached = false;                  // registered in the prefix cache
  uint64_t hash = 0;
  std::vector<int32_t> tokens;          // contents of a cached (full) block
  std::list<int32_t>::iterator lru_it;  // position in the eviction list while ref == 0
  bool in_lru = false;
};

struct Sequence {
  std::vector<int32_t> table;   // physical block per logical block
  std::vector<int32_t> tokens;  // token ids of the whole context
  uint64_t chain = 0;           // hash of the last registered full block
  int32_t hashed = 0;           // leading full blocks already hashed
  uint64_t mark = 0;            // call number of the last append call that touched it
  int32_t pending = 0;          // appends to it counted so far in that call
};

// 64-bit FNV-1a over the parent hash and the block's token ids, then a
// splitmix finaliser: the hash of a block depends on its whole prefix.
uint64_t chain_hash(uint64_t parent, const int32_t* tokens, int32_t n) {
  uint64_t h = 0xcbf29ce484222325ull;
  auto mix = [&](uint64_t v) {
    for (int i = 0; i < 8; ++i) {
      h ^= (v >> (8 * i)) & 0xffu;
      h *= 0x100000001b3ull;
    }
  };
  mix(parent);
  for (int32_t i = 0; i < n; ++i) mix(static_cast<uint32_t>(tokens[i]));
  h ^= h >> 30;
  h *= 0xbf58476d1ce4e5b9ull;
  h ^= h >> 27;
  h *= 0x94d049bb133111ebull;
  h ^= h >> 31;
  return h;
}

}  // namespace

struct pkv_block_manager {
  int32_t num_blocks;
  int32_t bs;
  bool prefix_caching;
  std::vector<Block> blocks;
  std::vector<int32_t> free_list;                 // back = next to hand out
  std::list<int32_t> lru;                         // evictable cached blocks, front = oldest
  std::unordered_map<uint64_t, int32_t> cache;    // chain hash -> block
  std::unordered_map<int64_t, Sequence> seqs;
  std::vector<std::pair<int64_t, int64_t>> copies;
  uint64_t calls = 0;                             // append calls so far
  std::vector<Sequence*> scratch;                 // per-call sequence pointers

  int32_t available() const { return static_cast<int32_t>(free_list.size() + lru.size()); }

  // Take a block: a never-used or returned one first, else evict the least
  // recently used cached block.  The caller checked availability.
  int32_t allocate() {
    int32_t b;
    if (!free_list.empty()) {
      b = free_list.back();
      free_list.pop_back();
    } else {
      b = lru.front();
      lru.pop_front();
      Block& e = blocks[b];
      e.in_lru = false;
      auto it = cache.find(e.hash);
      if (it != cache.end() && it->second == b) cache.erase(it);
      e.cached = false;
      e.tokens.clear();
    }
    blocks[b].ref = 1;
    return b;
  }

  void acquire(int32_t b) {
    Block& e = blocks[b];
    if (e.ref == 0 && e.in_lru) {
      lru.erase(e.lru_it);
      e.in_lru = false;
    }
    ++e.ref;
  }

  void release(int32_t b) {
    Block& e = blocks[b];
    if (--e.ref > 0) return;
    if (e.cached) {
      e.lru_it = lru.insert(lru.end(), b);
      e.in_lru = true;
    } else {
      free_list.push_back(b);
    }
  }

  // Register the full blocks of `s` that are not hashed yet.
  void register_full_blocks(Sequence& s) {
    if (!prefix_caching) return;
    const int32_t full = static_cast<int32_t>(s.tokens.size()) / bs;
    while (s.hashed < full) {
      const int32_t i = s.hashed;
      const int32_t* t = s.tokens.data() + static_cast<size_t>(i) * bs;
      const uint64_t h = chain_hash(s.chain, t, bs);
      const int32_t b = s.table[i];
      Block& e = blocks[b];
      if (!e.cached && cache.find(h) == cache.end()) {
        e.cached = true;
        e.hash = h;
        e.tokens.assign(t, t + bs);
        cache.emplace(h, b);
      }
      s.chain = h;
      ++s.hashed;
    }
  }

  int64_t slot(const Sequence& s, int32_t pos) const {
    return static_cast<int64_t>(s.table[pos / bs]) * bs + pos % bs;
  }
};

extern "C" {

pkv_block_manager* pkv_bm_create(int32_t num_blocks, int32_t block_size, uint64_t seed,
                                 int32_t prefix_caching) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  auto* bm = new pkv_block_manager();
  bm->num_blocks = num_blocks;
  bm->bs = block_size;
  bm->prefix_caching = prefix_caching != 0;
  bm->blocks.resize(static_cast<size_t>(num_blocks));
  bm->free_list.resize(static_cast<size_t>(num_blocks));
  for (int32_t i = 0; i < num_blocks; ++i) bm->free_list[i] = i;
  std::mt19937_64 rng(seed);
  std::shuffle(bm->free_list.begin(), bm->free_list.end(), rng);
  return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                               int32_t n, int32_t* cached_tokens) {
  if (!bm || (!tokens && n > 0)) return PKV_ERR_NULL;
  if (n < 0) return PKV_ERR_SHAPE;
  if (bm->seqs.count(seq_id)) return PKV_ERR_NOT_FOUND;
  const int32_t bs = bm->bs;
  // find the cached prefix: full blocks only, matched block by block exactly
  std::vector<int32_t> hits;
  uint64_t chain = 0;
  if (bm->prefix_caching) {
    for (int32_t i = 0; i < n / bs; ++i) {
      const int32_t* t = tokens + static_cast<size_t>(i) * bs;
      const uint64_t h = chain_hash(chain, t, bs);
      auto it = bm->cache.find(h);
      if (it == bm->cache.end()) break;
      const Block& e = bm->blocks[it->second];
      if (!std::equal(e.tokens.begin(), e.tokens.end(), t)) break;  // hash collision
      hits.push_back(it->second);
      chain = h;
    }
  }
  const int32_t need = (n + bs - 1) / bs - static_cast<int32_t>(hits.size());
  // cached hits held by nobody come out of the eviction list, so they do not count
  int32_t evictable_hits = 0;
  for (int32_t b : hits) evictable_hits += bm->blocks[b].ref == 0 ? 1 : 0;
  if (need > bm->available() - evictable_hits) return PKV_ERR_NO_BLOCKS;
  Sequence s;
  for (int32_t b : hits) {
    bm->acquire(b);
    s.table.push_back(b);
  }
  for (int32_t i = 0; i < need; ++i) s.table.push_back(bm->allocate());
  s.tokens.assign(tokens, tokens + n);
  s.chain = chain;
  s.hashed = static_cast<int32_t>(hits.size());
  bm->register_full_blocks(s);
  if (cached_tokens) *cached_tokens = static_cast<int32_t>(hits.size()) * bs;
  bm->seqs.emplace(seq_id, std::move(s));
  return PKV_OK;
}

pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child) {
  if (!bm) return PKV_ERR_NULL;
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end() || bm->seqs.count(child)) return PKV_ERR_NOT_FOUND;
  Sequence s = it->second;
  for (int32_t b : s.table) bm->acquire(b);
  bm->seqs.emplace(child, std::move(s));
  return PKV_OK;
}

pkv_status pkv_bm_append_tokens(pkv_block_manager* bm, const int64_t* seq_ids,
                                const int32_t* tokens, int32_t n, int64_t* slots_out) {
  if (!bm || ((!seq_ids || !tokens || !slots_out) && n > 0)) return PKV_ERR_NULL;
  if (n < 0) return PKV_ERR_SHAPE;
  // check first (all or nothing): sequences exist and enough blocks for new
  // blocks and copies.  A sequence may appear more than once in a call; the
  // per-sequence mark counts its appends within this call.
  const uint64_t call = ++bm->calls;
  bm->scratch.resize(static_cast<size_t>(n));
  int32_t need = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    Sequence& s = it->second;
    bm->scratch[i] = &s;
    if (s.mark != call) {
      s.mark = call;
      s.pending = 0;
    }
    const int32_t k = s.pending++;
    const int32_t pos = static_cast<int32_t>(s.tokens.size()) + k;
    if (pos % bm->bs == 0) {
      ++need;                                            // a new block
    } else if (k == 0 && bm->blocks[s.table[pos / bm->bs]].ref > 1) {
      ++need;                                            // a copy of the shared last block
    }
  }
  if (need > bm->available()) return PKV_ERR_NO_BLOCKS;
  for (int32_t i = 0; i < n; ++i) {
    Sequence& s = *bm->scratch[i];
    const int32_t pos = static_cast<int32_t>(s.tokens.size());
    const int32_t li = pos / bm->bs;
    if (li == static_cast<int32_t>(s.table.size())) {
      s.table.push_back(bm->allocate());
    } else {
      const int32_t b = s.table[li];
      if (bm->blocks[b].ref > 1) {                       // copy on write
        const int32_t nb = bm->allocate();
        bm->copies.emplace_back(b, nb);
        bm->release(b);
        s.table[li] = nb;
      }
    }
    slots_out[i] = bm->slot(s, pos);
    s.tokens.push_back(tokens[i]);
    bm->register_full_blocks(s);
  }
  return PKV_OK;
}

pkv_status pkv_bm_slots(pkv_block_manager* bm, int64_t seq_id, int32_t pos_begin,
                        int32_t pos_end, int64_t* slots_out) {
  if (!bm || (!slots_out && pos_end > pos_begin)) return PKV_ERR_NULL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
  const Sequence& s = it->second;
  if (pos_begin < 0 || pos_end < pos_begin || pos_end > static_cast<int32_t>(s.tokens.size()))
    return PKV_ERR_SHAPE;
  for (int32_t p = pos_begin; p < pos_end; ++p) slots_out[p - pos_begin] = bm->slot(s, p);
  return PKV_OK;
}

pkv_status pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq_id) {
  if (!bm) return PKV_ERR_NULL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
  // tail first, so that a prefix outlives its tails in the eviction order
  const std::vector<int32_t>& t = it->second.table;
  for (auto b = t.rbegin(); b != t.rend(); ++b) bm->release(*b);
  bm->seqs.erase(it);
  return PKV_OK;
}

int32_t pkv_bm_take_copies(pkv_block_manager* bm, int64_t* pairs_out, int32_t max_pairs) {
  if (!bm) return 0;
  const int32_t n = static_cast<int32_t>(bm->copies.size());
  if (n > max_pairs || (!pairs_out && n > 0)) return -n;
  for (int32_t i = 0; i < n; ++i) {
    pairs_out[2 * i] = bm->copies[i].first;
    pairs_out[2 * i + 1] = bm->copies[i].second;
  }
  bm->copies.clear();
  return n;
}

pkv_status pkv_bm_block_tables(pkv_block_manager* bm, const int64_t* seq_ids, int32_t n,
                               int32_t max_blocks, int32_t* tables_out, int32_t* lens_out) {
  if (!bm || ((!seq_ids || !tables_out || !lens_out) && n > 0)) return PKV_ERR_NULL;
  if (n < 0 || max_blocks <= 0) return PKV_ERR_SHAPE;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    if (static_cast<int32_t>(it->second.table.size()) > max_blocks) return PKV_ERR_SHAPE;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Sequence& s = bm->seqs.find(seq_ids[i])->second;
    int32_t* row = tables_out + static_cast<size_t>(i) * max_blocks;
    const int32_t nb = static_cast<int32_t>(s.table.size());
    std::memcpy(row, s.table.data(), sizeof(int32_t) * nb);
    std::fill(row + nb, row + max_blocks, -1);
    lens_out[i] = static_cast<int32_t>(s.tokens.size());
  }
  return PKV_OK;
}

pkv_status pkv_bm_prefix_order(pkv_block_manager* bm, const int64_t* seq_ids, int32_t n,
                               int32_t* order_out) {
  if (!bm || ((!seq_ids || !order_out) && n > 0)) return PKV_ERR_NULL;
  if (n < 0) return PKV_ERR_SHAPE;
  std::vector<const Sequence*> seqs(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    seqs[i] = &it->second;
  }
  // lexicographic order of the full blocks' physical ids: sequences that
  // begin with the same blocks end up next to each other, and the longer the
  // common run the closer (ties keep the given order)
  std::vector<int32_t> idx(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) idx[i] = i;
  const size_t bs = static_cast<size_t>(bm->bs);
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t x, int32_t y) {
    const Sequence& a = *seqs[x];
    const Sequence& b = *seqs[y];
    const size_t fa = std::min(a.tokens.size() / bs, a.table.size());
    const size_t fb = std::min(b.tokens.size() / bs, b.table.size());
    return std::lexicographical_compare(a.table.begin(), a.table.begin() + fa, b.table.begin(),
                                        b.table.begin() + fb);
  });
  std::copy(idx.begin(), idx.end(), order_out);
  return PKV_OK;
}

pkv_status pkv_bm_shared_prefix_groups(pkv_block_manager* bm, const int64_t* seq_ids, int32_t n,
                                       int32_t min_shared_blocks, int32_t* group_start_out,
                                       int32_t* shared_blocks_out, int32_t* num_groups_out) {
  if (!bm || !group_start_out || !num_groups_out || ((!seq_ids || !shared_blocks_out) && n > 0))
    return PKV_ERR_NULL;
  if (n < 0 || min_shared_blocks < 1) return PKV_ERR_SHAPE;
  std::vector<const Sequence*> seqs(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    seqs[i] = &it->second;
  }
  // leading physical blocks two sequences hold in common, among the full
  // blocks of both
  auto common = [&](const Sequence& a, const Sequence& b) {
    const size_t full = std::min(a.tokens.size(), b.tokens.size()) / static_cast<size_t>(bm->bs);
    size_t c = 0;
    while (c < full && c < a.table.size() && c < b.table.size() && a.table[c] == b.table[c]) ++c;
    return static_cast<int32_t>(c);
  };
  int32_t g = 0;
  group_start_out[0] = 0;
  for (int32_t i = 0; i < n;) {
    // a run starts at i and takes the following sequences while they keep at
    // least min_shared_blocks leading blocks in common with its first member
    int32_t shared = 0, j = i + 1;
    for (; j < n; ++j) {
      const int32_t c = common(*seqs[i], *seqs[j]);
      const int32_t p = j == i + 1 ? c : std::min(shared, c);
      if (p < min_shared_blocks) break;
      shared = p;
    }
    shared_blocks_out[g] = j - i >= 2 ? shared : 0;
    group_start_out[++g] = j;
    i = j;
  }
  *num_groups_out = g;
  return PKV_OK;
}

pkv_status pkv_bm_stats(const pkv_block_manager* bm, int32_t* free_blocks,
                        int32_t* evictable_blocks, int32_t* used_blocks, int32_t* sequences) {
  if (!bm) return PKV_ERR_NULL;
  const int32_t f = static_cast<int32_t>(bm->free_list.size());
  const int32_t e = static_cast<int32_t>(bm->lru.size());
  if (free_blocks) *free_blocks = f;
  if (evictable_blocks) *evictable_blocks = e;
  if (used_blocks) *used_blocks = bm->num_blocks - f - e;
  if (sequences) *sequences = static_cast<int32_t>(bm->seqs.size());
  return PKV_OK;
}

int32_t pkv_bm_refcount(const pkv_block_manager* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->blocks[block].ref;
}

}  // extern "C"
