// Host-side KV block manager: the ledger in front of the append.
//
// "vLLM 推理引擎源码级拆解" (chenxutan.com/d/5333): §2.1 (fixed-size blocks,
// sharing by reference count and copy-on-write), §2.2 (a token fills the last
// block, else a block from the free pool), §3.1 (can_allocate / allocate,
// can_append / append_slot), §3.2 (preemption by freeing or by swapping to
// host memory), §3.3 (the manager only keeps accounts), §4.2 (prefix caching:
// a block is named by a hash of its token ids and of its predecessor's hash;
// unheld cached blocks are reclaimed least-recently-used first). The C ABI and
// the semantics of each call are in include/pagedkv_blocks.h.
//
// The block hash is 64-bit FNV-1a (Fowler-Noll-Vo) over the predecessor's hash
// (8 bytes, little-endian) followed by the block's token ids (4 bytes each);
// the first block's predecessor hash is 0. A hash hit is taken only when the
// cached block's predecessor hash and token ids are equal as well, so a hash
// collision can cost a cache miss but never a wrong share.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pagedkv_blocks.h"

namespace {

constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

uint64_t fnv1a(uint64_t h, const void* data, size_t n) {
  const unsigned char* p = static_cast<const unsigned char*>(data);
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= kFnvPrime;
  }
  return h;
}

uint64_t block_hash(uint64_t parent, const int32_t* tokens, int bs) {
  unsigned char buf[8];
  for (int i = 0; i < 8; ++i) buf[i] = (unsigned char)(parent >> (8 * i));
  uint64_t h = fnv1a(kFnvOffset, buf, 8);
  for (int t = 0; t < bs; ++t) {
    const uint32_t v = (uint32_t)tokens[t];
    unsigned char b[4] = {(unsigned char)v, (unsigned char)(v >> 8), (unsigned char)(v >> 16),
                          (unsigned char)(v >> 24)};
    h = fnv1a(h, b, 4);
  }
  return h;
}

struct Block {
  int32_t ref = 0;
  bool hashed = false;  // registered in the prefix cache
  uint64_t hash = 0, parent = 0;
  std::vector<int32_t> tokens;  // the block's token ids, when hashed
  bool in_lru = false;          // cached and held by no sequence
  std::list<int32_t>::iterator lru_it;
};

struct Seq {
  std::vector<int32_t> blocks;  // device ids, or host ids while swapped out
  int64_t len = 0;
  bool swapped = false;
  uint64_t last_hash = 0;       // hash of the last full block (0: none)
  std::vector<int32_t> tail;    // token ids in the partial last block
};

}  // namespace

struct pkv_block_manager {
  int bs = 16;
  bool prefix = false;
  std::vector<Block> dev;
  std::vector<int32_t> free_dev;  // stack; the back is handed out first
  std::list<int32_t> lru;         // cached unheld blocks, least recent at the front
  std::unordered_map<uint64_t, int32_t> cache;  // block hash -> block
  std::vector<int32_t> host_ref;
  std::vector<int32_t> free_host;
  std::unordered_map<int64_t, Seq> seqs;

  int64_t available() const { return (int64_t)free_dev.size() + (int64_t)lru.size(); }

  // A device block for new contents, or -1: a free block, else the least
  // recently used cached block, which leaves the cache.
  int32_t take_block() {
    int32_t b;
    if (!free_dev.empty()) {
      b = free_dev.back();
      free_dev.pop_back();
    } else if (!lru.empty()) {
      b = lru.front();
      lru.pop_front();
      Block& blk = dev[b];
      blk.in_lru = false;
      uncache(b);
    } else {
      return -1;
    }
    dev[b].ref = 1;
    return b;
  }

  void uncache(int32_t b) {
    Block& blk = dev[b];
    if (!blk.hashed) return;
    auto it = cache.find(blk.hash);
    if (it != cache.end() && it->second == b) cache.erase(it);
    blk.hashed = false;
    blk.tokens.clear();
  }

  // One reference fewer; an unheld block goes to the LRU list if cached, else
  // to the free pool.
  void release(int32_t b) {
    Block& blk = dev[b];
    if (--blk.ref > 0) return;
    if (blk.hashed) {
      blk.in_lru = true;
      blk.lru_it = lru.insert(lru.end(), b);
    } else {
      free_dev.push_back(b);
    }
  }

  void hold(int32_t b) {
    Block& blk = dev[b];
    if (blk.in_lru) {
      lru.erase(blk.lru_it);
      blk.in_lru = false;
    }
    ++blk.ref;
  }

  // The cached block for (parent, tokens), or -1.
  int32_t lookup(uint64_t h, uint64_t parent, const int32_t* tokens) const {
    auto it = cache.find(h);
    if (it == cache.end()) return -1;
    const Block& blk = dev[it->second];
    if (blk.parent != parent || (int)blk.tokens.size() != bs ||
        std::memcmp(blk.tokens.data(), tokens, sizeof(int32_t) * bs) != 0)
      return -1;
    return it->second;
  }

  void register_block(int32_t b, uint64_t h, uint64_t parent, const int32_t* tokens) {
    if (cache.count(h)) return;  // an equal (or colliding) block is cached already
    Block& blk = dev[b];
    blk.hashed = true;
    blk.hash = h;
    blk.parent = parent;
    blk.tokens.assign(tokens, tokens + bs);
    cache.emplace(h, b);
  }

  void release_seq(Seq& s) {
    for (auto it = s.blocks.rbegin(); it != s.blocks.rend(); ++it) release(*it);
    s.blocks.clear();
  }
};

extern "C" {

pkv_block_manager* pkv_bm_create(int64_t num_blocks, int64_t num_host_blocks, int block_size,
                                 int prefix_caching) {
  if (num_blocks < 0 || num_blocks > INT32_MAX || num_host_blocks < 0 ||
      num_host_blocks > INT32_MAX || block_size <= 0)
    return nullptr;
  pkv_block_manager* bm = new (std::nothrow) pkv_block_manager();
  if (!bm) return nullptr;
  try {
    bm->bs = block_size;
    bm->prefix = prefix_caching != 0;
    bm->dev.resize((size_t)num_blocks);
    bm->free_dev.reserve((size_t)num_blocks);
    for (int64_t b = num_blocks - 1; b >= 0; --b) bm->free_dev.push_back((int32_t)b);
    bm->host_ref.assign((size_t)num_host_blocks, 0);
    for (int64_t b = num_host_blocks - 1; b >= 0; --b) bm->free_host.push_back((int32_t)b);
  } catch (...) {
    delete bm;
    return nullptr;
  }
  return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int64_t pkv_bm_num_free(const pkv_block_manager* bm) { return bm ? bm->available() : 0; }

int64_t pkv_bm_num_free_host(const pkv_block_manager* bm) {
  return bm ? (int64_t)bm->free_host.size() : 0;
}

int pkv_bm_can_allocate(const pkv_block_manager* bm, int64_t num_tokens) {
  if (!bm || num_tokens < 0) return 0;
  return (num_tokens + bm->bs - 1) / bm->bs <= bm->available() ? 1 : 0;
}

int pkv_bm_allocate(pkv_block_manager* bm, int64_t seq_id, const int32_t* token_ids,
                    int64_t num_tokens, int64_t* slot_mapping, int64_t* num_cached) {
  if (!bm) return PKV_ERR_NULL;
  if (num_tokens < 0) return PKV_ERR_SHAPE;
  if (bm->prefix && num_tokens > 0 && !token_ids) return PKV_ERR_NULL;
  if (bm->seqs.count(seq_id)) return PKV_ERR_SEQ;
  const int bs = bm->bs;
  const int64_t nblk = (num_tokens + bs - 1) / bs, nfull = num_tokens / bs;
  Seq s;
  s.len = num_tokens;
  // Pass 1: hashes and cache lookups, changing nothing; count what must be
  // taken, so that a call that cannot be served changes nothing.
  std::vector<int32_t> hitb((size_t)nblk, -1);
  std::vector<uint64_t> hashes((size_t)nblk, 0), parents((size_t)nblk, 0);
  uint64_t parent = 0;
  int64_t misses = 0, unheld_hits = 0;
  std::unordered_set<int32_t> hit_set;
  for (int64_t i = 0; i < nblk; ++i) {
    parents[(size_t)i] = parent;
    if (bm->prefix && i < nfull) {
      const uint64_t h = block_hash(parent, token_ids + i * bs, bs);
      hashes[(size_t)i] = h;
      const int32_t b = bm->lookup(h, parent, token_ids + i * bs);
      if (b >= 0 && hit_set.insert(b).second) {  // (a block is shared at most once here)
        hitb[(size_t)i] = b;
        if (bm->dev[b].ref == 0) ++unheld_hits;
      }
      parent = h;
    }
    if (hitb[(size_t)i] < 0) ++misses;
  }
  if (misses > bm->available() - unheld_hits) return PKV_ERR_NO_BLOCKS;
  // Pass 2: hold the hits first (so that taking blocks cannot evict them),
  // then take a block for every miss and name the full ones.
  for (int64_t i = 0; i < nblk; ++i)
    if (hitb[(size_t)i] >= 0) bm->hold(hitb[(size_t)i]);
  int64_t cached = 0;
  bool leading = true;
  for (int64_t i = 0; i < nblk; ++i) {
    int32_t b = hitb[(size_t)i];
    if (b < 0) {
      b = bm->take_block();  // cannot fail: counted above
      if (bm->prefix && i < nfull)
        bm->register_block(b, hashes[(size_t)i], parents[(size_t)i], token_ids + i * bs);
    }
    leading = leading && hitb[(size_t)i] >= 0;
    if (leading) cached += bs;
    s.blocks.push_back(b);
  }
  s.last_hash = parent;
  if (bm->prefix && num_tokens > nfull * bs)
    s.tail.assign(token_ids + nfull * bs, token_ids + num_tokens);
  if (slot_mapping) {
    for (int64_t t = 0; t < num_tokens; ++t) {
      const int64_t i = t / bs;
      slot_mapping[t] = hitb[(size_t)i] >= 0 ? -1 : (int64_t)s.blocks[(size_t)i] * bs + t % bs;
    }
  }
  if (num_cached) *num_cached = cached;
  bm->seqs.emplace(seq_id, std::move(s));
  return PKV_OK;
}

int pkv_bm_can_append(const pkv_block_manager* bm, int64_t seq_id) {
  if (!bm) return 0;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end() || it->second.swapped) return 0;
  const Seq& s = it->second;
  if (s.len % bm->bs != 0 && bm->dev[s.blocks.back()].ref == 1) return 1;
  return bm->available() > 0 ? 1 : 0;
}

int pkv_bm_append_slot(pkv_block_manager* bm, int64_t seq_id, int32_t token_id, int64_t* slot,
                       int64_t* cow_src, int64_t* cow_dst) {
  if (!bm || !slot || !cow_src || !cow_dst) return PKV_ERR_NULL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end() || it->second.swapped) return PKV_ERR_SEQ;
  Seq& s = it->second;
  const int bs = bm->bs;
  const int64_t off = s.len % bs;
  int64_t src = -1, dst = -1;
  if (off == 0) {
    const int32_t b = bm->take_block();
    if (b < 0) return PKV_ERR_NO_BLOCKS;
    s.blocks.push_back(b);
  } else {
    const int32_t last = s.blocks.back();
    if (bm->dev[last].ref > 1) {  // shared partial block: copy on write
      const int32_t b = bm->take_block();
      if (b < 0) return PKV_ERR_NO_BLOCKS;
      bm->release(last);
      s.blocks.back() = b;
      src = last;
      dst = b;
    }
  }
  *slot = (int64_t)s.blocks.back() * bs + off;
  *cow_src = src;
  *cow_dst = dst;
  s.len += 1;
  if (bm->prefix) {
    s.tail.push_back(token_id);
    if ((int)s.tail.size() == bs) {  // the block is full: name it
      const uint64_t h = block_hash(s.last_hash, s.tail.data(), bs);
      bm->register_block(s.blocks.back(), h, s.last_hash, s.tail.data());
      s.last_hash = h;
      s.tail.clear();
    }
  }
  return PKV_OK;
}

int pkv_bm_append_slots(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* token_ids,
                        int n, int64_t* slot_mapping, int64_t* cow_pairs, int64_t* num_cow) {
  if (!bm || !num_cow) return PKV_ERR_NULL;
  if (n < 0) return PKV_ERR_SHAPE;
  if (n > 0 && (!seq_ids || !token_ids || !slot_mapping || !cow_pairs)) return PKV_ERR_NULL;
  // Check everything first: known, resident, distinct; count the blocks needed.
  std::vector<Seq*> seqs((size_t)n);
  std::unordered_set<int64_t> seen;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || it->second.swapped || !seen.insert(seq_ids[i]).second)
      return PKV_ERR_SEQ;
    Seq& sq = it->second;
    seqs[(size_t)i] = &sq;
    if (sq.len % bm->bs == 0 || bm->dev[sq.blocks.back()].ref > 1) ++need;
  }
  // A shared partial block copied by one sequence of the batch may leave the
  // last sharer writing in place, so `need` is an upper bound.
  if (need > bm->available()) return PKV_ERR_NO_BLOCKS;
  int64_t ncow = 0;
  for (int i = 0; i < n; ++i) {
    int64_t src, dst;
    const int st = pkv_bm_append_slot(bm, seq_ids[i], token_ids[i], slot_mapping + i, &src, &dst);
    if (st != PKV_OK) return st;  // unreachable: checked above
    if (src >= 0) {
      cow_pairs[2 * ncow] = src;
      cow_pairs[2 * ncow + 1] = dst;
      ++ncow;
    }
  }
  *num_cow = ncow;
  return PKV_OK;
}

int pkv_bm_fork(pkv_block_manager* bm, int64_t parent_id, int64_t child_id) {
  if (!bm) return PKV_ERR_NULL;
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end() || it->second.swapped || bm->seqs.count(child_id)) return PKV_ERR_SEQ;
  Seq c = it->second;
  for (int32_t b : c.blocks) bm->hold(b);
  bm->seqs.emplace(child_id, std::move(c));
  return PKV_OK;
}

int pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
  if (!bm) return PKV_ERR_NULL;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PKV_ERR_SEQ;
  Seq& s = it->second;
  if (s.swapped) {
    for (int32_t b : s.blocks)
      if (--bm->host_ref[b] == 0) bm->free_host.push_back(b);
  } else {
    bm->release_seq(s);
  }
  bm->seqs.erase(it);
  return PKV_OK;
}

// Checks a group for swapping: known, distinct, all resident (want_swapped 0)
// or all swapped out (1).
static int check_group(const pkv_block_manager* bm, const int64_t* ids, int n, bool want_swapped) {
  if (n < 0) return PKV_ERR_SHAPE;
  if (n > 0 && !ids) return PKV_ERR_NULL;
  std::unordered_set<int64_t> seen;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(ids[i]);
    if (it == bm->seqs.end() || it->second.swapped != want_swapped || !seen.insert(ids[i]).second)
      return PKV_ERR_SEQ;
  }
  return PKV_OK;
}

int pkv_bm_swap_out(pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int64_t* pairs,
                    int64_t max_pairs, int64_t* num_pairs) {
  if (!bm || !num_pairs) return PKV_ERR_NULL;
  int st = check_group(bm, seq_ids, num_seqs, false);
  if (st != PKV_OK) return st;
  // Distinct device blocks of the group, in first-seen order.
  std::unordered_map<int32_t, int32_t> map;
  std::vector<int32_t> order;
  for (int i = 0; i < num_seqs; ++i)
    for (int32_t b : bm->seqs.at(seq_ids[i]).blocks)
      if (map.emplace(b, -1).second) order.push_back(b);
  if ((int64_t)order.size() > (int64_t)bm->free_host.size()) return PKV_ERR_NO_BLOCKS;
  if ((int64_t)order.size() > max_pairs || (!order.empty() && !pairs)) return PKV_ERR_SHAPE;
  for (size_t k = 0; k < order.size(); ++k) {
    const int32_t h = bm->free_host.back();
    bm->free_host.pop_back();
    map[order[k]] = h;
    pairs[2 * k] = order[k];
    pairs[2 * k + 1] = h;
  }
  for (int i = 0; i < num_seqs; ++i) {
    Seq& s = bm->seqs.at(seq_ids[i]);
    std::vector<int32_t> hb;
    hb.reserve(s.blocks.size());
    for (int32_t b : s.blocks) {
      const int32_t h = map[b];
      ++bm->host_ref[h];
      hb.push_back(h);
    }
    bm->release_seq(s);
    s.blocks = std::move(hb);
    s.swapped = true;
  }
  *num_pairs = (int64_t)order.size();
  return PKV_OK;
}

int pkv_bm_swap_in(pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int64_t* pairs,
                   int64_t max_pairs, int64_t* num_pairs) {
  if (!bm || !num_pairs) return PKV_ERR_NULL;
  int st = check_group(bm, seq_ids, num_seqs, true);
  if (st != PKV_OK) return st;
  std::unordered_map<int32_t, int32_t> map;
  std::vector<int32_t> order;
  for (int i = 0; i < num_seqs; ++i)
    for (int32_t h : bm->seqs.at(seq_ids[i]).blocks)
      if (map.emplace(h, -1).second) order.push_back(h);
  if ((int64_t)order.size() > bm->available()) return PKV_ERR_NO_BLOCKS;
  if ((int64_t)order.size() > max_pairs || (!order.empty() && !pairs)) return PKV_ERR_SHAPE;
  for (size_t k = 0; k < order.size(); ++k) {
    const int32_t b = bm->take_block();  // cannot fail: counted above
    bm->dev[b].ref = 0;                  // references are added per sequence below
    map[order[k]] = b;
    pairs[2 * k] = order[k];
    pairs[2 * k + 1] = b;
  }
  for (int i = 0; i < num_seqs; ++i) {
    Seq& s = bm->seqs.at(seq_ids[i]);
    for (int32_t& h : s.blocks) {
      const int32_t b = map[h];
      ++bm->dev[b].ref;
      if (--bm->host_ref[h] == 0) bm->free_host.push_back(h);
      h = b;
    }
    s.swapped = false;
    // Blocks come back private and unnamed; later full blocks are named again
    // from the sequence's hash chain.
  }
  *num_pairs = (int64_t)order.size();
  return PKV_OK;
}

int pkv_bm_block_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs,
                        int max_blocks_per_seq, int32_t* table, int32_t* seq_lens) {
  if (!bm) return PKV_ERR_NULL;
  if (num_seqs < 0 || max_blocks_per_seq < 0) return PKV_ERR_SHAPE;
  if (num_seqs > 0 && (!seq_ids || !table || !seq_lens)) return PKV_ERR_NULL;
  for (int i = 0; i < num_seqs; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || it->second.swapped) return PKV_ERR_SEQ;
    if ((int64_t)it->second.blocks.size() > max_blocks_per_seq || it->second.len > INT32_MAX)
      return PKV_ERR_SHAPE;
  }
  for (int i = 0; i < num_seqs; ++i) {
    const Seq& s = bm->seqs.at(seq_ids[i]);
    int32_t* row = table + (int64_t)i * max_blocks_per_seq;
    for (int j = 0; j < max_blocks_per_seq; ++j)
      row[j] = j < (int)s.blocks.size() ? s.blocks[(size_t)j] : -1;
    seq_lens[i] = (int32_t)s.len;
  }
  return PKV_OK;
}

int64_t pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id) {
  if (!bm) return PKV_ERR_NULL;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? (int64_t)PKV_ERR_SEQ : it->second.len;
}

int pkv_bm_refcount(const pkv_block_manager* bm, int32_t block) {
  if (!bm) return PKV_ERR_NULL;
  if (block < 0 || (size_t)block >= bm->dev.size()) return PKV_ERR_SHAPE;
  return bm->dev[block].ref;
}

int pkv_bm_usage(const pkv_block_manager* bm, int64_t* out) {
  if (!bm || !out) return PKV_ERR_NULL;
  std::unordered_map<int32_t, int64_t> fill;  // held block -> fullest use
  int64_t tokens = 0;
  for (const auto& kv : bm->seqs) {
    const Seq& s = kv.second;
    if (s.swapped) continue;
    tokens += s.len;
    for (size_t j = 0; j < s.blocks.size(); ++j) {
      const int64_t f = std::min<int64_t>(bm->bs, s.len - (int64_t)j * bm->bs);
      int64_t& cur = fill[s.blocks[j]];
      cur = std::max(cur, f);
    }
  }
  int64_t used = 0;
  for (const auto& kv : fill) used += kv.second;
  out[0] = (int64_t)bm->dev.size();
  out[1] = (int64_t)fill.size();
  out[2] = (int64_t)bm->lru.size();
  out[3] = (int64_t)bm->free_dev.size();
  out[4] = tokens;
  out[5] = used;
  return PKV_OK;
}

int pkv_bm_check(const pkv_block_manager* bm) {
  if (!bm) return PKV_ERR_NULL;
  const size_t nb = bm->dev.size(), nh = bm->host_ref.size();
  std::vector<int64_t> dref(nb, 0), href(nh, 0);
  for (const auto& kv : bm->seqs) {
    const Seq& s = kv.second;
    if ((int64_t)s.blocks.size() != (s.len + bm->bs - 1) / bm->bs) return PKV_ERR_SHAPE;
    for (int32_t b : s.blocks) {
      if (s.swapped) {
        if (b < 0 || (size_t)b >= nh) return PKV_ERR_SHAPE;
        ++href[b];
      } else {
        if (b < 0 || (size_t)b >= nb) return PKV_ERR_SHAPE;
        ++dref[b];
      }
    }
  }
  std::vector<char> state(nb, 0);  // 1 held, 2 free, 3 cached-unheld
  for (size_t b = 0; b < nb; ++b) {
    if (bm->dev[b].ref != dref[b]) return PKV_ERR_SHAPE;
    if (dref[b] > 0) state[b] = 1;
  }
  for (int32_t b : bm->free_dev) {
    if (b < 0 || (size_t)b >= nb || state[b] != 0 || bm->dev[b].hashed) return PKV_ERR_SHAPE;
    state[b] = 2;
  }
  for (int32_t b : bm->lru) {
    if (b < 0 || (size_t)b >= nb || state[b] != 0 || !bm->dev[b].hashed || !bm->dev[b].in_lru)
      return PKV_ERR_SHAPE;
    state[b] = 3;
  }
  for (size_t b = 0; b < nb; ++b)
    if (state[b] == 0) return PKV_ERR_SHAPE;
  for (const auto& kv : bm->cache) {
    const int32_t b = kv.second;
    if (b < 0 || (size_t)b >= nb || !bm->dev[b].hashed || bm->dev[b].hash != kv.first)
      return PKV_ERR_SHAPE;
  }
  for (size_t b = 0; b < nb; ++b) {
    if (!bm->dev[b].hashed) continue;
    auto it = bm->cache.find(bm->dev[b].hash);
    if (it == bm->cache.end() || it->second != (int32_t)b) return PKV_ERR_SHAPE;
  }
  std::vector<char> hfree(nh, 0);
  for (int32_t h : bm->free_host) {
    if (h < 0 || (size_t)h >= nh || hfree[h] || href[h] != 0) return PKV_ERR_SHAPE;
    hfree[h] = 1;
  }
  for (size_t h = 0; h < nh; ++h) {
    if (bm->host_ref[h] != href[h]) return PKV_ERR_SHAPE;
    if ((href[h] > 0) == (hfree[h] != 0)) return PKV_ERR_SHAPE;
  }
  return PKV_OK;
}

}  // extern "C"
