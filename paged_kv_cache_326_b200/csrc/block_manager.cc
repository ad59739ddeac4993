// Host block manager: free list, per-block reference counts, copy-on-write.
//
// "The KV Cache and PagedAttention": a text's logical blocks map to physical
// blocks anywhere in the pool (section "Like Pages of Memory"); a text gets
// its next block once its current ones are full, and returns them all when it
// finishes (section "The Block Table"); samples of one prompt share its
// blocks, each block counting its users, and a text that needs to change a
// shared block copies it first (section "Shared, Copied on Write"); a text
// either has every block it needs or none of them (section "When Memory Runs
// Out"), so every operation here either succeeds completely or changes
// nothing.
//
// Prefix reuse ("The KV Cache and PagedAttention", section "What Came After":
// every full block is identified by a hash of its own tokens chained with
// the hash of everything before it, and a new text that begins like an
// earlier one takes over the earlier text's blocks).  pa_bm_add_seq_tokens
// walks the prompt's full blocks in order and reuses cached blocks up to
// the first miss.  A cached block whose count falls to zero stays cached
// while it waits in the free list; a hit takes it back out; the allocator
// evicts it (drops its hash) when it hands the block out again.  Only
// prompt blocks registered by pa_bm_add_seq_tokens are cached.  A hash match
// alone never shares a block: a hit also needs the block's own token ids to
// be equal, and a second, independent 64-bit hash of the whole prefix (FNV-1a)
// to be equal, so a collision of the chained hash is caught.
#include <cstdint>
#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"

namespace pa {
int64_t option_prefix_key_bits();
}

struct pa_bm {
  int64_t num_blocks;
  int block_size;
  // Free list: take from the front, return to the back.  A cached block can
  // leave it from the middle (a prefix hit), so entries carry the stamp the
  // block got when it was returned; an entry whose block has since left, or
  // was returned again later, is stale and skipped.
  std::deque<std::pair<int32_t, uint32_t>> free_list;
  std::vector<uint8_t> in_free;
  std::vector<uint32_t> free_stamp;
  int64_t free_count = 0;
  std::vector<int32_t> ref;                      // texts using each block
  // prefix cache: key (the chained hash, masked by key_mask) -> block; each
  // cached block's key, its token ids and the second hash of its prefix
  std::unordered_map<uint64_t, int32_t> cache;
  std::vector<uint8_t> cached;
  std::vector<uint64_t> cached_hash;
  std::vector<uint64_t> cached_check;  // FNV-1a of every token up to the block's end
  std::vector<int32_t> cached_tokens;  // block_size ids per block, sized on first use
  uint64_t key_mask = ~0ull;
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t tokens;
  };
  std::unordered_map<int64_t, Seq> seqs;
};

namespace {

// SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): drives the Fisher-Yates shuffle of the initial
// free list when a seed is given.
uint64_t splitmix64(uint64_t& x) {
  uint64_t z = (x += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void drop_stale(pa_bm* bm) {
  while (!bm->free_list.empty()) {
    const auto& f = bm->free_list.front();
    if (bm->in_free[f.first] && bm->free_stamp[f.first] == f.second) return;
    bm->free_list.pop_front();
  }
}

// Drop every stale entry, keeping the order of the live ones, once they
// outnumber the live ones (prefix hits leave one behind each).
void compact(pa_bm* bm) {
  if (static_cast<int64_t>(bm->free_list.size()) <= 2 * bm->free_count + 64) return;
  std::deque<std::pair<int32_t, uint32_t>> live;
  for (const auto& f : bm->free_list)
    if (bm->in_free[f.first] && bm->free_stamp[f.first] == f.second) live.push_back(f);
  bm->free_list.swap(live);
}

void give_back(pa_bm* bm, int32_t b) {
  bm->in_free[b] = 1;
  bm->free_stamp[b] += 1;
  bm->free_list.emplace_back(b, bm->free_stamp[b]);
  bm->free_count += 1;
}

void uncache(pa_bm* bm, int32_t b) {
  if (!bm->cached[b]) return;
  auto it = bm->cache.find(bm->cached_hash[b]);
  if (it != bm->cache.end() && it->second == b) bm->cache.erase(it);
  bm->cached[b] = 0;
}

// The front of the free list; a block handed out again leaves the cache.
int32_t take(pa_bm* bm) {
  drop_stale(bm);
  const int32_t b = bm->free_list.front().first;
  bm->free_list.pop_front();
  bm->in_free[b] = 0;
  bm->free_count -= 1;
  uncache(bm, b);
  bm->ref[b] = 1;
  return b;
}

// SplitMix64's output mix (the same paper) as the step of the chained hash.
uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Hash of one full block: the hash of everything before it, then its tokens.
uint64_t block_hash(uint64_t prev, const int32_t* tokens, int n) {
  uint64_t h = prev;
  for (int i = 0; i < n; ++i)
    h = mix64(h ^ (static_cast<uint64_t>(static_cast<uint32_t>(tokens[i])) +
                   0x9E3779B97F4A7C15ull));
  return h;
}

// The check hash: 64-bit FNV-1a (Fowler, Noll, Vo) over the four
// little-endian bytes of every token id, continued from `prev` (the FNV
// offset basis before the first block).  Independent of the chained hash, so
// two different prefixes pass as equal only if both 64-bit hashes collide.
constexpr uint64_t kFnvBasis = 0xcbf29ce484222325ull;
uint64_t check_hash(uint64_t prev, const int32_t* tokens, int n) {
  uint64_t h = prev;
  for (int i = 0; i < n; ++i) {
    const uint32_t t = static_cast<uint32_t>(tokens[i]);
    for (int b = 0; b < 4; ++b) {
      h ^= (t >> (8 * b)) & 0xffu;
      h *= 0x100000001b3ull;
    }
  }
  return h;
}

}  // namespace

extern "C" {

pa_bm* pa_bm_create(int64_t num_blocks, int block_size, uint64_t shuffle_seed) {
  if (num_blocks <= 0 || num_blocks > INT32_MAX || block_size <= 0) return nullptr;
  pa_bm* bm = new (std::nothrow) pa_bm();
  if (!bm) return nullptr;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  std::vector<int32_t> order(static_cast<size_t>(num_blocks));
  for (int64_t i = 0; i < num_blocks; ++i) order[i] = static_cast<int32_t>(i);
  if (shuffle_seed != 0) {
    uint64_t st = shuffle_seed;
    for (int64_t i = num_blocks - 1; i > 0; --i) {
      int64_t j = static_cast<int64_t>(splitmix64(st) % static_cast<uint64_t>(i + 1));
      std::swap(order[i], order[j]);
    }
  }
  bm->in_free.assign(static_cast<size_t>(num_blocks), 0);
  bm->free_stamp.assign(static_cast<size_t>(num_blocks), 0);
  for (int32_t b : order) give_back(bm, b);
  bm->ref.assign(static_cast<size_t>(num_blocks), 0);
  bm->cached.assign(static_cast<size_t>(num_blocks), 0);
  bm->cached_hash.assign(static_cast<size_t>(num_blocks), 0);
  bm->cached_check.assign(static_cast<size_t>(num_blocks), 0);
  const int64_t bits = pa::option_prefix_key_bits();
  bm->key_mask = bits >= 64 ? ~0ull : ((1ull << bits) - 1);
  return bm;
}

void pa_bm_destroy(pa_bm* bm) { delete bm; }

int pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int num_tokens) {
  if (!bm || num_tokens < 0) return PA_ERR_INVALID;
  if (bm->seqs.count(seq_id)) return PA_ERR_EXISTS;
  int64_t need = (static_cast<int64_t>(num_tokens) + bm->block_size - 1) / bm->block_size;
  if (bm->free_count < need) return PA_ERR_OUT_OF_BLOCKS;
  pa_bm::Seq s;
  s.tokens = num_tokens;
  s.blocks.reserve(static_cast<size_t>(need));
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(take(bm));
  bm->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

int pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child) {
  if (!bm) return PA_ERR_INVALID;
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end()) return PA_ERR_NO_SEQ;
  if (bm->seqs.count(child)) return PA_ERR_EXISTS;
  pa_bm::Seq copy = it->second;
  for (int32_t b : copy.blocks) bm->ref[b] += 1;
  bm->seqs.emplace(child, std::move(copy));
  return PA_OK;
}

int pa_bm_append_slot(pa_bm* bm, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                      int32_t* cow_dst) {
  if (!bm || !slot || !cow_src || !cow_dst) return PA_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_NO_SEQ;
  pa_bm::Seq& s = it->second;
  const int64_t place = s.tokens % bm->block_size;
  int32_t src = -1, dst = -1;
  if (place == 0) {
    if (bm->free_count == 0) return PA_ERR_OUT_OF_BLOCKS;
    s.blocks.push_back(take(bm));
  } else {
    int32_t last = s.blocks.back();
    if (bm->ref[last] > 1) {
      if (bm->free_count == 0) return PA_ERR_OUT_OF_BLOCKS;
      dst = take(bm);
      bm->ref[last] -= 1;
      s.blocks.back() = dst;
      src = last;
    }
  }
  s.tokens += 1;
  *slot = static_cast<int64_t>(s.blocks.back()) * bm->block_size + place;
  *cow_src = src;
  *cow_dst = dst;
  return PA_OK;
}

int pa_bm_free_seq(pa_bm* bm, int64_t seq_id) {
  if (!bm) return PA_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_NO_SEQ;
  for (int32_t b : it->second.blocks)
    if (bm->ref[b] <= 0) return PA_ERR_CORRUPT;
  for (int32_t b : it->second.blocks) {
    if (--bm->ref[b] == 0) give_back(bm, b);
  }
  bm->seqs.erase(it);
  return PA_OK;
}

int64_t pa_bm_num_free(const pa_bm* bm) { return bm ? bm->free_count : PA_ERR_INVALID; }

int64_t pa_bm_num_cached_blocks(const pa_bm* bm) {
  return bm ? static_cast<int64_t>(bm->cache.size()) : PA_ERR_INVALID;
}

int pa_bm_add_seq_tokens(pa_bm* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                         int* num_cached_tokens) {
  if (!bm || num_tokens < 0 || (num_tokens > 0 && !tokens)) return PA_ERR_INVALID;
  if (bm->seqs.count(seq_id)) return PA_ERR_EXISTS;
  const int B = bm->block_size;
  const int64_t full = num_tokens / B;
  const int64_t need = (static_cast<int64_t>(num_tokens) + B - 1) / B;
  if (full > 0 && bm->cached_tokens.empty())
    bm->cached_tokens.assign(static_cast<size_t>(bm->num_blocks) * B, 0);
  // the keys of the full blocks, and the cached run at the front: a cached
  // block is a hit only if its token ids and its prefix's check hash agree
  std::vector<uint64_t> h(static_cast<size_t>(full)), chk(static_cast<size_t>(full));
  std::vector<int32_t> hit;
  bool run = true;
  uint64_t prev = 0, prev_chk = kFnvBasis;
  for (int64_t j = 0; j < full; ++j) {
    const int32_t* tj = tokens + j * B;
    prev = block_hash(prev, tj, B);
    prev_chk = check_hash(prev_chk, tj, B);
    h[j] = prev & bm->key_mask;
    chk[j] = prev_chk;
    if (run) {
      auto it = bm->cache.find(h[j]);
      const bool same =
          it != bm->cache.end() && bm->cached_check[it->second] == prev_chk &&
          std::memcmp(bm->cached_tokens.data() + static_cast<size_t>(it->second) * B, tj,
                      sizeof(int32_t) * B) == 0;
      if (same) {
        hit.push_back(it->second);
      } else {
        run = false;
      }
    }
  }
  int64_t hits_free = 0;
  for (int32_t b : hit) hits_free += bm->in_free[b] ? 1 : 0;
  const int64_t fresh = need - static_cast<int64_t>(hit.size());
  if (bm->free_count - hits_free < fresh) return PA_ERR_OUT_OF_BLOCKS;
  pa_bm::Seq s;
  s.tokens = num_tokens;
  s.blocks.reserve(static_cast<size_t>(need));
  for (int32_t b : hit) {  // reuse: a waiting block leaves the free list
    if (bm->in_free[b]) {
      bm->in_free[b] = 0;
      bm->free_count -= 1;
    }
    bm->ref[b] += 1;
    s.blocks.push_back(b);
  }
  compact(bm);
  for (int64_t j = static_cast<int64_t>(hit.size()); j < need; ++j) {
    const int32_t b = take(bm);
    s.blocks.push_back(b);
    if (j < full && !bm->cache.count(h[j])) {  // register a new full block
      bm->cache.emplace(h[j], b);
      bm->cached[b] = 1;
      bm->cached_hash[b] = h[j];
      bm->cached_check[b] = chk[j];
      std::memcpy(bm->cached_tokens.data() + static_cast<size_t>(b) * B, tokens + j * B,
                  sizeof(int32_t) * B);
    }
  }
  bm->seqs.emplace(seq_id, std::move(s));
  if (num_cached_tokens) *num_cached_tokens = static_cast<int>(hit.size()) * B;
  return PA_OK;
}

int pa_bm_refcount(const pa_bm* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return PA_ERR_INVALID;
  return bm->ref[block];
}

int64_t pa_bm_num_tokens(const pa_bm* bm, int64_t seq_id) {
  if (!bm) return PA_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? PA_ERR_NO_SEQ : it->second.tokens;
}

int pa_bm_export(const pa_bm* bm, const int64_t* seq_ids, int n, int32_t* block_tables,
                 int max_blocks_per_seq, int32_t* context_lens) {
  if (!bm || n < 0 || max_blocks_per_seq <= 0 || (n > 0 && (!seq_ids || !block_tables ||
                                                             !context_lens)))
    return PA_ERR_INVALID;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PA_ERR_NO_SEQ;
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks_per_seq)
      return PA_ERR_TABLE_FULL;
    if (it->second.tokens > INT32_MAX) return PA_ERR_INVALID;
  }
  for (int i = 0; i < n; ++i) {
    const pa_bm::Seq& s = bm->seqs.find(seq_ids[i])->second;
    int32_t* row = block_tables + static_cast<int64_t>(i) * max_blocks_per_seq;
    size_t k = 0;
    for (; k < s.blocks.size(); ++k) row[k] = s.blocks[k];
    for (; k < static_cast<size_t>(max_blocks_per_seq); ++k) row[k] = -1;
    context_lens[i] = static_cast<int32_t>(s.tokens);
  }
  return PA_OK;
}

int pa_split_shared_prefix(const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                           int max_blocks_per_seq, int block_size, int group_size,
                           int32_t* prefix_tables, int max_prefix_blocks, int32_t* prefix_lens,
                           int32_t* tail_tables, int max_tail_blocks, int32_t* tail_lens) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || group_size <= 0 ||
      num_seqs % group_size != 0 || max_prefix_blocks <= 0 || max_tail_blocks <= 0)
    return PA_ERR_INVALID;
  if (num_seqs == 0) return PA_OK;
  if (!block_tables || !context_lens || !prefix_tables || !prefix_lens || !tail_tables ||
      !tail_lens)
    return PA_ERR_INVALID;
  const int64_t cap = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  for (int s = 0; s < num_seqs; ++s)
    if (context_lens[s] < 0 || context_lens[s] > cap) return PA_ERR_INVALID;
  const int groups = num_seqs / group_size;
  std::vector<int> shared(groups);
  // Shared blocks of a group: the leading table entries that every text of
  // the group holds at the same index and has filled completely.
  for (int g = 0; g < groups; ++g) {
    const int s0 = g * group_size;
    const int32_t* row0 = block_tables + static_cast<int64_t>(s0) * max_blocks_per_seq;
    int p = 0;
    while (p < max_prefix_blocks && p < max_blocks_per_seq) {
      bool same = true;
      for (int s = s0; s < s0 + group_size && same; ++s) {
        const int32_t* row = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq;
        same = row[p] == row0[p] && static_cast<int64_t>(p + 1) * block_size <= context_lens[s];
      }
      if (!same) break;
      ++p;
    }
    shared[g] = p;
    for (int s = s0; s < s0 + group_size; ++s) {
      const int64_t tail = context_lens[s] - static_cast<int64_t>(p) * block_size;
      if ((tail + block_size - 1) / block_size > max_tail_blocks) return PA_ERR_TABLE_FULL;
    }
  }
  for (int g = 0; g < groups; ++g) {
    const int p = shared[g];
    const int32_t* row0 = block_tables + static_cast<int64_t>(g) * group_size * max_blocks_per_seq;
    int32_t* prow = prefix_tables + static_cast<int64_t>(g) * max_prefix_blocks;
    for (int k = 0; k < max_prefix_blocks; ++k) prow[k] = k < p ? row0[k] : -1;
    prefix_lens[g] = p * block_size;
    for (int s = g * group_size; s < (g + 1) * group_size; ++s) {
      const int32_t* row = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq;
      int32_t* trow = tail_tables + static_cast<int64_t>(s) * max_tail_blocks;
      const int tail = context_lens[s] - p * block_size;
      const int nb = (tail + block_size - 1) / block_size;
      for (int k = 0; k < max_tail_blocks; ++k) trow[k] = k < nb ? row[p + k] : -1;
      tail_lens[s] = tail;
    }
  }
  return PA_OK;
}

}  // extern "C"
